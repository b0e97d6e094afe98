"""Context-parallel CSA prefill of one long sequence over the ranks of a
process group.

"DeepSeek V4 CSA + CP 迁移到 HP：困难点深度分析" describes this layout in the
pipeline that opens the page (and §3.2 names its risk).
- Each rank holds one contiguous shard of the tokens.
- Stage-1 compression runs locally. It needs a left halo, because an
  overlapping entry reads the block before it.
- The compressed entries are all-gathered, since any query may select any
  earlier entry.
- The indexer, top-k and attention then run locally for the rank's own
  queries, with the sliding window reading the halo too.

The page names the risk of this layout: CP > 1 disagreeing with CP = 1 at the
shard edges.  A CP run must reproduce the single-rank result.  The page
gathers the halo with an all-gather; here the left neighbour sends it point
to point, since one neighbour's rows are all a rank needs.

This module moves data and does the bookkeeping (which rows, which positions).
The arithmetic is done by a backend object with three calls:

    compress(x [L, d_in], W, m, overlap, fp8) -> entries [L//m, d_out]
                                                   (fp8: (codes, scales))
    indexer_topk(qI [L, H_I, d_I], kI, kI_scale, m, topk, q_pos [L], n_entries)
        -> idx [L, topk]
    sparse_attn(q [L, H, D], kv_c, idx, kv_raw [R, D], window, q_pos, raw_pos0)
        -> out [L, H, D]

`CudaBackend` runs them through this library's entry points (the
positioned, decode-shaped kernels, since a shard's queries start at p0 > 0).
Exchanges go through torch.distributed: NCCL for CUDA tensors, gloo for host
tensors.  Nothing here computes the method itself.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass
class Shard:
    rank: int
    world: int
    p0: int        # first position of the rank's tokens
    p1: int        # one past the last


def shard_of(n: int, world: int, rank: int, m: int) -> Shard:
    """Equal contiguous shards whose edges fall on block boundaries."""
    if n % (world * m):
        raise ValueError("n must be a multiple of world * m for equal, block-aligned shards")
    per = n // world
    return Shard(rank, world, rank * per, (rank + 1) * per)


def _exchange_left_halo(local: torch.Tensor, rows: int, shard: Shard, group=None) -> torch.Tensor:
    """The last `rows` rows of the left neighbour's shard (empty on rank 0)."""
    if rows == 0 or shard.world == 1:
        return local[:0]
    if local.shape[0] < rows:
        raise ValueError("a shard must hold at least the halo's rows")
    ops = []
    recv = torch.empty((rows,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    if shard.rank + 1 < shard.world:
        ops.append(dist.P2POp(dist.isend, local[-rows:].contiguous(), shard.rank + 1, group))
    if shard.rank > 0:
        ops.append(dist.P2POp(dist.irecv, recv, shard.rank - 1, group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    return recv if shard.rank > 0 else local[:0]


def _all_gather_rows(local: torch.Tensor, shard: Shard, group=None) -> torch.Tensor:
    if shard.world == 1:
        return local
    parts = [torch.empty_like(local) for _ in range(shard.world)]
    dist.all_gather(parts, local.contiguous(), group=group)
    return torch.cat(parts, dim=0)


def cp_prefill(shard: Shard, q, kv, qI, kI_raw, W_c, W_Ic, m: int, topk: int, window: int,
               backend, indexer_fp8: bool = True, group=None) -> dict:
    """The CSA prefill of the rank's queries [p0, p1) of one sequence.

    q [L, H, D], kv [L, D], qI [L, H_I, d_I], kI_raw [L, d_I] are the rank's
    shard (L = p1 - p0); W_c, W_Ic are replicated.  Returns the rank's out
    [L, H, D] and idx [L, topk] plus the gathered compressed caches.
    """
    L = shard.p1 - shard.p0
    if kv.shape[0] != L:
        raise ValueError("the shard tensors must hold p1 - p0 rows")
    # 1. left halo: one block for the overlapping compressor, W-1 rows for the
    #    window (every rank takes part in the exchange, rank 0 only sends)
    h_kv = max(m, window - 1) if shard.world > 1 else 0
    if L < h_kv:
        raise ValueError("each shard must hold at least max(m, window - 1) tokens")
    halo_kv = _exchange_left_halo(kv, h_kv, shard, group)
    halo_kI = _exchange_left_halo(kI_raw, m if shard.world > 1 else 0, shard, group)
    # 2. compression over [p0 - m, p1): the first entry of that call belongs to
    #    the left neighbour (and saw a clipped window), so it is dropped
    def local_entries(x, halo, W, fp8):
        if shard.p0 == 0:
            return backend.compress(x, W, m, True, fp8)
        ext = torch.cat([halo[-m:], x], dim=0)
        res = backend.compress(ext, W, m, True, fp8)
        return (res[0][1:], res[1][1:]) if fp8 else res[1:]
    kv_c_loc = local_entries(kv, halo_kv, W_c, False)
    kI = local_entries(kI_raw, halo_kI, W_Ic, indexer_fp8)
    # 3. every rank needs every entry
    kv_c = _all_gather_rows(kv_c_loc, shard, group)
    if indexer_fp8:
        kI_c = _all_gather_rows(kI[0], shard, group)
        kI_s = _all_gather_rows(kI[1], shard, group)
    else:
        kI_c, kI_s = _all_gather_rows(kI, shard, group), None
    N_c = kv_c.shape[0]
    # 4. the rank's queries at their absolute positions
    q_pos = torch.arange(shard.p0, shard.p1, dtype=torch.int32, device=q.device)
    idx = backend.indexer_topk(qI, kI_c, kI_s, m, topk, q_pos, N_c)
    # 5. attention: the window reads the halo rows before p0 and the shard
    kv_raw = torch.cat([halo_kv, kv], dim=0) if halo_kv.shape[0] else kv
    raw_pos0 = shard.p0 - halo_kv.shape[0]
    out = backend.sparse_attn(q, kv_c, idx, kv_raw, window, q_pos, raw_pos0)
    return dict(out=out, idx=idx, kv_c=kv_c, kI_c=kI_c, kI_scale=kI_s)


class CudaBackend:
    """The context-parallel arithmetic through this library's entry points."""

    def __init__(self, stream=None):
        from . import api
        self.api = api
        self.stream = stream

    def compress(self, x, W, m, overlap, fp8):
        x = x[None].contiguous()
        if fp8:
            codes, scales = self.api.compress(x, W, m, overlap, out_dtype=torch.uint8,
                                              stream=self.stream)
            return codes[0], scales[0]
        return self.api.compress(x, W, m, overlap, stream=self.stream)[0]

    def indexer_topk(self, qI, kI, kI_scale, m, topk, q_pos, n_entries):
        ne = torch.tensor([n_entries], dtype=torch.int32, device=qI.device)
        idx = self.api.indexer_topk(qI[None].contiguous(), kI[None].contiguous(), m, topk,
                                    kI_scale=None if kI_scale is None else kI_scale[None].contiguous(),
                                    n_entries=ne, q_pos=q_pos[None].contiguous(),
                                    stream=self.stream)
        return idx[0]

    def sparse_attn(self, q, kv_c, idx, kv_raw, window, q_pos, raw_pos0):
        dev = q.device
        p0 = torch.tensor([raw_pos0], dtype=torch.int32, device=dev)
        ln = torch.tensor([kv_raw.shape[0]], dtype=torch.int32, device=dev)
        out = self.api.sparse_attn(q[None].contiguous(), kv_c[None].contiguous(),
                                   idx[None].contiguous(), kv_raw[None].contiguous(), window,
                                   raw_pos0=p0, raw_len=ln, q_pos=q_pos[None].contiguous(),
                                   stream=self.stream)
        return out[0]
