"""Context-parallel CSA prefill of one long sequence over the ranks of a
process group.

"DeepSeek V4 CSA + CP 迁移到 HP：困难点深度分析" describes this layout in the
pipeline that opens the page (and §3.2 names its risk).
- The sequence is cut into chunks of consecutive tokens, block aligned, and
  each rank holds some of them (its spans).
- Stage-1 compression runs locally, per span.  It needs a left halo, because
  an overlapping entry reads the block before it.
- The compressed entries are all-gathered, since any query may select any
  earlier entry.
- The indexer, top-k and attention then run locally for the rank's own
  queries, with the sliding window reading the halo too.

Causal work grows with the position (a query at t scores about t/m
entries), so equal contiguous shards leave the last rank with the most
indexer work.  The zigzag layout cuts the sequence into 2W chunks and gives
rank r chunks r and 2W-1-r: every rank then holds one early and one late
chunk and the same total work.  The contiguous layout (one chunk per rank)
is kept as an option.

The page names the risk of this layout: CP > 1 disagreeing with CP = 1 at the
shard edges.  A CP run must reproduce the single-rank result.  The page
gathers the halo with an all-gather; here the owner of the chunk before a
span sends it point to point, since one chunk's tail is all a span needs.

This module moves data and does the bookkeeping (which rows, which positions).
The arithmetic is done by a backend object with three calls:

    compress(x [L, d_in], W, m, overlap, fp8) -> entries [L//m, d_out]
                                                   (fp8: (codes, scales))
    indexer_topk(qI [L, H_I, d_I], kI, kI_scale, m, topk, q_pos0, n_entries)
        -> idx [L, topk]                    (query i at position q_pos0 + i)
    sparse_attn(q [L, H, D], kv_c, idx, kv_raw [R, D], window, q_pos0, raw_pos0)
        -> out [L, H, D]                    (raw row j at position raw_pos0 + j)

`CudaBackend` runs them through this library's entry points at an offset
(csa_*_at), which take the tensor-core prefill kernels.  Exchanges go through
torch.distributed: NCCL for CUDA tensors, gloo for host tensors.  Nothing
here computes the method itself.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class Shard:
    rank: int
    world: int
    n: int                                  # sequence length
    chunk: int                              # tokens per chunk
    owners: tuple                           # owners[c]: the rank holding chunk c
    spans: tuple                            # this rank's chunks as [a, b), ascending

    @property
    def length(self) -> int:
        return sum(b - a for a, b in self.spans)


def chunk_owners(world: int, layout: str) -> tuple:
    """The rank that holds each chunk, in sequence order."""
    if layout == "zigzag":
        return tuple(c if c < world else 2 * world - 1 - c for c in range(2 * world))
    if layout == "contiguous":
        return tuple(range(world))
    raise ValueError(f"unknown layout {layout!r}")


def shard_of(n: int, world: int, rank: int, m: int, layout: str = "zigzag") -> Shard:
    """Rank `rank`'s spans: equal chunks whose edges fall on block boundaries."""
    owners = chunk_owners(world, layout)
    C = len(owners)
    if n % (C * m):
        raise ValueError(f"n must be a multiple of {C} * m for equal, block-aligned chunks")
    ch = n // C
    spans = tuple((c * ch, (c + 1) * ch) for c in range(C) if owners[c] == rank)
    return Shard(rank, world, n, ch, owners, spans)


def take_rows(x: torch.Tensor, shard: Shard) -> torch.Tensor:
    """The rank's rows of a full-sequence tensor, spans concatenated."""
    return torch.cat([x[a:b] for a, b in shard.spans], dim=0)


def place_rows(parts: list, shards: list, n: int) -> torch.Tensor:
    """Inverse of take_rows over all ranks: the per-rank results (span order)
    put back in sequence order."""
    out = torch.empty((n,) + tuple(parts[0].shape[1:]), dtype=parts[0].dtype,
                      device=parts[0].device)
    for part, sh in zip(parts, shards):
        o = 0
        for a, b in sh.spans:
            out[a:b] = part[o:o + (b - a)]
            o += b - a
    return out


def _span_rows(local: torch.Tensor, shard: Shard) -> list:
    """The rank's rows split per span."""
    res, o = [], 0
    for a, b in shard.spans:
        res.append(local[o:o + (b - a)])
        o += b - a
    return res


def exchange_halos(local: torch.Tensor, rows: int, shard: Shard, group=None) -> list:
    """Per span, the `rows` rows just before it (empty for the span at 0):
    the tail of chunk c-1, sent by its owner to the owner of chunk c.
    Every rank walks the chunks in the same order; a rank that holds both
    chunks copies locally."""
    per = _span_rows(local, shard)
    mine = {a // shard.chunk: i for i, (a, _) in enumerate(shard.spans)}
    halos = [local[:0] for _ in shard.spans]
    if rows == 0:
        return halos
    if shard.chunk < rows:
        raise ValueError("a chunk must hold at least the halo's rows")
    ops, recvs = [], []
    for c in range(1, len(shard.owners)):
        src, dst = shard.owners[c - 1], shard.owners[c]
        if src == shard.rank and dst == shard.rank:
            halos[mine[c]] = per[mine[c - 1]][-rows:]
        elif src == shard.rank:
            ops.append(dist.P2POp(dist.isend, per[mine[c - 1]][-rows:].contiguous(), dst, group,
                                  tag=c))
        elif dst == shard.rank:
            buf = torch.empty((rows,) + tuple(local.shape[1:]), dtype=local.dtype,
                              device=local.device)
            ops.append(dist.P2POp(dist.irecv, buf, src, group, tag=c))
            recvs.append((mine[c], buf))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    for i, buf in recvs:
        halos[i] = buf
    return halos


def order_spans(parts: list, shard: Shard) -> torch.Tensor:
    """Per-rank rows (each rank's chunks in its span order, equal counts per
    chunk) put in sequence order."""
    per_chunk = parts[0].shape[0] // len(shard.spans)
    order = []
    for c, r in enumerate(shard.owners):
        k = sum(1 for cc in range(c) if shard.owners[cc] == r)   # c is rank r's k-th chunk
        order.append(parts[r][k * per_chunk:(k + 1) * per_chunk])
    return torch.cat(order, dim=0)


def all_gather_spans(local: torch.Tensor, shard: Shard, group=None) -> torch.Tensor:
    """Every rank's per-span rows, in sequence order."""
    if shard.world == 1:
        parts = [local]
    else:
        parts = [torch.empty_like(local) for _ in range(shard.world)]
        dist.all_gather(parts, local.contiguous(), group=group)
    return order_spans(parts, shard)


def compress_spans(shard: Shard, x: torch.Tensor, halos: list, W, m: int, fp8: bool, backend):
    """Stage 1 per span over [a - m, b): the first entry of that call belongs
    to the chunk before (and saw a clipped window), so it is dropped."""
    codes, scales = [], []
    for (a, _), xs, h in zip(shard.spans, _span_rows(x, shard), halos):
        if a == 0:
            res = backend.compress(xs, W, m, True, fp8)
        else:
            ext = torch.cat([h[-m:], xs], dim=0)
            res = backend.compress(ext, W, m, True, fp8)
            res = (res[0][1:], res[1][1:]) if fp8 else res[1:]
        if fp8:
            codes.append(res[0])
            scales.append(res[1])
        else:
            codes.append(res)
    if fp8:
        return torch.cat(codes, dim=0), torch.cat(scales, dim=0)
    return torch.cat(codes, dim=0)


def attend_spans(shard: Shard, q, qI, kv, halos_kv: list, kv_c, kI_c, kI_s, m: int, topk: int,
                 window: int, backend):
    """Stages 2 and 3 for the rank's queries, span by span, at their absolute
    positions; the window reads the halo rows before each span."""
    N_c = kv_c.shape[0]
    outs, idxs = [], []
    for (a, _), qs, qIs, kvs, h in zip(shard.spans, _span_rows(q, shard), _span_rows(qI, shard),
                                       _span_rows(kv, shard), halos_kv):
        idx = backend.indexer_topk(qIs, kI_c, kI_s, m, topk, a, N_c)
        kv_raw = torch.cat([h, kvs], dim=0) if h.shape[0] else kvs
        outs.append(backend.sparse_attn(qs, kv_c, idx, kv_raw, window, a, a - h.shape[0]))
        idxs.append(idx)
    return torch.cat(outs, dim=0), torch.cat(idxs, dim=0)


def cp_prefill(shard: Shard, q, kv, qI, kI_raw, W_c, W_Ic, m: int, topk: int, window: int,
               backend, indexer_fp8: bool = True, group=None) -> dict:
    """The CSA prefill of the rank's queries (its spans) of one sequence.

    q [L, H, D], kv [L, D], qI [L, H_I, d_I], kI_raw [L, d_I] are the rank's
    rows (take_rows: spans concatenated, L = shard.length); W_c, W_Ic are
    replicated.  Returns the rank's out [L, H, D] and idx [L, topk] (span
    order) plus the gathered compressed caches.
    """
    if kv.shape[0] != shard.length:
        raise ValueError("the shard tensors must hold the rank's span rows")
    # 1. left halos: one block for the overlapping compressor, W-1 rows for the
    #    window (every rank walks the same exchange list)
    many = len(shard.owners) > 1
    h_kv = max(m, window - 1) if many else 0
    if shard.chunk < h_kv:
        raise ValueError("each chunk must hold at least max(m, window - 1) tokens")
    halo_kv = exchange_halos(kv, h_kv, shard, group)
    halo_kI = exchange_halos(kI_raw, m if many else 0, shard, group)
    # 2. compression of the rank's spans
    kv_c_loc = compress_spans(shard, kv, halo_kv, W_c, m, False, backend)
    kI = compress_spans(shard, kI_raw, halo_kI, W_Ic, m, indexer_fp8, backend)
    # 3. every rank needs every entry
    kv_c = all_gather_spans(kv_c_loc, shard, group)
    if indexer_fp8:
        kI_c = all_gather_spans(kI[0], shard, group)
        kI_s = all_gather_spans(kI[1], shard, group)
    else:
        kI_c, kI_s = all_gather_spans(kI, shard, group), None
    # 4. the rank's queries at their absolute positions
    out, idx = attend_spans(shard, q, qI, kv, halo_kv, kv_c, kI_c, kI_s, m, topk, window,
                            backend)
    return dict(out=out, idx=idx, kv_c=kv_c, kI_c=kI_c, kI_scale=kI_s)


class CudaBackend:
    """The context-parallel arithmetic through this library's entry points:
    the positioned calls (csa_*_at) keep the prefill shape, so a span runs
    on the tensor-core indexer and attention kernels."""

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

    def indexer_topk(self, qI, kI, kI_scale, m, topk, q_pos0, n_entries):
        L = qI.shape[0]
        idx = torch.empty(1, L, topk, dtype=torch.int32, device=qI.device)
        ne = torch.tensor([n_entries], dtype=torch.int32, device=qI.device)
        self.api.csa_indexer_topk_at(
            qI[None].contiguous(), kI[None].contiguous(), m, topk, idx, q_pos0,
            kI_scale=None if kI_scale is None else kI_scale[None].contiguous(), n_entries=ne,
            stream=self.stream)
        return idx[0]

    def sparse_attn(self, q, kv_c, idx, kv_raw, window, q_pos0, raw_pos0):
        q1 = q[None].contiguous()
        out = torch.empty_like(q1)
        self.api.csa_sparse_attn_at(q1, kv_c[None].contiguous(), idx[None].contiguous(),
                                    kv_raw[None].contiguous(), window, out, q_pos0, raw_pos0,
                                    stream=self.stream)
        return out[0]
