"""Context-parallel prefill on host cores: two and four gloo ranks run the context-parallel
code (zigzag and contiguous layouts) with the oracle as the arithmetic, and the gathered
result must equal, bit for bit, the single-rank oracle run over the whole sequence.  This is
the CP = 1 vs CP > 1 agreement that the migration analysis names as the
risk of the layout.  Only the exchanges and bookkeeping are under
test; the oracle is plugged in from here."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N, H, D, H_I, d_I, M, K, WIN = 256, 4, 16, 2, 16, 4, 12, 24


class OracleBackend:
    """The oracle's stages on fp64 host tensors, shaped as cp_prefill calls them."""

    def __init__(self):
        import oracle
        self.o = oracle

    def compress(self, x, W, m, overlap, fp8):
        e = self.o.compress(x.numpy()[None], W.numpy(), m, overlap)[0]
        if fp8:
            codes, scales = self.o.quantize_rows_e4m3(e.astype(np.float32))
            return torch.from_numpy(codes), torch.from_numpy(scales)
        return torch.from_numpy(e)

    def indexer_topk(self, qI, kI, kI_scale, m, topk, q_pos0, n_entries):
        keys = kI.numpy()[None]
        sc = None if kI_scale is None else kI_scale.numpy()[None]
        L = qI.shape[0]
        q_pos = np.arange(q_pos0, q_pos0 + L, dtype=np.int32)
        idx, _, _ = self.o.indexer_topk_rows(qI.numpy(), np.zeros(L, np.int32), q_pos,
                                             keys, m, topk, np.array([n_entries], np.int32), sc)
        return torch.from_numpy(idx)

    def sparse_attn(self, q, kv_c, idx, kv_raw, window, q_pos0, raw_pos0):
        L = q.shape[0]
        q_pos = np.arange(q_pos0, q_pos0 + L, dtype=np.int32)
        o, _ = self.o.sparse_attn_rows(q.numpy(), np.zeros(L, np.int32), q_pos,
                                       kv_c.numpy()[None], idx.numpy(), kv_raw.numpy()[None],
                                       window, np.array([raw_pos0], np.int32),
                                       np.array([kv_raw.shape[0]], np.int32))
        return torch.from_numpy(o)


def _inputs():
    g = torch.Generator().manual_seed(4)
    f = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    return dict(q=f(N, H, D), kv=f(N, D), qI=f(N, H_I, d_I), kI_raw=f(N, d_I),
                W_c=f(D, D) / D ** 0.5, W_Ic=f(d_I, d_I) / d_I ** 0.5)


def _run(rank, world, inp, fp8, layout="zigzag", group=None):
    sys.path.insert(0, ROOT)
    from long_context_compressed_03_b200 import cp
    sh = cp.shard_of(N, world, rank, M, layout)
    loc = {k: (cp.take_rows(v, sh).contiguous() if k in ("q", "kv", "qI", "kI_raw") else v)
           for k, v in inp.items()}
    if fp8:       # cp_prefill hands fp8 query rows to the backend as values
        import oracle
        qv = oracle.quantized_query_rows(loc["qI"].numpy().astype(np.float32))
        loc["qI"] = torch.from_numpy(qv)
    return cp.cp_prefill(sh, loc["q"], loc["kv"], loc["qI"], loc["kI_raw"], loc["W_c"],
                         loc["W_Ic"], M, K, WIN, OracleBackend(), indexer_fp8=fp8, group=group)


def _rank_main(rank, world, port, fp8, layout, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = _run(rank, world, _inputs(), fp8, layout)
        q.put((rank, res["out"].numpy(), res["idx"].numpy(), res["kv_c"].numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,fp8,layout", [(2, True, "zigzag"), (4, False, "zigzag"),
                                              (4, True, "zigzag"), (2, False, "contiguous")])
def test_cp_ranks_reproduce_the_single_rank_run(world, fp8, layout):
    sys.path.insert(0, ROOT)
    from long_context_compressed_03_b200 import cp
    ref = _run(0, 1, _inputs(), fp8, "contiguous")       # one rank, one span: no exchange
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, fp8, layout, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=300) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shards = [cp.shard_of(N, world, r, M, layout) for r in range(world)]
    out = cp.place_rows([torch.from_numpy(g[1]) for g in got], shards, N).numpy()
    idx = cp.place_rows([torch.from_numpy(g[2]) for g in got], shards, N).numpy()
    for g in got:
        assert np.array_equal(g[3], ref["kv_c"].numpy())          # every rank holds every entry
    assert np.array_equal(idx, ref["idx"].numpy())
    assert np.array_equal(out, ref["out"].numpy())


def test_zigzag_spans_balance_the_causal_work():
    sys.path.insert(0, ROOT)
    from long_context_compressed_03_b200 import cp
    sh = cp.shard_of(64, 4, 1, 4)
    assert sh.spans == ((8, 16), (48, 56)) and sh.length == 16
    assert cp.chunk_owners(4, "zigzag") == (0, 1, 2, 3, 3, 2, 1, 0)
    # every position is held by exactly one rank
    cover = sorted(p for r in range(4) for a, b in cp.shard_of(64, 4, r, 4).spans
                   for p in range(a, b))
    assert cover == list(range(64))
    # indexer work (visible entries summed over the rank's queries) is equal across
    # zigzag ranks, and the contiguous last rank carries about (2W-1)/W^2 of it
    n, m, W = 65536, 4, 8
    work = lambda sh: sum(sum(range((a + 1) // m, (b + 1) // m)) for a, b in sh.spans)
    z = [work(cp.shard_of(n, W, r, m)) for r in range(W)]
    c = [work(cp.shard_of(n, W, r, m, "contiguous")) for r in range(W)]
    assert max(z) / min(z) < 1.001
    assert c[-1] / sum(c) == pytest.approx((2 * W - 1) / W ** 2, rel=1e-3)
    # take_rows / place_rows are inverse over the ranks
    x = torch.arange(64 * 3).reshape(64, 3)
    shs = [cp.shard_of(64, 4, r, 4) for r in range(4)]
    assert torch.equal(cp.place_rows([cp.take_rows(x, s) for s in shs], shs, 64), x)
    parts = [torch.full((2 * 2, 1), r) for r in range(4)]      # 2 rows per chunk
    assert cp.order_spans(parts, shs[0]).flatten().tolist() == \
        [0, 0, 1, 1, 2, 2, 3, 3, 3, 3, 2, 2, 1, 1, 0, 0]


def test_shards_must_cover_the_halo():
    sys.path.insert(0, ROOT)
    from long_context_compressed_03_b200 import cp
    sh = cp.shard_of(64, 2, 1, 4)              # zigzag: chunks of 16 tokens
    assert sh.spans == ((16, 32), (32, 48))
    with pytest.raises(ValueError):
        cp.shard_of(66, 4, 1, 4)
    loc = _inputs()
    with pytest.raises(ValueError):   # 16 tokens per chunk < window - 1
        cp.cp_prefill(sh, loc["q"][:32], loc["kv"][:32], loc["qI"][:32], loc["kI_raw"][:32],
                      loc["W_c"], loc["W_Ic"], 4, 4, 24, OracleBackend())
