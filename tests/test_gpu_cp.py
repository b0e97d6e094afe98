"""The context-parallel prefill on one GPU with this library's kernels as the
arithmetic.  The spans of a shard run through the positioned entry points
(csa_indexer_topk_at / csa_sparse_attn_at), which keep the prefill shape and
so the tensor-core kernels.  A CP run must reproduce the single-call result
bit for bit: the span starts are multiples of the attention kernel's
4-token unit, so every query meets the same key tiles in the same order, and
the indexer writes each row's entries in ascending order.

Ranks are emulated in one process: each rank's halos are the rows before its
spans, read from the full sequence (what the exchange delivers), and the
all-gather is the per-rank entries put in sequence order.  The exchanges
themselves run on host cores with gloo ranks (test_cp_cpu.py)."""
import numpy as np
import pytest
import torch

import oracle
from csa_checks import check_out, check_topk, np64

from long_context_compressed_03_b200 import api, cp

pytestmark = pytest.mark.gpu
DEV = "cuda"
N, H, D, H_I, d_I, M, K, WIN = 4096, 64, 128, 4, 64, 4, 64, 128


def _inputs(seed=6):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *s, std=1.0: (torch.randn(*s, generator=g) * std).to(torch.bfloat16).to(DEV)
    return dict(q=bf(N, H, D), kv=bf(N, D), qI=bf(N, H_I, d_I), kI_raw=bf(N, d_I),
                W_c=bf(D, D, std=D ** -0.5), W_Ic=bf(d_I, d_I, std=d_I ** -0.5))


def _full(inp, fp8):
    r = api.csa_prefill(inp["q"][None], inp["kv"][None], inp["qI"][None], inp["kI_raw"][None],
                        inp["W_c"], inp["W_Ic"], M, K, WIN, indexer_fp8=fp8)
    return {k: (None if v is None else v[0]) for k, v in r.items()}


def _same(a, b):
    assert a.shape == b.shape and a.dtype == b.dtype
    assert torch.equal(a, b), f"{(a != b).sum().item()} of {a.numel()} elements differ"


@pytest.mark.parametrize("fp8", [True, False])
def test_one_rank_zigzag_matches_the_single_call(fp8):
    # world 1, zigzag: rank 0 holds both chunks; the second runs at q_pos0 = N/2
    inp = _inputs()
    sh = cp.shard_of(N, 1, 0, M)
    assert sh.spans == ((0, N // 2), (N // 2, N))
    res = cp.cp_prefill(sh, inp["q"], inp["kv"], inp["qI"], inp["kI_raw"], inp["W_c"],
                        inp["W_Ic"], M, K, WIN, cp.CudaBackend(), indexer_fp8=fp8)
    ref = _full(inp, fp8)
    torch.cuda.synchronize()
    for key in ("kv_c", "kI_c", "kI_scale", "idx", "out"):
        if ref[key] is not None:
            _same(res[key], ref[key])
    # and against the oracle on sampled rows of the second span
    rows = np.arange(N // 2, N, 97)
    kI = res["kI_c"].cpu().numpy()[None] if fp8 else np64(res["kI_c"])[None]
    sc = res["kI_scale"].cpu().numpy()[None] if fp8 else None
    qrows = inp["qI"][rows].float().cpu().numpy()
    qrows = oracle.quantized_query_rows(qrows) if fp8 else qrows.astype(np.float64)
    scores = oracle.indexer_scores_rows(qrows, np.zeros(rows.size, np.int32),
                                        rows.astype(np.int32), kI, M, np.array([N // M], np.int32), sc)
    idx = res["idx"].cpu().numpy()[rows]
    check_topk(idx, scores, K, label=f"CP span indexer (fp8={fp8})")
    ro, _ = oracle.sparse_attn_rows(np64(inp["q"])[rows], np.zeros(rows.size, np.int32),
                                    rows.astype(np.int32), np64(res["kv_c"])[None], idx,
                                    np64(inp["kv"])[None], WIN)
    check_out(np64(res["out"])[rows], ro, torch.bfloat16, label=f"CP span attention (fp8={fp8})")


@pytest.mark.parametrize("world,fp8", [(2, True), (4, True), (4, False)])
def test_emulated_zigzag_ranks_reproduce_the_single_call(world, fp8):
    inp = _inputs(seed=7)
    be = cp.CudaBackend()
    shards = [cp.shard_of(N, world, r, M) for r in range(world)]
    h_kv = max(M, WIN - 1)
    halos = lambda x, sh, rows: [x[max(0, a - rows):a] if a else x[:0] for a, _ in sh.spans]
    loc = [{k: cp.take_rows(inp[k], sh) for k in ("q", "kv", "qI", "kI_raw")} for sh in shards]
    # stage 1 on every rank, then the all-gather (entries in sequence order)
    kv_parts = [cp.compress_spans(sh, l["kv"], halos(inp["kv"], sh, h_kv), inp["W_c"], M, False, be)
                for sh, l in zip(shards, loc)]
    kI_parts = [cp.compress_spans(sh, l["kI_raw"], halos(inp["kI_raw"], sh, M), inp["W_Ic"], M,
                                  fp8, be) for sh, l in zip(shards, loc)]
    kv_c = cp.order_spans(kv_parts, shards[0])
    if fp8:
        kI_c = cp.order_spans([p[0] for p in kI_parts], shards[0])
        kI_s = cp.order_spans([p[1] for p in kI_parts], shards[0])
    else:
        kI_c, kI_s = cp.order_spans(kI_parts, shards[0]), None
    # stages 2 and 3 on every rank, results put back in sequence order
    outs, idxs = [], []
    for sh, l in zip(shards, loc):
        o, i = cp.attend_spans(sh, l["q"], l["qI"], l["kv"], halos(inp["kv"], sh, h_kv), kv_c,
                               kI_c, kI_s, M, K, WIN, be)
        outs.append(o)
        idxs.append(i)
    ref = _full(inp, fp8)
    torch.cuda.synchronize()
    _same(kv_c, ref["kv_c"])
    _same(kI_c, ref["kI_c"])
    if fp8:
        _same(kI_s, ref["kI_scale"])
    _same(cp.place_rows(idxs, shards, N), ref["idx"])
    _same(cp.place_rows(outs, shards, N), ref["out"])


def test_positioned_calls_equal_explicit_positions():
    # csa_*_at with offsets == the same calls with per-element position arrays
    # (the row kernels), on rows checked against the oracle: a span at 1000
    inp = _inputs(seed=8)
    a, L = 1000, 512
    full = _full(inp, True)
    kI_c, kI_s, kv_c = full["kI_c"][None], full["kI_scale"][None], full["kv_c"][None]
    idx_at = torch.empty(1, L, K, dtype=torch.int32, device=DEV)
    api.csa_indexer_topk_at(inp["qI"][None, a:a + L].contiguous(), kI_c, M, K, idx_at, a,
                            kI_scale=kI_s)
    q_pos = torch.arange(a, a + L, dtype=torch.int32, device=DEV)[None].contiguous()
    idx_pos = api.indexer_topk(inp["qI"][None, a:a + L].contiguous(), kI_c, M, K, kI_scale=kI_s,
                               q_pos=q_pos)
    torch.cuda.synchronize()
    # both are exact top-k sets; the row kernel's order within a row is its own
    _same(torch.sort(idx_at, dim=-1).values, torch.sort(idx_pos, dim=-1).values)
    raw0 = a - (WIN - 1)
    raw = inp["kv"][None, raw0:a + L].contiguous()
    out_at = torch.empty(1, L, H, D, dtype=torch.bfloat16, device=DEV)
    api.csa_sparse_attn_at(inp["q"][None, a:a + L].contiguous(), kv_c, idx_at, raw, WIN, out_at,
                           a, raw0)
    out_pos = api.sparse_attn(inp["q"][None, a:a + L].contiguous(), kv_c, idx_at, raw, WIN,
                              raw_pos0=torch.tensor([raw0], dtype=torch.int32, device=DEV),
                              q_pos=q_pos)
    torch.cuda.synchronize()
    rows = np.arange(0, L, 37)
    ro, _ = oracle.sparse_attn_rows(np64(inp["q"])[a + rows], np.zeros(rows.size, np.int32),
                                    (a + rows).astype(np.int32), np64(kv_c),
                                    idx_at.cpu().numpy()[0, rows], np64(raw), WIN,
                                    np.array([raw0], np.int32))
    check_out(np64(out_at)[0, rows], ro, torch.bfloat16, label="attention at an offset")
    check_out(np64(out_pos)[0, rows], ro, torch.bfloat16, label="attention, position arrays")
    # HCA dense at an offset against the oracle
    out_h = torch.empty_like(out_at)
    m_h = 128
    kvh = api.compress(inp["kv"][None], inp["W_c"], m_h, False)
    api.hca_dense_attn_at(inp["q"][None, a:a + L].contiguous(), kvh, m_h, raw, WIN, out_h, a, raw0)
    torch.cuda.synchronize()
    rh, _ = oracle.hca_attn_rows(np64(inp["q"])[a + rows], np.zeros(rows.size, np.int32),
                                 (a + rows).astype(np.int32), np64(kvh), m_h, np64(raw), WIN,
                                 raw_pos0=np.array([raw0], np.int32))
    check_out(np64(out_h)[0, rows], rh, torch.bfloat16, label="HCA at an offset")
