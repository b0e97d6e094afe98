"""GPU parity of the packed (varlen) prefill entry points.  Sequences of mixed
lengths (including an empty one and ones shorter than a block) are packed
along the token dimension; every result must equal, bit for bit, the
unpacked call on each sequence alone, and match the oracle run per sequence."""
import numpy as np
import pytest
import torch

import oracle
from csa_checks import check_out, check_topk, np64

from long_context_compressed_03_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"
LENS = [700, 1, 0, 1303, 64, 2]      # m = 4: 175, 0, 0, 325, 16, 0 entries


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def _inputs(seed, lens, H=64, D=128, H_I=4, d_I=64):
    g = _gen(seed)
    T = int(sum(lens))
    return dict(
        q=torch.randn(T, H, D, generator=g).to(torch.bfloat16),
        kv=torch.randn(T, D, generator=g).to(torch.bfloat16),
        qI=torch.randn(T, H_I, d_I, generator=g).to(torch.bfloat16),
        kI_raw=torch.randn(T, d_I, generator=g).to(torch.bfloat16),
        W_c=(torch.randn(D, D, generator=g) / D ** 0.5).to(torch.bfloat16),
        W_Ic=(torch.randn(d_I, d_I, generator=g) / d_I ** 0.5).to(torch.bfloat16))


def test_entry_offsets():
    assert api.varlen_entry_offsets(_cu(LENS), 4).tolist() == [0, 175, 175, 175, 500, 516, 516]


def test_varlen_prefill_equals_per_sequence_calls_and_oracle():
    m, k, W = 4, 64, 128
    cu = _cu(LENS)
    e = api.varlen_entry_offsets(cu, m)
    inp = _inputs(1, LENS)
    d = {n: v.to(DEV) for n, v in inp.items()}
    T, E = int(cu[-1]), int(e[-1])
    kv_c = torch.empty(E, 128, dtype=torch.bfloat16, device=DEV)
    kI_c = torch.empty(E, 64, dtype=torch.uint8, device=DEV)
    kI_s = torch.empty(E, dtype=torch.float32, device=DEV)
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    out = torch.empty_like(d["q"])
    lse = torch.empty(T, 64, device=DEV)
    api.csa_compress_varlen(d["kv"], cu, d["W_c"], m, True, kv_c)
    api.csa_compress_varlen(d["kI_raw"], cu, d["W_Ic"], m, True, kI_c, kI_s)
    api.csa_indexer_topk_varlen(d["qI"], kI_c, cu, m, k, idx, kI_scale=kI_s)
    api.csa_sparse_attn_varlen(d["q"], cu, kv_c, m, idx, d["kv"], W, out, lse_out=lse)
    torch.cuda.synchronize()
    for s, L in enumerate(LENS):
        t0, t1, e0, e1 = cu[s], cu[s + 1], e[s], e[s + 1]
        if L == 0:
            continue
        # the unpacked calls on this sequence alone: identical bits
        ref_kv = api.compress(d["kv"][None, t0:t1].contiguous(), d["W_c"], m, True)
        ref_kI, ref_s = api.compress(d["kI_raw"][None, t0:t1].contiguous(), d["W_Ic"], m, True,
                                     out_dtype=torch.uint8)
        assert torch.equal(kv_c[e0:e1], ref_kv[0])
        assert torch.equal(kI_c[e0:e1], ref_kI[0]) and torch.equal(kI_s[e0:e1], ref_s[0])
        ref_idx = api.indexer_topk(d["qI"][None, t0:t1].contiguous(), ref_kI, m, k, kI_scale=ref_s)
        assert torch.equal(idx[t0:t1], ref_idx[0])
        ref_o, ref_l = api.sparse_attn(d["q"][None, t0:t1].contiguous(), ref_kv, ref_idx,
                                       d["kv"][None, t0:t1].contiguous(), W, with_lse=True)
        assert torch.equal(out[t0:t1], ref_o[0]) and torch.equal(lse[t0:t1], ref_l[0])
        # the oracle on this sequence
        orc_kv = oracle.compress(np64(inp["kv"][None, t0:t1]), np64(inp["W_c"]), m, True)
        check_out(np64(kv_c[e0:e1])[None], orc_kv, torch.bfloat16)
        n_e = e1 - e0
        rows = np.arange(L, dtype=np.int32)
        q_rows = oracle.quantized_query_rows(inp["qI"][t0:t1].float().numpy())
        scores = oracle.indexer_scores_rows(q_rows, np.zeros(L, np.int32), rows,
                                            kI_c[e0:e1].cpu().numpy()[None], m,
                                            np.array([n_e], np.int32), kI_s[e0:e1].cpu().numpy()[None])
        check_topk(idx[t0:t1].cpu().numpy(), scores, k)
        ro, _ = oracle.sparse_attn(np64(inp["q"][None, t0:t1]), np64(kv_c[e0:e1])[None],
                                   idx[t0:t1].cpu().numpy()[None], np64(inp["kv"][None, t0:t1]), W)
        check_out(np64(out[t0:t1])[None], ro, torch.bfloat16)


def test_varlen_hca_equals_per_sequence_calls_and_oracle():
    m, W = 128, 256
    lens = [700, 0, 1500, 130]
    cu = _cu(lens)
    e = api.varlen_entry_offsets(cu, m)
    inp = _inputs(2, lens)
    d = {n: v.to(DEV) for n, v in inp.items()}
    kv_c = torch.empty(int(e[-1]), 128, dtype=torch.bfloat16, device=DEV)
    out = torch.empty_like(d["q"])
    api.csa_compress_varlen(d["kv"], cu, d["W_c"], m, False, kv_c)
    api.hca_dense_attn_varlen(d["q"], cu, kv_c, m, d["kv"], W, out)
    torch.cuda.synchronize()
    for s, L in enumerate(lens):
        t0, t1, e0, e1 = cu[s], cu[s + 1], e[s], e[s + 1]
        if L == 0:
            continue
        ref_kv = api.compress(d["kv"][None, t0:t1].contiguous(), d["W_c"], m, False)
        ref_o = api.hca_attn(d["q"][None, t0:t1].contiguous(), ref_kv, m,
                             d["kv"][None, t0:t1].contiguous(), W)
        assert torch.equal(out[t0:t1], ref_o[0])
        ro, _ = oracle.hca_attn(np64(inp["q"][None, t0:t1]), np64(kv_c[e0:e1])[None], m,
                                np64(inp["kv"][None, t0:t1]), W)
        check_out(np64(out[t0:t1])[None], ro, torch.bfloat16)


def test_varlen_many_sequences_and_fallback_shapes():
    """130 short sequences (more than one launch's parameter map holds) and
    fp32 / 16-head operands (not served by the tensor-core kernels): both go
    through one launch per sequence and must equal the per-sequence calls."""
    m, k, W, H, D, H_I, d_I = 4, 8, 16, 16, 64, 2, 32
    rng = np.random.default_rng(5)
    lens = rng.integers(0, 40, size=130).tolist()
    cu = _cu(lens)
    e = api.varlen_entry_offsets(cu, m)
    T, E = int(cu[-1]), int(e[-1])
    g = _gen(9)
    q = torch.randn(T, H, D, generator=g).to(DEV)
    kv = torch.randn(T, D, generator=g).to(DEV)
    qI = torch.randn(T, H_I, d_I, generator=g).to(DEV)
    kI_raw = torch.randn(T, d_I, generator=g).to(DEV)
    W_c = (torch.randn(D, D, generator=g) / D ** 0.5).to(DEV)
    W_Ic = (torch.randn(d_I, d_I, generator=g) / d_I ** 0.5).to(DEV)
    kv_c = torch.empty(E, D, device=DEV)
    kI_c = torch.empty(E, d_I, device=DEV)
    idx = torch.empty(T, k, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    api.csa_compress_varlen(kv, cu, W_c, m, True, kv_c)
    api.csa_compress_varlen(kI_raw, cu, W_Ic, m, True, kI_c)
    api.csa_indexer_topk_varlen(qI, kI_c, cu, m, k, idx)
    api.csa_sparse_attn_varlen(q, cu, kv_c, m, idx, kv, W, out)
    torch.cuda.synchronize()
    for s, L in enumerate(lens):
        t0, t1, e0, e1 = cu[s], cu[s + 1], e[s], e[s + 1]
        if L == 0:
            continue
        rk = api.compress(kv[None, t0:t1].contiguous(), W_c, m, True)
        ri = api.compress(kI_raw[None, t0:t1].contiguous(), W_Ic, m, True)
        assert torch.equal(kv_c[e0:e1], rk[0]) and torch.equal(kI_c[e0:e1], ri[0])
        rx = api.indexer_topk(qI[None, t0:t1].contiguous(), ri, m, k)
        assert torch.equal(idx[t0:t1], rx[0])
        ro = api.sparse_attn(q[None, t0:t1].contiguous(), rk, rx, kv[None, t0:t1].contiguous(), W)
        assert torch.equal(out[t0:t1], ro[0])
