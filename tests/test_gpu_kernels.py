"""GPU parity of each C-ABI entry point against the fp64 oracle, on seeded
inputs sized so the oracle finishes in seconds while the kernels still see
several tiles and ragged tails, plus the method's degenerate cases."""
import math

import numpy as np
import pytest
import torch

import oracle
from csa_checks import (ATOL_BF16, ATOL_F32, check_compress_stored, check_e4m3_rows, check_out,
                        check_topk, compress_bound, max_abs, np64, rotated_bound)
from long_context_compressed_03_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _randn(g, *shape, dtype=torch.float32, std=1.0):
    return (torch.randn(*shape, generator=g) * std).to(dtype)


# ---------------------------------------------------------------- compression
COMPRESS_CASES = [
    # (B, n, d_in, d_out, m, overlap, x dtype, out kind)
    (1, 512, 64, 64, 4, True, torch.float32, "f32"),        # fp32 main compressor
    (1, 512, 32, 32, 4, True, torch.float32, "f32"),        # fp32 indexer compressor
    (2, 1003, 128, 128, 4, True, torch.bfloat16, "bf16"),   # ragged tail, several tiles
    (2, 1003, 64, 64, 4, True, torch.bfloat16, "e4m3"),     # fp8 indexer keys
    (1, 4 * 128 + 77, 128, 128, 128, False, torch.bfloat16, "bf16"),   # HCA ratio
    (3, 37, 16, 48, 4, False, torch.bfloat16, "bf16"),
    (1, 9, 16, 16, 1, False, torch.float32, "f32"),         # m = 1
    (1, 8, 32, 32, 8, True, torch.float32, "f32"),          # n == m: one entry
]


@pytest.mark.parametrize("case", COMPRESS_CASES)
def test_compress_matches_oracle(case):
    B, n, d_in, d_out, m, overlap, dt, kind = case
    g = _gen(100 + n)
    x = _randn(g, B, n, d_in, dtype=dt)
    W = _randn(g, d_in, d_out, dtype=dt, std=1 / math.sqrt(d_in))
    ref = oracle.compress(np64(x), np64(W), m, overlap)
    bound = compress_bound(np64(x), np64(W), m, overlap)
    xd, Wd = x.to(DEV), W.to(DEV)
    if kind == "e4m3":
        codes, scale = api.compress(xd, Wd, m, overlap, out_dtype=torch.uint8)
        check_e4m3_rows(codes.cpu().numpy(), scale.cpu().numpy(), ref, bound)
        return
    out_dt = torch.float32 if kind == "f32" else torch.bfloat16
    out = api.compress(xd, Wd, m, overlap, out_dtype=out_dt)
    torch.cuda.synchronize()
    got = np64(out)
    assert got.shape == ref.shape
    check_compress_stored(got, ref, bound, out_dt)


def _hadamard64(d):
    """Normalised Sylvester-Hadamard matrix in fp64 (symmetric, orthonormal),
    built independently of the kernels' butterfly order."""
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h / math.sqrt(d)


@pytest.mark.parametrize("case", [
    # (B, n, d_in, d_out, m, overlap, x dtype)
    (2, 1003, 64, 64, 4, True, torch.bfloat16),     # fp8 indexer keys, ragged tail
    (1, 700, 128, 128, 4, True, torch.float32),
    (1, 300, 256, 256, 4, True, torch.bfloat16),
    (1, 200, 32, 16, 1, False, torch.bfloat16),
])
def test_compress_hadamard_fp8_matches_rotated_oracle(case):
    """Rows rotated by the normalised Walsh-Hadamard matrix before the fp8
    cast: the codes dequantise to H @ (oracle row) within one E4M3 step."""
    B, n, d_in, d_out, m, overlap, dt = case
    g = _gen(500 + n)
    x = _randn(g, B, n, d_in, dtype=dt)
    W = _randn(g, d_in, d_out, dtype=dt, std=1.0 / math.sqrt(d_in))
    unrot = oracle.compress(np64(x), np64(W), m, overlap)
    ref = unrot @ _hadamard64(d_out)
    bound = rotated_bound(compress_bound(np64(x), np64(W), m, overlap), np64(x), np64(W), m, overlap)
    codes, scale = api.compress(x.to(DEV), W.to(DEV), m, overlap, out_dtype=torch.uint8,
                                hadamard=True)
    codes, scale = codes.cpu().numpy(), scale.cpu().numpy()
    check_e4m3_rows(codes, scale, ref, bound)
    # rotating back recovers the row to within the fp8 error spread by H
    back = oracle.dequantize_rows_e4m3(codes, scale) @ _hadamard64(d_out)
    assert max_abs(back, unrot) <= 0.1 * np.abs(unrot).max()


GATED_CASES = [
    # (B, n, d_in, d_out, m, overlap, x dtype, out kind)
    (2, 1003, 64, 64, 4, True, torch.bfloat16, "bf16"),         # ratio 4, overlapping, ragged tail
    (1, 700, 128, 128, 4, True, torch.float32, "f32"),
    (1, 128 * 5 + 77, 128, 128, 128, False, torch.bfloat16, "bf16"),   # ratio 128: windows span steps
    (2, 300, 32, 48, 4, True, torch.bfloat16, "e4m3"),          # a half slice (48 = 32 + 16), fp8 out
    (1, 260, 64, 64, 4, True, torch.bfloat16, "e4m3_rot"),
    (1, 130, 16, 16, 1, True, torch.float32, "f32"),            # m = 1: 63 entries per CTA
    (1, 500, 16, 32, 64, True, torch.bfloat16, "bf16"),         # m = 64 overlapping: 128 positions
    (3, 37, 16, 16, 4, False, torch.float32, "f32"),
]


@pytest.mark.parametrize("case", GATED_CASES)
def test_compress_gated_matches_oracle(case):
    B, n, d_in, d_out, m, overlap, dt, kind = case
    c = 2 if overlap else 1
    g = _gen(300 + n + m)
    x = _randn(g, B, n, d_in, dtype=dt)
    W_kv = _randn(g, d_in, c * d_out, dtype=dt, std=1 / math.sqrt(d_in))
    W_g = _randn(g, d_in, c * d_out, dtype=dt, std=2 / math.sqrt(d_in))
    ape = _randn(g, m, c * d_out)
    ref = oracle.compress_gated(np64(x), np64(W_kv), np64(W_g), np64(ape), m, overlap)
    args = (x.to(DEV), W_kv.to(DEV), W_g.to(DEV), ape.to(DEV), m, overlap)
    if kind in ("e4m3", "e4m3_rot"):
        rot = kind == "e4m3_rot"
        if rot:
            ref = ref @ _hadamard64(d_out)
        codes, scale = api.compress_gated(*args, out_dtype=torch.uint8, hadamard=rot)
        codes, scale = codes.cpu().numpy(), scale.cpu().numpy()
        deq = oracle.dequantize_rows_e4m3(codes, scale)
        np.testing.assert_allclose(scale, np.abs(ref).max(axis=-1) / 448.0, rtol=1e-5)
        assert np.all(np.abs(deq - ref) <= np.abs(ref) * 2.0 ** -3 + scale[..., None] * 2.0 ** -9)
        return
    out_dt = torch.float32 if kind == "f32" else torch.bfloat16
    out = api.compress_gated(*args, out_dtype=out_dt)
    torch.cuda.synchronize()
    got = np64(out)
    assert got.shape == ref.shape
    check_out(got, ref, out_dt)
    if kind != "f32":
        # and within one bf16 step of the exact value
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5)


def test_compress_gated_flat_gates_equal_the_mean_pool_kernel():
    """Zero gate weights, constant APE and W_kv = [W | W]: the two compressors
    of this library agree (uniform softmax = mean, and the projection is linear)."""
    g = _gen(9)
    B, n, d, m = 2, 515, 64, 4
    x = _randn(g, B, n, d).to(DEV)
    W = _randn(g, d, d, std=1 / math.sqrt(d)).to(DEV)
    gated = api.compress_gated(x, torch.cat([W, W], 1), torch.zeros(d, 2 * d, device=DEV),
                               torch.full((m, 2 * d), 0.3, device=DEV), m, True)
    mean = api.compress(x, W, m, True)
    assert torch.allclose(gated, mean, atol=2e-5, rtol=1e-5)


def test_compress_no_entries_is_a_noop():
    x = torch.zeros(1, 3, 16, device=DEV, dtype=torch.bfloat16)
    W = torch.zeros(16, 16, device=DEV, dtype=torch.bfloat16)
    out = api.compress(x, W, 4, True)
    assert out.shape == (1, 0, 16)


# ---------------------------------------------------------------- indexer + top-k
def _index_case(seed, B, n, H_I, d_I, kind, k, n_entries=None, q_pos=None, ties=False):
    """Returns device inputs and the oracle's view of them."""
    g = _gen(seed)
    m = 4
    N = n // m
    if kind == "f32":
        qI = _randn(g, B, n, H_I, d_I)
        kI = _randn(g, B, N, d_I)
    else:
        qI = _randn(g, B, n, H_I, d_I, dtype=torch.bfloat16)
        kI = _randn(g, B, N, d_I, dtype=torch.bfloat16)
    if ties:
        kI[:, 1::3] = kI[:, 0:1]          # many exact duplicates of entry 0
    dev = dict(qI=qI.to(DEV))
    orc = {}
    qrows = np64(qI).reshape(B * n, H_I, d_I)
    if kind in ("f32", "bf16"):
        dev["kI"] = kI.to(DEV)
        orc["kI"] = np64(kI)
        orc["kI_scale"] = None
        orc["q_rows"] = qrows
    else:
        # fp8 keys come from the oracle-independent input cast in torch
        amax = kI.float().abs().amax(-1)
        sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        codes = (kI.float() / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
        dev["kI"], dev["kI_scale"] = codes.to(DEV), sc.to(DEV)
        orc["kI"], orc["kI_scale"] = codes.numpy(), sc.numpy()
        if kind == "e4m3_rot":
            # keys rotated in fp64 by an independent Sylvester matrix, cast by torch
            kr = torch.from_numpy(np64(kI) @ _hadamard64(d_I)).float()
            amax = kr.abs().amax(-1)
            sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
            codes = (kr / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
            dev["kI"], dev["kI_scale"] = codes.to(DEV), sc.to(DEV)
            orc["kI"], orc["kI_scale"] = codes.numpy(), sc.numpy()
            orc["q_rows"] = oracle.quantized_query_rows(qrows.astype(np.float32), rotate=True)
        elif kind == "e4m3_given":
            qa = qI.float().abs().amax(-1)
            qs = torch.where(qa > 0, qa / 448.0, torch.ones_like(qa))
            qc = (qI.float() / qs[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
            dev["qI"], dev["qI_scale"] = qc.to(DEV), qs.to(DEV)
            orc["q_rows"] = oracle.dequantize_rows_e4m3(qc.numpy(), qs.numpy()).reshape(B * n, H_I, d_I)
        else:
            orc["q_rows"] = oracle.quantized_query_rows(qrows.astype(np.float32))
    ne = np.full(B, N, np.int32) if n_entries is None else np.asarray(n_entries, np.int32)
    qp = np.broadcast_to(np.arange(n, dtype=np.int32), (B, n)) if q_pos is None else q_pos
    if n_entries is not None:
        dev["n_entries"] = torch.from_numpy(ne).to(DEV)
    if q_pos is not None:
        dev["q_pos"] = torch.from_numpy(np.ascontiguousarray(qp)).to(DEV)
    rows_b = np.repeat(np.arange(B, dtype=np.int32), n)
    rows_t = np.asarray(qp, np.int32).reshape(-1)
    return dev, orc, ne, rows_b, rows_t, m


INDEXER_CASES = [
    # (B, n, H_I, d_I, kind, k)
    (1, 512, 1, 32, "f32", 8),            # fp32: generic kernel
    (2, 700, 4, 64, "bf16", 32),          # tensor-core path, ragged last tile
    (2, 901, 4, 64, "e4m3", 64),          # bf16 queries quantised in the kernel
    (2, 912, 4, 64, "e4m3", 64),          # entry count a multiple of 4 (vector scales)
    (1, 1200, 4, 64, "e4m3_given", 100),
    (1, 4100, 2, 64, "e4m3", 300),        # two indexer heads, several CTAs
    (1, 333, 16, 32, "bf16", 7),          # 16 heads: generic kernel
    (2, 901, 4, 64, "e4m3_rot", 64),      # Hadamard-rotated keys, queries rotated in the kernel
    (1, 4100, 2, 64, "e4m3_rot", 300),
]


@pytest.mark.parametrize("case", INDEXER_CASES)
def test_indexer_topk_matches_oracle(case):
    B, n, H_I, d_I, kind, k = case
    dev, orc, ne, rb, rt, m = _index_case(7 + n, B, n, H_I, d_I, kind, k)
    idx = api.indexer_topk(dev["qI"], dev["kI"], m, k, qI_scale=dev.get("qI_scale"),
                           kI_scale=dev.get("kI_scale"), kI_rotated=kind == "e4m3_rot")
    got = idx.cpu().numpy().reshape(B * n, k)
    scores = oracle.indexer_scores_rows(orc["q_rows"], rb, rt, orc["kI"], m, ne, orc["kI_scale"])
    stats = check_topk(got, scores, k)
    assert stats["exact"] + stats["near_ties"] == stats["rows"]


@pytest.mark.parametrize("case", [
    # (B, n, H_I, d_I, kind, k, weight sign)
    (2, 700, 4, 64, "bf16", 32, "mixed"),        # tensor-core kernel, bf16
    (2, 901, 4, 64, "e4m3", 64, "mixed"),        # tensor-core kernel, fp8
    (1, 4100, 2, 64, "e4m3", 300, "mixed"),
    (1, 1200, 4, 64, "e4m3_rot", 100, "mixed"),  # with rotated keys
    (2, 901, 4, 64, "e4m3", 64, "negative"),     # every score <= 0: zeros first, lowest index
    (1, 512, 3, 32, "f32", 8, "mixed"),          # SIMT kernel
    (1, 333, 16, 32, "bf16", 7, "mixed"),
])
def test_indexer_gated_matches_oracle(case):
    """score = sum_h w_h ReLU(q_h . k) with per-(query, head) weights of any sign."""
    B, n, H_I, d_I, kind, k, sign = case
    dev, orc, ne, rb, rt, m = _index_case(31 + n, B, n, H_I, d_I, kind, k)
    w = torch.randn(B, n, H_I, generator=_gen(77 + n))
    if sign == "negative":
        w = -w.abs()
    idx = api.indexer_topk(dev["qI"], dev["kI"], m, k, qI_scale=dev.get("qI_scale"),
                           kI_scale=dev.get("kI_scale"), kI_rotated=kind == "e4m3_rot",
                           qI_weight=w.to(DEV))
    got = idx.cpu().numpy().reshape(B * n, k)
    scores = oracle.indexer_scores_rows(orc["q_rows"], rb, rt, orc["kI"], m, ne, orc["kI_scale"],
                                        weights=w.double().numpy().reshape(B * n, H_I))
    stats = check_topk(got, scores, k)
    assert stats["exact"] + stats["near_ties"] == stats["rows"]
    if sign == "negative":
        # rows with at least k zero scores take exactly the k lowest-index zeros
        for r in range(B * n):
            V = int(np.sum(~np.isnan(scores[r])))
            zeros = np.flatnonzero(scores[r][:V] == 0.0)
            if V > k and zeros.size >= k + 8:
                near = np.flatnonzero(np.abs(scores[r][:V]) < 1e-3)
                if near.size == zeros.size:          # no fp32-vs-fp64 sign doubt near zero
                    assert np.array_equal(np.sort(got[r]), zeros[:k])


def test_indexer_decode_positions_and_entry_counts():
    B, n_q, k = 3, 5, 16
    n = 400
    dev, orc, _, _, _, m = _index_case(11, B, n, 4, 64, "bf16", k)
    # decode-like: a few queries per element at arbitrary positions, fewer valid entries
    ne = np.array([100, 37, 3], np.int32)
    qp = np.array([[399, 150, 20, 3, 2], [399, 399, 399, 148, 0], [11, 12, 13, 14, 15]], np.int32)
    qsel = dev["qI"][:, :n_q].contiguous()
    idx = api.indexer_topk(qsel, dev["kI"], m, k, n_entries=torch.from_numpy(ne).to(DEV),
                           q_pos=torch.from_numpy(qp).to(DEV))
    got = idx.cpu().numpy().reshape(B * n_q, k)
    qrows = orc["q_rows"].reshape(B, n, 4, 64)[:, :n_q].reshape(B * n_q, 4, 64)
    rb = np.repeat(np.arange(B, dtype=np.int32), n_q)
    scores = oracle.indexer_scores_rows(qrows, rb, qp.reshape(-1), orc["kI"], m, ne)
    check_topk(got, scores, k)


def test_indexer_exact_ties_take_lowest_indices():
    B, n, k = 1, 600, 24
    dev, orc, ne, rb, rt, m = _index_case(12, B, n, 4, 64, "bf16", k, ties=True)
    idx = api.indexer_topk(dev["qI"], dev["kI"], m, k)
    got = idx.cpu().numpy().reshape(B * n, k)
    want, kth, _ = oracle.indexer_topk_rows(orc["q_rows"], rb, rt, orc["kI"], m, k, ne)
    scores = oracle.indexer_scores_rows(orc["q_rows"], rb, rt, orc["kI"], m, ne)
    check_topk(got, scores, k)
    # rows whose boundary is an exact tie: the GPU must take the same lowest indices
    tie_rows = np.flatnonzero(kth[:, 0] == kth[:, 1])
    assert tie_rows.size > 0
    for r in tie_rows:
        assert np.array_equal(np.sort(got[r][got[r] >= 0]), np.sort(want[r][want[r] >= 0]))


def test_indexer_all_zero_scores_pick_first_entries():
    B, n, k = 2, 256, 10
    qI = torch.zeros(B, n, 4, 64, dtype=torch.bfloat16, device=DEV)
    kI = torch.randn(B, n // 4, 64, generator=_gen(3)).to(torch.bfloat16).to(DEV)
    idx = api.indexer_topk(qI, kI, 4, k).cpu().numpy()
    for t in range(n):
        V = (t + 1) // 4
        sel = np.sort(idx[0, t][idx[0, t] >= 0])
        assert np.array_equal(sel, np.arange(min(V, k)))


def test_indexer_is_deterministic():
    dev, _, _, _, _, m = _index_case(13, 2, 901, 4, 64, "e4m3", 64)
    a = api.indexer_topk(dev["qI"], dev["kI"], m, 64, kI_scale=dev["kI_scale"])
    b = api.indexer_topk(dev["qI"], dev["kI"], m, 64, kI_scale=dev["kI_scale"])
    assert torch.equal(a, b)


# ---------------------------------------------------------------- attention
def _attn_inputs(seed, B, n_q, H, D, N_cap, L_raw, dt):
    g = _gen(seed)
    q = _randn(g, B, n_q, H, D, dtype=dt)
    kv_c = _randn(g, B, N_cap, D, dtype=dt)
    kv_raw = _randn(g, B, L_raw, D, dtype=dt)
    return q, kv_c, kv_raw


@pytest.mark.parametrize("dt,H,D", [(torch.float32, 8, 64), (torch.bfloat16, 64, 128),
                                    (torch.bfloat16, 16, 64), (torch.float32, 128, 128)])
def test_sparse_attention_matches_oracle(dt, H, D):
    B, n, W, k = 2, 97, 13, 9
    N = n // 4
    q, kv_c, kv = _attn_inputs(5 + H, B, n, H, D, N, n, dt)
    g = np.random.default_rng(H)
    idx = g.integers(-3, N + 3, size=(B, n, k)).astype(np.int32)   # padding + ignored + repeats
    idx[0, 5, :3] = 2                                               # duplicate entries count twice
    out, lse = api.sparse_attn(q.to(DEV), kv_c.to(DEV), torch.from_numpy(idx).to(DEV),
                               kv.to(DEV), W, with_lse=True)
    ro, rl = oracle.sparse_attn(np64(q), np64(kv_c), idx, np64(kv), W)
    check_out(np64(out).reshape(ro.shape), ro, dt)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(rl.shape), rl, atol=1e-3)


@pytest.mark.parametrize("m,W,n", [(128, 64, 700), (4, 40, 301), (1, 0, 50)])
def test_hca_attention_matches_oracle(m, W, n):
    B, H, D = 2, 64, 128
    N = n // m
    q, kv_c, kv = _attn_inputs(9 + n, B, n, H, D, N, n, torch.bfloat16)
    out, lse = api.hca_attn(q.to(DEV), kv_c.to(DEV), m, kv.to(DEV), W, with_lse=True)
    ro, rl = oracle.hca_attn(np64(q), np64(kv_c), m, np64(kv), W)
    got_o = np64(out).reshape(ro.shape)
    got_l = lse.cpu().numpy().reshape(rl.shape)
    empty = np.isneginf(rl)
    assert np.all(got_o[empty.all(axis=1)] == 0.0)
    assert np.array_equal(np.isneginf(got_l), empty)
    check_out(got_o, ro, torch.bfloat16)
    np.testing.assert_allclose(got_l[~empty], rl[~empty], atol=1e-3)


def test_decode_caches_with_partial_swa_and_entry_counts():
    B, H, D, N_cap, W, k = 4, 64, 128, 300, 32, 20
    q, kv_c, swa = _attn_inputs(21, B, 1, H, D, N_cap, W, torch.bfloat16)
    ctx = np.array([1000, 17, 40, 1200], np.int32)          # element 1: partly filled SWA
    q_pos = (ctx - 1).reshape(B, 1)
    raw_pos0 = ctx - W
    raw_len = np.full(B, W, np.int32)
    ne = np.minimum(ctx // 4, N_cap).astype(np.int32)
    g = np.random.default_rng(4)
    idx = np.stack([np.sort(g.choice(max(e, 1), size=k, replace=e < k)) for e in ne])
    idx = idx.reshape(B, 1, k).astype(np.int32)
    idx[1, 0, ne[1]:] = -1
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    out, lse = api.sparse_attn(q.to(DEV), kv_c.to(DEV), T(idx), swa.to(DEV), W, with_lse=True,
                               raw_pos0=T(raw_pos0), raw_len=T(raw_len), q_pos=T(q_pos))
    ro, rl = oracle.sparse_attn(np64(q), np64(kv_c), idx, np64(swa), W, q_pos=q_pos,
                                raw_pos0=raw_pos0, raw_len=raw_len)
    check_out(np64(out).reshape(ro.shape), ro, torch.bfloat16)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(rl.shape), rl, atol=1e-3)
    # HCA over the same caches
    out2, lse2 = api.hca_attn(q.to(DEV), kv_c.to(DEV), 4, swa.to(DEV), W, with_lse=True,
                              n_entries=T(ne), raw_pos0=T(raw_pos0), raw_len=T(raw_len),
                              q_pos=T(q_pos))
    ro2, rl2 = oracle.hca_attn(np64(q), np64(kv_c), 4, np64(swa), W, n_entries=ne, q_pos=q_pos,
                               raw_pos0=raw_pos0, raw_len=raw_len)
    check_out(np64(out2).reshape(ro2.shape), ro2, torch.bfloat16)


def test_window_only_and_explicit_scale():
    B, n, H, D, W = 1, 200, 8, 64, 50
    q, kv_c, kv = _attn_inputs(31, B, n, H, D, 4, n, torch.float32)
    out = api.sparse_attn(q.to(DEV), kv_c.to(DEV), None, kv.to(DEV), W, softmax_scale=0.3)
    ro, _ = oracle.sparse_attn(np64(q), np64(kv_c), np.zeros((B, n, 0), np.int32), np64(kv), W,
                               scale=0.3)
    check_out(np64(out).reshape(ro.shape), ro, torch.float32)


def test_attention_is_deterministic():
    q, kv_c, kv = _attn_inputs(41, 2, 64, 64, 128, 16, 64, torch.bfloat16)
    idx = torch.randint(-1, 16, (2, 64, 8), dtype=torch.int32, generator=_gen(1)).to(DEV)
    a = api.sparse_attn(q.to(DEV), kv_c.to(DEV), idx, kv.to(DEV), 16)
    b = api.sparse_attn(q.to(DEV), kv_c.to(DEV), idx, kv.to(DEV), 16)
    assert torch.equal(a, b)


def test_binding_rejects_host_tensors():
    x = torch.zeros(1, 8, 16)
    with pytest.raises(ValueError):
        api.csa_compress(x, torch.zeros(16, 16), 4, True, torch.zeros(1, 2, 16))


# ---------------------------------------------------------------- decode-time compression
@pytest.mark.parametrize("case", [
    # (B, n, d_in, d_out, m, overlap, x dtype, cache kind, N_cap)
    (3, 37, 128, 128, 4, True, torch.bfloat16, "bf16", 16),     # CSA main compressor, ragged
    (2, 41, 64, 64, 4, True, torch.bfloat16, "e4m3", 12),       # fp8 indexer-key cache
    (2, 57, 64, 64, 4, True, torch.bfloat16, "e4m3_rot", 16),   # Hadamard-rotated fp8 keys
    (2, 300, 128, 128, 128, False, torch.bfloat16, "bf16", 3),  # HCA ratio
    (1, 24, 32, 48, 4, False, torch.float32, "f32", 4),         # cache shorter than the stream
])
def test_compress_append_stream_matches_oracle(case):
    """Tokens fed one at a time through csa_compress_append rebuild the entries
    of the oracle's batch compression (positions staggered per element)."""
    B, n, d_in, d_out, m, overlap, dt, kind, N_cap = case
    g = _gen(200 + n)
    x = _randn(g, B, n, d_in, dtype=dt)
    W = _randn(g, d_in, d_out, dtype=dt, std=1 / math.sqrt(d_in))
    start = np.arange(B) * 3                     # element b starts its sequence at step 3b
    steps = n + int(start.max())
    state = torch.zeros(B, 2, d_in, dtype=torch.float32, device=DEV)
    if kind in ("e4m3", "e4m3_rot"):
        cache = torch.zeros(B, N_cap, d_out, dtype=torch.uint8, device=DEV)
        scale = torch.zeros(B, N_cap, dtype=torch.float32, device=DEV)
    else:
        cache = torch.zeros(B, N_cap, d_out, dtype=torch.float32 if kind == "f32" else torch.bfloat16,
                            device=DEV)
        scale = None
    n_ent = torch.zeros(B, dtype=torch.int32, device=DEV)
    xd, Wd = x.to(DEV), W.to(DEV)
    rows = torch.arange(B, device=DEV)
    for s in range(steps):
        p = s - start
        pos = torch.from_numpy(np.where((p >= 0) & (p < n), p, -1).astype(np.int32)).to(DEV)
        tok = xd[rows, torch.from_numpy(np.clip(p, 0, n - 1)).to(DEV)].contiguous()
        api.csa_compress_append(tok, Wd, m, overlap, pos, state, cache, cache_scale=scale,
                                n_entries=n_ent, hadamard=kind == "e4m3_rot")
    torch.cuda.synchronize()
    ref = oracle.compress(np64(x), np64(W), m, overlap)
    bound = compress_bound(np64(x), np64(W), m, overlap)
    if kind == "e4m3_rot":
        ref = ref @ _hadamard64(d_out)
        bound = rotated_bound(bound, np64(x), np64(W), m, overlap)
    N_w = min(N_cap, ref.shape[1])
    assert np.array_equal(n_ent.cpu().numpy(), np.full(B, min(n // m, N_cap), np.int32))
    if kind in ("e4m3", "e4m3_rot"):
        check_e4m3_rows(cache.cpu().numpy()[:, :N_w], scale.cpu().numpy()[:, :N_w], ref[:, :N_w],
                        bound[:, :N_w])
    else:
        check_compress_stored(np64(cache)[:, :N_w], ref[:, :N_w], bound[:, :N_w],
                              torch.float32 if kind == "f32" else torch.bfloat16)
