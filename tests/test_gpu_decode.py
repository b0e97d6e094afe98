"""GPU parity of the decode-shaped calls (few query rows over long caches)
against the fp64 oracle.  These shapes take the cluster-split kernels: one
row's entries or keys are shared by up to 16 CTAs whose partial results are
merged over distributed shared memory, so the cases below vary the cluster
size, put ties and invalid slots across CTA boundaries, and include rows
with nothing visible."""
import math

import numpy as np
import pytest
import torch

import oracle
from csa_checks import check_out, check_topk, np64

from long_context_compressed_03_b200 import api

pytestmark = pytest.mark.gpu
DEV = "cuda"


def T(a):
    if isinstance(a, torch.Tensor):
        return a.contiguous().to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _fp8_rows(x: torch.Tensor):
    """Per-row e4m3 codes and scales made by torch's own cast (not the oracle)."""
    amax = x.float().abs().amax(-1)
    sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (x.float() / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, sc


def _sylvester(d):
    """Normalised Sylvester-Hadamard matrix (fp64), independent of the kernels."""
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h / math.sqrt(d)


def _decode_indexer(seed, B, n_q, N_cap, H_I, d_I, k, ctx, q_kind="bf16", m=4, tie_rows=False,
                    gated=False):
    g = _gen(seed)
    qI = torch.randn(B, n_q, H_I, d_I, generator=g).to(torch.bfloat16)
    kI = torch.randn(B, N_cap, d_I, generator=g)
    if tie_rows:
        kI[:] = kI[:, :1]                        # every entry identical: all scores tie
    rot = q_kind == "bf16_rot"
    if rot:                                      # keys stored Hadamard-rotated
        kI = torch.from_numpy(kI.double().numpy() @ _sylvester(d_I)).float()
    codes, sc = _fp8_rows(kI)
    ne = np.minimum(np.asarray(ctx) // m, N_cap).astype(np.int32)
    q_pos = np.stack([np.asarray(ctx) - 1 - j for j in range(n_q)], axis=1).astype(np.int32)
    kw = dict(kI_scale=T(sc), n_entries=T(ne), q_pos=T(q_pos))
    w = torch.randn(B, n_q, H_I, generator=g) if gated else None
    if gated:
        kw["qI_weight"] = T(w)
    if q_kind == "e4m3":
        qc, qs = _fp8_rows(qI)
        idx = api.indexer_topk(T(qc), T(codes), m, k, qI_scale=T(qs), **kw)
        q_rows = oracle.dequantize_rows_e4m3(qc.numpy(), qs.numpy())
    else:
        idx = api.indexer_topk(T(qI), T(codes), m, k, kI_rotated=rot, **kw)
        q_rows = oracle.quantized_query_rows(qI.float().numpy(), rotate=rot)
    q_rows = q_rows.reshape(B * n_q, H_I, d_I)
    rb = np.repeat(np.arange(B, dtype=np.int32), n_q)
    wr = None if w is None else w.double().numpy().reshape(B * n_q, H_I)
    scores = oracle.indexer_scores_rows(q_rows, rb, q_pos.reshape(-1), codes.numpy(), m, ne, sc.numpy(),
                                        weights=wr)
    return idx.cpu().numpy().reshape(B * n_q, k), scores, ne, q_pos


@pytest.mark.parametrize("case", [
    # (B, n_q, N_cap, H_I, d_I, k, q kind)
    (5, 1, 3000, 4, 64, 64, "bf16"),        # a few CTAs per row
    (2, 2, 50000, 8, 128, 512, "e4m3"),     # 16-CTA clusters, more entries than one CTA holds
    (64, 4, 2100, 4, 64, 100, "bf16"),      # many rows: small clusters
    (3, 1, 9000, 1, 64, 2048, "bf16"),      # one head, the largest k
    (4, 1, 6000, 4, 64, 256, "bf16_rot"),   # Hadamard-rotated keys, query rotated in the kernel
    (2, 2, 30000, 8, 128, 512, "bf16_rot"), # d_I = 128: butterflies across a lane's own elements
])
def test_decode_indexer_matches_oracle(case):
    B, n_q, N_cap, H_I, d_I, k, qk = case
    rng = np.random.default_rng(N_cap)
    ctx = rng.integers(4 * k // 2, 4 * N_cap + 40, size=B)
    ctx[0] = 4 * N_cap + 3                  # every entry visible
    if B > 1:
        ctx[1] = 4 * k + 7                  # just above k visible
    if B > 2:
        ctx[2] = 4 * (k // 2)               # fewer visible than k: -1 padding
    got, scores, _, _ = _decode_indexer(17 + B, B, n_q, N_cap, H_I, d_I, k, ctx, qk)
    stats = check_topk(got, scores, k)
    assert stats["exact"] + stats["near_ties"] == stats["rows"]


@pytest.mark.parametrize("case", [
    # (B, n_q, N_cap, H_I, d_I, k, q kind)
    (5, 1, 3000, 4, 64, 64, "bf16"),
    (2, 2, 50000, 8, 128, 512, "e4m3"),     # 16-CTA clusters, signed keys across ranks
    (4, 1, 6000, 4, 64, 256, "bf16_rot"),
])
def test_decode_indexer_gated_matches_oracle(case):
    B, n_q, N_cap, H_I, d_I, k, qk = case
    rng = np.random.default_rng(N_cap + 1)
    ctx = rng.integers(4 * k, 4 * N_cap + 40, size=B)
    ctx[0] = 4 * N_cap + 3
    got, scores, _, _ = _decode_indexer(57 + B, B, n_q, N_cap, H_I, d_I, k, ctx, qk, gated=True)
    assert np.nanmin(scores) < 0.0                  # the weights made negative scores
    stats = check_topk(got, scores, k)
    assert stats["exact"] + stats["near_ties"] == stats["rows"]


def test_decode_indexer_ties_span_cluster_ranks():
    # all scores equal: the lowest k indices win, whichever CTA holds them
    B, N_cap, k = 2, 20000, 700
    got, scores, ne, _ = _decode_indexer(5, B, 1, N_cap, 4, 64, k, [4 * N_cap, 4 * 9000 + 2], tie_rows=True)
    for r in range(B):
        assert np.array_equal(np.sort(got[r]), np.arange(k))


def test_decode_indexer_is_deterministic():
    args = (9, 4, 1, 30000, 4, 64, 512, [120000, 90000, 70001, 4000])
    a, _, _, _ = _decode_indexer(*args)
    b, _, _, _ = _decode_indexer(*args)
    assert np.array_equal(a, b)


def _decode_attn_inputs(seed, B, H, D, N_cap, W):
    g = _gen(seed)
    q = torch.randn(B, 1, H, D, generator=g).to(torch.bfloat16)
    kv_c = torch.randn(B, N_cap, D, generator=g).to(torch.bfloat16)
    swa = torch.randn(B, W, D, generator=g).to(torch.bfloat16)
    return q, kv_c, swa


@pytest.mark.parametrize("H,D", [(64, 128), (16, 64), (32, 128), (128, 64), (128, 128)])
def test_decode_hca_matches_oracle(H, D):
    B, N_cap, W, m = 3, 5000, 256, 4
    q, kv_c, swa = _decode_attn_inputs(40 + H + D, B, H, D, N_cap, W)
    ctx = np.array([4 * N_cap + 1, 700, 1], np.int64)        # full, short, first token
    q_pos = (ctx - 1).reshape(B, 1).astype(np.int32)
    raw_pos0 = (ctx - W).astype(np.int32)
    raw_len = np.minimum(ctx, W).astype(np.int32)
    ne = np.minimum(ctx // m, N_cap).astype(np.int32)
    out, lse = api.hca_attn(T(q), T(kv_c), m, T(swa), W, with_lse=True, n_entries=T(ne),
                            raw_pos0=T(raw_pos0), raw_len=T(raw_len), q_pos=T(q_pos))
    ro, rl = oracle.hca_attn(np64(q), np64(kv_c), m, np64(swa), W, n_entries=ne, q_pos=q_pos,
                             raw_pos0=raw_pos0, raw_len=raw_len)
    check_out(np64(out).reshape(ro.shape), ro, torch.bfloat16)
    np.testing.assert_allclose(lse.cpu().numpy().reshape(rl.shape), rl, atol=1e-3)


def test_decode_csa_sparse_with_padding_repeats_and_empty_rows():
    B, H, D, N_cap, W, k = 6, 64, 128, 4000, 128, 512
    q, kv_c, swa = _decode_attn_inputs(77, B, H, D, N_cap, W)
    ctx = np.array([16000, 600, 1, 9000, 12345, 2], np.int64)
    q_pos = (ctx - 1).reshape(B, 1).astype(np.int32)
    raw_pos0 = (ctx - W).astype(np.int32)
    raw_len = np.minimum(ctx, W).astype(np.int32)
    raw_len[4] = 0                                    # an element whose window cache is empty
    ne = np.minimum(ctx // 4, N_cap).astype(np.int32)
    rng = np.random.default_rng(3)
    idx = np.full((B, 1, k), -1, np.int32)
    for b in range(B):
        v = int(ne[b])
        if v:
            idx[b, 0, :min(k, v)] = rng.choice(v, size=min(k, v), replace=False)
    idx[3, 0, 100:140] = idx[3, 0, 0]                 # repeated entries count every time
    idx[3, 0, 200:210] = -1                           # padding inside the row
    raw_len_dev = raw_len.copy()
    out, lse = api.sparse_attn(T(q), T(kv_c), T(idx), T(swa), W, with_lse=True,
                               raw_pos0=T(raw_pos0), raw_len=T(raw_len_dev), q_pos=T(q_pos))
    ro, rl = oracle.sparse_attn(np64(q), np64(kv_c), idx, np64(swa), W, q_pos=q_pos,
                                raw_pos0=raw_pos0, raw_len=raw_len)
    got_o = np64(out).reshape(ro.shape)
    got_l = lse.cpu().numpy().reshape(rl.shape)
    empty = np.isneginf(rl)
    assert np.array_equal(np.isneginf(got_l), empty)
    assert np.all(got_o[empty.all(axis=1)] == 0.0)
    check_out(got_o, ro, torch.bfloat16)
    np.testing.assert_allclose(got_l[~empty], rl[~empty], atol=1e-3)


def test_decode_attention_nothing_visible():
    # position 0 with an empty window cache and only padded index slots
    B, H, D, k, W = 2, 64, 128, 16, 8
    q, kv_c, swa = _decode_attn_inputs(8, B, H, D, 32, W)
    idx = np.full((B, 1, k), -1, np.int32)
    zeros = np.zeros(B, np.int32)
    out, lse = api.sparse_attn(T(q), T(kv_c), T(idx), T(swa), W, with_lse=True,
                               raw_pos0=T(zeros), raw_len=T(zeros), q_pos=T(zeros.reshape(B, 1)))
    assert torch.all(out == 0)
    assert torch.all(torch.isneginf(lse))


def test_decode_attention_is_deterministic():
    B, H, D, N_cap, W = 4, 64, 128, 6000, 512
    q, kv_c, swa = _decode_attn_inputs(12, B, H, D, N_cap, W)
    ctx = np.array([24000, 20000, 9000, 512], np.int64)
    kw = dict(n_entries=T(np.minimum(ctx // 4, N_cap).astype(np.int32)),
              raw_pos0=T((ctx - W).astype(np.int32)), raw_len=T(np.full(B, W, np.int32)),
              q_pos=T((ctx - 1).reshape(B, 1).astype(np.int32)))
    a = api.hca_attn(T(q), T(kv_c), 4, T(swa), W, **kw)
    b = api.hca_attn(T(q), T(kv_c), 4, T(swa), W, **kw)
    assert torch.equal(a, b)


@pytest.mark.parametrize("B", [3, 160])
def test_decode_csa_rows_of_mixed_shape_both_decode_kernels(B):
    # 64 heads x 128: up to one row per SM takes the tcgen05 decode kernel
    # (transposed score tiles, TMA window tiles, clusters sized by occupancy);
    # more rows than SMs take the mma.sync cluster kernel.  Rows mix a full
    # selection, a short context (index padding, a window shorter than W and
    # a compressed part that does not fill a tile) and the first token.
    H, D, N_cap, W, k = 64, 128, 3000, 256, 320
    q, kv_c, swa = _decode_attn_inputs(90 + B, B, H, D, N_cap, W)
    rng = np.random.default_rng(B)
    ctx = rng.integers(W + 1, 4 * N_cap, size=B).astype(np.int64)
    ctx[1] = 150                                      # 37 entries, window of 150
    ctx[2] = 1                                        # nothing compressed, one raw row
    q_pos = (ctx - 1).reshape(B, 1).astype(np.int32)
    raw_pos0 = (ctx - W).astype(np.int32)
    raw_len = np.minimum(ctx, W).astype(np.int32)
    ne = np.minimum(ctx // 4, N_cap)
    idx = np.full((B, 1, k), -1, np.int32)
    for b in range(B):
        v = int(ne[b])
        if v:
            idx[b, 0, :min(k, v)] = rng.choice(v, size=min(k, v), replace=False)
    out, lse = api.sparse_attn(T(q), T(kv_c), T(idx), T(swa), W, with_lse=True,
                               raw_pos0=T(raw_pos0), raw_len=T(raw_len), q_pos=T(q_pos))
    rows = np.unique(np.concatenate([[0, 1, 2], rng.choice(B, size=min(B, 12), replace=False)]))
    ro, rl = oracle.sparse_attn(np64(q)[rows], np64(kv_c)[rows], idx[rows], np64(swa)[rows], W,
                                q_pos=q_pos[rows], raw_pos0=raw_pos0[rows], raw_len=raw_len[rows])
    check_out(np64(out)[rows].reshape(ro.shape), ro, torch.bfloat16,
              label=f"decode attention, {B} rows of mixed shape")
    np.testing.assert_allclose(lse.cpu().numpy()[rows].reshape(rl.shape), rl, atol=1e-3)
