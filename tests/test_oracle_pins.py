"""Pins of the fp64 oracle to facts other than itself.

Each test checks the oracle against something the pages or the mathematics
fix: numbers printed on the pages (tests/golden), closed forms, special cases
that reduce to a library routine (torch's fp8 cast, scaled-dot-product
attention, numpy sorting), hand-enumerated windows and invariants.  They are
chosen so that a dropped term, a wrong sign or index, or a transposed operand
in the oracle fails at least one of them.  CPU only.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- fp8 E4M3
def _torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_matches_torch_for_every_code():
    ours = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    ref = _torch_e4m3_values()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x08] == 2.0 ** -6 and ours[0x01] == 2.0 ** -9


def _encode_grid():
    vals = _torch_e4m3_values()
    pos = np.unique(vals[(~np.isnan(vals)) & (vals >= 0)])
    mids = (pos[:-1] + pos[1:]) / 2.0                       # exact ties
    pts = [pos, mids]
    m32 = mids.astype(np.float32)
    pts.append(np.nextafter(m32, np.float32(np.inf)).astype(np.float64))
    pts.append(np.nextafter(m32, np.float32(-np.inf)).astype(np.float64))
    rng = np.random.default_rng(0)
    pts.append(rng.uniform(0, 448, 20000))
    pts.append(np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 20000)))
    g = np.concatenate(pts)
    g = g[g <= 448.0]
    return np.concatenate([g, -g]).astype(np.float32)


def test_e4m3_encode_matches_torch_cast():
    x = _encode_grid()
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch keeps the sign of a value that rounds to zero; so do we
    assert np.array_equal(ours, ref), np.flatnonzero(ours != ref)[:10]


def test_e4m3_saturates_above_448():
    x = np.array([448.0, 460.0, 464.0, 1e6, -1e30], dtype=np.float32)
    assert list(oracle.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_quantize_rows_scale_and_error_bound():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 64)).astype(np.float32)
    x[3] = 0.0
    codes, scales = oracle.quantize_rows_e4m3(x)
    assert scales[3] == 1.0 and not codes[3].any()
    amax = np.abs(x).max(axis=1)
    nz = amax > 0
    assert np.array_equal(scales[nz], (amax[nz] / np.float32(448.0)).astype(np.float32))
    # the row maximum lands on +-448 exactly
    arg = np.abs(x).argmax(axis=1)
    top = codes[np.arange(64), arg][nz]
    assert set(np.unique(top & 0x7F)) == {0x7E}
    # round-to-nearest error bound: half a quantum of E4M3 (3 mantissa bits)
    deq = oracle.dequantize_rows_e4m3(codes, scales)
    y = x.astype(np.float64) / scales[:, None]
    q = np.where(np.abs(y) < 2.0 ** -6, 2.0 ** -9,
                 2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 1e-30))) - 3))
    assert np.all(np.abs(deq / scales[:, None] - y) <= q / 2 + 1e-12)


# ---------------------------------------------------------------- compression
def test_entry_counts_printed_on_the_pages():
    rows = []
    with open(os.path.join(GOLDEN, "page_numbers.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(tuple(int(v) for v in line.split()))
    assert len(rows) == 3
    for n, m, want in rows:
        assert oracle.num_entries(n, m) == want


@pytest.mark.parametrize("overlap", [True, False])
def test_compress_constant_input_closed_form(overlap):
    rng = np.random.default_rng(2)
    c = 0.37
    W = rng.standard_normal((8, 5))
    x = np.full((2, 37, 8), c)
    out = oracle.compress(x, W, 4, overlap)
    assert out.shape == (2, 9, 5)
    # every entry -- including entry 0, whose overlapping window is clipped
    # at the sequence start -- equals c times the column sums of W
    np.testing.assert_allclose(out, np.broadcast_to(c * W.sum(axis=0), out.shape), rtol=0,
                               atol=1e-14)


def test_compress_hand_enumerated_windows():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 7, 3))
    I = np.eye(3)
    # m=2, n=7 -> floor(7/2) = 3 entries; token 6 forms no entry.
    overlap_windows = [[0, 1], [0, 1, 2, 3], [2, 3, 4, 5]]
    plain_windows = [[0, 1], [2, 3], [4, 5]]
    got_o = oracle.compress(x, I, 2, True)[0]
    got_p = oracle.compress(x, I, 2, False)[0]
    for i in range(3):
        np.testing.assert_allclose(got_o[i], x[0, overlap_windows[i]].mean(axis=0), atol=1e-15)
        np.testing.assert_allclose(got_p[i], x[0, plain_windows[i]].mean(axis=0), atol=1e-15)


def test_compress_projection_orientation():
    # one active input feature c: out[i] = pooled_c * W[c, :]  (row c of W)
    W = np.arange(12, dtype=np.float64).reshape(3, 4)
    x = np.zeros((1, 8, 3))
    x[0, :, 1] = 2.0
    out = oracle.compress(x, W, 4, True)[0]
    np.testing.assert_allclose(out, np.broadcast_to(2.0 * W[1], out.shape), atol=1e-14)


@pytest.mark.parametrize("overlap", [True, False])
def test_compress_invariant_to_order_inside_a_block(overlap):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1, 32, 6))
    W = rng.standard_normal((6, 6))
    ref = oracle.compress(x, W, 4, overlap)
    y = x.copy()
    y[0, 8:12] = y[0, [10, 8, 11, 9]]
    np.testing.assert_allclose(oracle.compress(y, W, 4, overlap), ref, atol=1e-13)
    # but moving a token across a block boundary changes the entries
    z = x.copy()
    z[0, [11, 12]] = z[0, [12, 11]]
    assert not np.allclose(oracle.compress(z, W, 4, overlap), ref)


def test_compress_ratio_one_is_identity():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 9, 4))
    np.testing.assert_array_equal(oracle.compress(x, np.eye(4), 1, False), x)


def test_compress_overlap_is_mean_of_two_plain_blocks():
    # with overlap, entry i (i >= 1) pools blocks i-1 and i, each of m rows
    rng = np.random.default_rng(6)
    x = rng.standard_normal((1, 40, 5))
    W = rng.standard_normal((5, 3))
    plain = oracle.compress(x, W, 4, False)[0]
    ov = oracle.compress(x, W, 4, True)[0]
    np.testing.assert_allclose(ov[1:], (plain[1:] + plain[:-1]) / 2, atol=1e-13)
    np.testing.assert_allclose(ov[0], plain[0], atol=1e-14)


# ---------------------------------------------------------------- indexer / top-k
def _lexsort_topk(scores_row, k):
    """numpy reference selection: score descending, index ascending."""
    idx = np.arange(scores_row.size)
    order = np.lexsort((idx, -scores_row))
    return order[:k]


def test_visible_entries_rule():
    # entry i becomes visible once its block [m i, m(i+1)) is complete
    assert [oracle.visible_entries(t, 4, 100) for t in range(10)] == [0, 0, 0, 1, 1, 1, 1, 2, 2, 2]
    assert oracle.visible_entries(1000, 4, 7) == 7
    assert oracle.visible_entries(-1, 4, 7) == 0


def test_single_head_positive_scores_order_like_plain_dot_product():
    # all-positive inputs: ReLU is inactive and the score is the dot product
    # of the page's einsum; top-k must agree with numpy's sort of q.k
    rng = np.random.default_rng(7)
    qI = rng.uniform(0.1, 1.0, (1, 64, 1, 16))
    kI = rng.uniform(0.1, 1.0, (1, 16, 16))
    idx, _, _ = oracle.indexer_topk(qI, kI, 4, 5)
    for t in range(64):
        V = min((t + 1) // 4, 16)
        dots = kI[0, :V] @ qI[0, t, 0]
        want = _lexsort_topk(dots, 5)
        got = idx[t][idx[t] >= 0]
        assert np.array_equal(got, want)


def test_relu_per_head_gives_absolute_dot_for_opposite_heads():
    # heads (q, -q): ReLU(x) + ReLU(-x) = |x|
    rng = np.random.default_rng(8)
    q1 = rng.standard_normal((1, 40, 1, 8))
    qI = np.concatenate([q1, -q1], axis=2)
    kI = rng.standard_normal((1, 10, 8))
    s = oracle.indexer_scores(qI, kI, 4)
    for t in range(40):
        V = min((t + 1) // 4, 10)
        np.testing.assert_allclose(s[t, :V], np.abs(kI[0, :V] @ q1[0, t, 0]), atol=1e-13)
        assert np.all(np.isnan(s[t, V:]))
    idx, _, _ = oracle.indexer_topk(qI, kI, 4, 3)
    for t in range(40):
        V = min((t + 1) // 4, 10)
        want = _lexsort_topk(np.abs(kI[0, :V] @ q1[0, t, 0]), 3)
        assert np.array_equal(idx[t][idx[t] >= 0], want)


def test_negative_dot_products_contribute_nothing():
    # single head, key = -query direction: score is exactly 0, not negative
    q = np.zeros((1, 8, 1, 4))
    q[0, :, 0, 0] = 1.0
    k = np.zeros((1, 2, 4))
    k[0, 0, 0] = -3.0
    k[0, 1, 0] = 2.0
    s = oracle.indexer_scores(q, k, 4)
    assert s[7, 0] == 0.0 and s[7, 1] == 2.0


def test_topk_causality_padding_and_full_sets():
    rng = np.random.default_rng(9)
    qI = rng.standard_normal((2, 50, 2, 8))
    kI = rng.standard_normal((2, 12, 8))
    n_ent = np.array([12, 9], dtype=np.int32)
    k = 6
    idx, kth, _ = oracle.indexer_topk(qI, kI, 4, k, n_entries=n_ent)
    idx = idx.reshape(2, 50, k)
    for b in range(2):
        for t in range(50):
            V = min((t + 1) // 4, n_ent[b])
            row = idx[b, t]
            sel = row[row >= 0]
            assert np.all(sel < V)
            assert len(set(sel.tolist())) == sel.size
            if V <= k:
                assert sorted(sel.tolist()) == list(range(V))
                assert np.all(row[V:] == -1)
            else:
                assert sel.size == k


def test_topk_ties_take_lowest_indices():
    qI = np.ones((1, 40, 1, 4))
    kI = np.ones((1, 10, 4))          # every score equal
    kI[0, 7] *= 2.0                   # one clear winner
    idx, _, _ = oracle.indexer_topk(qI, kI, 4, 3)
    assert sorted(idx[39].tolist()) == [0, 1, 7]


def test_topk_invariant_to_positive_query_scale():
    rng = np.random.default_rng(10)
    qI = rng.standard_normal((1, 80, 3, 8))
    kI = rng.standard_normal((1, 20, 8))
    a, _, _ = oracle.indexer_topk(qI, kI, 4, 7)
    b, _, _ = oracle.indexer_topk(qI * 3.7, kI, 4, 7)
    assert np.array_equal(a, b)


def test_kth_scores_match_numpy_sort():
    rng = np.random.default_rng(11)
    qI = rng.standard_normal((1, 60, 2, 8))
    kI = rng.standard_normal((1, 15, 8))
    k = 4
    _, kth, smax = oracle.indexer_topk(qI, kI, 4, k)
    s = oracle.indexer_scores(qI, kI, 4)
    for t in range(60):
        row = s[t][~np.isnan(s[t])]
        srt = np.sort(row)[::-1]
        if row.size >= k:
            assert kth[t, 0] == srt[k - 1]
        if row.size > k:
            assert kth[t, 1] == srt[k]
        if row.size:
            assert smax[t] == np.abs(row).max()


# ---------------------------------------------------------------- gated compressor
def test_gated_compress_hand_worked_example():
    # m = 2, no overlap, d_in = d_out = 1, W_kv = 1, W_gate = ln 2, ape = 0:
    # weights are 2^x, so block (1, 2) pools to (2*1 + 4*2)/6 = 5/3 and block
    # (3, 4) to (8*3 + 16*4)/24 = 11/3; the trailing position 5 makes no entry
    x = np.array([[[1.0], [2.0], [3.0], [4.0], [5.0]]])
    out = oracle.compress_gated(x, np.ones((1, 1)), np.full((1, 1), math.log(2.0)),
                                np.zeros((2, 1)), 2, False)
    np.testing.assert_allclose(out[0, :, 0], [5.0 / 3.0, 11.0 / 3.0], rtol=1e-15)


def test_gated_compress_overlap_routes_channel_halves_by_block():
    # d_out = 1, overlap: the previous block is read through projected channel
    # 0 and the current block through channel 1.  W_kv = (1, 10) and equal
    # logits: entry 0 = mean of 10 x over block 0; entry i > 0 = mean of
    # (x over block i-1, 10 x over block i)
    x = np.arange(1.0, 9.0).reshape(1, 8, 1)
    out = oracle.compress_gated(x, np.array([[1.0, 10.0]]), np.zeros((1, 2)), np.zeros((2, 2)),
                                2, True)
    assert out.shape == (1, 4, 1)
    np.testing.assert_allclose(out[0, 0, 0], 10 * (1 + 2) / 2)
    for i in range(1, 4):
        prev = x[0, 2 * i - 2:2 * i, 0]
        cur = 10 * x[0, 2 * i:2 * i + 2, 0]
        np.testing.assert_allclose(out[0, i, 0], (prev.sum() + cur.sum()) / 4, rtol=1e-15)


@pytest.mark.parametrize("overlap", [True, False])
def test_gated_compress_with_flat_gates_is_the_mean_pool(overlap):
    # zero gate weights and a constant APE give a uniform softmax; with both
    # channel halves of W_kv equal to W this is mean-then-project (linear)
    rng = np.random.default_rng(31)
    B, n, d_in, d_out, m = 2, 37, 6, 5, 4
    x = rng.standard_normal((B, n, d_in))
    W = rng.standard_normal((d_in, d_out))
    c = 2 if overlap else 1
    W_kv = np.concatenate([W] * c, axis=1)
    ape = np.full((m, c * d_out), 0.7)
    got = oracle.compress_gated(x, W_kv, np.zeros((d_in, c * d_out)), ape, m, overlap)
    np.testing.assert_allclose(got, oracle.compress(x, W, m, overlap), rtol=1e-12, atol=1e-12)


def test_gated_compress_dominant_gate_selects_one_position():
    # a logit 60 above the rest puts weight 1 - O(e^-60) on one position
    rng = np.random.default_rng(32)
    B, n, d_in, d_out, m = 1, 16, 3, 2, 4
    x = rng.standard_normal((B, n, d_in))
    W_kv = rng.standard_normal((d_in, 2 * d_out))
    ape = np.zeros((m, 2 * d_out))
    ape[1, d_out:] = 60.0          # current block, its position 1, every channel
    out = oracle.compress_gated(x, W_kv, np.zeros((d_in, 2 * d_out)), ape, m, True)
    for i in range(n // m):
        v = x[0, m * i + 1] @ W_kv[:, d_out:]
        np.testing.assert_allclose(out[0, i], v, rtol=1e-12, atol=1e-12)


def test_gated_compress_is_causal_and_shift_invariant_in_the_logits():
    rng = np.random.default_rng(33)
    B, n, d_in, d_out, m = 1, 24, 4, 3, 4
    x = rng.standard_normal((B, n, d_in))
    W_kv = rng.standard_normal((d_in, 2 * d_out))
    W_g = rng.standard_normal((d_in, 2 * d_out))
    ape = rng.standard_normal((m, 2 * d_out))
    a = oracle.compress_gated(x, W_kv, W_g, ape, m, True)
    y = x.copy()
    y[0, 13:] += 5.0               # entries 0..2 end before position 12
    b = oracle.compress_gated(y, W_kv, W_g, ape, m, True)
    assert np.array_equal(a[0, :3], b[0, :3]) and not np.allclose(a[0, 3:], b[0, 3:])
    c = oracle.compress_gated(x, W_kv, W_g, ape + 3.25, m, True)
    np.testing.assert_allclose(c, a, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- gated indexer
def test_gated_scores_hand_worked_example():
    # two heads, d = 2, weights (2, -3); worked by hand:
    #   key (1,0):  dots ( 1, -1) -> 2*1 + -3*0 =  2
    #   key (0,1):  dots ( 2,  1) -> 2*2 + -3*1 =  1
    #   key (1,1):  dots ( 3,  0) -> 2*3 + -3*0 =  6
    #   key (-1,-1): dots (-3, 0) -> 0
    #   key (-1,0): dots (-1,  1) -> 0 + -3*1  = -3
    q = np.array([[[[1.0, 2.0], [-1.0, 1.0]]]])                     # [1, 1, 2, 2]
    k = np.array([[[1, 0], [0, 1], [1, 1], [-1, -1], [-1, 0]]], dtype=np.float64)
    w = np.array([[[2.0, -3.0]]])
    pos = np.array([[19]], np.int32)                                 # all 5 entries visible
    s = oracle.indexer_scores(q, k, 4, q_pos=pos, weights=w)
    assert s[0].tolist() == [2.0, 1.0, 6.0, 0.0, -3.0]
    idx, kth, smax = oracle.indexer_topk(q, k, 4, 5, q_pos=pos, weights=w)
    assert idx[0].tolist() == [2, 0, 1, 3, 4]                        # negatives rank below zero
    idx3, kth3, _ = oracle.indexer_topk(q, k, 4, 3, q_pos=pos, weights=w)
    assert idx3[0].tolist() == [2, 0, 1] and kth3[0].tolist() == [1.0, 0.0]
    assert smax[0] == 6.0


def test_unit_weights_and_one_hot_weights_reduce_to_known_scores():
    rng = np.random.default_rng(21)
    qI = rng.standard_normal((2, 30, 4, 8))
    kI = rng.standard_normal((2, 9, 8))
    plain = oracle.indexer_scores(qI, kI, 4)
    ones = oracle.indexer_scores(qI, kI, 4, weights=np.ones((2, 30, 4)))
    assert np.array_equal(np.isnan(plain), np.isnan(ones))
    assert np.array_equal(plain[~np.isnan(plain)], ones[~np.isnan(ones)])
    for j in range(4):
        onehot = np.zeros((2, 30, 4))
        onehot[..., j] = 1.0
        got = oracle.indexer_scores(qI, kI, 4, weights=onehot)
        single = oracle.indexer_scores(qI[:, :, j:j + 1], kI, 4)
        ok = ~np.isnan(single)
        assert np.array_equal(got[ok], single[ok])


def test_gated_scores_are_linear_and_odd_in_the_weights():
    rng = np.random.default_rng(22)
    qI = rng.standard_normal((1, 40, 3, 8))
    kI = rng.standard_normal((1, 10, 8))
    w1 = rng.standard_normal((1, 40, 3))
    w2 = rng.standard_normal((1, 40, 3))
    s1 = oracle.indexer_scores(qI, kI, 4, weights=w1)
    s2 = oracle.indexer_scores(qI, kI, 4, weights=w2)
    s12 = oracle.indexer_scores(qI, kI, 4, weights=2.5 * w1 + w2)
    ok = ~np.isnan(s1)
    np.testing.assert_allclose(s12[ok], 2.5 * s1[ok] + s2[ok], rtol=1e-12, atol=1e-12)
    neg = oracle.indexer_scores(qI, kI, 4, weights=-w1)
    assert np.array_equal(neg[ok], -s1[ok])                         # each term negates exactly


def test_gated_topk_matches_brute_force_on_tiny_inputs():
    # per-head ReLU dots and the weighted sum written out with Python loops
    rng = np.random.default_rng(23)
    H, d, N, n, k = 3, 4, 11, 48, 5
    qI = rng.standard_normal((1, n, H, d))
    kI = rng.standard_normal((1, N, d))
    w = rng.standard_normal((1, n, H))
    idx, _, _ = oracle.indexer_topk(qI, kI, 4, k, weights=w)
    for t in range(n):
        V = min((t + 1) // 4, N)
        scores = []
        for s_ in range(V):
            tot = 0.0
            for h in range(H):
                dot = sum(float(qI[0, t, h, c]) * float(kI[0, s_, c]) for c in range(d))
                tot += float(w[0, t, h]) * max(dot, 0.0)
            scores.append(tot)
        want = sorted(range(V), key=lambda i: (-scores[i], i))[:k]
        assert idx[t][:min(k, V)].tolist() == want


# ---------------------------------------------------------------- attention
def _sdpa_mqa(q, kv, mask=None, causal=False):
    """torch scaled_dot_product_attention in fp64 with one shared KV head."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                   # [B, H, n, D]
    kt = torch.from_numpy(kv)[:, None].expand(-1, q.shape[2], -1, -1)
    m = None if mask is None else torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(qt, kt, kt, attn_mask=m, is_causal=causal)
    return o.permute(0, 2, 1, 3).numpy()


def test_hca_ratio_one_identity_projection_is_causal_sdpa():
    rng = np.random.default_rng(12)
    B, n, H, D = 2, 33, 3, 16
    q = rng.standard_normal((B, n, H, D))
    kv = rng.standard_normal((B, n, D))
    kv_c = oracle.compress(kv, np.eye(D), 1, False)
    o, lse = oracle.hca_attn(q, kv_c, 1, kv, 0)
    ref = _sdpa_mqa(q, kv, causal=True)
    np.testing.assert_allclose(o.reshape(B, n, H, D), ref, atol=1e-12)
    assert np.all(np.isfinite(lse))


def test_window_only_is_banded_sdpa():
    rng = np.random.default_rng(13)
    B, n, H, D, W = 1, 40, 2, 8, 7
    q = rng.standard_normal((B, n, H, D))
    kv = rng.standard_normal((B, n, D))
    idx = np.full((B, n, 3), -1, np.int32)
    o, _ = oracle.sparse_attn(q, np.zeros((B, 1, D)), idx, kv, W)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    band = (j <= i) & (j >= i - W + 1)        # the page's start = max(0, i-W+1)
    ref = _sdpa_mqa(q, kv, mask=band)
    np.testing.assert_allclose(o.reshape(B, n, H, D), ref, atol=1e-12)
    # a window covering everything is plain causal attention
    o2, _ = oracle.sparse_attn(q, np.zeros((B, 1, D)), idx, kv, n + 5)
    np.testing.assert_allclose(o2.reshape(B, n, H, D), _sdpa_mqa(q, kv, causal=True), atol=1e-12)


def _dense_masked_reference(q, kv_c, kv_raw, m, W, scale):
    """Softmax over the concatenation [kv_c ; kv_raw] with the visibility
    mask of compressed entries and the window mask of raw rows (numpy)."""
    B, n, H, D = q.shape
    N = kv_c.shape[1]
    out = np.zeros_like(q)
    for b in range(B):
        keys = np.concatenate([kv_c[b], kv_raw[b]], axis=0)
        t = np.arange(n)[:, None]
        s = np.arange(N)[None, :]
        p = np.arange(kv_raw.shape[1])[None, :]
        mask = np.concatenate([s < (t + 1) // m, (p <= t) & (p >= t - W + 1)], axis=1)
        z = np.einsum("thd,kd->thk", q[b], keys) * scale
        z = np.where(mask[:, None, :], z, -np.inf)
        z = z - z.max(axis=-1, keepdims=True)
        w = np.exp(z)
        w /= w.sum(axis=-1, keepdims=True)
        out[b] = np.einsum("thk,kd->thd", w, keys)
    return out


def test_sparse_with_every_entry_selected_equals_dense_and_hca():
    rng = np.random.default_rng(14)
    B, n, H, D, m, W = 2, 48, 4, 8, 4, 9
    q = rng.standard_normal((B, n, H, D))
    kv = rng.standard_normal((B, n, D))
    Wc = rng.standard_normal((D, D)) / math.sqrt(D)
    kv_c = oracle.compress(kv, Wc, m, True)
    N = kv_c.shape[1]
    idx = np.full((B, n, N), -1, np.int32)
    for t in range(n):
        V = (t + 1) // m
        idx[:, t, :V] = np.arange(V)[::-1]        # order must not matter
    o_s, lse_s = oracle.sparse_attn(q, kv_c, idx, kv, W)
    o_h, lse_h = oracle.hca_attn(q, kv_c, m, kv, W)
    ref = _dense_masked_reference(q, kv_c, kv, m, W, 1 / math.sqrt(D))
    np.testing.assert_allclose(o_s.reshape(ref.shape), ref, atol=1e-12)
    np.testing.assert_allclose(o_h, o_s, atol=1e-12)
    np.testing.assert_allclose(lse_h, lse_s, atol=1e-12)


def test_constant_keys_give_the_constant_and_log_count_lse():
    B, n, H, D = 1, 20, 2, 4
    rng = np.random.default_rng(15)
    q = rng.standard_normal((B, n, H, D))
    v = np.array([0.5, -1.0, 2.0, 0.25])
    kv = np.broadcast_to(v, (B, n, D)).copy()
    kv_c = np.broadcast_to(v, (B, 5, D)).copy()
    idx = np.tile(np.array([0, 1, -1], np.int32), (B, n, 1))
    W = 6
    o, lse = oracle.sparse_attn(q, kv_c, idx, kv, W)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), atol=1e-14)
    t = np.arange(n)
    count = 2 + np.minimum(t + 1, W)
    z = (q[0] @ v) / 2.0                             # scale 1/sqrt(4)
    np.testing.assert_allclose(lse, z + np.log(count)[:, None], atol=1e-12)


def test_compressed_and_raw_copies_of_one_vector_both_count():
    # multiset union: a compressed entry equal to a raw row is a second key
    a = np.array([1.0, 0.0])
    c = np.array([0.0, 1.0])
    q = np.array([[[[2.0, 0.0]]]])                   # [1,1,1,2], position 0
    kv_raw = a[None, None, :]                        # raw position 0 = a
    kv_c = np.stack([a, c])[None]                    # entries: a, c
    idx = np.array([[[0, 1]]], np.int32)
    o, lse = oracle.sparse_attn(q, kv_c, idx, kv_raw, 1, scale=1.0)
    za, zc = 2.0, 0.0
    want = (2 * math.exp(za) * a + math.exp(zc) * c) / (2 * math.exp(za) + math.exp(zc))
    np.testing.assert_allclose(o[0, 0], want, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], math.log(2 * math.exp(za) + math.exp(zc)), atol=1e-14)


def test_empty_key_set_gives_zero_and_minus_inf():
    q = np.ones((1, 3, 2, 4))
    kv_c = np.ones((1, 2, 4))
    kv = np.ones((1, 3, 4))
    o, lse = oracle.hca_attn(q, kv_c, 4, kv, 0)     # no entry visible yet, no window
    assert np.all(o == 0.0) and np.all(np.isneginf(lse))


def test_decode_window_uses_absolute_positions_and_drops_negative_ones():
    # SWA cache slots hold positions raw_pos0 + j; negative positions are void
    rng = np.random.default_rng(16)
    D = 4
    q = rng.standard_normal((1, 1, 1, D))
    swa = rng.standard_normal((1, 4, D))
    idx = np.full((1, 1, 1), -1, np.int32)
    # context of 2 tokens held in a 4-slot cache: slots 0,1 are positions -2,-1
    o, _ = oracle.sparse_attn(q, np.zeros((1, 1, D)), idx, swa, 4, q_pos=np.array([[1]]),
                              raw_pos0=np.array([-2]), raw_len=np.array([4]))
    keys = swa[0, 2:4]
    z = keys @ q[0, 0, 0] / 2.0
    w = np.exp(z - z.max())
    np.testing.assert_allclose(o[0, 0], (w / w.sum()) @ keys, atol=1e-14)


def test_end_to_end_is_causal():
    # perturbing tokens after t leaves every output at positions <= t unchanged
    rng = np.random.default_rng(17)
    B, n, H, D, HI, dI = 1, 64, 2, 8, 2, 8
    q = rng.standard_normal((B, n, H, D))
    kv = rng.standard_normal((B, n, D))
    qI = rng.standard_normal((B, n, HI, dI))
    kI = rng.standard_normal((B, n, dI))
    Wc = rng.standard_normal((D, D))
    WIc = rng.standard_normal((dI, dI))
    o1, l1, i1 = oracle.csa_forward(q, kv, qI, kI, Wc, WIc, 4, 3, 5)
    t = 37
    q2, kv2, qI2, kI2 = (a.copy() for a in (q, kv, qI, kI))
    for a in (q2, kv2, qI2, kI2):
        a[:, t + 1:] = rng.standard_normal(a[:, t + 1:].shape)
    o2, l2, i2 = oracle.csa_forward(q2, kv2, qI2, kI2, Wc, WIc, 4, 3, 5)
    assert np.array_equal(o1[:t + 1], o2[:t + 1])
    assert np.array_equal(i1[:t + 1], i2[:t + 1])
    assert not np.allclose(o1[t + 1:], o2[t + 1:])


# ---------------------------------------------------------------- decode-time compression state
def test_append_stream_equals_batch_compression():
    # feeding a sequence one token at a time must rebuild exactly the entries
    # the (separately pinned) batch compressor computes, ragged tails included
    rng = np.random.default_rng(31)
    for B, n, d_in, d_out, m, overlap in [(2, 37, 16, 24, 4, True), (3, 300, 32, 16, 128, False),
                                          (1, 9, 8, 8, 1, False), (2, 64, 16, 16, 4, False),
                                          (1, 4, 8, 8, 4, True)]:
        x = rng.standard_normal((B, n, d_in))
        W = rng.standard_normal((d_in, d_out))
        np.testing.assert_allclose(oracle.compress_stream(x, W, m, overlap),
                                   oracle.compress(x, W, m, overlap), rtol=0, atol=1e-12)


def test_append_writes_only_on_block_completion_and_skips_absent_tokens():
    rng = np.random.default_rng(32)
    B, d, m = 3, 8, 4
    W = rng.standard_normal((d, d))
    state = np.zeros((B, 2, d))
    out = np.full((B, 5, d), 7.0)
    # element 0 at positions 0..3 (completes entry 0 at p=3), element 1 has no token, element 2
    # starts at position 4 (its first block is absent: only block 1 completes, alone)
    for p in range(4):
        x = rng.standard_normal((B, d))
        done = oracle.compress_append(state, x, W, m, True, np.array([p, -1, 4 + p], np.int32), out, 5)
        want = [0 if p == 3 else -1, -1, 1 if p == 3 else -1]
        assert list(done) == want
    assert np.all(out[1] == 7.0) and np.all(state[1] == 0.0)      # untouched element
    assert np.all(out[0, 1:] == 7.0) and np.all(out[2, [0, 2, 3, 4]] == 7.0)
    assert np.all(state[:, 1][[0, 2]] == 0.0)                      # running sums restarted


def test_append_constant_input_and_cache_bound():
    # constant rows c: every entry is c * (column sums of W), overlap or not;
    # an entry past N_cap is not written but the state still advances
    d, m, c = 8, 4, 0.75
    W = np.random.default_rng(33).standard_normal((d, 5))
    for overlap in (True, False):
        state = np.zeros((1, 2, d))
        out = np.zeros((1, 2, 5))
        for p in range(4 * m):
            done = oracle.compress_append(state, np.full((1, d), c), W, m, overlap,
                                          np.array([p], np.int32), out, 2)
            if (p + 1) % m == 0:
                assert done[0] == p // m
        np.testing.assert_allclose(out[0], np.tile(c * W.sum(axis=0), (2, 1)), rtol=0, atol=1e-12)
        assert np.allclose(state[0, 0], m * c)                   # last complete block's sum


# ---------------------------------------------------------------- Hadamard rotation (indexer rows)
def _sylvester(d):
    H = np.array([[1.0]])
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H / np.sqrt(d)


def test_hadamard_rows_match_the_sylvester_matrix():
    rng = np.random.default_rng(41)
    for d in (16, 64, 128):
        x = rng.standard_normal((5, d)).astype(np.float32)
        got = oracle.hadamard_rows_f32(x).astype(np.float64)
        want = x.astype(np.float64) @ _sylvester(d).T
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-5 * np.abs(want).max())


def test_hadamard_is_an_involution_and_keeps_dot_products():
    rng = np.random.default_rng(42)
    q = rng.standard_normal((64, 64)).astype(np.float32)
    k = rng.standard_normal((64, 64)).astype(np.float32)
    hq, hk = oracle.hadamard_rows_f32(q), oracle.hadamard_rows_f32(k)
    np.testing.assert_allclose(oracle.hadamard_rows_f32(hq), q, rtol=0, atol=1e-5)
    dots = (q.astype(np.float64) * k).sum(-1)
    hdots = (hq.astype(np.float64) * hk).sum(-1)
    np.testing.assert_allclose(hdots, dots, rtol=0, atol=1e-4)
    # an outlier channel is spread over every coordinate: the row amax drops
    x = np.zeros((1, 64), np.float32)
    x[0, 5] = 100.0
    assert np.allclose(np.abs(oracle.hadamard_rows_f32(x)), 12.5)


def test_rotated_query_quantisation_is_rotate_then_quantise():
    rng = np.random.default_rng(43)
    q = rng.standard_normal((7, 4, 64)).astype(np.float32)
    codes, scales = oracle.quantize_rows_e4m3(oracle.hadamard_rows_f32(q))
    np.testing.assert_array_equal(oracle.quantized_query_rows(q, rotate=True),
                                  oracle.dequantize_rows_e4m3(codes, scales))
