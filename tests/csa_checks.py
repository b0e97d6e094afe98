"""Shared comparison helpers for the parity tests (no method arithmetic here).

Tolerances (stated once, used by every parity test):
  * attention outputs, max-abs against the fp64 oracle: 1e-4 for fp32
    paths; 2e-2 for bf16 paths wherever half a bf16 ulp of the exact value
    is at most 2e-2 (|ref| < 8).  From |ref| >= 8 on no bf16 value need lie
    within 2e-2 of the exact result, so there the stored value must be the
    bf16 rounding of some value within 2e-2 of it: |got - ref| <= 2e-2 +
    half an ulp of |ref|;
  * compression outputs (fp32 or bf16 storage) are held to the fp32
    arithmetic they need: the stored value is the correct rounding of a
    value within gamma_n * S of the exact one, where S = mean|x| @ |W| is
    the sum of the absolute terms and n the terms one output adds up;
  * fp8 (E4M3) compression codes: bit-exact against the oracle's fp32
    quantiser applied to the oracle's row, except for elements whose scaled
    value lies within the fp32 error bound of an E4M3 rounding midpoint
    (counted and reported: there either neighbour is a correct rounding);
  * top-k index sets: identical except where the oracle's k-th and (k+1)-th
    scores lie within delta = 1e-3 * max(|s_k|, |s_k+1|) + 1e-6 * max_s |s|
    of each other (a near-tie); inside a near-tie every index scoring above
    s_k + delta must be chosen and every chosen index must score at least
    s_k+1 - delta.
Near-ties are common by construction at large V (thousands of visible
entries put consecutive order statistics ~1e-4 apart relative, and ReLU
makes exact ties at 0), so their count is reported, not bounded.

Every check records its observed error and margin in ``LOG``; the test
session prints the log at the end (tests/conftest.py).
"""
from __future__ import annotations

import os

import numpy as np
import torch

ATOL_BF16 = 2e-2
ATOL_F32 = 1e-4
TOPK_REL = 1e-3
TOPK_ABS_FRAC = 1e-6
U32 = 2.0 ** -24           # unit roundoff of fp32

LOG: list[str] = []


def _label(label):
    if label:
        return label
    cur = os.environ.get("PYTEST_CURRENT_TEST", "?")
    return cur.split(" ")[0].split("::")[-1]


def record(label, **vals) -> None:
    parts = ", ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}" for k, v in vals.items())
    line = f"{_label(label)}: {parts}"
    LOG.append(line)
    print("[parity] " + line)


def np64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a float tensor (any device)."""
    return t.detach().to("cpu", torch.float64).numpy()


def atol_for(dtype: torch.dtype) -> float:
    return ATOL_F32 if dtype == torch.float32 else ATOL_BF16


def half_ulp(x: np.ndarray, mant_bits: int) -> np.ndarray:
    """Half the spacing of a binary format with `mant_bits` stored mantissa
    bits at magnitude |x| (normal range; bf16: 7, fp32: 23)."""
    ax = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(ax > 0, 2.0 ** (e - mant_bits - 1), 2.0 ** (-126 - mant_bits - 1))


def bf16_out_tol(ref: np.ndarray) -> np.ndarray:
    """Per-element bound for a bf16-stored output (see the module header)."""
    h = half_ulp(ref, 7)
    return np.where(h <= ATOL_BF16, ATOL_BF16, ATOL_BF16 + h)


def check_out(got: np.ndarray, ref: np.ndarray, dtype, label: str | None = None) -> float:
    """Output tolerance for a kernel result stored in `dtype`; returns the
    max abs error."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if got.shape != ref.shape:            # the same elements with a unit axis more or less
        assert got.size == ref.size, f"shape {got.shape} != {ref.shape}"
        got = got.reshape(ref.shape)
    if got.size == 0:
        return 0.0
    err = np.abs(got - ref)
    if dtype == torch.float32:
        tol = np.full(err.shape, ATOL_F32)
    else:
        tol = bf16_out_tol(ref)
    margin = float(np.min(tol - err))
    worst = int(np.argmax(err - tol))
    record(label, max_abs=float(err.max()), min_margin=margin, n=int(err.size),
           big=int(np.count_nonzero(np.abs(ref) >= 8)))
    assert margin >= 0, (f"error {err.flat[worst]} > tolerance {tol.flat[worst]} at |ref| = "
                         f"{abs(ref.flat[worst])}")
    return float(err.max())


def compress_error_bound(S: np.ndarray, n_terms: int) -> np.ndarray:
    """gamma_n * S: the fp32 error bound of an output that adds n_terms terms
    whose absolute values sum to at most S."""
    g = n_terms * U32 / (1.0 - n_terms * U32)
    return g * np.asarray(S, np.float64)


def check_compress_stored(got: np.ndarray, ref: np.ndarray, bound: np.ndarray, dtype,
                          label: str | None = None) -> None:
    """A stored compression output is the correct rounding (bf16 or fp32) of
    a value within `bound` of the exact one, and within the north-star
    tolerance."""
    got = np.asarray(got, np.float64)
    if got.shape != ref.shape:
        assert got.size == ref.size, f"shape {got.shape} != {ref.shape}"
        got = got.reshape(ref.shape)
    err = np.abs(got - ref)
    mant = 23 if dtype == torch.float32 else 7
    tol = bound + half_ulp(np.abs(ref) + bound, mant)
    margin = float(np.min(tol - err)) if err.size else 0.0
    record(label, max_abs=float(err.max()) if err.size else 0.0, min_margin_rounding=margin,
           n=int(err.size))
    assert margin >= 0, "stored output is not a correct rounding of the fp32 result"
    assert float(err.max() if err.size else 0.0) <= atol_for(dtype)


_MIDS = None


def _e4m3_midpoints() -> np.ndarray:
    """Midpoints between consecutive non-negative finite E4M3 values."""
    global _MIDS
    if _MIDS is None:
        import oracle
        v = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))   # 0x00 .. 0x7E (0x7F is NaN)
        v = np.sort(v)
        _MIDS = (v[:-1] + v[1:]) / 2.0
    return _MIDS


def check_e4m3_rows(codes: np.ndarray, scale: np.ndarray, ref: np.ndarray, bound: np.ndarray,
                    label: str | None = None) -> dict:
    """fp8 rows from the GPU against the oracle's fp32 quantiser applied to
    the oracle's row (`ref`, fp64, cast to fp32 first).  `bound` bounds the
    GPU row's fp32 error per element.  Codes must be identical except where
    the scaled value lies within its error bound of a rounding midpoint."""
    import oracle
    ref = np.asarray(ref, np.float64)
    codes = np.asarray(codes, np.uint8)
    scale = np.asarray(scale, np.float64)
    rcodes, rscale = oracle.quantize_rows_e4m3(ref.astype(np.float32))
    amax = np.abs(ref).max(axis=-1)
    brow = np.asarray(bound).max(axis=-1)
    # scale = amax / 448 of the GPU's row: within the row's bound / 448
    s_tol = brow / 448.0 + 2.0 ** -23 * np.abs(rscale) + 1e-30
    zero = amax == 0
    s_ref = np.where(zero, 1.0, amax / 448.0)
    assert np.all(np.abs(scale - s_ref) <= s_tol), "per-row scale off by more than its bound"
    t = np.abs(ref) / s_ref[..., None]
    rel_s = brow / np.where(zero, 1.0, amax) + 2.0 ** -23
    delta = np.asarray(bound) / s_ref[..., None] + t * (2 * rel_s[..., None] + 4 * U32)
    mids = _e4m3_midpoints()
    j = np.clip(np.searchsorted(mids, t), 1, mids.size - 1)
    dist = np.minimum(np.abs(t - mids[j - 1]), np.abs(t - mids[j]))
    near = dist <= delta
    same = (codes == rcodes) | (((codes & 0x7F) == 0) & ((rcodes & 0x7F) == 0))
    bad = ~same & ~near
    nmis = int(np.count_nonzero(~same))
    stats = dict(elements=int(codes.size), mismatches=nmis,
                 exempt_near_midpoint=int(np.count_nonzero(~same & near)),
                 near_midpoint_total=int(np.count_nonzero(near)))
    record(label, **stats)
    assert not np.any(bad), (f"{int(np.count_nonzero(bad))} E4M3 codes differ away from a rounding "
                             f"midpoint")
    # an exempt element may only sit one code step away
    if nmis:
        dv = np.abs(oracle.e4m3_decode(codes[~same]) - oracle.e4m3_decode(rcodes[~same]))
        step = 2.0 * np.abs(oracle.e4m3_decode(rcodes[~same])) * 2.0 ** -3 + 2.0 ** -9
        assert np.all(dv <= step), "an exempt code is more than one E4M3 step away"
    return stats


def check_topk(gpu_idx: np.ndarray, scores: np.ndarray, k: int, label: str | None = None) -> dict:
    """Check GPU top-k rows against the oracle's full score rows.

    gpu_idx [R, k] int32; scores [R, N_cap] fp64 with NaN for invisible
    entries.  Returns counters; raises AssertionError with the first failing
    row."""
    R = gpu_idx.shape[0]
    near = 0
    exact = 0
    for r in range(R):
        row = gpu_idx[r]
        srow = scores[r]
        vis = np.flatnonzero(~np.isnan(srow))
        V = vis.size
        if V:
            assert vis[-1] == V - 1, f"row {r}: visible entries are not a prefix"
        chosen = row[row >= 0]
        assert np.all(row[chosen.size:] == -1), f"row {r}: -1 padding is not a suffix"
        assert chosen.size == min(k, V), f"row {r}: {chosen.size} chosen, expected {min(k, V)}"
        assert np.unique(chosen).size == chosen.size, f"row {r}: duplicate indices"
        assert np.all(chosen < V), f"row {r}: index beyond the visible entries (V={V})"
        if V <= k:
            exact += 1
            continue
        s = srow[:V]
        order = np.lexsort((np.arange(V), -s))
        sk, sk1 = s[order[k - 1]], s[order[k]]
        delta = TOPK_REL * max(abs(sk), abs(sk1)) + TOPK_ABS_FRAC * np.abs(s).max()
        if sk - sk1 > delta:
            want = np.sort(order[:k])
            got = np.sort(chosen)
            assert np.array_equal(want, got), (
                f"row {r}: set mismatch outside a near-tie "
                f"(s_k={sk}, s_k+1={sk1}); missing {np.setdiff1d(want, got)[:8]}, "
                f"extra {np.setdiff1d(got, want)[:8]}")
            exact += 1
        else:
            near += 1
            must = np.flatnonzero(s > sk + delta)
            assert np.all(np.isin(must, chosen)), f"row {r}: near-tie row misses a clear winner"
            assert np.all(s[chosen] >= sk1 - delta), f"row {r}: near-tie row chose a clear loser"
    stats = dict(rows=R, exact=exact, near_ties=near)
    record(label, **stats)
    return stats


def max_abs(a: np.ndarray, b: np.ndarray) -> float:
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))


def compress_bound(x: np.ndarray, W: np.ndarray, m: int, overlap: bool) -> np.ndarray:
    """fp32 error bound of each compression output: gamma_n * (mean|x| @ |W|)
    with n = the window's additions (at most 2m) + the projection's d_in
    terms + the division and the final rounding."""
    import oracle
    S = oracle.compress(np.abs(x), np.abs(W), m, overlap)
    return compress_error_bound(S, (2 * m if overlap else m) + x.shape[-1] + 2)


def rotated_bound(bound: np.ndarray, x: np.ndarray, W: np.ndarray, m: int, overlap: bool) -> np.ndarray:
    """Error bound after the normalised Walsh-Hadamard rotation in fp32
    (log2 d butterfly stages, then the 1/sqrt(d) product): the row's bounds
    spread by |H|, plus one rounding per stage of partial sums bounded by
    sum|S|."""
    import oracle
    S = oracle.compress(np.abs(x), np.abs(W), m, overlap)
    d = S.shape[-1]
    stages = int(np.log2(d))
    row = (bound.sum(axis=-1) + (stages + 2) * U32 * S.sum(axis=-1)) / np.sqrt(d)
    return np.broadcast_to(row[..., None], S.shape)
