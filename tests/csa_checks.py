"""Shared comparison helpers for the parity tests (no method arithmetic here).

Tolerances (stated once, used by every parity test):
  * attention / compression outputs, max-abs against the fp64 oracle:
    2e-2 for bf16 paths, 1e-4 for fp32 paths; a bf16-stored output may in
    addition carry its own storage rounding, at most 2^-8 |ref| (half an
    ulp, rounded up): above |ref| ~ 8 no bf16 value lies within 2e-2 of the
    exact result, so the 2e-2 budget is applied on top of that rounding;
  * bf16-stored compression outputs additionally within one bf16 ulp:
    |gpu - ref| <= 2^-8 |ref| + 1e-5;
  * top-k index sets: identical except where the oracle's k-th and (k+1)-th
    scores lie within delta = 1e-3 * max(|s_k|, |s_k+1|) + 1e-6 * max_s |s|
    of each other (a near-tie); inside a near-tie every index scoring above
    s_k + delta must be chosen and every chosen index must score at least
    s_k+1 - delta.
Near-ties are common by construction at large V (thousands of visible
entries put consecutive order statistics ~1e-4 apart relative, and ReLU
makes exact ties at 0), so their count is reported, not bounded.
"""
from __future__ import annotations

import numpy as np
import torch

ATOL_BF16 = 2e-2
ATOL_F32 = 1e-4
TOPK_REL = 1e-3
TOPK_ABS_FRAC = 1e-6


def np64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a float tensor (any device)."""
    return t.detach().to("cpu", torch.float64).numpy()


def atol_for(dtype: torch.dtype) -> float:
    return ATOL_F32 if dtype == torch.float32 else ATOL_BF16


def check_topk(gpu_idx: np.ndarray, scores: np.ndarray, k: int) -> dict:
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
    return dict(rows=R, exact=exact, near_ties=near)


def excess_bf16(got: np.ndarray, ref: np.ndarray) -> float:
    """max over elements of |got - ref| - 2^-8 |ref| (storage rounding of a
    bf16 output removed); compare with ATOL_BF16."""
    if got.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref) - np.abs(ref) * 2.0 ** -8))


def check_out(got: np.ndarray, ref: np.ndarray, dtype) -> None:
    """Output tolerance for a kernel result stored in `dtype`."""
    if dtype == torch.float32:
        err = max_abs(got, ref)
        assert err <= ATOL_F32, f"max abs error {err} > {ATOL_F32}"
    else:
        err = excess_bf16(got, ref)
        assert err <= ATOL_BF16, f"error beyond bf16 storage rounding {err} > {ATOL_BF16}"


def max_abs(a: np.ndarray, b: np.ndarray) -> float:
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))
