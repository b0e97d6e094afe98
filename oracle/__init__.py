"""Plain fp64 CPU oracle for the CSA / HCA hot path -- TEST INFRASTRUCTURE.

Only the tests, the smoke check in ``__graft_entry__`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The product path (the CUDA
library and its Python binding) never imports, links or executes anything
here, and this package imports nothing from the product.

The arithmetic lives in ``csa_oracle.c`` (plain C, fp64, OpenMP over query
rows); this module only compiles it with gcc and marshals numpy arrays.
Every function states which passage of the pages it follows:

* [P1] "DeepSeek V4 CSA + CP 迁移到 HP：困难点深度分析" (gitcode issue)
* [P3] "DS-V4 分析&学习"
* [P5] "百万上下文从「奢侈品」变「日用品」：DeepSeek V4 CSA/HCA 混合注意力架构深度解析"

Parity of the indexer's head combination (sum over heads of ReLU(q_h . k))
against the method as DeepSeek runs it is unpinned: the pages print no
formula for it; the oracle pins it only to its own stated reading.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``csa_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_long
        lib.oracle_num_threads.restype = i32
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_quantize_rows_e4m3.argtypes = [P, i64, i32, P, P]
        lib.oracle_hadamard_rows_f32.argtypes = [P, i64, i32]
        lib.oracle_num_entries.argtypes = [i64, i64]
        lib.oracle_num_entries.restype = i64
        lib.oracle_visible_entries.argtypes = [i64, i32, i64]
        lib.oracle_visible_entries.restype = i64
        lib.oracle_compress.argtypes = [P, i32, i32, i32, P, i32, i32, i32, P]
        lib.oracle_compress_gated.argtypes = [P, i32, i32, i32, P, P, P, i32, i32, i32, P]
        lib.oracle_compress_append.argtypes = [P, P, i32, i32, P, i32, i32, i32, P, P, i32, P]
        dbl = ctypes.c_double
        lib.oracle_indexer_scores.argtypes = [P, P, P, P, i64, i32, i32, P, P, P, i32, P, i32, P]
        lib.oracle_indexer_topk.argtypes = [P, P, P, P, i64, i32, i32, P, P, P, i32, P, i32, i32, P,
                                            P, P]
        lib.oracle_sparse_attn.argtypes = [P, P, P, i64, i32, i32, P, i32, P, i32, P, i32, P, P,
                                           i32, dbl, P, P]
        lib.oracle_hca_attn.argtypes = [P, P, P, i64, i32, i32, P, i32, P, i32, P, i32, P, P, i32,
                                        dbl, P, P]
        _lib = lib
        return lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    """OpenMP threads the oracle uses (``OMP_NUM_THREADS`` or all host cores)."""
    return int(_load().oracle_num_threads())


# --------------------------------------------------------------------------
# FP8 E4M3 (OCP 8-bit floating point specification, E4M3 encoding)
# --------------------------------------------------------------------------
def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code (uint8), as fp64 (NaN for the NaN codes)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_decode(int(v)) for v in c.ravel()]).reshape(c.shape)


def e4m3_encode(x) -> np.ndarray:
    """Round fp32 values to E4M3 codes: nearest, ties to even, saturate at 448."""
    lib = _load()
    a = np.asarray(x, dtype=np.float32)
    return np.array([lib.oracle_e4m3_encode(float(v)) for v in a.ravel()],
                    dtype=np.uint8).reshape(a.shape)


def quantize_rows_e4m3(x) -> tuple[np.ndarray, np.ndarray]:
    """Per-row E4M3 quantisation in fp32: scale = amax/448 (1 for a zero row),
    code = E4M3(x / scale).  Returns (codes uint8 [..., d], scales fp32 [...])."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    d = a.shape[-1]
    rows = a.size // d if d else 0
    codes = np.empty(a.shape, dtype=np.uint8)
    scales = np.empty(a.shape[:-1], dtype=np.float32)
    _load().oracle_quantize_rows_e4m3(_ptr(a), rows, d, _ptr(codes), _ptr(scales))
    return codes, scales


def hadamard_rows_f32(x) -> np.ndarray:
    """Rows rotated by the normalised Walsh-Hadamard matrix, in fp32, in the
    fixed butterfly order the kernels use (see csa_oracle.c)."""
    a = np.array(x, dtype=np.float32, copy=True, order="C")
    d = a.shape[-1]
    assert d > 0 and d & (d - 1) == 0, "d must be a power of two"
    _load().oracle_hadamard_rows_f32(_ptr(a), a.size // d, d)
    return a


def dequantize_rows_e4m3(codes, scales) -> np.ndarray:
    """codes * scale per row, exactly, in fp64."""
    table = e4m3_decode(np.arange(256, dtype=np.uint8))
    return table[np.asarray(codes, dtype=np.uint8)] * np.asarray(scales, np.float64)[..., None]


# --------------------------------------------------------------------------
# Stage 1: compression ([P5] §3.2; [P3] §1.3; [P1] §3.2)
# --------------------------------------------------------------------------
def num_entries(n: int, m: int) -> int:
    """floor(n/m): a trailing partial block yields no entry ([P5] §3.2)."""
    return int(_load().oracle_num_entries(n, m))


def visible_entries(t: int, m: int, n_entries: int) -> int:
    """Entries visible to the query at position t: min(floor((t+1)/m), n_entries)."""
    return int(_load().oracle_visible_entries(t, m, n_entries))


def compress(x, W, m: int, overlap: bool) -> np.ndarray:
    """out[b,i] = mean(x[b, win(i)]) @ W for i < floor(n/m) (fp64).
    x: [B, n, d_in]; W: [d_in, d_out]."""
    x = _f64(x)
    W = _f64(W)
    B, n, d_in = x.shape
    d_out = W.shape[1]
    assert W.shape[0] == d_in
    N_c = num_entries(n, m)
    out = np.zeros((B, N_c, d_out), dtype=np.float64)
    if N_c:
        _load().oracle_compress(_ptr(x), B, n, d_in, _ptr(W), d_out, m, int(bool(overlap)),
                                _ptr(out))
    return out


def compress_gated(x, W_kv, W_gate, ape, m: int, overlap: bool) -> np.ndarray:
    """The gated-softmax compressor (reading in csa_oracle.c): per channel, a
    softmax over the window's positions of (x @ W_gate + ape[p mod m]) weights
    x @ W_kv; overlapping windows take the first half of the projected
    channels from the previous block and the second half from the current one.
    x [B, n, d_in]; W_kv, W_gate [d_in, c*d_out]; ape [m, c*d_out], c = 2 if
    overlap else 1.  Returns [B, floor(n/m), d_out] (fp64)."""
    x, W_kv, W_gate, ape = _f64(x), _f64(W_kv), _f64(W_gate), _f64(ape)
    B, n, d_in = x.shape
    c = 2 if overlap else 1
    assert W_kv.shape == W_gate.shape and W_kv.shape[0] == d_in and W_kv.shape[1] % c == 0
    d_out = W_kv.shape[1] // c
    assert ape.shape == (m, c * d_out)
    N_c = num_entries(n, m)
    out = np.zeros((B, N_c, d_out), dtype=np.float64)
    if N_c:
        _load().oracle_compress_gated(_ptr(x), B, n, d_in, _ptr(W_kv), _ptr(W_gate), _ptr(ape),
                                      d_out, m, int(bool(overlap)), _ptr(out))
    return out


def compress_append(state, x_new, W, m: int, overlap: bool, pos, out, N_cap: int) -> np.ndarray:
    """One decode step of the compressor state ("DS-V4 分析&学习" opening summary
    and §1.3): adds each element's new token to its running block sum and, when
    the token completes block j = pos // m, writes entry j (mean over its window,
    then @ W) into ``out[b, j]``.  ``state`` [B, 2, d_in] fp64 and ``out``
    [B, N_cap, d_out] fp64 are updated in place; returns done [B] (the entry
    written, or -1)."""
    x_new = _f64(x_new)
    W = _f64(W)
    B, d_in = x_new.shape
    d_out = W.shape[1]
    assert state.dtype == np.float64 and state.flags.c_contiguous and state.shape == (B, 2, d_in)
    assert out.dtype == np.float64 and out.flags.c_contiguous and out.shape == (B, N_cap, d_out)
    pos = _i32(pos)
    done = np.empty(B, np.int32)
    _load().oracle_compress_append(_ptr(state), _ptr(x_new), B, d_in, _ptr(W), d_out, m,
                                   int(bool(overlap)), _ptr(pos), _ptr(out), N_cap, _ptr(done))
    return done


def compress_stream(x, W, m: int, overlap: bool) -> np.ndarray:
    """Feeds x [B, n, d_in] to ``compress_append`` one position at a time and
    returns the entries it wrote, [B, floor(n/m), d_out]."""
    x = _f64(x)
    B, n, d_in = x.shape
    N_c = num_entries(n, m)
    state = np.zeros((B, 2, d_in), np.float64)
    out = np.zeros((B, N_c, _f64(W).shape[1]), np.float64)
    for p in range(n):
        compress_append(state, x[:, p], W, m, overlap, np.full(B, p, np.int32), out, N_c)
    return out


# --------------------------------------------------------------------------
# Stage 2: indexer scores and top-k ([P5] §3.2; [P3] §1.2, §4)
# --------------------------------------------------------------------------
def _rows_arg(rows, total):
    if rows is None:
        return np.arange(total, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def _defaults(B, n_q, N_cap, n_entries, q_pos):
    if n_entries is None:
        n_entries = np.full(B, N_cap, dtype=np.int32)
    if q_pos is None:
        q_pos = np.broadcast_to(np.arange(n_q, dtype=np.int32), (B, n_q))
    return _i32(n_entries), _i32(q_pos)


def _keys_arg(kI, kI_scale):
    """(fp64 values, codes, scales) pointers for fp64 keys or E4M3 codes + scales."""
    if kI_scale is None:
        k = _f64(kI)
        return k, None, None, (_ptr(k), None, None)
    c = np.ascontiguousarray(np.asarray(kI, dtype=np.uint8))
    sc = np.ascontiguousarray(np.asarray(kI_scale, dtype=np.float32))
    return None, c, sc, (None, _ptr(c), _ptr(sc))


def quantized_query_rows(qI_rows, rotate: bool = False) -> np.ndarray:
    """fp64 values of query rows after the per-(row, head) E4M3 quantisation
    the indexer applies to bf16 queries against fp8 keys (fp32 procedure);
    with ``rotate`` the rows are Hadamard-rotated (fp32) first, as against
    rotated keys."""
    q = np.asarray(qI_rows, dtype=np.float32)
    if rotate:
        q = hadamard_rows_f32(q)
    codes, scales = quantize_rows_e4m3(q)
    return dequantize_rows_e4m3(codes, scales)


def _weights_arg(weights, R, H_I):
    if weights is None:
        return None, None
    w = np.ascontiguousarray(np.asarray(weights, dtype=np.float64).reshape(R, H_I))
    return w, _ptr(w)


def indexer_scores_rows(qI_rows, row_b, row_t, kI, m: int, n_entries, kI_scale=None,
                        weights=None):
    """Scores sum_h w_h ReLU(qI_h . kI[s]) of listed query rows against every
    entry.  qI_rows [R, H_I, d_I] fp64 (dequantised); weights [R, H_I] per-head
    gate weights (None: all 1); row_b/row_t [R] batch element and absolute
    position; kI [B, N_cap, d_I] fp64 values, or E4M3 codes with kI_scale
    [B, N_cap]; n_entries [B].  Returns [R, N_cap], NaN where the entry is not
    visible."""
    q = _f64(qI_rows)
    R, H_I, d_I = q.shape
    w, wp = _weights_arg(weights, R, H_I)
    keep = _keys_arg(kI, kI_scale)
    N_cap = np.asarray(kI).shape[1]
    rb, rt, ne = _i32(row_b), _i32(row_t), _i32(n_entries)
    out = np.empty((R, N_cap), dtype=np.float64)
    _load().oracle_indexer_scores(_ptr(q), wp, _ptr(rb), _ptr(rt), R, H_I, d_I, *keep[3], N_cap,
                                  _ptr(ne), m, _ptr(out))
    return out


def indexer_topk_rows(qI_rows, row_b, row_t, kI, m: int, topk: int, n_entries, kI_scale=None,
                      weights=None):
    """Per listed query row: the topk largest visible scores (ties -> lower
    index, -1 padding).  Returns (idx [R, topk] int32 in (score desc, index
    asc) order, kth [R, 2] = k-th and (k+1)-th largest scores (NaN if
    absent), smax [R] = largest |score|)."""
    q = _f64(qI_rows)
    R, H_I, d_I = q.shape
    w, wp = _weights_arg(weights, R, H_I)
    keep = _keys_arg(kI, kI_scale)
    N_cap = np.asarray(kI).shape[1]
    rb, rt, ne = _i32(row_b), _i32(row_t), _i32(n_entries)
    idx = np.empty((R, topk), dtype=np.int32)
    kth = np.empty((R, 2), dtype=np.float64)
    smax = np.empty(R, dtype=np.float64)
    _load().oracle_indexer_topk(_ptr(q), wp, _ptr(rb), _ptr(rt), R, H_I, d_I, *keep[3], N_cap,
                                _ptr(ne), m, topk, _ptr(idx), _ptr(kth), _ptr(smax))
    return idx, kth, smax


def _full_rows(B, n_q, q_pos, rows):
    r = _rows_arg(rows, B * n_q)
    qp = np.asarray(q_pos).reshape(-1)
    return r, (r // n_q).astype(np.int32), qp[r].astype(np.int32)


def indexer_scores(qI, kI, m: int, n_entries=None, q_pos=None, rows=None, kI_scale=None,
                   weights=None):
    """indexer_scores_rows over full tensors qI [B, n_q, H_I, d_I] (weights
    [B, n_q, H_I] or None); rows are flattened b*n_q+q (all by default)."""
    qI = _f64(qI)
    B, n_q, H_I, d_I = qI.shape
    N_cap = np.asarray(kI).shape[1]
    n_entries, q_pos = _defaults(B, n_q, N_cap, n_entries, q_pos)
    r, rb, rt = _full_rows(B, n_q, q_pos, rows)
    w = None if weights is None else _f64(weights).reshape(B * n_q, H_I)[r]
    return indexer_scores_rows(qI.reshape(B * n_q, H_I, d_I)[r], rb, rt, kI, m, n_entries,
                               kI_scale, w)


def indexer_topk(qI, kI, m: int, topk: int, n_entries=None, q_pos=None, rows=None, kI_scale=None,
                 weights=None):
    """indexer_topk_rows over full tensors (see indexer_scores)."""
    qI = _f64(qI)
    B, n_q, H_I, d_I = qI.shape
    N_cap = np.asarray(kI).shape[1]
    n_entries, q_pos = _defaults(B, n_q, N_cap, n_entries, q_pos)
    r, rb, rt = _full_rows(B, n_q, q_pos, rows)
    w = None if weights is None else _f64(weights).reshape(B * n_q, H_I)[r]
    return indexer_topk_rows(qI.reshape(B * n_q, H_I, d_I)[r], rb, rt, kI, m, topk, n_entries,
                             kI_scale, w)


# --------------------------------------------------------------------------
# Stage 3: joint-softmax attention ([P3] §1.2, §1.4, §1.5; [P5] §4.3, §5.2)
# --------------------------------------------------------------------------
def _raw_defaults(B, L_raw, raw_pos0, raw_len):
    if raw_pos0 is None:
        raw_pos0 = np.zeros(B, dtype=np.int32)
    if raw_len is None:
        raw_len = np.full(B, L_raw, dtype=np.int32)
    return _i32(raw_pos0), _i32(raw_len)


def sparse_attn_rows(q_rows, row_b, row_t, kv_c, idx_rows, kv_raw, window: int, raw_pos0=None,
                     raw_len=None, scale: float | None = None):
    """Joint softmax over {kv_c[b, idx] : 0 <= idx < N_cap} ∪ window raw rows
    for listed query rows.  q_rows [R, H, D]; row_b/row_t [R]; kv_c
    [B, N_cap, D]; idx_rows [R, topk]; kv_raw [B, L_raw, D].
    Returns (o [R, H, D], lse [R, H])."""
    q = _f64(q_rows)
    R, H, D = q.shape
    kv_c = _f64(kv_c)
    kv_raw = _f64(kv_raw)
    idx = _i32(idx_rows).reshape(R, -1) if R else _i32(np.zeros((0, 0)))
    topk = idx.shape[1] if R else 0
    B, N_cap = kv_c.shape[0], kv_c.shape[1]
    L_raw = kv_raw.shape[1]
    raw_pos0, raw_len = _raw_defaults(B, L_raw, raw_pos0, raw_len)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    rb, rt = _i32(row_b), _i32(row_t)
    out = np.empty((R, H, D), dtype=np.float64)
    lse = np.empty((R, H), dtype=np.float64)
    _load().oracle_sparse_attn(_ptr(q), _ptr(rb), _ptr(rt), R, H, D, _ptr(kv_c), N_cap,
                               _ptr(idx), topk, _ptr(kv_raw), L_raw, _ptr(raw_pos0),
                               _ptr(raw_len), window, float(scale), _ptr(out), _ptr(lse))
    return out, lse


def hca_attn_rows(q_rows, row_b, row_t, kv_c, m: int, kv_raw, window: int, n_entries=None,
                  raw_pos0=None, raw_len=None, scale: float | None = None):
    """Dense attention over every visible entry s < min(floor((t+1)/m),
    n_entries) plus the window, one softmax, for listed query rows."""
    q = _f64(q_rows)
    R, H, D = q.shape
    kv_c = _f64(kv_c)
    kv_raw = _f64(kv_raw)
    B, N_cap = kv_c.shape[0], kv_c.shape[1]
    L_raw = kv_raw.shape[1]
    if n_entries is None:
        n_entries = np.full(B, N_cap, dtype=np.int32)
    ne = _i32(n_entries)
    raw_pos0, raw_len = _raw_defaults(B, L_raw, raw_pos0, raw_len)
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    rb, rt = _i32(row_b), _i32(row_t)
    out = np.empty((R, H, D), dtype=np.float64)
    lse = np.empty((R, H), dtype=np.float64)
    _load().oracle_hca_attn(_ptr(q), _ptr(rb), _ptr(rt), R, H, D, _ptr(kv_c), N_cap, _ptr(ne), m,
                            _ptr(kv_raw), L_raw, _ptr(raw_pos0), _ptr(raw_len), window,
                            float(scale), _ptr(out), _ptr(lse))
    return out, lse


def sparse_attn(q, kv_c, idx, kv_raw, window: int, q_pos=None, raw_pos0=None, raw_len=None,
                scale: float | None = None, rows=None):
    """sparse_attn_rows over full tensors q [B, n_q, H, D], idx [B, n_q, topk]."""
    q = _f64(q)
    B, n_q, H, D = q.shape
    _, q_pos = _defaults(B, n_q, 0, None, q_pos)
    r, rb, rt = _full_rows(B, n_q, q_pos, rows)
    idx = _i32(idx).reshape(B * n_q, -1)
    return sparse_attn_rows(q.reshape(B * n_q, H, D)[r], rb, rt, kv_c, idx[r], kv_raw, window,
                            raw_pos0, raw_len, scale)


def hca_attn(q, kv_c, m: int, kv_raw, window: int, n_entries=None, q_pos=None, raw_pos0=None,
             raw_len=None, scale: float | None = None, rows=None):
    """hca_attn_rows over full tensors q [B, n_q, H, D]."""
    q = _f64(q)
    B, n_q, H, D = q.shape
    _, q_pos = _defaults(B, n_q, 0, None, q_pos)
    r, rb, rt = _full_rows(B, n_q, q_pos, rows)
    return hca_attn_rows(q.reshape(B * n_q, H, D)[r], rb, rt, kv_c, m, kv_raw, window, n_entries,
                         raw_pos0, raw_len, scale)


# --------------------------------------------------------------------------
# End to end: stage 1 -> 2 -> 3 (a composition of the functions above)
# --------------------------------------------------------------------------
def csa_forward(q, kv, qI, kI_raw, W_c, W_Ic, m: int, topk: int, window: int, rows=None):
    """Whole CSA prefill for a batch of sequences (positions 0..n-1): compress
    kv and the indexer keys with overlap, score + top-k, attend.
    Returns (o [R, H, D], lse [R, H], idx [R, topk]) for the listed rows."""
    kv_c = compress(kv, W_c, m, True)
    kI_c = compress(kI_raw, W_Ic, m, True)
    idx, _, _ = indexer_topk(qI, kI_c, m, topk, rows=rows)
    B, n_q = np.asarray(q).shape[:2]
    q = _f64(q)
    r, rb, rt = _full_rows(B, n_q, np.broadcast_to(np.arange(n_q), (B, n_q)), rows)
    o, lse = sparse_attn_rows(q.reshape(B * n_q, *q.shape[2:])[r], rb, rt, kv_c, idx, kv, window)
    return o, lse, idx
