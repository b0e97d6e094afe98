"""Thin Python binding of libcsa_b200.so (see include/csa_b200.h).

Argument marshalling only: each function of the C ABI has a Python function
of the same name that takes torch CUDA tensors, derives sizes and dtype
codes from them, passes raw device pointers and the current CUDA stream, and
raises ``CsaError`` on a non-OK status.  Every step of the computation runs
in the library's kernels; there is no fallback of any kind -- if the library
is missing or fails to load, the first call raises.

Convenience wrappers (``compress``, ``indexer_topk``, ``sparse_attn``,
``hca_attn``, ``csa_prefill``) allocate their outputs with ``torch.empty``
and call the ABI functions.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa_b200.so")

CSA_OK, CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_MISALIGNED, CSA_ERR_CUDA, \
    CSA_ERR_TIMEOUT = range(6)
DT_F32, DT_BF16, DT_E4M3, DT_E4M3_HADAMARD = 0, 1, 2, 3

# symbol -> (restype, argtypes); mirrors include/csa_b200.h
P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "csa_status_string": (ctypes.c_char_p, [I]),
    "csa_last_error_detail": (ctypes.c_char_p, []),
    "csa_version": (I, []),
    "csa_kernel_launches": (ctypes.c_ulonglong, []),
    "csa_check_device_error": (I, [P, I]),
    "csa_debug_inject_launch_error": (I, [I]),
    "csa_debug_set_wait_limit": (I, [ctypes.c_longlong, I]),
    "csa_compress": (I, [P, I, I, I, I, P, I, I, I, P, I, P, P]),
    "csa_compress_gated": (I, [P, I, I, I, I, P, P, P, I, I, I, P, I, P, P]),
    "csa_compress_append": (I, [P, I, I, I, P, I, I, I, P, P, P, I, P, I, P, P]),
    "csa_indexer_topk": (I, [P, I, P, P, P, I, P, I, I, I, I, I, P, P, I, I, P, P]),
    "csa_sparse_attn": (I, [P, I, I, I, I, I, P, I, P, I, P, I, P, P, I, P, F, P, P, P]),
    "hca_dense_attn": (I, [P, I, I, I, I, I, P, I, P, I, P, I, P, P, I, P, F, P, P, P]),
    "csa_varlen_entry_offsets": (I, [P, I, I, P]),
    "csa_compress_varlen": (I, [P, I, I, P, I, P, I, I, I, P, I, P, P]),
    "csa_indexer_topk_varlen": (I, [P, I, P, P, P, I, P, I, P, I, I, I, I, P, P]),
    "csa_sparse_attn_varlen": (I, [P, I, I, P, I, I, P, I, P, I, P, I, F, P, P, P]),
    "hca_dense_attn_varlen": (I, [P, I, I, P, I, I, P, I, P, I, F, P, P, P]),
    "csa_compress_append_paged": (I, [P, I, I, I, P, I, I, I, P, P, P, I, P, P, I, I, I, P, P]),
    "csa_indexer_topk_paged": (I, [P, I, P, P, P, I, P, P, I, I, I, I, I, I, I, P, P, I, I, P, P]),
    "csa_sparse_attn_paged": (I, [P, I, I, I, I, I, P, P, I, I, I, P, I, P, I, P, P, I, P, F, P, P,
                                  P]),
    "hca_dense_attn_paged": (I, [P, I, I, I, I, I, P, P, I, I, I, P, I, P, I, P, P, I, P, F, P, P,
                                 P]),
    "csa_indexer_topk_at": (I, [P, I, P, P, P, I, P, I, I, I, I, I, P, I, I, I, P, P]),
    "csa_sparse_attn_at": (I, [P, I, I, I, I, I, P, I, P, I, P, I, I, I, I, F, P, P, P]),
    "hca_dense_attn_at": (I, [P, I, I, I, I, I, P, I, P, I, P, I, I, I, I, F, P, P, P]),
}


class CsaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{_status_name(status)}: {detail}")
        self.status = status
        self.detail = detail


_lock = threading.Lock()
_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library (once).  Raises if it is missing: there is no fallback."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"libcsa_b200.so not found at {p}; build it with "
                               "`python -m long_context_compressed_03_b200.build`")
        lib = ctypes.CDLL(p)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def _status_name(status: int) -> str:
    try:
        return load().csa_status_string(status).decode()
    except Exception:  # pragma: no cover - only when the library cannot load
        return f"status {status}"


def _check(status: int) -> None:
    if status != CSA_OK:
        raise CsaError(status, load().csa_last_error_detail().decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DT_F32
    if t.dtype == torch.bfloat16:
        return DT_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DT_E4M3
    raise ValueError(f"unsupported dtype {t.dtype}")


def _dt_rot(t: torch.Tensor, rotated: bool) -> int:
    """dtype code of an fp8 tensor whose rows are (or are to be) Hadamard-rotated."""
    d = _dt(t)
    if rotated:
        if d != DT_E4M3:
            raise ValueError("Hadamard rotation applies to fp8 (uint8 / float8_e4m3fn) rows only")
        return DT_E4M3_HADAMARD
    return d


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _i32(t: torch.Tensor | None, name: str):
    if t is not None and t.dtype != torch.int32:
        raise ValueError(f"{name} must be int32")
    return _ptr(t)


# ---------------------------------------------------------------- the ABI, by name
def csa_version() -> int:
    return int(load().csa_version())


def csa_kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(load().csa_kernel_launches())


def csa_check_device_error(clear: bool = True, stream=None) -> None:
    """Synchronise the stream and raise CsaError(CSA_ERR_TIMEOUT) if a kernel's
    bounded on-chip wait expired since the last check."""
    _check(load().csa_check_device_error(_stream(stream), int(bool(clear))))


def csa_compress(x: torch.Tensor, W: torch.Tensor, m: int, overlap: bool, out: torch.Tensor,
                 out_row_scale: torch.Tensor | None = None, hadamard: bool = False,
                 stream=None) -> None:
    """x [B, n, d_in], W [d_in, d_out] -> out [B, n//m, d_out] (+ scales for fp8;
    ``hadamard``: fp8 rows rotated by the normalised Walsh-Hadamard matrix first)."""
    B, n, d_in = x.shape
    d_out = W.shape[1]
    _check(load().csa_compress(_ptr(x), _dt(x), B, n, d_in, _ptr(W), d_out, m, int(bool(overlap)),
                               _ptr(out), _dt_rot(out, hadamard), _ptr(out_row_scale),
                               _stream(stream)))


def csa_compress_gated(x: torch.Tensor, W_kv: torch.Tensor, W_gate: torch.Tensor,
                       ape: torch.Tensor, m: int, overlap: bool, out: torch.Tensor,
                       out_row_scale: torch.Tensor | None = None, hadamard: bool = False,
                       stream=None) -> None:
    """x [B, n, d_in]; W_kv, W_gate [d_in, c*d_out]; ape [m, c*d_out] fp32
    (c = 2 if overlap else 1) -> out [B, n//m, d_out] (+ scales for fp8)."""
    B, n, d_in = x.shape
    c = 2 if overlap else 1
    d_out = W_kv.shape[1] // c
    if ape.dtype != torch.float32:
        raise ValueError("ape must be float32")
    if tuple(W_gate.shape) != tuple(W_kv.shape) or tuple(ape.shape) != (m, c * d_out):
        raise ValueError("W_kv, W_gate must be [d_in, c*d_out] and ape [m, c*d_out]")
    _check(load().csa_compress_gated(_ptr(x), _dt(x), B, n, d_in, _ptr(W_kv), _ptr(W_gate),
                                     _ptr(ape), d_out, m, int(bool(overlap)), _ptr(out),
                                     _dt_rot(out, hadamard), _ptr(out_row_scale),
                                     _stream(stream)))


def csa_compress_append(x_new: torch.Tensor, W: torch.Tensor, m: int, overlap: bool,
                        pos: torch.Tensor, state: torch.Tensor, cache: torch.Tensor,
                        cache_scale: torch.Tensor | None = None,
                        n_entries: torch.Tensor | None = None, hadamard: bool = False,
                        stream=None) -> None:
    """x_new [B, d_in], pos [B] int32, state [B, 2, d_in] fp32 (zero before the first
    token), cache [B, N_cap, d_out] (+ cache_scale [B, N_cap] for fp8; ``hadamard`` as
    in csa_compress)."""
    B, d_in = x_new.shape
    d_out = W.shape[1]
    if state.dtype != torch.float32:
        raise ValueError("state must be float32")
    _check(load().csa_compress_append(_ptr(x_new), _dt(x_new), B, d_in, _ptr(W), d_out, m,
                                      int(bool(overlap)), _i32(pos, "pos"), _ptr(state),
                                      _ptr(cache), _dt_rot(cache, hadamard), _ptr(cache_scale),
                                      cache.shape[1],
                                      _i32(n_entries, "n_entries"), _stream(stream)))


def csa_indexer_topk(qI: torch.Tensor, kI: torch.Tensor, m: int, topk: int, idx_out: torch.Tensor,
                     qI_scale: torch.Tensor | None = None, kI_scale: torch.Tensor | None = None,
                     n_entries: torch.Tensor | None = None, q_pos: torch.Tensor | None = None,
                     kI_rotated: bool = False, qI_weight: torch.Tensor | None = None,
                     stream=None) -> None:
    """qI [B, n_q, H_I, d_I], kI [B, N_cap, d_I] -> idx_out [B, n_q, topk] int32.
    ``kI_rotated``: fp8 keys written with the Hadamard rotation (bf16 queries are
    rotated in the kernel; fp8 query codes are taken as already rotated).
    ``qI_weight`` [B, n_q, H_I] fp32: per-head gate weights, any sign
    (score = sum_h w_h ReLU(q_h . k))."""
    B, n_q, H_I, d_I = qI.shape
    N_cap = kI.shape[1]
    if qI_weight is not None and (qI_weight.dtype != torch.float32 or
                                  tuple(qI_weight.shape) != (B, n_q, H_I)):
        raise ValueError("qI_weight must be float32 [B, n_q, H_I]")
    _check(load().csa_indexer_topk(_ptr(qI), _dt(qI), _ptr(qI_scale), _ptr(qI_weight), _ptr(kI),
                                   _dt_rot(kI, kI_rotated),
                                   _ptr(kI_scale), B, n_q, H_I, d_I, N_cap,
                                   _i32(n_entries, "n_entries"), _i32(q_pos, "q_pos"), m, topk,
                                   _i32(idx_out, "idx_out"), _stream(stream)))


def csa_sparse_attn(q: torch.Tensor, kv_c: torch.Tensor, idx: torch.Tensor | None,
                    kv_raw: torch.Tensor, window: int, out: torch.Tensor,
                    lse_out: torch.Tensor | None = None, raw_pos0: torch.Tensor | None = None,
                    raw_len: torch.Tensor | None = None, q_pos: torch.Tensor | None = None,
                    softmax_scale: float = 0.0, stream=None) -> None:
    """q [B, n_q, H, D], kv_c [B, N_cap, D], idx [B, n_q, topk], kv_raw [B, L_raw, D]."""
    B, n_q, H, D = q.shape
    topk = 0 if idx is None else idx.shape[-1]
    _check(load().csa_sparse_attn(_ptr(q), _dt(q), B, n_q, H, D, _ptr(kv_c), kv_c.shape[1],
                                  _i32(idx, "idx"), topk, _ptr(kv_raw), kv_raw.shape[1],
                                  _i32(raw_pos0, "raw_pos0"), _i32(raw_len, "raw_len"), window,
                                  _i32(q_pos, "q_pos"), float(softmax_scale), _ptr(out),
                                  _ptr(lse_out), _stream(stream)))


def hca_dense_attn(q: torch.Tensor, kv_c: torch.Tensor, m: int, kv_raw: torch.Tensor, window: int,
                   out: torch.Tensor, lse_out: torch.Tensor | None = None,
                   n_entries: torch.Tensor | None = None, raw_pos0: torch.Tensor | None = None,
                   raw_len: torch.Tensor | None = None, q_pos: torch.Tensor | None = None,
                   softmax_scale: float = 0.0, stream=None) -> None:
    """Dense attention over every visible entry of kv_c plus the window."""
    B, n_q, H, D = q.shape
    _check(load().hca_dense_attn(_ptr(q), _dt(q), B, n_q, H, D, _ptr(kv_c), kv_c.shape[1],
                                 _i32(n_entries, "n_entries"), m, _ptr(kv_raw), kv_raw.shape[1],
                                 _i32(raw_pos0, "raw_pos0"), _i32(raw_len, "raw_len"), window,
                                 _i32(q_pos, "q_pos"), float(softmax_scale), _ptr(out),
                                 _ptr(lse_out), _stream(stream)))


# ---------------------------------------------------------------- packed (varlen) prefill
def _host_cu(cu_seqlens) -> tuple:
    """cu_seqlens as a host int32 array (kept alive by the caller's frame) + S."""
    cu = np.ascontiguousarray(np.asarray(cu_seqlens.cpu() if isinstance(cu_seqlens, torch.Tensor)
                                         else cu_seqlens, dtype=np.int32))
    return cu, cu.size - 1, cu.ctypes.data_as(ctypes.c_void_p)


def varlen_entry_offsets(cu_seqlens, m: int) -> np.ndarray:
    """e(0..S): where each sequence's compressed entries start in the packed cache."""
    cu, S, p = _host_cu(cu_seqlens)
    out = np.zeros(S + 1, np.int32)
    if load().csa_varlen_entry_offsets(p, S, m, out.ctypes.data_as(ctypes.c_void_p)) < 0:
        raise ValueError("invalid cu_seqlens or m")
    return out


def csa_compress_varlen(x: torch.Tensor, cu_seqlens, W: torch.Tensor, m: int, overlap: bool,
                        out: torch.Tensor, out_row_scale: torch.Tensor | None = None,
                        hadamard: bool = False, stream=None) -> None:
    """x [T, d_in] packed -> out [E, d_out] packed (E = varlen_entry_offsets(...)[-1])."""
    cu, S, cup = _host_cu(cu_seqlens)
    _check(load().csa_compress_varlen(_ptr(x), _dt(x), S, cup, x.shape[-1], _ptr(W), W.shape[1], m,
                                      int(bool(overlap)), _ptr(out), _dt_rot(out, hadamard),
                                      _ptr(out_row_scale), _stream(stream)))


def csa_indexer_topk_varlen(qI: torch.Tensor, kI: torch.Tensor, cu_seqlens, m: int, topk: int,
                            idx_out: torch.Tensor, qI_scale=None, kI_scale=None,
                            kI_rotated: bool = False, qI_weight=None, stream=None) -> None:
    """qI [T, H_I, d_I], kI [E, d_I] packed -> idx_out [T, topk] (sequence-local entries)."""
    cu, S, cup = _host_cu(cu_seqlens)
    _, H_I, d_I = qI.shape
    _check(load().csa_indexer_topk_varlen(_ptr(qI), _dt(qI), _ptr(qI_scale), _ptr(qI_weight),
                                          _ptr(kI), _dt_rot(kI, kI_rotated), _ptr(kI_scale), S, cup,
                                          H_I, d_I, m, topk, _i32(idx_out, "idx_out"),
                                          _stream(stream)))


def csa_sparse_attn_varlen(q: torch.Tensor, cu_seqlens, kv_c: torch.Tensor, m: int,
                           idx: torch.Tensor | None, kv_raw: torch.Tensor, window: int,
                           out: torch.Tensor, lse_out: torch.Tensor | None = None,
                           softmax_scale: float = 0.0, stream=None) -> None:
    """q / out [T, H, D], kv_c [E, D], idx [T, topk], kv_raw [T, D] (packed)."""
    cu, S, cup = _host_cu(cu_seqlens)
    _, H, D = q.shape
    topk = 0 if idx is None else idx.shape[-1]
    _check(load().csa_sparse_attn_varlen(_ptr(q), _dt(q), S, cup, H, D, _ptr(kv_c), m,
                                         _i32(idx, "idx"), topk, _ptr(kv_raw), window,
                                         float(softmax_scale), _ptr(out), _ptr(lse_out),
                                         _stream(stream)))


def hca_dense_attn_varlen(q: torch.Tensor, cu_seqlens, kv_c: torch.Tensor, m: int,
                          kv_raw: torch.Tensor, window: int, out: torch.Tensor,
                          lse_out: torch.Tensor | None = None, softmax_scale: float = 0.0,
                          stream=None) -> None:
    cu, S, cup = _host_cu(cu_seqlens)
    _, H, D = q.shape
    _check(load().hca_dense_attn_varlen(_ptr(q), _dt(q), S, cup, H, D, _ptr(kv_c), m, _ptr(kv_raw),
                                        window, float(softmax_scale), _ptr(out), _ptr(lse_out),
                                        _stream(stream)))


# ---------------------------------------------------------------- spans at an offset
def csa_indexer_topk_at(qI: torch.Tensor, kI: torch.Tensor, m: int, topk: int,
                        idx_out: torch.Tensor, q_pos0: int, kI_scale: torch.Tensor | None = None,
                        n_entries: torch.Tensor | None = None, qI_scale: torch.Tensor | None = None,
                        kI_rotated: bool = False, qI_weight: torch.Tensor | None = None,
                        stream=None) -> None:
    """csa_indexer_topk with query q of every element at position q_pos0 + q."""
    B, n_q, H_I, d_I = qI.shape
    _check(load().csa_indexer_topk_at(_ptr(qI), _dt(qI), _ptr(qI_scale), _ptr(qI_weight),
                                      _ptr(kI), _dt_rot(kI, kI_rotated), _ptr(kI_scale), B, n_q,
                                      H_I, d_I, kI.shape[1], _i32(n_entries, "n_entries"),
                                      int(q_pos0), m, topk, _i32(idx_out, "idx_out"),
                                      _stream(stream)))


def csa_sparse_attn_at(q: torch.Tensor, kv_c: torch.Tensor, idx: torch.Tensor | None,
                       kv_raw: torch.Tensor, window: int, out: torch.Tensor, q_pos0: int,
                       raw_pos0: int, lse_out: torch.Tensor | None = None,
                       softmax_scale: float = 0.0, stream=None) -> None:
    """csa_sparse_attn with query q at position q_pos0 + q and raw row j at raw_pos0 + j."""
    B, n_q, H, D = q.shape
    topk = 0 if idx is None else idx.shape[-1]
    _check(load().csa_sparse_attn_at(_ptr(q), _dt(q), B, n_q, H, D, _ptr(kv_c), kv_c.shape[1],
                                     _i32(idx, "idx"), topk, _ptr(kv_raw), kv_raw.shape[1],
                                     int(raw_pos0), window, int(q_pos0), float(softmax_scale),
                                     _ptr(out), _ptr(lse_out), _stream(stream)))


def hca_dense_attn_at(q: torch.Tensor, kv_c: torch.Tensor, m: int, kv_raw: torch.Tensor,
                      window: int, out: torch.Tensor, q_pos0: int, raw_pos0: int,
                      lse_out: torch.Tensor | None = None, n_entries: torch.Tensor | None = None,
                      softmax_scale: float = 0.0, stream=None) -> None:
    """hca_dense_attn with query q at position q_pos0 + q and raw row j at raw_pos0 + j."""
    B, n_q, H, D = q.shape
    _check(load().hca_dense_attn_at(_ptr(q), _dt(q), B, n_q, H, D, _ptr(kv_c), kv_c.shape[1],
                                    _i32(n_entries, "n_entries"), m, _ptr(kv_raw),
                                    kv_raw.shape[1], int(raw_pos0), window, int(q_pos0),
                                    float(softmax_scale), _ptr(out), _ptr(lse_out),
                                    _stream(stream)))


# ---------------------------------------------------------------- paged caches
class PagedCache:
    """A page pool and its block table: ``pool`` [num_pages, page_size, row...]
    (and ``scale`` [num_pages, page_size] for fp8 rows), ``block_table``
    [B, max_pages] int32 (ids outside [0, num_pages) mark absent pages)."""

    def __init__(self, pool: torch.Tensor, block_table: torch.Tensor,
                 scale: torch.Tensor | None = None):
        if pool.dim() < 3:
            raise ValueError("pool must be [num_pages, page_size, row...]")
        self.pool, self.block_table, self.scale = pool, block_table, scale
        self.num_pages, self.page_size = pool.shape[0], pool.shape[1]
        self.max_pages = block_table.shape[1]

    @property
    def args(self):
        return (_i32(self.block_table, "block_table"), self.max_pages, self.page_size,
                self.num_pages)


def csa_compress_append_paged(x_new: torch.Tensor, W: torch.Tensor, m: int, overlap: bool,
                              pos: torch.Tensor, state: torch.Tensor, cache: PagedCache,
                              n_entries: torch.Tensor | None = None, hadamard: bool = False,
                              stream=None) -> None:
    """csa_compress_append into a paged cache (entry j of element b goes to its page)."""
    B, d_in = x_new.shape
    d_out = W.shape[1]
    if state.dtype != torch.float32:
        raise ValueError("state must be float32")
    _check(load().csa_compress_append_paged(
        _ptr(x_new), _dt(x_new), B, d_in, _ptr(W), d_out, m, int(bool(overlap)),
        _i32(pos, "pos"), _ptr(state), _ptr(cache.pool), _dt_rot(cache.pool, hadamard),
        _ptr(cache.scale), *cache.args, _i32(n_entries, "n_entries"), _stream(stream)))


def csa_indexer_topk_paged(qI: torch.Tensor, kI: PagedCache, m: int, topk: int,
                           idx_out: torch.Tensor, qI_scale: torch.Tensor | None = None,
                           n_entries: torch.Tensor | None = None, q_pos: torch.Tensor | None = None,
                           kI_rotated: bool = False, qI_weight: torch.Tensor | None = None,
                           stream=None) -> None:
    """csa_indexer_topk over a paged indexer-key cache (kI.scale: fp8 row scales)."""
    B, n_q, H_I, d_I = qI.shape
    _check(load().csa_indexer_topk_paged(
        _ptr(qI), _dt(qI), _ptr(qI_scale), _ptr(qI_weight), _ptr(kI.pool),
        _dt_rot(kI.pool, kI_rotated), _ptr(kI.scale), *kI.args, B, n_q, H_I, d_I,
        _i32(n_entries, "n_entries"), _i32(q_pos, "q_pos"), m, topk, _i32(idx_out, "idx_out"),
        _stream(stream)))


def csa_sparse_attn_paged(q: torch.Tensor, kv_c: PagedCache, idx: torch.Tensor | None,
                          kv_raw: torch.Tensor, window: int, out: torch.Tensor,
                          lse_out: torch.Tensor | None = None, raw_pos0: torch.Tensor | None = None,
                          raw_len: torch.Tensor | None = None, q_pos: torch.Tensor | None = None,
                          softmax_scale: float = 0.0, stream=None) -> None:
    B, n_q, H, D = q.shape
    topk = 0 if idx is None else idx.shape[-1]
    _check(load().csa_sparse_attn_paged(
        _ptr(q), _dt(q), B, n_q, H, D, _ptr(kv_c.pool), *kv_c.args, _i32(idx, "idx"), topk,
        _ptr(kv_raw), kv_raw.shape[1], _i32(raw_pos0, "raw_pos0"), _i32(raw_len, "raw_len"),
        window, _i32(q_pos, "q_pos"), float(softmax_scale), _ptr(out), _ptr(lse_out),
        _stream(stream)))


def hca_dense_attn_paged(q: torch.Tensor, kv_c: PagedCache, m: int, kv_raw: torch.Tensor,
                         window: int, out: torch.Tensor, lse_out: torch.Tensor | None = None,
                         n_entries: torch.Tensor | None = None,
                         raw_pos0: torch.Tensor | None = None, raw_len: torch.Tensor | None = None,
                         q_pos: torch.Tensor | None = None, softmax_scale: float = 0.0,
                         stream=None) -> None:
    B, n_q, H, D = q.shape
    _check(load().hca_dense_attn_paged(
        _ptr(q), _dt(q), B, n_q, H, D, _ptr(kv_c.pool), *kv_c.args, _i32(n_entries, "n_entries"),
        m, _ptr(kv_raw), kv_raw.shape[1], _i32(raw_pos0, "raw_pos0"), _i32(raw_len, "raw_len"),
        window, _i32(q_pos, "q_pos"), float(softmax_scale), _ptr(out), _ptr(lse_out),
        _stream(stream)))


# ---------------------------------------------------------------- allocating wrappers
def compress(x: torch.Tensor, W: torch.Tensor, m: int, overlap: bool, out_dtype=None,
             hadamard: bool = False, stream=None):
    """Returns out (and the per-row scales when out_dtype is fp8: (codes, scales))."""
    B, n, _ = x.shape
    N_c = n // m
    out_dtype = x.dtype if out_dtype is None else out_dtype
    if out_dtype in (torch.uint8, torch.float8_e4m3fn):
        out = torch.empty(B, N_c, W.shape[1], dtype=torch.uint8, device=x.device)
        scale = torch.empty(B, N_c, dtype=torch.float32, device=x.device)
        csa_compress(x, W, m, overlap, out, scale, hadamard=hadamard, stream=stream)
        return out, scale
    out = torch.empty(B, N_c, W.shape[1], dtype=out_dtype, device=x.device)
    csa_compress(x, W, m, overlap, out, stream=stream)
    return out


def compress_gated(x, W_kv, W_gate, ape, m: int, overlap: bool, out_dtype=None,
                   hadamard: bool = False, stream=None):
    """Allocating form of csa_compress_gated: out (or (codes, scales) for fp8)."""
    B, n, _ = x.shape
    N_c = n // m
    d_out = W_kv.shape[1] // (2 if overlap else 1)
    out_dtype = x.dtype if out_dtype is None else out_dtype
    if out_dtype in (torch.uint8, torch.float8_e4m3fn):
        out = torch.empty(B, N_c, d_out, dtype=torch.uint8, device=x.device)
        scale = torch.empty(B, N_c, dtype=torch.float32, device=x.device)
        csa_compress_gated(x, W_kv, W_gate, ape, m, overlap, out, scale, hadamard=hadamard,
                           stream=stream)
        return out, scale
    out = torch.empty(B, N_c, d_out, dtype=out_dtype, device=x.device)
    csa_compress_gated(x, W_kv, W_gate, ape, m, overlap, out, stream=stream)
    return out


def indexer_topk(qI, kI, m: int, topk: int, qI_scale=None, kI_scale=None, n_entries=None,
                 q_pos=None, kI_rotated: bool = False, qI_weight=None,
                 stream=None) -> torch.Tensor:
    B, n_q = qI.shape[:2]
    idx = torch.empty(B, n_q, topk, dtype=torch.int32, device=qI.device)
    csa_indexer_topk(qI, kI, m, topk, idx, qI_scale=qI_scale, kI_scale=kI_scale,
                     n_entries=n_entries, q_pos=q_pos, kI_rotated=kI_rotated,
                     qI_weight=qI_weight, stream=stream)
    return idx


def sparse_attn(q, kv_c, idx, kv_raw, window: int, with_lse: bool = False, **kw):
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if with_lse else None
    csa_sparse_attn(q, kv_c, idx, kv_raw, window, out, lse_out=lse, **kw)
    return (out, lse) if with_lse else out


def hca_attn(q, kv_c, m: int, kv_raw, window: int, with_lse: bool = False, **kw):
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if with_lse else None
    hca_dense_attn(q, kv_c, m, kv_raw, window, out, lse_out=lse, **kw)
    return (out, lse) if with_lse else out


def csa_prefill(q, kv, qI, kI_raw, W_c, W_Ic, m: int, topk: int, window: int,
                indexer_fp8: bool, indexer_hadamard: bool = False, qI_weight=None, stream=None):
    """The whole CSA prefill hot path (positions 0..n-1 of each sequence):
    compress kv, compress the indexer keys (fp8 + row scales when
    ``indexer_fp8``, Hadamard-rotated first when ``indexer_hadamard``),
    indexer + top-k (gated by ``qI_weight`` [B, n, H_I] when given), joint
    sparse attention.
    Returns dict(out, idx, kv_c, kI_c, kI_scale)."""
    kv_c = compress(kv, W_c, m, True, stream=stream)
    rot = bool(indexer_fp8 and indexer_hadamard)
    if indexer_fp8:
        kI_c, kI_scale = compress(kI_raw, W_Ic, m, True, out_dtype=torch.uint8, hadamard=rot,
                                  stream=stream)
    else:
        kI_c, kI_scale = compress(kI_raw, W_Ic, m, True, stream=stream), None
    idx = indexer_topk(qI, kI_c, m, topk, kI_scale=kI_scale, kI_rotated=rot, qI_weight=qI_weight,
                       stream=stream)
    out = sparse_attn(q, kv_c, idx, kv, window, stream=stream)
    return dict(out=out, idx=idx, kv_c=kv_c, kI_c=kI_c, kI_scale=kI_scale)
