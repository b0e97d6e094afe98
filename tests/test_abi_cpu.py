"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, the binding's signature table matches the header, and
argument validation rejects bad calls before anything reaches the GPU.
CPU only: every call here fails validation (or is a no-op), so no kernel
is launched and no device memory is touched."""
import ctypes
import os
import re

import pytest

from long_context_compressed_03_b200 import api, build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa_b200.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return api.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = {}
    for m in re.finditer(r"(?:csa_status_t|const char\s*\*|unsigned long long|int)\s+(\w+)\s*\(([^)]*)\)\s*;",
                         text):
        name, params = m.group(1), m.group(2).strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        protos[name] = n
    return protos


def test_header_declares_the_four_stage_entry_points():
    d = _declared()
    for name in ("csa_compress", "csa_compress_append", "csa_indexer_topk", "csa_sparse_attn",
                 "hca_dense_attn", "csa_status_string", "csa_last_error_detail", "csa_version"):
        assert name in d


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_signatures_match_header_arity():
    d = _declared()
    for name, n in d.items():
        assert name in api.SIGNATURES, name
        assert len(api.SIGNATURES[name][1]) == n, name


def test_status_strings(lib):
    assert api.csa_version() == 100
    assert lib.csa_status_string(0) == b"CSA_OK"
    assert lib.csa_status_string(3) == b"CSA_ERR_MISALIGNED"
    assert lib.csa_status_string(99) == b"CSA_ERR_UNKNOWN"


FAKE = ctypes.c_void_p(0x10000)     # never dereferenced: validation fails first
ODD = ctypes.c_void_p(0x10001)


def _detail(lib):
    return lib.csa_last_error_detail().decode()


def test_compress_validation(lib):
    f = lib.csa_compress
    assert f(FAKE, 1, 1, 64, 128, FAKE, 128, 0, 1, FAKE, 1, None, None) == api.CSA_ERR_INVALID_ARG
    assert "m must be" in _detail(lib)
    assert f(FAKE, 1, 1, 64, 128, FAKE, 128, 4, 2, FAKE, 1, None, None) == api.CSA_ERR_INVALID_ARG
    assert f(FAKE, 1, 1, 64, 120, FAKE, 128, 4, 1, FAKE, 1, None, None) == api.CSA_ERR_UNSUPPORTED
    assert f(FAKE, 1, 1, 64, 128, FAKE, 128, 4, 1, FAKE, 0, None, None) == api.CSA_ERR_UNSUPPORTED
    # fp8 output without a scale buffer, and a scale buffer without fp8
    assert f(FAKE, 1, 1, 64, 128, FAKE, 128, 4, 1, FAKE, 2, None, None) == api.CSA_ERR_INVALID_ARG
    assert f(FAKE, 1, 1, 64, 128, FAKE, 128, 4, 1, FAKE, 1, FAKE, None) == api.CSA_ERR_INVALID_ARG
    assert f(ODD, 1, 1, 64, 128, FAKE, 128, 4, 1, FAKE, 1, None, None) == api.CSA_ERR_MISALIGNED
    assert f(None, 1, 1, 64, 128, FAKE, 128, 4, 1, FAKE, 1, None, None) == api.CSA_ERR_INVALID_ARG
    # no entries (n < m, or B = 0): nothing to do, nothing launched
    assert f(None, 1, 1, 3, 128, None, 128, 4, 1, None, 1, None, None) == api.CSA_OK
    assert f(None, 1, 0, 64, 128, None, 128, 4, 1, None, 1, None, None) == api.CSA_OK


def test_compress_gated_validation(lib):
    f = lib.csa_compress_gated
    #       x   dt B  n   d_in Wkv  Wg   ape  d_out m  ov out  dt scale stream
    args = [FAKE, 1, 1, 64, 64, FAKE, FAKE, FAKE, 64, 4, 1, FAKE, 1, None, None]
    bad = list(args); bad[9] = 0                       # m = 0
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[8] = 40                      # d_out not a multiple of 16
    assert f(*bad) == api.CSA_ERR_UNSUPPORTED
    bad = list(args); bad[7] = None                    # no APE
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[12] = 2                      # fp8 output without scales
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[1] = 2                       # fp8 input
    assert f(*bad) == api.CSA_ERR_UNSUPPORTED
    bad = list(args); bad[6] = ODD                     # misaligned gate weights
    assert f(*bad) == api.CSA_ERR_MISALIGNED
    bad = list(args); bad[12] = 0                      # F32 output from BF16 input
    assert f(*bad) == api.CSA_ERR_UNSUPPORTED
    ok = list(args); ok[3] = 3                         # n < m: no entries, no-op
    assert f(*ok) == api.CSA_OK


def test_compress_append_validation(lib):
    f = lib.csa_compress_append
    #       x_new dt B  d_in W    d_out m  ov pos   state cache dt scale N_cap n_ent stream
    args = [FAKE, 1, 2, 64, FAKE, 64, 4, 1, FAKE, FAKE, FAKE, 1, None, 16, None, None]
    bad = list(args); bad[6] = 0                       # m = 0
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[3] = 40                      # d_in not a multiple of 16
    assert f(*bad) == api.CSA_ERR_UNSUPPORTED
    bad = list(args); bad[11] = 2                      # fp8 cache without scales
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[8] = None                    # no positions
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[9] = ODD                     # misaligned state
    assert f(*bad) == api.CSA_ERR_MISALIGNED
    ok = list(args); ok[2] = 0                         # B = 0: no-op
    assert f(*ok) == api.CSA_OK


def test_indexer_validation(lib):
    f = lib.csa_indexer_topk
    #       qI  dt scale wt  kI   dt scale B  n_q H  d   N   ne    pos   m  k  idx   stream
    args = [FAKE, 1, None, None, FAKE, 1, None, 1, 8, 4, 64, 16, None, None, 4, 8, FAKE, None]
    bad = list(args); bad[15] = 0                      # topk = 0
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[15] = 4096                   # topk > 2048
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[5] = 2                       # fp8 keys without scales
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[10] = 60                     # d_I not a multiple of 16
    assert f(*bad) == api.CSA_ERR_UNSUPPORTED
    bad = list(args); bad[0] = ODD
    assert f(*bad) == api.CSA_ERR_MISALIGNED
    bad = list(args); bad[3] = ODD                     # misaligned gate weights
    assert f(*bad) == api.CSA_ERR_MISALIGNED
    bad = list(args); bad[14] = 0                      # m = 0
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    ok = list(args); ok[8] = 0                         # n_q = 0: no-op
    assert f(*ok) == api.CSA_OK


def test_hadamard_type_validation(lib):
    # the rotated fp8 type: d_out / d_I must be powers of two, scales are
    # required, queries are never given as that type, attention rejects it
    H = api.DT_E4M3_HADAMARD
    f = lib.csa_compress
    #       x   dt B  n   d_in W    d_out m  ov out  dt scale stream
    args = [FAKE, 1, 1, 64, 64, FAKE, 64, 4, 1, FAKE, H, FAKE, None]
    bad = list(args); bad[6] = 48                      # d_out not a power of two
    assert f(*bad) == api.CSA_ERR_UNSUPPORTED
    assert "power of two" in _detail(lib)
    bad = list(args); bad[11] = None                   # no scales
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    ok = list(args); ok[2] = 0                         # B = 0: no-op
    assert f(*ok) == api.CSA_OK
    g = lib.csa_compress_append
    args = [FAKE, 1, 2, 64, FAKE, 96, 4, 1, FAKE, FAKE, FAKE, H, FAKE, 16, None, None]
    assert g(*args) == api.CSA_ERR_UNSUPPORTED        # d_out = 96
    ok = list(args); ok[5] = 128; ok[2] = 0
    assert g(*ok) == api.CSA_OK
    h = lib.csa_indexer_topk
    args = [FAKE, 1, None, None, FAKE, H, FAKE, 1, 8, 4, 64, 16, None, None, 4, 8, FAKE, None]
    bad = list(args); bad[10] = 48                     # d_I not a power of two
    assert h(*bad) == api.CSA_ERR_UNSUPPORTED
    bad = list(args); bad[6] = None                    # rotated keys without scales
    assert h(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[1] = H; bad[2] = FAKE        # queries as the rotated type
    assert h(*bad) == api.CSA_ERR_UNSUPPORTED
    ok = list(args); ok[8] = 0
    assert h(*ok) == api.CSA_OK
    a = lib.csa_sparse_attn
    args = [FAKE, H, 1, 8, 64, 128, FAKE, 16, FAKE, 4, FAKE, 8, None, None, 4, None,
            ctypes.c_float(0.0), FAKE, None, None]
    assert a(*args) == api.CSA_ERR_UNSUPPORTED


def test_paged_entry_point_validation(lib):
    # the page map is checked before anything is launched
    f = lib.csa_sparse_attn_paged
    #       q   dt B  nq H   D    pool  bt   maxp P   np   idx  k  raw  L  p0    len   W  qpos
    args = [FAKE, 1, 1, 8, 64, 128, FAKE, FAKE, 16, 64, 40, FAKE, 4, FAKE, 8, None, None, 4, None,
            ctypes.c_float(0.0), FAKE, None, None]
    bad = list(args); bad[9] = 48                      # page size not a power of two
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[7] = None                    # no block table
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[7] = ODD
    assert f(*bad) == api.CSA_ERR_MISALIGNED
    bad = list(args); bad[8] = 1 << 20; bad[9] = 1 << 12   # capacity above 2^30 entries
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    ok = list(args); ok[2] = 0                         # B = 0: no-op
    assert f(*ok) == api.CSA_OK
    g = lib.csa_indexer_topk_paged
    #       qI  dt sc   wt   pool dt  scale bt   maxp P  np  B  nq H  d   ne    pos   m  k  idx  stream
    args = [FAKE, 1, None, None, FAKE, 2, None, FAKE, 16, 64, 40, 1, 1, 4, 64, None, FAKE, 4, 8, FAKE, None]
    assert g(*args) == api.CSA_ERR_INVALID_ARG        # fp8 keys without their scale pool
    bad = list(args); bad[6] = FAKE; bad[9] = 0        # page size 0
    assert g(*bad) == api.CSA_ERR_INVALID_ARG
    h = lib.csa_compress_append_paged
    #       x   dt B  d_in W    d_out m  ov pos   state cache dt scale bt  maxp P  np  n_ent stream
    args = [FAKE, 1, 2, 64, FAKE, 64, 4, 1, FAKE, FAKE, FAKE, 1, None, FAKE, 4, 3, 8, None, None]
    assert h(*args) == api.CSA_ERR_INVALID_ARG        # page size 3
    k = lib.hca_dense_attn_paged
    args = [FAKE, 2, 1, 1, 64, 128, FAKE, FAKE, 16, 64, 40, None, 4, FAKE, 8, None, None, 4, None,
            ctypes.c_float(0.0), FAKE, None, None]
    assert k(*args) == api.CSA_ERR_UNSUPPORTED        # fp8 attention operands


def test_varlen_offsets_and_validation(lib):
    cu = (ctypes.c_int * 4)(0, 5, 5, 13)
    off = (ctypes.c_int * 4)()
    assert lib.csa_varlen_entry_offsets(cu, 3, 4, off) == 3
    assert list(off) == [0, 1, 1, 3]
    assert lib.csa_varlen_entry_offsets(cu, 3, 0, off) == -1
    f = lib.csa_indexer_topk_varlen
    #       qI  dt sc   wt   kI   dt sc   S  cu  H  d   m  k  idx   stream
    args = [FAKE, 1, None, None, FAKE, 1, None, 3, cu, 4, 64, 4, 8, FAKE, None]
    bad = list(args); bad[8] = (ctypes.c_int * 4)(0, 5, 4, 13)    # decreasing
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[8] = (ctypes.c_int * 4)(1, 5, 5, 13)    # must start at 0
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[0] = ODD             # sequence 0's query rows off the 16-byte grid
    assert f(*bad) == api.CSA_ERR_MISALIGNED
    bad = list(args); bad[13] = None
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    ok = list(args); ok[7] = 0                 # no sequences: nothing to do
    assert f(*ok) == api.CSA_OK
    g = lib.csa_sparse_attn_varlen
    #       q   dt S  cu  H   D    kv_c m  idx  k  raw  W  scale             out   lse   stream
    args = [FAKE, 2, 3, cu, 64, 128, FAKE, 4, FAKE, 8, FAKE, 8, ctypes.c_float(0.0), FAKE, None, None]
    assert g(*args) == api.CSA_ERR_UNSUPPORTED                    # fp8 attention operands
    h = lib.csa_compress_varlen
    #       x   dt S  cu  d_in W    d_out m  ov out  dt scale stream
    args = [FAKE, 1, 3, cu, 64, FAKE, 64, 4, 1, FAKE, 1, FAKE, None]
    assert h(*args) == api.CSA_ERR_INVALID_ARG                    # scales with bf16 output


def test_attention_validation(lib):
    f = lib.csa_sparse_attn
    args = [FAKE, 1, 1, 8, 64, 128, FAKE, 16, FAKE, 4, FAKE, 8, None, None, 4, None,
            ctypes.c_float(0.0), FAKE, None, None]
    bad = list(args); bad[14] = -1
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[5] = 100
    assert f(*bad) == api.CSA_ERR_UNSUPPORTED
    bad = list(args); bad[1] = 2
    assert f(*bad) == api.CSA_ERR_UNSUPPORTED
    bad = list(args); bad[8] = None                    # idx NULL with topk > 0
    assert f(*bad) == api.CSA_ERR_INVALID_ARG
    bad = list(args); bad[17] = ODD
    assert f(*bad) == api.CSA_ERR_MISALIGNED
    ok = list(args); ok[2] = 0
    assert f(*ok) == api.CSA_OK
    g = lib.hca_dense_attn
    hargs = [FAKE, 1, 1, 8, 64, 128, FAKE, 16, None, 0, FAKE, 8, None, None, 4, None,
             ctypes.c_float(0.0), FAKE, None, None]
    assert g(*hargs) == api.CSA_ERR_INVALID_ARG          # m = 0
    assert "m must be" in _detail(lib)


def test_binding_raises_loudly_without_library(tmp_path):
    import importlib
    mod = importlib.reload(api)
    try:
        with pytest.raises(RuntimeError, match="not found"):
            mod._lib = None
            mod.load(str(tmp_path / "missing.so"))
    finally:
        importlib.reload(api)


def test_binding_rejects_host_tensors_and_bad_shapes(lib):
    # the binding marshals CUDA tensors only and checks what it can before the
    # C call; nothing here reaches a kernel
    import torch
    x = torch.zeros(1, 8, 16)
    W = torch.zeros(16, 16)
    with pytest.raises(ValueError, match="CUDA"):
        api.csa_compress(x, W, 4, True, torch.zeros(1, 2, 16))
    with pytest.raises(ValueError, match="int32"):
        api._i32(torch.zeros(3, dtype=torch.int64), "q_pos")
    with pytest.raises(ValueError, match="fp8"):
        api._dt_rot(torch.zeros(2, 2), True)      # rotation applies to fp8 rows only
    assert api._dt_rot(torch.zeros(2, 2, dtype=torch.uint8), True) == api.DT_E4M3_HADAMARD
    with pytest.raises(ValueError, match="pool"):
        api.PagedCache(torch.zeros(4, 4), torch.zeros(1, 2, dtype=torch.int32))
    with pytest.raises(ValueError, match="cu_seqlens"):
        api.varlen_entry_offsets([0, 5, 3], 4)     # decreasing
    assert api.varlen_entry_offsets([0, 5, 5, 13], 4).tolist() == [0, 1, 1, 3]


def test_injected_launch_error_maps_to_cuda_status(lib):
    # validation runs first, then the injected error stands in for the launch
    # (one shot).  The arguments are valid device buffers when a GPU is
    # present, so even a hook that failed to fire would compute on real memory.
    import torch
    if torch.cuda.is_available():
        dev = [torch.zeros(1, 8, 16, device="cuda"), torch.zeros(16, 16, device="cuda"),
               torch.zeros(1, 2, 16, device="cuda")]
        x, W, out = (ctypes.c_void_p(t.data_ptr()) for t in dev)
    else:
        x = W = out = FAKE
    assert lib.csa_debug_inject_launch_error(0) == api.CSA_ERR_INVALID_ARG
    # 801 would be read by the packed entry points as "take the per-sequence path"
    assert lib.csa_debug_inject_launch_error(801) == api.CSA_ERR_INVALID_ARG
    assert lib.csa_debug_inject_launch_error(719) == api.CSA_OK      # cudaErrorLaunchFailure
    # an invalid call reports its own error and leaves the injection pending
    assert lib.csa_compress(x, 0, 1, 8, 16, W, 16, 0, 1, out, 0, None, None) == api.CSA_ERR_INVALID_ARG
    before = lib.csa_kernel_launches()
    assert lib.csa_compress(x, 0, 1, 8, 16, W, 16, 4, 1, out, 0, None, None) == api.CSA_ERR_CUDA
    # the injected code's own message (a real launch on fake pointers would
    # report a different error), and nothing was launched
    assert "csa_compress" in _detail(lib) and "unspecified launch failure" in _detail(lib)
    assert lib.csa_kernel_launches() == before
    if not torch.cuda.is_available():
        return
    # consumed: the next call launches normally
    assert lib.csa_compress(x, 0, 1, 8, 16, W, 16, 4, 1, out, 0, None, None) == api.CSA_OK


def test_wait_limit_hook_validates_and_resets(lib):
    assert lib.csa_debug_set_wait_limit(-1, 0) == api.CSA_ERR_INVALID_ARG
    assert lib.csa_debug_set_wait_limit(2_000_000, 0) == api.CSA_OK
    assert lib.csa_debug_set_wait_limit(0, 0) == api.CSA_OK          # back to the default
