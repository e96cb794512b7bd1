"""The C-ABI library builds for sm_100a, loads without a GPU, exports every
entry point that include/nvfp4_trace.h declares, and rejects bad arguments
before touching the device (CPU only: validation never reaches CUDA)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib_path():
    from train_rollout_alignment_b200 import build
    return build.build()


def _declared():
    names = []
    for fname in os.listdir(os.path.join(ROOT, "include")):
        if fname.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fname)).read()
            names += re.findall(r"^\s*(?:nvfp4_status|const char\*|int64_t|int)\s+((?:nvfp4|mxfp8)_\w+)\s*\(", text, re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    want = {"nvfp4_quantize_rtn", "nvfp4_emit_hint", "nvfp4_guided_requant",
            "nvfp4_sr_transpose_requant", "nvfp4_rht_quantize", "nvfp4_mismatch_stats",
            "nvfp4_tensor_amax", "nvfp4_status_string", "nvfp4_quantize_tile16",
            "nvfp4_transpose_tile16", "mxfp8_sr_transpose_requant", "nvfp4_dequantize",
            "mxfp8_dequantize", "nvfp4_quantize_rtn_rows", "nvfp4_guided_requant_rows",
            "nvfp4_scales_to_mma", "nvfp4_gemm_quantize", "nvfp4_wait_selftest",
            "nvfp4_moe_gemm_quantize"}
    assert want <= set(_declared())


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib_path())
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_exports_only_the_c_abi():
    """Everything but the C ABI is local to the library, so two copies loaded
    in one process (or another library) cannot share its internals, e.g. the
    launchers' per-device shared-memory opt-in flags."""
    import shutil
    import subprocess
    if shutil.which("nm") is None:
        pytest.skip("nm not available")
    out = subprocess.run(["nm", "-D", "--defined-only", _lib_path()], capture_output=True, text=True,
                         check=True).stdout
    names = [line.split()[-1] for line in out.splitlines() if line.strip()]
    extra = [n for n in names if not (n.startswith("nvfp4_") or n.startswith("mxfp8_"))]
    assert not extra, extra[:10]
    assert set(_declared()) <= set(names)


def test_status_strings():
    lib = ctypes.CDLL(_lib_path())
    lib.nvfp4_status_string.restype = ctypes.c_char_p
    for s in range(6):
        assert lib.nvfp4_status_string(s)
    assert b"unknown" in lib.nvfp4_status_string(99)


def test_last_cuda_error_names_the_failure_without_a_gpu():
    """A call that passes validation but cannot launch (no driver or no GPU
    here) returns NVFP4_ERR_CUDA, and nvfp4_last_cuda_error keeps the CUDA
    error behind it; the binding puts its text into the exception."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a machine without a usable GPU (the call would launch)")
    lib = ctypes.CDLL(_lib_path())
    lib.nvfp4_last_cuda_error.restype = ctypes.c_int
    lib.nvfp4_last_cuda_error_string.restype = ctypes.c_char_p
    f = lib.nvfp4_tensor_amax
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    fake = 1 << 20  # the launch fails before any kernel could touch it
    assert f(fake, 16, fake, None) == 4
    err = lib.nvfp4_last_cuda_error()
    assert err != 0
    assert lib.nvfp4_last_cuda_error_string() not in (b"", b"no error")
    # not reset by a later call that fails validation
    assert f(fake, 15, fake, None) == 3
    assert lib.nvfp4_last_cuda_error() == err
    from train_rollout_alignment_b200 import _binding as b
    with pytest.raises(b.Nvfp4Error) as ei:
        b._check("nvfp4_tensor_amax", 4)
    assert ei.value.cuda_error == err and "CUDA error %d" % err in str(ei.value)


def test_validation_rejects_bad_arguments_without_a_gpu():
    lib = ctypes.CDLL(_lib_path())
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    q = lib.nvfp4_quantize_rtn
    q.restype = I
    q.argtypes = [P, I64, I64, P, I, P, P, P, P, I, P]
    fake = 1 << 20  # never dereferenced: every call below fails validation first
    assert q(fake, 4, 40, fake, 0, fake, fake, fake, None, 0, None) == 3          # cols % 16
    assert q(fake, -1, 64, fake, 0, fake, fake, fake, None, 0, None) == 1         # negative rows
    assert q(None, 4, 64, fake, 0, fake, fake, fake, None, 0, None) == 1          # null input
    assert q(fake + 16, 4, 64, fake, 0, fake, fake, fake, None, 0, None) == 2     # x not 32-B aligned
    assert q(fake, 4, 64, fake, 0, fake + 8, fake, fake, None, 0, None) == 2      # codes misaligned
    assert q(fake, 4, 64, fake, 0, fake, fake, fake, fake, 3, None) == 5          # hint bits
    assert q(fake, 4, 64, fake, 2, fake, fake, fake, None, 0, None) == 1          # unknown flag
    assert q(fake, 1 << 21, 1 << 20, fake, 0, fake, fake, fake, None, 0, None) == 3  # >= 2^40
    r = lib.nvfp4_rht_quantize
    r.restype = I
    r.argtypes = [P, I64, I64, ctypes.c_uint64, P, P, P, P, P, P]
    assert r(fake, 4, 48, 3, fake, fake, fake, fake, None, None) == 3              # cols % 32
    s = lib.nvfp4_sr_transpose_requant
    s.restype = I
    s.argtypes = [P, P, P, I64, I64, I64, ctypes.c_uint64, ctypes.c_uint32, P, P, P, P, P]
    assert s(fake, fake, fake, 2, 24, 32, 2, 0, fake, fake, fake, fake, None) == 3  # rows % 16
    assert s(fake, fake, fake, 70000, 16, 16, 2, 0, fake, fake, fake, fake, None) == 3
    assert s(fake, fake, fake, 0, 16, 16, 2, 0, None, None, None, None, None) == 0  # empty stack
    e = lib.nvfp4_emit_hint
    e.restype = I
    e.argtypes = [P, I64, I, P, P]
    assert e(fake, 32, 3, fake, None) == 5
    assert e(fake, 24, 2, fake, None) == 3
    assert e(fake, 32, 2, fake + 4, None) == 2


def test_validation_of_the_tile_and_mxfp8_entry_points_without_a_gpu():
    lib = ctypes.CDLL(_lib_path())
    P, I64, I, U64, U32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint32
    fake = 1 << 20
    q = lib.nvfp4_quantize_tile16
    q.restype = I
    q.argtypes = [P, I64, I64, P, I, P, P, P, P]
    assert q(fake, 24, 32, fake, 0, fake, fake, fake, None) == 3      # rows % 16
    assert q(fake, 32, 40, fake, 0, fake, fake, fake, None) == 3      # cols % 16
    assert q(None, 32, 32, fake, 0, fake, fake, fake, None) == 1
    assert q(fake + 16, 32, 32, fake, 0, fake, fake, fake, None) == 2
    assert q(fake, 32, 32, fake, 4, fake, fake, fake, None) == 1      # unknown flag
    t = lib.nvfp4_transpose_tile16
    t.restype = I
    t.argtypes = [P, P, I64, I64, I64, P, P, P]
    assert t(fake, fake, 1, 16, 24, fake, fake, None) == 3
    assert t(fake, fake, 70000, 16, 16, fake, fake, None) == 3
    assert t(fake, fake, 0, 16, 16, None, None, None) == 0            # empty stack
    assert t(fake, fake, 1, 16, 16, fake + 8, fake, None) == 2
    m = lib.mxfp8_sr_transpose_requant
    m.restype = I
    m.argtypes = [P, P, P, I64, I64, I64, U64, U32, P, P, P]
    assert m(fake, fake, fake, 1, 48, 32, 2, 0, fake, fake, None) == 3  # rows % 32
    assert m(fake, fake, fake, 1, 64, 24, 2, 0, fake, fake, None) == 3  # cols % 16
    assert m(fake, fake, None, 1, 64, 32, 2, 0, fake, fake, None) == 1
    assert m(fake, fake, fake, 1, 64, 32, 2, 0, fake + 4, fake, None) == 2
    d = lib.nvfp4_dequantize
    d.restype = I
    d.argtypes = [P, P, P, I64, I64, I, P, P]
    assert d(fake, fake, fake, 4, 32, 2, fake, None) == 1              # unknown layout
    assert d(fake, fake, fake, 8, 32, 1, fake, None) == 3              # tiles need rows % 16
    assert d(fake, fake, fake, 4, 32, 0, fake + 16, None) == 2         # out 32-B aligned
    x = lib.mxfp8_dequantize
    x.restype = I
    x.argtypes = [P, P, I64, P, P]
    assert x(fake, fake, 48, fake, None) == 3
    assert x(fake, fake, 64, fake + 16, None) == 2
    assert x(fake, fake, 0, None, None) == 0


def test_validation_of_the_kv_row_entry_points_without_a_gpu():
    lib = ctypes.CDLL(_lib_path())
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fake = 1 << 20
    q = lib.nvfp4_quantize_rtn_rows
    q.restype = I
    q.argtypes = [P, I64, I64, P, P, P, P, I, P]
    assert q(fake, 8, 96, fake, fake, fake, None, 0, None) == 3        # head_dim not a power of two
    assert q(fake, 8, 1024, fake, fake, fake, None, 0, None) == 3      # head_dim > 512
    assert q(fake, -1, 128, fake, fake, fake, None, 0, None) == 1
    assert q(None, 8, 128, fake, fake, fake, None, 0, None) == 1
    assert q(fake + 16, 8, 128, fake, fake, fake, None, 0, None) == 2
    assert q(fake, 8, 128, fake, fake, fake + 2, None, 0, None) == 2   # row scales 4-B aligned
    assert q(fake, 8, 128, fake, fake, fake, fake, 3, None) == 5
    assert q(fake, 0, 128, None, None, None, None, 0, None) == 0       # empty cache
    g = lib.nvfp4_guided_requant_rows
    g.restype = I
    g.argtypes = [P, I64, I64, P, I, P, P, P, P, P]
    assert g(fake, 8, 128, fake, 3, fake, fake, fake, None, None) == 5
    assert g(fake, 8, 128, fake, 2, fake, fake, fake, fake + 4, None) == 2  # stats 8-B aligned


def test_validation_of_the_producer_entry_points_without_a_gpu():
    lib = ctypes.CDLL(_lib_path())
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    g = lib.nvfp4_gemm_quantize
    g.restype = I
    g.argtypes = [P, P, P, P, P, P, I64, I64, I64, P, P, P, P, P, P, I, P, P]
    f = 1 << 20  # never dereferenced: every call below fails validation first

    def call(m=256, n=256, k=512, a=f, ws=f, codes=f, hints=None, hb=0, d_out=None, ts=f):
        return g(a, f, f, f, f, f, m, n, k, ws, codes, f, None, ts, hints, hb, d_out, None)

    assert call(m=200) == 3                       # m % 128
    assert call(n=100) == 3                       # n % 128
    assert call(k=384) == 3                       # k % 256
    assert call(k=0) == 3                         # k > 0
    assert call(m=-128) == 1                      # negative size
    assert call(ws=None) == 1                     # no scratch
    assert call(a=None) == 1                      # null operand
    assert call(codes=f + 16) == 2                # output codes not 32-B aligned
    assert call(ws=f + 4) == 2                    # ws not 16-B aligned
    assert call(d_out=f + 16) == 2                # D output not 32-B aligned
    assert call(hints=f, hb=3) == 5               # hint_bits not in {1, 2, 4}
    s2m = lib.nvfp4_scales_to_mma
    s2m.restype = I
    s2m.argtypes = [P, I64, I64, P, P]
    assert s2m(f, -1, 4, f, None) == 1
    assert s2m(f, 128, 4, f + 8, None) == 2
    assert s2m(None, 128, 4, f, None) == 1
    assert s2m(None, 0, 4, None, None) == 0       # empty: nothing to do
    mg = lib.nvfp4_moe_gemm_quantize
    mg.restype = I
    mg.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I64, P, P, P, P, P, P, I, P, P]
    assert mg(f, f, f, f, f, f, f, 0, 256, 256, 512, f, f, f, None, f, None, 0, None, None) == 1  # no experts
    assert mg(f, f, f, f, f, f, None, 4, 256, 256, 512, f, f, f, None, f, None, 0, None, None) == 1  # no offsets
    assert mg(f, f, f, f, f, f, f + 2, 4, 256, 256, 512, f, f, f, None, f, None, 0, None, None) == 2  # offsets align
    assert mg(f, f, f, f, f, f, f, 4, 200, 256, 512, f, f, f, None, f, None, 0, None, None) == 3  # m % 128


def test_noalloc_sr_transpose_returns_the_allocating_forms_status_without_a_gpu():
    """The no-allocation SR transpose checks its arguments exactly as the
    allocating form does, before it looks up its scratch array: an empty batch
    is a no-op and bad shapes or pointers give the same status."""
    lib = ctypes.CDLL(_lib_path())
    P, I64, U64, U32, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int
    a = lib.nvfp4_sr_transpose_requant
    a.restype = I
    a.argtypes = [P, P, P, I64, I64, I64, U64, U32, P, P, P, P, P]
    n = lib.nvfp4_sr_transpose_requant_noalloc
    n.restype = I
    n.argtypes = [P, P, P, I64, I64, I64, U64, U32, P, P, P, P]
    fake = 1 << 20
    cases = [
        (None, None, None, 0, 16, 16),        # empty batch: nothing to do
        (fake, fake, fake, 0, 16, 16),
        (fake, fake, fake, 2, 24, 16),        # rows % 16
        (fake, fake, fake, -1, 16, 16),       # negative batch
        (None, fake, fake, 2, 16, 16),        # null input
        (fake + 4, fake, fake, 2, 16, 16),    # misaligned codes
    ]
    for c_, s_, t_, batch, rows, cols in cases:
        want = a(c_, s_, t_, batch, rows, cols, 2, 0, fake, fake, fake, fake, None)
        got = n(c_, s_, t_, batch, rows, cols, 2, 0, fake, fake, fake, None)
        assert got == want, (batch, rows, cols, got, want)
    assert n(fake, fake, fake, 4097, 16, 16, 2, 0, fake, fake, fake, None) == 6   # over the scratch limit


def test_validation_of_the_fused_train_pass_without_a_gpu():
    lib = ctypes.CDLL(_lib_path())
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f = lib.nvfp4_guided_requant_stats
    f.restype = I
    f.argtypes = [P, I64, I64, P, I, P, I, P, P, P, P, P, P, P, P, P]
    a = 1 << 20  # never dereferenced: every call below fails validation first

    def call(x=a, rows=4, cols=64, hints=None, hb=2, ws=a, flags=0, codes=a, rc=a, rs=a, rts=a, s8=a, s4=None):
        return f(x, rows, cols, hints, hb, ws, flags, codes, a, a, s4, rc, rs, rts, s8, None)

    assert call(cols=40) == 3                 # cols % 16
    assert call(rows=-1) == 1                 # negative size
    assert call(s8=None) == 1                 # the counters are required
    assert call(rc=None) == 1                 # the rollout tensor is required
    assert call(rts=None) == 1
    assert call(flags=2) == 1                 # unknown flag
    assert call(hints=a, hb=3) == 5           # hint width
    assert call(x=a + 16) == 2                # BF16 input 32-byte aligned
    assert call(rc=a + 8) == 2                # rollout codes 16-byte aligned
    assert call(s8=a + 4) == 2                # counters 8-byte aligned
    assert call(s4=a + 4) == 2


def test_hint_pack_validation_and_size_without_a_gpu():
    lib = ctypes.CDLL(_lib_path())
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    size = lib.nvfp4_hint_pack_size
    size.restype = I64
    size.argtypes = [P, I64]
    pack = lib.nvfp4_hint_pack
    pack.restype = I
    pack.argtypes = [P, P, I64, P, P, P]
    sizes = (ctypes.c_int64 * 4)(16, 1, 0, 33)
    assert size(sizes, 4) == 16 + 16 + 0 + 48
    assert size(sizes, 0) == 0
    assert size(None, 2) == -1
    assert size((ctypes.c_int64 * 1)(-1), 1) == -1
    assert size((ctypes.c_int64 * 1)(1 << 40), 1) == -1
    a = 1 << 20
    srcs = (ctypes.c_void_p * 4)(a, a + 16, None, a + 32)
    assert pack(srcs, sizes, 4, None, None, None) == 1            # no staging buffer
    assert pack(srcs, sizes, 4, a + 8, None, None) == 2           # staging not 16-byte aligned
    bad = (ctypes.c_void_p * 4)(a, a + 8, None, a + 32)
    assert pack(bad, sizes, 4, a, None, None) == 2                # a stream not 16-byte aligned
    nul = (ctypes.c_void_p * 4)(a, None, None, a)
    assert pack(nul, sizes, 4, a, None, None) == 1                # a non-empty stream without a pointer
    assert pack(srcs, sizes, -1, a, None, None) == 1
    assert pack(None, None, 0, None, None, None) == 0             # nothing to do
    zeros = (ctypes.c_int64 * 2)(0, 0)
    assert pack((ctypes.c_void_p * 2)(None, None), zeros, 2, None, None, None) == 0


def test_moe_dispatch_sizes_and_validation_without_a_gpu():
    lib = ctypes.CDLL(_lib_path())
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    cap = lib.nvfp4_moe_rows_cap
    cap.restype, cap.argtypes = I64, [I64, I64]
    words = lib.nvfp4_moe_route_ws_words
    words.restype, words.argtypes = I64, [I64, I64]
    assert cap(6, 3) == 384 and cap(0, 1) == 0 and cap(256, 1) == 256 and cap(257, 2) == 384
    assert cap(-1, 3) == -1 and cap(5, 0) == -1 and cap(5, 1025) == -1
    assert words(6, 3) == 2 * 3 and words(4097, 5) == (3 + 1) * 5
    route = lib.nvfp4_moe_route
    route.restype = I
    route.argtypes = [P, I64, I64, I64, P, P, P, I64, P, P]
    a = 1 << 20
    assert route(a, 3, 2, 3, a, a, a, 384, a, None) != 3              # capacity large enough
    assert route(a, 3, 2, 3, a, a, a, 383, a, None) == 3              # capacity too small
    assert route(a, 3, 2, 2000, a, a, a, 1 << 20, a, None) == 3       # too many experts
    assert route(a, 3, 0, 3, a, a, a, 384, a, None) == 1              # top_k 0
    assert route(a, 3, 2, 3, None, a, a, 384, a, None) == 1           # no scratch
    assert route(a + 2, 3, 2, 3, a, a, a, 384, a, None) == 2          # ids not 4-byte aligned
    gather = lib.nvfp4_moe_gather
    gather.restype = I
    gather.argtypes = [P, P, I64, I64, P, I64, I64, P, P, P]
    assert gather(a, a, 3, 96, a, 128, 2, a, a, None) == 3            # k % 64
    assert gather(a, a, 3, 128, a, 100, 2, a, a, None) == 3           # m_cap % 128
    assert gather(a, a, 3, 128, a, 128, 2, a + 8, a, None) == 2       # a_codes 16-byte aligned
    assert gather(a, a, 3, 128, None, 128, 2, a, a, None) == 1
    assert gather(None, None, 0, 128, None, 0, 2, None, None, None) == 0
