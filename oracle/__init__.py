"""CPU oracle for NVFP4 quantization with train/rollout rounding alignment.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``train_rollout_alignment_b200``) never imports it and has no CPU
fallback.

The arithmetic lives in ``nvfp4_oracle.c`` (plain scalar C, every FP32 step one
IEEE round-to-nearest operation).  This module only compiles it with gcc and
marshals numpy arrays.  ctypes releases the GIL during each call, so callers
may run independent tensors on a thread pool.

Pages followed: "TRACE explainer" (blog.ontle.kr/blog/286), "Quantization in RL
training" (ai-systems-engineering.com) and "Thinking Machines Lab releases 4-bit
training" (metallab.ai); the C file cites the paragraph behind each step.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_nvfp4.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc) if missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            F = ctypes.c_float
            sig = {
                "oracle_e2m1_value": (ctypes.c_double, [ctypes.c_int]),
                "oracle_e2m1_rne": (ctypes.c_int, [F]),
                "oracle_e4m3_value": (ctypes.c_double, [ctypes.c_int]),
                "oracle_e4m3_rne_satfinite": (ctypes.c_int, [F]),
                "oracle_bf16_to_f32": (F, [ctypes.c_uint16]),
                "oracle_amax_f32": (F, [P, I64]),
                "oracle_amax_bf16": (F, [P, I64]),
                "oracle_tensor_scale": (F, [F]),
                "oracle_block_scale": (ctypes.c_int, [F, F]),
                "oracle_quantize_f32": (None, [P, I64, I64, F, P, P, P]),
                "oracle_emit_hint": (None, [P, I64, ctypes.c_int, P]),
                "oracle_quantize_rtn_bf16": (None, [P, I64, I64, F, P, P, P, P, ctypes.c_int]),
                "oracle_guided_bf16": (None, [P, I64, I64, F, P, ctypes.c_int, P, P, P, P]),
                "oracle_dequant_one": (F, [ctypes.c_int, ctypes.c_int, F]),
                "oracle_dequant": (None, [P, P, F, I64, P]),
                "oracle_mismatch_stats": (None, [P, P, F, P, P, F, I64, I64, P]),
                "oracle_philox4x32_10": (None, [P, P, P]),
                "oracle_sr_magnitude": (ctypes.c_int, [F, ctypes.c_uint32]),
                "oracle_sr_transpose_requant": (
                    None, [P, P, P, I64, I64, I64, ctypes.c_uint64, ctypes.c_uint32, P, P, P]),
                "oracle_sr_transpose_requant_from": (
                    None, [P, P, P, I64, I64, I64, I64, ctypes.c_uint64, ctypes.c_uint32, P, P, P]),
                "oracle_quantize_tile16_bf16": (None, [P, I64, I64, F, P, P, P]),
                "oracle_transpose_tile16": (None, [P, P, I64, I64, I64, P, P]),
                "oracle_dequant_tile16": (None, [P, P, F, I64, I64, P]),
                "oracle_e8m0_exponent": (ctypes.c_int, [F]),
                "oracle_e4m3_sr": (ctypes.c_int, [F, ctypes.c_uint32]),
                "oracle_mxfp8_sr_transpose_requant": (
                    None, [P, P, P, I64, I64, I64, ctypes.c_uint64, ctypes.c_uint32, P, P]),
                "oracle_mxfp8_sr_transpose_requant_from": (
                    None, [P, P, P, I64, I64, I64, I64, ctypes.c_uint64, ctypes.c_uint32, P, P]),
                "oracle_mxfp8_dequant": (None, [P, P, I64, P]),
                "oracle_quantize_rtn_rows_bf16": (None, [P, I64, I64, P, P, P, P, ctypes.c_int]),
                "oracle_guided_rows_bf16": (None, [P, I64, I64, P, ctypes.c_int, P, P, P, P]),
                "oracle_rht_signs": (None, [ctypes.c_uint64, P]),
                "oracle_rht32_f64": (None, [P, I64, I64, ctypes.c_uint64, P]),
                "oracle_rht_quantize": (None, [P, I64, I64, ctypes.c_uint64, P, P, P, P]),
                "oracle_gemm_nvfp4": (None, [P, P, F, P, P, F, I64, I64, I64, P, P]),
                "oracle_scales_to_mma": (None, [P, I64, I64, P]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(x) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "BF16 inputs are passed as uint16 bit patterns"
    return x


# --------------------------------------------------------------------------- scalars
def e2m1_value(m: int) -> float:
    return _load().oracle_e2m1_value(int(m))


def e2m1_rne(a: float) -> int:
    return _load().oracle_e2m1_rne(float(a))


def e4m3_value(b: int) -> float:
    return _load().oracle_e4m3_value(int(b))


def e4m3_rne_satfinite(f: float) -> int:
    return _load().oracle_e4m3_rne_satfinite(float(f))


def tensor_scale(A: float) -> float:
    return _load().oracle_tensor_scale(float(A))


def block_scale(amax_block: float, s_t: float) -> int:
    return _load().oracle_block_scale(float(amax_block), float(s_t))


def sr_magnitude(a: float, r: int) -> int:
    return _load().oracle_sr_magnitude(float(a), int(r) & 0xFFFFFFFF)


def philox4x32_10(ctr, key) -> tuple:
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    _load().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return tuple(int(v) for v in out)


def rht_signs(seed: int) -> np.ndarray:
    s = np.zeros(32, dtype=np.int32)
    _load().oracle_rht_signs(int(seed), _ptr(s))
    return s


# --------------------------------------------------------------------------- tensors
def amax_bf16(x) -> float:
    x = _u16(x)
    return float(_load().oracle_amax_bf16(_ptr(x), x.size))


def amax_f32(y) -> float:
    y = np.ascontiguousarray(y, dtype=np.float32)
    return float(_load().oracle_amax_f32(_ptr(y), y.size))


def _alloc_q(rows, cols):
    return (np.zeros((rows, cols // 2), np.uint8), np.zeros((rows, cols // 16), np.uint8),
            np.zeros(1, np.float32))


def quantize_f32(y, A: float | None = None):
    """Round-to-nearest NVFP4 of an FP32 [rows, cols] array -> (codes, scales, s_t)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    rows, cols = y.shape
    if A is None:
        A = amax_f32(y)
    codes, scales, ts = _alloc_q(rows, cols)
    _load().oracle_quantize_f32(_ptr(y), rows, cols, float(A), _ptr(codes), _ptr(scales), _ptr(ts))
    return codes, scales, float(ts[0])


def quantize_rtn(x, A: float | None = None, hint_bits: int = 0):
    """Rollout side: BF16 [rows, cols] -> (codes, scales, s_t, hints or None).

    ``A`` is the tensor amax; pass the full tensor's amax when ``x`` holds only
    some rows of it (sampled checking)."""
    x = _u16(x)
    rows, cols = x.shape
    if A is None:
        A = amax_bf16(x)
    codes, scales, ts = _alloc_q(rows, cols)
    hints = None
    hp = None
    if hint_bits:
        hints = np.zeros((rows * cols * hint_bits + 7) // 8, np.uint8)
        hp = _ptr(hints)
    _load().oracle_quantize_rtn_bf16(_ptr(x), rows, cols, float(A), _ptr(codes), _ptr(scales),
                                     _ptr(ts), hp, int(hint_bits))
    return codes, scales, float(ts[0]), hints


def emit_hint(codes, n: int, hint_bits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    hints = np.zeros((n * hint_bits + 7) // 8, np.uint8)
    _load().oracle_emit_hint(_ptr(codes), int(n), int(hint_bits), _ptr(hints))
    return hints


def guided_requant(x, hints, hint_bits: int, A: float | None = None):
    """Train side: BF16 [rows, cols] + rollout hints -> (codes, scales, s_t, stats4)."""
    x = _u16(x)
    rows, cols = x.shape
    if A is None:
        A = amax_bf16(x)
    codes, scales, ts = _alloc_q(rows, cols)
    stats = np.zeros(4, np.uint64)
    hp = None
    if hints is not None:
        hints = np.ascontiguousarray(hints, dtype=np.uint8)
        hp = _ptr(hints)
    _load().oracle_guided_bf16(_ptr(x), rows, cols, float(A), hp, int(hint_bits), _ptr(codes),
                               _ptr(scales), _ptr(ts), _ptr(stats))
    return codes, scales, float(ts[0]), stats


def quantize_rtn_rows(x, hint_bits: int = 0):
    """KV-cache layout: every row of BF16 [rows, cols] is its own tensor ->
    (codes, scales, row_scales [rows], hints or None)."""
    x = _u16(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    rs = np.zeros(rows, np.float32)
    hints = np.zeros((rows * cols * hint_bits + 7) // 8, np.uint8) if hint_bits else None
    _load().oracle_quantize_rtn_rows_bf16(_ptr(x), rows, cols, _ptr(codes), _ptr(scales), _ptr(rs),
                                          _ptr(hints) if hints is not None else None, int(hint_bits))
    return codes, scales, rs, hints


def guided_requant_rows(x, hints, hint_bits: int):
    """KV-cache layout, train side -> (codes, scales, row_scales, stats4)."""
    x = _u16(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    rs = np.zeros(rows, np.float32)
    stats = np.zeros(4, np.uint64)
    hp = None
    if hints is not None:
        hints = np.ascontiguousarray(hints, dtype=np.uint8)
        hp = _ptr(hints)
    _load().oracle_guided_rows_bf16(_ptr(x), rows, cols, hp, int(hint_bits), _ptr(codes), _ptr(scales),
                                    _ptr(rs), _ptr(stats))
    return codes, scales, rs, stats


def dequant_one(code: int, scale_byte: int, s_t: float) -> float:
    return float(_load().oracle_dequant_one(int(code), int(scale_byte), float(s_t)))


def dequant(codes, scales, s_t: float, n: int) -> np.ndarray:
    """NVFP4 -> FP32 values, flat, n elements."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out = np.zeros(n, np.float32)
    _load().oracle_dequant(_ptr(codes), _ptr(scales), float(s_t), int(n), _ptr(out))
    return out


def mismatch_stats(codes_a, scales_a, ts_a, codes_b, scales_b, ts_b, rows, cols) -> np.ndarray:
    ca = np.ascontiguousarray(codes_a, dtype=np.uint8)
    sa = np.ascontiguousarray(scales_a, dtype=np.uint8)
    cb = np.ascontiguousarray(codes_b, dtype=np.uint8)
    sb = np.ascontiguousarray(scales_b, dtype=np.uint8)
    stats = np.zeros(8, np.uint64)
    _load().oracle_mismatch_stats(_ptr(ca), _ptr(sa), float(ts_a), _ptr(cb), _ptr(sb), float(ts_b),
                                  int(rows), int(cols), _ptr(stats))
    return stats


def sr_transpose_requant(codes, scales, ts, batch, rows, cols, seed, draw, first: int = 0):
    """[batch, rows, cols] NVFP4 -> transposed [batch, cols, rows] NVFP4 by SR.

    ``first``: index of the first given matrix within the whole stack (the
    random counter is the element's index in the whole output stack)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    ts = np.ascontiguousarray(ts, dtype=np.float32)
    ct = np.zeros((batch, cols, rows // 2), np.uint8)
    st = np.zeros((batch, cols, rows // 16), np.uint8)
    tst = np.zeros(batch, np.float32)
    _load().oracle_sr_transpose_requant_from(_ptr(codes), _ptr(scales), _ptr(ts), int(first),
                                             int(batch), int(rows), int(cols), int(seed),
                                             int(draw) & 0xFFFFFFFF, _ptr(ct), _ptr(st), _ptr(tst))
    return ct, st, tst


def quantize_tile16(x, A: float | None = None):
    """BF16 [rows, cols] -> (codes [rows, cols/2], tile scales [rows/16, cols/16], s_t)."""
    x = _u16(x)
    rows, cols = x.shape
    if A is None:
        A = amax_bf16(x)
    codes = np.zeros((rows, cols // 2), np.uint8)
    tscales = np.zeros((rows // 16, cols // 16), np.uint8)
    ts = np.zeros(1, np.float32)
    _load().oracle_quantize_tile16_bf16(_ptr(x), rows, cols, float(A), _ptr(codes), _ptr(tscales),
                                        _ptr(ts))
    return codes, tscales, float(ts[0])


def transpose_tile16(codes, tscales, batch, rows, cols):
    """[batch, rows, cols] tile-scaled codes -> [batch, cols, rows] (lossless)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    tscales = np.ascontiguousarray(tscales, dtype=np.uint8)
    ct = np.zeros((batch, cols, rows // 2), np.uint8)
    st = np.zeros((batch, cols // 16, rows // 16), np.uint8)
    _load().oracle_transpose_tile16(_ptr(codes), _ptr(tscales), int(batch), int(rows), int(cols),
                                    _ptr(ct), _ptr(st))
    return ct, st


def dequant_tile16(codes, tscales, s_t: float, rows: int, cols: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    tscales = np.ascontiguousarray(tscales, dtype=np.uint8)
    out = np.zeros((rows, cols), np.float32)
    _load().oracle_dequant_tile16(_ptr(codes), _ptr(tscales), float(s_t), int(rows), int(cols),
                                  _ptr(out))
    return out


def e8m0_exponent(amax: float) -> int:
    return _load().oracle_e8m0_exponent(float(amax))


def e4m3_sr(a: float, r: int) -> int:
    return _load().oracle_e4m3_sr(float(a), int(r) & 0xFFFFFFFF)


def mxfp8_sr_transpose_requant(codes, scales, ts, batch, rows, cols, seed, draw, first: int = 0):
    """[batch, rows, cols] NVFP4 -> (E4M3 bytes [batch, cols, rows],
    E8M0 bytes [batch, cols, rows/32]) by dequantize, transpose and SR.

    ``first``: index of the first given matrix within the whole stack (the
    random counter is the element's index in the whole output stack)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    ts = np.ascontiguousarray(ts, dtype=np.float32)
    q = np.zeros((batch, cols, rows), np.uint8)
    e8 = np.zeros((batch, cols, rows // 32), np.uint8)
    _load().oracle_mxfp8_sr_transpose_requant_from(_ptr(codes), _ptr(scales), _ptr(ts), int(first),
                                                   int(batch), int(rows), int(cols), int(seed),
                                                   int(draw) & 0xFFFFFFFF, _ptr(q), _ptr(e8))
    return q, e8


def mxfp8_dequant(q, e8) -> np.ndarray:
    """MXFP8 -> FP32, flat; blocks of 32 consecutive elements."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    e8 = np.ascontiguousarray(e8, dtype=np.uint8)
    out = np.zeros(q.size, np.float32)
    _load().oracle_mxfp8_dequant(_ptr(q), _ptr(e8), int(q.size), _ptr(out))
    return out


def rht32_f64(x, seed: int) -> np.ndarray:
    x = _u16(x)
    rows, cols = x.shape
    y = np.zeros((rows, cols), np.float64)
    _load().oracle_rht32_f64(_ptr(x), rows, cols, int(seed), _ptr(y))
    return y


def rht_quantize(x, seed: int):
    """-> (codes, scales, s_t, y_f32) with y the FP32-rounded double transform."""
    x = _u16(x)
    rows, cols = x.shape
    codes, scales, ts = _alloc_q(rows, cols)
    y = np.zeros((rows, cols), np.float32)
    _load().oracle_rht_quantize(_ptr(x), rows, cols, int(seed), _ptr(codes), _ptr(scales), _ptr(ts),
                                _ptr(y))
    return codes, scales, float(ts[0]), y


def gemm_nvfp4(a_codes, a_scales, a_ts: float, b_codes, b_scales, b_ts: float, m: int, n: int,
               k: int):
    """D = dec(A) @ dec(B)^T for NVFP4 A [m, k], B [n, k] (row-layout scales).

    -> (d, dabs) float64 [m, n]: D (exact sum, one final rounding) and the
    same sum of |terms|."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8).reshape(-1)
    b_codes = np.ascontiguousarray(b_codes, dtype=np.uint8).reshape(-1)
    a_scales = np.ascontiguousarray(a_scales, dtype=np.uint8).reshape(-1)
    b_scales = np.ascontiguousarray(b_scales, dtype=np.uint8).reshape(-1)
    assert a_codes.size == m * k // 2 and b_codes.size == n * k // 2
    assert a_scales.size == m * k // 16 and b_scales.size == n * k // 16
    d = np.zeros((m, n), np.float64)
    dabs = np.zeros((m, n), np.float64)
    _load().oracle_gemm_nvfp4(_ptr(a_codes), _ptr(a_scales), float(a_ts), _ptr(b_codes),
                              _ptr(b_scales), float(b_ts), m, n, k, _ptr(d), _ptr(dabs))
    return d, dabs


def moe_gemm_nvfp4(a_codes, a_scales, a_ts: float, w_codes, w_scales, w_ts, expert_rows, n: int,
                   k: int):
    """The MoE form of gemm_nvfp4: A rows expert_rows[e] .. expert_rows[e+1]-1
    times expert e's weight W_e [n, k] (w_* indexed by expert).  Each expert's
    block is the plain GEMM of its rows ("Thinking Machines Lab releases 4-bit
    training", configuration paragraph: the MoE forward runs in NVFP4).

    -> (d, dabs) float64 [m, n]."""
    rows = [int(r) for r in expert_rows]
    m = rows[-1]
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8).reshape(m, k // 2)
    a_scales = np.ascontiguousarray(a_scales, dtype=np.uint8).reshape(m, k // 16)
    d = np.zeros((m, n), np.float64)
    dabs = np.zeros((m, n), np.float64)
    for e in range(len(rows) - 1):
        r0, r1 = rows[e], rows[e + 1]
        if r1 == r0:
            continue
        d[r0:r1], dabs[r0:r1] = gemm_nvfp4(a_codes[r0:r1], a_scales[r0:r1], a_ts, w_codes[e], w_scales[e],
                                           float(w_ts[e]), r1 - r0, n, k)
    return d, dabs


def moe_route(topk_ids, experts: int):
    """The dispatch of routed tokens to the experts ("Thinking Machines Lab
    releases 4-bit training", communication paragraph: tokens are sent to the
    experts in NVFP4; configuration paragraph: the MoE forward runs in NVFP4).
    The pages give no layout; the reading taken: the (token, slot)
    assignments a = token * top_k + slot are grouped by expert, in increasing
    a within an expert, and every expert's group is padded with empty rows to
    a multiple of 128 (the tile height of the expert GEMM); an assignment whose
    expert id is outside 0 .. experts - 1 is dropped.

    -> (expert_rows [experts + 1], row_src [expert_rows[-1]] with the
    assignment of each grouped row or -1 for a padding row, assign_row [A]
    with the grouped row of each assignment or -1), all int64."""
    ids = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    rows = [0]
    row_src = []
    assign_row = np.full(ids.size, -1, np.int64)
    for e in range(experts):
        idx = np.nonzero(ids == e)[0]
        start = rows[-1]
        assign_row[idx] = start + np.arange(idx.size)
        pad = (-idx.size) % 128
        row_src.extend(idx.tolist() + [-1] * pad)
        rows.append(start + idx.size + pad)
    return np.array(rows, np.int64), np.array(row_src, np.int64), assign_row


def scales_to_mma(scales, rows: int, sf_cols: int) -> np.ndarray:
    """Row-layout block scales [rows, sf_cols] -> the 128x4-tiled MMA layout."""
    scales = np.ascontiguousarray(scales, dtype=np.uint8).reshape(-1)
    assert scales.size == rows * sf_cols
    out = np.zeros(mma_scale_bytes(rows, sf_cols), np.uint8)
    _load().oracle_scales_to_mma(_ptr(scales), rows, sf_cols, _ptr(out))
    return out


def mma_scale_bytes(rows: int, sf_cols: int) -> int:
    return ((rows + 127) // 128) * ((sf_cols + 3) // 4) * 512


# --------------------------------------------------------------------------- helpers
def unpack_codes(codes, n: int | None = None) -> np.ndarray:
    """Packed nibbles -> one uint8 code per element (element 2j = low nibble)."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(c.size * 2, np.uint8)
    out[0::2] = c & 15
    out[1::2] = c >> 4
    return out if n is None else out[:n]
