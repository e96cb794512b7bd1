"""ctypes binding of libnvfp4trace.so: one Python function per C-ABI entry
point, same names, argument marshalling only.

Tensors are torch CUDA tensors (torch provides device memory and streams, the
library does all the work).  Each function passes ``data_ptr()``s, sizes and
the current CUDA stream, and raises ``Nvfp4Error`` on a non-zero status.  There
is no CPU path: importing this module fails if the library is not built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4trace.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        "libnvfp4trace.so is not built; run `python -m train_rollout_alignment_b200.build` "
        "(nvcc, sm_100a).  There is no CPU fallback.")
_lib = ctypes.CDLL(_LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SIGS = {
    "nvfp4_status_string": (ctypes.c_char_p, [_I]),
    "nvfp4_last_cuda_error": (_I, []),
    "nvfp4_last_cuda_error_string": (ctypes.c_char_p, []),
    "nvfp4_tensor_amax": (_I, [_P, _I64, _P, _P]),
    "nvfp4_quantize_rtn": (_I, [_P, _I64, _I64, _P, _I, _P, _P, _P, _P, _I, _P]),
    "nvfp4_emit_hint": (_I, [_P, _I64, _I, _P, _P]),
    "nvfp4_guided_requant": (_I, [_P, _I64, _I64, _P, _I, _P, _I, _P, _P, _P, _P, _P]),
    "nvfp4_mismatch_stats": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _P, _P]),
    "nvfp4_guided_requant_stats": (
        _I, [_P, _I64, _I64, _P, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "nvfp4_sr_transpose_requant": (
        _I, [_P, _P, _P, _I64, _I64, _I64, ctypes.c_uint64, ctypes.c_uint32, _P, _P, _P, _P, _P]),
    "nvfp4_rht_quantize": (_I, [_P, _I64, _I64, ctypes.c_uint64, _P, _P, _P, _P, _P, _P]),
    "nvfp4_sr_transpose_requant_noalloc": (
        _I, [_P, _P, _P, _I64, _I64, _I64, ctypes.c_uint64, ctypes.c_uint32, _P, _P, _P, _P]),
    "nvfp4_quantize_tile16": (_I, [_P, _I64, _I64, _P, _I, _P, _P, _P, _P]),
    "nvfp4_quantize_rtn_rows": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _I, _P]),
    "nvfp4_guided_requant_rows": (_I, [_P, _I64, _I64, _P, _I, _P, _P, _P, _P, _P]),
    "nvfp4_transpose_tile16": (_I, [_P, _P, _I64, _I64, _I64, _P, _P, _P]),
    "mxfp8_sr_transpose_requant": (
        _I, [_P, _P, _P, _I64, _I64, _I64, ctypes.c_uint64, ctypes.c_uint32, _P, _P, _P]),
    "nvfp4_dequantize": (_I, [_P, _P, _P, _I64, _I64, _I, _P, _P]),
    "mxfp8_dequantize": (_I, [_P, _P, _I64, _P, _P]),
    "nvfp4_scales_to_mma": (_I, [_P, _I64, _I64, _P, _P]),
    "nvfp4_wait_selftest": (_I, [_P, _P]),
    "nvfp4_hint_pack": (_I, [_P, _P, _I64, _P, _P, _P]),
    "nvfp4_hint_pack_size": (_I64, [_P, _I64]),
    "nvfp4_moe_rows_cap": (_I64, [_I64, _I64]),
    "nvfp4_measure_mul_wide": (_I, [_I64, _I64, _P, _P, _P]),
    "nvfp4_moe_route_ws_words": (_I64, [_I64, _I64]),
    "nvfp4_moe_route": (_I, [_P, _I64, _I64, _I64, _P, _P, _P, _I64, _P, _P]),
    "nvfp4_moe_gather": (_I, [_P, _P, _I64, _I64, _P, _I64, _I64, _P, _P, _P]),
    "nvfp4_moe_gemm_quantize": (
        _I, [_P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _I, _P, _P]),
    "nvfp4_gemm_quantize": (
        _I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _I, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

# Constants mirrored from include/nvfp4_trace.h
NVFP4_WS_WORDS = 8
NVFP4_STATS8_WORDS = 8
NVFP4_STATS4_WORDS = 4
NVFP4_AMAX_PRECOMPUTED = 1
NVFP4_WARN_NONFINITE = 1
NVFP4_WARN_TIMEOUT = 2
NVFP4_ERR_SCRATCH_LIMIT = 6
NVFP4_SR_NOALLOC_MAX_BATCH = 4096
NVFP4_SCALES_BLOCK16 = 0
NVFP4_SCALES_TILE16 = 1


NVFP4_ERR_CUDA = 4


class Nvfp4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = "%s: %s (status %d)" % (fn, nvfp4_status_string(status), status)
        if status == NVFP4_ERR_CUDA:
            self.cuda_error = nvfp4_last_cuda_error()
            msg += ": CUDA error %d, %s" % (self.cuda_error, nvfp4_last_cuda_error_string())
        super().__init__(msg)


def library_path() -> str:
    return _LIB_PATH


def nvfp4_status_string(status: int) -> str:
    return _lib.nvfp4_status_string(int(status)).decode()


def nvfp4_last_cuda_error() -> int:
    return int(_lib.nvfp4_last_cuda_error())


def nvfp4_last_cuda_error_string() -> str:
    return _lib.nvfp4_last_cuda_error_string().decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("NVFP4 kernels take CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("NVFP4 kernels take contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, status: int):
    if status != 0:
        raise Nvfp4Error(fn, status)


def _rows_cols(x):
    if x.dim() != 2:
        raise ValueError("expected a 2-D [rows, cols] tensor")
    return int(x.shape[0]), int(x.shape[1])


def nvfp4_tensor_amax(x, ws, stream=None):
    _check("nvfp4_tensor_amax", _lib.nvfp4_tensor_amax(_ptr(x), x.numel(), _ptr(ws), _stream(stream)))


def nvfp4_quantize_rtn(x, ws, codes, scales, tensor_scale, hints=None, hint_bits=0, flags=0,
                       stream=None):
    rows, cols = _rows_cols(x)
    _check("nvfp4_quantize_rtn", _lib.nvfp4_quantize_rtn(
        _ptr(x), rows, cols, _ptr(ws), int(flags), _ptr(codes), _ptr(scales), _ptr(tensor_scale),
        _ptr(hints), int(hint_bits), _stream(stream)))


def nvfp4_emit_hint(codes, n, hint_bits, hints, stream=None):
    _check("nvfp4_emit_hint", _lib.nvfp4_emit_hint(_ptr(codes), int(n), int(hint_bits), _ptr(hints),
                                                   _stream(stream)))


def nvfp4_guided_requant(x, hints, hint_bits, ws, codes, scales, tensor_scale, stats4=None, flags=0,
                         stream=None):
    rows, cols = _rows_cols(x)
    _check("nvfp4_guided_requant", _lib.nvfp4_guided_requant(
        _ptr(x), rows, cols, _ptr(hints), int(hint_bits), _ptr(ws), int(flags), _ptr(codes),
        _ptr(scales), _ptr(tensor_scale), _ptr(stats4), _stream(stream)))


def nvfp4_guided_requant_stats(x, hints, hint_bits, ws, codes, scales, tensor_scale, stats4, roll_codes,
                               roll_scales, roll_tensor_scale, stats8, flags=0, stream=None):
    rows, cols = _rows_cols(x)
    _check("nvfp4_guided_requant_stats", _lib.nvfp4_guided_requant_stats(
        _ptr(x), rows, cols, _ptr(hints), int(hint_bits), _ptr(ws), int(flags), _ptr(codes),
        _ptr(scales), _ptr(tensor_scale), _ptr(stats4), _ptr(roll_codes), _ptr(roll_scales),
        _ptr(roll_tensor_scale), _ptr(stats8), _stream(stream)))


def nvfp4_mismatch_stats(codes_a, scales_a, ts_a, codes_b, scales_b, ts_b, rows, cols, stats8,
                         stream=None):
    _check("nvfp4_mismatch_stats", _lib.nvfp4_mismatch_stats(
        _ptr(codes_a), _ptr(scales_a), _ptr(ts_a), _ptr(codes_b), _ptr(scales_b), _ptr(ts_b),
        int(rows), int(cols), _ptr(stats8), _stream(stream)))


def nvfp4_sr_transpose_requant(codes, scales, tensor_scale, batch, rows, cols, seed, draw, ws,
                               codes_t, scales_t, tensor_scale_t, stream=None):
    _check("nvfp4_sr_transpose_requant", _lib.nvfp4_sr_transpose_requant(
        _ptr(codes), _ptr(scales), _ptr(tensor_scale), int(batch), int(rows), int(cols),
        int(seed) & 0xFFFFFFFFFFFFFFFF, int(draw) & 0xFFFFFFFF, _ptr(ws), _ptr(codes_t),
        _ptr(scales_t), _ptr(tensor_scale_t), _stream(stream)))


def nvfp4_sr_transpose_requant_noalloc(codes, scales, tensor_scale, batch, rows, cols, seed, draw,
                                       codes_t, scales_t, tensor_scale_t, stream=None):
    """SR transpose without a scratch argument, for callers that cannot
    allocate device memory (the library keeps a fixed scratch array of
    NVFP4_SR_NOALLOC_MAX_BATCH words per GPU; see include/nvfp4_trace.h)."""
    _check("nvfp4_sr_transpose_requant_noalloc", _lib.nvfp4_sr_transpose_requant_noalloc(
        _ptr(codes), _ptr(scales), _ptr(tensor_scale), int(batch), int(rows), int(cols),
        int(seed) & 0xFFFFFFFFFFFFFFFF, int(draw) & 0xFFFFFFFF, _ptr(codes_t), _ptr(scales_t),
        _ptr(tensor_scale_t), _stream(stream)))


def nvfp4_rht_quantize(x, sign_seed, ws, codes, scales, tensor_scale, y_out=None, stream=None):
    rows, cols = _rows_cols(x)
    _check("nvfp4_rht_quantize", _lib.nvfp4_rht_quantize(
        _ptr(x), rows, cols, int(sign_seed) & 0xFFFFFFFFFFFFFFFF, _ptr(ws), _ptr(codes), _ptr(scales),
        _ptr(tensor_scale), _ptr(y_out), _stream(stream)))


# ----------------------------------------------------------------- output buffers
def empty_nvfp4(rows: int, cols: int, device, hint_bits: int = 0):
    """Device buffers for one quantized [rows, cols] tensor: codes, scales,
    tensor scale, scratch words and (optionally) hints."""
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=device)
    ts = torch.empty(1, dtype=torch.float32, device=device)
    ws = torch.zeros(NVFP4_WS_WORDS, dtype=torch.int32, device=device)  # words 4..7 must start at zero
    hints = None
    if hint_bits:
        hints = torch.empty(((rows * cols * hint_bits + 7) // 8,), dtype=torch.uint8, device=device)
    return codes, scales, ts, ws, hints


# ----------------------------------------------------------------- alternatives to SR transpose
def nvfp4_quantize_tile16(x, ws, codes, tile_scales, tensor_scale, flags=0, stream=None):
    rows, cols = _rows_cols(x)
    _check("nvfp4_quantize_tile16", _lib.nvfp4_quantize_tile16(
        _ptr(x), rows, cols, _ptr(ws), int(flags), _ptr(codes), _ptr(tile_scales), _ptr(tensor_scale),
        _stream(stream)))


def nvfp4_transpose_tile16(codes, tile_scales, batch, rows, cols, codes_t, tile_scales_t, stream=None):
    _check("nvfp4_transpose_tile16", _lib.nvfp4_transpose_tile16(
        _ptr(codes), _ptr(tile_scales), int(batch), int(rows), int(cols), _ptr(codes_t),
        _ptr(tile_scales_t), _stream(stream)))


def mxfp8_sr_transpose_requant(codes, scales, tensor_scale, batch, rows, cols, seed, draw, q_t, e8_t,
                               stream=None):
    _check("mxfp8_sr_transpose_requant", _lib.mxfp8_sr_transpose_requant(
        _ptr(codes), _ptr(scales), _ptr(tensor_scale), int(batch), int(rows), int(cols),
        int(seed) & 0xFFFFFFFFFFFFFFFF, int(draw) & 0xFFFFFFFF, _ptr(q_t), _ptr(e8_t), _stream(stream)))


def nvfp4_dequantize(codes, scales, tensor_scale, rows, cols, scale_layout, out, stream=None):
    _check("nvfp4_dequantize", _lib.nvfp4_dequantize(
        _ptr(codes), _ptr(scales), _ptr(tensor_scale), int(rows), int(cols), int(scale_layout), _ptr(out),
        _stream(stream)))


def mxfp8_dequantize(q, e8, n, out, stream=None):
    _check("mxfp8_dequantize", _lib.mxfp8_dequantize(_ptr(q), _ptr(e8), int(n), _ptr(out), _stream(stream)))


# ----------------------------------------------------------------- KV-cache rows
def nvfp4_quantize_rtn_rows(x, codes, scales, row_scales, hints=None, hint_bits=0, stream=None):
    rows, cols = _rows_cols(x)
    _check("nvfp4_quantize_rtn_rows", _lib.nvfp4_quantize_rtn_rows(
        _ptr(x), rows, cols, _ptr(codes), _ptr(scales), _ptr(row_scales), _ptr(hints), int(hint_bits),
        _stream(stream)))


def nvfp4_guided_requant_rows(x, hints, hint_bits, codes, scales, row_scales, stats4=None, stream=None):
    rows, cols = _rows_cols(x)
    _check("nvfp4_guided_requant_rows", _lib.nvfp4_guided_requant_rows(
        _ptr(x), rows, cols, _ptr(hints), int(hint_bits), _ptr(codes), _ptr(scales), _ptr(row_scales),
        _ptr(stats4), _stream(stream)))


# ----------------------------------------------------------------- rollout producer
def mma_scale_bytes(rows: int, sf_cols: int) -> int:
    """Size of the 128x4-tiled tensor-core scale layout of [rows, sf_cols] scales."""
    return ((rows + 127) // 128) * ((sf_cols + 3) // 4) * 512


def nvfp4_scales_to_mma(scales, rows, sf_cols, scales_mma, stream=None):
    _check("nvfp4_scales_to_mma", _lib.nvfp4_scales_to_mma(
        _ptr(scales), int(rows), int(sf_cols), _ptr(scales_mma), _stream(stream)))


def nvfp4_gemm_quantize(a_codes, a_scales_mma, a_ts, b_codes, b_scales_mma, b_ts, m, n, k, ws, codes,
                        scales, tensor_scale, scales_mma=None, hints=None, hint_bits=0, d_out=None,
                        stream=None):
    _check("nvfp4_gemm_quantize", _lib.nvfp4_gemm_quantize(
        _ptr(a_codes), _ptr(a_scales_mma), _ptr(a_ts), _ptr(b_codes), _ptr(b_scales_mma), _ptr(b_ts),
        int(m), int(n), int(k), _ptr(ws), _ptr(codes), _ptr(scales), _ptr(scales_mma), _ptr(tensor_scale),
        _ptr(hints), int(hint_bits), _ptr(d_out), _stream(stream)))


def nvfp4_moe_gemm_quantize(a_codes, a_scales_mma, a_ts, w_codes, w_scales_mma, w_ts, expert_rows, experts, m,
                            n, k, ws, codes, scales, tensor_scale, scales_mma=None, hints=None, hint_bits=0,
                            d_out=None, stream=None):
    _check("nvfp4_moe_gemm_quantize", _lib.nvfp4_moe_gemm_quantize(
        _ptr(a_codes), _ptr(a_scales_mma), _ptr(a_ts), _ptr(w_codes), _ptr(w_scales_mma), _ptr(w_ts),
        _ptr(expert_rows), int(experts), int(m), int(n), int(k), _ptr(ws), _ptr(codes), _ptr(scales),
        _ptr(scales_mma), _ptr(tensor_scale), _ptr(hints), int(hint_bits), _ptr(d_out), _stream(stream)))


def nvfp4_hint_pack_size(sizes) -> int:
    arr = (ctypes.c_int64 * max(1, len(sizes)))(*[int(v) for v in sizes])
    total = _lib.nvfp4_hint_pack_size(arr, len(sizes))
    if total < 0:
        raise ValueError("invalid hint stream sizes")
    return int(total)


def nvfp4_hint_pack(streams, staging, host_dst=None, stream=None):
    """Gather the device byte tensors `streams` into `staging` (each stream on
    a 16-byte boundary, padding zeroed) and copy that to `host_dst` (a CPU
    uint8 tensor, pinned for an asynchronous copy) when given."""
    n = len(streams)
    srcs = (ctypes.c_void_p * max(1, n))(*[_ptr(t) if t.numel() else None for t in streams])
    sizes = (ctypes.c_int64 * max(1, n))(*[t.numel() * t.element_size() for t in streams])
    host = None
    if host_dst is not None:
        if host_dst.is_cuda or not host_dst.is_contiguous():
            raise ValueError("host_dst must be a contiguous CPU tensor")
        host = host_dst.data_ptr()
    _check("nvfp4_hint_pack", _lib.nvfp4_hint_pack(srcs, sizes, n, _ptr(staging), host, _stream(stream)))


def nvfp4_moe_rows_cap(assignments: int, experts: int) -> int:
    v = int(_lib.nvfp4_moe_rows_cap(int(assignments), int(experts)))
    if v < 0:
        raise ValueError("unsupported routing size")
    return v


def nvfp4_moe_route_ws_words(assignments: int, experts: int) -> int:
    v = int(_lib.nvfp4_moe_route_ws_words(int(assignments), int(experts)))
    if v < 0:
        raise ValueError("unsupported routing size")
    return v


def nvfp4_moe_route(topk_ids, experts, ws, expert_rows, row_src, assign_row, stream=None):
    """topk_ids: int32 [tokens, top_k] (CUDA)."""
    tokens, top_k = int(topk_ids.shape[0]), int(topk_ids.shape[1])
    _check("nvfp4_moe_route", _lib.nvfp4_moe_route(
        _ptr(topk_ids), tokens, top_k, int(experts), _ptr(ws), _ptr(expert_rows), _ptr(row_src),
        int(row_src.numel()), _ptr(assign_row), _stream(stream)))


def nvfp4_moe_gather(codes, scales, tokens, k, row_src, top_k, a_codes, a_scales_mma, stream=None):
    _check("nvfp4_moe_gather", _lib.nvfp4_moe_gather(
        _ptr(codes), _ptr(scales), int(tokens), int(k), _ptr(row_src), int(row_src.numel()), int(top_k),
        _ptr(a_codes), _ptr(a_scales_mma), _stream(stream)))


def nvfp4_measure_mul_wide(ctas, iters, cycles, sink, stream=None):
    _check("nvfp4_measure_mul_wide", _lib.nvfp4_measure_mul_wide(int(ctas), int(iters), _ptr(cycles), _ptr(sink),
                                                                 _stream(stream)))


def nvfp4_wait_selftest(ws, stream=None):
    _check("nvfp4_wait_selftest", _lib.nvfp4_wait_selftest(_ptr(ws), _stream(stream)))
