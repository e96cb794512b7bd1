"""GPU parity of the fused rollout producer ("Thinking Machines Lab releases
4-bit training", configuration paragraph: the MoE forward GEMMs run in NVFP4):
the tcgen05 block-scaled GEMM with its quantizing epilogue, and the conversion
of row-layout scales into the tensor-core scale layout.

* scales_to_mma: bit-exact against the oracle's layout, ragged shapes included.
* D (the FP32 GEMM output, written on request) against the oracle's exact sum:
  the tensor core accumulates K/16 block partial sums in FP32 (order and
  internal rounding are the hardware's), then one multiply by fl(s_a s_b).  The
  bound used, per element, is
      |D_gpu - D| <= (K/16) * 2^-22 * sum|terms| + 2^-23 |D|
  -- twice the textbook recursive-summation bound for K/16 addends at unit
  roundoff 2^-23 (truncating adds), plus the final multiply.  A wrong scale,
  row or operand moves D by the size of whole terms, far above it.  This is
  also the pin of the scale layout: the tensor core reads the scales in the
  layout the oracle defines, and D matches only if they agree.
* The epilogue's quantization is bit-exact against the oracle quantizer fed
  the GPU's own D (codes, row-layout and MMA-layout scales, tensor scale,
  hints, observed amax) -- the same reading as for the RHT path, because the
  accumulation order cannot be reproduced on the CPU.
* Against the oracle's own D (no GPU value in its input): every code or scale
  that differs sits within the D bound of a rounding boundary.
"""
import numpy as np
import pytest
import torch

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import Buf, f32_bits, lib

pytestmark = pytest.mark.gpu

MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _operand(rows, k, seed, kind):
    x = syn.random_case((rows, k), seed, kind)
    codes, scales, ts, _ = oracle.quantize_rtn(x)
    return codes, scales, np.float32(ts)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _dev_mma_scales(scales, rows, sf_cols):
    b = lib()
    out = Buf(b.mma_scale_bytes(rows, sf_cols))
    b.nvfp4_scales_to_mma(_dev(scales.reshape(-1)), rows, sf_cols, out.t)
    return out


def gpu_gemm(ca, sa, ta, cb, sb, tb, m, n, k, a_out, hint_bits=2, want_d=True):
    b = lib()
    sfa = _dev_mma_scales(sa, m, k // 16)
    sfb = _dev_mma_scales(sb, n, k // 16)
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    ws[0] = np.int32(np.uint32(f32_bits(a_out)).view(np.int32))
    codes, scales = Buf(m * n // 2), Buf(m * n // 16)
    smma = Buf(b.mma_scale_bytes(m, n // 16))
    ts = Buf(4, torch.float32)
    hints = Buf(m * n * hint_bits // 8) if hint_bits else None
    d = Buf(4 * m * n, torch.float32) if want_d else None
    b.nvfp4_gemm_quantize(_dev(ca), sfa.t, _dev(np.array([ta], np.float32)), _dev(cb), sfb.t,
                          _dev(np.array([tb], np.float32)), m, n, k, ws, codes.t, scales.t, ts.t,
                          scales_mma=smma.t, hints=hints.t if hints else None, hint_bits=hint_bits,
                          d_out=d.t if d else None)
    torch.cuda.synchronize()
    out = dict(codes=codes.np(), scales=scales.np(), smma=smma.np(), ts=ts.np(),
               ws=ws.cpu().numpy().view(np.uint32), hints=hints.np() if hints else None,
               d=d.np().reshape(m, n) if d else None)
    sfa.check_tail()
    sfb.check_tail()
    return out


def _d_bound(d, dabs, k):
    return (k / 16) * 2.0 ** -22 * dabs + 2.0 ** -23 * np.abs(d)


def _check_against_own_d(got, m, n, a_out, hint_bits):
    """Epilogue parity: the oracle quantizer fed the GPU's D, bit for bit."""
    D = got["d"]
    codes, scales, ts = oracle.quantize_f32(D, a_out)
    assert np.float32(got["ts"][0]).view(np.uint32) == np.float32(ts).view(np.uint32)
    assert np.array_equal(got["scales"], scales.reshape(-1)), "row-layout scales"
    assert np.array_equal(got["codes"], codes.reshape(-1)), "codes"
    assert np.array_equal(got["smma"], oracle.scales_to_mma(scales, m, n // 16)), "MMA-layout scales"
    if hint_bits:
        assert np.array_equal(got["hints"], oracle.emit_hint(codes, m * n, hint_bits)), "hints"
    assert got["ws"][2] == np.float32(np.abs(D).max()).view(np.uint32), "observed amax"
    assert got["ws"][1] == 0, "warning bits"


def _check_against_oracle_d(got, d_ref, dabs, k, a_out):
    """Independent check: quantize the oracle's D; differences only at boundaries."""
    m, n = d_ref.shape
    tol = _d_bound(d_ref, dabs, k)
    D32 = d_ref.astype(np.float32)
    codes, scales, ts = oracle.quantize_f32(D32, a_out)
    gs = got["scales"].reshape(m, n // 16)
    rs = scales.reshape(m, n // 16)
    # a block scale may differ only by one E4M3 step, where the block amax is
    # within the bound of the other side's
    ds = gs.astype(int) - rs.astype(int)
    assert np.all(np.abs(ds) <= 1)
    same_scale = np.repeat(ds == 0, 16, axis=1)
    gc = oracle.unpack_codes(got["codes"]).reshape(m, n)
    rc = oracle.unpack_codes(codes).reshape(m, n)
    diff = (gc != rc) & same_scale & ~(((gc & 7) == 0) & ((rc & 7) == 0))
    if diff.any():
        sbv = np.vectorize(oracle.e4m3_value)(np.repeat(rs, 16, axis=1))[diff]
        inv = 1.0 / (sbv * float(ts))
        v = np.abs(d_ref[diff]) * inv
        near = np.min(np.abs(v[:, None] - MIDPOINTS[None, :]), axis=1)
        assert np.all(near <= tol[diff] * inv * 1.01 + 1e-12), "code differs away from a boundary"
        assert np.all(np.abs((gc[diff] & 7).astype(int) - (rc[diff] & 7).astype(int)) == 1)
    assert diff.sum() <= max(4, 1e-3 * m * n)
    assert (ds != 0).sum() <= max(2, 1e-3 * m * n // 16)


def _run_case(m, n, k, seed, kinds=("normal", "heavy"), hint_bits=2, a_scale=1.0):
    ca, sa, ta = _operand(m, k, seed, kinds[0])
    cb, sb, tb = _operand(n, k, seed + 1, kinds[1])
    d_ref, dabs = oracle.gemm_nvfp4(ca, sa, ta, cb, sb, tb, m, n, k)
    a_out = np.float32(np.abs(d_ref).max() * a_scale)
    got = gpu_gemm(ca, sa, ta, cb, sb, tb, m, n, k, a_out, hint_bits)
    err = np.abs(got["d"].astype(np.float64) - d_ref)
    bound = _d_bound(d_ref, dabs, k)
    worst = np.argmax(err - bound)
    assert np.all(err <= bound), "D off by %g (bound %g) at %s" % (
        err.flat[worst], bound.flat[worst], np.unravel_index(worst, err.shape))
    _check_against_own_d(got, m, n, a_out, hint_bits)
    _check_against_oracle_d(got, d_ref, dabs, k, a_out)
    return got


# ----------------------------------------------------------------- scale layout
@pytest.mark.parametrize("rows,sf_cols", [(128, 4), (256, 256), (200, 6), (1, 1), (130, 5),
                                          (1000, 33)])
def test_scales_to_mma_matches_oracle(rows, sf_cols):
    rng = np.random.Generator(np.random.PCG64(rows * 7 + sf_cols))
    s = rng.integers(0, 127, size=(rows, sf_cols), dtype=np.uint8)
    got = _dev_mma_scales(s, rows, sf_cols).np()
    assert np.array_equal(got, oracle.scales_to_mma(s, rows, sf_cols))


# ----------------------------------------------------------------- GEMM + quantize
@pytest.mark.parametrize("hint_bits", [0, 1, 2, 4])
def test_gemm_quantize_small(hint_bits):
    _run_case(256, 256, 512, 11, hint_bits=hint_bits)


@pytest.mark.parametrize("m,n,k,kinds", [
    (128, 128, 256, ("normal", "normal")),         # one tile, one K-block
    (384, 512, 1024, ("heavy", "outlier")),        # 3 x 4 tiles, 4 K-blocks: ring wraps
    (128, 256, 4096, ("normal", "tiny")),          # long K, subnormal block scales
    (256, 128, 768, ("sparse", "ties")),           # zeros, -0, grid midpoints
    # 256 x 256 tiles over CTA pairs (m, n multiples of 256)
    (512, 768, 2048, ("normal", "heavy")),         # 2 x 3 pair tiles, ring wraps
    (256, 512, 256, ("outlier", "normal")),        # one K-block per tile
    (768, 256, 4096, ("tiny", "normal")),          # long K, subnormal block scales
    (1024, 1024, 512, ("sparse", "ties")),         # 16 pair tiles
])
def test_gemm_quantize_shapes(m, n, k, kinds):
    _run_case(m, n, k, 23 + m + k, kinds)


def test_gemm_quantize_saturating_tensor_scale():
    # A_out a quarter of the true max: the largest blocks saturate (scale 448, code 7)
    got = _run_case(256, 256, 512, 5, a_scale=0.25)
    assert np.any(got["scales"] == 0x7E)


def test_gemm_quantize_zero_amax_gives_unit_tensor_scale():
    m = n = 128
    k = 256
    ca, sa, ta = _operand(m, k, 3, "normal")
    cb, sb, tb = _operand(n, k, 4, "normal")
    got = gpu_gemm(ca, sa, ta, cb, sb, tb, m, n, k, np.float32(0.0))
    assert got["ts"][0] == 1.0
    _check_against_own_d(got, m, n, np.float32(0.0), 2)


def test_gemm_quantize_without_d_output_matches():
    m, n, k = 256, 256, 512
    ca, sa, ta = _operand(m, k, 9, "normal")
    cb, sb, tb = _operand(n, k, 10, "normal")
    with_d = gpu_gemm(ca, sa, ta, cb, sb, tb, m, n, k, np.float32(8.0))
    no_d = gpu_gemm(ca, sa, ta, cb, sb, tb, m, n, k, np.float32(8.0), want_d=False)
    for key in ("codes", "scales", "smma", "hints"):
        assert np.array_equal(with_d[key], no_d[key]), key


def test_gemm_quantize_empty_rows_only_write_the_tensor_scale():
    b = lib()
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    ws[0] = np.int32(f32_bits(2688.0 * 2))
    ts = Buf(4, torch.float32)
    b.nvfp4_gemm_quantize(None, None, None, None, None, None, 0, 256, 512, ws, None, None, ts.t)
    torch.cuda.synchronize()
    assert ts.np()[0] == 2.0


def test_gemm_quantize_full_size_sampled_rows():
    """The workload the bench times (8192 tokens x 4096 -> 4096), one launch;
    the oracle checks 12 sampled rows of D and the quantization of all of D."""
    m, n, k = 8192, 4096, 4096
    rng = np.random.Generator(np.random.PCG64(77))
    xa = rng.standard_normal((m, k), dtype=np.float32)
    xb = (rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.02))
    ca, sa, ta, _ = oracle.quantize_rtn(syn.bf16_bits(xa))
    cb, sb, tb, _ = oracle.quantize_rtn(syn.bf16_bits(xb))
    rows = np.sort(rng.choice(m, 12, replace=False))
    rows[0], rows[-1] = 0, m - 1
    ca_rows = ca.reshape(m, k // 2)[rows]
    sa_rows = sa.reshape(m, k // 16)[rows]
    d_ref, dabs = oracle.gemm_nvfp4(ca_rows, sa_rows, ta, cb, sb, tb, len(rows), n, k)
    a_out = np.float32(np.abs(d_ref).max() * 1.5)
    got = gpu_gemm(ca, sa, np.float32(ta), cb, sb, np.float32(tb), m, n, k, a_out)
    D = got["d"]
    err = np.abs(D[rows].astype(np.float64) - d_ref)
    assert np.all(err <= _d_bound(d_ref, dabs, k))
    _check_against_own_d(got, m, n, a_out, 2)


def test_bounded_wait_reports_timeout_and_the_gpu_stays_usable():
    """Failure detection without a fault: the pipeline's bounded wait on a
    barrier nothing completes gives up after ~2 s with NVFP4_WARN_TIMEOUT, and
    a GEMM right after it still matches the oracle."""
    import time
    b = lib()
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    b.nvfp4_wait_selftest(ws)
    torch.cuda.synchronize()
    dt = time.time() - t0
    assert int(ws[1]) & b.NVFP4_WARN_TIMEOUT
    assert 1.5 < dt < 30.0, dt
    _run_case(128, 128, 256, 41)


# ----------------------------------------------------------------- MoE form
def gpu_moe(ca, sa, ta, experts, rows, n, k, a_out, hint_bits=2):
    """experts: list of (codes [n, k/2], scales [n, k/16], s_t) per expert."""
    b = lib()
    m, E = rows[-1], len(experts)
    sfa = _dev_mma_scales(sa, m, k // 16)
    w_scales = np.concatenate([np.asarray(w[1]).reshape(n, k // 16) for w in experts])
    sfw = _dev_mma_scales(w_scales, E * n, k // 16)       # = the experts' layouts, concatenated
    w_codes = np.concatenate([np.asarray(w[0]).reshape(n, k // 2) for w in experts])
    w_ts = np.array([w[2] for w in experts], np.float32)
    offs = torch.tensor(rows, dtype=torch.int32, device="cuda")
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    ws[0] = np.int32(np.uint32(f32_bits(a_out)).view(np.int32))
    codes, scales = Buf(m * n // 2), Buf(m * n // 16)
    smma = Buf(b.mma_scale_bytes(m, n // 16))
    ts = Buf(4, torch.float32)
    hints = Buf(m * n * hint_bits // 8) if hint_bits else None
    d = Buf(4 * m * n, torch.float32)
    b.nvfp4_moe_gemm_quantize(_dev(ca), sfa.t, _dev(np.array([ta], np.float32)), _dev(w_codes), sfw.t,
                              _dev(w_ts), offs, E, m, n, k, ws, codes.t, scales.t, ts.t, scales_mma=smma.t,
                              hints=hints.t if hints else None, hint_bits=hint_bits, d_out=d.t)
    torch.cuda.synchronize()
    return dict(codes=codes.np(), scales=scales.np(), smma=smma.np(), ts=ts.np(),
                ws=ws.cpu().numpy().view(np.uint32), hints=hints.np() if hints else None,
                d=d.np().reshape(m, n))


@pytest.mark.parametrize("rows,n,k,kinds", [
    ([0, 256, 256, 640, 768], 256, 512, ("normal", "heavy")),    # expert 1 gets no tokens
    ([0, 128, 256, 384, 512, 640, 768, 896, 1024], 128, 1024, ("outlier", "normal")),
])
def test_moe_gemm_quantize(rows, n, k, kinds):
    m, E = rows[-1], len(rows) - 1
    ca, sa, ta = _operand(m, k, 90 + E, kinds[0])
    experts = [_operand(n, k, 100 + e, kinds[1]) for e in range(E)]
    d_ref, dabs = oracle.moe_gemm_nvfp4(ca, sa, ta, [w[0] for w in experts], [w[1] for w in experts],
                                        [w[2] for w in experts], rows, n, k)
    a_out = np.float32(np.abs(d_ref).max())
    got = gpu_moe(ca, sa, ta, experts, rows, n, k, a_out)
    err = np.abs(got["d"].astype(np.float64) - d_ref)
    assert np.all(err <= _d_bound(d_ref, dabs, k))
    _check_against_own_d(got, m, n, a_out, 2)
    _check_against_oracle_d(got, d_ref, dabs, k, a_out)
