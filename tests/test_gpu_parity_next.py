"""GPU parity for the alternatives to the SR transpose step ("Thinking Machines
Lab releases 4-bit training", forward/backward mismatch paragraph): 16x16-tile
NVFP4 quantize and lossless transpose, MXFP8 stochastic-rounding transpose
re-quantize, and the dequantize entry points -- bit for bit against the oracle
through the C ABI, on small shapes that span several tiles with ragged edges,
on the edge cases, and on the 128x512x2048 expert stack at full size."""
import numpy as np
import pytest
import torch

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import Buf, assert_codes_equal, dev_bf16, f32_bits, lib, pool

pytestmark = pytest.mark.gpu

KINDS = ["normal", "heavy", "tiny", "outlier", "zeros", "ties", "sparse"]


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()


def gpu_tile16(x, precomputed=False):
    b = lib()
    xt = dev_bf16(x)
    rows, cols = xt.shape
    n = rows * cols
    codes, tsc, ts = Buf(n // 2), Buf(n // 256), Buf(4, torch.float32)
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    flags = 0
    if precomputed:
        b.nvfp4_tensor_amax(xt, ws)
        flags = b.NVFP4_AMAX_PRECOMPUTED
    b.nvfp4_quantize_tile16(xt, ws, codes.t, tsc.t, ts.t, flags)
    torch.cuda.synchronize()
    return codes.np().reshape(rows, cols // 2), tsc.np().reshape(rows // 16, cols // 16), float(ts.np()[0])


def gpu_transpose_tile16(codes, tsc, batch, rows, cols):
    b = lib()
    n = rows * cols
    ct, tt = Buf(batch * n // 2), Buf(batch * n // 256)
    b.nvfp4_transpose_tile16(dev(codes), dev(tsc), batch, rows, cols, ct.t, tt.t)
    torch.cuda.synchronize()
    return ct.np().reshape(batch, cols, rows // 2), tt.np().reshape(batch, cols // 16, rows // 16)


def gpu_mxfp8(codes, scales, ts, batch, rows, cols, seed, draw):
    b = lib()
    n = batch * rows * cols
    q, e8 = Buf(n), Buf(n // 32)
    b.mxfp8_sr_transpose_requant(dev(codes), dev(scales), dev(np.asarray(ts, np.float32)), batch, rows, cols,
                                 seed, draw, q.t, e8.t)
    torch.cuda.synchronize()
    return q.np().reshape(batch, cols, rows), e8.np().reshape(batch, cols, rows // 32)


def _rtn_stack(w):
    batch = w.shape[0]
    with pool(batch) as ex:
        outs = list(ex.map(lambda e: oracle.quantize_rtn(w[e]), range(batch)))
    return (np.stack([o[0] for o in outs]), np.stack([o[1] for o in outs]),
            np.array([o[2] for o in outs], np.float32))


# ----------------------------------------------------------------------------- tile-16
@pytest.mark.parametrize("shape", [(16, 16), (16, 48), (48, 80), (128, 2048), (272, 528)])
@pytest.mark.parametrize("kind", KINDS)
def test_tile16_quantize_matches_oracle(shape, kind):
    x = syn.random_case(shape, 7000 + shape[0] + shape[1], kind)
    oc, ot, os_ = oracle.quantize_tile16(x)
    for pre in (False, True):
        gc, gt, gs = gpu_tile16(x, pre)
        assert f32_bits(gs) == f32_bits(os_)
        assert_codes_equal(gt, ot, "tile scales")
        assert_codes_equal(gc, oc, "tile codes")


@pytest.mark.parametrize("shape", [(1, 16, 16), (3, 48, 80), (2, 64, 64), (2, 80, 144), (1, 208, 48)])
def test_tile16_transpose_matches_oracle(shape):
    batch, rows, cols = shape
    w = syn.random_case(shape, 7100 + rows, "heavy")
    q = [oracle.quantize_tile16(w[e]) for e in range(batch)]
    codes, tsc = np.stack([a[0] for a in q]), np.stack([a[1] for a in q])
    gc, gt = gpu_transpose_tile16(codes, tsc, batch, rows, cols)
    oc, ot = oracle.transpose_tile16(codes, tsc, batch, rows, cols)
    assert_codes_equal(gt, ot, "transposed tile scales")
    assert_codes_equal(gc, oc, "transposed codes")


def test_tile16_transpose_of_gpu_quantize_is_gpu_quantize_of_transpose():
    x = syn.random_case((96, 160), 7200, "outlier")
    c, t, s = gpu_tile16(x)
    ct, tt = gpu_transpose_tile16(c[None], t[None], 1, 96, 160)
    c2, t2, s2 = gpu_tile16(np.ascontiguousarray(x.T))
    assert s == s2
    assert_codes_equal(ct[0], c2, "codes")
    assert_codes_equal(tt[0], t2, "tile scales")


# ----------------------------------------------------------------------------- MXFP8
@pytest.mark.parametrize("shape", [(1, 32, 16), (2, 64, 48), (3, 128, 64), (2, 160, 208), (1, 256, 16)])
@pytest.mark.parametrize("kind", ["normal", "heavy", "tiny", "outlier", "zeros"])
def test_mxfp8_sr_transpose_matches_oracle(shape, kind):
    batch, rows, cols = shape
    w = syn.random_case(shape, 7300 + rows + cols, kind)
    codes, scales, ts = _rtn_stack(w)
    for seed, draw in ((2, 0), (2, 1), ((5 << 32) | 17, 123456)):
        gq, ge = gpu_mxfp8(codes, scales, ts, batch, rows, cols, seed, draw)
        oq, oe = oracle.mxfp8_sr_transpose_requant(codes, scales, ts, batch, rows, cols, seed, draw)
        assert_codes_equal(ge, oe, "E8M0 scales")
        assert_codes_equal(gq, oq, "E4M3 bytes")


def test_mxfp8_sr_transpose_extreme_tensor_scales():
    """Tensor scales that push the E8M0 exponent to its clamps and the FP32
    products into the subnormal range."""
    batch, rows, cols = 4, 64, 32
    w = syn.random_case((batch, rows, cols), 7400, "heavy")
    codes, scales, _ = _rtn_stack(w)
    ts = np.array([2.0 ** -120, 2.0 ** -140, 3.0e30, 1.0], np.float32)
    gq, ge = gpu_mxfp8(codes, scales, ts, batch, rows, cols, 3, 9)
    oq, oe = oracle.mxfp8_sr_transpose_requant(codes, scales, ts, batch, rows, cols, 3, 9)
    assert_codes_equal(ge, oe, "E8M0 scales")
    assert_codes_equal(gq, oq, "E4M3 bytes")


# ----------------------------------------------------------------------------- dequantize
@pytest.mark.parametrize("shape", [(16, 16), (48, 80), (208, 1024)])
def test_nvfp4_dequantize_matches_oracle(shape):
    b = lib()
    rows, cols = shape
    x = syn.random_case(shape, 7500 + rows, "heavy")
    c, s, t, _ = oracle.quantize_rtn(x)
    out = Buf(4 * rows * cols, torch.float32)
    b.nvfp4_dequantize(dev(c), dev(s), dev(np.array([t], np.float32)), rows, cols, b.NVFP4_SCALES_BLOCK16, out.t)
    torch.cuda.synchronize()
    want = oracle.dequant(c, s, t, rows * cols)
    assert np.array_equal(out.np().view(np.uint32), want.view(np.uint32))
    ct, tt, tst = oracle.quantize_tile16(x)
    out2 = Buf(4 * rows * cols, torch.float32)
    b.nvfp4_dequantize(dev(ct), dev(tt), dev(np.array([tst], np.float32)), rows, cols, b.NVFP4_SCALES_TILE16,
                       out2.t)
    torch.cuda.synchronize()
    want2 = oracle.dequant_tile16(ct, tt, tst, rows, cols).reshape(-1)
    assert np.array_equal(out2.np().view(np.uint32), want2.view(np.uint32))


def test_mxfp8_dequantize_matches_oracle():
    b = lib()
    rng = np.random.default_rng(9)
    n = 32 * 4001
    q = rng.integers(0, 256, n).astype(np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x7E  # no NaN encodings
    e8 = rng.integers(0, 255, n // 32).astype(np.uint8)
    e8[:8] = [0, 1, 2, 126, 127, 128, 253, 254]
    out = Buf(4 * n, torch.float32)
    b.mxfp8_dequantize(dev(q), dev(e8), n, out.t)
    torch.cuda.synchronize()
    want = oracle.mxfp8_dequant(q, e8)
    got = out.np()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


# ----------------------------------------------------------------------------- edge cases
def test_empty_and_invalid_calls_write_nothing():
    b = lib()
    e = torch.empty(0, dtype=torch.uint8, device="cuda")
    ts = Buf(4, torch.float32)
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    x0 = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    b.nvfp4_quantize_tile16(x0, ws, e, e, ts.t)
    torch.cuda.synchronize()
    assert ts.np()[0] == 1.0
    b.nvfp4_transpose_tile16(e, e, 0, 16, 16, e, e)
    b.mxfp8_sr_transpose_requant(e, e, e, 0, 32, 16, 2, 0, e, e)
    b.mxfp8_dequantize(e, e, 0, e)
    codes = Buf(16 * 48 // 2)
    with pytest.raises(b.Nvfp4Error) as err:
        b.mxfp8_sr_transpose_requant(codes.t, codes.t, ts.t, 1, 16, 48, 2, 0, codes.t, codes.t)  # rows % 32
    assert err.value.status == 3
    torch.cuda.synchronize()
    assert np.all(codes.np() == 0xAB)


# ----------------------------------------------------------------------------- expert stack, full size
def test_expert_stack_tile16_and_mxfp8_full_size():
    """128x512x2048 expert stack (seed 2), the launch configuration the bench
    times: tile quantize of experts 0, 1, 127 and the transpose of the whole
    stack against the oracle; MXFP8 SR transpose of the whole stack, experts
    0, 1 and 127 bit-exact, and every element within one E4M3 step of y."""
    b = lib()
    batch, rows, cols = syn.CFG2_SHAPE
    w = syn.cfg2()
    sample = [0, 1, batch - 1]
    # tile path: GPU quantize of every expert, oracle check on the sample
    n = rows * cols
    tc_all = np.zeros((batch, rows, cols // 2), np.uint8)
    tt_all = np.zeros((batch, rows // 16, cols // 16), np.uint8)
    for e in range(batch):
        gc, gt, gs = gpu_tile16(w[e])
        tc_all[e], tt_all[e] = gc, gt
        if e in sample:
            oc, ot, os_ = oracle.quantize_tile16(w[e])
            assert f32_bits(gs) == f32_bits(os_)
            assert_codes_equal(gt, ot, "expert %d tile scales" % e)
            assert_codes_equal(gc, oc, "expert %d tile codes" % e)
    ct, tt = gpu_transpose_tile16(tc_all, tt_all, batch, rows, cols)
    for e in sample:
        oc, ot = oracle.transpose_tile16(tc_all[e:e + 1], tt_all[e:e + 1], 1, rows, cols)
        assert_codes_equal(ct[e], oc[0], "expert %d transposed codes" % e)
        assert_codes_equal(tt[e], ot[0], "expert %d transposed tile scales" % e)
    # MXFP8 path from the oracle's 16-value RTN of every expert
    codes, scales, ts = _rtn_stack(w)
    gq, ge = gpu_mxfp8(codes, scales, ts, batch, rows, cols, syn.CFG2_SR_SEED, 0)

    def one(e):
        return oracle.mxfp8_sr_transpose_requant(codes[e:e + 1], scales[e:e + 1], ts[e:e + 1], 1, rows, cols,
                                                 syn.CFG2_SR_SEED, 0, first=e)
    with pool(len(sample)) as ex:
        outs = list(ex.map(one, sample))
    for e, (oq, oe) in zip(sample, outs):
        assert_codes_equal(ge[e], oe[0], "expert %d E8M0" % e)
        assert_codes_equal(gq[e], oq[0], "expert %d E4M3" % e)
    # every element: |dequant - y| <= one E4M3 step at its magnitude, or the
    # distance to 448 units where |y| / unit saturates (a property at any size)
    out = torch.empty(batch * n, dtype=torch.float32, device="cuda")
    b.mxfp8_dequantize(dev(gq), dev(ge), batch * n, out)
    yq = torch.empty(batch * n, dtype=torch.float32, device="cuda")
    for e in range(batch):
        b.nvfp4_dequantize(dev(codes[e]), dev(scales[e]), dev(ts[e:e + 1]), rows, cols, b.NVFP4_SCALES_BLOCK16,
                           yq[e * n:(e + 1) * n])
    y = yq.reshape(batch, rows, cols).transpose(1, 2).reshape(-1).double()
    d = (out.double() - y).abs()
    unit = torch.pow(2.0, dev(ge).double() - 127).repeat_interleave(32)
    step = torch.where(y.abs() / unit >= 2.0 ** -6, torch.pow(2.0, torch.floor(torch.log2(y.abs().clamp_min(1e-300)))) / 8,
                       unit * 2.0 ** -9)
    a = y.abs() / unit
    bound = torch.where(a >= 448, (a - 448) * unit, step)
    assert bool((d <= bound * (1 + 1e-12)).all())
