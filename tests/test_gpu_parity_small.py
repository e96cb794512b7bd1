"""GPU parity on small and adversarial inputs: every CUDA kernel, through the C
ABI, against the CPU oracle, element by element.  Codes, scales, tensor scales,
hints and counters must match bit for bit; RHT outputs follow the tolerance
rule of the RHT tests below.  Sizes span several CTAs, ragged tails and the
degenerate cases (one block, all zeros, subnormal block scales, exact ties)."""
import numpy as np
import pytest
import torch

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import (Buf, assert_codes_equal, dev_bf16, f32_bits, gpu_emit_hint, gpu_guided,
                       gpu_guided_stats, gpu_rht, gpu_rtn, gpu_sr, gpu_stats, lib, rht_boundary_check)

pytestmark = pytest.mark.gpu

SHAPES = [(1, 16), (3, 48), (37, 528), (64, 1024), (257, 2080)]
KINDS = ["normal", "heavy", "tiny", "outlier", "zeros", "ties", "sparse"]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("kind", KINDS)
def test_rtn_matches_oracle(shape, kind):
    x = syn.random_case(shape, 1000 + shape[0], kind)
    for bits in (0, 1, 2, 4):
        g = gpu_rtn(x, bits)
        c, s, t, h = oracle.quantize_rtn(x, hint_bits=bits)
        assert f32_bits(g["ts"]) == f32_bits(t)
        assert_codes_equal(g["scales"], s, "scales")
        assert_codes_equal(g["codes"], c, "codes")
        if bits:
            assert_codes_equal(g["hints"], h, "hints")
        assert f32_bits(np.uint32(g["ws"][0]).view(np.float32)) == f32_bits(oracle.amax_bf16(x))


def test_amax_precomputed_flag_and_standalone_amax():
    b = lib()
    x = syn.random_case((128, 256), 5, "heavy")
    xt = dev_bf16(x)
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    b.nvfp4_tensor_amax(xt, ws)
    torch.cuda.synchronize()
    assert f32_bits(np.uint32(ws.cpu().numpy()[0]).view(np.float32)) == f32_bits(oracle.amax_bf16(x))
    g = gpu_rtn(x, 0, ws=ws, flags=b.NVFP4_AMAX_PRECOMPUTED)
    c, s, t, _ = oracle.quantize_rtn(x)
    assert_codes_equal(g["codes"], c)
    # a planted amax is used as given: scales follow A = 2 * true amax
    ws2 = torch.tensor([f32_bits(2 * oracle.amax_bf16(x)), 0, 0, 0, 0, 0, 0, 0], dtype=torch.int64).to(torch.int32).cuda()
    g2 = gpu_rtn(x, 0, ws=ws2, flags=b.NVFP4_AMAX_PRECOMPUTED)
    c2, s2, t2, _ = oracle.quantize_rtn(x, A=2 * oracle.amax_bf16(x))
    assert f32_bits(g2["ts"]) == f32_bits(t2)
    assert_codes_equal(g2["codes"], c2)


def test_amax_passes_in_a_row_leave_no_state_behind():
    """The amax pass publishes A from the CTA that finishes last, without a
    clearing launch: calls in a row on one scratch buffer must each give their
    own tensor's amax (a smaller one after a larger one, a non-finite one,
    then a finite one, an empty one), set the warning bit only when it applies,
    and leave the arrival counter and the running maximum (words 4 and 5) zero."""
    b = lib()
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    ws[2] = 12345  # a result left by another call: cleared by the amax pass
    big = syn.random_case((1024, 4096), 11, "outlier")          # many CTAs
    small = (syn.bf16_to_f32(syn.random_case((333, 64), 12, "normal")) * np.float32(1e-3))
    small = syn.bf16_bits(small)
    bad = syn.random_case((64, 256), 13, "normal").copy()
    bad[7, 9] = 0x7FC0  # a NaN pattern
    for x, warn in ((big, 0), (small, 0), (bad, 1), (small, 0)):
        b.nvfp4_tensor_amax(dev_bf16(x), ws)
        torch.cuda.synchronize()
        w = ws.cpu().numpy().view(np.uint32)
        if warn:
            assert w[0] >= 0x7F800000 and w[1] == b.NVFP4_WARN_NONFINITE
        else:
            assert f32_bits(np.uint32(w[0]).view(np.float32)) == f32_bits(oracle.amax_bf16(x))
            assert w[1] == 0
        assert w[2] == 0 and w[3] == 0
        assert not w[4:].any()
    b.nvfp4_tensor_amax(torch.empty(0, dtype=torch.bfloat16, device="cuda"), ws)
    torch.cuda.synchronize()
    assert not ws.cpu().numpy().any()


@pytest.mark.parametrize("shape", [(1, 16), (37, 528), (129, 2048)])
@pytest.mark.parametrize("noise", [2.0 ** -8, 2.0 ** -3, None])
def test_guided_matches_oracle(shape, noise):
    rng = np.random.default_rng(shape[0])
    xt = syn.random_case(shape, 2000 + shape[0], "heavy")
    xr = syn.rollout_copy(xt, rng, noise) if noise else syn.random_case(shape, 77, "heavy")
    for bits in (1, 2, 4):
        _, _, _, hints = oracle.quantize_rtn(xr, hint_bits=bits)
        g = gpu_guided(xt, hints, bits)
        c, s, t, st = oracle.guided_requant(xt, hints, bits)
        assert f32_bits(g["ts"]) == f32_bits(t)
        assert_codes_equal(g["scales"], s, "scales")
        assert_codes_equal(g["codes"], c, "guided codes")
        assert list(g["stats"][:3]) == list(st[:3])
    g = gpu_guided(xt, None, 2)
    c, s, t, _ = oracle.quantize_rtn(xt)
    assert_codes_equal(g["codes"], c)
    assert not g["stats"].any()


def test_guided_on_grid_values_ignore_hints():
    x = syn.random_case((32, 256), 3, "ties")
    rng = np.random.default_rng(1)
    for bits in (1, 2, 4):
        hints = rng.integers(0, 256, 32 * 256 * bits // 8).astype(np.uint8)
        g = gpu_guided(x, hints, bits)
        c, s, t, st = oracle.guided_requant(x, hints, bits)
        assert_codes_equal(g["codes"], c)
        assert list(g["stats"][:3]) == list(st[:3])


@pytest.mark.parametrize("shape", [(3, 48), (64, 1024)])
def test_guided_zeros_subnormals_adversarial_hints(shape):
    """Exact zeros (+0 and -0) sit on the grid and must ignore the hint; BF16
    subnormals are off the grid (bracket 0 / 0.5) and must follow it."""
    x = syn.random_case(shape, 11, "sparse")
    rng = np.random.default_rng(shape[0])
    n = x.size
    for bits in (1, 2, 4):
        hints = rng.integers(0, 256, (n * bits + 7) // 8).astype(np.uint8)
        g = gpu_guided(x, hints, bits)
        c, s, t, st = oracle.guided_requant(x, hints, bits)
        assert_codes_equal(g["scales"], s, "scales")
        assert_codes_equal(g["codes"], c, "guided codes")
        assert list(g["stats"][:3]) == list(st[:3])
        r = gpu_rtn(x, bits)
        oc, os_, ot, oh = oracle.quantize_rtn(x, hint_bits=bits)
        assert_codes_equal(r["codes"], oc, "rtn codes")


@pytest.mark.parametrize("n", [16, 48, 16 * 1001, 1 << 20])
def test_emit_hint_matches_oracle(n):
    rng = np.random.default_rng(n)
    codes = rng.integers(0, 256, n // 2).astype(np.uint8)
    for bits in (1, 2, 4):
        assert_codes_equal(gpu_emit_hint(codes, n, bits), oracle.emit_hint(codes, n, bits), "hints")


@pytest.mark.parametrize("shape", [(1, 16), (37, 528), (129, 2048), (300, 4096)])
@pytest.mark.parametrize("kind", ["normal", "heavy", "sparse", "ties", "outlier", "tiny"])
def test_guided_requant_stats_matches_guided_then_stats(shape, kind):
    """The fused train pass equals the guided re-quantization followed by the
    counters against the rollout tensor, bit for bit, for every hint width
    (none = round-to-nearest), with rollout tensors that are a noisy copy (few
    differing blocks), an unrelated tensor (most blocks differ) and the train
    side's own round-to-nearest result (equal tensor scales)."""
    rng = np.random.default_rng(shape[0] + len(kind))
    rows, cols = shape
    xt = syn.random_case(shape, 6000 + rows, kind)
    xr = syn.rollout_copy(xt, rng, 2.0 ** -8)
    other = syn.random_case(shape, 6100 + rows, "heavy")
    for bits in (0, 1, 2, 4):
        hb = bits if bits else 2
        ro = oracle.quantize_rtn(xr, hint_bits=bits)
        hints = ro[3] if bits else None
        gc, gs, gt, gst = oracle.guided_requant(xt, hints, hb)
        rollouts = [ro[:3], oracle.quantize_rtn(other)[:3]]
        if bits == 0:
            rollouts.append(oracle.quantize_rtn(xt)[:3])
        for roll in rollouts:
            g = gpu_guided_stats(xt, hints, hb, roll, stats8_init=[5, 0, 0, 0, 0, 0, 0, 77])
            assert f32_bits(g["ts"]) == f32_bits(gt)
            assert_codes_equal(g["scales"], gs, "scales")
            assert_codes_equal(g["codes"], gc, "guided codes")
            if bits:
                assert list(g["stats"][:3]) == list(gst[:3])
            else:
                assert not g["stats"].any()
            o = oracle.mismatch_stats(roll[0], roll[1], roll[2], gc, gs, gt, rows, cols)
            want = [int(o[0]) + 5] + [int(v) for v in o[1:7]] + [77]  # added to; word 7 untouched
            assert [int(v) for v in g["stats8"]] == want


@pytest.mark.parametrize("shape", [(1, 16), (37, 528), (200, 1024)])
def test_mismatch_stats_matches_oracle(shape):
    rng = np.random.default_rng(7)
    rows, cols = shape
    xt = syn.random_case(shape, 3000 + rows, "normal")
    xr = syn.rollout_copy(xt, rng, 2.0 ** -6)
    a = oracle.quantize_rtn(xr, hint_bits=2)
    b = oracle.guided_requant(xt, a[3], 2)
    r = oracle.quantize_rtn(xt)
    for (ca, sa, ta), (cb, sb, tb) in [((a[0], a[1], a[2]), (b[0], b[1], b[2])),
                                       ((a[0], a[1], a[2]), (r[0], r[1], r[2])),
                                       ((r[0], r[1], r[2]), (r[0], r[1], r[2])),
                                       ((a[0], a[1], a[2]), (a[0], a[1], np.float32(a[2]) * 3))]:
        g = gpu_stats(ca, sa, ta, cb, sb, tb, rows, cols)
        o = oracle.mismatch_stats(ca, sa, ta, cb, sb, tb, rows, cols)
        assert list(g[:7]) == list(o[:7])
        assert g[7] == 0


@pytest.mark.parametrize("ratio", [1.001, 1.0 + 2.0 ** -20, 0.75, 1.0])
def test_mismatch_stats_arbitrary_codes_and_scale_ratios(ratio):
    """Random code bytes and scale bytes (zero scales with nonzero codes, E4M3
    subnormal scales) under tensor-scale ratios that are far from every grid
    ratio (1.001), within 2^-17 of one (1 + 2^-20), exactly one (0.75), or
    equal (1.0): every path of the value counter, against the oracle."""
    rng = np.random.default_rng(int(ratio * 1e6))
    rows, cols = 96, 4096
    n = rows * cols
    ca = rng.integers(0, 256, n // 2).astype(np.uint8)
    cb = ca.copy()
    flip = rng.random(n // 2) < 0.3
    cb[flip] = rng.integers(0, 256, int(flip.sum())).astype(np.uint8)
    sa = rng.integers(0, 127, n // 16).astype(np.uint8)
    sa[rng.random(n // 16) < 0.05] = 0
    sa[rng.random(n // 16) < 0.05] = rng.integers(1, 8)  # subnormal scales
    sb = sa.copy()
    move = rng.random(n // 16) < 0.2
    sb[move] = rng.integers(0, 127, int(move.sum())).astype(np.uint8)
    ta = np.float32(0.0123)
    tb = np.float32(ta * np.float32(ratio))
    g = gpu_stats(ca, sa, ta, cb, sb, tb, rows, cols)
    o = oracle.mismatch_stats(ca, sa, ta, cb, sb, tb, rows, cols)
    assert list(g[:7]) == list(o[:7])


def _rtn_stack(w):
    batch = w.shape[0]
    outs = [oracle.quantize_rtn(w[e]) for e in range(batch)]
    return (np.stack([o[0] for o in outs]), np.stack([o[1] for o in outs]),
            np.array([o[2] for o in outs], np.float32))


@pytest.mark.parametrize("shape", [(1, 16, 16), (3, 32, 48), (2, 80, 208), (2, 128, 64)])
@pytest.mark.parametrize("kind", ["normal", "heavy", "tiny", "zeros"])
def test_sr_transpose_matches_oracle(shape, kind):
    w = syn.random_case(shape, 4000 + shape[1], kind)
    batch, rows, cols = shape
    codes, scales, ts = _rtn_stack(w)
    for seed, draw in ((2, 0), (2, 1), ((5 << 32) | 17, 123456)):
        ct, st, tst = gpu_sr(codes, scales, ts, batch, rows, cols, seed, draw)
        oc, osc, ots = oracle.sr_transpose_requant(codes, scales, ts, batch, rows, cols, seed, draw)
        assert [f32_bits(v) for v in tst] == [f32_bits(v) for v in ots]
        assert_codes_equal(st, osc, "transposed scales")
        assert_codes_equal(ct, oc, "transposed SR codes")


def _rht_check(x, seed):
    g = gpu_rht(x, seed)
    rows, cols = x.shape
    # 1) the GPU transform is within 1e-6 * ||x_group||_2 of the double-precision one
    yd = oracle.rht32_f64(x, seed)
    xg = syn.bf16_to_f32(x).astype(np.float64).reshape(-1, 32)
    norm = np.linalg.norm(xg, axis=1)
    err = np.abs(g["y"].astype(np.float64).reshape(-1, 32) - yd.reshape(-1, 32))
    assert np.all(err <= 1e-6 * norm[:, None] + 1e-45)
    # 2) quantization of the GPU's own y is bit-exact
    c, s, t = oracle.quantize_f32(g["y"])
    assert f32_bits(g["ts"]) == f32_bits(t)
    assert_codes_equal(g["scales"], s, "rht scales")
    assert_codes_equal(g["codes"], c, "rht codes")
    # 3) against the full oracle, codes may differ only where the oracle's value
    #    is within the transform tolerance (propagated to the scaled domain) of
    #    a rounding boundary: an E4M3 midpoint for the block scale, an E2M1
    #    midpoint for the code.
    oc, osc, ot, oy = oracle.rht_quantize(x, seed)
    rht_boundary_check(x, yd, oc, osc, ot, g["codes"], g["scales"], g["ts"])
    return g


@pytest.mark.parametrize("shape", [(1, 32), (5, 96), (64, 1024), (131, 2048)])
@pytest.mark.parametrize("kind", ["normal", "outlier", "heavy", "zeros"])
def test_rht_matches_oracle(shape, kind):
    _rht_check(syn.random_case(shape, 5000 + shape[0], kind), 3)


def test_rht_without_y_out_gives_same_codes():
    x = syn.random_case((64, 512), 9, "heavy")
    a = gpu_rht(x, 11, want_y=True)
    b = gpu_rht(x, 11, want_y=False)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])


# ----------------------------------------------------------------- edge cases
def test_empty_tensors():
    b = lib()
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    ts = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    e = torch.empty(0, dtype=torch.uint8, device="cuda")
    b.nvfp4_quantize_rtn(x, ws, e, e, ts, None, 0)
    torch.cuda.synchronize()
    assert ts.item() == 1.0
    ts.zero_()
    b.nvfp4_guided_requant(x, None, 2, ws, e, e, ts)
    torch.cuda.synchronize()
    assert ts.item() == 1.0
    stats = torch.zeros(8, dtype=torch.int64, device="cuda")
    b.nvfp4_mismatch_stats(e, e, ts, e, e, ts, 0, 64, stats)
    b.nvfp4_emit_hint(e, 0, 2, e)
    torch.cuda.synchronize()
    assert not stats.any()


def test_invalid_arguments_write_nothing():
    b = lib()
    x = dev_bf16(syn.random_case((4, 64), 1, "normal"))
    codes = Buf(128)
    scales = Buf(16)
    ts = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    raw = torch.zeros(4 * 64 + 16, dtype=torch.int16, device="cuda")
    x_mis = raw[8:8 + 256].view(torch.bfloat16).view(4, 64)  # 16-byte aligned, not 32
    cases = [
        (lambda: b.nvfp4_quantize_rtn(x_mis, ws, codes.t, scales.t, ts), 2),
        (lambda: b.nvfp4_quantize_rtn(x, ws, codes.t[1:], scales.t, ts), 2),
        (lambda: b.nvfp4_quantize_rtn(x, ws, codes.t, scales.t, ts, codes.t, 3), 5),
        (lambda: b.nvfp4_quantize_rtn(x, ws, codes.t, scales.t, ts, flags=8), 1),
        (lambda: b.nvfp4_quantize_rtn(x[:, :40].contiguous(), ws, codes.t, scales.t, ts), 3),
        (lambda: b.nvfp4_rht_quantize(x[:, :48].contiguous(), 1, ws, codes.t, scales.t, ts), 3),
        (lambda: b.nvfp4_emit_hint(codes.t, 20, 2, scales.t), 3),
    ]
    for fn, status in cases:
        with pytest.raises(b.Nvfp4Error) as ei:
            fn()
        assert ei.value.status == status
    torch.cuda.synchronize()
    assert np.all(codes.np() == 0xAB) and np.all(scales.np() == 0xAB) and ts.item() == 0.0


def test_nonfinite_input_sets_warning_without_fault():
    x = syn.random_case((8, 64), 2, "normal").copy()
    x[3, 5] = 0x7F80  # +inf
    x[6, 7] = 0x7FC1  # NaN
    g = gpu_rtn(x, 2)
    assert g["ws"][1] & 1
    ok = syn.random_case((8, 64), 2, "normal")
    assert gpu_rtn(ok, 2)["ws"][1] == 0


def test_subnormal_tensor_scales_every_path():
    """Inputs so small that the tensor (or row) scale is an FP32 subnormal and
    1 / (sb * s_t) overflows to +inf: RTN, hints, guided, the KV rows, the
    tile quantizer, RHT and SR must all give the oracle's codes (nonzero ->
    saturated, zero -> +-0)."""
    b = lib()
    rng = np.random.default_rng(22)
    xf = (rng.standard_normal((64, 256)) * 1e-39).astype(np.float32)
    xf[rng.random(xf.shape) < 0.3] = 0.0
    xf[1, :3] = [-0.0, 0.0, 1e-40]
    x = syn.bf16_bits(xf)
    g = gpu_rtn(x, 2)
    oc, os_, ot, oh = oracle.quantize_rtn(x, hint_bits=2)
    assert f32_bits(g["ts"]) == f32_bits(ot) and 0 < ot < 2.0 ** -126
    assert_codes_equal(g["scales"], os_, "scales")
    assert_codes_equal(g["codes"], oc, "codes")
    assert_codes_equal(g["hints"], oh, "hints")
    gg = gpu_guided(x, oh, 2)
    gc, gs, gt, gst = oracle.guided_requant(x, oh, 2)
    assert_codes_equal(gg["codes"], gc, "guided codes")
    assert list(gg["stats"][:3]) == list(gst[:3])
    # KV rows: every row its own tensor, each with a subnormal scale
    xt = dev_bf16(x)
    rows, cols = x.shape
    codes, scales, rs = Buf(rows * cols // 2), Buf(rows * cols // 16), Buf(4 * rows, torch.float32)
    b.nvfp4_quantize_rtn_rows(xt, codes.t, scales.t, rs.t)
    torch.cuda.synchronize()
    rc, rsc, rr, _ = oracle.quantize_rtn_rows(x)
    assert_codes_equal(codes.np(), rc.reshape(-1), "row codes")
    # tile quantizer
    tcodes, tsc, tts = Buf(rows * cols // 2), Buf(rows * cols // 256), Buf(4, torch.float32)
    b.nvfp4_quantize_tile16(xt, torch.zeros(8, dtype=torch.int32, device="cuda"), tcodes.t, tsc.t, tts.t)
    torch.cuda.synchronize()
    tc, tt, tst = oracle.quantize_tile16(x)
    assert_codes_equal(tcodes.np(), tc.reshape(-1), "tile codes")
    # RHT: the transform of tiny inputs stays tiny
    gr = gpu_rht(x, 3)
    qc, qs, qt = oracle.quantize_f32(gr["y"])
    assert_codes_equal(gr["codes"], qc, "rht codes")
    # SR transpose with a subnormal tensor scale on the input stack
    w = syn.random_case((2, 32, 64), 23, "normal")
    codes2, scales2, ts2 = _rtn_stack(w)
    ts2 = np.array([1e-44, 2e-45], np.float32)
    ct, st, tst2 = gpu_sr(codes2, scales2, ts2, 2, 32, 64, 2, 0)
    oc2, osc2, ots2 = oracle.sr_transpose_requant(codes2, scales2, ts2, 2, 32, 64, 2, 0)
    assert_codes_equal(st, osc2, "sr scales")
    assert_codes_equal(ct, oc2, "sr codes")
