"""GPU parity on the five synthetic workloads at their full sizes.

* single 1024x2048 tensor: the whole rollout -> hint -> guided -> counters
  pipeline, every output bit-exact, the fused train pass included;
* 24-layer MoE activation stack (8192x2048, Student-t): every layer bit-exact,
  hints on layers 12..23;
* 128x512x2048 expert stack: SR transpose of draw 0 bit-exact on all experts,
  draws 0..1023 bit-exact on experts 0..1, and the mean of 1024 GPU draws
  unbiased (Hoeffding bound per element, z-score overall and per p-bucket);
* 16384x4096 activation with outliers: RHT + quantize, every element under
  the RHT tolerance rule (differences only at rounding boundaries);
* 48-layer 65536x4096 throughput stack, in the launch configuration the bench
  times: every layer bit-exact over every row (codes, scales, hints, both
  counter sets), sampled rows of every layer against the oracle (which gets
  the full layer's amax), the fused counters equal to the standalone
  kernel's on every layer.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import (assert_codes_equal, dev_bf16, f32_bits, gpu_guided, gpu_guided_stats, gpu_rht, gpu_rtn,
                       gpu_sr, gpu_stats, lib, oracle_guided_parallel, oracle_rtn_parallel, pool,
                       oracle_stats_parallel, amax_parallel, rht_boundary_check, to_u16)

pytestmark = pytest.mark.gpu


def _pipeline_check(xt, xr, bits, label):
    rows, cols = xt.shape
    A_r, A_t = oracle.amax_bf16(xr), oracle.amax_bf16(xt)
    gr = gpu_rtn(xr, bits)
    oc, os_, ot, oh = oracle_rtn_parallel(xr, A_r, bits)
    assert f32_bits(gr["ts"]) == f32_bits(ot)
    assert_codes_equal(gr["scales"], os_, label + " rollout scales")
    assert_codes_equal(gr["codes"], oc, label + " rollout codes")
    if bits:
        assert_codes_equal(gr["hints"], oh, label + " hints")
    gg = gpu_guided(xt, gr["hints"] if bits else None, bits if bits else 2)
    gc, gs, gt, gst = oracle_guided_parallel(xt, oh, bits if bits else 2, A_t)
    assert f32_bits(gg["ts"]) == f32_bits(gt)
    assert_codes_equal(gg["scales"], gs, label + " train scales")
    assert_codes_equal(gg["codes"], gc, label + " guided codes")
    assert list(gg["stats"][:3]) == list(gst[:3])
    s_gpu = gpu_stats(gr["codes"], gr["scales"], gr["ts"], gg["codes"], gg["scales"], gg["ts"], rows, cols)
    s_or = oracle.mismatch_stats(oc, os_, ot, gc, gs, gt, rows, cols)
    assert list(s_gpu[:7]) == list(s_or[:7])
    # the fused train pass (guided + counters against the rollout tensor)
    gf = gpu_guided_stats(xt, gr["hints"] if bits else None, bits if bits else 2,
                          (gr["codes"], gr["scales"], gr["ts"]))
    assert_codes_equal(gf["codes"], gc, label + " fused guided codes")
    assert_codes_equal(gf["scales"], gs, label + " fused train scales")
    assert list(gf["stats"][:3]) == (list(gst[:3]) if bits else [0, 0, 0])
    assert list(gf["stats8"][:7]) == list(s_or[:7])
    return s_or


def test_single_tensor_pipeline_all_hint_widths():
    xt, xr = syn.cfg0()
    rows, cols = xt.shape
    rtn = oracle.quantize_rtn(xt)
    ro = oracle.quantize_rtn(xr)
    base = oracle.mismatch_stats(ro[0], ro[1], ro[2], rtn[0], rtn[1], rtn[2], rows, cols)
    g = gpu_stats(ro[0], ro[1], ro[2], rtn[0], rtn[1], rtn[2], rows, cols)
    assert list(g[:7]) == list(base[:7])
    for bits in (2, 1, 4):
        st = _pipeline_check(xt, xr, bits, "cfg0/%d-bit" % bits)
        assert st[1] < base[1]  # guidance removes mismatches
        print("single tensor, %d-bit hints: code mismatches %d -> %d (RTN vs RTN %d adjacent / %d far)"
              % (bits, base[1], st[1], base[2], base[3]))


def test_moe_activation_stack_24_layers():
    L, rows, cols = syn.CFG1_LAYERS, *syn.CFG1_SHAPE
    total_before = total_after = 0
    for layer in range(L):
        xt, xr = syn.cfg1_layer(layer)
        bits = 2 if layer >= syn.CFG1_HINT_FROM else 0
        st = _pipeline_check(xt, xr, bits, "cfg1 layer %d" % layer)
        if bits:
            total_after += int(st[1])
    print("MoE stack, back-half layers: code mismatches after guidance %d" % total_after)


def _rtn_stack_parallel(w):
    batch = w.shape[0]
    with pool(batch) as ex:
        outs = list(ex.map(lambda e: oracle.quantize_rtn(w[e]), range(batch)))
    return (np.stack([o[0] for o in outs]), np.stack([o[1] for o in outs]),
            np.array([o[2] for o in outs], np.float32))


def _oracle_sr_parallel(codes, scales, ts, rows, cols, seed, draw, experts):
    def one(e):
        return oracle.sr_transpose_requant(codes[e:e + 1], scales[e:e + 1], ts[e:e + 1], 1, rows, cols,
                                           seed, draw, first=e)
    with pool(len(experts)) as ex:
        return list(ex.map(one, experts))


def _dequant_torch(codes, scales, ts, shape):
    """Test-side decode of NVFP4 on the GPU (torch ops): [batch, r, c] FP32."""
    grid = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6],
                        dtype=torch.float32, device=codes.device)
    b, r, c = shape
    nib = torch.stack([codes & 15, codes >> 4], dim=-1).reshape(b, r, c).long()
    e4 = torch.tensor([oracle.e4m3_value(k) for k in range(256)], dtype=torch.float32,
                      device=codes.device)
    sb = e4[scales.long()].reshape(b, r, c // 16).repeat_interleave(16, dim=2)
    return (grid[nib] * sb) * ts.reshape(b, 1, 1)


def test_expert_stack_sr_transpose():
    batch, rows, cols = syn.CFG2_SHAPE
    w = syn.cfg2()
    codes, scales, ts = _rtn_stack_parallel(w)
    seed = syn.CFG2_SR_SEED
    # draw 0: every expert bit-exact
    ct, st, tst = gpu_sr(codes, scales, ts, batch, rows, cols, seed, 0)
    outs = _oracle_sr_parallel(codes, scales, ts, rows, cols, seed, 0, list(range(batch)))
    for e, (oc, osc, ots) in enumerate(outs):
        assert f32_bits(tst[e]) == f32_bits(ots[0])
        assert_codes_equal(st[e], osc[0], "expert %d scales" % e)
        assert_codes_equal(ct[e], oc[0], "expert %d SR codes" % e)
    # draws 1..1023 on experts 0 and 1 (the whole stack launched each time,
    # so the counters are those of the full launch), in batches of draws
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    c_in, s_in, t_in = dev(codes), dev(scales), dev(np.asarray(ts, np.float32))
    n = batch * rows * cols
    ct_d = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    st_d = torch.empty(n // 16, dtype=torch.uint8, device="cuda")
    tst_d = torch.empty(batch, dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(batch, 8), dtype=torch.int32, device="cuda")
    per_e = rows * cols // 2
    b = lib()
    for d0 in range(1, 1024, 64):
        draws = list(range(d0, min(1024, d0 + 64)))
        got = {}
        for draw in draws:
            b.nvfp4_sr_transpose_requant(c_in, s_in, t_in, batch, rows, cols, seed, draw, ws, ct_d, st_d, tst_d)
            got[draw] = ct_d[:2 * per_e].cpu().numpy().reshape(2, cols, rows // 2)
        tasks = [(draw, e) for draw in draws for e in (0, 1)]
        with pool(len(tasks)) as ex:
            outs = list(ex.map(lambda t: oracle.sr_transpose_requant(
                codes[t[1]:t[1] + 1], scales[t[1]:t[1] + 1], ts[t[1]:t[1] + 1], 1, rows, cols, seed, t[0],
                first=t[1])[0], tasks))
        for (draw, e), oc in zip(tasks, outs):
            assert_codes_equal(got[draw][e], oc[0], "draw %d expert %d" % (draw, e))


def test_expert_stack_sr_mean_of_1024_draws_is_unbiased():
    b = lib()
    batch, rows, cols = syn.CFG2_SHAPE
    w = syn.cfg2()
    codes, scales, ts = _rtn_stack_parallel(w)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    c_in, s_in, t_in = dev(codes), dev(scales), dev(ts)
    n = batch * rows * cols
    ct = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    st = torch.empty(n // 16, dtype=torch.uint8, device="cuda")
    tst = torch.empty(batch, dtype=torch.float32, device="cuda")
    ws = torch.zeros(batch, dtype=torch.int32, device="cuda")
    draws = 1024
    acc = torch.zeros((batch, cols, rows), dtype=torch.float64, device="cuda")
    for d in range(draws):
        b.nvfp4_sr_transpose_requant(c_in, s_in, t_in, batch, rows, cols, syn.CFG2_SR_SEED, d, ws, ct, st, tst)
        acc += _dequant_torch(ct, st, tst, (batch, cols, rows))
    mean = acc / draws
    y = _dequant_torch(c_in, s_in, t_in, (batch, rows, cols)).transpose(1, 2).double()
    e4 = torch.tensor([oracle.e4m3_value(k) for k in range(256)], dtype=torch.float64, device="cuda")
    scale = e4[st.long()].reshape(batch, cols, rows // 16).repeat_interleave(16, dim=2) * tst.double().reshape(batch, 1, 1)
    grid = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=torch.float64, device="cuda")
    a = torch.where(scale > 0, y.abs() / torch.where(scale > 0, scale, 1), torch.zeros_like(y))
    lo = (torch.bucketize(a, grid, right=True) - 1).clamp(0, 6)
    width = grid[lo + 1] - grid[lo]
    p = ((a - grid[lo]) / width).clamp(0, 1)
    sat = a >= 6
    p = torch.where(sat, torch.zeros_like(p), p)
    expect = torch.where(sat, torch.sign(y) * 6 * scale, y)
    dev_units = (mean - expect) / torch.where(scale > 0, scale * width, torch.ones_like(scale))
    # per element: Hoeffding, P(|mean - p| > t) <= 2 exp(-2 n t^2); t for 1e-12
    t = float(np.sqrt(np.log(2 / 1e-12) / (2 * draws)))
    assert dev_units.abs().max().item() <= t + 1e-6
    var = (p * (1 - p) / draws)
    z = dev_units.sum() / var.sum().sqrt()
    assert abs(z.item()) < 5, z.item()
    for lo_p, hi_p in ((0, .1), (.1, .3), (.3, .7), (.7, .9), (.9, 1.0)):
        m = (p > lo_p) & (p <= hi_p)
        zb = dev_units[m].sum() / var[m].sum().sqrt()
        assert abs(zb.item()) < 5, (lo_p, hi_p, zb.item())
    print("SR 1024 draws: overall z %.2f, max per-element deviation %.4f cells" % (z.item(), dev_units.abs().max().item()))


def test_activation_rht_quantize():
    x = syn.cfg3()
    rows, cols = x.shape
    seed = syn.CFG3_SIGN_SEED
    g = gpu_rht(x, seed)
    step = 512
    with pool(rows // step) as ex:
        yd = np.concatenate(list(ex.map(lambda r: oracle.rht32_f64(x[r:r + step], seed), range(0, rows, step))))
    xg = syn.bf16_to_f32(x).astype(np.float64).reshape(-1, 32)
    norm = np.linalg.norm(xg, axis=1)
    err = np.abs(g["y"].astype(np.float64).reshape(-1, 32) - yd.reshape(-1, 32))
    assert np.all(err <= 1e-6 * norm[:, None])
    # quantization of the GPU's own y: bit-exact
    Ag = oracle.amax_f32(g["y"])
    with pool(rows // step) as ex:
        outs = list(ex.map(lambda r: oracle.quantize_f32(g["y"][r:r + step], Ag), range(0, rows, step)))
    assert f32_bits(g["ts"]) == f32_bits(outs[0][2])
    assert_codes_equal(g["scales"], np.concatenate([o[1] for o in outs]), "rht scales")
    assert_codes_equal(g["codes"], np.concatenate([o[0] for o in outs]), "rht codes")
    # full oracle (double transform): codes and scales may differ only next to
    # a rounding boundary (the RHT tolerance rule, applied to every element)
    oy = yd.astype(np.float32)
    Ao = oracle.amax_f32(oy)
    with pool(rows // step) as ex:
        oo = list(ex.map(lambda r: oracle.quantize_f32(oy[r:r + step], Ao), range(0, rows, step)))
    oc = np.concatenate([o[0] for o in oo])
    ot = oo[0][2]
    n_blk = n_code = 0
    for r in range(0, rows, step):
        nb, nc = rht_boundary_check(x[r:r + step], yd[r:r + step], oo[r // step][0], oo[r // step][1], ot,
                                    g["codes"][r:r + step], g["scales"][r:r + step], g["ts"])
        n_blk += nb
        n_code += nc
    agree = np.mean(oracle.unpack_codes(oc) == oracle.unpack_codes(g["codes"]))
    # reported: RHT vs plain quantization error (per element MSE, in the domain it was quantized in)
    osc = np.concatenate([o[1] for o in oo])
    dq = oracle.dequant(oc, osc, oo[0][2], x.size)
    mse_rht = float(np.mean((dq.astype(np.float64) - yd.reshape(-1)) ** 2))
    pc, ps, pt, _ = oracle_rtn_parallel(x, oracle.amax_bf16(x))
    dqp = oracle.dequant(pc, ps, pt, x.size)
    mse_plain = float(np.mean((dqp.astype(np.float64) - xg.reshape(-1)) ** 2))
    print("RHT32: code agreement with the double-precision oracle %.7f (%d scales and %d codes differ, all "
          "at rounding boundaries); MSE rht %.4g vs plain %.4g" % (agree, n_blk, n_code, mse_rht, mse_plain))


def test_throughput_stack_sampled_rows_every_layer():
    b = lib()
    L, (rows, cols) = syn.CFG4_LAYERS, syn.CFG4_SHAPE
    n = rows * cols
    rng = np.random.default_rng(4)
    dev = "cuda"
    codes_r = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales_r = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    codes_t = torch.empty_like(codes_r)
    scales_t = torch.empty_like(scales_r)
    ts_r = torch.empty(1, dtype=torch.float32, device=dev)
    ts_t = torch.empty(1, dtype=torch.float32, device=dev)
    ws_r = torch.zeros(8, dtype=torch.int32, device=dev)
    ws_t = torch.zeros(8, dtype=torch.int32, device=dev)
    hints = torch.empty(n * 2 // 8, dtype=torch.uint8, device=dev)
    for layer in range(L):
        xt_d, xr_d = syn.cfg4_layer_device(layer, dev)
        bits = 2 if layer >= syn.CFG4_HINT_FROM else 0
        h = hints if bits else None
        stats4 = torch.zeros(4, dtype=torch.int64, device=dev)
        stats8 = torch.zeros(8, dtype=torch.int64, device=dev)
        stats8_sep = torch.zeros(8, dtype=torch.int64, device=dev)
        b.nvfp4_tensor_amax(xr_d, ws_r)
        b.nvfp4_quantize_rtn(xr_d, ws_r, codes_r, scales_r, ts_r, h, bits, flags=b.NVFP4_AMAX_PRECOMPUTED)
        b.nvfp4_tensor_amax(xt_d, ws_t)
        b.nvfp4_guided_requant_stats(xt_d, h, 2, ws_t, codes_t, scales_t, ts_t, stats4, codes_r, scales_r,
                                     ts_r, stats8, flags=b.NVFP4_AMAX_PRECOMPUTED)
        b.nvfp4_mismatch_stats(codes_r, scales_r, ts_r, codes_t, scales_t, ts_t, rows, cols, stats8_sep)
        torch.cuda.synchronize()
        assert torch.equal(stats8, stats8_sep)  # fused counters == the standalone kernel's
        sel = np.unique(np.concatenate([[0, rows - 1], rng.choice(rows, 30, replace=False)]))
        sel_t = torch.from_numpy(sel).to(dev)
        xr, xt = to_u16(xr_d), to_u16(xt_d)
        with pool(16) as ex:
            A_r = max(ex.map(oracle.amax_bf16, np.array_split(xr, 16)))
            A_t = max(ex.map(oracle.amax_bf16, np.array_split(xt, 16)))
        xr_s, xt_s = xr[sel], xt[sel]
        oc, os_, ot, oh = oracle.quantize_rtn(xr_s, A_r, bits)
        assert f32_bits(ts_r.item()) == f32_bits(ot)
        assert_codes_equal(codes_r[sel_t].cpu().numpy(), oc, "layer %d rollout codes" % layer)
        assert_codes_equal(scales_r[sel_t].cpu().numpy(), os_, "layer %d rollout scales" % layer)
        hrow = cols * 2 // 8
        h_sel = None
        if bits:
            h_gpu = hints.cpu().numpy().reshape(rows, hrow)[sel]
            assert_codes_equal(h_gpu, oh.reshape(len(sel), hrow), "layer %d hints" % layer)
            h_sel = oh
        gc, gs, gt, gst = oracle.guided_requant(xt_s, h_sel, 2, A_t)
        assert f32_bits(ts_t.item()) == f32_bits(gt)
        assert_codes_equal(codes_t[sel_t].cpu().numpy(), gc, "layer %d train codes" % layer)
        assert_codes_equal(scales_t[sel_t].cpu().numpy(), gs, "layer %d train scales" % layer)
        s8 = stats8.cpu().numpy()
        s4 = stats4.cpu().numpy()
        assert s8[0] == n and s8[1] == s8[2] + s8[3] and s8[4] >= s8[1] and s8[7] == 0
        assert s4[0] >= s4[1] + s4[2]
        if not bits:
            assert not s4.any()
        # counters on the sampled rows: GPU kernel on GPU outputs == oracle on oracle outputs
        so = oracle.mismatch_stats(oc, os_, ot, gc, gs, gt, len(sel), cols)
        sg = gpu_stats(codes_r[sel_t].cpu().numpy(), scales_r[sel_t].cpu().numpy(), ts_r.item(),
                       codes_t[sel_t].cpu().numpy(), scales_t[sel_t].cpu().numpy(), ts_t.item(), len(sel), cols)
        assert list(sg[:7]) == list(so[:7])
        del xt_d, xr_d


# Every layer of the stack (about 5 s each on a 16-core host);
# NVFP4_PARITY_QUICK=1 keeps the first and last layer of each half.
_FULL_LAYERS = ([0, 23, 24, 47] if os.environ.get("NVFP4_PARITY_QUICK") == "1"
                else list(range(syn.CFG4_LAYERS)))


@pytest.mark.parametrize("layer", _FULL_LAYERS)
def test_throughput_stack_full_layer(layer):
    """Whole layers of the 48-layer stack against the oracle over every row:
    codes, scales, tensor scales, hints, the guidance counters and the
    mismatch counters, all bit-exact, in the launch configuration the bench
    times (amax pass, then the quantizers with the amax precomputed, the
    train side fused with its counters); the standalone counter kernel must
    agree too."""
    b = lib()
    rows, cols = syn.CFG4_SHAPE
    n = rows * cols
    dev = "cuda"
    bits = 2 if layer >= syn.CFG4_HINT_FROM else 0
    xt_d, xr_d = syn.cfg4_layer_device(layer, dev)
    codes_r, scales_r, ts_r, ws_r, _ = b.empty_nvfp4(rows, cols, dev)
    codes_t, scales_t, ts_t, ws_t, _ = b.empty_nvfp4(rows, cols, dev)
    hints = torch.empty(n * 2 // 8, dtype=torch.uint8, device=dev) if bits else None
    stats4 = torch.zeros(4, dtype=torch.int64, device=dev)
    stats8 = torch.zeros(8, dtype=torch.int64, device=dev)
    b.nvfp4_tensor_amax(xr_d, ws_r)
    b.nvfp4_quantize_rtn(xr_d, ws_r, codes_r, scales_r, ts_r, hints, bits, flags=b.NVFP4_AMAX_PRECOMPUTED)
    b.nvfp4_tensor_amax(xt_d, ws_t)
    b.nvfp4_guided_requant_stats(xt_d, hints, 2, ws_t, codes_t, scales_t, ts_t, stats4, codes_r, scales_r, ts_r,
                                 stats8, flags=b.NVFP4_AMAX_PRECOMPUTED)
    stats8_sep = torch.zeros(8, dtype=torch.int64, device=dev)
    b.nvfp4_mismatch_stats(codes_r, scales_r, ts_r, codes_t, scales_t, ts_t, rows, cols, stats8_sep)
    torch.cuda.synchronize()
    assert torch.equal(stats8, stats8_sep)
    xr, xt = to_u16(xr_d), to_u16(xt_d)
    del xt_d, xr_d
    A_r, A_t = amax_parallel(xr), amax_parallel(xt)
    oc, os_, ot, oh = oracle_rtn_parallel(xr, A_r, bits)
    assert f32_bits(ts_r.item()) == f32_bits(ot)
    assert_codes_equal(codes_r.cpu().numpy(), oc, "layer %d rollout codes" % layer)
    assert_codes_equal(scales_r.cpu().numpy(), os_, "layer %d rollout scales" % layer)
    if bits:
        assert_codes_equal(hints.cpu().numpy(), oh, "layer %d hints" % layer)
    gc, gs, gt, gst = oracle_guided_parallel(xt, oh, 2, A_t)
    assert f32_bits(ts_t.item()) == f32_bits(gt)
    assert_codes_equal(codes_t.cpu().numpy(), gc, "layer %d train codes" % layer)
    assert_codes_equal(scales_t.cpu().numpy(), gs, "layer %d train scales" % layer)
    assert list(stats4.cpu().numpy()[:3].astype(np.uint64)) == list(gst[:3])
    so = oracle_stats_parallel(oc, os_, ot, gc, gs, gt, rows, cols)
    assert list(stats8.cpu().numpy()[:7].astype(np.uint64)) == list(so[:7])
    print("layer %d: %d code mismatches (%d adjacent, %d far), %d scale mismatches, guidance consulted %d, "
          "changed %d" % (layer, so[1], so[2], so[3], so[5], gst[0], gst[1]))
