"""GPU parity of the KV-cache row-scale quantizers (one FP32 scale per
(token, head) row; TRACE explainer, hyper-parameter table): codes, block
scales, row scales, hints and guidance counters bit for bit against the oracle,
for every supported head_dim, input kinds with ragged row counts, and a cache
of 65536 tokens x 16 heads x 128 sampled in the launch configuration the bench
times."""
import numpy as np
import pytest
import torch

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import Buf, assert_codes_equal, dev_bf16, f32_bits, lib

pytestmark = pytest.mark.gpu


def gpu_rows(x, hint_bits=0):
    b = lib()
    xt = dev_bf16(x)
    rows, cols = xt.shape
    n = rows * cols
    codes, scales, rs = Buf(n // 2), Buf(n // 16), Buf(4 * rows, torch.float32)
    hints = Buf(n * hint_bits // 8) if hint_bits else None
    b.nvfp4_quantize_rtn_rows(xt, codes.t, scales.t, rs.t, hints.t if hints else None, hint_bits)
    torch.cuda.synchronize()
    return codes.np(), scales.np(), rs.np(), hints.np() if hints else None


def gpu_guided_rows(x, hints_np, hint_bits):
    b = lib()
    xt = dev_bf16(x)
    rows, cols = xt.shape
    n = rows * cols
    codes, scales, rs = Buf(n // 2), Buf(n // 16), Buf(4 * rows, torch.float32)
    hints = torch.from_numpy(np.ascontiguousarray(hints_np)).cuda() if hints_np is not None else None
    stats = torch.zeros(4, dtype=torch.int64, device="cuda")
    b.nvfp4_guided_requant_rows(xt, hints, hint_bits, codes.t, scales.t, rs.t, stats)
    torch.cuda.synchronize()
    return codes.np(), scales.np(), rs.np(), stats.cpu().numpy().astype(np.uint64)


def _check(got, want, label):
    gc, gs, gr = got[:3]
    oc, os_, orr = want[:3]
    assert np.array_equal(np.asarray(gr, np.float32).view(np.uint32), np.asarray(orr, np.float32).view(np.uint32)), label + " row scales"
    assert_codes_equal(gs.reshape(-1), os_.reshape(-1), label + " scales")
    assert_codes_equal(gc.reshape(-1), oc.reshape(-1), label + " codes")


@pytest.mark.parametrize("dim", [16, 32, 64, 128, 256, 512])
@pytest.mark.parametrize("kind", ["normal", "heavy", "tiny", "outlier", "zeros", "ties", "sparse"])
def test_rows_rtn_and_guided_match_oracle(dim, kind):
    rows = 37 * (32 // max(1, min(32, dim // 16))) + 5  # several warps and a ragged last group
    xt = syn.random_case((rows, dim), 8000 + dim, kind)
    xr = syn.rollout_copy(xt, np.random.default_rng(dim), 2.0 ** -6)
    for bits in (0, 1, 2, 4):
        g = gpu_rows(xr, bits)
        o = oracle.quantize_rtn_rows(xr, bits)
        _check(g, o, "rollout rows bits=%d" % bits)
        if bits:
            assert_codes_equal(g[3], o[3], "rows hints")
            gg = gpu_guided_rows(xt, o[3], bits)
            og = oracle.guided_requant_rows(xt, o[3], bits)
            _check(gg, og, "train rows bits=%d" % bits)
            assert list(gg[3][:3]) == list(og[3][:3])


def test_rows_without_hints_is_rtn():
    x = syn.random_case((64, 128), 8100, "normal")
    g = gpu_guided_rows(x, None, 2)
    o = oracle.quantize_rtn_rows(x)
    _check(g, o, "guided without hints")


def test_kv_cache_at_bench_size_sampled_rows():
    """65536 tokens x 16 heads x 128: the whole cache on the GPU (the bench's
    launch configuration), every 997th row and the last rows against the
    oracle (each row is its own tensor, so a row sample is exact)."""
    tokens, heads, dim = 65536, 16, 128
    rows = tokens * heads
    gen = torch.Generator(device="cuda").manual_seed(5)
    xt = (torch.randn((rows, dim), device="cuda", generator=gen) *
          torch.exp(torch.empty((1, dim), device="cuda").uniform_(np.log(0.1), np.log(10.0), generator=gen)))
    xt = xt.to(torch.bfloat16)
    xr = (xt.float() * (1 + torch.randn(xt.shape, device="cuda", generator=gen) * 2.0 ** -8)).to(torch.bfloat16)
    g = gpu_rows(xr, 2)
    gg = gpu_guided_rows(xt, g[3], 2)
    sample = np.concatenate([np.arange(0, rows, 997), np.arange(rows - 5, rows)])
    to_np = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    xr_s, xt_s = to_np(xr[torch.from_numpy(sample).cuda()]), to_np(xt[torch.from_numpy(sample).cuda()])
    o = oracle.quantize_rtn_rows(xr_s, 2)
    og = oracle.guided_requant_rows(xt_s, o[3], 2)
    hb = dim * 2 // 8
    pick = lambda a, per: a.reshape(rows, per)[sample]
    _check((pick(g[0], dim // 2), pick(g[1], dim // 16), g[2][sample]), o, "rollout sample")
    assert_codes_equal(pick(g[3], hb).reshape(-1), o[3], "hints sample")
    _check((pick(gg[0], dim // 2), pick(gg[1], dim // 16), gg[2][sample]), og, "train sample")
