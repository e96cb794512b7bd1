"""The row-sharded helpers through the real C ABI on one GPU (a group of one:
no collective runs): the precomputed-amax path they use gives the oracle's
codes, scales, hints, guidance and mismatch counters bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import dev_bf16, lib

pytestmark = pytest.mark.gpu


def test_sharded_helpers_on_one_rank_match_the_oracle():
    from train_rollout_alignment_b200 import sharded
    b = lib()
    rows, cols = 192, 512
    x = syn.random_case((rows, cols), 12, "heavy")
    xr = syn.bf16_bits(syn.bf16_to_f32(x) * np.float32(1.0 + 2.0 ** -7))
    cr, sr, tr, ws, h = b.empty_nvfp4(rows, cols, "cuda", hint_bits=2)
    sharded.quantize_rtn(dev_bf16(xr), ws, cr, sr, tr, h, 2)
    ct, st, tt, ws2, _ = b.empty_nvfp4(rows, cols, "cuda")
    s4 = torch.zeros(4, dtype=torch.int64, device="cuda")
    sharded.guided_requant(dev_bf16(x), h, 2, ws2, ct, st, tt, s4)
    s8 = torch.zeros(8, dtype=torch.int64, device="cuda")
    sharded.mismatch_stats(cr, sr, tr, ct, st, tt, rows, cols, s8)
    torch.cuda.synchronize()
    oc, os_, ot, oh = oracle.quantize_rtn(xr, hint_bits=2)
    gc, gs, gt, gst = oracle.guided_requant(x, oh, 2)
    ost = oracle.mismatch_stats(oc, os_, ot, gc, gs, gt, rows, cols)
    assert np.array_equal(cr.cpu().numpy(), oc) and np.array_equal(sr.cpu().numpy(), os_)
    assert np.array_equal(h.cpu().numpy(), oh) and float(tr.item()) == ot
    assert np.array_equal(ct.cpu().numpy(), gc) and np.array_equal(st.cpu().numpy(), gs)
    assert list(s4.cpu().numpy()[:3].astype(np.uint64)) == list(gst[:3])
    assert list(s8.cpu().numpy()[:7].astype(np.uint64)) == list(ost[:7])
