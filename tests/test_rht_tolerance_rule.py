"""The checker behind the RHT parity tests, exercised on the CPU with the
oracle on both sides (no GPU): with nothing changed it finds no difference;
a code or a block scale changed away from a rounding boundary is caught.

The rule it implements ("Thinking Machines Lab releases 4-bit training",
communication paragraph: a 32-point random Hadamard transform before
quantizing): the transform may differ from the double-precision one by
1e-6 * ||x_group||_2, so a quantized result may differ only where that
difference can move the value across an E2M1 or E4M3 rounding midpoint.
"""
import numpy as np
import pytest

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import rht_boundary_check


def _case():
    x = syn.random_case((64, 512), 77, "outlier")
    yd = oracle.rht32_f64(x, 3)
    oc, osc, ot, oy = oracle.rht_quantize(x, 3)
    return x, yd, oc, osc, ot


def test_identical_outputs_pass():
    x, yd, oc, osc, ot = _case()
    assert rht_boundary_check(x, yd, oc, osc, ot, oc.copy(), osc.copy(), ot) == (0, 0)


def _cells(x, yd, osc, ot):
    """|v| of every element in its own block's scale (the oracle's)."""
    e4 = np.array([oracle.e4m3_value(k) for k in range(256)])
    y = yd.astype(np.float32).astype(np.float64).reshape(-1, 16)
    sc = e4[np.asarray(osc).reshape(-1)] * ot
    return np.abs(y) / np.where(sc > 0, sc, 1)[:, None], sc


def test_code_changed_mid_cell_is_caught():
    x, yd, oc, osc, ot = _case()
    a, sc = _cells(x, yd, osc, ot)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    dist = np.min(np.abs(a.reshape(-1)[:, None] - mids[None, :]), axis=1)
    dist[np.repeat(sc, 16) == 0] = 0
    i = int(np.argmax(dist))  # the element farthest from any boundary
    assert dist[i] > 0.1
    codes = oracle.unpack_codes(oc)
    m = codes[i] & 7
    codes[i] = (codes[i] & 8) | (m + 1 if m < 7 else m - 1)
    bad = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8).reshape(oc.shape)
    with pytest.raises(AssertionError, match="E2M1"):
        rht_boundary_check(x, yd, oc, osc, ot, bad, osc, ot)


def test_scale_changed_mid_step_is_caught():
    x, yd, oc, osc, ot = _case()
    y = yd.astype(np.float32).astype(np.float64).reshape(-1, 16)
    sbf = np.abs(y).max(axis=1) / 6.0 / ot
    e4 = np.array([oracle.e4m3_value(k) for k in range(127)])
    mid = (e4[:-1] + e4[1:]) / 2
    dist = np.min(np.abs(sbf[:, None] - mid[None, :]), axis=1) / sbf
    b = int(np.argmax(dist))
    s2 = np.asarray(osc).reshape(-1).copy()
    s2[b] = s2[b] + 1
    with pytest.raises(AssertionError, match="E4M3"):
        rht_boundary_check(x, yd, oc, osc, ot, oc, s2.reshape(osc.shape), ot)


def test_sign_of_zero_is_not_a_difference():
    x = syn.random_case((8, 64), 5, "zeros")
    yd = oracle.rht32_f64(x, 3)
    oc, osc, ot, _ = oracle.rht_quantize(x, 3)
    codes = oracle.unpack_codes(oc)
    flipped = np.where((codes & 7) == 0, codes ^ 8, codes).astype(np.uint8)
    g = (flipped[0::2] | (flipped[1::2] << 4)).astype(np.uint8).reshape(oc.shape)
    assert rht_boundary_check(x, yd, oc, osc, ot, g, osc, ot)[1] == 0
