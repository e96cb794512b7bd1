"""Pins for the oracle's Philox generator, stochastic-rounding transpose and
32-point random Hadamard transform (CPU only).

* Philox4x32-10: the published known-answer vectors (tests/golden).
* SR: the worked example of "Thinking Machines Lab releases 4-bit training"
  (forward/backward mismatch paragraph: 2.25 -> 2 three times in four, 3 once,
  mean 2.25) -- exactly 2^22 of the 2^24 possible 24-bit draws round up;
  unbiasedness of the mean over many draws; a transpose whose values are
  already on the grid comes back as the transposed codes.
* RHT: scipy's Sylvester Hadamard matrix, the unit-vector closed form, norm
  preservation and inversion.
"""
import json
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from train_rollout_alignment_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_philox_known_answers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(t, 16) for t in r]
        assert oracle.philox4x32_10(v[0:4], v[4:6]) == tuple(v[6:10])


def _count_round_up(a: float) -> int:
    """Number of 24-bit draws k (r = k << 8) that round a up (decisions are
    monotone in k, so bisect for the first k that rounds down)."""
    lo_m = oracle.sr_magnitude(a, 0xFFFFFF00)
    hi_m = oracle.sr_magnitude(a, 0)
    if lo_m == hi_m:
        return 0
    lo, hi = 0, 1 << 24
    while lo < hi:
        mid = (lo + hi) // 2
        if oracle.sr_magnitude(a, mid << 8) == hi_m:
            lo = mid + 1
        else:
            hi = mid
    rng = np.random.default_rng(1)
    for k in rng.integers(0, 1 << 24, 200):
        assert oracle.sr_magnitude(a, int(k) << 8) == (hi_m if k < lo else lo_m)
    return lo


def test_sr_worked_example_2p25():
    ex = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["tml4_sr_2p25"]
    a = ex["value"]
    assert GRID[oracle.sr_magnitude(a, 0)] == ex["high"]
    assert GRID[oracle.sr_magnitude(a, 0xFFFFFFFF)] == ex["low"]
    up = _count_round_up(a)
    assert up == int(ex["p_high"] * 2 ** 24)
    mean = (ex["high"] * up + ex["low"] * (2 ** 24 - up)) / 2 ** 24
    assert mean == ex["mean"]


@pytest.mark.parametrize("a,p", [(0.125, 0.25), (1.25, 0.5), (2.75, 0.75), (4.5, 0.25), (5.5, 0.75)])
def test_sr_probability_is_exact_for_dyadic_fractions(a, p):
    assert _count_round_up(a) == int(p * 2 ** 24)


def test_sr_on_grid_and_saturation_are_deterministic():
    for m, g in enumerate(GRID):
        for r in (0, 0x12345678, 0xFFFFFFFF):
            assert oracle.sr_magnitude(g, r) == m
    for v in (6.0, 6.5, 100.0):
        assert oracle.sr_magnitude(v, 0) == 7


def _rtn_stack(w):
    batch, rows, cols = w.shape
    codes = np.zeros((batch, rows, cols // 2), np.uint8)
    scales = np.zeros((batch, rows, cols // 16), np.uint8)
    ts = np.zeros(batch, np.float32)
    for e in range(batch):
        c, s, t, _ = oracle.quantize_rtn(w[e])
        codes[e], scales[e], ts[e] = c, s, t
    return codes, scales, ts


def test_sr_transpose_mean_is_unbiased():
    batch, rows, cols, draws = 2, 32, 48, 400
    w = syn.random_case((batch, rows, cols), 17, "normal")
    codes, scales, ts = _rtn_stack(w)
    n = rows * cols
    y = np.stack([oracle.dequant(codes[e], scales[e], ts[e], n).reshape(rows, cols).T
                  for e in range(batch)])  # [batch, cols, rows]
    acc = np.zeros((batch, cols * rows))
    for d in range(draws):
        ct, st, tst = oracle.sr_transpose_requant(codes, scales, ts, batch, rows, cols, 2, d)
        for e in range(batch):
            acc[e] += oracle.dequant(ct[e], st[e], tst[e], n)
    mean = acc / draws
    # expected value is v * sb' * s_t' ~= y; the spread of one draw is the cell
    # width (in value units) times sqrt(p (1 - p))
    z_num, z_var = 0.0, 0.0
    for e in range(batch):
        _, st, tst = oracle.sr_transpose_requant(codes, scales, ts, batch, rows, cols, 2, 0)[0:3]
        scale = np.array([oracle.e4m3_value(b) for b in st[e].reshape(-1)]).repeat(16) * tst[e]
        a = np.abs(y[e].reshape(-1)) / np.where(scale > 0, scale, 1)
        lo = np.clip(np.searchsorted(GRID, a, side="right") - 1, 0, 6)
        w_cell = GRID[lo + 1] - GRID[lo]
        p = np.clip((a - GRID[lo]) / w_cell, 0, 1)
        p[a >= 6] = 0
        sd = w_cell * scale * np.sqrt(p * (1 - p) / draws)
        # a block scale rounded down can put |v| above 6: those elements clip
        # to 6 deterministically, so their expected value is 6 * scale
        expect = np.where(a >= 6, np.sign(y[e].reshape(-1)) * 6 * scale, y[e].reshape(-1))
        diff = mean[e] - expect
        assert np.all(np.abs(diff) <= 5 * sd + 1e-6 * np.abs(expect) + 1e-30)
        z_num += diff.sum()
        z_var += (sd ** 2).sum()
    assert abs(z_num / np.sqrt(z_var)) < 5


def test_sr_transpose_of_on_grid_values_is_the_transpose():
    rows, cols = 32, 32
    rng = np.random.default_rng(4)
    m = rng.integers(0, 8, (rows, cols))
    m[np.arange(rows), np.arange(cols)] = 7          # every row and column block holds a 6
    m[np.arange(rows), (np.arange(cols) + 16) % cols] = 7
    sign = rng.integers(0, 2, (rows, cols)) << 3
    c = (sign | m).astype(np.uint8).reshape(-1)
    codes = (c[0::2] | (c[1::2] << 4)).astype(np.uint8).reshape(1, rows, cols // 2)
    scales = np.full((1, rows, cols // 16), oracle.e4m3_rne_satfinite(2.0), np.uint8)
    ts = np.array([0.75], np.float32)
    ct, st, tst = oracle.sr_transpose_requant(codes, scales, ts, 1, rows, cols, 2, 0)
    got = oracle.unpack_codes(ct[0]).reshape(cols, rows)
    want = c.reshape(rows, cols).T
    # values land within a few ulps of grid points, so a draw moves a code with
    # probability ~1e-7; zero codes keep their sign
    assert np.array_equal(got, want)
    y = oracle.dequant(codes[0], scales[0], ts[0], rows * cols).reshape(rows, cols).T
    yt = oracle.dequant(ct[0], st[0], tst[0], rows * cols).reshape(cols, rows)
    assert np.allclose(yt, y, rtol=1e-6, atol=0)


def test_sr_transpose_index_counter():
    """The random word of output element i is Philox(key=seed, ctr=(i, 0, draw, 0)).x0."""
    batch, rows, cols = 2, 16, 32
    w = syn.random_case((batch, rows, cols), 23, "normal")
    codes, scales, ts = _rtn_stack(w)
    seed, draw = (7 << 32) | 5, 3
    ct, st, tst = oracle.sr_transpose_requant(codes, scales, ts, batch, rows, cols, seed, draw)
    n = rows * cols
    for e in range(batch):
        y = oracle.dequant(codes[e], scales[e], ts[e], n).reshape(rows, cols).T.reshape(-1)
        got = oracle.unpack_codes(ct[e])
        for local in range(n):
            i = e * n + local
            r = oracle.philox4x32_10([i & 0xFFFFFFFF, i >> 32, draw, 0], [seed & 0xFFFFFFFF, seed >> 32])[0]
            sbv = np.float32(oracle.e4m3_value(st[e].reshape(-1)[local // 16]))
            inv = np.float32(1.0) / (sbv * np.float32(tst[e]))
            a = abs(np.float32(y[local]) * inv)
            assert got[local] & 7 == oracle.sr_magnitude(a, r)


def test_rht_signs_come_from_philox_bit0():
    for seed in (3, (1 << 32) | 9):
        s = oracle.rht_signs(seed)
        for j in range(32):
            x0 = oracle.philox4x32_10([j, 0, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])[0]
            assert s[j] == (-1 if x0 & 1 else 1)
        assert 4 < np.sum(s < 0) < 28


def test_rht_matches_sylvester_matrix_product():
    x = syn.random_case((4, 96), 5, "heavy")
    seed = 3
    y = oracle.rht32_f64(x, seed)
    H = scipy.linalg.hadamard(32).astype(np.float64)
    sig = oracle.rht_signs(seed).astype(np.float64)
    xg = syn.bf16_to_f32(x).astype(np.float64).reshape(-1, 32)
    want = (xg * sig) @ H.T / np.sqrt(32.0)
    assert np.allclose(y.reshape(-1, 32), want, rtol=0, atol=1e-12 * np.abs(xg).max())
    # orthogonality: norm kept, and sigma (.) (H y) / sqrt(32) gives x back
    assert np.allclose(np.linalg.norm(y.reshape(-1, 32), axis=1), np.linalg.norm(xg, axis=1), rtol=1e-12)
    back = (y.reshape(-1, 32) @ H.T / np.sqrt(32.0)) * sig
    assert np.allclose(back, xg, rtol=0, atol=1e-12 * np.abs(xg).max())


def test_rht_unit_vectors():
    seed = 11
    sig = oracle.rht_signs(seed)
    H = scipy.linalg.hadamard(32)
    for k in (0, 1, 5, 31):
        e = np.zeros((1, 32), np.float32)
        e[0, k] = 1.0
        y = oracle.rht32_f64(syn.bf16_bits(e), seed)[0]
        assert np.array_equal(y, sig[k] * H[:, k] / np.sqrt(32.0))


def test_rht_quantize_equals_quantize_of_rounded_transform():
    x = syn.random_case((8, 64), 6, "outlier")
    codes, scales, ts, y = oracle.rht_quantize(x, 3)
    yd = oracle.rht32_f64(x, 3)
    assert np.array_equal(y, yd.astype(np.float32))
    c2, s2, t2 = oracle.quantize_f32(y)
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2) and ts == t2


def test_sr_transpose_per_matrix_calls_match_whole_stack():
    batch, rows, cols = 3, 16, 48
    w = syn.random_case((batch, rows, cols), 29, "normal")
    codes, scales, ts = _rtn_stack(w)
    whole = oracle.sr_transpose_requant(codes, scales, ts, batch, rows, cols, 9, 4)
    for e in range(batch):
        part = oracle.sr_transpose_requant(codes[e:e + 1], scales[e:e + 1], ts[e:e + 1], 1, rows, cols,
                                           9, 4, first=e)
        assert np.array_equal(part[0][0], whole[0][e]) and np.array_equal(part[1][0], whole[1][e])
        assert part[2][0] == whole[2][e]
