"""Pins for the oracle's two alternatives to the dequantize -> transpose -> SR
re-quantize step ("Thinking Machines Lab releases 4-bit training",
forward/backward mismatch paragraph): NVIDIA's 16x16-tile scaling, and the
backward in MXFP8 with stochastic rounding (CPU only).

* Tile scaling: a transpose maps a tile-scaled matrix onto the tile
  quantization of the transposed input (the property the page names); when
  every 16-value row of each tile reaches its tile's maximum the tile result
  equals the 16-value block result (tying it to the pinned block path); exact
  rational brute force on small matrices; one large value flattens the rest of
  its tile (the page's objection).
* MXFP8: 8.25 bits per value (the page's format table); the E8M0 exponent puts
  every block maximum in the top E4M3 binade; E4M3 decode and the SR bracket
  against ml_dtypes; exact round-up counts for dyadic fractions; unbiasedness
  over draws; the Philox counter of every element; on-grid values transpose
  losslessly.
"""
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import oracle
from train_rollout_alignment_b200 import synthetic as syn

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
E4M3 = [oracle.e4m3_value(b) for b in range(0x7F)]
E4M3_LIB = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def _nearest_with_margin(target: Fraction, cands):
    ds = [abs(target - Fraction(c)) for c in cands]
    best = min(range(len(cands)), key=lambda k: (ds[k], k % 2))
    safe = all(not (m != 0 and abs(target - m) <= abs(m) * Fraction(1, 2 ** 18))
               for m in ((Fraction(cands[k]) + Fraction(cands[k + 1])) / 2 for k in range(len(cands) - 1)))
    return best, safe


# ----------------------------------------------------------------------------- tile scaling
@pytest.mark.parametrize("shape,kind", [((16, 16), "normal"), ((32, 48), "heavy"), ((64, 32), "outlier"),
                                        ((48, 16), "tiny"), ((32, 32), "zeros"), ((16, 64), "sparse")])
def test_tile16_transpose_is_the_tile_quantization_of_the_transpose(shape, kind):
    x = syn.random_case(shape, 900 + shape[0], kind)
    rows, cols = shape
    c, t, s = oracle.quantize_tile16(x)
    ct, tt = oracle.transpose_tile16(c[None], t[None], 1, rows, cols)
    c2, t2, s2 = oracle.quantize_tile16(np.ascontiguousarray(x.T))
    assert s == s2
    assert np.array_equal(ct[0], c2) and np.array_equal(tt[0], t2)
    # and the transpose is an involution
    cb, tb = oracle.transpose_tile16(ct, tt, 1, cols, rows)
    assert np.array_equal(cb[0], c) and np.array_equal(tb[0], t)


def test_tile16_equals_blocks_when_every_row_reaches_the_tile_max():
    rng = np.random.default_rng(3)
    rows, cols = 64, 96
    xf = rng.standard_normal((rows, cols)).astype(np.float32)
    for ti in range(rows // 16):
        for tj in range(cols // 16):
            tile = xf[16 * ti:16 * ti + 16, 16 * tj:16 * tj + 16]
            m = np.float32(np.abs(tile).max() * 1.5)
            tile[np.arange(16), rng.integers(0, 16, 16)] = m * np.where(rng.random(16) < 0.5, -1, 1)
    x = syn.bf16_bits(xf)
    c, t, s = oracle.quantize_tile16(x)
    cb, sb, sbt, _ = oracle.quantize_rtn(x)
    assert s == sbt
    assert np.array_equal(c, cb)
    assert np.array_equal(np.repeat(t, 16, axis=0), sb)


@pytest.mark.parametrize("shape,seed,kind", [((16, 16), 1, "normal"), ((32, 32), 2, "heavy"),
                                             ((16, 48), 3, "tiny"), ((32, 16), 4, "outlier")])
def test_tile16_recipe_brute_force(shape, seed, kind):
    x = syn.random_case(shape, seed, kind)
    xf = syn.bf16_to_f32(x).astype(np.float64)
    c, t, s_t = oracle.quantize_tile16(x)
    codes = oracle.unpack_codes(c).reshape(shape)
    checked = total = 0
    for ti in range(shape[0] // 16):
        for tj in range(shape[1] // 16):
            tile = xf[16 * ti:16 * ti + 16, 16 * tj:16 * tj + 16]
            target = Fraction(float(np.abs(tile).max())) / (6 * Fraction(s_t))
            sb, safe = _nearest_with_margin(target, E4M3)
            if not safe:
                continue
            assert t[ti, tj] == sb
            scale = Fraction(E4M3[sb]) * Fraction(s_t)
            for (r, cc), v in np.ndenumerate(tile):
                total += 1
                sign = 8 if np.signbit(v) else 0
                if scale == 0:
                    assert codes[16 * ti + r, 16 * tj + cc] == sign
                    checked += 1
                    continue
                m, safe_m = _nearest_with_margin(abs(Fraction(float(v))) / scale, GRID)
                if safe_m:
                    checked += 1
                    assert codes[16 * ti + r, 16 * tj + cc] == sign | m
    assert checked >= 0.8 * total


def test_one_large_value_flattens_its_tile():
    rng = np.random.default_rng(5)
    xf = rng.uniform(0.5, 1.0, (32, 32)).astype(np.float32)
    xf[3, 5] = 1000.0  # one large value in tile (0, 0)
    x = syn.bf16_bits(xf)
    c, t, _ = oracle.quantize_tile16(x)
    codes = oracle.unpack_codes(c).reshape(32, 32)
    tile0 = codes[:16, :16].copy()
    tile0[3, 5] = 0
    assert not (tile0 & 7).any()                  # everything else in the tile rounds to 0
    assert (codes[16:, :] & 7).all() and (codes[:16, 16:] & 7).all()  # other tiles keep their values
    cb, _, _, _ = oracle.quantize_rtn(x)
    blocks = oracle.unpack_codes(cb).reshape(32, 32)
    assert (blocks[:16, :16][np.arange(16) != 3] & 7).all()  # 16-value blocks lose only row 3


def test_tile16_dequant_is_block_dequant_with_broadcast_scales():
    x = syn.random_case((48, 64), 11, "heavy")
    c, t, s = oracle.quantize_tile16(x)
    y = oracle.dequant_tile16(c, t, s, 48, 64)
    yb = oracle.dequant(c, np.repeat(t, 16, axis=0), s, 48 * 64).reshape(48, 64)
    assert np.array_equal(y.view(np.uint32), yb.view(np.uint32))


# ----------------------------------------------------------------------------- MXFP8
def test_mxfp8_is_eight_and_a_quarter_bits_per_value():
    batch, rows, cols = 1, 64, 32
    codes = np.zeros((batch, rows, cols // 2), np.uint8)
    scales = np.zeros((batch, rows, cols // 16), np.uint8)
    q, e8 = oracle.mxfp8_sr_transpose_requant(codes, scales, np.ones(1, np.float32), batch, rows, cols, 1, 0)
    assert (q.nbytes + e8.nbytes) * 8 / (rows * cols) == 8.25


def test_e4m3_decode_matches_library():
    assert np.array_equal(np.array(E4M3), E4M3_LIB)


@pytest.mark.parametrize("k", [-119, -20, -3, 0, 1, 7, 8, 30])
def test_e8m0_exponent_puts_the_block_max_in_the_top_binade(k):
    for f in (1.0, 1.5, 1.9999999):
        amax = np.float32(f * 2.0 ** k)
        e = oracle.e8m0_exponent(float(amax))
        assert e == k - 8
        scaled = float(amax) * 2.0 ** -e
        assert 256.0 <= scaled < 512.0  # the binade of 256..448 (values above 448 saturate)
    assert oracle.e8m0_exponent(float(np.float32(2.0 ** k) * np.float32(1 - 2 ** -24))) == max(k - 9, -127)


def test_e8m0_exponent_edges():
    assert oracle.e8m0_exponent(0.0) == -127
    assert oracle.e8m0_exponent(2.0 ** -140) == -127  # clamped
    assert oracle.e8m0_exponent(2.0 ** -120) == -127  # -128 clamped
    assert oracle.e8m0_exponent(3.0e38) == 119


def test_e4m3_sr_bracket_matches_library_values():
    rng = np.random.default_rng(8)
    a = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 3000)),
                        E4M3_LIB, (E4M3_LIB[:-1] + E4M3_LIB[1:]) / 2]).astype(np.float32)
    for v in a:
        v = float(v)
        lo_b = oracle.e4m3_sr(v, 0xFFFFFFFF)  # the largest draw never rounds up
        hi_b = oracle.e4m3_sr(v, 0)           # the smallest always does, off the grid
        below = E4M3_LIB[E4M3_LIB <= v]
        assert E4M3_LIB[lo_b] == below.max()
        if v in E4M3_LIB:
            assert hi_b == lo_b
        elif v < 448:
            assert E4M3_LIB[hi_b] == E4M3_LIB[E4M3_LIB > v].min()
    for v in (448.0, 460.0, 1e6):
        assert oracle.e4m3_sr(v, 0) == 0x7E


def _count_round_up(a: float) -> int:
    lo_b, hi_b = oracle.e4m3_sr(a, 0xFFFFFF00), oracle.e4m3_sr(a, 0)
    if lo_b == hi_b:
        return 0
    lo, hi = 0, 1 << 24
    while lo < hi:
        mid = (lo + hi) // 2
        if oracle.e4m3_sr(a, mid << 8) == hi_b:
            lo = mid + 1
        else:
            hi = mid
    return lo


@pytest.mark.parametrize("lo_b,p", [(0x01, 0.25), (0x38, 0.5), (0x41, 0.75), (0x7D, 0.125), (0x10, 0.375)])
def test_e4m3_sr_probability_is_exact_for_dyadic_fractions(lo_b, p):
    a = E4M3[lo_b] + p * (E4M3[lo_b + 1] - E4M3[lo_b])
    assert _count_round_up(a) == int(p * 2 ** 24)


def _nvfp4_stack(w):
    outs = [oracle.quantize_rtn(w[e]) for e in range(w.shape[0])]
    return (np.stack([o[0] for o in outs]), np.stack([o[1] for o in outs]),
            np.array([o[2] for o in outs], np.float32))


def test_mxfp8_sr_transpose_mean_is_unbiased():
    batch, rows, cols, draws = 2, 64, 32, 300
    w = syn.random_case((batch, rows, cols), 41, "normal")
    codes, scales, ts = _nvfp4_stack(w)
    n = rows * cols
    y = np.stack([oracle.dequant(codes[e], scales[e], ts[e], n).reshape(rows, cols).T.reshape(-1)
                  for e in range(batch)])
    acc = np.zeros((batch, n))
    for d in range(draws):
        q, e8 = oracle.mxfp8_sr_transpose_requant(codes, scales, ts, batch, rows, cols, 9, d)
        for e in range(batch):
            acc[e] += oracle.mxfp8_dequant(q[e], e8[e])
    q, e8 = oracle.mxfp8_sr_transpose_requant(codes, scales, ts, batch, rows, cols, 9, 0)
    z_num = z_var = 0.0
    for e in range(batch):
        unit = 2.0 ** (e8[e].reshape(-1).astype(np.float64) - 127).repeat(32)
        a = np.abs(y[e]) / unit
        lo = np.array([E4M3_LIB[E4M3_LIB <= v].max() for v in a])
        hi = np.array([E4M3_LIB[E4M3_LIB > v].min() if v < 448 else 448.0 for v in a])
        p = np.where(hi > lo, (a - lo) / np.where(hi > lo, hi - lo, 1), 0)
        expect = np.sign(y[e]) * np.where(a >= 448, 448, a) * unit
        sd = (hi - lo) * unit * np.sqrt(p * (1 - p) / draws)
        diff = acc[e] / draws - expect
        assert np.all(np.abs(diff) <= 5 * sd + 1e-12 * np.abs(expect) + 1e-30)
        z_num += diff.sum()
        z_var += (sd ** 2).sum()
    assert abs(z_num / np.sqrt(z_var)) < 5


def test_mxfp8_sr_transpose_index_counter():
    """Random word of output element i (row-major in [batch, cols, rows]):
    Philox(key=seed, ctr=(i lo, i hi, draw, 0)).x0; the block exponent from the
    block maximum; v = y * 2^-e."""
    batch, rows, cols = 2, 32, 16
    w = syn.random_case((batch, rows, cols), 43, "heavy")
    codes, scales, ts = _nvfp4_stack(w)
    seed, draw = (3 << 32) | 11, 5
    q, e8 = oracle.mxfp8_sr_transpose_requant(codes, scales, ts, batch, rows, cols, seed, draw)
    n = rows * cols
    for e in range(batch):
        yt = oracle.dequant(codes[e], scales[e], ts[e], n).reshape(rows, cols).T.reshape(-1)
        for b in range(n // 32):
            blk = yt[32 * b:32 * b + 32]
            ex = oracle.e8m0_exponent(float(np.abs(blk).max()))
            assert e8[e].reshape(-1)[b] == ex + 127
            for k in range(32):
                i = e * n + 32 * b + k
                r = oracle.philox4x32_10([i & 0xFFFFFFFF, i >> 32, draw, 0], [seed & 0xFFFFFFFF, seed >> 32])[0]
                v = abs(float(np.float32(blk[k]) * np.float32(2.0 ** -ex)))
                got = int(q[e].reshape(-1)[32 * b + k])
                assert got & 0x7F == oracle.e4m3_sr(v, r)
                assert got >> 7 == int(np.signbit(blk[k]))


def test_mxfp8_on_grid_values_transpose_losslessly():
    rows, cols = 32, 32
    rng = np.random.default_rng(6)
    m = rng.integers(0, 8, (rows, cols))
    m[np.arange(rows), np.arange(cols)] = 7
    sign = rng.integers(0, 2, (rows, cols)) << 3
    c = (sign | m).astype(np.uint8).reshape(-1)
    codes = (c[0::2] | (c[1::2] << 4)).astype(np.uint8).reshape(1, rows, cols // 2)
    scales = np.full((1, rows, cols // 16), oracle.e4m3_rne_satfinite(2.0), np.uint8)  # power-of-two scale
    ts = np.array([0.125], np.float32)                                                # and tensor scale
    y = oracle.dequant(codes[0], scales[0], ts[0], rows * cols).reshape(rows, cols).T.reshape(-1)
    for draw in (0, 1, 77):
        q, e8 = oracle.mxfp8_sr_transpose_requant(codes, scales, ts, 1, rows, cols, 2, draw)
        yt = oracle.mxfp8_dequant(q[0], e8[0])
        assert np.array_equal(yt.view(np.uint32), y.view(np.uint32)) or np.array_equal(yt, y)


def test_mxfp8_per_matrix_calls_match_whole_stack():
    batch, rows, cols = 3, 32, 32
    w = syn.random_case((batch, rows, cols), 47, "normal")
    codes, scales, ts = _nvfp4_stack(w)
    q, e8 = oracle.mxfp8_sr_transpose_requant(codes, scales, ts, batch, rows, cols, 4, 2)
    for e in range(batch):
        qe, e8e = oracle.mxfp8_sr_transpose_requant(codes[e:e + 1], scales[e:e + 1], ts[e:e + 1], 1, rows,
                                                    cols, 4, 2, first=e)
        assert np.array_equal(qe[0], q[e]) and np.array_equal(e8e[0], e8[e])
