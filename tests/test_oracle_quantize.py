"""Pins for the oracle's quantize, hint, guided re-quantize and mismatch steps.

What pins what (none of these re-types the oracle's FP32 chain):
* scale recipe / code choice: brute force over all 16 codes and all 127 finite
  E4M3 scales, in exact rational arithmetic, on tiny tensors; elements whose
  exact value sits within 2^-18 of a decision boundary are excluded (the
  oracle's rounded FP32 chain may legitimately fall either side there);
* closed forms: the tensor's largest element takes the top code; an all-zero
  tensor gives s_t = 1 and zero scales;
* TRACE explainer, rounding-analogy / prescription paragraphs: the 2.49 / 2.51
  example;
* hints: unpacking with numpy's unpackbits and the stated field order;
* guided rounding: guiding a tensor by its own hints changes nothing; the
  distance guarantee of the prescription paragraph (never further from the
  rollout than round-to-nearest) for full codes everywhere, for 2-bit hints
  inside the window where modular aliasing cannot occur;
* mismatch counters: pairs built with a known number of changes.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from train_rollout_alignment_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
E4M3 = [oracle.e4m3_value(b) for b in range(0x7F)]


def _codes(codes, n):
    return oracle.unpack_codes(codes, n)


def _pos(c):
    c = c.astype(np.int64)
    return np.where(c & 8, -(c & 7), c & 7)


def _nearest_with_margin(target: Fraction, cands, even_of):
    """Index of the nearest candidate (ties -> even_of(index) True), and
    whether target is at least 2^-18 (relative) away from every midpoint."""
    ds = [abs(target - Fraction(c)) for c in cands]
    best = min(range(len(cands)), key=lambda k: (ds[k], not even_of(k)))
    safe = True
    for k in range(len(cands) - 1):
        mid = (Fraction(cands[k]) + Fraction(cands[k + 1])) / 2
        if mid != 0 and abs(target - mid) <= abs(mid) * Fraction(1, 2 ** 18):
            safe = False
    return best, safe


@pytest.mark.parametrize("shape,seed,kind", [((1, 16), 1, "normal"), ((2, 32), 2, "normal"),
                                             ((4, 64), 3, "heavy"), ((3, 48), 4, "tiny"),
                                             ((2, 64), 5, "ties"), ((4, 32), 6, "outlier")])
def test_block_recipe_brute_force(shape, seed, kind):
    x = syn.random_case(shape, seed, kind)
    xf = syn.bf16_to_f32(x).astype(np.float64)
    codes, scales, s_t, _ = oracle.quantize_rtn(x)
    A = float(np.max(np.abs(xf)))
    # tensor scale: A / 2688 correctly rounded (division of two floats done in
    # double then rounded to float is correctly rounded)
    assert np.float32(s_t) == np.float32(A / 2688.0) if A > 0 else s_t == 1.0
    c = _codes(codes, x.size).reshape(shape)
    checked = total = 0
    for r in range(shape[0]):
        for b in range(shape[1] // 16):
            blk = xf[r, 16 * b:16 * b + 16]
            amax_b = Fraction(float(np.max(np.abs(blk))))
            target = amax_b / (6 * Fraction(s_t))
            sb, safe_sb = _nearest_with_margin(target, E4M3, lambda k: k % 2 == 0)
            if not safe_sb:
                continue
            assert scales[r, b] == sb, (r, b)
            scale = Fraction(E4M3[sb]) * Fraction(s_t)
            for k in range(16):
                total += 1
                if scale == 0:
                    assert c[r, 16 * b + k] == (8 if np.signbit(blk[k]) else 0)
                    checked += 1
                    continue
                a = abs(Fraction(float(blk[k]))) / scale
                m, safe = _nearest_with_margin(a, GRID, lambda k2: k2 % 2 == 0)
                if not safe:
                    continue
                checked += 1
                want = (8 if np.signbit(blk[k]) else 0) | m
                assert c[r, 16 * b + k] == want, (r, b, k, float(a))
    assert checked >= 0.8 * total or kind == "ties"


def test_tensor_max_takes_top_code_and_zero_tensor():
    for seed in range(5):
        x = syn.random_case((8, 64), 100 + seed, "heavy")
        codes, scales, s_t, _ = oracle.quantize_rtn(x)
        xf = syn.bf16_to_f32(x)
        i = int(np.argmax(np.abs(xf)))
        assert _codes(codes, x.size)[i] & 7 == 7
        assert scales.reshape(-1)[i // 16] == 0x7E  # block of A: scale 448
    z = syn.random_case((2, 32), 0, "zeros")
    codes, scales, s_t, _ = oracle.quantize_rtn(z)
    assert s_t == 1.0 and not scales.any()
    want = np.where(np.signbit(syn.bf16_to_f32(z).reshape(-1)), 8, 0)
    assert np.array_equal(_codes(codes, z.size), want)


def test_trace_rounding_analogy_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["trace_rounding_analogy"]
    row = np.zeros((1, 16), np.float32)
    row[0, 0] = ex["block_max"]
    train, roll = row.copy(), row.copy()
    train[0, 1], roll[0, 1] = ex["train_value"], ex["rollout_value"]
    xt, xr = syn.bf16_bits(train), syn.bf16_bits(roll)
    for bits in (1, 2, 4):
        rc, rs, rts, hints = oracle.quantize_rtn(xr, hint_bits=bits)
        tc, ts_, tts, _ = oracle.quantize_rtn(xt)
        gc, gs, gts, st = oracle.guided_requant(xt, hints, bits)
        dq = lambda c, s, t: oracle.dequant(c, s, t, 16)[1]
        assert dq(tc, ts_, tts) == pytest.approx(ex["expected_train_rtn_value"], rel=1e-6)
        assert dq(rc, rs, rts) == pytest.approx(ex["expected_rollout_rtn_value"], rel=1e-6)
        assert dq(gc, gs, gts) == pytest.approx(ex["expected_guided_value"], rel=1e-6)
        assert st[1] == 1  # exactly one element changed by the guidance


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_hint_pack_round_trip(bits):
    rng = np.random.default_rng(bits)
    n = 16 * 37
    c = rng.integers(0, 16, n).astype(np.uint8)
    packed = (c[0::2] | (c[1::2] << 4)).astype(np.uint8)
    h = oracle.emit_hint(packed, n, bits)
    assert h.size == (n * bits + 7) // 8
    fields = np.unpackbits(h, bitorder="little")[: n * bits].reshape(n, bits)
    vals = (fields * (1 << np.arange(bits))).sum(1)
    want = c if bits == 4 else (c & 7) & ((1 << bits) - 1)
    if bits != 4:
        # inside each 16-element block, field f holds element (f >> 1) + 8 * (f & 1)
        order = np.array([(f >> 1) + 8 * (f & 1) for f in range(16)])
        want = want.reshape(-1, 16)[:, order].reshape(-1)
    assert np.array_equal(vals, want)


def test_sparse_case_zeros_are_on_grid():
    """Exact zeros never consult the hint; BF16 subnormals next to a large
    value quantize to zero magnitude but are off the grid (bracket 0 / 0.5)."""
    x = syn.random_case((4, 64), 11, "sparse")
    xf = syn.bf16_to_f32(x)
    zero = xf.reshape(-1) == 0
    assert zero.sum() > 64
    for bits in (1, 2):
        h_all = np.full(x.size * bits // 8, 0xFF, np.uint8)  # always names the odd cell
        gc, _, _, st = oracle.guided_requant(x, h_all, bits)
        c = _codes(gc, x.size)
        assert np.all(c[zero] & 7 == 0)
        assert np.array_equal(c[zero] >> 3, np.signbit(xf.reshape(-1)[zero]).astype(np.uint8))
        assert st[0] <= x.size - zero.sum()


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_guided_by_own_hints_is_rtn(bits):
    x = syn.random_case((16, 128), 7, "heavy")
    codes, scales, s_t, hints = oracle.quantize_rtn(x, hint_bits=bits)
    gc, gs, gts, st = oracle.guided_requant(x, hints, bits)
    assert np.array_equal(gc, codes) and np.array_equal(gs, scales) and gts == s_t
    assert st[1] == 0 and st[2] == 0 and st[0] > 0
    nc, ns, nts, nst = oracle.guided_requant(x, None, bits)
    assert np.array_equal(nc, codes) and not nst.any()


def _scaled_abs(x, scales, s_t):
    """|x| / (sb * s_t) per element in double (approximates the FP32 v)."""
    xf = syn.bf16_to_f32(x).astype(np.float64).reshape(-1)
    sbv = np.array(E4M3, np.float64)[scales.reshape(-1).repeat(16)]
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(sbv > 0, np.abs(xf) / (sbv * s_t), 0.0), np.signbit(xf)


@pytest.mark.parametrize("noise", [2.0 ** -8, 2.0 ** -4, 0.5, None])
def test_guided_distance_guarantee(noise):
    rng = np.random.default_rng(3)
    xt = syn.random_case((32, 256), 9, "normal")
    if noise is None:
        xr = syn.random_case((32, 256), 10, "normal")  # unrelated rollout
    else:
        xr = syn.rollout_copy(xt, rng, noise)
    n = xt.size
    rtn_c, rtn_s, rtn_t, _ = oracle.quantize_rtn(xt)
    ro_c, _, _, _ = oracle.quantize_rtn(xr)
    p_rtn, p_ro = _pos(_codes(rtn_c, n)), _pos(_codes(ro_c, n))
    a, neg = _scaled_abs(xt, rtn_s, rtn_t)
    grid = np.array(GRID)
    lo = np.searchsorted(grid, a, side="right") - 1
    margin = np.min(np.abs(a[:, None] - grid[None, :]), axis=1) > 1e-6
    r_mag = np.abs(p_ro)
    r_neg = p_ro < 0
    for bits in (1, 2, 4):
        _, _, _, hints = oracle.quantize_rtn(xr, hint_bits=bits)
        gc, _, _, st = oracle.guided_requant(xt, hints, bits)
        p_g = _pos(_codes(gc, n))
        worse = np.abs(p_g - p_ro) > np.abs(p_rtn - p_ro)
        # the guided cell is always one of the two cells bracketing v
        assert np.all(np.isin(np.abs(p_g) - lo, [0, 1]) | ~margin | (a >= 6))
        same_sign = (r_neg == neg) | (r_mag == 0)
        if bits == 4:
            assert not worse.any()
        elif bits == 2:
            window = (r_mag >= lo - 2) & (r_mag <= lo + 3) & same_sign & margin
            assert not (worse & window).any()
        else:
            hit = ((r_mag == lo) | (r_mag == lo + 1)) & same_sign & margin & (a < 6)
            assert np.all(p_g[hit] == p_ro[hit])
        changed = int(np.sum(p_g != p_rtn))
        assert st[1] == changed
        if noise == 2.0 ** -8:  # small wobble: guidance helps and never hurts
            assert np.sum(p_g != p_ro) < np.sum(p_rtn != p_ro)


def _exact_grid_tensor(seed):
    """A tensor whose scaled values are exact: A = 2688 gives s_t = 1, a block
    with max 6 * 2^j gets sb = 2^j and inv = 2^-j, so grid values times 2^j sit
    exactly on the grid.  Returns (bf16 bits, on-grid mask)."""
    rng = np.random.default_rng(seed)
    rows, cols = 8, 64
    x = np.zeros((rows, cols), np.float32)
    grid = np.array(GRID, np.float32)
    on = np.zeros((rows, cols), bool)
    for r in range(rows):
        for b in range(cols // 16):
            j = int(rng.integers(-3, 4))
            blk = rng.choice(grid, 16) * np.float32(2.0 ** j)
            blk[0] = 6.0 * 2.0 ** j
            off = rng.random(16) < 0.4
            off[0] = False
            blk[off] = (rng.uniform(0, 6, off.sum()) * 2.0 ** j).astype(np.float32)
            blk *= rng.choice(np.array([-1, 1], np.float32), 16)
            x[r, 16 * b:16 * b + 16] = blk
            on[r, 16 * b:16 * b + 16] = ~off
    x[0, 0] = 2688.0
    on[0, :16] = False  # that block's scale is 448: not exact
    xb = syn.bf16_bits(x)
    on &= syn.bf16_to_f32(xb) == x  # off-grid draws that BF16 rounding put on-grid
    return xb, on


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_guided_ignores_hints_on_grid(bits):
    xb, on = _exact_grid_tensor(5)
    rows, cols = xb.shape
    n = xb.size
    rc, rs, rt, _ = oracle.quantize_rtn(xb)
    assert rt == 1.0
    rng = np.random.default_rng(bits)
    hints = rng.integers(0, 256, (n * bits + 7) // 8).astype(np.uint8)  # adversarial
    gc, gs, gt, st = oracle.guided_requant(xb, hints, bits)
    c_rtn, c_g = _codes(rc, n).reshape(rows, cols), _codes(gc, n).reshape(rows, cols)
    assert np.array_equal(c_g[on], c_rtn[on])
    a, _ = _scaled_abs(xb, rs, rt)
    exact_on = np.isin(a.reshape(rows, cols), np.array(GRID)) | (a.reshape(rows, cols) >= 6)
    assert np.all(exact_on[on])
    assert st[0] == np.sum(~exact_on)


def test_guided_outside_bracket_count_two_bit():
    xt = syn.random_case((8, 128), 21, "normal")
    xr = syn.random_case((8, 128), 22, "normal")
    n = xt.size
    rc, rs, rt, hints = oracle.quantize_rtn(xr, hint_bits=2)
    tc, ts_, tt, _ = oracle.quantize_rtn(xt)
    gc, _, _, st = oracle.guided_requant(xt, hints, 2)
    a, _ = _scaled_abs(xt, ts_, tt)
    grid = np.array(GRID)
    on_grid = np.isin(a, grid)
    lo = np.searchsorted(grid, a, side="right") - 1
    h = _codes(rc, n) & 3
    consulted = (~on_grid) & (a < 6)
    outside = consulted & (h != (lo & 3)) & (h != ((lo + 1) & 3))
    assert st[0] == consulted.sum()
    assert st[2] == outside.sum()


def test_mismatch_stats_identity_and_constructed_pairs():
    x = syn.random_case((8, 128), 31, "normal")
    n = x.size
    c, s, t, _ = oracle.quantize_rtn(x)
    st = oracle.mismatch_stats(c, s, t, c, s, t, 8, 128)
    assert list(st) == [n, 0, 0, 0, 0, 0, 0, 0]
    flat = _codes(c, n).copy()
    rng = np.random.default_rng(5)
    idx = rng.choice(np.nonzero((flat & 7) < 6)[0], 40, replace=False)
    b = flat.copy()
    b[idx[:30]] += 1                 # 30 adjacent changes (|d| = 1)
    b[idx[30:]] = (b[idx[30:]] & 8) | (((b[idx[30:]] & 7) + 2) & 7)  # 10 changes by 2
    zeros = np.nonzero(flat & 7 == 0)[0]
    b[zeros] ^= 8                    # +0 <-> -0 is not a mismatch
    packed = (b[0::2] | (b[1::2] << 4)).astype(np.uint8)
    st = oracle.mismatch_stats(c, s, t, packed, s, t, 8, 128)
    assert list(st) == [n, 40, 30, 10, 30 + 20, 0, 40, 0]
    s2 = s.copy()
    s2.reshape(-1)[[0, 5]] += 1      # two blocks get another scale
    nz = np.count_nonzero(flat.reshape(-1, 16)[[0, 5]] & 7)
    st = oracle.mismatch_stats(c, s, t, c, s2, t, 8, 128)
    assert list(st) == [n, 0, 0, 0, 0, 2, nz, 0]
    st = oracle.mismatch_stats(c, s, t, c, s, np.float32(t) * np.float32(1.5), 8, 128)
    assert st[6] == np.count_nonzero(flat & 7) and st[1] == 0
    # sign flip of a nonzero code: distance 2m
    b = flat.copy()
    k = int(np.nonzero((flat & 7) == 3)[0][0])
    b[k] ^= 8
    packed = (b[0::2] | (b[1::2] << 4)).astype(np.uint8)
    st = oracle.mismatch_stats(c, s, t, packed, s, t, 8, 128)
    assert list(st[1:5]) == [1, 0, 1, 6]


def test_subnormal_tensor_scale_saturates_nonzero_and_keeps_zeros():
    """A tensor of BF16 subnormals: s_t = A / 2688 is deep in the FP32
    subnormal range and 1 / (sb * s_t) overflows to +inf; every nonzero value
    then takes the top code and zeros keep code sign << 3 (closed form)."""
    rng = np.random.default_rng(21)
    xf = (rng.standard_normal((4, 64)) * 1e-39).astype(np.float32)
    xf[rng.random(xf.shape) < 0.3] = 0.0
    xf[0, :4] = [-0.0, 0.0, 1e-40, -1e-40]
    x = syn.bf16_bits(xf)
    codes, scales, s_t, hints = oracle.quantize_rtn(x, hint_bits=2)
    assert 0 < s_t < 2.0 ** -126
    c = _codes(codes, x.size)
    xb = syn.bf16_to_f32(x).reshape(-1)
    sign = np.signbit(xb).astype(np.uint8) << 3
    assert np.array_equal(c, np.where(xb != 0, sign | 7, sign))
    gc, gs, gt, st = oracle.guided_requant(x, hints, 2)
    assert np.array_equal(gc, codes) and st[0] == 0  # no rounding decisions
