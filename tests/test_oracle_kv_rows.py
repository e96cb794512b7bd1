"""Pins for the oracle's KV-cache layout (TRACE explainer, hyper-parameter
table: the rollout keeps the KV cache in FP4 too), read as one FP32 scale per
row of [tokens x heads, head_dim] (CPU only).

* scaling one row by a power of two scales only that row's scale and keeps its
  codes and block scales (so each row uses its own amax, not the tensor's);
* the largest element of every row takes the top code with block scale 448;
* permuting rows permutes the outputs (no cross-row state);
* guiding a cache by its own hints gives round-to-nearest, and the hint stream
  of each row sits at its block offset;
* a single row equals the tensor quantizer on that row.
"""
import numpy as np
import pytest

import oracle
from train_rollout_alignment_b200 import synthetic as syn


def _kv(tokens, heads, dim, seed, kind="normal"):
    return syn.random_case((tokens * heads, dim), seed, kind)


@pytest.mark.parametrize("dim", [16, 64, 128, 256])
def test_power_of_two_row_scaling_only_moves_that_row_scale(dim):
    x = _kv(8, 4, dim, 11)
    c, s, r, _ = oracle.quantize_rtn_rows(x)
    xf = syn.bf16_to_f32(x).copy()
    k = np.arange(x.shape[0]) % 7 - 3          # a different power of two per row
    xs = syn.bf16_bits((xf * (2.0 ** k)[:, None]).astype(np.float32))
    c2, s2, r2, _ = oracle.quantize_rtn_rows(xs)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)
    assert np.array_equal(r2, (r * (2.0 ** k)).astype(np.float32))


def test_row_max_takes_top_code_with_scale_448():
    x = _kv(16, 2, 128, 12, "heavy")
    c, s, r, _ = oracle.quantize_rtn_rows(x)
    xf = syn.bf16_to_f32(x)
    codes = oracle.unpack_codes(c).reshape(x.shape)
    for row in range(x.shape[0]):
        j = int(np.argmax(np.abs(xf[row])))
        assert codes[row, j] & 7 == 7
        assert s[row, j // 16] == 0x7E
        assert np.float32(r[row]) == np.float32(np.float32(np.abs(xf[row]).max()) / np.float32(2688))


def test_rows_are_independent():
    x = _kv(12, 4, 64, 13, "outlier")
    perm = np.random.default_rng(0).permutation(x.shape[0])
    c, s, r, h = oracle.quantize_rtn_rows(x, 2)
    cp, sp, rp, hp = oracle.quantize_rtn_rows(np.ascontiguousarray(x[perm]), 2)
    assert np.array_equal(cp, c[perm]) and np.array_equal(sp, s[perm]) and np.array_equal(rp, r[perm])
    hb = 64 * 2 // 8
    assert np.array_equal(hp.reshape(-1, hb), h.reshape(-1, hb)[perm])


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_guided_by_own_hints_is_rtn_and_rows_match_the_tensor_quantizer(bits):
    x = _kv(10, 3, 128, 14)
    c, s, r, h = oracle.quantize_rtn_rows(x, bits)
    gc, gs, gr, st = oracle.guided_requant_rows(x, h, bits)
    assert np.array_equal(gc, c) and np.array_equal(gs, s) and np.array_equal(gr, r)
    assert st[1] == 0  # nothing changed
    row = 7
    tc, ts, tt, th = oracle.quantize_rtn(np.ascontiguousarray(x[row:row + 1]), hint_bits=bits)
    assert np.array_equal(tc[0], c[row]) and np.array_equal(ts[0], s[row]) and np.float32(tt) == r[row]
    hb = 128 * bits // 8
    assert np.array_equal(th, h[row * hb:(row + 1) * hb])
