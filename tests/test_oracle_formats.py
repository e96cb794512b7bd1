"""Pins for the oracle's number formats (CPU only).

E2M1 and E4M3 rounding are checked against the ``ml_dtypes`` library casts
(float4_e2m1fn, float8_e4m3fn), which implement the OCP formats with
round-to-nearest-even; decoding against the same library; the dequantization
rule against the worked example of "Quantization in RL training"
(shared-convention paragraph: code 3 x scale 0.1 = 0.3, x scale 0.2 = 0.6).
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ml_e2m1_index(values: np.ndarray) -> np.ndarray:
    q = values.astype(np.float32).astype(ml_dtypes.float4_e2m1fn)
    return q.view(np.uint8) & 7


def _midpoints_and_neighbours(points):
    pts = np.asarray(points, np.float32)
    mids = ((pts[:-1].astype(np.float64) + pts[1:]) / 2).astype(np.float32)
    out = [mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0))]
    out += [pts, np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))]
    return np.concatenate(out)


def test_e2m1_grid_matches_library_decode():
    dec = np.arange(8, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    assert [oracle.e2m1_value(m) for m in range(8)] == list(dec)
    assert len(set(dec.tolist() + (-dec).tolist())) == 15  # 16 codes, +0 and -0 coincide


def test_e2m1_rne_all_bf16_magnitudes_vs_library():
    bits = np.arange(0, 0x7F80, dtype=np.uint32)  # every finite non-negative BF16
    base = (bits << 16).view(np.float32)
    vals = np.concatenate([base[base <= 64.0] * np.float32(f) for f in (1.0, 0.3, 1.7, 5.3, 0.011)])
    vals = np.concatenate([vals, _midpoints_and_neighbours([0, .5, 1, 1.5, 2, 3, 4, 6]),
                           np.array([6.0, 6.5, 7.0, 1e30, np.float32(np.inf)], np.float32)])
    want = _ml_e2m1_index(np.minimum(vals, np.float32(6.0)))
    got = np.array([oracle.e2m1_rne(v) for v in vals], np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, list(zip(vals[bad][:8], got[bad][:8], want[bad][:8]))


def test_e2m1_ties_go_to_even_index():
    # midpoints: 0.25 0.75 1.25 1.75 2.5 3.5 5 -> indices 0 2 2 4 4 6 6
    assert [oracle.e2m1_rne(v) for v in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)] == [0, 2, 2, 4, 4, 6, 6]


def test_e4m3_decode_vs_library():
    for b in range(256):
        if (b & 0x7F) == 0x7F:
            continue  # NaN encodings
        lib = float(np.array([b], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)[0])
        assert oracle.e4m3_value(b) == lib, b
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_rne_satfinite_vs_library():
    rng = np.random.default_rng(11)
    rand = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(460.0), 60000)).astype(np.float32)
    finite = np.array([oracle.e4m3_value(b) for b in range(0x7F)], np.float64)
    vals = np.concatenate([rand, _midpoints_and_neighbours(finite), np.float32([0.0, 2.0 ** -10, 2.0 ** -11])])
    vals = vals[vals <= 460.0]
    want = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = np.array([oracle.e4m3_rne_satfinite(v) for v in vals], np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, list(zip(vals[bad][:8], got[bad][:8], want[bad][:8]))


def test_e4m3_saturates_instead_of_overflowing():
    for v in (448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3.4e38, float("inf")):
        assert oracle.e4m3_rne_satfinite(v) == 0x7E


def test_dequant_code_times_scale_worked_example():
    ex = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["rlq_code_times_scale"]
    m = [k for k in range(8) if oracle.e2m1_value(k) == ex["code_value"]][0]
    one = oracle.e4m3_rne_satfinite(1.0)
    assert oracle.e4m3_value(one) == 1.0
    for scale, expect in ex["cases"]:
        got = oracle.dequant_one(m, one, np.float32(scale))
        assert got == pytest.approx(expect, rel=2 ** -23)
        assert oracle.dequant_one(m | 8, one, np.float32(scale)) == -got
    # same code, different scale -> different value
    assert oracle.dequant_one(m, one, 0.1) != oracle.dequant_one(m, one, 0.2)


def test_storage_is_four_and_a_half_bits_per_value():
    ex = json.load(open(os.path.join(GOLDEN, "worked_examples.json")))["format_bits_per_value"]
    rows, cols = 4, 64
    x = np.zeros((rows, cols), np.uint16)
    codes, scales, _, _ = oracle.quantize_rtn(x)
    bits = (codes.nbytes + scales.nbytes) * 8 / (rows * cols)
    assert bits == ex["bits_per_value"]
    assert cols // scales.shape[1] == ex["values_per_scale"]
