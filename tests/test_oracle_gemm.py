"""Pins for the oracle's NVFP4 GEMM of the rollout producer ("Thinking Machines
Lab releases 4-bit training", configuration paragraph: the MoE forward GEMMs
run in NVFP4) and for the tensor-core scale-factor layout (CPU only).

GEMM, D = dec(A) dec(B)^T:
* equals numpy's float64 matmul of the blockwise-dequantized operands (exact
  there for k <= 512) times s_a s_b;
* closed forms: all-ones operands give k s_a s_b; one-hot operands give the
  single product;
* D(A, B) = D(B, A)^T, so neither operand is read transposed;
* dabs = |D| when every term is positive, and dabs >= |D| always.

Scale layout (the hardware's contract, not the pages'): parity unpinned on the
CPU beyond structure -- every 512-byte tile holds exactly the scales of its
128 rows x 4 columns, tiles are ordered column tile fastest, padding is zero,
and each 16-byte lane group holds 4 rows 32 apart.  The tensor core pins it on
the GPU: its block-scaled MMA fed scales in this layout must reproduce the
oracle GEMM of the row-layout scales.
"""
import numpy as np
import pytest

import oracle
from train_rollout_alignment_b200 import synthetic as syn

E4M3_ONE = 0x38      # 1.0
E4M3_TWO = 0x40      # 2.0
E4M3_HALF = 0x30     # 0.5


def _nvfp4(rows, cols, seed, kind="normal"):
    x = syn.random_case((rows, cols), seed, kind)
    codes, scales, ts, _ = oracle.quantize_rtn(x)
    return codes, scales, ts


def _dequant_unit(codes, scales, rows, cols):
    """Dequantized values without the tensor scale (exact in FP32)."""
    return oracle.dequant(codes, scales, 1.0, rows * cols).reshape(rows, cols).astype(np.float64)


@pytest.mark.parametrize("m,n,k", [(16, 32, 64), (40, 24, 256), (8, 8, 512)])
def test_gemm_matches_float64_matmul_of_dequantized_operands(m, n, k):
    ca, sa, ta = _nvfp4(m, k, 101 + m)
    cb, sb, tb = _nvfp4(n, k, 202 + n, "heavy")
    d, dabs = oracle.gemm_nvfp4(ca, sa, ta, cb, sb, tb, m, n, k)
    A = _dequant_unit(ca, sa, m, k)
    B = _dequant_unit(cb, sb, n, k)
    st = float(ta) * float(tb)                 # exact in double
    ref = (A @ B.T) * st
    assert np.allclose(d, ref, rtol=1e-15, atol=0.0)
    assert np.allclose(dabs, (np.abs(A) @ np.abs(B).T) * abs(st), rtol=1e-15, atol=0.0)
    assert np.all(dabs >= np.abs(d) * (1 - 1e-15))


def test_gemm_all_ones_closed_form():
    m, n, k = 4, 6, 128
    a = np.full(m * k // 2, 0x22, np.uint8)            # every element code 2 = 1.0
    b = np.full(n * k // 2, 0x22, np.uint8)
    sa = np.full(m * k // 16, E4M3_ONE, np.uint8)
    sb = np.full(n * k // 16, E4M3_ONE, np.uint8)
    d, dabs = oracle.gemm_nvfp4(a, sa, 0.5, b, sb, 0.25, m, n, k)
    assert np.all(d == k * 0.125) and np.all(dabs == k * 0.125)


def test_gemm_one_hot_closed_form():
    m, n, k = 3, 5, 64
    a = np.zeros(m * k // 2, np.uint8)
    b = np.zeros(n * k // 2, np.uint8)
    sa = np.full(m * k // 16, E4M3_TWO, np.uint8)
    sb = np.full(n * k // 16, E4M3_HALF, np.uint8)
    ea = [5, 17, 40]          # the nonzero element of each A row
    eb = [17, 5, 40, 41, 5]   # ... of each B row
    for i, e in enumerate(ea):
        idx = i * k + e
        a[idx // 2] |= 7 << (4 * (idx % 2))             # +6
    for j, e in enumerate(eb):
        idx = j * k + e
        b[idx // 2] |= 0xD << (4 * (idx % 2))           # -3
    d, _ = oracle.gemm_nvfp4(a, sa, 1.0, b, sb, 1.0, m, n, k)
    want = np.array([[(6 * 2) * (-3 * 0.5) if ea[i] == eb[j] else 0.0 for j in range(n)]
                     for i in range(m)])
    assert np.array_equal(d, want)


def test_gemm_swapping_operands_transposes():
    m, n, k = 24, 40, 192
    ca, sa, ta = _nvfp4(m, k, 7)
    cb, sb, tb = _nvfp4(n, k, 8, "outlier")
    d1, a1 = oracle.gemm_nvfp4(ca, sa, ta, cb, sb, tb, m, n, k)
    d2, a2 = oracle.gemm_nvfp4(cb, sb, tb, ca, sa, ta, n, m, k)
    assert np.array_equal(d1, d2.T) and np.array_equal(a1, a2.T)


def test_gemm_sign_bits_flip_the_terms():
    m, n, k = 8, 8, 64
    ca, sa, ta = _nvfp4(m, k, 31)
    cb, sb, tb = _nvfp4(n, k, 32)
    d, _ = oracle.gemm_nvfp4(ca, sa, ta, cb, sb, tb, m, n, k)
    neg = np.frombuffer(ca, np.uint8) ^ 0x88                # negate every element of A
    dn, _ = oracle.gemm_nvfp4(neg, sa, ta, cb, sb, tb, m, n, k)
    assert np.array_equal(dn, -d)


# ----------------------------------------------------------------- scale layout
def _labelled(rows, sf_cols):
    r, c = np.meshgrid(np.arange(rows), np.arange(sf_cols), indexing="ij")
    return ((r * 7 + c * 13) % 251 + 1).astype(np.uint8)   # never 0, so padding shows


@pytest.mark.parametrize("rows,sf_cols", [(128, 4), (256, 12), (200, 6), (1, 1), (130, 5)])
def test_scale_layout_tiles_hold_their_rows_and_columns(rows, sf_cols):
    s = _labelled(rows, sf_cols)
    out = oracle.scales_to_mma(s, rows, sf_cols)
    rt_n, kt_n = (rows + 127) // 128, (sf_cols + 3) // 4
    assert out.size == rt_n * kt_n * 512
    for rt in range(rt_n):
        for kt in range(kt_n):
            tile = out[(rt * kt_n + kt) * 512:(rt * kt_n + kt + 1) * 512]
            block = s[rt * 128:(rt + 1) * 128, kt * 4:(kt + 1) * 4]
            want = np.sort(np.concatenate([block.reshape(-1),
                                           np.zeros(512 - block.size, np.uint8)]))
            assert np.array_equal(np.sort(tile), want)


def test_scale_layout_lane_groups_hold_rows_32_apart():
    rows, sf_cols = 128, 4
    s = np.zeros((rows, sf_cols), np.uint8)
    for lane in (0, 5, 31):
        s[:] = 0
        s[[lane, lane + 32, lane + 64, lane + 96], :] = np.arange(1, 17, dtype=np.uint8).reshape(4, 4)
        out = oracle.scales_to_mma(s, rows, sf_cols)
        nz = np.nonzero(out)[0]
        assert nz.min() == 16 * lane and nz.max() == 16 * lane + 15
        # the 4 scales of one row are adjacent and in column order
        assert np.array_equal(out[16 * lane:16 * lane + 16], np.arange(1, 17, dtype=np.uint8))


def test_scale_layout_padding_is_zero():
    rows, sf_cols = 70, 3
    out = oracle.scales_to_mma(_labelled(rows, sf_cols), rows, sf_cols)
    assert out.size == 512 and np.count_nonzero(out) == rows * sf_cols


# ----------------------------------------------------------------- MoE form
def test_moe_gemm_is_the_plain_gemm_per_expert_block():
    n, k = 24, 128
    rows = [0, 16, 16, 48, 56]          # expert 1 has no tokens
    m = rows[-1]
    ca, sa, ta = _nvfp4(m, k, 51)
    ws = [_nvfp4(n, k, 60 + e, "heavy") for e in range(4)]
    d, dabs = oracle.moe_gemm_nvfp4(ca, sa, ta, [w[0] for w in ws], [w[1] for w in ws],
                                    [w[2] for w in ws], rows, n, k)
    A = _dequant_unit(ca, sa, m, k)
    for e in range(4):
        r0, r1 = rows[e], rows[e + 1]
        B = _dequant_unit(ws[e][0], ws[e][1], n, k)
        want = (A[r0:r1] @ B.T) * (float(ta) * float(ws[e][2]))
        assert np.allclose(d[r0:r1], want, rtol=1e-15, atol=0.0)


def test_moe_gemm_with_one_expert_is_the_plain_gemm():
    m, n, k = 32, 16, 64
    ca, sa, ta = _nvfp4(m, k, 71)
    cb, sb, tb = _nvfp4(n, k, 72)
    d1, a1 = oracle.gemm_nvfp4(ca, sa, ta, cb, sb, tb, m, n, k)
    d2, a2 = oracle.moe_gemm_nvfp4(ca, sa, ta, [cb], [sb], [tb], [0, m], n, k)
    assert np.array_equal(d1, d2) and np.array_equal(a1, a2)


@pytest.mark.parametrize("case", range(12))
def test_gemm_random_shapes_and_kinds(case):
    rng = np.random.Generator(np.random.PCG64(900 + case))
    kinds = ["normal", "heavy", "outlier", "tiny", "sparse", "ties", "zeros"]
    m, n = int(rng.integers(1, 24)), int(rng.integers(1, 24))
    k = 16 * int(rng.integers(1, 24))                  # ragged: any multiple of 16 up to 368
    ca, sa, ta = _nvfp4(m, k, 1000 + case, kinds[case % len(kinds)])
    cb, sb, tb = _nvfp4(n, k, 2000 + case, kinds[(case + 3) % len(kinds)])
    d, dabs = oracle.gemm_nvfp4(ca, sa, ta, cb, sb, tb, m, n, k)
    A = _dequant_unit(ca, sa, m, k)
    B = _dequant_unit(cb, sb, n, k)
    st = float(ta) * float(tb)
    assert np.allclose(d, (A @ B.T) * st, rtol=1e-15, atol=0.0)
    assert np.allclose(dabs, (np.abs(A) @ np.abs(B).T) * abs(st), rtol=1e-15, atol=0.0)


# ----------------------------------------------------------------- dispatch
def test_moe_route_worked_example():
    """3 tokens, top-2, 3 experts, worked by hand: assignments a = 2 t + j
    with experts [[1, 0], [1, 2], [0, 1]] -> expert 0 gets a = 1, 4; expert 1
    a = 0, 2, 5; expert 2 a = 3; each group padded to 128 rows."""
    rows, src, arow = oracle.moe_route([[1, 0], [1, 2], [0, 1]], 3)
    assert list(rows) == [0, 128, 256, 384]
    assert list(src[:2]) == [1, 4] and list(src[128:131]) == [0, 2, 5] and src[256] == 3
    assert np.all(src[2:128] == -1) and np.all(src[131:256] == -1) and np.all(src[257:] == -1)
    assert list(arow) == [128, 0, 129, 256, 1, 130]


def test_moe_route_invariants():
    rng = np.random.Generator(np.random.PCG64(5))
    tokens, top_k, E = 500, 3, 7
    ids = rng.integers(-1, E + 1, (tokens, top_k))     # some ids out of range: dropped
    rows, src, arow = oracle.moe_route(ids, E)
    flat = ids.reshape(-1)
    assert rows[0] == 0 and np.all(np.diff(rows) % 128 == 0) and np.all(np.diff(rows) >= 0)
    for e in range(E):
        grp = src[rows[e]:rows[e + 1]]
        real = grp[grp >= 0]
        assert np.array_equal(real, np.nonzero(flat == e)[0])      # all of expert e, in order
        assert np.all(grp[real.size:] == -1) and rows[e + 1] - rows[e] - real.size < 128
    ok = (flat >= 0) & (flat < E)
    assert np.all(arow[~ok] == -1)
    assert np.array_equal(src[arow[ok]], np.nonzero(ok)[0])        # the inverse permutation
    assert rows[-1] <= ((ok.sum() + 127 * E + 127) // 128) * 128
