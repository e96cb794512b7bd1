"""Helpers for the GPU parity tests: run the CUDA path through the C ABI on
host-generated inputs, with sentinel-filled outputs and canary tails that catch
unwritten bytes and out-of-bounds writes.  The binding is imported lazily so the
CPU-only test run never needs the GPU."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle

CANARY = 0xAB
TAIL = 256


def lib():
    from train_rollout_alignment_b200 import _binding
    return _binding


def pool(n_tasks: int):
    return ThreadPoolExecutor(max_workers=max(1, min(n_tasks, len(os.sched_getaffinity(0)))))


def dev_bf16(x) -> torch.Tensor:
    if isinstance(x, torch.Tensor):
        return x
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16
    return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()


def to_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class Buf:
    """A device byte buffer with a canary tail; .t is the exact-size view."""

    def __init__(self, nbytes: int, dtype=torch.uint8):
        item = torch.empty((), dtype=dtype).element_size()
        self.n = nbytes // item
        self.raw = torch.full((nbytes + TAIL,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[:nbytes].view(dtype)

    def check_tail(self):
        tail = self.raw[self.raw.numel() - TAIL:].cpu().numpy()
        assert np.all(tail == CANARY), "write past the end of an output buffer"

    def np(self):
        self.check_tail()
        return self.t.cpu().numpy()


def f32_bits(v) -> int:
    return int(np.float32(v).view(np.uint32))


def gpu_rtn(x, hint_bits: int = 0, ws=None, flags: int = 0):
    b = lib()
    xt = dev_bf16(x)
    rows, cols = xt.shape
    n = rows * cols
    codes, scales, ts = Buf(n // 2), Buf(n // 16), Buf(4, torch.float32)
    ws = ws if ws is not None else torch.zeros(8, dtype=torch.int32, device="cuda")
    hints = Buf((n * hint_bits + 7) // 8) if hint_bits else None
    b.nvfp4_quantize_rtn(xt, ws, codes.t, scales.t, ts.t, hints.t if hints else None, hint_bits, flags)
    torch.cuda.synchronize()
    return dict(codes=codes.np().reshape(rows, cols // 2), scales=scales.np().reshape(rows, cols // 16),
                ts=float(ts.np()[0]), hints=hints.np() if hints else None, ws=ws.cpu().numpy())


def gpu_guided(x, hints_np, hint_bits: int, with_stats: bool = True):
    b = lib()
    xt = dev_bf16(x)
    rows, cols = xt.shape
    n = rows * cols
    codes, scales, ts = Buf(n // 2), Buf(n // 16), Buf(4, torch.float32)
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    hints = torch.from_numpy(np.ascontiguousarray(hints_np)).cuda() if hints_np is not None else None
    stats = torch.zeros(4, dtype=torch.int64, device="cuda") if with_stats else None
    b.nvfp4_guided_requant(xt, hints, hint_bits, ws, codes.t, scales.t, ts.t, stats)
    torch.cuda.synchronize()
    return dict(codes=codes.np().reshape(rows, cols // 2), scales=scales.np().reshape(rows, cols // 16),
                ts=float(ts.np()[0]), stats=stats.cpu().numpy().astype(np.uint64) if with_stats else None)


def gpu_emit_hint(codes_np, n: int, hint_bits: int):
    b = lib()
    codes = torch.from_numpy(np.ascontiguousarray(codes_np).reshape(-1)).cuda()
    hints = Buf((n * hint_bits + 7) // 8)
    b.nvfp4_emit_hint(codes, n, hint_bits, hints.t)
    torch.cuda.synchronize()
    return hints.np()


def gpu_stats(ca, sa, ta, cb, sb, tb, rows, cols):
    b = lib()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    tsa = torch.tensor([ta], dtype=torch.float32, device="cuda")
    tsb = torch.tensor([tb], dtype=torch.float32, device="cuda")
    stats = torch.zeros(8, dtype=torch.int64, device="cuda")
    b.nvfp4_mismatch_stats(dev(ca), dev(sa), tsa, dev(cb), dev(sb), tsb, rows, cols, stats)
    torch.cuda.synchronize()
    return stats.cpu().numpy().astype(np.uint64)


def gpu_sr(codes, scales, ts, batch, rows, cols, seed, draw):
    b = lib()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    n = batch * rows * cols
    ct, st, tst = Buf(n // 2), Buf(n // 16), Buf(4 * batch, torch.float32)
    ws = torch.zeros(max(batch, 8), dtype=torch.int32, device="cuda")
    b.nvfp4_sr_transpose_requant(dev(codes), dev(scales), dev(np.asarray(ts, np.float32)), batch, rows,
                                 cols, seed, draw, ws, ct.t, st.t, tst.t)
    torch.cuda.synchronize()
    return (ct.np().reshape(batch, cols, rows // 2), st.np().reshape(batch, cols, rows // 16),
            tst.np().reshape(batch))


def gpu_rht(x, seed: int, want_y: bool = True):
    b = lib()
    xt = dev_bf16(x)
    rows, cols = xt.shape
    n = rows * cols
    codes, scales, ts = Buf(n // 2), Buf(n // 16), Buf(4, torch.float32)
    y = Buf(4 * n, torch.float32) if want_y else None
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    b.nvfp4_rht_quantize(xt, seed, ws, codes.t, scales.t, ts.t, y.t if y else None)
    torch.cuda.synchronize()
    return dict(codes=codes.np().reshape(rows, cols // 2), scales=scales.np().reshape(rows, cols // 16),
                ts=float(ts.np()[0]), y=y.np().reshape(rows, cols) if y else None, ws=ws.cpu().numpy())


def assert_codes_equal(got, want, what="codes"):
    got, want = np.asarray(got), np.asarray(want)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        i = tuple(bad[0])
        raise AssertionError("%s differ at %d places; first %s: got 0x%02x want 0x%02x"
                             % (what, len(bad), i, got[i], want[i]))


def oracle_rtn_parallel(x, A, hint_bits=0, chunks=16):
    """Oracle RTN over row chunks on a thread pool (same tensor amax A)."""
    rows = x.shape[0]
    step = max(1, (rows + chunks - 1) // chunks)
    parts = [x[r:r + step] for r in range(0, rows, step)]
    with pool(len(parts)) as ex:
        outs = list(ex.map(lambda p: oracle.quantize_rtn(p, A, hint_bits), parts))
    codes = np.concatenate([o[0] for o in outs])
    scales = np.concatenate([o[1] for o in outs])
    hints = np.concatenate([o[3] for o in outs]) if hint_bits else None
    return codes, scales, outs[0][2], hints


def oracle_guided_parallel(x, hints, hint_bits, A, chunks=16):
    rows, cols = x.shape
    step = max(1, (rows + chunks - 1) // chunks)
    # hint bytes per row chunk: step * cols * bits / 8 (cols % 16 == 0 keeps it whole)
    hb = lambda r0, r1: None if hints is None else hints[r0 * cols * hint_bits // 8:r1 * cols * hint_bits // 8]
    parts = [(x[r:r + step], hb(r, min(rows, r + step))) for r in range(0, rows, step)]
    with pool(len(parts)) as ex:
        outs = list(ex.map(lambda p: oracle.guided_requant(p[0], p[1], hint_bits, A), parts))
    codes = np.concatenate([o[0] for o in outs])
    scales = np.concatenate([o[1] for o in outs])
    stats = np.sum([o[3] for o in outs], axis=0).astype(np.uint64)
    return codes, scales, outs[0][2], stats


# ----------------------------------------------------------------- RHT tolerance rule
_E4M3_VALUES = None


def _e4m3_midpoints():
    global _E4M3_VALUES
    if _E4M3_VALUES is None:
        e4 = np.array([oracle.e4m3_value(k) for k in range(127)], np.float64)  # 0 .. 448
        _E4M3_VALUES = (e4, (e4[:-1] + e4[1:]) / 2)
    return _E4M3_VALUES


_E2M1_MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _nearest_dist(vals, mids):
    """Distance of each value to the nearest entry of the sorted array mids."""
    j = np.clip(np.searchsorted(mids, vals), 1, len(mids) - 1)
    return np.minimum(np.abs(vals - mids[j - 1]), np.abs(vals - mids[j]))


def rht_boundary_check(x_rows, yd_rows, oc, osc, ot, g_codes, g_scales, g_ts):
    """The RHT tolerance rule against the full double-precision oracle, on a
    row range: the transform may differ from the double one by
    tol = 1e-6 * ||x_group||_2 per element, so
      * a block scale may differ only where the oracle's (amax_b / 6) / s_t is
        within that tolerance (carried into the scale domain) of an E4M3
        rounding midpoint;
      * in a block whose scale agrees, a code may differ (as a signed grid
        position: +0 and -0 are one value) only where the oracle's |v| is
        within the tolerance (carried into v) of an E2M1 midpoint.
    A difference between the two tensor scales (they come from the two
    transforms' maxima) widens both by its relative size.
    x_rows: BF16 bits [r, cols]; yd_rows: the double transform [r, cols];
    oc/osc: the oracle's codes/scales of these rows (of y = fl32(yd)), ot its
    tensor scale; g_*: the GPU's.  -> (scale diffs, code diffs); raises on a
    difference away from a boundary."""
    from train_rollout_alignment_b200 import synthetic as syn
    e4, e4_mid = _e4m3_midpoints()
    norm = np.linalg.norm(syn.bf16_to_f32(x_rows).astype(np.float64).reshape(-1, 32), axis=1)
    tol_y = 1e-6 * np.repeat(norm, 2)                       # per 16-block: the bound of its 32-group
    rel_ts = abs(float(g_ts) - float(ot)) / float(ot) + 1e-6
    oy = yd_rows.astype(np.float32).astype(np.float64).reshape(-1, 16)
    amax_b = np.abs(oy).max(axis=1)
    sbf = amax_b / 6.0 / ot
    osc = np.asarray(osc).reshape(-1)
    blk_diff = osc != np.asarray(g_scales).reshape(-1)
    if blk_diff.any():
        d = _nearest_dist(sbf[blk_diff], e4_mid)
        allowed = (tol_y[blk_diff] / 6.0 / ot) * 1.01 + rel_ts * sbf[blk_diff]
        bad = d > allowed
        assert not bad.any(), "%d block scales differ away from an E4M3 boundary" % int(bad.sum())
    pos = lambda c: np.where(c & 8, -(c & 7).astype(np.int8), (c & 7).astype(np.int8))
    pc_o = pos(oracle.unpack_codes(oc)).reshape(-1, 16)
    pc_g = pos(oracle.unpack_codes(g_codes)).reshape(-1, 16)
    diff = (pc_o != pc_g) & ~blk_diff[:, None]
    n_code = int(diff.sum())
    if n_code:
        bi, ki = np.nonzero(diff)
        sbv = e4[osc[bi]]
        assert np.all(sbv > 0), "a code differs in a block whose scale is zero"
        scale = sbv * ot
        a = np.abs(oy[bi, ki]) / scale
        d = _nearest_dist(a, _E2M1_MIDS)
        allowed = tol_y[bi] / scale * 1.01 + rel_ts * a
        bad = d > allowed
        assert not bad.any(), "%d codes differ away from an E2M1 boundary" % int(bad.sum())
    return int(blk_diff.sum()), n_code


def oracle_stats_parallel(ca, sa, ta, cb, sb, tb, rows, cols, chunks=16):
    """Oracle mismatch counters over row chunks (every counter is a sum over rows)."""
    step = max(1, (rows + chunks - 1) // chunks)
    ca, sa = np.asarray(ca).reshape(rows, -1), np.asarray(sa).reshape(rows, -1)
    cb, sb = np.asarray(cb).reshape(rows, -1), np.asarray(sb).reshape(rows, -1)
    parts = [(r, min(rows, r + step)) for r in range(0, rows, step)]
    with pool(len(parts)) as ex:
        outs = list(ex.map(lambda p: oracle.mismatch_stats(ca[p[0]:p[1]], sa[p[0]:p[1]], ta, cb[p[0]:p[1]],
                                                           sb[p[0]:p[1]], tb, p[1] - p[0], cols), parts))
    return np.sum(outs, axis=0).astype(np.uint64)


def amax_parallel(x, chunks=16):
    with pool(chunks) as ex:
        return max(ex.map(oracle.amax_bf16, np.array_split(x, chunks)))


def gpu_guided_stats(x, hints_np, hint_bits: int, roll, stats8_init=None):
    """nvfp4_guided_requant_stats on host inputs; roll = (codes, scales, ts) of
    the rollout side.  -> dict like gpu_guided plus stats8."""
    b = lib()
    xt = dev_bf16(x)
    rows, cols = xt.shape
    n = rows * cols
    codes, scales, ts = Buf(n // 2), Buf(n // 16), Buf(4, torch.float32)
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    hints = torch.from_numpy(np.ascontiguousarray(hints_np)).cuda() if hints_np is not None else None
    stats4 = torch.zeros(4, dtype=torch.int64, device="cuda")
    stats8 = (torch.zeros(8, dtype=torch.int64, device="cuda") if stats8_init is None
              else torch.from_numpy(np.asarray(stats8_init, np.int64)).cuda())
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    rts = torch.tensor([roll[2]], dtype=torch.float32, device="cuda")
    b.nvfp4_guided_requant_stats(xt, hints, hint_bits, ws, codes.t, scales.t, ts.t, stats4, dev(roll[0]),
                                 dev(roll[1]), rts, stats8)
    torch.cuda.synchronize()
    return dict(codes=codes.np().reshape(rows, cols // 2), scales=scales.np().reshape(rows, cols // 16),
                ts=float(ts.np()[0]), stats=stats4.cpu().numpy().astype(np.uint64),
                stats8=stats8.cpu().numpy().astype(np.uint64))
