"""The dispatch half of the rollout producer on one GPU ("Thinking Machines
Lab releases 4-bit training": tokens reach the experts in NVFP4 and the MoE
forward runs in NVFP4), through the C ABI: the grouping of the routed tokens
by expert equals the oracle's (a stable counting sort, so row for row), the
gather of their NVFP4 rows equals the oracle's grouped rows and scale layout
byte for byte, and the expert GEMM over the gathered rows -- launched with the
grouping's capacity as m, the real row count read on the GPU -- matches the
oracle's MoE GEMM (D within the accumulation bound, its quantization bit-exact)
and leaves the rows past the grouping untouched."""
import numpy as np
import pytest
import torch

import oracle
from train_rollout_alignment_b200 import synthetic as syn

from _gpu_util import Buf, f32_bits, lib

pytestmark = pytest.mark.gpu


def _route(ids, E):
    b = lib()
    tokens, top_k = ids.shape
    A = tokens * top_k
    cap = b.nvfp4_moe_rows_cap(A, E)
    ws = torch.full((b.nvfp4_moe_route_ws_words(A, E),), 12345, dtype=torch.int32, device="cuda")
    rows = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    src = torch.full((cap,), -7, dtype=torch.int32, device="cuda")
    arow = torch.full((max(A, 1),), -7, dtype=torch.int32, device="cuda")
    b.nvfp4_moe_route(torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda(), E, ws, rows, src,
                      arow[:A] if A else arow)
    torch.cuda.synchronize()
    return rows.cpu().numpy(), src.cpu().numpy(), arow.cpu().numpy()[:A], cap


@pytest.mark.parametrize("tokens,top_k,E", [(1, 1, 1), (300, 2, 5), (5000, 2, 128), (4099, 8, 1024),
                                            (777, 3, 7), (0, 2, 4)])
def test_route_matches_oracle(tokens, top_k, E):
    rng = np.random.Generator(np.random.PCG64(tokens + E))
    ids = rng.integers(-1, E + 1, (tokens, top_k)).astype(np.int32)   # some out of range: dropped
    if tokens > 1000:  # skewed load: a few hot experts
        hot = rng.random((tokens, top_k)) < 0.5
        ids[hot] = rng.integers(0, min(E, 3), int(hot.sum()))
    rows, src, arow, cap = _route(ids, E)
    o_rows, o_src, o_arow = oracle.moe_route(ids, E)
    assert list(rows) == list(o_rows)
    assert np.array_equal(src[:o_rows[-1]], o_src)
    assert np.all(src[o_rows[-1]:] == -1) and src.size == cap
    assert np.array_equal(arow, o_arow)
    # the same call again gives the same rows
    rows2, src2, arow2, _ = _route(ids, E)
    assert np.array_equal(src, src2) and np.array_equal(arow, arow2)


def _tokens(tokens, k, seed):
    x = syn.random_case((tokens, k), seed, "heavy")
    codes, scales, ts, _ = oracle.quantize_rtn(x)
    return codes, scales, np.float32(ts)


@pytest.mark.parametrize("tokens,top_k,E,k", [(200, 2, 3, 256), (1000, 4, 16, 512)])
def test_gather_matches_oracle_grouping(tokens, top_k, E, k):
    b = lib()
    rng = np.random.Generator(np.random.PCG64(k))
    ids = rng.integers(0, E, (tokens, top_k)).astype(np.int32)
    codes, scales, _ = _tokens(tokens, k, 3)
    rows, src, arow, cap = _route(ids, E)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    src_d = torch.from_numpy(src).cuda()
    ac, asf = Buf(cap * k // 2), Buf(b.mma_scale_bytes(cap, k // 16))
    b.nvfp4_moe_gather(d(codes), d(scales), tokens, k, src_d, top_k, ac.t, asf.t)
    torch.cuda.synchronize()
    tok = np.where(src >= 0, src // top_k, -1)
    want_c = np.zeros((cap, k // 2), np.uint8)
    want_s = np.zeros((cap, k // 16), np.uint8)
    want_c[tok >= 0] = codes.reshape(tokens, k // 2)[tok[tok >= 0]]
    want_s[tok >= 0] = scales.reshape(tokens, k // 16)[tok[tok >= 0]]
    assert np.array_equal(ac.np().reshape(cap, k // 2), want_c)
    assert np.array_equal(asf.np(), oracle.scales_to_mma(want_s, cap, k // 16))


def test_route_gather_expert_gemm_end_to_end():
    b = lib()
    tokens, top_k, E, n, k = 700, 2, 6, 256, 512
    rng = np.random.Generator(np.random.PCG64(11))
    ids = rng.integers(0, E, (tokens, top_k)).astype(np.int32)
    ids[rng.random((tokens, top_k)) < 0.05] = -1                  # a few dropped slots
    codes, scales, ta = _tokens(tokens, k, 21)
    experts = [oracle.quantize_rtn(syn.random_case((n, k), 30 + e, "normal")) for e in range(E)]
    rows, src, arow, cap = _route(ids, E)
    # oracle side: the grouped A from the oracle's own routing, its MoE GEMM
    o_rows, o_src, _ = oracle.moe_route(ids, E)
    m = int(o_rows[-1])
    tok = np.where(o_src >= 0, o_src // top_k, -1)
    ga = np.zeros((m, k // 2), np.uint8)
    gs = np.zeros((m, k // 16), np.uint8)
    ga[tok >= 0] = codes.reshape(tokens, k // 2)[tok[tok >= 0]]
    gs[tok >= 0] = scales.reshape(tokens, k // 16)[tok[tok >= 0]]
    d_ref, dabs = oracle.moe_gemm_nvfp4(ga, gs, ta, [w[0] for w in experts], [w[1] for w in experts],
                                        [w[2] for w in experts], o_rows, n, k)
    a_out = np.float32(np.abs(d_ref).max())
    # GPU side: route -> gather -> expert GEMM with m = the capacity
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda()
    ac, asf = Buf(cap * k // 2), Buf(b.mma_scale_bytes(cap, k // 16))
    b.nvfp4_moe_gather(d(codes), d(scales), tokens, k, torch.from_numpy(src).cuda(), top_k, ac.t, asf.t)
    w_codes = np.concatenate([np.asarray(w[0]).reshape(n, k // 2) for w in experts])
    w_sc = np.concatenate([np.asarray(w[1]).reshape(n, k // 16) for w in experts])
    wsf = Buf(b.mma_scale_bytes(E * n, k // 16))
    b.nvfp4_scales_to_mma(d(w_sc), E * n, k // 16, wsf.t)
    w_ts = np.array([w[2] for w in experts], np.float32)
    ws = torch.zeros(8, dtype=torch.int32, device="cuda")
    ws[0] = np.int32(np.uint32(f32_bits(a_out)).view(np.int32))
    oc, osc = Buf(cap * n // 2), Buf(cap * n // 16)
    osm = Buf(b.mma_scale_bytes(cap, n // 16))
    ots, oh = Buf(4, torch.float32), Buf(cap * n // 4)
    dd = Buf(4 * cap * n, torch.float32)
    for t in (oc, osc, oh, dd):
        t.raw[:t.raw.numel() - 256].fill_(0xAB)
    b.nvfp4_moe_gemm_quantize(ac.t, asf.t, d(np.array([ta], np.float32)), d(w_codes), wsf.t, d(w_ts),
                              torch.from_numpy(rows).cuda(), E, cap, n, k, ws, oc.t, osc.t, ots.t,
                              scales_mma=osm.t, hints=oh.t, hint_bits=2, d_out=dd.t)
    torch.cuda.synchronize()
    D = dd.np().reshape(cap, n)
    assert np.all(np.abs(D[:m].astype(np.float64) - d_ref) <= (k / 16) * 2.0 ** -22 * dabs + 2.0 ** -23 * np.abs(d_ref))
    qc, qs, qt = oracle.quantize_f32(np.ascontiguousarray(D[:m]), a_out)
    assert np.array_equal(oc.np().reshape(cap, n // 2)[:m], qc)
    assert np.array_equal(osc.np().reshape(cap, n // 16)[:m], qs)
    assert np.array_equal(oh.np().reshape(cap, n // 4)[:m], oracle.emit_hint(qc, m * n, 2).reshape(m, n // 4))
    # rows past the grouping were not computed: their bytes are as they were
    assert np.all(oc.np().reshape(cap, n // 2)[m:] == 0xAB)
    assert np.all(dd.np().view(np.uint8).reshape(cap, 4 * n)[m:] == 0xAB)
    assert int(ws.cpu().numpy().view(np.uint32)[1]) == 0
    # every token slot's product row is where assign_row says
    assert np.array_equal(arow, oracle.moe_route(ids, E)[2])
