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


def _nccl_worker(rank, world, port, q):
    import os
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank), NCCL_NVLS_ENABLE="0")
    import torch
    from train_rollout_alignment_b200 import _binding as b
    from train_rollout_alignment_b200 import dist as d
    from train_rollout_alignment_b200 import sharded
    torch.cuda.set_device(rank)
    d.init("nccl", timeout_s=60)
    rows, cols = 256, 512
    x = syn.random_case((rows, cols), 12, "heavy")
    xr = syn.bf16_bits(syn.bf16_to_f32(x) * np.float32(1.0 + 2.0 ** -7))
    per = rows // world
    sl = slice(rank * per, (rank + 1) * per)
    cr, sr, tr, ws, h = b.empty_nvfp4(per, cols, "cuda", hint_bits=2)
    sharded.quantize_rtn(dev_bf16(xr[sl]), ws, cr, sr, tr, h, 2)
    ct, st, tt, ws2, _ = b.empty_nvfp4(per, cols, "cuda")
    s4 = torch.zeros(4, dtype=torch.int64, device="cuda")
    sharded.guided_requant(dev_bf16(x[sl]), h, 2, ws2, ct, st, tt, s4)
    s8 = torch.zeros(8, dtype=torch.int64, device="cuda")
    sharded.mismatch_stats(cr, sr, tr, ct, st, tt, per, cols, s8)
    torch.cuda.synchronize()
    q.put({"rank": rank, "cr": cr.cpu().numpy(), "h": h.cpu().numpy(), "ct": ct.cpu().numpy(),
           "tr": float(tr.item()), "tt": float(tt.item()), "s4": s4.cpu().numpy(), "s8": s8.cpu().numpy()})
    d.finish()


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs two GPUs (NCCL between processes)")
def test_sharded_helpers_over_nccl_on_two_gpus():
    """Two ranks on two GPUs, rows split in halves: the amax all-reduce and
    the counter sums run over NCCL, and every rank's rows equal the oracle's
    rows of the whole tensor."""
    import socket
    import torch.multiprocessing as mp
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_nccl_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted([q.get(timeout=300) for _ in procs], key=lambda o: o["rank"])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    rows, cols = 256, 512
    x = syn.random_case((rows, cols), 12, "heavy")
    xr = syn.bf16_bits(syn.bf16_to_f32(x) * np.float32(1.0 + 2.0 ** -7))
    oc, os_, ot, oh = oracle.quantize_rtn(xr, hint_bits=2)
    gc, gs, gt, gst = oracle.guided_requant(x, oh, 2)
    ost = oracle.mismatch_stats(oc, os_, ot, gc, gs, gt, rows, cols)
    per = rows // 2
    for o in out:
        r = o["rank"]
        assert o["tr"] == ot and o["tt"] == gt
        assert np.array_equal(o["cr"], oc[r * per:(r + 1) * per])
        assert np.array_equal(o["ct"], gc[r * per:(r + 1) * per])
        assert np.array_equal(o["h"], oh[r * per * cols // 4:(r + 1) * per * cols // 4])
        assert list(o["s4"][:3].astype(np.uint64)) == list(gst[:3])
        assert list(o["s8"][:7].astype(np.uint64)) == list(ost[:7])
