"""The multi-GPU plumbing of the benchmark, run as two gloo ranks on CPU:
every rank generates its own layer stack (weak scaling: no data-path
collective), the job time is the max over ranks, and the whole-job rate is the
units all ranks processed divided by that time."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from train_rollout_alignment_b200 import dist as d
    from train_rollout_alignment_b200 import synthetic as syn
    d.init("gloo", timeout_s=60)
    w, r, lr = d.world()
    seconds = 1.0 + 0.5 * r  # this rank's elapsed time
    m = d.max_over_ranks(seconds)
    xt, xr = syn.cfg4_layer_device(3, "cpu", r, shape=(64, 256))
    xt2, _ = syn.cfg4_layer_device(3, "cpu", r, shape=(64, 256))
    q.put({"rank": r, "world": w, "max": m, "rate": d.aggregate_rate(100.0, w, m),
           "sum": float(xt.float().sum()), "again": bool(torch.equal(xt, xt2)),
           "rollout_close": float((xr.float() - xt.float()).abs().max() / xt.float().abs().max())})
    d.finish()


def test_two_gloo_ranks_weak_scaling_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort(key=lambda o: o["rank"])
    assert [o["world"] for o in out] == [2, 2]
    assert all(o["max"] == 1.5 for o in out)          # slowest rank's time
    assert all(o["rate"] == 200.0 / 1.5 for o in out)  # 2 ranks x 100 units / 1.5 s
    assert out[0]["sum"] != out[1]["sum"]               # each rank its own stack
    assert all(o["again"] for o in out)                 # seeded: reproducible
    assert all(o["rollout_close"] < 0.05 for o in out)  # rollout = train x (1 + N(0, 2^-8))
