"""Row sharding of one tensor across ranks (train_rollout_alignment_b200.sharded),
run as two gloo ranks on CPU.  The GPU kernels are replaced by a test double
built from the oracle (the kernels' own parity is the GPU tests' job); what is
checked here is the exchange: the MAX all-reduce of the amax scratch words and
the SUM all-reduce of the counters, so that

* every rank quantizes its rows with the whole tensor's tensor scale, even
  when its own rows have a smaller amax;
* each rank's codes, scales and hints are the rows of the unsharded result;
* the guidance counters and the mismatch counters are the whole tensor's;
* warning bits of any rank reach every rank."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

ROWS, COLS = 64, 256


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class OracleKernels:
    """Stand-in for the C-ABI binding on CPU tensors (test only)."""
    NVFP4_AMAX_PRECOMPUTED = 1

    def __init__(self, warn=0):
        import oracle
        self.o = oracle
        self.warn = warn

    @staticmethod
    def _u16(x):
        return x.contiguous().view(torch.int16).numpy().view(np.uint16)

    @staticmethod
    def _A(ws):
        return float(np.int32(ws[0].item()).view(np.float32))

    def nvfp4_tensor_amax(self, x, ws):
        ws.zero_()
        ws[0] = int(np.float32(self.o.amax_bf16(self._u16(x))).view(np.int32))
        ws[1] = self.warn

    def nvfp4_quantize_rtn(self, x, ws, codes, scales, ts, hints=None, hint_bits=0, flags=0):
        assert flags == self.NVFP4_AMAX_PRECOMPUTED
        c, s, t, h = self.o.quantize_rtn(self._u16(x), A=self._A(ws), hint_bits=hint_bits)
        codes.copy_(torch.from_numpy(c.reshape(codes.shape)))
        scales.copy_(torch.from_numpy(s.reshape(scales.shape)))
        ts.fill_(t)
        if hints is not None:
            hints.copy_(torch.from_numpy(h.reshape(hints.shape)))

    def nvfp4_guided_requant(self, x, hints, hint_bits, ws, codes, scales, ts, stats4=None, flags=0):
        assert flags == self.NVFP4_AMAX_PRECOMPUTED
        c, s, t, st = self.o.guided_requant(self._u16(x), hints.numpy(), hint_bits, A=self._A(ws))
        codes.copy_(torch.from_numpy(c.reshape(codes.shape)))
        scales.copy_(torch.from_numpy(s.reshape(scales.shape)))
        ts.fill_(t)
        if stats4 is not None:
            stats4 += torch.from_numpy(st.astype(np.int64))

    def nvfp4_mismatch_stats(self, ca, sa, ta, cb, sb, tb, rows, cols, stats8):
        st = self.o.mismatch_stats(ca.numpy(), sa.numpy(), float(ta.item()), cb.numpy(), sb.numpy(),
                                   float(tb.item()), rows, cols)
        stats8[:7] += torch.from_numpy(st[:7].astype(np.int64))


def _tensors():
    from train_rollout_alignment_b200 import synthetic as syn
    x = syn.random_case((ROWS, COLS), 5, "normal")
    x[ROWS - 3, 7] = syn.bf16_bits(np.float32([40.0]))[0]    # the global max sits in rank 1's rows
    xr = syn.bf16_bits(syn.bf16_to_f32(x) * np.float32(1.0 + 2.0 ** -7))
    return x, xr


def _bf16(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from train_rollout_alignment_b200 import dist as d
    from train_rollout_alignment_b200 import sharded
    d.init("gloo", timeout_s=60)
    lib = OracleKernels(warn=1 if rank == 0 else 0)
    x, xr = _tensors()
    rows = ROWS // world
    sl = slice(rank * rows, (rank + 1) * rows)
    n = rows * COLS
    u8 = dict(dtype=torch.uint8)
    # rollout side on this rank's rows, with 2-bit hints
    ws = torch.zeros(8, dtype=torch.int32)
    cr, sr, tr = torch.zeros(n // 2, **u8), torch.zeros(n // 16, **u8), torch.zeros(1)
    h = torch.zeros(n * 2 // 8, **u8)
    sharded.quantize_rtn(_bf16(xr[sl]), ws, cr, sr, tr, h, 2, lib=lib)
    warn = int(ws[1])
    # train side guided by the same rows' hints, counters summed over ranks
    ct, st_, tt = torch.zeros(n // 2, **u8), torch.zeros(n // 16, **u8), torch.zeros(1)
    s4 = torch.zeros(4, dtype=torch.int64)
    sharded.guided_requant(_bf16(x[sl]), h, 2, ws, ct, st_, tt, s4, lib=lib)
    s8 = torch.zeros(8, dtype=torch.int64)
    sharded.mismatch_stats(cr, sr, tr, ct, st_, tt, rows, COLS, s8, lib=lib)
    q.put({"rank": rank, "codes_r": cr.numpy().copy(), "scales_r": sr.numpy().copy(), "ts_r": float(tr),
           "hints": h.numpy().copy(), "codes_t": ct.numpy().copy(), "ts_t": float(tt),
           "s4": s4.numpy().copy(), "s8": s8.numpy().copy(), "warn": warn})
    d.finish()


def test_row_sharded_quantization_matches_the_unsharded_tensor():
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted([q.get(timeout=180) for _ in procs], key=lambda o: o["rank"])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, xr = _tensors()
    oc, os_, ot, oh = oracle.quantize_rtn(xr, hint_bits=2)
    gc, gs, gt, gst = oracle.guided_requant(x, oh, 2)
    ost = oracle.mismatch_stats(oc, os_, ot, gc, gs, gt, ROWS, COLS)
    half = ROWS * COLS // 2
    for o in out:
        r = o["rank"]
        assert o["ts_r"] == ot and o["ts_t"] == gt           # the whole tensor's scale on both ranks
        assert np.array_equal(o["codes_r"], oc.reshape(-1)[r * half // 2:(r + 1) * half // 2])
        assert np.array_equal(o["scales_r"], os_.reshape(-1)[r * half // 16:(r + 1) * half // 16])
        assert np.array_equal(o["hints"], oh[r * half // 4:(r + 1) * half // 4])
        assert np.array_equal(o["codes_t"], gc.reshape(-1)[r * half // 2:(r + 1) * half // 2])
        assert list(o["s4"][:3]) == [int(v) for v in gst[:3]]  # counters of the whole tensor
        assert list(o["s8"][:7]) == [int(v) for v in ost[:7]]
        assert o["warn"] == 1                                  # rank 0's warning reached rank 1
    # without the exchange, rank 0 would have used its own (smaller) amax
    c0, _, t0, _ = oracle.quantize_rtn(xr[:ROWS // 2], hint_bits=2)
    assert t0 != ot
