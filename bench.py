"""Throughput of the NVFP4 train/rollout alignment path on B200.

One step = the whole path over the 48-layer stack of 65536x4096 BF16
activations (per-column scales log-uniform in [0.1, 10]), for every layer:
  rollout: tensor amax -> round-to-nearest quantize (+ fused 2-bit hints on
           layers 24..47)
  train:   tensor amax -> guided re-quantize (hints on layers 24..47, plain
           round-to-nearest before) with its guidance counters, fused with
           the mismatch counters between the rollout and the train codes
           (counted from registers: the train codes are not read back).
Inputs (48 GiB per GPU) are resident in HBM and larger than L2, so no L2 flush
is needed between steps.  `value` is algorithmic GB/s (bytes each kernel must
move, summed over the step, divided by the step time), `elements_per_s` the
train + rollout elements processed per second.  The timed step runs the
rollout chain and the train chain on two streams; a second timed pass runs
the same steps on one stream with events around every launch, and its
per-kernel durations give the `kernels` table and the roofline figures.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--layers L] [--impl reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own 48-layer stack
(weak scaling, no collective on the data path); the time is the max over
ranks.  `--impl reference` times the CPU oracle on a bounded sample of the
same workload instead.
"""
from __future__ import annotations

import argparse
import gc
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "NVFP4 quantize+guided-requant GB/s and elements/s; fraction of B200 HBM roofline"
ROWS, COLS = 65536, 4096
HINT_BITS = 2

# Algorithmic bytes per element of each kernel (what it must read + write).
BYTES = {
    "amax": 2.0,                                   # BF16 in
    "quantize_rtn": 2.0 + 0.5 + 1 / 16,            # BF16 in, codes + scales out
    "quantize_rtn+hint": 2.0 + 0.5 + 1 / 16 + HINT_BITS / 8,
    "guided_requant": 2.0 + 0.5 + 1 / 16,          # no hints: plain RTN
    "guided_requant+hint": 2.0 + HINT_BITS / 8 + 0.5 + 1 / 16,
    # guided (or RTN) + counters in one pass: BF16 in (+ hints), the rollout's
    # codes + scales in, the train codes + scales out
    "guided_requant_stats": 2.0 + 2 * (0.5 + 1 / 16),
    "guided_requant_stats+hint": 2.0 + HINT_BITS / 8 + 2 * (0.5 + 1 / 16),
    "mismatch_stats": 2 * (0.5 + 1 / 16),
    "emit_hint": 0.5 + HINT_BITS / 8,
}


SPEC_HBM_GBS = 8000.0  # B200 HBM3e data-sheet bandwidth, reported beside the measured peak
# Philox-bound kernels: each random word costs 18 32x32->64-bit multiplies per
# element (10 rounds of 2; the first round's product of the shared draw word is
# computed once, the last round needs one).  The multiply rate per SM is
# measured in the same run (nvfp4_measure_mul_wide: one 1024-thread CTA per SM,
# 8 independent multiply chains per thread, SM clock cycles read in the kernel).
PHILOX_MULS_PER_ELEM = 18


def measure_mul_wide(b, device, iters=20000):
    """32x32->64-bit multiplies per clock per SM, median over the SMs."""
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device=device)
    sink = torch.zeros(sms, dtype=torch.int32, device=device)
    b.nvfp4_measure_mul_wide(sms, 100, cycles, sink)           # warm-up
    b.nvfp4_measure_mul_wide(sms, iters, cycles, sink)
    torch.cuda.synchronize()
    c = statistics.median(cycles.cpu().tolist())
    return 1024 * 8 * iters / c


def _philox_roofline(elems_per_s, sms, sm_mhz, lanes_per_clk):
    peak = sms * sm_mhz * 1e6 * lanes_per_clk / PHILOX_MULS_PER_ELEM
    return {"bound": "alu", "unit": "elements/s", "achieved": round(elems_per_s, 1), "peak": round(peak, 1),
            "frac": round(elems_per_s / peak, 4),
            "basis": "%d Philox wide multiplies per element at %.1f lanes/clk/SM (measured in this run by "
                     "nvfp4_measure_mul_wide), %d SMs, %.0f MHz"
                     % (PHILOX_MULS_PER_ELEM, lanes_per_clk, sms, sm_mhz)}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# dense FP4 tensor-core peak = measured cuBLAS BF16 burst x the nominal FP4/BF16
# ratio (9 / 2.25 PFLOP/s)
FP4_PER_BF16 = 4.0


def _fp4_peak_tflops():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))["bf16_tflops"]) * FP4_PER_BF16, "measured bf16 burst x 4"
    return 1590.0 * FP4_PER_BF16, "fallback bf16 x 4"


# --------------------------------------------------------------------------- clocks
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, "--query-gpu=" + CLOCK_QUERY, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [t.strip() for t in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = max(smax, float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- workload
class Stack:
    """Device-resident 48-layer workload and its output buffers."""

    def __init__(self, layers: int, hint_from: int, device, rank: int, shape=(ROWS, COLS), gen=None):
        """gen(layer) -> (train, rollout) BF16 device tensors of `shape`; the
        throughput stack's generator by default."""
        from train_rollout_alignment_b200 import synthetic as syn
        self.layers, self.hint_from, self.device = layers, hint_from, device
        rows, cols = self.rows, self.cols = shape
        self.n = rows * cols
        if gen is None:
            gen = lambda l: syn.cfg4_layer_device(l, device, rank, shape)
        self.xt, self.xr = [], []
        for l in range(layers):
            t, r = gen(l)
            self.xt.append(t)
            self.xr.append(r)
        u8 = dict(dtype=torch.uint8, device=device)
        self.cr = [torch.empty((rows, cols // 2), **u8) for _ in range(layers)]
        self.sr = [torch.empty((rows, cols // 16), **u8) for _ in range(layers)]
        self.ct = [torch.empty((rows, cols // 2), **u8) for _ in range(layers)]
        self.st = [torch.empty((rows, cols // 16), **u8) for _ in range(layers)]
        self.hints = [torch.empty(self.n * HINT_BITS // 8, **u8) if l >= hint_from else None
                      for l in range(layers)]
        self.ts = torch.empty((layers, 2), dtype=torch.float32, device=device)
        self.ws = torch.zeros((layers, 2, 8), dtype=torch.int32, device=device)
        self.stats = torch.zeros((layers, 12), dtype=torch.int64, device=device)

    def kernels_of_layer(self, l):
        """(kernel label, algorithmic bytes) in launch order for layer l."""
        q = "quantize_rtn+hint" if l >= self.hint_from else "quantize_rtn"
        g = "guided_requant_stats+hint" if l >= self.hint_from else "guided_requant_stats"
        return [("amax", BYTES["amax"] * self.n),
                (q, BYTES[q] * self.n),
                ("amax", BYTES["amax"] * self.n),
                (g, BYTES[g] * self.n)]

    def step_bytes(self):
        return sum(b for l in range(self.layers) for _, b in self.kernels_of_layer(l))

    def run_layer(self, b, l, xr, xt, events=None):
        """The four kernels of layer l; events: list to append (start, end) pairs to."""
        ws_r, ws_t = self.ws[l, 0], self.ws[l, 1]
        ts_r, ts_t = self.ts[l, 0:1], self.ts[l, 1:2]
        h = self.hints[l]
        bits = HINT_BITS if h is not None else 0
        st = self.stats[l]
        calls = [
            lambda: b.nvfp4_tensor_amax(xr, ws_r),
            lambda: b.nvfp4_quantize_rtn(xr, ws_r, self.cr[l], self.sr[l], ts_r, h, bits,
                                         flags=b.NVFP4_AMAX_PRECOMPUTED),
            lambda: b.nvfp4_tensor_amax(xt, ws_t),
            lambda: b.nvfp4_guided_requant_stats(xt, h, HINT_BITS, ws_t, self.ct[l], self.st[l], ts_t, st[8:12],
                                                 self.cr[l], self.sr[l], ts_r, st[0:8],
                                                 flags=b.NVFP4_AMAX_PRECOMPUTED),
        ]
        for fn in calls:
            if events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                events.append((e0, e1))
            else:
                fn()

    def step(self, b, events=None):
        """The step serialized on the current stream (events: per-kernel timing)."""
        self.stats.zero_()
        for l in range(self.layers):
            self.run_layer(b, l, self.xr[l], self.xt[l], events)

    def step_pipelined(self, b, s_roll, s_train):
        """The step on two streams: the rollout chain (amax, quantize + hints)
        on s_roll, the train chain (amax, guided + counters) on s_train; layer
        l's guided pass waits for layer l's rollout codes and hints.  Kernel
        tails of one chain overlap the other chain's next kernel."""
        main = torch.cuda.current_stream(self.device)
        self.stats.zero_()
        start = torch.cuda.Event()
        start.record(main)
        s_roll.wait_event(start)
        s_train.wait_event(start)
        for l in range(self.layers):
            ws_r, ws_t = self.ws[l, 0], self.ws[l, 1]
            ts_r, ts_t = self.ts[l, 0:1], self.ts[l, 1:2]
            h = self.hints[l]
            bits = HINT_BITS if h is not None else 0
            st = self.stats[l]
            with torch.cuda.stream(s_roll):
                b.nvfp4_tensor_amax(self.xr[l], ws_r)
                b.nvfp4_quantize_rtn(self.xr[l], ws_r, self.cr[l], self.sr[l], ts_r, h, bits,
                                     flags=b.NVFP4_AMAX_PRECOMPUTED)
                rolled = torch.cuda.Event()
                rolled.record(s_roll)
            with torch.cuda.stream(s_train):
                b.nvfp4_tensor_amax(self.xt[l], ws_t)
                s_train.wait_event(rolled)
                b.nvfp4_guided_requant_stats(self.xt[l], h, HINT_BITS, ws_t, self.ct[l], self.st[l], ts_t,
                                             st[8:12], self.cr[l], self.sr[l], ts_r, st[0:8],
                                             flags=b.NVFP4_AMAX_PRECOMPUTED)
        for s in (s_roll, s_train):
            done = torch.cuda.Event()
            done.record(s)
            main.wait_event(done)


# --------------------------------------------------------------------------- CPU oracle
def _oracle_pipeline(xt, xr, hint_bits):
    import oracle
    A_r, A_t = oracle.amax_bf16(xr), oracle.amax_bf16(xt)
    rc, rs, rt, h = oracle.quantize_rtn(xr, A_r, hint_bits)
    gc, gs, gt, _ = oracle.guided_requant(xt, h, HINT_BITS, A_t)
    oracle.mismatch_stats(rc, rs, rt, gc, gs, gt, xt.shape[0], xt.shape[1])


def oracle_sample(device, rank, rows_per_core: int, cores: int):
    """Host arrays for the CPU oracle: `cores` chunks of `rows_per_core` rows of
    layer 24 (a hinted layer), each chunk quantized as a tensor of its own."""
    from train_rollout_alignment_b200 import synthetic as syn
    xt, xr = syn.cfg4_layer_device(24, device, rank)
    rows = min(ROWS, rows_per_core * cores)
    to_np = lambda t: t[:rows].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    xt_h, xr_h = to_np(xt), to_np(xr)
    del xt, xr
    return [(xt_h[i:i + rows_per_core], xr_h[i:i + rows_per_core]) for i in range(0, rows, rows_per_core)]


def time_oracle(chunks):
    """Wall time of the oracle pipeline over all chunks, one thread per chunk
    (the C oracle releases the GIL)."""
    from concurrent.futures import ThreadPoolExecutor
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=len(chunks)) as ex:
        list(ex.map(lambda c: _oracle_pipeline(c[0], c[1], HINT_BITS), chunks))
    return time.perf_counter() - t0


def oracle_bytes(chunks):
    """Algorithmic bytes of the oracle's work, counted as for the GPU step of
    a hinted layer (the same work moves the same algorithmic bytes)."""
    per_elem = BYTES["amax"] * 2 + BYTES["quantize_rtn+hint"] + BYTES["guided_requant_stats+hint"]
    return sum(c[0].size for c in chunks) * per_elem, sum(c[0].size for c in chunks)


def _cores():
    return len(os.sched_getaffinity(0))


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--layers", type=int, default=48)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    args = ap.parse_args()
    from train_rollout_alignment_b200 import dist as tdist
    world, rank, local = tdist.world()
    if args.impl == "reference":
        return run_reference(args, world, rank, local)
    return run_ours(args, world, rank, local)


def _config(layers):
    return {"workload": "%d-layer stack of %dx%d BF16 activations, N(0,1) x per-column log-uniform "
                        "[0.1, 10] scales, seed 4: rollout RTN + 2-bit hints on layers %d-%d, train "
                        "guided requant, mismatch stats" % (layers, ROWS, COLS, layers // 2, layers - 1),
            "layers": layers, "rows": ROWS, "cols": COLS, "hint_bits": HINT_BITS,
            "inputs_bf16_gib_per_gpu": round(layers * 2 * ROWS * COLS * 2 / 2 ** 30, 1),
            "l2": "no flush: every input tensor (512 MiB) is larger than L2 (126 MB)"}


def run_ours(args, world, rank, local):
    from train_rollout_alignment_b200 import _binding as b
    from train_rollout_alignment_b200 import dist as tdist
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        tdist.init("nccl")
    peak, peak_kind = _peaks()

    stack = Stack(args.layers, args.layers // 2, device, rank)
    torch.cuda.synchronize()
    step_bytes = stack.step_bytes()
    step_elems = 2 * stack.n * args.layers

    s_roll, s_train = torch.cuda.Stream(device), torch.cuda.Stream(device)
    gc.collect()
    gc.disable()  # no collector pauses inside the timed regions
    for _ in range(args.warmup):
        stack.step_pipelined(b, s_roll, s_train)
    torch.cuda.synchronize()

    # ---- device-timed region: K pipelined steps, no per-kernel events inside
    sampler = ClockSampler(local)
    time.sleep(0.3)
    tdist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for _ in range(args.steps):
        stack.step_pipelined(b, s_roll, s_train)
    t_end.record()
    torch.cuda.synchronize()
    tdist.barrier()
    t_max = tdist.max_over_ranks(t_start.elapsed_time(t_end) / 1e3, device)

    # ---- second timed region: K serialized steps with events around every
    # launch on the launching stream (per-kernel durations for the roofline;
    # concurrent kernels would blur them, so this pass runs one at a time)
    tdist.barrier()
    torch.cuda.synchronize()
    events = []
    k_start = torch.cuda.Event(enable_timing=True)
    k_end = torch.cuda.Event(enable_timing=True)
    k_start.record()
    for _ in range(args.steps):
        stack.step(b, events)
    k_end.record()
    torch.cuda.synchronize()
    tdist.barrier()
    clocks = sampler.stop()
    t_serial = tdist.max_over_ranks(k_start.elapsed_time(k_end) / 1e3, device)

    # per-kernel durations (average over launches in the serialized pass)
    labels = [lab for l in range(args.layers) for lab, _ in stack.kernels_of_layer(l)] * args.steps
    nbytes = [nb for l in range(args.layers) for _, nb in stack.kernels_of_layer(l)] * args.steps
    per = {}
    for lab, nb, (e0, e1) in zip(labels, nbytes, events):
        d = per.setdefault(lab, {"launches": 0, "ms": 0.0, "bytes": 0.0})
        d["launches"] += 1
        d["ms"] += e0.elapsed_time(e1)
        d["bytes"] += nb
    total_ms = sum(d["ms"] for d in per.values())
    kernels = {}
    for lab, d in per.items():
        gbs = d["bytes"] / (d["ms"] / 1e3) / 1e9
        kernels[lab] = {"launches": d["launches"], "avg_us": round(1e3 * d["ms"] / d["launches"], 2),
                        "share": round(d["ms"] / total_ms, 4), "GB/s": round(gbs, 1),
                        "frac": round(gbs / peak, 4)}
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    dom_bytes_per_launch = per[dom]["bytes"] / per[dom]["launches"]
    dom_gbs = per[dom]["bytes"] / (per[dom]["ms"] / 1e3) / 1e9
    traffic = _ncu_traffic(dom)

    value = tdist.aggregate_rate(args.steps * step_bytes, world, t_max) / 1e9
    elems = tdist.aggregate_rate(args.steps * step_elems, world, t_max)

    # ---- the other rows of the path, each timed alone (rank-local)
    sm_mhz = clocks["sm_max_mhz"] if clocks else 1965.0
    other = time_other_kernels(b, stack, device, peak, sm_mhz)

    other["hint_transport"] = time_hint_transport(b, stack, device)
    other.update(time_kv_rows(b, device, peak))
    other["l2_resident_configs"] = time_small_configs(b, device, peak, rank)
    other["rollout_producer"] = time_producer(b, device)

    # ---- end to end through the C ABI with host buffers (rank-local)
    e2e = run_e2e(b, stack, device, steps=min(args.steps, 2))

    gc.enable()

    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if world == 1:
        cores = _cores()
        chunks = oracle_sample(device, rank, rows_per_core=1024, cores=cores)
        nbytes_cpu, nel = oracle_bytes(chunks)
        dt = time_oracle(chunks)
        one = chunks[:1]
        nbytes_1, nel_1 = oracle_bytes(one)
        dt_1 = time_oracle(one)
        cpu = {"value": round(nbytes_cpu / dt / 1e9, 3), "unit": "GB/s", "cores": len(chunks),
               "kind": "oracle",
               "sample": "%d rows x %d cols of layer 24 (train + rollout), split in %d chunks of 1024 "
                         "rows each quantized as its own tensor, one thread per chunk; %.1f s wall"
                         % (len(chunks) * 1024, COLS, len(chunks), dt),
               "elements_per_s": round(2 * nel / dt, 1),
               "single_thread": {"value": round(nbytes_1 / dt_1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                                 "elements_per_s": round(2 * nel_1 / dt_1, 1),
                                 "sample": "one chunk of 1024 rows on one thread; %.1f s wall" % dt_1}}

    launches = 4 * args.layers * args.steps
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t_max / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded, generated on the GPU; BF16 inputs, FP32 arithmetic)",
        "config": _config(args.layers),
        "value_basis": ("algorithmic bytes (what each kernel must read and write, summed over the step) / "
                        "step time; consecutive kernels can hit in L2 (the quantizer reads the tail of the "
                        "tensor the amax pass just read), so this is not DRAM traffic: see dram_bytes_per_step "
                        "and the per-kernel serialized figures"),
        "algorithmic_bytes_per_step": int(step_bytes),
        "dram_bytes_per_step": _dram_bytes_per_step(stack),
        "elements_per_s": round(elems, 1),
        "schedule": "rollout chain and train chain on two streams (guided waits for its layer's hints)",
        "serialized": {"ms_per_step": round(1e3 * t_serial / args.steps, 3),
                       "value": round(tdist.aggregate_rate(args.steps * step_bytes, world, t_serial) / 1e9, 1),
                       "note": "one stream, events around every launch; source of the kernels table"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(dom_gbs, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dom_gbs / peak, 4),
                     "frac_of_spec": round(dom_gbs / SPEC_HBM_GBS, 4),
                     "bytes_per_launch": dom_bytes_per_launch, "traffic": traffic},
        "kernels": kernels,
        "other_kernels": other,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    tdist.finish()
    if rank == 0:
        print(json.dumps(out))


def _sources_sha(files):
    """sha256 (first 16 hex digits) of the named kernel source files, in order."""
    import hashlib
    from train_rollout_alignment_b200 import build as bld
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(bld.CSRC, f), "rb").read())
    return h.hexdigest()[:16]


def _ncu_traffic_all():
    """DRAM bytes per launch of each kernel of the step from the committed ncu
    summary, for the kernels whose line was taken on their current sources
    (the files the line names): {label: bytes}."""
    path = os.path.join(ROOT, "profiles", "ncu_dram_traffic.txt")
    out = {}
    if not os.path.exists(path):
        return out
    for line in open(path):
        if line.startswith("#") or "=" not in line:
            continue
        kv = dict(tok.split("=", 1) for tok in line.split())
        if "label" not in kv or "files" not in kv:
            continue
        if kv.get("src_sha") == _sources_sha(kv["files"].split(",")):
            out[kv["label"]] = float(kv["dram_bytes_per_launch"])
    return out


def _ncu_traffic(kernel_label):
    """DRAM bytes per launch of one kernel (see _ncu_traffic_all), or None."""
    return _ncu_traffic_all().get(kernel_label)


def _dram_bytes_per_step(stack):
    """DRAM bytes of one step from the per-launch ncu traffic of its kernels,
    when every kernel of the step has a current line; else None."""
    per = _ncu_traffic_all()
    total = 0.0
    for l in range(stack.layers):
        for lab, _ in stack.kernels_of_layer(l):
            if lab not in per:
                return None
            total += per[lab]
    return total


def _flush_l2(bufs):
    """Write 256 MiB, then read another 256 MiB: the timed call finds none of
    its inputs in L2 (126 MB).  Some of the flush's written lines can still be
    in L2 and are written back during the timed call: on B200 a 512 MiB read
    took 92 us after this flush against 84 us after a read-only one, so
    figures taken this way are a few percent low for short kernels."""
    w, r = bufs
    w.add_(1)
    torch.sum(r, dtype=torch.float32)


def _timed(fn, reps, flush):
    """Median device time of fn over reps calls, L2 flushed before each (outside
    the events).  A short spin kernel ahead of the start event keeps the GPU
    busy while the host enqueues the call, so host-side delays do not land
    between the events."""
    times = []
    for r in range(reps):
        _flush_l2(flush)
        torch.cuda._sleep(100_000)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn(r)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times) / 1e3


def _timed_b2b(fn, count=10, reps=3):
    """Device time per call of `count` calls launched back to back between one
    pair of events (median over `reps` such runs), no L2 flush: for kernels
    whose inputs are more than twice the L2, so a call cannot find its input
    left in L2 by the one before.  Each call also pays for writing back the
    previous call's output, as it would in a stream of work; and the event
    timer's granularity (about a microsecond) is spread over `count` calls."""
    times = []
    for r in range(reps):
        torch.cuda._sleep(100_000)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(count):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / count)
    return statistics.median(times) / 1e3


def time_other_kernels(b, stack, device, peak, sm_mhz, reps=10):
    """Standalone hint emit (throughput stack, layer 24), SR transpose
    re-quantize (128 x 512 x 2048 expert stack) and RHT32 + quantize
    (16384 x 4096 activation with outliers): seconds per call and algorithmic
    GB/s (median of `reps` calls), L2 flushed before every call; kernels whose
    inputs are more than twice the L2 (the amax pass, the counters, the two
    quantizers alone, tile quantize) are timed back to back, the flushed
    figure beside it."""
    from train_rollout_alignment_b200 import synthetic as syn
    flush = (torch.zeros(64 << 20, dtype=torch.float32, device=device),
             torch.ones(64 << 20, dtype=torch.float32, device=device))
    out = {}
    mul_rate = measure_mul_wide(b, device)
    out["mul_wide_lanes_per_clk_per_sm"] = round(mul_rate, 2)
    # hint emit from the codes of a hinted layer
    l = stack.hint_from
    h = torch.empty(stack.n * HINT_BITS // 8, dtype=torch.uint8, device=device)
    t = _timed(lambda r: b.nvfp4_emit_hint(stack.cr[l], stack.n, HINT_BITS, h), reps, flush)
    gbs = BYTES["emit_hint"] * stack.n / t / 1e9
    out["emit_hint"] = {"workload": "%dx%d codes, 2-bit hints" % (ROWS, COLS), "avg_us": round(t * 1e6, 2),
                        "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4), "bytes_per_elem": BYTES["emit_hint"]}
    # the amax pass alone on that layer's rollout input (in the step each launch
    # follows a writer and pays for its output write-back): back to back and flushed
    ws_tmp = torch.zeros(8, dtype=torch.int32, device=device)
    amax_call = lambda r: b.nvfp4_tensor_amax(stack.xr[l], ws_tmp)
    t = _timed_b2b(amax_call)
    t_f = _timed(amax_call, reps, flush)
    gbs = BYTES["amax"] * stack.n / t / 1e9
    out["amax (alone)"] = {"workload": "%dx%d BF16 layer %d" % (ROWS, COLS, l),
                           "timing": "10 calls back to back, inputs > 2x L2",
                           "avg_us": round(t * 1e6, 2), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4),
                           "flushed_us": round(t_f * 1e6, 2),
                           "flushed_frac": round(BYTES["amax"] * stack.n / t_f / 1e9 / peak, 4),
                           "bytes_per_elem": BYTES["amax"]}
    # the standalone counters (the step counts inside the guided pass) between
    # the rollout and train tensors of that layer
    # (inputs of 302 MB: timed back to back, the L2-flushed figure beside it)
    s8 = torch.zeros(8, dtype=torch.int64, device=device)
    stats_call = lambda r: b.nvfp4_mismatch_stats(stack.cr[l], stack.sr[l], stack.ts[l, 0:1], stack.ct[l],
                                                  stack.st[l], stack.ts[l, 1:2], ROWS, COLS, s8)
    t = _timed_b2b(stats_call)
    t_f = _timed(stats_call, reps, flush)
    gbs = BYTES["mismatch_stats"] * stack.n / t / 1e9
    out["mismatch_stats"] = {"workload": "%dx%d rollout vs train NVFP4 (layer %d)" % (ROWS, COLS, l),
                             "timing": "10 calls back to back, inputs > 2x L2",
                             "avg_us": round(t * 1e6, 2), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4),
                             "flushed_us": round(t_f * 1e6, 2),
                             "flushed_frac": round(BYTES["mismatch_stats"] * stack.n / t_f / 1e9 / peak, 4),
                             "bytes_per_elem": BYTES["mismatch_stats"]}
    # the two quantizers of that layer alone (in the step they may find part
    # of their input in L2 behind the amax pass): back to back and L2-flushed
    c_tmp, s_tmp = torch.empty_like(stack.ct[l]), torch.empty_like(stack.st[l])
    ts_tmp = torch.empty(1, dtype=torch.float32, device=device)
    s4 = torch.zeros(4, dtype=torch.int64, device=device)
    for name, fn in (("quantize_rtn+hint", lambda r: b.nvfp4_quantize_rtn(
                         stack.xr[l], stack.ws[l, 0], c_tmp, s_tmp, ts_tmp, h, HINT_BITS,
                         flags=b.NVFP4_AMAX_PRECOMPUTED)),
                     ("guided_requant+hint", lambda r: b.nvfp4_guided_requant(
                         stack.xt[l], stack.hints[l], HINT_BITS, stack.ws[l, 1], c_tmp, s_tmp, ts_tmp, s4,
                         flags=b.NVFP4_AMAX_PRECOMPUTED))):
        t = _timed_b2b(fn)
        t_f = _timed(fn, reps, flush)
        gbs = BYTES[name] * stack.n / t / 1e9
        out[name + " (alone)"] = {"workload": "%dx%d BF16 layer %d, amax precomputed" % (ROWS, COLS, l),
                                  "timing": "10 calls back to back, inputs > 2x L2",
                                  "avg_us": round(t * 1e6, 2), "GB/s": round(gbs, 1),
                                  "frac": round(gbs / peak, 4), "flushed_us": round(t_f * 1e6, 2),
                                  "flushed_frac": round(BYTES[name] * stack.n / t_f / 1e9 / peak, 4),
                                  "bytes_per_elem": BYTES[name]}
    del c_tmp, s_tmp
    # SR transpose: the expert stack quantized by the library's own RTN path
    batch, er, ec = syn.CFG2_SHAPE
    w = torch.from_numpy(syn.cfg2().view(np.int16)).view(torch.bfloat16).to(device)
    ne = er * ec
    codes = torch.empty(batch * ne // 2, dtype=torch.uint8, device=device)
    scales = torch.empty(batch * ne // 16, dtype=torch.uint8, device=device)
    ts = torch.empty(batch, dtype=torch.float32, device=device)
    ws = torch.zeros(max(batch, 8), dtype=torch.int32, device=device)
    for e in range(batch):
        b.nvfp4_quantize_rtn(w[e], ws, codes[e * ne // 2:(e + 1) * ne // 2],
                             scales[e * ne // 16:(e + 1) * ne // 16], ts[e:e + 1])
    ct, st, tst = torch.empty_like(codes), torch.empty_like(scales), torch.empty_like(ts)
    t = _timed(lambda r: b.nvfp4_sr_transpose_requant(codes, scales, ts, batch, er, ec, syn.CFG2_SR_SEED, r,
                                                      ws, ct, st, tst), reps, flush)
    n = batch * ne
    sr_bytes = 3 * (0.5 + 1 / 16)  # amax pre-pass reads codes+scales, main pass reads and writes them
    out["sr_transpose_requant"] = {
        "workload": "%dx%dx%d expert stack, one Philox4x32-10 word per element" % (batch, er, ec),
        "avg_us": round(t * 1e6, 2), "GB/s": round(sr_bytes * n / t / 1e9, 1),
        "frac": round(sr_bytes * n / t / 1e9 / peak, 4), "bytes_per_elem": sr_bytes,
        "elements_per_s": round(n / t, 1),
        "alu_roofline": _philox_roofline(n / t, torch.cuda.get_device_properties(device).multi_processor_count, sm_mhz,
                                         mul_rate)}
    b.nvfp4_sr_transpose_requant(codes, scales, ts, batch, er, ec, syn.CFG2_SR_SEED, 0, ws, ct, st, tst)
    out.update(time_transpose_alternatives(b, stack, w, codes, scales, ts, (ct, st, tst), device, peak, reps,
                                           flush))
    out["mxfp8_sr_transpose_requant"]["alu_roofline"] = _philox_roofline(
        out["mxfp8_sr_transpose_requant"]["elements_per_s"], torch.cuda.get_device_properties(device).multi_processor_count,
        sm_mhz, mul_rate)
    del w, codes, scales, ct, st
    # RHT32 + quantize
    x = torch.from_numpy(syn.cfg3().view(np.int16)).view(torch.bfloat16).to(device)
    rr, cc = x.shape
    c3 = torch.empty((rr, cc // 2), dtype=torch.uint8, device=device)
    s3 = torch.empty((rr, cc // 16), dtype=torch.uint8, device=device)
    t3 = torch.empty(1, dtype=torch.float32, device=device)
    t = _timed(lambda r: b.nvfp4_rht_quantize(x, syn.CFG3_SIGN_SEED, ws, c3, s3, t3), reps, flush)
    n = rr * cc
    rht_bytes = 2 + 2 + 0.5 + 1 / 16
    out["rht_quantize"] = {"workload": "%dx%d activation, 0.1%% outliers x100" % (rr, cc),
                           "avg_us": round(t * 1e6, 2), "GB/s": round(rht_bytes * n / t / 1e9, 1),
                           "frac": round(rht_bytes * n / t / 1e9 / peak, 4), "bytes_per_elem": rht_bytes}
    return out


def time_transpose_alternatives(b, stack, w, codes, scales, ts, sr_out, device, peak, reps, flush):
    """The two alternatives to the SR transpose on the expert stack: 16x16-tile
    NVFP4 (tile quantize timed on a 65536x4096 layer, lossless transpose of the
    stack) and MXFP8 SR transpose re-quantize; then the error of each way of
    getting a quantized W^T, against the BF16 W^T (relative squared error,
    relative bias, share of nonzero values decoded as 0)."""
    batch, er, ec = w.shape
    ne, n = er * ec, batch * er * ec
    out = {}
    # tile quantize, streaming: the train input of a hinted layer, its amax precomputed
    l = stack.hint_from
    ct16 = torch.empty((ROWS, COLS // 2), dtype=torch.uint8, device=device)
    tt16 = torch.empty((ROWS // 16, COLS // 16), dtype=torch.uint8, device=device)
    ts16 = torch.empty(1, dtype=torch.float32, device=device)
    wsl = stack.ws[l, 1]
    b.nvfp4_tensor_amax(stack.xt[l], wsl)
    tile_call = lambda r: b.nvfp4_quantize_tile16(stack.xt[l], wsl, ct16, tt16, ts16, flags=b.NVFP4_AMAX_PRECOMPUTED)
    t = _timed_b2b(tile_call)
    t_f = _timed(tile_call, reps, flush)
    qb = 2 + 0.5 + 1 / 256
    out["quantize_tile16"] = {"workload": "%dx%d BF16 layer, amax precomputed" % (ROWS, COLS),
                              "timing": "10 calls back to back, inputs > 2x L2",
                              "avg_us": round(t * 1e6, 2), "GB/s": round(qb * stack.n / t / 1e9, 1),
                              "frac": round(qb * stack.n / t / 1e9 / peak, 4), "flushed_us": round(t_f * 1e6, 2),
                              "bytes_per_elem": qb}
    del ct16, tt16
    # tile codes of the expert stack, then the lossless transpose
    tc = torch.empty(n // 2, dtype=torch.uint8, device=device)
    tt = torch.empty(n // 256, dtype=torch.uint8, device=device)
    tts = torch.empty(batch, dtype=torch.float32, device=device)
    wse = torch.zeros(8, dtype=torch.int32, device=device)
    for e in range(batch):
        b.nvfp4_quantize_tile16(w[e], wse, tc[e * ne // 2:(e + 1) * ne // 2], tt[e * ne // 256:(e + 1) * ne // 256],
                                tts[e:e + 1])
    tct, ttt = torch.empty_like(tc), torch.empty_like(tt)
    t = _timed(lambda r: b.nvfp4_transpose_tile16(tc, tt, batch, er, ec, tct, ttt), reps, flush)
    tb = 0.5 + 0.5 + 2 / 256
    out["transpose_tile16"] = {"workload": "%dx%dx%d expert stack" % (batch, er, ec), "avg_us": round(t * 1e6, 2),
                               "GB/s": round(tb * n / t / 1e9, 1), "frac": round(tb * n / t / 1e9 / peak, 4),
                               "bytes_per_elem": tb}
    # MXFP8 SR transpose from the 16-value NVFP4 codes
    q = torch.empty(n, dtype=torch.uint8, device=device)
    e8 = torch.empty(n // 32, dtype=torch.uint8, device=device)
    t = _timed(lambda r: b.mxfp8_sr_transpose_requant(codes, scales, ts, batch, er, ec, 2, r, q, e8), reps, flush)
    mb = 0.5 + 1 / 16 + 1 + 1 / 32
    out["mxfp8_sr_transpose_requant"] = {
        "workload": "%dx%dx%d expert stack, one Philox4x32-10 word per element" % (batch, er, ec),
        "avg_us": round(t * 1e6, 2), "GB/s": round(mb * n / t / 1e9, 1), "frac": round(mb * n / t / 1e9 / peak, 4),
        "bytes_per_elem": mb, "elements_per_s": round(n / t, 1)}
    b.mxfp8_sr_transpose_requant(codes, scales, ts, batch, er, ec, 2, 0, q, e8)
    # quality of each quantized W^T against the BF16 W^T
    wt = w.float().transpose(1, 2).contiguous()
    deq = torch.empty((batch, ec, er), dtype=torch.float32, device=device)

    def err(y):
        d = (y - wt).double()
        nz = wt != 0
        return {"rel_sq_err": float((d * d).sum() / (wt.double() ** 2).sum()),
                "rel_bias": float(d.sum() / wt.double().abs().sum()),
                "nonzero_to_zero": float(((y == 0) & nz).sum() / nz.sum())}

    quality = {}
    ct_, st_, tst_ = sr_out
    for e in range(batch):
        b.nvfp4_dequantize(ct_[e * ne // 2:(e + 1) * ne // 2], st_[e * ne // 16:(e + 1) * ne // 16], tst_[e:e + 1],
                           ec, er, b.NVFP4_SCALES_BLOCK16, deq[e])
    quality["nvfp4_16_sr_transpose"] = err(deq)
    for e in range(batch):
        b.nvfp4_dequantize(tct[e * ne // 2:(e + 1) * ne // 2], ttt[e * ne // 256:(e + 1) * ne // 256], tts[e:e + 1],
                           ec, er, b.NVFP4_SCALES_TILE16, deq[e])
    quality["nvfp4_tile16_transpose"] = err(deq)
    b.mxfp8_dequantize(q, e8, n, deq)
    quality["mxfp8_sr_transpose"] = err(deq)
    cd = torch.empty(ne // 2, dtype=torch.uint8, device=device)
    sd = torch.empty(ne // 16, dtype=torch.uint8, device=device)
    td = torch.empty(1, dtype=torch.float32, device=device)
    for e in range(batch):
        b.nvfp4_quantize_rtn(w[e].t().contiguous(), wse, cd, sd, td)
        b.nvfp4_dequantize(cd, sd, td, ec, er, b.NVFP4_SCALES_BLOCK16, deq[e])
    quality["nvfp4_16_rtn_of_transposed_bf16"] = err(deq)
    quality["note"] = ("W^T of the %dx%dx%d expert stack; each row is one way to obtain a quantized W^T from "
                       "the forward's quantized W (the last row quantizes the BF16 W^T directly, for reference)"
                       % (batch, er, ec))
    out["transpose_quality"] = quality
    return out


def time_small_configs(b, device, peak, rank, reps=30):
    """The whole step on the two smaller activation workloads, whose tensors
    fit in L2 (126 MB): the single 1024x2048 N(0,1) tensor with 2-bit hints,
    and the 24-layer 8192x2048 Student-t (nu=4) stack with 16 outlier channels
    x50 per layer, hints on layers 12-23 (generated on the GPU: the same
    distribution as the host generator of the parity tests).  Their kernels
    last microseconds, so the step is captured once in a CUDA graph (both
    streams) and replayed: "warm" = graph replays back to back (median of
    per-replay times over `reps` replays in one timed region; L2 may hold the
    inputs), "flushed" = L2 flushed before every replay.  Flagged L2-resident:
    these numbers can exceed the HBM roofline."""
    from train_rollout_alignment_b200 import synthetic as syn
    flush = (torch.zeros(64 << 20, dtype=torch.float32, device=device),
             torch.ones(64 << 20, dtype=torch.float32, device=device))
    out = {}
    x0 = syn.cfg0()
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    stacks = {
        "single_tensor_1024x2048": lambda: Stack(1, 0, device, rank, syn.CFG0_SHAPE,
                                                 gen=lambda l: (to_dev(x0[0]), to_dev(x0[1]))),
        "moe_activation_stack_24x8192x2048": lambda: Stack(
            syn.CFG1_LAYERS, syn.CFG1_HINT_FROM, device, rank, syn.CFG1_SHAPE,
            gen=lambda l: syn.cfg1_layer_device(l, device, rank)),
    }
    for name, make in stacks.items():
        st = make()
        nbytes, nel = st.step_bytes(), 2 * st.n * st.layers
        cap = torch.cuda.Stream(device)
        s_roll, s_train = torch.cuda.Stream(device), torch.cuda.Stream(device)
        with torch.cuda.stream(cap):
            for _ in range(3):  # warm-up outside capture (first-call set-up of the kernels)
                st.step_pipelined(b, s_roll, s_train)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            st.step_pipelined(b, s_roll, s_train)
        torch.cuda.synchronize()
        res = {}
        # warm: replays back to back between two events
        graph.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(1_000_000)
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / reps
        res["warm"] = {"us_per_step": round(t * 1e6, 2), "GB/s": round(nbytes / t / 1e9, 1),
                       "frac": round(nbytes / t / 1e9 / peak, 4), "elements_per_s": round(nel / t, 1)}
        times = []
        for _ in range(reps):
            _flush_l2(flush)
            torch.cuda._sleep(1_000_000)
            a = torch.cuda.Event(enable_timing=True)
            z = torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            z.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(z) / 1e3)
        t = statistics.median(times)
        res["flushed"] = {"us_per_step": round(t * 1e6, 2), "GB/s": round(nbytes / t / 1e9, 1),
                          "frac": round(nbytes / t / 1e9 / peak, 4), "elements_per_s": round(nel / t, 1)}
        res.update({"layers": st.layers, "shape": [st.rows, st.cols], "bytes_per_step": int(nbytes),
                    "kernels_per_step": 4 * st.layers, "l2_resident": True, "timing": "CUDA graph replay"})
        out[name] = res
        del graph, st
        torch.cuda.synchronize()
    return out


def time_kv_rows(b, device, peak, reps=10):
    """KV-cache layout (one FP32 scale per (token, head) row): a cache of
    65536 tokens x 16 heads x 128 (head_dim), the rollout's RTN + 2-bit hints
    and the train side's guided re-quantization, each timed as 10 calls back
    to back and as the median of `reps` calls with an L2 flush before each."""
    tokens, heads, dim = 65536, 16, 128
    rows = tokens * heads
    n = rows * dim
    gen = torch.Generator(device=device).manual_seed(6)
    xt = (torch.randn((rows, dim), device=device, generator=gen)
          * torch.exp(torch.empty((1, dim), device=device).uniform_(np.log(0.1), np.log(10.0), generator=gen)))
    xt = xt.to(torch.bfloat16)
    xr = (xt.float() * (1 + torch.randn(xt.shape, device=device, generator=gen) * 2.0 ** -8)).to(torch.bfloat16)
    u8 = dict(dtype=torch.uint8, device=device)
    cr, sr_, rr = torch.empty(n // 2, **u8), torch.empty(n // 16, **u8), torch.empty(rows, dtype=torch.float32, device=device)
    ct, st_, rt = torch.empty(n // 2, **u8), torch.empty(n // 16, **u8), torch.empty(rows, dtype=torch.float32, device=device)
    h = torch.empty(n * HINT_BITS // 8, **u8)
    s4 = torch.zeros(4, dtype=torch.int64, device=device)
    flush = (torch.zeros(64 << 20, dtype=torch.float32, device=device),
             torch.ones(64 << 20, dtype=torch.float32, device=device))
    rtn = lambda r: b.nvfp4_quantize_rtn_rows(xr, cr, sr_, rr, h, HINT_BITS)
    gd = lambda r: b.nvfp4_guided_requant_rows(xt, h, HINT_BITS, ct, st_, rt, s4)
    nb = 2 + 0.5 + 1 / 16 + HINT_BITS / 8 + 4 / dim  # BF16 in; codes, scales, hints, row scale
    work = "KV cache %d tokens x %d heads x %d, one FP32 scale per row, 2-bit hints" % (tokens, heads, dim)
    out = {}
    # inputs of 268 MB (more than twice the L2): back to back, the flushed figure beside it
    for name, fn in (("kv_rows_rollout_rtn+hint", rtn), ("kv_rows_train_guided+hint", gd)):
        t = _timed_b2b(fn)
        t_f = _timed(fn, reps, flush)
        gbs = nb * n / t / 1e9
        out[name] = {"workload": work, "timing": "10 calls back to back, inputs > 2x L2",
                     "avg_us": round(t * 1e6, 2), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4),
                     "flushed_us": round(t_f * 1e6, 2), "flushed_frac": round(nb * n / t_f / 1e9 / peak, 4),
                     "bytes_per_elem": nb, "elements_per_s": round(n / t, 1)}
    return out


def time_producer(b, device, reps=10, m=8192, n=4096, k=4096):
    """The fused rollout producer: an NVFP4 activation [m tokens, k] times an
    NVFP4 weight [n, k] on the tensor cores, the product quantized to NVFP4
    with 2-bit hints and both scale layouts in the epilogue.  Operands come from
    the library's own quantizer on synthetic N(0, 1) activations and N(0, 0.02^2)
    weights; the output tensor scale uses the max |D| recorded by a previous
    call (delayed scaling).  Also the MoE form (routed rows grouped by expert,
    one weight per expert, one launch).  Median of `reps` calls, L2 flushed
    before each."""
    gen = torch.Generator(device=device).manual_seed(8)
    u8 = dict(dtype=torch.uint8, device=device)

    def nvfp4_operand_k(rows, kk, std):
        x = (torch.randn((rows, kk), device=device, generator=gen) * std).to(torch.bfloat16)
        codes, scales, ts, ws, _ = b.empty_nvfp4(rows, kk, device)
        b.nvfp4_quantize_rtn(x, ws, codes, scales, ts)
        smma = torch.empty(b.mma_scale_bytes(rows, kk // 16), **u8)
        b.nvfp4_scales_to_mma(scales, rows, kk // 16, smma)
        return codes, smma, ts

    def nvfp4_operand(rows, std):
        return nvfp4_operand_k(rows, k, std)

    a_codes, a_sf, a_ts = nvfp4_operand(m, 1.0)
    w_codes, w_sf, w_ts = nvfp4_operand(n, 0.02)
    codes, scales, ts, ws, hints = b.empty_nvfp4(m, n, device, hint_bits=HINT_BITS)
    smma = torch.empty(b.mma_scale_bytes(m, n // 16), **u8)
    d = torch.empty((m, n), dtype=torch.float32, device=device)
    ws.zero_()

    def call(r, d_out=None):
        b.nvfp4_gemm_quantize(a_codes, a_sf, a_ts, w_codes, w_sf, w_ts, m, n, k, ws, codes, scales, ts,
                              scales_mma=smma, hints=hints, hint_bits=HINT_BITS, d_out=d_out)

    call(0)
    torch.cuda.synchronize()
    ws[0] = ws[2]                       # delayed scaling: the amax this product just produced
    flush = (torch.zeros(64 << 20, dtype=torch.float32, device=device),
             torch.ones(64 << 20, dtype=torch.float32, device=device))
    t = _timed(call, reps, flush)
    t_d = _timed(lambda r: call(r, d), reps, flush)
    warn = int(ws[1].item())
    peak, basis = _fp4_peak_tflops()
    flops = 2.0 * m * n * k
    out_bytes = m * n * (0.5 + 1 / 16 + 1 / 16 + HINT_BITS / 8)
    tf = flops / t / 1e12
    out = {"workload": "NVFP4 [%d tokens x %d] x NVFP4 weight [%d x %d]^T -> NVFP4 + %d-bit hints + "
                       "tensor-core scale layout" % (m, k, n, k, HINT_BITS),
           "avg_us": round(t * 1e6, 2), "TFLOP/s": round(tf, 1),
           "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": round(peak, 1),
                        "unit": "TFLOP/s", "frac": round(tf / peak, 4), "peak_basis": basis},
           "epilogue_out_bytes": int(out_bytes),
           "with_fp32_D_written_us": round(t_d * 1e6, 2),
           "warning_bits": warn}
    del a_codes, a_sf, w_codes, w_sf, codes, scales, smma, d, hints

    # the same product with a 4x longer reduction (k = 16384): the epilogue's
    # share shrinks and the main loop's rate shows
    k_long = 4 * k
    a_codes, a_sf, a_ts = nvfp4_operand_k(m, k_long, 1.0)
    w_codes, w_sf, w_ts = nvfp4_operand_k(n, k_long, 0.02)
    codes, scales, ts, ws, hints = b.empty_nvfp4(m, n, device, hint_bits=HINT_BITS)
    smma = torch.empty(b.mma_scale_bytes(m, n // 16), **u8)
    ws.zero_()

    def call_long(r):
        b.nvfp4_gemm_quantize(a_codes, a_sf, a_ts, w_codes, w_sf, w_ts, m, n, k_long, ws, codes, scales,
                              ts, scales_mma=smma, hints=hints, hint_bits=HINT_BITS)

    call_long(0)
    torch.cuda.synchronize()
    ws[0] = ws[2]
    t_l = _timed(call_long, reps, flush)
    tf_l = 2.0 * m * n * k_long / t_l / 1e12
    out["long_k"] = {"workload": "NVFP4 [%d x %d] x NVFP4 weight [%d x %d]^T -> NVFP4 + %d-bit hints"
                                 % (m, k_long, n, k_long, HINT_BITS),
                     "avg_us": round(t_l * 1e6, 2), "TFLOP/s": round(tf_l, 1), "frac": round(tf_l / peak, 4),
                     "warning_bits": int(ws[1].item())}
    del a_codes, a_sf, w_codes, w_sf, codes, scales, smma, hints

    # MoE form: 8 experts x 2048 routed rows (8192 tokens, top-2), hidden k ->
    # expert width n_e, one launch for all experts, each expert its own scale
    E, rows_e, n_e = 8, 2048, 2048
    mm = E * rows_e
    a_codes, a_sf, a_ts = nvfp4_operand(mm, 1.0)
    parts = [nvfp4_operand(n_e, 0.02) for _ in range(E)]
    w_codes = torch.cat([p_[0] for p_ in parts])
    w_sf = torch.cat([p_[1] for p_ in parts])
    w_ts = torch.cat([p_[2] for p_ in parts])
    offs = torch.arange(0, mm + 1, rows_e, dtype=torch.int32, device=device)
    codes, scales, ts, ws, hints = b.empty_nvfp4(mm, n_e, device, hint_bits=HINT_BITS)
    smma = torch.empty(b.mma_scale_bytes(mm, n_e // 16), **u8)
    ws.zero_()

    def moe(r):
        b.nvfp4_moe_gemm_quantize(a_codes, a_sf, a_ts, w_codes, w_sf, w_ts, offs, E, mm, n_e, k, ws, codes,
                                  scales, ts, scales_mma=smma, hints=hints, hint_bits=HINT_BITS)

    moe(0)
    torch.cuda.synchronize()
    ws[0] = ws[2]
    t_m = _timed(moe, reps, flush)
    tf_m = 2.0 * mm * n_e * k / t_m / 1e12
    out["moe"] = {"workload": "%d experts x %d routed rows, NVFP4 [%d x %d] x per-expert NVFP4 weight [%d x %d]^T "
                              "-> NVFP4 + %d-bit hints, one launch" % (E, rows_e, mm, k, n_e, k, HINT_BITS),
                  "avg_us": round(t_m * 1e6, 2), "TFLOP/s": round(tf_m, 1), "frac": round(tf_m / peak, 4),
                  "warning_bits": int(ws[1].item())}
    return out


def time_hint_transport(b, stack, device, reps=5):
    """The guidance that leaves the GPU in one step: the back-half layers'
    hints to pinned host memory, (1) through the library (nvfp4_hint_pack:
    one gather kernel into a staging buffer, then one copy) and (2) as one
    copy per layer on a copy stream; median of `reps` transfers each, with the
    size against the uncompacted NVFP4 of the same layers (4 + 0.5 bits per
    element)."""
    hinted = [l for l in range(stack.layers) if stack.hints[l] is not None]
    streams = [stack.hints[l] for l in hinted]
    nbytes = sum(t.numel() for t in streams)
    total = b.nvfp4_hint_pack_size([t.numel() for t in streams])
    staging = torch.empty(total, dtype=torch.uint8, device=device)
    host = torch.empty(max(total, nbytes), dtype=torch.uint8).pin_memory()
    copy = torch.cuda.Stream(device)

    def timed(fn):
        times, gather = [], []
        for _ in range(reps):
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            with torch.cuda.stream(copy):
                fn(ev)
            torch.cuda.synchronize()
            times.append(ev[0].elapsed_time(ev[2]) / 1e3)
            gather.append(ev[0].elapsed_time(ev[1]) / 1e3)
        return statistics.median(times), statistics.median(gather)

    def packed(ev):
        ev[0].record(copy)
        b.nvfp4_hint_pack(streams, staging, stream=copy)
        ev[1].record(copy)
        host[:total].copy_(staging, non_blocking=True)
        ev[2].record(copy)

    def per_layer(ev):
        ev[0].record(copy)
        ev[1].record(copy)
        off = 0
        for t in streams:
            host[off:off + t.numel()].copy_(t, non_blocking=True)
            off += t.numel()
        ev[2].record(copy)

    # the library call as one unit (gather + its own copy), for the record
    def library(ev):
        ev[0].record(copy)
        ev[1].record(copy)
        b.nvfp4_hint_pack(streams, staging, host, stream=copy)
        ev[2].record(copy)

    t_lib, _ = timed(library)
    t_pack, t_gather = timed(packed)
    t_direct, _ = timed(per_layer)
    uncompacted = stack.n * len(hinted) * 4.5 / 8
    return {"layers": "%d-%d" % (hinted[0], hinted[-1]), "hint_bits": HINT_BITS, "bytes_per_step": nbytes,
            "library_call": {"entry": "nvfp4_hint_pack (gather kernel + one copy to pinned host memory)",
                             "seconds": round(t_lib, 5), "GB/s": round(total / t_lib / 1e9, 2)},
            "gather_kernel": {"seconds": round(t_gather, 6), "GB/s": round(2 * total / t_gather / 1e9, 1),
                              "note": "device-to-device, read + write"},
            "per_layer_copies": {"seconds": round(t_direct, 5), "GB/s": round(nbytes / t_direct / 1e9, 2)},
            "uncompacted_nvfp4_bytes": int(uncompacted), "compaction": round(nbytes / uncompacted, 4),
            "context": "the TRACE explainer sizes guidance transport at 300 GB/s GPU->CPU (GB200); "
                       "this is the B200 host link with pinned memory"}


def run_e2e(b, stack, device, steps):
    """The same step with inputs copied from pinned host memory every step and
    the hints + counters read back, timed on the host around the device work.
    Host copies of 4 distinct layers are reused cyclically (host memory bound);
    copies run on a second stream, double-buffered against the kernels."""
    P = min(4, stack.layers)
    pin = lambda t: t.cpu().pin_memory()
    h_xr = [pin(stack.xr[l]) for l in range(P)]
    h_xt = [pin(stack.xt[l]) for l in range(P)]
    h_hints = [torch.empty(stack.n * HINT_BITS // 8, dtype=torch.uint8).pin_memory()
               for l in range(stack.layers) if stack.hints[l] is not None]
    h_stats = torch.empty_like(stack.stats, device="cpu").pin_memory()
    slots_r = [torch.empty_like(stack.xr[0]) for _ in range(2)]
    slots_t = [torch.empty_like(stack.xt[0]) for _ in range(2)]
    copy = torch.cuda.Stream(device)
    comp = torch.cuda.current_stream(device)
    h2d = d2h = 0

    def one_step():
        nonlocal h2d, d2h
        free = [torch.cuda.Event(), torch.cuda.Event()]
        for e in free:
            e.record(comp)
        stack.stats.zero_()
        hi = 0
        for l in range(stack.layers):
            s = l % 2
            ready = torch.cuda.Event()
            with torch.cuda.stream(copy):
                copy.wait_event(free[s])
                slots_r[s].copy_(h_xr[l % P], non_blocking=True)
                slots_t[s].copy_(h_xt[l % P], non_blocking=True)
                ready.record(copy)
            h2d += 2 * slots_r[s].numel() * 2
            comp.wait_event(ready)
            stack.run_layer(b, l, slots_r[s], slots_t[s])
            free[s].record(comp)
            if stack.hints[l] is not None:
                h_hints[hi].copy_(stack.hints[l], non_blocking=True)
                d2h += stack.hints[l].numel()
                hi += 1
        h_stats.copy_(stack.stats, non_blocking=True)
        d2h += stack.stats.numel() * 8

    one_step()  # warm-up (pins, first copies)
    torch.cuda.synchronize()
    h2d = d2h = 0
    t0 = time.perf_counter()
    for _ in range(steps):
        one_step()
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    return {"value": round(steps * stack.step_bytes() / dt / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d // steps, "d2h_bytes_per_step": d2h // steps, "steps": steps,
            "host_layers": "%d distinct layers in pinned host memory, used cyclically" % P}


def run_reference(args, world, rank, local):
    """The CPU oracle as the reference arm, on a bounded sample of the same
    workload per step (rank 0 only; other ranks exit)."""
    if rank != 0:
        return
    device = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    cores = _cores()
    rows_per_core = 256
    if device.type == "cuda":
        chunks = oracle_sample(device, 0, rows_per_core=rows_per_core, cores=cores)
    else:
        from train_rollout_alignment_b200 import synthetic as syn
        chunks = [syn.normal_pair((rows_per_core, COLS), 4 + i) for i in range(cores)]
        chunks = [(t, r) for t, r in chunks]
    nbytes, nel = oracle_bytes(chunks)
    for _ in range(args.warmup):
        time_oracle(chunks)
    dts = [time_oracle(chunks) for _ in range(args.steps)]
    dt = sum(dts)
    value = args.steps * nbytes / dt / 1e9
    sample = ("%d rows x %d cols of layer 24 (train + rollout) per step, %d chunks of %d rows, one "
              "thread per chunk" % (len(chunks) * rows_per_core, COLS, len(chunks), rows_per_core))
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * dt / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded)", "config": _config(args.layers),
        "elements_per_s": round(args.steps * 2 * nel / dt, 1),
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": len(chunks), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))


if __name__ == "__main__":
    main()
