"""Benchmark of the weight-only quantised GEMM library on B200.

Headline: packed-weight GEMV GB/s on a Llama-7B-shaped decoder layer (qkv
4096->12288, o 4096->4096, gate/up 4096->22016, down 11008->4096), 3-bit codes,
group 128, one decode token (M = 1).  A *step* is one decode pass over the
layer: the four ``wq_gemm`` calls, inputs resident in HBM, each step on the
next of several distinct copies of the packed weights so that the working set
(> 3x L2) never sits in L2 between steps.

    value = (packed codes + fp16 scales/zeros + x + y bytes of one step)
            / (device time of one step),   summed over ranks (weak scaling).

The same JSON line carries the other rows of the path, measured in the same
run: M = 4 and 16 on the same layer (GEMV), the Llama-13B-shaped prefill GEMMs
at M = 2048 (tensor cores, TFLOP/s) and the quantiser (GB/s of fp16 weights
read), the roofline of the dominant kernel, an end-to-end figure through the C
ABI with host buffers, and the CPU oracle timed on a bounded sample.

``--impl reference`` times the CPU oracle (``oracle/``) on the same workload
and metric instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import wq_inputs  # noqa: E402

HEADLINE = "llama7b_layer_3b_g128"
PREFILL = "llama13b_prefill_4b_g128"
METRIC = "packed-weight GEMV GB/s"
UNIT = "GB/s"


# ----------------------------------------------------------------- accounting
def groups(K, group):
    return 1 if group in (0, K) else K // group


def linear_bytes(N, K, bits, group, M):
    """Algorithmic bytes of one y = x . W'^T: codes + scales + zeros + x + y."""
    return N * K * bits // 8 + N * groups(K, group) * 4 + M * K * 2 + M * N * 2


def step_bytes(workload, M):
    w = wq_inputs.WORKLOADS[workload]
    return sum(linear_bytes(N, K, w["bits"], w["group"], M) for _, N, K in w["linears"])


def aggregate(per_rank_ms, bytes_per_rank_step):
    """Whole-job throughput (GB/s) from the per-rank device times of one step:
    every rank processes its own layer copy, the job takes as long as the
    slowest rank."""
    world = len(per_rank_ms)
    t = max(per_rank_ms)
    return world * bytes_per_rank_step / (t * 1e-3) / 1e9, t


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while active."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index=0, period_s=0.01):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._on = threading.Event()
        self._stop = threading.Event()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def _run(self):
        while not self._stop.is_set():
            if self._on.is_set() and self._nv is not None:
                try:
                    mhz = self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM)
                    rs = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                    self.samples.append(mhz)
                    for name, bit in self.REASONS.items():
                        if rs & bit and name != "gpu_idle":
                            self.reasons.add(name)
                except Exception:  # noqa: BLE001
                    pass
            time.sleep(self.period)

    def __enter__(self):
        self._on.set()
        return self

    def __exit__(self, *exc):
        self._on.clear()

    def summary(self):
        self._stop.set()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons)}


# ----------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def recorded_traffic(kernel_key, source_file):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    has not changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel_key)
    if not rec:
        return None
    h = hashlib.sha256(open(os.path.join(ROOT, source_file), "rb").read()).hexdigest()
    return rec["bytes_per_launch"] if rec.get("source_sha256") == h else None


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def reduce_max(value: float) -> float:
    """Max of a float over ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ----------------------------------------------------------------- GPU legs
class Layer:
    """R distinct device copies of one workload's packed linears."""

    def __init__(self, workload, copies, seed):
        import torch
        import quantized_gemm_wq_b200 as wq
        self.w = wq_inputs.WORKLOADS[workload]
        self.bits, self.group = self.w["bits"], self.w["group"]
        self.copies = []
        base = []
        for li, (name, N, K) in enumerate(self.w["linears"]):
            Wh = wq_inputs.weight_f16(seed, li, N, K, dist=self.w["dist"])
            W = torch.from_numpy(Wh).cuda()
            base.append((N, K) + tuple(wq.wq_quantize_rtn(W, self.bits, self.group)))
            del W
        for r in range(copies):
            self.copies.append([(N, K, c.clone(), s.clone(), z.clone()) if r else (N, K, c, s, z)
                                for (N, K, c, s, z) in base])
        torch.cuda.synchronize()


def gpu_leg_decode(layer, M, steps, warmup, seed, sampler=None, per_launch=False):
    """Device time per step (ms) of the decode pass at batch M.

    Each weight copy's step (one ``wq_gemm`` per projection) is captured once
    in a CUDA graph; the timed region replays exactly ``steps`` graphs,
    cycling over the copies, between two events on the capture stream.  With
    ``per_launch`` the graphs also hold an event between consecutive launches,
    and the kernels' durations are read from the last replay of every graph
    (the last ``len(copies)`` steps of the timed region)."""
    import torch
    import quantized_gemm_wq_b200 as wq
    lin = layer.w["linears"]
    xs = [wq_inputs.activations_bf16(seed, 500 + i, M, K).cuda() for i, (_, N, K) in enumerate(lin)]
    ys = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for (_, N, K) in lin]
    b, g = layer.bits, layer.group
    st = torch.cuda.Stream()
    graphs, gevents = [], []
    for cp in layer.copies:
        # external events: recorded as graph nodes whose timestamps stay readable
        evs = ([torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(lin) + 1)]
               if per_launch else None)
        with torch.cuda.stream(st):          # warm the launch path before capture
            for j, (N, K, c, s, z) in enumerate(cp):
                wq.wq_gemm(xs[j], c, s, z, b, g, N, K, y=ys[j], stream=st)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=st):
            for j, (N, K, c, s, z) in enumerate(cp):
                if evs is not None:
                    evs[j].record(st)
                wq.wq_gemm(xs[j], c, s, z, b, g, N, K, y=ys[j], stream=st)
            if evs is not None:
                evs[-1].record(st)
        graphs.append(gr)
        gevents.append(evs)
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        with torch.cuda.stream(st):
            e0.record(st)
            for i in range(steps):
                graphs[i % len(graphs)].replay()
            e1.record(st)
        torch.cuda.synchronize()
    barrier()
    launch_ms = []
    if per_launch:
        for evs in gevents:
            launch_ms.append([evs[j].elapsed_time(evs[j + 1]) for j in range(len(lin))])
    ms = e0.elapsed_time(e1) / steps
    del graphs
    return ms, launch_ms


def gpu_leg_e2e(layer, M, steps, warmup, seed):
    """Same step through the C ABI with host buffers: per step, each x is
    copied from pinned host memory and each y read back to pinned host memory
    inside the timed region."""
    import torch
    import quantized_gemm_wq_b200 as wq
    lin = layer.w["linears"]
    xh = [wq_inputs.activations_bf16(seed, 500 + i, M, K).pin_memory() for i, (_, N, K) in enumerate(lin)]
    yh = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for (_, N, K) in lin]
    xd = [torch.empty(M, K, dtype=torch.bfloat16, device="cuda") for (_, N, K) in lin]
    yd = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for (_, N, K) in lin]
    b, g = layer.bits, layer.group

    def step(i):
        cp = layer.copies[i % len(layer.copies)]
        for j, (N, K, c, s, z) in enumerate(cp):
            xd[j].copy_(xh[j], non_blocking=True)
            wq.wq_gemm(xd[j], c, s, z, b, g, N, K, y=yd[j])
            yh[j].copy_(yd[j], non_blocking=True)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    h2d = sum(M * K * 2 for (_, N, K) in lin)
    d2h = sum(M * N * 2 for (_, N, K) in lin)
    return e0.elapsed_time(e1) / steps, h2d, d2h


def gpu_leg_prefill(steps, warmup, seed, sampler=None):
    """Each prefill GEMM timed alone with CUDA events, L2 flushed before every
    timed launch (a 512 MB memset outside the timed interval)."""
    import torch
    import quantized_gemm_wq_b200 as wq
    w = wq_inputs.WORKLOADS[PREFILL]
    M = w["Ms"][0]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    out = []
    for li, (name, N, K) in enumerate(w["linears"]):
        W = torch.from_numpy(wq_inputs.weight_f16(seed, li, N, K, dist=w["dist"])).cuda()
        c, s, z = wq.wq_quantize_rtn(W, w["bits"], w["group"])
        del W
        x = wq_inputs.activations_bf16(seed, 300 + li, M, K).cuda()
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        for _ in range(warmup):
            wq.wq_gemm(x, c, s, z, w["bits"], w["group"], N, K, y=y)
        torch.cuda.synchronize()
        ts = []
        ctx = sampler if sampler is not None else _Null()
        with ctx:
            for _ in range(steps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                wq.wq_gemm(x, c, s, z, w["bits"], w["group"], N, K, y=y)
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
        t = statistics.median(ts)
        out.append({"linear": f"{name} {K}->{N}", "M": M, "us": t * 1e3,
                    "tflops": 2 * M * N * K / (t * 1e-3) / 1e12})
        del c, s, z, x, y
    return out


def gpu_leg_quantize(seed, reps=5):
    """Quantiser throughput on the headline layer (GB/s of fp16 weights read
    plus packed output written)."""
    import torch
    import quantized_gemm_wq_b200 as wq
    w = wq_inputs.WORKLOADS[HEADLINE]
    tot_b, tot_t = 0, 0.0
    for li, (name, N, K) in enumerate(w["linears"]):
        W = torch.from_numpy(wq_inputs.weight_f16(seed, li, N, K, dist=w["dist"])).cuda()
        c, s, z = wq.wq_quantize_rtn(W, w["bits"], w["group"])
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            wq.wq_quantize_rtn(W, w["bits"], w["group"], codes=c, scales=s, zeros=z)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        tot_t += statistics.median(ts) * 1e-3
        tot_b += N * K * 2 + N * K * w["bits"] // 8 + N * groups(K, w["group"]) * 4
        del W, c, s, z
    return {"GBps": tot_b / tot_t / 1e9, "us": tot_t * 1e6}


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


# ----------------------------------------------------------------- CPU oracle
def oracle_sample(seconds_target=8.0, max_rows=None):
    """The CPU oracle (as it stands) on a bounded sample of the headline step:
    for every projection, the first R output rows at M = 1 (quantise in fp64,
    unpack, fp64 matmul), R doubling up to the full layer and whole passes
    repeated until the timed oracle matmuls add up to seconds_target.
    Returns (GB/s of the same algorithmic bytes, threads used, description)."""
    import oracle
    w = wq_inputs.WORKLOADS[HEADLINE]
    nthreads = os.cpu_count() or 1
    R = 256
    prepared = {}
    tot_b, tot_t, passes = 0, 0.0, 0
    while True:
        pb, pt = 0, 0.0
        for li, (name, N, K) in enumerate(w["linears"]):
            rows = np.arange(min(R, N))
            key = (li, len(rows))
            if key not in prepared:
                Wh = wq_inputs.weight_f16(0, li, N, K, dist=w["dist"], rows=rows)
                x = wq_inputs.activations_bf16(0, 500 + li, 1, K)
                q, s, z = oracle.quantize_rtn(wq_inputs.f16_bits(Wh), w["bits"], w["group"])
                prepared[key] = (oracle.pack(q, w["bits"]), s, z, wq_inputs.bf16_bits(x))
            words, s, z, xb = prepared[key]
            t0 = time.perf_counter()
            oracle.gemm(xb, words, s, z, len(rows), K, w["bits"], w["group"], nthreads=nthreads)
            pt += time.perf_counter() - t0
            pb += linear_bytes(len(rows), K, w["bits"], w["group"], 1)
        full = all(R >= N for _, N, _ in w["linears"]) or (max_rows is not None and R >= max_rows)
        if pt < seconds_target / 4 and not full:
            R *= 2
            continue
        tot_b += pb
        tot_t += pt
        passes += 1
        if tot_t >= seconds_target or passes >= 64:
            return (tot_b / tot_t / 1e9, nthreads,
                    f"oracle fp64 gemm (unpack, dequantise, dot) over the first {R} output rows "
                    f"of each of the 4 projections at M=1, {passes} pass(es), {tot_t:.2f} s of CPU time")


def run_reference(args, rank, world):
    if rank != 0:
        return
    vals = []
    desc = ""
    cores = os.cpu_count() or 1
    for _ in range(args.warmup):
        oracle_sample(seconds_target=0.1, max_rows=256)
    per_step = max(0.5, min(5.0, 60.0 / max(1, args.steps)))
    for _ in range(args.steps):
        v, cores, desc = oracle_sample(seconds_target=per_step, max_rows=2048)
        vals.append(v)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": HEADLINE, "M": 1},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- main
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--copies", type=int, default=5,
                    help="distinct device copies of the layer rotated over the steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None,
                    help="run one small profiling case instead of the benchmark: "
                         "decode | gemv:<i> | prefill:<i>")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.case:
        run_case(args.case)
        return
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
            return
        run_ours(args, rank, world, local)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


def run_case(case: str) -> None:
    """One small profiling case (for ncu): ``decode`` runs one decode step of
    the headline layer (the four M = 1 GEMV launches, after 3 warm-up steps);
    ``gemv:<linear index>`` one M = 1 GEMV of that projection; ``gemv16:<linear
    index>`` the same with a batch of 16 rows (the tensor-core GEMV);
    ``prefill:<linear index>`` one prefill GEMM (M = 2048) of the
    Llama-13B-shaped workload."""
    import torch
    import quantized_gemm_wq_b200 as wq
    kind, _, arg = case.partition(":")
    wl = PREFILL if kind == "prefill" else HEADLINE
    w = wq_inputs.WORKLOADS[wl]
    lins = list(enumerate(w["linears"]))
    if kind in ("gemv", "gemv16", "prefill"):
        lins = [lins[int(arg or 0)]]
    M = w["Ms"][0] if kind == "prefill" else (16 if kind == "gemv16" else 1)
    ops = []
    for li, (name, N, K) in lins:
        W = torch.from_numpy(wq_inputs.weight_f16(0, li, N, K, dist=w["dist"])).cuda()
        c, s, z = wq.wq_quantize_rtn(W, w["bits"], w["group"])
        del W
        x = wq_inputs.activations_bf16(0, 700 + li, M, K).cuda()
        ops.append((x, c, s, z, N, K))
    for _ in range(3):
        for (x, c, s, z, N, K) in ops:
            wq.wq_gemm(x, c, s, z, w["bits"], w["group"], N, K)
    torch.cuda.synchronize()
    for (x, c, s, z, N, K) in ops:
        wq.wq_gemm(x, c, s, z, w["bits"], w["group"], N, K)
    torch.cuda.synchronize()
    assert wq.wq_last_device_error() == wq.WQ_OK
    print(json.dumps({"case": case, "launches": len(ops), "ok": True}))


def run_ours(args, rank, world, local):
    import torch
    torch.cuda.set_device(local)
    import quantized_gemm_wq_b200 as wq  # noqa: F401  (fails loudly without libwq.so)
    peaks = measured_peaks()
    sampler = ClockSampler(local)
    seed = 1000 + rank                      # each rank decodes its own layer
    layer = Layer(HEADLINE, args.copies, seed)
    w = wq_inputs.WORKLOADS[HEADLINE]
    b1 = step_bytes(HEADLINE, 1)

    # headline: M = 1 decode step, per-launch events for the roofline
    ms, launch_ms = gpu_leg_decode(layer, 1, args.steps, args.warmup, seed, sampler,
                                   per_launch=True)
    ms_max = reduce_max(ms)
    value, _ = aggregate([ms_max] * world, b1)
    # dominant kernel: the M = 1 GEMV; a step is its 4 launches back to back in
    # a CUDA graph, so its average throughput is the step's algorithmic bytes
    # over the step's device time.  Per-launch event times (graph event nodes,
    # ~2 us timestamp granularity) are reported alongside.
    per_lin_ms = [statistics.mean(r[j] for r in launch_ms) for j in range(len(w["linears"]))]
    lin_b = [linear_bytes(N, K, w["bits"], w["group"], 1) for _, N, K in w["linears"]]
    # the step without per-launch events (events add a little host work per launch)
    ms_plain, _ = gpu_leg_decode(layer, 1, args.steps, args.warmup, seed, sampler)
    ms_plain = reduce_max(ms_plain)
    value_plain, _ = aggregate([ms_plain] * world, b1)

    other_m = {}
    for M in (4, 16):
        t, _ = gpu_leg_decode(layer, M, args.steps, args.warmup, seed, sampler)
        t = reduce_max(t)
        other_m[str(M)] = {"GBps": world * step_bytes(HEADLINE, M) / (t * 1e-3) / 1e9,
                           "us_per_step": t * 1e3}
    e2e_ms, h2d, d2h = gpu_leg_e2e(layer, 1, args.steps, args.warmup, seed)
    e2e_ms = reduce_max(e2e_ms)
    del layer
    torch.cuda.empty_cache()
    prefill = gpu_leg_prefill(max(5, min(args.steps, 20)), args.warmup, seed, sampler)
    quant = gpu_leg_quantize(seed)
    clocks = sampler.summary()

    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        v, cores, desc = oracle_sample()
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
    best_pf = max(p["tflops"] for p in prefill)
    line = {
        "metric": METRIC, "value": value_plain, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_plain,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": HEADLINE, "M": 1, "bits": w["bits"], "group": w["group"],
                   "linears": [f"{n} {K}->{N}" for n, N, K in w["linears"]],
                   "bytes_per_step": b1, "l2": f"{args.copies} rotating weight copies "
                   f"({args.copies * b1 / 1e6:.0f} MB > L2)", "parallelism": f"replicas{world}"},
        "roofline": {"bound": "hbm", "kernel": "gemv_m1_tma_kernel<3>",
                     "achieved": value_plain / world, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": value_plain / world / peaks["hbm_gbs"],
                     "peak_source": peaks["source"] + " (copy bandwidth, MEASURED_PEAKS.json hbm_gbs)",
                     "traffic": recorded_traffic("gemv_m1_tma_kernel<3>@" + HEADLINE,
                                                 "quantized_gemm_wq_b200/csrc/gemv_tma.cu"),
                     "algorithmic_bytes_per_launch": lin_b,
                     "launch_us_events": [t * 1e3 for t in per_lin_ms]},
        "e2e": {"value": world * b1 / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * len(w["linears"]),
        "decode_other_M": other_m,
        "decode_step_with_launch_events": {"GBps": value, "ms_per_step": ms_max},
        "prefill": {"workload": PREFILL, "bound": "tensor", "gemms": prefill,
                    "peak_tflops": peaks["bf16_tflops"],
                    "frac_best": best_pf / peaks["bf16_tflops"]},
        "quantize": {"workload": HEADLINE, **quant},
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
