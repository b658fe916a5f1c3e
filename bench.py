"""Benchmark of the weight-only quantised GEMM library on B200.

Headline: packed-weight GEMV GB/s of one decode step (M = 1) over a 32-layer
Llama-7B-shaped linear stack (per layer q, k, v, o 4096->4096, gate, up
4096->11008, down 11008->4096), 4-bit codes, group 128: 224 linears, 3.44 GB of
packed weights per step, far larger than L2, so every step streams its weights
from HBM.  Each projection has its own activation vector (the projections are
independent: no activation chaining).  A *step* is one ``wq_gemm_grouped`` call
over the 224 linears (one preparation launch and two persistent GEMV launches),
captured once in a CUDA graph; the timed region replays exactly K graphs.

    value = (packed codes + fp16 scales/zeros + x + y bytes of one step)
            / (device time of one step),   summed over ranks (weak scaling).

The same JSON line carries the other rows of the path, measured in the same
run: the stack at M = 4, 16 (grouped) and 64 (tcgen05 GEMM per linear), the
stack through 224 separate ``wq_gemm`` launches, the single 4096x4096 linear,
the Llama-7B-shaped 3-bit layer (M = 1, 4, 16), the OPT-175B-shaped FC1/FC2
at 2 and 8 bits, the Llama-13B-shaped prefill GEMMs (tensor cores, TFLOP/s),
the quantiser, the roofline of the dominant kernel, an end-to-end figure with
host buffers, and the CPU oracle timed on a bounded sample.

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

HEADLINE = "llama7b_stack32_4b_g128"
LAYER3B = "llama7b_layer_3b_g128"
LINEAR1 = "linear4096_4b_g128"
OPT2B, OPT8B = "opt175b_fc_2b_rowwise", "opt175b_fc_8b_rowwise"
PREFILL = "llama13b_prefill_4b_g128"
METRIC = "packed-weight GEMV GB/s"
UNIT = "GB/s"
KERNEL = "gemv_grouped_kernel<4, 1>"


# ----------------------------------------------------------------- accounting
def groups(K, group):
    return 1 if group in (0, K) else K // group


def linear_bytes(N, K, bits, group, M):
    """Algorithmic bytes of one y = x . W'^T: codes + scales + zeros + x + y."""
    return N * K * bits // 8 + N * groups(K, group) * 4 + M * K * 2 + M * N * 2


def step_bytes(workload, M):
    w = wq_inputs.WORKLOADS[workload]
    return sum(linear_bytes(N, K, w["bits"], w["group"], M) for _, N, K in w["linears"])


def step_flops(workload, M):
    w = wq_inputs.WORKLOADS[workload]
    return sum(2 * M * N * K for _, N, K in w["linears"])


def aggregate(per_rank_ms, bytes_per_rank_step):
    """Whole-job throughput (GB/s) from the per-rank device times of one step:
    every rank processes its own copy of the workload, the job takes as long
    as the slowest rank."""
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

    def __init__(self, device_index=0, period_s=0.005):
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


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


# ----------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def recorded_traffic(key, source_file):
    """DRAM bytes per step from a committed ncu summary, if the kernel source
    has not changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(key)
    if not rec:
        return None
    h = hashlib.sha256(open(os.path.join(ROOT, source_file), "rb").read()).hexdigest()
    return rec["bytes_per_step"] if rec.get("source_sha256") == h else None


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


# ----------------------------------------------------------------- device data
def _gen(seed, tid):
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(int(seed) * 1_000_003 + int(tid))
    return g


def device_weight_f16(seed, tid, N, K, dist):
    """Seeded fp16 weights drawn on the device (same distributions as
    wq_inputs: 0.02 N(0,1), or 0.02 t(4) as z / sqrt(chi2_4 / 4))."""
    import torch
    g = _gen(seed, tid)
    W = torch.empty(N, K, dtype=torch.float16, device="cuda")
    step = max(1, (1 << 26) // K)
    for r0 in range(0, N, step):
        n = min(step, N - r0)
        z = torch.randn(n, K, generator=g, device="cuda")
        if dist == "t4":
            c = torch.randn(4, n, K, generator=g, device="cuda").pow_(2).sum(0).div_(4.0)
            z = z / c.sqrt_()
        W[r0:r0 + n] = (z * 0.02).half()
    return W


def device_x(seed, tid, M, K):
    import torch
    return torch.randn(M, K, generator=_gen(seed, 7_000_000 + tid), device="cuda").to(torch.bfloat16)


class Linears:
    """The packed linears of a workload on the device: one quantisation per
    linear (``wq_quantize_rtn``), weights drawn on the device."""

    def __init__(self, workload, seed, copies=1):
        import torch
        import quantized_gemm_wq_b200 as wq
        self.w = wq_inputs.WORKLOADS[workload]
        self.bits, self.group = self.w["bits"], self.w["group"]
        self.lins = []
        for cp in range(copies):
            for li, (name, N, K) in enumerate(self.w["linears"]):
                W = device_weight_f16(seed + 101 * cp, li, N, K, self.w["dist"])
                c, s, z = wq.wq_quantize_rtn(W, self.bits, self.group)
                del W
                self.lins.append((f"{name}#{cp}" if copies > 1 else name, N, K, c, s, z))
        torch.cuda.synchronize()
        self.per_copy = len(self.w["linears"])

    def items(self, M, seed, copy=0):
        """(x, codes, scales, zeros, N, K, group, y) of one copy, fresh x and y."""
        import torch
        out = []
        for j in range(self.per_copy):
            name, N, K, c, s, z = self.lins[copy * self.per_copy + j]
            x = device_x(seed, j, M, K)
            y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            out.append((x, c, s, z, N, K, self.group, y))
        return out


def graph_time(step_fns, steps, warmup, sampler=None):
    """Device ms per step: each of ``step_fns`` (one per rotating copy) is
    captured once in a CUDA graph; the timed region replays ``steps`` graphs,
    cycling over them, between two events on the capture stream."""
    import torch
    st = torch.cuda.Stream()
    graphs = []
    for fn in step_fns:
        with torch.cuda.stream(st):
            fn(st)                      # warm the launch path before capture
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=st):
            fn(st)
        graphs.append(gr)
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with (sampler if sampler is not None else _Null()):
        with torch.cuda.stream(st):
            e0.record(st)
            for i in range(steps):
                graphs[i % len(graphs)].replay()
            e1.record(st)
        torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1) / steps
    del graphs
    return ms


def grouped_fn(items, bits, ws):
    import quantized_gemm_wq_b200 as wq
    return lambda st: wq.wq_gemm_grouped(items, bits, workspace=ws, stream=st)


def per_linear_fn(items, bits):
    import quantized_gemm_wq_b200 as wq
    return lambda st: [wq.wq_gemm(x, c, s, z, bits, g, N, K, y=y, stream=st)
                       for (x, c, s, z, N, K, g, y) in items]


def gbps(nbytes, ms):
    return nbytes / (ms * 1e-3) / 1e9


# ----------------------------------------------------------------- legs
def leg_stack(args, seed, sampler, world):
    """Headline and the other batch sizes on the 32-layer stack."""
    import torch
    import quantized_gemm_wq_b200 as wq
    stack = Linears(HEADLINE, seed)
    bits = stack.bits
    out = {}
    items1 = stack.items(1, seed)
    ws1 = wq.grouped_workspace(items1, bits)
    ms = reduce_max(graph_time([grouped_fn(items1, bits, ws1)], args.steps, args.warmup, sampler))
    out["headline_ms"] = ms
    out["per_linear_M1"] = None
    n_pl = max(args.warmup, min(args.steps, 100))
    ms_pl = reduce_max(graph_time([per_linear_fn(items1, bits)], n_pl, args.warmup, sampler))
    out["per_linear_M1"] = {"us_per_step": ms_pl * 1e3,
                            "GBps": world * gbps(step_bytes(HEADLINE, 1), ms_pl),
                            "launches_per_step": len(items1)}
    other = {}
    for M in (4, 16, 64):
        items = stack.items(M, seed)
        n = max(args.warmup, min(args.steps, 100 if M < 64 else 50))
        ws = wq.grouped_workspace(items, bits)
        t = reduce_max(graph_time([grouped_fn(items, bits, ws)], n, args.warmup, sampler))
        path = ("wq_gemm_grouped (persistent warp-MMA GEMV)" if M <= 16 else
                "wq_gemm_grouped (swap-AB tcgen05 GEMM, one launch per 64 linears)")
        del ws
        other[str(M)] = {"us_per_step": t * 1e3, "GBps": world * gbps(step_bytes(HEADLINE, M), t),
                         "TFLOPs": world * step_flops(HEADLINE, M) / (t * 1e-3) / 1e12, "path": path}
        if M == 64:
            tp = reduce_max(graph_time([per_linear_fn(items, bits)], max(args.warmup, min(args.steps, 30)),
                                       args.warmup, sampler))
            other[str(M)]["per_linear"] = {"us_per_step": tp * 1e3,
                                           "GBps": world * gbps(step_bytes(HEADLINE, M), tp),
                                           "path": "wq_gemm per linear (swap-AB tcgen05 GEMM, split-K clusters)"}
        del items
    out["other_M"] = other
    # end to end: per step, every x from one pinned host buffer, every y back
    # into one pinned host buffer, the grouped call in between (one graph)
    K_all = [K for (_, _, _, _, _, K, _, _) in items1]
    N_all = [N for (_, _, _, _, N, _, _, _) in items1]
    xd = torch.empty(sum(K_all), dtype=torch.bfloat16, device="cuda")
    yd = torch.empty(sum(N_all), dtype=torch.bfloat16, device="cuda")
    xh = torch.empty(sum(K_all), dtype=torch.bfloat16).pin_memory()
    yh = torch.empty(sum(N_all), dtype=torch.bfloat16).pin_memory()
    xh.copy_(torch.cat([it[0].view(-1) for it in items1]).cpu())
    e_items, ko, no = [], 0, 0
    for (x, c, s, z, N, K, g, y) in items1:
        e_items.append((xd[ko:ko + K].view(1, K), c, s, z, N, K, g, yd[no:no + N].view(1, N)))
        ko += K
        no += N

    def e2e_step(st):
        xd.copy_(xh, non_blocking=True)
        wq.wq_gemm_grouped(e_items, bits, workspace=ws1, stream=st)
        yh.copy_(yd, non_blocking=True)

    ms_e2e = reduce_max(graph_time([e2e_step], max(args.warmup, min(args.steps, 200)), args.warmup))
    out["e2e"] = {"value": world * gbps(step_bytes(HEADLINE, 1), ms_e2e), "unit": UNIT,
                  "h2d_bytes_per_step": int(xh.numel() * 2), "d2h_bytes_per_step": int(yh.numel() * 2),
                  "us_per_step": ms_e2e * 1e3,
                  "how": "CUDA graph per step: one H2D copy of all 224 x from pinned memory, "
                         "wq_gemm_grouped, one D2H copy of all 224 y into pinned memory"}
    del stack, items1, ws1
    torch.cuda.empty_cache()
    return out


def leg_layer3b(args, seed, sampler, world):
    """The 3-bit Llama-7B-shaped layer: 5 rotating weight copies (> L2)."""
    import torch
    import quantized_gemm_wq_b200 as wq
    copies = 5
    L = Linears(LAYER3B, seed, copies=copies)
    out = {"l2": f"{copies} rotating weight copies ({copies * step_bytes(LAYER3B, 1) / 1e6:.0f} MB > L2)"}
    n = max(args.warmup, min(args.steps, 300))
    for M in (1, 4, 16):
        its = [L.items(M, seed, cp) for cp in range(copies)]
        wss = [wq.grouped_workspace(it, L.bits) for it in its]
        t = reduce_max(graph_time([grouped_fn(it, L.bits, w) for it, w in zip(its, wss)], n, args.warmup,
                                  sampler))
        tp = reduce_max(graph_time([per_linear_fn(it, L.bits) for it in its], n, args.warmup, sampler))
        out[str(M)] = {"grouped_us": t * 1e3, "grouped_GBps": world * gbps(step_bytes(LAYER3B, M), t),
                       "per_linear_us": tp * 1e3, "per_linear_GBps": world * gbps(step_bytes(LAYER3B, M), tp)}
    del L
    torch.cuda.empty_cache()
    return out


def leg_linear1(args, seed, sampler, world):
    """The single 4096x4096 4-bit linear at M = 1: 48 rotating copies (430 MB)
    launched back to back in one graph; time per linear."""
    import torch
    import quantized_gemm_wq_b200 as wq
    copies = 48
    L = Linears(LINEAR1, seed, copies=copies)
    its = [L.items(1, seed, cp) for cp in range(copies)]
    flat = [it[0] for it in its]
    wss = [wq.grouped_workspace([it], L.bits) for it in flat]
    n = max(args.warmup, min(args.steps // 10, 50))

    def per_linear(st):
        for it in flat:
            per_linear_fn([it], L.bits)(st)

    def grouped_each(st):
        for it, w in zip(flat, wss):
            wq.wq_gemm_grouped([it], L.bits, workspace=w, stream=st)

    b = step_bytes(LINEAR1, 1)
    t = reduce_max(graph_time([per_linear], n, args.warmup, sampler)) / copies
    tg = reduce_max(graph_time([grouped_each], n, args.warmup, sampler)) / copies
    del L, its, flat, wss
    torch.cuda.empty_cache()
    return {"l2": f"{copies} rotating copies in one graph", "per_linear_us": t * 1e3,
            "per_linear_GBps": world * gbps(b, t), "grouped_us": tg * 1e3, "grouped_GBps": world * gbps(b, tg)}


def leg_opt(args, seed, sampler, world):
    """OPT-175B-shaped FC1 + FC2, per-row grids, 2 and 8 bits, M = 1."""
    import torch
    import quantized_gemm_wq_b200 as wq
    out = {}
    for wl in (OPT2B, OPT8B):
        L = Linears(wl, seed)
        it = L.items(1, seed)
        ws = wq.grouped_workspace(it, L.bits)
        n = max(args.warmup, min(args.steps // 5, 40))
        t = reduce_max(graph_time([per_linear_fn(it, L.bits)], n, args.warmup, sampler))
        tg = reduce_max(graph_time([grouped_fn(it, L.bits, ws)], n, args.warmup, sampler))
        b = step_bytes(wl, 1)
        out[wl] = {"per_linear_us": t * 1e3, "per_linear_GBps": world * gbps(b, t),
                   "grouped_us": tg * 1e3, "grouped_GBps": world * gbps(b, tg)}
        del L, it, ws
        torch.cuda.empty_cache()
    return out


def leg_prefill(steps, warmup, seed, sampler=None):
    """Each prefill GEMM timed alone with CUDA events, L2 flushed before every
    timed launch (a 512 MB memset outside the timed interval)."""
    import torch
    import quantized_gemm_wq_b200 as wq
    w = wq_inputs.WORKLOADS[PREFILL]
    M = w["Ms"][0]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    out = []
    for li, (name, N, K) in enumerate(w["linears"]):
        W = device_weight_f16(seed, 300 + li, N, K, w["dist"])
        c, s, z = wq.wq_quantize_rtn(W, w["bits"], w["group"])
        del W
        x = device_x(seed, 300 + li, M, K)
        y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        for _ in range(warmup):
            wq.wq_gemm(x, c, s, z, w["bits"], w["group"], N, K, y=y)
        torch.cuda.synchronize()
        ts = []
        with (sampler if sampler is not None else _Null()):
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


def leg_quantize(seed, reps=5):
    """Quantiser throughput on the 3-bit layer (GB/s of fp16 weights read plus
    packed output written)."""
    import torch
    import quantized_gemm_wq_b200 as wq
    w = wq_inputs.WORKLOADS[LAYER3B]
    tot_b, tot_t = 0, 0.0
    for li, (name, N, K) in enumerate(w["linears"]):
        W = device_weight_f16(seed, 900 + li, N, K, w["dist"])
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
    return {"workload": LAYER3B, "GBps": tot_b / tot_t / 1e9, "us": tot_t * 1e6}


# ----------------------------------------------------------------- CPU oracle
def oracle_sample(seconds_target=8.0, max_rows=None):
    """The CPU oracle (as it stands) on a bounded sample of the headline step:
    for each of the 7 projection shapes of a layer, the first R output rows at
    M = 1 (quantise in fp64, unpack, fp64 matmul), R doubling up to the full
    projection, and whole passes repeated until the timed oracle matmuls add up
    to seconds_target.  Returns (GB/s of the same algorithmic bytes, threads
    used, description)."""
    import oracle
    w = wq_inputs.WORKLOADS[HEADLINE]
    layer = w["linears"][:7]
    nthreads = os.cpu_count() or 1
    R = 256
    prepared = {}
    tot_b, tot_t, passes = 0, 0.0, 0
    while True:
        pb, pt = 0, 0.0
        for li, (name, N, K) in enumerate(layer):
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
        full = all(R >= N for _, N, _ in layer) or (max_rows is not None and R >= max_rows)
        if pt < seconds_target / 4 and not full:
            R *= 2
            continue
        tot_b += pb
        tot_t += pt
        passes += 1
        if tot_t >= seconds_target or passes >= 64:
            return (tot_b / tot_t / 1e9, nthreads,
                    f"oracle fp64 gemm (unpack, dequantise, dot) over the first {R} output rows "
                    f"of each of the 7 projections of one layer at M=1, {passes} pass(es), "
                    f"{tot_t:.2f} s of CPU time")


def oracle_quantize_sample(seconds_target=2.0):
    """The CPU oracle's quantiser (fp64 RTN on every host thread, then its
    packer) on the first rows of each projection of the 3-bit layer, the
    workload of the GPU quantiser line; GB/s of fp16 weights read plus codes,
    scales and zeros written.  Returns (GB/s, description)."""
    import oracle
    w = wq_inputs.WORKLOADS[LAYER3B]
    nthreads = os.cpu_count() or 1
    R = 64
    while True:
        tb, tt = 0, 0.0
        for li, (name, N, K) in enumerate(w["linears"]):
            rows = np.arange(min(R, N))
            Wb = wq_inputs.f16_bits(wq_inputs.weight_f16(0, 900 + li, N, K, dist=w["dist"], rows=rows))
            t0 = time.perf_counter()
            q, s, z = oracle.quantize_rtn(Wb, w["bits"], w["group"], nthreads=nthreads)
            oracle.pack(q, w["bits"])
            tt += time.perf_counter() - t0
            n = len(rows)
            tb += n * K * 2 + n * K * w["bits"] // 8 + n * groups(K, w["group"]) * 4
        if tt >= seconds_target or all(R >= N for _, N, _ in w["linears"]):
            return (tb / tt / 1e9, f"oracle fp64 quantise + pack of the first {R} rows of each projection "
                                   f"of the 3-bit layer, {tt:.2f} s of CPU time")
        R *= 2


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


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
                             "sample": desc, "cpu": cpu_model()},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- main
def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="measure the headline leg only (the stack at M = 1, 4, 16, 64)")
    ap.add_argument("--case", default=None,
                    help="run one small profiling case instead of the benchmark: "
                         "stack:<M>:<layers> | stackpl:<M>:<layers> | gemv:<i> | gemv16:<i> | prefill:<i>")
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
    """One small profiling case (for ncu), after 3 untimed repetitions:
    ``stack:<M>:<layers>`` one decode step over the first <layers> layers of
    the 32-layer stack (layers >= 2 exceed L2) as one wq_gemm_grouped call
    (``stackpl:`` the same as one wq_gemm per linear); ``gemv:<i>`` /
    ``gemv16:<i>`` one wq_gemm of projection i of the 3-bit layer at M = 1 / 16;
    ``prefill:<i>`` one prefill GEMM (M = 2048) of the 13B-shaped workload."""
    import torch
    import quantized_gemm_wq_b200 as wq
    kind, _, arg = case.partition(":")
    if kind in ("stack", "stackpl"):
        per_linear = kind == "stackpl"
        Ms, _, nl = arg.partition(":")
        M, layers = int(Ms or 1), int(nl or 4)
        w = wq_inputs.WORKLOADS[HEADLINE]
        items = []
        for li, (name, N, K) in enumerate(w["linears"][:7 * layers]):
            W = device_weight_f16(0, li, N, K, w["dist"])
            c, s, z = wq.wq_quantize_rtn(W, w["bits"], w["group"])
            del W
            items.append((device_x(0, li, M, K), c, s, z, N, K, w["group"]))
        ws = wq.grouped_workspace(items, w["bits"])
        for _ in range(4):
            if per_linear:
                for (x, c, s, z, N, K, g) in items:
                    wq.wq_gemm(x, c, s, z, w["bits"], g, N, K)
            else:
                wq.wq_gemm_grouped(items, w["bits"], workspace=ws)
        torch.cuda.synchronize()
        assert wq.wq_last_device_error() == wq.WQ_OK
        print(json.dumps({"case": case, "linears": len(items), "ok": True}))
        return
    wl = PREFILL if kind == "prefill" else LAYER3B
    w = wq_inputs.WORKLOADS[wl]
    lins = list(enumerate(w["linears"]))
    if kind in ("gemv", "gemv16", "prefill"):
        lins = [lins[int(arg or 0)]]
    M = w["Ms"][0] if kind == "prefill" else (16 if kind == "gemv16" else 1)
    ops = []
    for li, (name, N, K) in lins:
        W = device_weight_f16(0, li, N, K, w["dist"])
        c, s, z = wq.wq_quantize_rtn(W, w["bits"], w["group"])
        del W
        ops.append((device_x(0, 700 + li, M, K), c, s, z, N, K))
    for _ in range(4):
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
    seed = 1000 + rank                      # each rank decodes its own stack
    w = wq_inputs.WORKLOADS[HEADLINE]
    b1 = step_bytes(HEADLINE, 1)

    stack = leg_stack(args, seed, sampler, world)
    ms = stack["headline_ms"]
    value, _ = aggregate([ms] * world, b1)
    extra = {}
    if not args.headline_only:
        extra["llama7b_layer_3b_g128"] = leg_layer3b(args, seed, sampler, world)
        extra["linear4096_4b_g128"] = leg_linear1(args, seed, sampler, world)
        extra["opt175b_fc"] = leg_opt(args, seed, sampler, world)
        pf = leg_prefill(max(5, min(args.steps, 20)), args.warmup, seed, sampler)
        best = max(p["tflops"] for p in pf)
        extra["prefill"] = {"workload": PREFILL, "bound": "tensor", "gemms": pf,
                            "peak_tflops": peaks["bf16_tflops"], "frac_best": best / peaks["bf16_tflops"]}
        extra["quantize"] = leg_quantize(seed)
    clocks = sampler.summary()
    if wq.wq_last_device_error() != wq.WQ_OK:
        raise RuntimeError("a kernel gave up a bounded wait during the bench")

    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        v, cores, desc = oracle_sample()
        qv, qdesc = oracle_quantize_sample()
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
               "cpu": cpu_model(), "quantize": {"GBps": qv, "sample": qdesc}}
    per_rank = value / world
    nlaunch = 1 + (len(w["linears"]) + 127) // 128
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": HEADLINE, "M": 1, "bits": w["bits"], "group": w["group"],
                   "linears": len(w["linears"]), "layer": [f"{n} {K}->{N}" for n, N, K in w["linears"][:7]],
                   "bytes_per_step": b1, "path": "wq_gemm_grouped, one CUDA graph per step",
                   "l2": f"inputs larger than L2 ({b1 / 1e9:.2f} GB of packed weights per step)",
                   "parallelism": f"replicas{world}"},
        "roofline": {"bound": "hbm", "kernel": KERNEL, "achieved": per_rank, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": per_rank / peaks["hbm_gbs"],
                     "peak_source": peaks["source"] + " (copy bandwidth, MEASURED_PEAKS.json hbm_gbs)",
                     "traffic": recorded_traffic(f"{KERNEL}@{HEADLINE}", "quantized_gemm_wq_b200/csrc/gemv_grouped.cu"),
                     "algorithmic_bytes_per_step": b1,
                     "timed_span": f"the whole step: {nlaunch} launches (1 activation preparation, "
                                   f"{nlaunch - 1} persistent GEMV)"},
        "e2e": {k: v for k, v in stack["e2e"].items()},
        "gpu_launches": args.steps * nlaunch,
        "decode_stack32": {"per_linear_M1": stack["per_linear_M1"], "other_M": stack["other_M"]},
        **extra,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
