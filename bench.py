"""Benchmark of the BitLinear W1.58A8 forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one pass of the whole hot path over one batch: for every linear
of the workload, the RMSNorm/absmax int8 quantisation of its input and the
W1.58A8 product with dequant epilogue.  Decode shapes (M <= 8) run it as one
kernel per linear (bitnet_bitlinear_gemv); the two-kernel path
(bitnet_quant_act + bitnet_linear_gemv) is timed alongside under
"unfused_step".  Larger batches use bitnet_quant_act + the tcgen05 GEMM.  Weight packing (absmean ternarisation) is the offline
step: it runs once before timing and is reported separately under "stages".

Timed region: W untimed warm-up steps, then exactly K steps replayed from
CUDA graphs, bracketed by a barrier and a device synchronisation, timed with
CUDA events on the launching stream; the max over ranks is taken.  Each step
reads a different copy of the packed weights (32 copies per linear, more
than twice the 126 MB L2 in total), the way successive layers of a model do,
so the weights come from HBM.  value = algorithmic bytes of all ranks' steps
/ max elapsed time.  With N > 1 every rank runs an independent replica (the
path has no exchange step), so scaling is weak.

Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle (the
plain single-threaded C++ definition) on a bounded sample of the same
workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bitlinear_absmean_ternary_b200 import synth  # noqa: E402

METRIC = "BitLinear W1.58A8: decode GB/s & prefill TOPS, % of B200 roofline"
DEFAULT_WORKLOAD = "decode_m1_2p5b_ffn"
EPS_W = 1e-5
EPS_RMS = 1e-5
COPIES = 32
GRAPH_STEPS = 128
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "gemv_decode_m1_2p5b_ffn.md")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- helpers

def load_peaks() -> tuple:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(names) -> str:
    """Hash of the kernel sources with comments and whitespace removed, so that
    an edit of a comment does not orphan an ncu summary of the same code."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "bitlinear_absmean_ternary_b200", "csrc", n), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(re.sub(r"\s+", "", text).encode())
    return h.hexdigest()[:16]


def profiled_traffic(path: str, src_hash: str):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    summary is missing or was taken on a different kernel source."""
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != src_hash:
        return None
    return float(m.group(1))


def linear_bytes(lin) -> dict:
    """Algorithmic bytes of one linear: quant (x in, x_q/a/rowsum out) and
    product (packed W, x_q, a, rowsum, gamma in; y out)."""
    xin = lin.M * lin.K * (2 if lin.x_dtype == "bf16" else 4) + (lin.K * 2 if lin.norm else 0)
    quant = xin + lin.M * lin.K + 8 * lin.M
    yb = lin.M * lin.N * (2 if lin.y_dtype == "bf16" else 4)
    prod = lin.N * lin.K // 4 + lin.M * lin.K + 8 * lin.M + 4 + yb
    return {"quant": quant, "product": prod, "x_in": xin, "y_out": yb}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self._nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                bits = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, group_active: bool, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if not group_active:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(group_active: bool, device=None):
    if group_active:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- CPU oracle

def oracle_step_sample(lins, time_budget_s: float):
    """Prepare oracle inputs and a callable running one bounded sample step.

    A sample step quantises every linear's input and forms the product for the
    first `rows` output features of each linear (all tokens), where `rows` is
    chosen so the step takes about time_budget_s.  Returns (step_fn,
    bytes_per_step, description)."""
    import oracle
    prep = []
    for lin in lins:
        W = lin.make_w(0)
        packed, gamma = oracle.pack_weights(W, EPS_W)
        x = lin.make_x(0)
        g = lin.make_gain(0)
        prep.append((lin, packed, gamma, x, g))

    def run(rows_frac: float):
        for lin, packed, gamma, x, g in prep:
            rows = max(1, int(round(lin.N * rows_frac)))
            xq, a, rs = oracle.quant_act(x, g, EPS_RMS)
            oracle.bitlinear(packed[:rows], gamma, lin.K, xq, a)

    # calibrate on a small fraction
    frac = 1.0 / 64
    t0 = time.perf_counter()
    run(frac)
    dt = max(time.perf_counter() - t0, 1e-6)
    frac = min(1.0, frac * time_budget_s / dt)

    def bytes_for(f):
        tot = 0
        for lin, *_ in prep:
            rows = max(1, int(round(lin.N * f)))
            b = linear_bytes(lin)
            tot += b["quant"] + rows * lin.K // 4 + lin.M * lin.K + 8 * lin.M + 4 + b["y_out"] * rows // lin.N
        return tot

    desc = (f"oracle on {frac * 100:.2f}% of the output features of every linear (all tokens; the full "
            f"quantisation of every input) per step")
    return (lambda: run(frac)), bytes_for(frac), desc, frac


def host_info() -> dict:
    """CPU model and logical core count of the host the oracle runs on."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def run_reference(args, lins, rank: int):
    if rank != 0:
        return
    budget = 100.0 / max(1, args.steps + args.warmup)  # whole run about 100 s of CPU work
    step, nbytes, desc, frac = oracle_step_sample(lins, budget)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = nbytes * args.steps / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": args.workload, "linears": [[l.M, l.K, l.N] for l in lins], "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": desc,
                         "host": host_info()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def run_ours(args, lins, ws: int, rank: int, local: int):
    import torch
    import bitlinear_absmean_ternary_b200 as bl

    if not torch.cuda.is_available():
        # no CPU fallback: the measured path is the CUDA library or nothing
        sys.exit("bench.py: no CUDA device; this arm times the CUDA library (the oracle is --impl reference)")
    group = False
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
        group = True
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    bl.lib()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.Stream(dev)

    # ---- inputs and offline weight packing (timed once, reported under "stages"); one
    # untimed pack first so that the library's first-call setup is not in the figure
    bl.bitnet_pack_weights(torch.ones((64, 64), dtype=torch.float32, device=dev), EPS_W)
    torch.cuda.synchronize(dev)
    packs, xs, gains, bufs = [], [], [], []
    pack_ms = []
    for lin in lins:
        W = torch.from_numpy(lin.make_w(0)).to(dev)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            P, G = bl.bitnet_pack_weights(W, EPS_W)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        pack_ms.append(e0.elapsed_time(e1))
        copies = [P] + [P.clone() for _ in range(COPIES - 1)]
        packs.append((copies, G))
        del W
        x = lin.make_x(0)
        if lin.x_dtype == "bf16":
            xt = torch.from_numpy(synth.f32_to_bf16_bits(x).view(np.int16).copy()).to(dev).view(torch.bfloat16)
        else:
            xt = torch.from_numpy(x).to(dev)
        xs.append(xt)
        g = lin.make_gain(0)
        if g is None:
            gains.append(None)
        elif lin.x_dtype == "bf16":
            gains.append(torch.from_numpy(synth.f32_to_bf16_bits(g).view(np.int16).copy()).to(dev).view(torch.bfloat16))
        else:
            gains.append(torch.from_numpy(g).to(dev))
        ydt = torch.bfloat16 if lin.y_dtype == "bf16" else torch.float32
        bufs.append({
            "xq": torch.empty((lin.M, lin.K), dtype=torch.int8, device=dev),
            "a": torch.empty(lin.M, dtype=torch.float32, device=dev),
            "rs": torch.empty(lin.M, dtype=torch.int32, device=dev),
            "y": torch.empty((lin.M, lin.N), dtype=ydt, device=dev),
        })
    torch.cuda.synchronize(dev)

    def quant(i, _c):
        b = bufs[i]
        bl.bitnet_quant_act(xs[i], gains[i], EPS_RMS, b["xq"], b["a"], b["rs"])

    def product(i, c):
        lin, b = lins[i], bufs[i]
        fn = bl.bitnet_linear_gemv if lin.M <= 8 else bl.bitnet_linear_gemm
        fn(packs[i][0][c % COPIES], packs[i][1], b["xq"], b["a"], b["rs"], y=b["y"])

    def fused(i, c):
        # quantisation + product in one kernel (decode shapes)
        b = bufs[i]
        bl.bitnet_bitlinear_gemv(xs[i], packs[i][0][c % COPIES], packs[i][1], gains[i], EPS_RMS, y=b["y"])

    def step_unfused(c):
        for i in range(len(lins)):
            quant(i, c)
            product(i, c)

    def step_fused(c):
        for i in range(len(lins)):
            fused(i, c)

    use_fused = all(l.M <= 8 and l.M * l.K <= 21504 for l in lins)
    step = step_fused if use_fused else step_unfused

    def capture(fn_per_step, nsteps: int, start: int = 0):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for s in range(nsteps):
                fn_per_step(start + s)
        return g

    def time_graph(graph, replays: int) -> float:
        barrier(group, dev)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):  # replay() launches on the current stream
            e0.record(stream)
            for _ in range(replays):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(group, dev)
        return e0.elapsed_time(e1)

    G = GRAPH_STEPS
    K = args.steps
    full, rem = divmod(K, G)
    g_main = capture(step, G)
    g_rem = capture(step, rem) if rem else None
    # warm-up: W untimed steps
    wfull, wrem = divmod(args.warmup, G)
    g_warm = capture(step, wrem) if wrem else None
    with torch.cuda.stream(stream):
        for _ in range(wfull):
            g_main.replay()
        if g_warm is not None:
            g_warm.replay()
    torch.cuda.synchronize(dev)
    # the timed region: exactly K steps
    kernels_per_step = (1 if use_fused else 2) * len(lins)
    with ClockSampler(dev.index) as clocks:
        barrier(group, dev)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # an event after every graph of G steps: per-step percentiles over the replays
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(full)]
        with torch.cuda.stream(stream):
            e0.record(stream)
            for r in range(full):
                g_main.replay()
                marks[r].record(stream)
            if g_rem is not None:
                g_rem.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(group, dev)
    el_ms = max_over_ranks(e0.elapsed_time(e1), group, dev)
    per_step_us = [(a.elapsed_time(b) if a is not None else e0.elapsed_time(b)) * 1e3 / G
                   for a, b in zip([None] + marks[:-1], marks)]
    step_stats = None
    if len(per_step_us) >= 2:
        qs = np.percentile(per_step_us, [10, 50, 90])
        step_stats = {"p10_us": float(qs[0]), "p50_us": float(qs[1]), "p90_us": float(qs[2]),
                      "samples": len(per_step_us), "per": f"graph replay of {G} steps"}
    step_bytes = sum(linear_bytes(l)["quant"] + linear_bytes(l)["product"] for l in lins)
    value = ws * K * step_bytes / (el_ms / 1e3) / 1e9

    # ---- per-kernel-kind graphs for the stage breakdown and the roofline (same
    # kernels, same launch configuration, same weight rotation, back to back)
    def per_stage(fn, label):
        g = capture(lambda c: [fn(i, c) for i in range(len(lins))], G)
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize(dev)
        reps = max(1, min(50, (K // G) // 4))
        ms = max_over_ranks(time_graph(g, reps), group, dev)
        return ms / (reps * G * len(lins))  # per launch

    prod_ms = per_stage(product, "product")
    quant_ms = per_stage(quant, "quant")
    fused_ms = per_stage(fused, "fused") if use_fused else None
    prod_bytes = statistics.mean(linear_bytes(l)["product"] for l in lins)
    quant_bytes = statistics.mean(linear_bytes(l)["quant"] for l in lins)
    hbm_peak = float(peaks["hbm_gbs"])
    if use_fused:
        # the dominant (only) kernel of the step: fused quantisation + GEMV;
        # its algorithmic bytes: x in, packed W, scales, y out
        kern, kern_ms = "gemv_kernel (fused quant + GEMV, bitnet_bitlinear_gemv)", fused_ms
        kern_bytes = statistics.mean(linear_bytes(l)["x_in"] + l.N * l.K // 4 + 4 + linear_bytes(l)["y_out"]
                                     for l in lins)
        src = kernel_source_hash(["gemv.cuh", "quant.cuh", "ptx.cuh"])
    elif lins[0].M <= 8:
        kern, kern_ms, kern_bytes = "gemv_kernel", prod_ms, prod_bytes
        src = kernel_source_hash(["gemv.cuh", "ptx.cuh"])
    else:
        kern, kern_ms, kern_bytes = "gemm_kernel", prod_ms, prod_bytes
        src = kernel_source_hash(["gemm.cuh", "ptx.cuh"])
    traffic = profiled_traffic(PROFILE_SUMMARY, src)
    achieved = kern_bytes / (kern_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                "traffic": traffic, "kernel": kern,
                "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)" if peak_src == "measured" else
                "fallback 6650 GB/s", "launch_us": kern_ms * 1e3, "bytes_per_launch": kern_bytes,
                "how": "back-to-back launches of this kernel alone in CUDA graphs over the rotating weight copies, "
                       "CUDA events on the launching stream; average time per launch"}

    # ---- the other path over the same K steps (four-call path when the fused one is timed above)
    unfused = None
    if use_fused:
        gu = capture(step_unfused, G)
        with torch.cuda.stream(stream):
            gu.replay()
        torch.cuda.synchronize(dev)
        reps = max(1, K // G)
        ms = max_over_ranks(time_graph(gu, reps), group, dev)
        unfused = {"value": ws * reps * G * step_bytes / (ms / 1e3) / 1e9, "unit": "GB/s",
                   "ms_per_step": ms / (reps * G), "steps": reps * G, "kernels_per_step": 2 * len(lins),
                   "what": "bitnet_quant_act + bitnet_linear_gemv per linear (two kernels)"}

    # ---- end to end through the public API with host buffers
    h2d = sum(linear_bytes(l)["x_in"] for l in lins)
    d2h = sum(linear_bytes(l)["y_out"] for l in lins)
    xs_host = [x.cpu().pin_memory() for x in xs]
    ys_host = [torch.empty_like(b["y"], device="cpu").pin_memory() for b in bufs]
    k_e2e = min(K, 4000)

    def e2e_step(c):
        for i, lin in enumerate(lins):
            xs[i].copy_(xs_host[i], non_blocking=True)
            if use_fused:
                fused(i, c)
            else:
                quant(i, c)
                product(i, c)
            ys_host[i].copy_(bufs[i]["y"], non_blocking=True)

    with torch.cuda.stream(stream):
        for c in range(min(200, k_e2e)):
            e2e_step(c)
        torch.cuda.synchronize(dev)
        barrier(group, dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for c in range(k_e2e):
            e2e_step(c)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(group, dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), group, dev)
    e2e = {"value": ws * k_e2e * step_bytes / (e2e_ms / 1e3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": k_e2e,
           "how": "eager Python calls of the public API per step: pinned H2D copy of every input, the BitLinear "
                  "call(s), D2H copy of every output"}

    # ---- prefill tensor-core GEMM (M = 4096), a secondary line of the same metric
    prefill = None
    if not args.no_prefill and lins[0].M <= 8:
        prefill = bench_prefill(torch, bl, dev, stream, peaks, peak_src, group)

    # ---- STE backward GEMMs at the prefill shapes, a secondary line
    ste = None
    if not args.no_ste and lins[0].M <= 8:
        ste = bench_ste(torch, bl, dev, stream, peaks, peak_src, group)

    # ---- the decode step on base-3 packed weights, a secondary line
    decode_b3 = None
    if not args.no_b3 and use_fused and all(l.M * ((l.K + 79) // 80 * 80) <= 24000 for l in lins):
        decode_b3 = bench_b3(torch, bl, dev, stream, lins, xs, gains, peaks, peak_src, group, el_ms / K)

    # ---- the one-launch decode FFN block (up, gate, squared-ReLU gating, down), a secondary line
    ffn_block = None
    if not args.no_ffn and lins[0].M <= 8:
        ffn_block = bench_ffn_block(torch, bl, dev, stream, peaks, peak_src, group)

    # ---- CPU oracle baseline (rank 0, N = 1)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        stepfn, nbytes, desc, _ = oracle_step_sample(lins, 1.0)
        stepfn()
        n, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < args.cpu_seconds:
            stepfn()
            n += 1
        el = time.perf_counter() - t0
        cpu = {"value": nbytes * n / el / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{n} steps, each {desc}; {el:.1f} s", "host": host_info()}

    if rank == 0:
        clk = clocks.summary()
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
            "ms_per_step": el_ms / K, "step_percentiles": step_stats, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": "int8", "data": "synthetic",
            "config": {"workload": args.workload, "linears": [[l.M, l.K, l.N] for l in lins],
                       "step": ("per linear: one bitnet_bitlinear_gemv kernel (RMSNorm/absmax int8 quantisation of "
                                "the input fused with the ternary GEMV and dequant)") if use_fused else
                               "per linear: bitnet_quant_act + ternary product with dequant",
                       "l2": f"{COPIES} rotating packed-weight copies per linear "
                             f"({COPIES * sum(l.N * l.K // 4 for l in lins) / 1e6:.0f} MB > 126 MB L2)",
                       "timing": f"CUDA graphs of {G} steps, programmatic dependent launch between kernels",
                       "parallelism": "replicas" if ws > 1 else "single"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": K * kernels_per_step,
            "clocks": clk,
            "unfused_step": unfused,
            "stages": {"quant_us_per_launch": quant_ms * 1e3, "quant_gbs": quant_bytes / (quant_ms / 1e3) / 1e9,
                       "product_us_per_launch": prod_ms * 1e3,
                       "fused_us_per_launch": None if fused_ms is None else fused_ms * 1e3,
                       "pack_ms": pack_ms, "pack_gbs": [l.N * l.K * 4.25 / (ms / 1e3) / 1e9
                                                        for l, ms in zip(lins, pack_ms)]},
            "prefill": prefill,
            "ffn_block": ffn_block,
            "decode_b3": decode_b3,
            "ste_backward": ste,
        }
        print(json.dumps(line), flush=True)
    if group:
        import torch.distributed as dist
        del g_main, g_rem
        dist.destroy_process_group()


def bench_b3(torch, bl, dev, stream, lins, xs, gains, peaks, peak_src, group, two_bit_step_ms):
    """The decode step with base-3 packed weights (bitnet_bitlinear_gemv_b3, five codes per byte): same
    linears, inputs, weight rotation and graphs as the 2-bit step; GB/s on the base-3 byte count."""
    packs = []
    for lin in lins:
        W = torch.from_numpy(lin.make_w(0)).to(dev)
        P, G = bl.bitnet_pack_weights_b3(W, EPS_W)
        del W
        packs.append(([P] + [P.clone() for _ in range(COPIES - 1)], G))
    ys = [torch.empty((l.M, l.N), dtype=torch.bfloat16 if l.y_dtype == "bf16" else torch.float32, device=dev)
          for l in lins]

    def step(c):
        for i in range(len(lins)):
            bl.bitnet_bitlinear_gemv_b3(xs[i], packs[i][0][c % COPIES], packs[i][1], gains[i], EPS_RMS, y=ys[i])

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in range(GRAPH_STEPS):
            step(c)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize(dev)
    reps = 40
    barrier(group, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(group, dev)
    ms = max_over_ranks(e0.elapsed_time(e1), group, dev) / (reps * GRAPH_STEPS)
    b3_bytes = sum(l.N * bl.bitnet_b3_row_bytes(l.K) for l in lins)
    step_bytes = b3_bytes + sum(linear_bytes(l)["x_in"] + 4 + linear_bytes(l)["y_out"] for l in lins)
    gbs = step_bytes / (ms / 1e3) / 1e9
    return {"us_per_step": ms * 1e3, "gbs": gbs, "frac": gbs / float(peaks["hbm_gbs"]),
            "weight_bytes_per_step": b3_bytes, "two_bit_us_per_step": two_bit_step_ms * 1e3,
            "device_status": bl.bitnet_get_device_status(),
            "timing": f"CUDA graphs of {GRAPH_STEPS} steps over {COPIES} rotating weight copies, per step"}


def bench_ste(torch, bl, dev, stream, peaks, peak_src, group):
    """Straight-through-estimator backward GEMMs (tcgen05 kind::f16, bf16 operands, fp32 accumulation) at the
    prefill shapes, M = 4096 tokens: input gradient dX = gamma dY q and weight gradient dW = bf16(dY a)^T x_q,
    per-launch CUDA-event time with L2 flushed (256 MB write) before each launch."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    bf16_peak = float(peaks["bf16_tflops"])
    out, tot_flop, tot_ms = {}, 0, 0.0
    for lin in synth.WORKLOADS["prefill_m4096_2p5b_ffn"]:
        M, N, K = lin.M, lin.N, lin.K
        W = torch.from_numpy(lin.make_w(0)).to(dev)
        P, G = bl.bitnet_pack_weights(W, EPS_W)
        del W
        x = torch.from_numpy(synth.f32_to_bf16_bits(lin.make_x(0)).view(np.int16).copy()).to(dev).view(torch.bfloat16)
        dY = torch.from_numpy(synth.f32_to_bf16_bits(synth.activations(M, N, 0, 99, "normal", 0.0, 1.0, "bf16"))
                              .view(np.int16).copy()).to(dev).view(torch.bfloat16)
        with torch.cuda.stream(stream):
            xq, a, _ = bl.bitnet_quant_act(x, None, EPS_RMS)
            dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
            dW = torch.empty((N, K), dtype=torch.float32, device=dev)
            ws = torch.empty(bl.bitnet_ste_weight_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
            wsx = torch.empty(bl.bitnet_ste_input_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
            tx, tw = [], []
            for it in range(13):
                flush.zero_()
                e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                e0.record(stream)
                bl.bitnet_ste_backward_input(P, G, dY, dX=dX, workspace=wsx)
                e1.record(stream)
                flush.zero_()
                e2.record(stream)
                e3 = torch.cuda.Event(enable_timing=True)
                bl.bitnet_ste_backward_weight(dY, xq, a, dW=dW, workspace=ws)
                e3.record(stream)
                torch.cuda.synchronize(dev)
                if it >= 3:
                    tx.append(e0.elapsed_time(e1))
                    tw.append(e2.elapsed_time(e3))
        flop = 2 * M * N * K
        msx = max_over_ranks(statistics.median(tx), group, dev)
        msw = max_over_ranks(statistics.median(tw), group, dev)
        out[f"K{K}_N{N}"] = {"dx_us": msx * 1e3, "dx_tflops": flop / (msx / 1e3) / 1e12,
                             "dw_us": msw * 1e3, "dw_tflops": flop / (msw / 1e3) / 1e12}
        tot_flop += 2 * flop
        tot_ms += msx + msw
    tf = tot_flop / (tot_ms / 1e3) / 1e12
    return {"workload": "prefill_m4096_2p5b_ffn", "tflops": tf, "unit": "TFLOP/s",
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16_peak, "unit": "TFLOP/s",
                         "frac": tf / bf16_peak, "peak_source": f"{peak_src} bf16_tflops"},
            "per_shape": out, "device_status": bl.bitnet_get_device_status(),
            "timing": "median of 10 single calls, L2 flushed before each; each call includes its operand "
                      "expansion pre-passes (codes to bf16 for dX; dY*a and x_q transposed to bf16 for dW)"}


def bench_ffn_block(torch, bl, dev, stream, peaks, peak_src, group, name="ffn_block_m1_2p5b"):
    """The one-launch decode FFN (bitnet_bitlinear_ffn_gemv: up and gate, squared-ReLU gating, sub-norm, down)
    back to back in CUDA graphs over rotating weight copies, beside the same three BitLinears as separate
    fused launches (without the gating step)."""
    blk = synth.FFN_BLOCKS[name]
    P = {}
    for which in ("up", "gate", "down"):
        W = torch.from_numpy(blk.make_w(which, 0)).to(dev)
        P[which] = bl.bitnet_pack_weights(W, EPS_W)
        del W
    copies = max(2, int(2 * 126e6 // blk.weight_bytes) + 1)
    cps = [[P[w][0]] + [P[w][0].clone() for _ in range(copies - 1)] for w in ("up", "gate", "down")]
    bf = lambda a: torch.from_numpy(synth.f32_to_bf16_bits(a).view(np.int16).copy()).to(dev).view(torch.bfloat16)
    x = bf(blk.make_x(0))
    gi, gs = (bf(g) for g in blk.make_gains(0))
    h = torch.empty((blk.M, blk.F), dtype=torch.bfloat16, device=dev)
    u = torch.empty((blk.M, blk.F), dtype=torch.bfloat16, device=dev)
    y = torch.empty((blk.M, blk.D), dtype=torch.bfloat16, device=dev)
    sync = torch.zeros(bl.BITNET_FFN_SYNC_BYTES, dtype=torch.uint8, device=dev)
    G = P["up"][1], P["gate"][1], P["down"][1]

    def ffn(c):
        bl.bitnet_bitlinear_ffn_gemv(x, cps[0][c % copies], G[0], cps[1][c % copies], G[1], cps[2][c % copies],
                                     G[2], gi, EPS_RMS, gs, EPS_RMS, h=h, y=y, sync=sync)

    def three(c):
        bl.bitnet_bitlinear_gemv(x, cps[0][c % copies], G[0], gi, EPS_RMS, y=u)
        bl.bitnet_bitlinear_gemv(x, cps[1][c % copies], G[1], gi, EPS_RMS, y=h)
        bl.bitnet_bitlinear_gemv(h, cps[2][c % copies], G[2], gs, EPS_RMS, y=y)

    def timed(fn, per=64, reps=40):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c in range(per):
                fn(c)
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
        torch.cuda.synchronize(dev)
        barrier(group, dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(group, dev)
        return max_over_ranks(e0.elapsed_time(e1), group, dev) / (per * reps)

    ms = timed(ffn)
    ms3 = timed(three)
    status = bl.bitnet_get_device_status()
    nbytes = blk.weight_bytes + 2 * blk.M * blk.D + 2 * (blk.D + blk.F) + 12 + 2 * blk.M * blk.F + 2 * blk.M * blk.D
    gbs = nbytes / (ms / 1e3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    traffic = profiled_traffic(os.path.join(ROOT, "profiles", "ffn_block_m1_2p5b.md"),
                               kernel_source_hash(["ffn.cuh", "gemv.cuh", "quant.cuh", "ptx.cuh"]))
    return {"workload": name, "M": blk.M, "D": blk.D, "F": blk.F, "us_per_ffn": ms * 1e3, "gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "traffic": traffic, "bytes_per_launch": nbytes,
                         "peak_source": f"{peak_src} hbm_gbs"},
            "three_fused_launches_us": ms3 * 1e3, "weight_copies": copies, "device_status": status,
            "timing": "CUDA graphs of 64 launches over rotating weight copies, CUDA events, per launch"}


def bench_prefill(torch, bl, dev, stream, peaks, peak_src, group):
    """Tensor-core GEMM at M = 4096 (K = 2560 -> N = 6912 and K = 6912 -> N = 2560):
    per-launch CUDA-event time with L2 flushed (256 MB write) before each launch."""
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    int8_peak = float(peaks["bf16_tflops"]) * 2.0  # dense int8 = 2x dense bf16 (nominal 4.5 vs 2.25 PFLOP/s)
    tot_ops, tot_ms = 0, 0.0
    for lin in synth.WORKLOADS["prefill_m4096_2p5b_ffn"]:
        W = torch.from_numpy(lin.make_w(0)).to(dev)
        P, G = bl.bitnet_pack_weights(W, EPS_W)
        del W
        x = torch.from_numpy(synth.f32_to_bf16_bits(lin.make_x(0)).view(np.int16).copy()).to(dev).view(torch.bfloat16)
        with torch.cuda.stream(stream):
            xq, a, rs = bl.bitnet_quant_act(x, None, EPS_RMS, want_rowsum=True)
            y = torch.empty((lin.M, lin.N), dtype=torch.bfloat16, device=dev)
            times = []
            qtimes = []
            for it in range(13):
                flush.zero_()
                e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                e0.record(stream)
                bl.bitnet_quant_act(x, None, EPS_RMS, xq, a, rs)
                e1.record(stream)
                bl.bitnet_linear_gemm(P, G, xq, a, rs, y=y)
                e2.record(stream)
                torch.cuda.synchronize(dev)
                if it >= 3:
                    qtimes.append(e0.elapsed_time(e1))
                    times.append(e1.elapsed_time(e2))
        ms = max_over_ranks(statistics.median(times), group, dev)
        qms = max_over_ranks(statistics.median(qtimes), group, dev)
        tops = lin.ops / (ms / 1e3) / 1e12
        qb = linear_bytes(lin)["quant"]
        out[f"K{lin.K}_N{lin.N}"] = {"gemm_us": ms * 1e3, "tops": tops, "frac": tops / int8_peak,
                                     "quant_us": qms * 1e3, "quant_gbs": qb / (qms / 1e3) / 1e9,
                                     "quant_frac": qb / (qms / 1e3) / 1e9 / float(peaks["hbm_gbs"])}
        tot_ops += lin.ops
        tot_ms += ms
    tops = tot_ops / (tot_ms / 1e3) / 1e12
    return {"workload": "prefill_m4096_2p5b_ffn", "tops": tops, "unit": "TOPS",
            "roofline": {"bound": "tensor", "achieved": tops, "peak": int8_peak, "unit": "TOP/s",
                         "frac": tops / int8_peak,
                         "peak_source": f"{peak_src} bf16_tflops x 2 (dense int8 / dense bf16 nominal ratio)"},
            "per_shape": out, "timing": "median of 10 single launches, L2 flushed before each"}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=51200)
    ap.add_argument("--warmup", type=int, default=1280)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-prefill", action="store_true", help="skip the secondary prefill GEMM measurement")
    ap.add_argument("--no-ffn", action="store_true", help="skip the secondary one-launch FFN block measurement")
    ap.add_argument("--no-b3", action="store_true", help="skip the secondary base-3 decode measurement")
    ap.add_argument("--no-ste", action="store_true", help="skip the secondary STE backward GEMM measurement")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    ws, rank, local = dist_setup()
    lins = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, lins, rank)
        return
    run_ours(args, lins, ws, rank, local)


if __name__ == "__main__":
    main()
