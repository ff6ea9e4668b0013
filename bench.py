"""Benchmark of the BitLinear W1.58A8 forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one pass of the whole hot path over one batch: for every linear
of the workload, the RMSNorm/absmax int8 quantisation of its input and the
W1.58A8 product with dequant epilogue.  Decode shapes (M <= 8) run it as one
kernel per linear (bitnet_bitlinear_gemv, quantisation fused into the GEMV);
batches of up to 64 tokens run bitnet_bitlinear_gemm (the quantisation, then
the stream-K or tile tcgen05 product); larger batches bitnet_quant_act + the
tcgen05 GEMM.  Weight packing
(absmean ternarisation) is the offline step: it runs once before timing and
is reported separately under "stages".

The headline workload is the largest configuration that fits one GPU: the
27B-class FFN at decode (M = 1, up 5376 -> 21504 and down 21504 -> 5376),
in GB/s.  Every other configuration of the benchmark set is measured in the
same run and reported under "configs", each with its own roofline and CPU
oracle baseline: the small correctness case, the 2.5B decode GEMV, the
batched decode through a 2.5B block (M = 64), the 2.5B prefill (M = 4096)
and the 27B FFN at M = 16 and M = 2048.

Timed region (headline): W untimed warm-up steps, then exactly K steps
replayed from CUDA graphs, bracketed by a barrier and a device
synchronisation, timed with CUDA events on the launching stream; the max over
ranks is taken.  Every graph the timed region replays has been replayed
before it starts.  Each step reads a different copy of the packed weights
(enough copies that one rotation is over three times the 126 MB L2), the way
successive layers of a model do, so the weights come from HBM.  value =
algorithmic bytes of all ranks' steps / max elapsed time.  With N > 1 every
rank runs an independent replica (the path has no exchange step), so scaling
is weak.

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
DEFAULT_WORKLOAD = "ffn27b_m1"
# the benchmark configurations, smallest first (each reported under "configs")
CONFIG_WORKLOADS = ["bitlinear_m4_k256_n256", "decode_m1_2p5b_ffn", "decode_m64_2p5b_block",
                    "prefill_m4096_2p5b_ffn", "ffn27b_m1", "ffn27b_m16", "ffn27b_m2048"]
EPS_W = 1e-5
EPS_RMS = 1e-5
L2_BYTES = 126e6
MAX_COPIES = 32
GRAPH_STEPS = 128
FLUSH_BYTES = 256 << 20
NOMINAL_INT8_TOPS = 4500.0
PROFILES = os.path.join(ROOT, "profiles")
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


def profiled_traffic(path: str, src_hash: str, key: str = "traffic_bytes_per_launch"):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    summary is missing or was taken on a different kernel source."""
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(re.escape(key) + r":\s*([0-9.eE+]+)", text)
    h = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    if not m or not h or h.group(1) != src_hash:
        return None
    return float(m.group(1))


def linear_bytes(lin) -> dict:
    """Algorithmic bytes of one linear: quant (x in, x_q/a/rowsum out) and
    product (packed W, x_q, a, rowsum, gamma in; y out); `fused` is the
    fused decode kernel's (x in, packed W, gamma, y out)."""
    xin = lin.M * lin.K * (2 if lin.x_dtype == "bf16" else 4) + (lin.K * 2 if lin.norm else 0)
    quant = xin + lin.M * lin.K + 8 * lin.M
    yb = lin.M * lin.N * (2 if lin.y_dtype == "bf16" else 4)
    w = lin.N * lin.K // 4
    prod = w + lin.M * lin.K + 8 * lin.M + 4 + yb
    return {"quant": quant, "product": prod, "fused": xin + w + 4 + yb, "x_in": xin, "y_out": yb, "w": w}


def gemv1_used(lin, sms: int = 148) -> bool:
    """Whether the decode GEMV of a linear runs the one-token whole-row-slot kernel: one token, more than 64 KB
    of packed weights per SM, K within its register budget -- the library's rule, restated to name the kernel."""
    rows = -(-lin.N // min(lin.N, sms))
    return lin.M == 1 and rows * (lin.K // 4) > 64 * 1024 and lin.K <= 65536


def sk_units(lin) -> int:
    """(128-row tile, 256-K step) units of the stream-K product of a linear with M <= 64 tokens."""
    bn = 16 if lin.M <= 16 else (32 if lin.M <= 32 else 64)
    return -(-lin.N // 128) * -(-lin.M // bn) * -(-lin.K // 256)


def step_bytes(lins) -> int:
    """Algorithmic bytes of one step (quantisation + product of every linear);
    the same count for the fused and the two-kernel path."""
    return sum(linear_bytes(l)["quant"] + linear_bytes(l)["product"] for l in lins)


def step_ops(lins) -> int:
    return sum(l.ops for l in lins)


def int8_peak(peaks) -> float:
    """Dense int8 tensor peak: the measured dense bf16 burst x 2 (the nominal
    int8 / bf16 ratio, 4.5 / 2.25 PFLOP/s)."""
    return float(peaks["bf16_tflops"]) * 2.0


def roofline_bound(nbytes: float, ops: float, peaks) -> str:
    """'tensor' when the int8 contraction takes longer at peak than moving the
    algorithmic bytes at the measured HBM rate, else 'hbm'."""
    t_hbm = nbytes / (float(peaks["hbm_gbs"]) * 1e9)
    t_tc = ops / (int8_peak(peaks) * 1e12)
    return "tensor" if t_tc > t_hbm else "hbm"


def roofline(kernel: str, nbytes: float, ops: float, seconds: float, peaks, peak_src: str, how: str,
             traffic=None, launches: int = 1) -> dict:
    """Roofline object of a kernel: achieved rate of its algorithmic bytes or
    ops (per launch, summed over `launches` launches taking `seconds`)."""
    bound = roofline_bound(nbytes, ops, peaks)
    src = "measured (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    if bound == "hbm":
        peak = float(peaks["hbm_gbs"])
        ach = nbytes / seconds / 1e9
        out = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
               "peak_source": f"{src} hbm_gbs"}
    else:
        peak = int8_peak(peaks)
        ach = ops / seconds / 1e12
        out = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TOP/s", "frac": ach / peak,
               "frac_of_nominal_int8": ach / NOMINAL_INT8_TOPS,
               "peak_source": f"{src} bf16_tflops x 2 (dense int8 / dense bf16 nominal ratio)"}
    out.update({"kernel": kernel, "traffic": traffic, "launch_us": seconds / launches * 1e6,
                "bytes_per_launch": nbytes / launches, "ops_per_launch": ops / launches, "how": how})
    return out


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

    def _sample(self):
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
            bits = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for b, name in self.REASONS.items():
                if bits & b:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
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
            self._sample()  # one sample at the end of the region as well

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


def config_unit(lins, peaks) -> str:
    """A configuration's rate unit: TOPS when its product is tensor-bound, else GB/s."""
    b = sum(linear_bytes(l)["product"] for l in lins)
    return "TOPS" if roofline_bound(b, step_ops(lins), peaks) == "tensor" else "GB/s"


# ----------------------------------------------------------------------------- CPU oracle

_WCACHE = {}


def weights_for(lin):
    """Latent fp32 weights of a linear, generated once per weight spec."""
    key = (lin.N, lin.K, lin.w_sigma, lin.w_id)
    if key not in _WCACHE:
        _WCACHE[key] = lin.make_w(0)
    return _WCACHE[key]


_OCACHE = {}


def oracle_packed(lin):
    import oracle
    key = (lin.N, lin.K, lin.w_sigma, lin.w_id)
    if key not in _OCACHE:
        _OCACHE[key] = oracle.pack_weights(weights_for(lin), EPS_W)
    return _OCACHE[key]


def oracle_sample(lins, budget_s: float, unit: str):
    """A bounded sample of one step of the workload on the CPU oracle.

    Every linear quantises `tok` token rows of its input (all of them, or a
    64-token slice for M >= 256, extrapolated per token) and forms the
    product for the first `rows` output features, `rows` chosen so that the
    call takes about budget_s.  Returns (call, work done per call in `unit`
    (bytes for GB/s, ops for TOPS), description)."""
    import oracle
    prep = []
    for lin in lins:
        packed, gamma = oracle_packed(lin)
        tok = lin.M if lin.M < 256 else 64
        x = lin.make_x(0)[:tok]
        g = lin.make_gain(0)
        prep.append((lin, packed, gamma, np.ascontiguousarray(x), g, tok))

    def run(frac: float):
        for lin, packed, gamma, x, g, tok in prep:
            rows = max(1, int(round(lin.N * frac)))
            xq, a, _ = oracle.quant_act(x, g, EPS_RMS)
            oracle.bitlinear(packed[:rows], gamma, lin.K, xq, a)

    frac = 1.0 / 256
    t0 = time.perf_counter()
    run(frac)
    dt = max(time.perf_counter() - t0, 1e-6)
    frac = min(1.0, frac * budget_s / dt)

    def work(f):
        tot = 0.0
        for lin, _p, _g, _x, _gn, tok in prep:
            rows = max(1, int(round(lin.N * f)))
            if unit == "TOPS":
                tot += 2.0 * tok * rows * lin.K
            else:
                b = linear_bytes(lin)
                tot += (b["quant"] * tok / lin.M + rows * lin.K // 4 + tok * lin.K + 8 * tok + 4
                        + b["y_out"] * tok / lin.M * rows / lin.N)
        return tot

    sliced = [p for p in prep if p[-1] != p[0].M]
    slice_note = f"; a {sliced[0][-1]}-token slice of every input, extrapolated per token" if sliced else ""
    desc = (f"oracle on {frac * 100:.2f}% of the output features of every linear (the full quantisation of the "
            f"tokens it takes){slice_note}")
    return (lambda: run(frac)), work(frac), desc


def cpu_baseline(lins, unit: str, seconds: float) -> dict:
    """The oracle as it stands, single-threaded, on a bounded sample (about `seconds` of CPU)."""
    step, work, desc = oracle_sample(lins, min(2.0, seconds / 3), unit)
    step()
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        step()
        n += 1
    el = time.perf_counter() - t0
    scale = 1e9 if unit == "GB/s" else 1e12
    return {"value": work * n / el / scale, "unit": unit, "cores": 1, "kind": "oracle",
            "sample": f"{n} calls in {el:.1f} s, each {desc}", "host": host_info()}


def run_reference(args, lins, rank: int):
    if rank != 0:
        return
    import oracle
    oracle.build()
    budget = 100.0 / max(1, args.steps + args.warmup)  # whole run about 100 s of CPU work
    unit = "GB/s"
    step, work, desc = oracle_sample(lins, budget, unit)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = work * args.steps / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": args.workload, "linears": [[l.M, l.K, l.N] for l in lins], "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": 1, "kind": "oracle", "sample": desc,
                         "host": host_info()},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

class Workload:
    """Device state of one workload: packed weights and, per linear, its input,
    quantised input and output buffers, all in `copies` rotated copies (one
    rotation over three times the 126 MB L2), and the launches of one step."""

    def __init__(self, torch, bl, dev, lins, packs, rotate: bool = True):
        self.torch, self.bl, self.dev, self.lins = torch, bl, dev, lins
        per_step = sum(linear_bytes(l)["quant"] + linear_bytes(l)["product"] for l in lins)
        self.copies = max(2, min(MAX_COPIES, math.ceil(3 * L2_BYTES / per_step))) if rotate else 1
        self.packs = [packs.get(torch, bl, dev, l, self.copies) for l in lins]
        self.xs, self.gains, self.bufs = [], [], []
        for lin in lins:
            x0 = self._act(lin.make_x(0), lin.x_dtype)
            self.xs.append([x0] + [x0.clone() for _ in range(self.copies - 1)])
            g = lin.make_gain(0)
            self.gains.append(None if g is None else self._act(g, lin.x_dtype))
            ydt = torch.bfloat16 if lin.y_dtype == "bf16" else torch.float32
            self.bufs.append([{
                "xq": torch.empty((lin.M, lin.K), dtype=torch.int8, device=dev),
                "a": torch.empty(lin.M, dtype=torch.float32, device=dev),
                "rs": torch.empty(lin.M, dtype=torch.int32, device=dev),
                "y": torch.empty((lin.M, lin.N), dtype=ydt, device=dev)} for _ in range(self.copies)])
        # the path of a step: one fused kernel per linear for decode-sized batches, else quantisation + product
        kmax = lambda l: 32768 if l.x_dtype == "bf16" else 16384
        if all(l.M <= 8 and l.M * l.K <= 21504 for l in lins):
            self.path = "gemv_fused"
        elif all(l.M <= 64 and l.K <= kmax(l) for l in lins):
            self.path = "gemm_fused"
        else:
            self.path = "quant_gemv" if all(l.M <= 8 for l in lins) else "quant_gemm"
        self.fused = self.path.endswith("_fused")
        # one workspace for the whole step (its calls run one after another on one stream)
        wsb = max([bl.bitnet_linear_gemm_workspace_bytes(l.M, l.N, l.K) for l in lins if l.M > 8] +
                  [bl.bitnet_bitlinear_gemm_workspace_bytes(l.M, l.N, l.K) for l in lins
                   if self.path == "gemm_fused"] or [0])
        self.ws = torch.zeros(wsb, dtype=torch.uint8, device=dev) if wsb else None
        # bitnet_bitlinear_gemm: the quantisation, then the stream-K product from 12 (row tile, K step)
        # units of work per SM, else the tile product -- the library's rule, restated here only to name
        # the product kernel
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        self.sk = [self.path == "gemm_fused" and sk_units(l) >= 12 * sms for l in lins]
        self.kernels_per_step = (1 if self.path == "gemv_fused" else 2) * len(lins)
        self.product_kernel = {
            "gemv_fused": ("gemv1_kernel (one token, whole-row slots; fused quantisation + GEMV, "
                           "bitnet_bitlinear_gemv)" if all(gemv1_used(l) for l in lins) else
                           "gemv_kernel (fused quantisation + GEMV, bitnet_bitlinear_gemv)"),
            "gemm_fused": ("gemm_sk_kernel (tcgen05 stream-K, after the quantisation, in bitnet_bitlinear_gemm)"
                           if all(self.sk) else
                           "gemm_kernel (tcgen05 tiles, after the quantisation, in bitnet_bitlinear_gemm)"
                           if not any(self.sk) else
                           "gemm_sk_kernel / gemm_kernel (tcgen05 stream-K or tiles per linear, after the "
                           "quantisation, in bitnet_bitlinear_gemm)"),
            "quant_gemv": "gemv_kernel (bitnet_linear_gemv)",
            "quant_gemm": ("gemm_sk_kernel (tcgen05 stream-K, bitnet_linear_gemm)" if all(l.M <= 64 for l in lins)
                           else "gemm_kernel (tcgen05, bitnet_linear_gemm)")}[self.path]

    @property
    def footprint_mb(self) -> float:
        return self.copies * sum(linear_bytes(l)["quant"] + linear_bytes(l)["product"] for l in self.lins) / 1e6

    def _act(self, a, dtype):
        torch = self.torch
        if dtype == "bf16":
            return torch.from_numpy(synth.f32_to_bf16_bits(a).view(np.int16).copy()).to(self.dev).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(self.dev)

    def x(self, i, c):
        return self.xs[i][c % self.copies]

    def buf(self, i, c):
        return self.bufs[i][c % self.copies]

    def quant(self, i, c):
        b = self.buf(i, c)
        self.bl.bitnet_quant_act(self.x(i, c), self.gains[i], EPS_RMS, b["xq"], b["a"], b["rs"])

    def product(self, i, c):
        lin, b = self.lins[i], self.buf(i, c)
        if lin.M <= 8:
            self.bl.bitnet_linear_gemv(self.packs[i][0][c % self.copies], self.packs[i][1], b["xq"], b["a"],
                                       b["rs"], y=b["y"])
        else:
            self.bl.bitnet_linear_gemm(self.packs[i][0][c % self.copies], self.packs[i][1], b["xq"], b["a"],
                                       b["rs"], y=b["y"], workspace=self.ws)

    def fused_linear(self, i, c):
        if self.path == "gemv_fused":
            self.bl.bitnet_bitlinear_gemv(self.x(i, c), self.packs[i][0][c % self.copies], self.packs[i][1],
                                          self.gains[i], EPS_RMS, y=self.buf(i, c)["y"])
        else:
            self.bl.bitnet_bitlinear_gemm(self.x(i, c), self.packs[i][0][c % self.copies], self.packs[i][1],
                                          self.gains[i], EPS_RMS, y=self.buf(i, c)["y"], workspace=self.ws)

    def fused_linear_host(self, i, c, x_host, y_host):
        """The one-token/few-token decode linear with host buffers: pinned x in,
        fused kernel, pinned y out, in one C call (bitnet_bitlinear_gemv_host)."""
        self.bl.bitnet_bitlinear_gemv_host(x_host, self.x(i, c), self.packs[i][0][c % self.copies], self.packs[i][1],
                                           self.buf(i, c)["y"], y_host, self.gains[i], EPS_RMS)

    def linear(self, i, c):
        if self.fused:
            self.fused_linear(i, c)
        else:
            self.quant(i, c)
            self.product(i, c)

    def step(self, c):
        for i in range(len(self.lins)):
            self.linear(i, c)

    def step_unfused(self, c):
        for i in range(len(self.lins)):
            self.quant(i, c)
            self.product(i, c)


class PackCache:
    """Packed weights (and their rotated copies) per weight spec, shared by the
    workloads that use the same matrices; the pack time is recorded."""

    def __init__(self):
        self.d = {}
        self.pack_ms = {}

    def get(self, torch, bl, dev, lin, copies):
        key = (lin.N, lin.K, lin.w_sigma, lin.w_id)
        if key not in self.d:
            W = torch.from_numpy(weights_for(lin)).to(dev)
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            P, G = bl.bitnet_pack_weights(W, EPS_W)
            e1.record()
            torch.cuda.synchronize(dev)
            self.pack_ms[f"{lin.N}x{lin.K}"] = e0.elapsed_time(e1)
            del W
            self.d[key] = ([P], G)
        lst, G = self.d[key]
        while len(lst) < copies:
            lst.append(lst[0].clone())
        return lst, G


def capture(torch, stream, fn_per_step, nsteps: int, start: int = 0):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for s in range(nsteps):
            fn_per_step(start + s)
    return g


def replay_ms(torch, dev, stream, graph, replays: int, group=False) -> float:
    """CUDA-event time of `replays` back-to-back replays (the graph was replayed before)."""
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
    return max_over_ranks(e0.elapsed_time(e1), group, dev)


def per_launch_ms(torch, dev, stream, wl, fn, i, steps: int = GRAPH_STEPS, replays: int = 10, group=False) -> float:
    """Average time of one launch kind of linear i, back to back in a CUDA graph
    over the rotating weight copies (after one untimed replay)."""
    g = capture(torch, stream, lambda c: fn(i, c), steps)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize(dev)
    return replay_ms(torch, dev, stream, g, replays, group) / (steps * replays)


def measure_rotating(torch, bl, dev, stream, wl, peaks, peak_src, group, steps=GRAPH_STEPS, replays=20) -> dict:
    """A decode-sized configuration: steps back to back in CUDA graphs over the
    rotating weight copies, and each kernel kind alone the same way."""
    g = capture(torch, stream, wl.step, steps)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize(dev)
    ms = replay_ms(torch, dev, stream, g, replays, group) / (steps * replays)
    lins = wl.lins
    per = []
    for i, lin in enumerate(lins):
        prod = wl.fused_linear if wl.fused else wl.product
        pms = per_launch_ms(torch, dev, stream, wl, prod, i, steps=steps, replays=max(2, replays // 2), group=group)
        qms = None if wl.fused else per_launch_ms(torch, dev, stream, wl, wl.quant, i, steps=steps,
                                                  replays=max(2, replays // 2), group=group)
        qb = linear_bytes(lin)["quant"]
        per.append({"linear": lin.name, "M": lin.M, "K": lin.K, "N": lin.N, "product_us": pms * 1e3,
                    "product_tops": lin.ops / (pms / 1e3) / 1e12,
                    "quant_us": None if qms is None else qms * 1e3,
                    "quant_gbs": None if qms is None else qb / (qms / 1e3) / 1e9,
                    "quant_frac": None if qms is None else qb / (qms / 1e3) / 1e9 / float(peaks["hbm_gbs"])})
    kbytes = sum(linear_bytes(l)["fused" if wl.fused else "product"] for l in lins)
    ksec = sum(p["product_us"] for p in per) * 1e-6
    rl = roofline(wl.product_kernel, kbytes, step_ops(lins), ksec, peaks, peak_src,
                  "each linear's product kernel alone, back to back in CUDA graphs over the rotating weight copies, "
                  "CUDA events on the launching stream; bytes and time summed over the linears", launches=len(lins))
    unfused = None
    if wl.fused:
        # the same steps as two kernels per linear (quantisation, then the product)
        gu = capture(torch, stream, wl.step_unfused, steps)
        with torch.cuda.stream(stream):
            gu.replay()
        torch.cuda.synchronize(dev)
        ums = replay_ms(torch, dev, stream, gu, replays, group) / (steps * replays)
        del gu
        unfused = {"ms_per_step": ums, "kernels_per_step": 2 * len(lins),
                   "what": "bitnet_quant_act + the product per linear (two kernels)"}
    return {"ms_per_step": ms, "per_linear": per, "roofline": rl, "copies": wl.copies, "unfused_step": unfused,
            "device_status": bl.bitnet_get_device_status(),
            "timing": f"CUDA graphs of {steps} steps back to back over {wl.copies} rotated copies of every buffer "
                      f"({wl.footprint_mb:.0f} MB per rotation > 3 x 126 MB L2), {replays} replays after one untimed "
                      "replay, CUDA events"}


def measure_flushed(torch, bl, dev, stream, wl, peaks, peak_src, group, reps=10) -> dict:
    """Single cold steps: each step with the L2 flushed (256 MB write) before
    it; CUDA events around every kernel; medians of reps steps after 3
    untimed ones.  (The write-back of the flush's dirty lines lands on the
    first kernel, so this is a pessimistic figure.)"""
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    lins = wl.lins
    qt = [[] for _ in lins]
    pt = [[] for _ in lins]
    st = []
    with torch.cuda.stream(stream):
        for it in range(reps + 3):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(lins) + 1)]
            ev[0].record(stream)
            for i in range(len(lins)):
                wl.quant(i, 0)
                ev[2 * i + 1].record(stream)
                wl.product(i, 0)
                ev[2 * i + 2].record(stream)
            torch.cuda.synchronize(dev)
            if it >= 3:
                for i in range(len(lins)):
                    qt[i].append(ev[2 * i].elapsed_time(ev[2 * i + 1]))
                    pt[i].append(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]))
                st.append(ev[0].elapsed_time(ev[-1]))
    med = lambda v: max_over_ranks(statistics.median(v), group, dev)
    per = []
    for i, lin in enumerate(lins):
        qb = linear_bytes(lin)["quant"]
        qms, pms = med(qt[i]), med(pt[i])
        per.append({"linear": lin.name, "M": lin.M, "K": lin.K, "N": lin.N, "product_us": pms * 1e3,
                    "product_tops": lin.ops / (pms / 1e3) / 1e12, "quant_us": qms * 1e3,
                    "quant_gbs": qb / (qms / 1e3) / 1e9, "quant_frac": qb / (qms / 1e3) / 1e9 / float(peaks["hbm_gbs"])})
    kbytes = sum(linear_bytes(l)["product"] for l in lins)
    ksec = sum(p["product_us"] for p in per) * 1e-6
    rl = roofline(wl.product_kernel, kbytes, step_ops(lins), ksec, peaks, peak_src,
                  "single launches with the L2 flushed before each step, CUDA events; median of "
                  f"{reps}; ops and time summed over the linears", launches=len(lins))
    return {"ms_per_step": med(st), "per_linear": per, "roofline": rl, "device_status": bl.bitnet_get_device_status(),
            "timing": f"one step at a time with a {FLUSH_BYTES >> 20} MB L2 flush before it; median of {reps} "
                      "steps after 3 untimed ones"}


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
    packs = PackCache()
    # one untimed pack first so that the library's first-call setup is not in the pack figures
    bl.bitnet_pack_weights(torch.ones((64, 64), dtype=torch.float32, device=dev), EPS_W)
    torch.cuda.synchronize(dev)

    # ------------------------------------------------------------------ headline: exactly K steps
    wl = Workload(torch, bl, dev, lins, packs, rotate=True)
    K = args.steps
    G = min(GRAPH_STEPS, K)
    full, rem = divmod(K, G)
    g_main = capture(torch, stream, wl.step, G)
    g_rem = capture(torch, stream, wl.step, rem, start=full * G) if rem else None
    # warm-up: at least W steps, and every graph of the timed region replayed once
    warm_replays = max(1, math.ceil(max(0, args.warmup - rem) / G)) if full else 0
    with torch.cuda.stream(stream):
        for _ in range(warm_replays):
            g_main.replay()
        if g_rem is not None:
            g_rem.replay()
    torch.cuda.synchronize(dev)
    warm_steps = warm_replays * G + rem
    with ClockSampler(dev.index) as clocks:
        barrier(group, dev)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
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
    head_status = bl.bitnet_get_device_status()
    per_rep = [(a.elapsed_time(b) if a is not None else e0.elapsed_time(b)) * 1e3 / G
               for a, b in zip([None] + marks[:-1], marks)]
    step_stats = None
    if len(per_rep) >= 2:
        qs = np.percentile(per_rep, [10, 50, 90])
        step_stats = {"p10_us": float(qs[0]), "p50_us": float(qs[1]), "p90_us": float(qs[2]),
                      "samples": len(per_rep), "per": f"graph replay of {G} steps"}
    sbytes = step_bytes(lins)
    value = ws * K * sbytes / (el_ms / 1e3) / 1e9
    del g_main, g_rem

    # ------------------------------------------------------------------ the headline's kernels and roofline
    head = measure_rotating(torch, bl, dev, stream, wl, peaks, peak_src, group)
    rl = head["roofline"]
    if wl.fused and lins[0].K == 5376 and lins[0].N == 21504:
        rl["traffic"] = profiled_traffic(os.path.join(PROFILES, "gemv_decode_m1_27b_ffn.md"),
                                         kernel_source_hash(["gemv1.cuh", "gemv.cuh", "quant.cuh", "ptx.cuh"]))
    unfused = head.get("unfused_step")
    if unfused is not None:
        unfused = dict(unfused, value=ws * sbytes / (unfused["ms_per_step"] / 1e3) / 1e9, unit="GB/s")

    # ------------------------------------------------------------------ end to end through the public API
    h2d = sum(linear_bytes(l)["x_in"] for l in lins)
    d2h = sum(linear_bytes(l)["y_out"] for l in lins)
    xs_host = [wl.x(i, 0).cpu().pin_memory() for i in range(len(lins))]
    ys_host = [torch.empty_like(wl.buf(i, 0)["y"], device="cpu").pin_memory() for i in range(len(lins))]
    k_e2e = min(max(K, 200), 2000)

    # the decode workloads' public call takes host buffers itself (one C call per linear)
    host_call = wl.path == "gemv_fused"

    def e2e_loop(n, copies=True, calls=True):
        with torch.cuda.stream(stream):
            torch.cuda.synchronize(dev)
            barrier(group, dev)
            t0 = time.perf_counter()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for c in range(n):
                for i in range(len(lins)):
                    if copies and calls and host_call:
                        wl.fused_linear_host(i, c, xs_host[i], ys_host[i])
                        continue
                    if copies:
                        wl.x(i, c).copy_(xs_host[i], non_blocking=True)
                    if calls:
                        wl.linear(i, c)
                    if copies:
                        ys_host[i].copy_(wl.buf(i, c)["y"], non_blocking=True)
            b.record(stream)
            torch.cuda.synchronize(dev)
            host_ms = (time.perf_counter() - t0) * 1e3
            barrier(group, dev)
        return max_over_ranks(a.elapsed_time(b), group, dev), host_ms

    e2e_loop(min(200, k_e2e))
    e2e_ms, _ = e2e_loop(k_e2e)
    copies_ms, _ = e2e_loop(min(500, k_e2e), calls=False)
    calls_ms, calls_host_ms = e2e_loop(min(500, k_e2e), copies=False)
    nb = min(500, k_e2e)
    e2e = {"value": ws * k_e2e * sbytes / (e2e_ms / 1e3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": k_e2e, "us_per_step": e2e_ms * 1e3 / k_e2e,
           "breakdown_us_per_step": {"copies_only": copies_ms * 1e3 / nb, "api_calls_only": calls_ms * 1e3 / nb,
                                     "api_calls_host_wall": calls_host_ms * 1e3 / nb,
                                     "kernels_back_to_back": head["ms_per_step"] * 1e3},
           "how": ("eager Python calls of the public API per step: for each linear one bitnet_bitlinear_gemv_host "
                   "call (pinned H2D copy of the input, the fused kernel, D2H copy of the output, issued from C)"
                   if host_call else
                   "eager Python calls of the public API per step: pinned H2D copy of every input (torch), the "
                   "BitLinear call(s), D2H copy of every output (torch)") +
                  "; the breakdown repeats the loop with torch copies alone and the device-buffer calls alone"}
    del xs_host, ys_host

    # ------------------------------------------------------------------ every configuration
    configs = {}
    if not args.no_configs:
        for name in CONFIG_WORKLOADS:
            if name == args.workload:
                continue
            configs[name] = bench_config(torch, bl, dev, stream, name, packs, peaks, peak_src, group,
                                         rank == 0 and ws == 1 and not args.no_cpu, args.config_cpu_seconds)

    # ------------------------------------------------------------------ secondary kernels
    ffn_block = None
    if not args.no_ffn:
        ffn_block = {n: bench_ffn_block(torch, bl, dev, stream, peaks, peak_src, group, n)
                     for n in ("ffn_block_m1_27b", "ffn_block_m1_2p5b")}
    decode_b3 = None
    if not args.no_b3 and wl.path == "gemv_fused" and all(l.M * ((l.K + 79) // 80 * 80) <= 24000 for l in lins):
        decode_b3 = bench_b3(torch, bl, dev, stream, wl, peaks, group, el_ms / K)
    ste = None
    if not args.no_ste:
        ste = bench_ste(torch, bl, dev, stream, peaks, peak_src, group)

    # ------------------------------------------------------------------ CPU oracle baseline (rank 0, N = 1)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        cpu = cpu_baseline(lins, "GB/s", args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
            "warmup_steps_run": warm_steps, "ms_per_step": el_ms / K, "step_percentiles": step_stats,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": args.workload, "linears": [[l.M, l.K, l.N] for l in lins],
                       "step": {"gemv_fused": "per linear: one bitnet_bitlinear_gemv kernel (RMSNorm/absmax int8 "
                                              "quantisation of the input fused with the ternary GEMV and dequant)",
                                "gemm_fused": ("per linear: one bitnet_bitlinear_gemm call = the quantisation kernel "
                                               "+ the tcgen05 product with dequant (stream-K from 12 units of work "
                                               f"per SM, else tiles; stream-K per linear: {wl.sk})")}.get(
                                    wl.path, "per linear: bitnet_quant_act + ternary product with dequant"),
                       "l2": f"{wl.copies} rotated copies of every buffer ({wl.footprint_mb:.0f} MB per rotation "
                             "> 3 x 126 MB L2): inputs larger than L2, no flush",
                       "timing": f"CUDA graphs of {G} steps, programmatic dependent launch between kernels; every "
                                 "graph of the timed region replayed during the warm-up",
                       "parallelism": "replicas" if ws > 1 else "single"},
            "roofline": rl,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": K * wl.kernels_per_step,
            "clocks": clocks.summary(),
            "device_status": head_status,
            "kernels": {"ms_per_step_back_to_back": head["ms_per_step"], "per_linear": head["per_linear"]},
            "unfused_step": unfused,
            "stages": {"pack_ms": packs.pack_ms,
                       "pack_gbs": {k: int(k.split("x")[0]) * int(k.split("x")[1]) * 4.25 / (v / 1e3) / 1e9
                                    for k, v in packs.pack_ms.items()}},
            "configs": configs,
            "ffn_block": ffn_block,
            "decode_b3": decode_b3,
            "ste_backward": ste,
        }
        print(json.dumps(line), flush=True)
    if group:
        import torch.distributed as dist
        dist.destroy_process_group()


def bench_config(torch, bl, dev, stream, name, packs, peaks, peak_src, group, with_cpu, cpu_seconds) -> dict:
    """One configuration of the benchmark set: its step time, value in its unit,
    the roofline of its product kernel and the CPU oracle beside it.  Steps run
    back to back over rotated copies of every buffer; large batches also get
    single cold steps after an L2 flush ("cold")."""
    lins = synth.WORKLOADS[name]
    unit = config_unit(lins, peaks)
    big = any(l.M >= 256 for l in lins)
    wl = Workload(torch, bl, dev, lins, packs)
    m = measure_rotating(torch, bl, dev, stream, wl, peaks, peak_src, group, steps=16 if big else GRAPH_STEPS,
                         replays=5 if big else 20)
    if big:
        m["cold"] = measure_flushed(torch, bl, dev, stream, wl, peaks, peak_src, group)
    sec = m["ms_per_step"] / 1e3
    value = step_ops(lins) / sec / 1e12 if unit == "TOPS" else step_bytes(lins) / sec / 1e9
    out = {"workload": name, "linears": [[l.M, l.K, l.N] for l in lins], "value": value, "unit": unit,
           "us_per_step": m["ms_per_step"] * 1e3, "kernels_per_step": wl.kernels_per_step,
           "path": wl.path, **m}
    del wl
    torch.cuda.empty_cache()
    if with_cpu:
        out["cpu_baseline"] = cpu_baseline(lins, unit, cpu_seconds)
    return out


def bench_b3(torch, bl, dev, stream, wl, peaks, group, two_bit_step_ms):
    """The decode step with base-3 packed weights (bitnet_bitlinear_gemv_b3, five codes per byte): same
    linears, inputs and weight rotation as the 2-bit step; GB/s on the base-3 byte count."""
    lins = wl.lins
    packs = []
    for lin in lins:
        W = torch.from_numpy(weights_for(lin)).to(dev)
        P, G = bl.bitnet_pack_weights_b3(W, EPS_W)
        del W
        packs.append(([P] + [P.clone() for _ in range(wl.copies - 1)], G))
    def step(c):
        for i in range(len(lins)):
            bl.bitnet_bitlinear_gemv_b3(wl.x(i, c), packs[i][0][c % wl.copies], packs[i][1], wl.gains[i], EPS_RMS,
                                        y=wl.buf(i, c)["y"])

    g = capture(torch, stream, step, GRAPH_STEPS)
    with torch.cuda.stream(stream):
        for _ in range(2):
            g.replay()
    torch.cuda.synchronize(dev)
    reps = 10
    ms = replay_ms(torch, dev, stream, g, reps, group) / (reps * GRAPH_STEPS)
    b3_bytes = sum(l.N * bl.bitnet_b3_row_bytes(l.K) for l in lins)
    sb = b3_bytes + sum(linear_bytes(l)["x_in"] + 4 + linear_bytes(l)["y_out"] for l in lins)
    gbs = sb / (ms / 1e3) / 1e9
    del g, packs
    return {"us_per_step": ms * 1e3, "gbs": gbs, "frac": gbs / float(peaks["hbm_gbs"]),
            "weight_bytes_per_step": b3_bytes, "two_bit_us_per_step": two_bit_step_ms * 1e3,
            "device_status": bl.bitnet_get_device_status(),
            "timing": f"CUDA graphs of {GRAPH_STEPS} steps over {wl.copies} rotating weight copies, per step"}


def bench_ste(torch, bl, dev, stream, peaks, peak_src, group):
    """Straight-through-estimator backward GEMMs (tcgen05 kind::f16, bf16 operands, fp32 accumulation) at the
    prefill shapes, M = 4096 tokens: input gradient dX = gamma dY q and weight gradient dW = bf16(dY a)^T x_q,
    per-launch CUDA-event time with L2 flushed (256 MB write) before each launch."""
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    bf16_peak = float(peaks["bf16_tflops"])
    out, tot_flop, tot_ms = {}, 0, 0.0
    for lin in synth.WORKLOADS["prefill_m4096_2p5b_ffn"]:
        M, N, K = lin.M, lin.N, lin.K
        W = torch.from_numpy(weights_for(lin)).to(dev)
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
                e0, e1, e2, e3 = (torch.cuda.Event(enable_timing=True) for _ in range(4))
                e0.record(stream)
                bl.bitnet_ste_backward_input(P, G, dY, dX=dX, workspace=wsx)
                e1.record(stream)
                flush.zero_()
                e2.record(stream)
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
    copies = max(2, int(3 * L2_BYTES // blk.weight_bytes) + 1)
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

    def timed(fn, per=32, reps=10):
        g = capture(torch, stream, fn, per)
        with torch.cuda.stream(stream):
            for _ in range(2):
                g.replay()
        torch.cuda.synchronize(dev)
        return replay_ms(torch, dev, stream, g, reps, group) / (per * reps)

    ms = timed(ffn)
    ms3 = timed(three)
    status = bl.bitnet_get_device_status()
    nbytes = blk.weight_bytes + 2 * blk.M * blk.D + 2 * (blk.D + blk.F) + 12 + 2 * blk.M * blk.F + 2 * blk.M * blk.D
    gbs = nbytes / (ms / 1e3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    traffic = profiled_traffic(os.path.join(PROFILES, f"{name}.md"),
                               kernel_source_hash(["ffn.cuh", "gemv.cuh", "quant.cuh", "ptx.cuh"]))
    del cps, P
    return {"workload": name, "M": blk.M, "D": blk.D, "F": blk.F, "us_per_ffn": ms * 1e3, "gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "traffic": traffic, "bytes_per_launch": nbytes,
                         "peak_source": f"{peak_src} hbm_gbs"},
            "three_fused_launches_us": ms3 * 1e3, "weight_copies": copies, "device_status": status,
            "timing": "CUDA graphs of 32 launches over rotating weight copies, CUDA events, per launch"}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2560)
    ap.add_argument("--warmup", type=int, default=256)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU oracle time for the headline baseline")
    ap.add_argument("--config-cpu-seconds", type=float, default=3.0, help="CPU oracle time per configuration")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baselines")
    ap.add_argument("--no-configs", action="store_true", help="skip the other configurations")
    ap.add_argument("--no-ffn", action="store_true", help="skip the one-launch FFN block measurement")
    ap.add_argument("--no-b3", action="store_true", help="skip the base-3 decode measurement")
    ap.add_argument("--no-ste", action="store_true", help="skip the STE backward GEMM measurement")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.steps < 1:
        ap.error("--steps must be at least 1")
    ws, rank, local = dist_setup()
    lins = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, lins, rank)
        return
    run_ours(args, lins, ws, rank, local)


if __name__ == "__main__":
    main()
