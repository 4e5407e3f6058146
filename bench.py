#!/usr/bin/env python
"""MoE-layer forward benchmark on B200: tokens/s and grouped-GEMM TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config mixtral] [--impl ours|reference]

One step = one whole layer forward (router, permute, up grouped GEMM with the
SiLU gate, down grouped GEMM, combine) over the workload's T tokens.  The
default workload is the Mixtral-shaped layer (T=4096, d=4096, E=8 top-2,
I=14336, Zipf s=1.0 routing skew).  Inputs are seeded synthetic tensors
resident in HBM; the L2 cache is flushed between timed steps, outside the
timed events: a 2x-L2 buffer is rewritten and then read back, so the step
starts with L2 holding only clean lines (no write-back of the flush's own
dirty lines is charged to the step).  Each step is timed with CUDA
events on the launching stream; with N > 1 (torchrun) every rank runs an
independent replica of the layer on its own tokens (the layer has no
exchange step on one node's data-parallel path), and the reported time is the
max over ranks.

Printed: ONE JSON line (rank 0) with the contract keys plus
  kernels      per-kernel average device time (staged run of the same kernels;
               router, permute and combine also on their own, back to back)
  roofline     the up-projection grouped GEMM against the measured bf16 peak
  e2e          the same metric through moe_forward_host (host buffers, H2D of x
               and D2H of the output inside the timed region; consecutive steps
               on two streams so copies overlap kernels; `serial` one at a time)
  cpu_baseline the fp64 oracle on a bounded token sample, on this host's cores
  clocks       SM clock / throttle reasons sampled during the timed region
  workloads    (default run at N=1) the same measurement -- ms_per_step,
               kernels, roofline, clocks, graph, e2e -- for the other layers
               of the pages' workloads (fine-grained balanced / skewed, their
               FP8 versions, decode) and the router microbenchmark
`--impl reference` times the oracle alone (the slow CPU reference arm), on
the same token batches the cpu_baseline leg uses.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workload import CONFIGS, make_inputs, make_router_logits, shape_of  # noqa: E402
from workload.gen import ROUTER_MICRO  # noqa: E402

METRIC = "MoE-layer tokens/s at 1 B200; grouped-GEMM TFLOP/s as % of dense tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# --------------------------------------------------------------------------- ranks
def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """The largest value of x over all ranks (the job is as slow as its slowest rank)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput of independent replicas: every rank's tokens over the slowest rank's step."""
    return world * tokens_per_rank / (ms_per_step_max * 1e-3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def workload_desc(s) -> str:
    parts = [f"{s.name}: T={s.T} d={s.d} E={s.E} top-{s.k} I={s.inter}"]
    if s.shared_inter:
        parts.append(f"+1 shared (I={s.shared_inter})")
    parts.append(("mx-e4m3 experts (power-of-two scales)" if s.mx else "fp8 e4m3 experts") if s.fp8 else "bf16")
    parts.append(f"Zipf s={s.zipf_s} logit bias" if s.zipf_s else "balanced router")
    if s.gather:
        parts.append("up GEMM gathers its A rows in the load")
    return ", ".join(parts)


L2_NOTE = "flushed between timed steps (2x L2 buffer rewritten then read back, outside the events)"


def config_block(s):
    return {"workload": workload_desc(s), "tokens_per_step": s.T, "seed": 1234, "l2": L2_NOTE,
            "parallelism": "replicas (one independent layer per GPU)",
            "kernels_note": "kernels.<stage>.us: inside whole forwards, an event before each kernel; "
                            "kernels.<stage>.isolated: " + ISOLATED_NOTE}


def host_cpu():
    """The host's CPU model and core count (reported beside the CPU baseline)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        usable = os.cpu_count()
    return {"cpu_model": model, "host_cores": os.cpu_count(), "usable_cores": usable}


class Flusher:
    """Evicts L2 between timed steps: a buffer of twice the L2 size is
    rewritten and then summed, so what L2 holds afterwards is clean lines of
    this buffer (the dirty ones were written back during the flush)."""

    def __init__(self, dev):
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        n = max(2 * l2, 256 << 20) // 4
        self.buf = torch.empty(n, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.fill_(1.0)
        torch.sum(self.buf, dim=0, out=self.sink)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every 10 ms through NVML
    on a background thread while the timed region runs; without NVML the
    summary says so instead of giving a number."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self.error = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(self.gpu)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def __enter__(self):
        import threading
        try:
            nv, h = self._handle()
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of a number
            self.error = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for b, name in self.REASONS.items():
                        if bits & b:
                            self.reasons.add(name)
                except Exception as e:
                    self.error = str(e)
                    return
                self._stop.wait(0.01)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [self.error or "no samples"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_min_mhz": float(min(self.samples)),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples),
                "sampler": "nvml every 10 ms during the timed region"}


# --------------------------------------------------------------------------- our arm
def build_lib():
    from grouped_gemm_03_b200.build import build
    build()
    import grouped_gemm_03_b200 as gg
    gg.lib()
    return gg


def make_cfg(gg, s):
    xdt = gg.MOE_F32 if s.x_dtype == "f32" else gg.MOE_BF16
    rdt = gg.MOE_F32 if s.router_dtype == "f32" else gg.MOE_BF16
    odt = gg.MOE_F32 if s.x_dtype == "f32" else gg.MOE_BF16
    edt = (gg.MOE_MXE4M3 if s.mx else gg.MOE_E4M3) if s.fp8 else gg.MOE_BF16
    return gg.make_config(s.T, s.d, s.E, s.k, s.inter, s.shared_inter, xdt, rdt, edt, odt, s.renormalize,
                          flags=gg.MOE_FLAG_GATHER_A if s.gather else 0)


HOLD_CYCLES = 2_000_000  # ~1 ms spin queued ahead of each timed step


def time_steps(fn, steps, warmup, flush, stream, hold=True):
    """Per-step device time.  With hold, a short spin kernel is queued after the
    L2 flush so the step's launches are already enqueued when its start event
    fires: the events then bracket device work, not host enqueue latency."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush()
        if hold:
            torch.cuda._sleep(HOLD_CYCLES)
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


STAGES = ("router", "permute", "up_gemm", "down_gemm", "combine")


def time_marked(gg, cfg, inp, weights, out, counts, ws, steps, flush, stream):
    """Per-kernel device time inside whole forwards: moe_forward_marked records an
    event before each of the layer's five kernels and one after the last."""
    def run(evs):
        gg.moe_forward_marked(cfg, inp["x"], inp["W_r"], inp["bias"], weights, evs, out, counts_out=counts, ws=ws)

    for _ in range(2):
        run([torch.cuda.Event(enable_timing=True) for _ in range(6)])
    torch.cuda.synchronize()
    per = {n: [] for n in STAGES}
    for _ in range(steps):
        flush()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        for e in evs:  # create the CUDA events before the hold so the timed launches are not delayed
            e.record(stream)
        torch.cuda._sleep(HOLD_CYCLES)
        run(evs)
        torch.cuda.synchronize()
        for i, n in enumerate(STAGES):
            per[n].append(evs[i].elapsed_time(evs[i + 1]))
    return {n: float(np.mean(v)) for n, v in per.items()}


E2E_NOTE = ("moe_forward_host with pinned host buffers, every step's host-to-device copy of x and "
            "device-to-host copy of the output inside the timed region; consecutive steps alternate "
            "between two streams (each with its own workspace and buffers), so one step's copies "
            "overlap the other's kernels; one event pair over all steps (the expert weights, larger "
            "than L2, stream from HBM every step)")
ISOLATED_HOLD_CYCLES = 8_000_000  # ~4 ms spin: every launch of the run is enqueued before it ends
ISOLATED_NOTE = ("the stage's own launches back to back through the library's entry point (moe_router_topk, "
                 "moe_permute, moe_combine), queued behind a spin kernel, each on its own copy of the "
                 "stage's input (copies totalling >= 2x L2, so every launch reads HBM); one event pair "
                 "over all launches")


def rotating_copies(t, dev, at_least=2):
    """Copies of `t` whose total size is at least twice the L2 cache (at most 16)."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    nbytes = t.numel() * t.element_size()
    n = int(min(16, max(at_least, -(-2 * l2 // max(nbytes, 1)))))
    return [t.clone() for _ in range(n)]


def time_back_to_back(fn, reps, flush, stream):
    """Device time per call of fn(i), i = 0..reps-1, launched back to back."""
    for i in range(2):
        fn(i)
    torch.cuda.synchronize()
    flush()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(ISOLATED_HOLD_CYCLES)
    a.record(stream)
    for i in range(reps):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def time_isolated(gg, s, inp, alg, dev, flush, stream, reps=16):
    """Per-launch device time of the router, permute and combine stages on their own
    (the in-forward breakdown puts an event between kernels, which also times each
    launch's latency; here consecutive launches overlap as they do in the forward)."""
    shared = bool(s.shared_inter)
    xs = rotating_copies(inp["x"], dev)
    rws = torch.empty(gg.lib().moe_router_workspace_size(s.T, s.E), dtype=torch.uint8, device=dev)
    pws = torch.empty(gg.lib().moe_permute_workspace_size(s.T, s.E), dtype=torch.uint8, device=dev)
    out = {}

    def router(i):
        return gg.router_topk(xs[i % len(xs)], inp["W_r"], s.k, bias=inp["bias"], renormalize=s.renormalize,
                              ws=rws)

    out["router"] = time_back_to_back(router, reps, flush, stream)
    idx, w = router(0)

    def permute(i):
        return gg.permute(xs[i % len(xs)], idx, s.E, append_shared=shared, fp8=s.fp8, mx=s.mx, ws=pws)

    if not s.gather:  # (with the gather flag the forward's permute writes only the plan)
        out["permute"] = time_back_to_back(permute, reps, flush, stream)
    plan = permute(0)
    rows = plan["row_to_token"].numel()
    Y = torch.randn((rows, s.d), device=dev).to(torch.bfloat16)
    Ys = rotating_copies(Y, dev)
    del Y, xs
    o = torch.empty((s.T, s.d), dtype=torch.bfloat16 if s.x_dtype != "f32" else torch.float32, device=dev)

    def combine(i):
        gg.combine(Ys[i % len(Ys)], plan["token_to_row"], w, shared, out_dtype=o.dtype, out=o)

    out["combine"] = time_back_to_back(combine, reps, flush, stream)
    del Ys
    torch.cuda.empty_cache()
    res = {}
    for name, t_ms in out.items():
        res[name] = {"us": round(t_ms * 1e3, 2), "gbs": round(alg[name]["bytes"] / (t_ms * 1e-3) / 1e9, 1)}
    return res


def traffic_from_profile(workload, stage, kernel_src_hash):
    """DRAM bytes per launch of `stage` on `workload` from the committed ncu summary, if it
    was taken on the kernel sources as they are now."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p)).get(workload, {}).get(stage)
    except (OSError, ValueError):
        return None
    if not d or d.get("source_sha256") != kernel_src_hash:
        return None
    return d.get("bytes_per_launch")


STAGE_SOURCES = {"router": ("router.cu", "router_tc.cu"), "permute": ("permute.cu",),
                 "up_gemm": ("grouped_gemm.cu",), "down_gemm": ("grouped_gemm.cu",), "combine": ("combine.cu",)}


def kernel_source_hash(stage):
    h = hashlib.sha256()
    for f in STAGE_SOURCES[stage] + ("ptx.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "grouped_gemm_03_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def algorithmic(s, counts=None):
    """Per-kernel algorithmic FLOPs / bytes of one forward (bf16)."""
    T, d, E, k, I = s.T, s.d, s.E, s.k, s.inter
    sh = 1 if s.shared_inter else 0
    R = T * k
    Rp = R + sh * T
    active = E if counts is None else int((np.asarray(counts) > 0).sum())
    eb = 1 if s.fp8 else 2
    xb = 4 if s.x_dtype == "f32" else 2
    ob = 4 if s.x_dtype == "f32" else 2
    return {
        "router": {"bytes": T * d * xb + E * d * (4 if s.router_dtype == "f32" else 2) + T * k * 8},
        "permute": {"bytes": T * d * xb + Rp * d * eb + T * k * 4 * 3},
        "up_gemm": {"flops": 2.0 * Rp * 2 * I * d,
                    "bytes": (active + sh) * 2 * I * d * eb + Rp * d * eb + Rp * I * eb},
        "down_gemm": {"flops": 2.0 * Rp * d * I,
                      "bytes": (active + sh) * d * I * eb + Rp * I * eb + Rp * d * 2},
        "combine": {"bytes": Rp * d * 2 + T * d * ob + T * k * 8},
    }


STAGE_NAMES = {"router": "router GEMM + softmax + top-k", "permute": "histogram / scan / scatter",
               "up_gemm": "up-projection grouped GEMM (SiLU gate)", "down_gemm": "down-projection grouped GEMM",
               "combine": "combine (gather, weight, sum + shared)"}


def roofline(s, alg, kernels, peaks, peak_kind):
    """The roofline entry of the kernel with the largest share of the step.  A GEMM
    whose algorithmic FLOP per byte is below the ridge point (tensor peak / HBM peak)
    is bound by HBM (the expert weights), otherwise by the tensor pipe."""
    if not kernels:
        return None
    stage = max(kernels, key=lambda n: kernels[n]["us"])
    t = kernels[stage]["us"] * 1e-6
    a = alg[stage]
    hbm = float(peaks["hbm_gbs"])
    tensor = float(peaks["bf16_tflops"]) * (2.0 if s.fp8 else 1.0)
    tensor_kind = "bf16 burst (cuBLAS 8192^3)" + (" x 2, the nominal e4m3 / bf16 dense ratio" if s.fp8 else "")
    if "flops" in a and a["flops"] / a["bytes"] >= tensor * 1e12 / (hbm * 1e9):
        achieved, peak, unit, bound, kind = a["flops"] / t / 1e12, tensor, "TFLOP/s", "tensor", tensor_kind
    else:
        achieved, peak, unit, bound, kind = a["bytes"] / t / 1e9, hbm, "GB/s", "hbm", "HBM copy bandwidth"
    return {"bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4),
            "traffic": traffic_from_profile(s.name, stage, kernel_source_hash(stage)),
            "kernel": STAGE_NAMES[stage], "algorithmic": a, "peak_kind": f"{peak_kind} {kind}"}


class HostExperts:
    """[e] -> host fp64 copy of expert e of a stacked device weight tensor.

    With cache=True the copies are kept (staged once, outside the timed
    oracle calls); with cache=False every access converts afresh, so host
    memory holds one expert at a time (the fine-grained layers' 257 experts
    would take ~90 GB as fp64) and the conversion counts as oracle time."""

    def __init__(self, t, cache=True):
        self.t, self.cache, self.keep = t, {}, cache

    def __getitem__(self, e):
        import oracle
        e = int(e)
        if not self.keep:
            return oracle.as_f64(self.t[e])
        if e not in self.cache:
            self.cache[e] = oracle.as_f64(self.t[e])
        return self.cache[e]

    def stage(self, experts):
        if self.keep:
            for e in experts:
                self[e]


HOST_CACHE_BYTES = 24 << 30  # fp64 expert copies the oracle legs may keep on the host


def oracle_batch_tokens(s) -> int:
    """Tokens per oracle batch: the CPU-baseline leg and the reference arm use the same batches."""
    return min(s.T, 512)


class OracleRunner:
    """The fp64 oracle forward (routing, the selected experts, shared expert) on
    seeded random token batches of the workload, timed on the host's cores."""

    def __init__(self, s, inp, seed=7):
        import oracle
        self.oracle, self.s, self.inp = oracle, s, inp
        expert_bytes = s.E * 3 * s.inter * s.d * 8
        self.cached = expert_bytes <= HOST_CACHE_BYTES
        self.W1 = HostExperts(inp["W1"], cache=self.cached)
        self.W2 = HostExperts(inp["W2"], cache=self.cached)
        self.W1s = oracle.as_f64(inp["W1s"]) if inp["W1s"] is not None else None
        self.W2s = oracle.as_f64(inp["W2s"]) if inp["W2s"] is not None else None
        self.rng = np.random.default_rng(seed)
        self.batch = oracle_batch_tokens(s)

    def step(self) -> float:
        """One batch; returns the seconds spent in the oracle call itself."""
        s, o = self.s, self.oracle
        toks = np.sort(self.rng.choice(s.T, size=self.batch, replace=False))
        xs = self.inp["x"][toks]
        if self.cached:  # staging the weights is input preparation, not oracle work
            need = np.unique(o.route(xs, self.inp["W_r"], self.inp["bias"], s.k)["idx"])
            self.W1.stage(need)
            self.W2.stage(need)
        kw = dict(pow2=s.mx) if s.fp8 else {}
        fwd = o.moe_forward_fp8 if s.fp8 else o.moe_forward
        t0 = time.perf_counter()
        fwd(xs, self.inp["W_r"], self.inp["bias"], self.W1, self.W2, self.W1s, self.W2s, k=s.k,
            renormalize=s.renormalize, **kw)
        return time.perf_counter() - t0

    def describe(self, batches, spent) -> str:
        how = ("expert weights staged to host fp64 outside the timed calls" if self.cached else
               "expert weights converted to fp64 inside the timed calls, one expert at a time")
        return (f"fp64 numpy oracle forward (routing, selected experts, shared) on {batches} batch(es) of "
                f"{self.batch} random tokens of {self.s.T}, {spent:.1f} s; {how}")


def blas_threads() -> int:
    from threadpoolctl import threadpool_info
    return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])


def cpu_baseline(s, inp, budget_s=12.0):
    """The oracle on the reference arm's token batches until ~budget_s of CPU time; tokens/s."""
    r = OracleRunner(s, inp)
    batches, spent = 0, 0.0
    while spent < budget_s and batches < 64:
        spent += r.step()
        batches += 1
    return {"value": round(batches * r.batch / spent, 3), "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle", "sample": r.describe(batches, spent), **host_cpu()}


# --------------------------------------------------------------------------- one workload
def prepare(gg, s, dev, seed):
    """Device inputs, weights (quantised for FP8 layers, outside any timing), outputs, workspace."""
    inp = make_inputs(s, seed=seed, device=dev)
    cfg = make_cfg(gg, s)
    ws = torch.empty(gg.workspace_size(cfg) + gg.host_staging_size(cfg), dtype=torch.uint8, device=dev)
    if s.fp8:  # weights quantised once per 128x128 block (offline, outside the timed region)
        quant = gg.quantize_weights_mx if s.mx else gg.quantize_weights_fp8
        W1q, W1sc = quant(inp["W1"])
        W2q, W2sc = quant(inp["W2"])
        weights = gg.ExpertWeights(W1=W1q, W2=W2q, W1_scales=W1sc, W2_scales=W2sc)
        if s.shared_inter:
            weights.W1s, weights.W1s_scales = quant(inp["W1s"])
            weights.W2s, weights.W2s_scales = quant(inp["W2s"])
    else:
        weights = gg.ExpertWeights(W1=inp["W1"], W2=inp["W2"], W1s=inp["W1s"], W2s=inp["W2s"])
    out = torch.empty((s.T, s.d), dtype=torch.bfloat16 if s.x_dtype != "f32" else torch.float32, device=dev)
    counts = torch.empty(s.E, dtype=torch.int32, device=dev)
    return inp, cfg, ws, weights, out, counts


def measure_layer(gg, s, steps, warmup, world, dev, flush, seed, graph=True, e2e=True):
    """Times one workload's forward: the headline steps, the CUDA-graph replay,
    the host-buffer entry point and the per-kernel breakdown."""
    stream = torch.cuda.current_stream()
    inp, cfg, ws, weights, out, counts = prepare(gg, s, dev, seed)

    def step():
        gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], weights, out=out, counts_out=counts, ws=ws)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        times = time_steps(step, steps, warmup, flush, stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    status = gg.read_device_status(ws)
    if status != 0:
        raise RuntimeError(f"{s.name}: device status {status}")
    r = dict(ms=max_over_ranks(float(np.mean(times)), world, dev), clocks=clk.summary())

    # the per-kernel breakdown right after the headline steps (same clock and
    # thermal state; the two-stream e2e phase below loads the GPU harder)
    with ClockSampler(dev) as kclk:
        kt = time_marked(gg, cfg, inp, weights, out, counts, ws, max(3, steps // 2), flush, stream)
    c = counts.cpu().numpy()
    alg = algorithmic(s, c)
    kern = {}
    for name, t_ms in kt.items():
        a = alg[name]
        e = {"us": round(t_ms * 1e3, 2)}
        if "flops" in a:
            e["tflops"] = round(a["flops"] / (t_ms * 1e-3) / 1e12, 1)
        e["gbs"] = round(a["bytes"] / (t_ms * 1e-3) / 1e9, 1)
        kern[name] = e
    iso = time_isolated(gg, s, inp, alg, dev, flush, stream)
    for name, e in iso.items():
        kern[name]["isolated"] = e
    r["kernels_clocks"] = kclk.summary()

    if graph:  # the same forward replayed from a CUDA graph (one launch of the whole layer)
        gstream = torch.cuda.Stream()
        gstream.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gstream):
            step()  # warm the capture stream
            with torch.cuda.graph(g, stream=gstream):
                step()
        stream.wait_stream(gstream)
        torch.cuda.synchronize()
        gt = time_steps(g.replay, max(3, steps // 2), 3, flush, stream)
        r["graph_ms"] = max_over_ranks(float(np.mean(gt)), world, dev)
        del g

    if e2e:  # host buffers through moe_forward_host, copies inside the timed region
        xh = [inp["x"].cpu().pin_memory() for _ in range(2)]
        oh = [torch.empty((s.T, s.d), dtype=out.dtype).pin_memory() for _ in range(2)]

        def step_host():
            gg.moe_forward_host(cfg, xh[0], inp["W_r"], inp["bias"], weights, oh[0], ws)

        # one step at a time on one stream, L2 flushed between steps
        et = time_steps(step_host, max(3, steps // 2), 2, flush, stream, hold=False)
        r["e2e_serial_ms"] = max_over_ranks(float(np.mean(et)), world, dev)
        # consecutive steps on two streams, each with its own workspace and pinned
        # buffers: one step's host copies overlap the other's kernels
        wss = [ws, torch.empty_like(ws)]
        sts = [torch.cuda.Stream(), torch.cuda.Stream()]

        def run(n):
            for i in range(n):
                j = i % 2
                gg.moe_forward_host(cfg, xh[j], inp["W_r"], inp["bias"], weights, oh[j], wss[j], stream=sts[j])

        for st in sts:
            st.wait_stream(stream)
        run(4)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for st in sts:
            st.wait_stream(stream)
        run(steps)
        for st in sts:
            stream.wait_stream(st)
        b.record(stream)
        torch.cuda.synchronize()
        r["e2e_ms"] = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
        if gg.read_device_status(wss[1]) != 0:
            raise RuntimeError(f"{s.name}: device status in the second workspace")
        del wss, sts
        r["h2d"] = xh[0].numel() * xh[0].element_size()
        r["d2h"] = oh[0].numel() * oh[0].element_size()

    r.update(kernels=kern, counts=c, alg=alg, inp=inp)
    return r


def layer_report(s, r, peaks, peak_kind, world):
    """The per-workload part of the JSON line."""
    T = s.T
    roof = roofline(s, r["alg"], r["kernels"], peaks, peak_kind)
    gemm_us = r["kernels"]["up_gemm"]["us"] + r["kernels"]["down_gemm"]["us"]
    gemm_tf = s.gemm_flops() / (gemm_us * 1e-6) / 1e12
    tensor_peak = float(peaks["bf16_tflops"]) * (2.0 if s.fp8 else 1.0)
    c = r["counts"]
    hbm = float(peaks["hbm_gbs"])
    for e in r["kernels"].values():
        if "isolated" in e:
            e["isolated"]["frac_of_hbm"] = round(e["isolated"]["gbs"] / hbm, 4)
    rep = {"workload": workload_desc(s), "tokens_per_step": T,
           "dtype": ("mx-e4m3" if s.mx else "e4m3") if s.fp8 else "bf16",
           "ms_per_step": round(r["ms"], 4), "value": round(job_tokens_per_s(T, world, r["ms"]), 1),
           "unit": "tokens/s",
           # grouped-GEMM FLOP over the two GEMM kernels' own time, against the dense tensor peak
           "gemm_tflops": round(gemm_tf, 1), "gemm_frac_of_peak": round(gemm_tf / tensor_peak, 4),
           "roofline": roof, "kernels": r["kernels"], "clocks": r["clocks"], "kernels_clocks": r["kernels_clocks"],
           "expert_counts": {"min": int(c.min()), "max": int(c.max()), "mean": float(c.mean()),
                             "zeros": int((c == 0).sum())}}
    if "graph_ms" in r:
        rep["graph"] = {"ms_per_step": round(r["graph_ms"], 4),
                        "value": round(job_tokens_per_s(T, world, r["graph_ms"]), 1), "unit": "tokens/s",
                        "note": "the same forward captured once in a CUDA graph and replayed"}
    if "e2e_ms" in r:
        rep["e2e"] = {"value": round(job_tokens_per_s(T, world, r["e2e_ms"]), 1), "unit": "tokens/s",
                      "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                      "ms_per_step": round(r["e2e_ms"], 4), "note": E2E_NOTE,
                      "serial": {"value": round(job_tokens_per_s(T, world, r["e2e_serial_ms"]), 1),
                                 "unit": "tokens/s", "ms_per_step": round(r["e2e_serial_ms"], 4),
                                 "note": "one step at a time on one stream, L2 flushed between steps"}}
    return rep


SIDE_WORKLOADS = ("fine", "fine_skew", "fine_fp8", "fine_fp8_skew", "fine_mx", "fine_mx_skew", "fine_gather",
                  "decode", "tiny")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="mixtral", choices=sorted(CONFIGS) + ["router_micro"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workloads", default="auto",
                    help="'auto' (the other layers and the router microbenchmark, with the default "
                         "config at N=1), 'none', or a comma list of workload names")
    ap.add_argument("--set", default="", help="shape overrides for profiling runs, e.g. E=32,T=512")
    args = ap.parse_args()
    args.overrides = {}
    for kv in filter(None, args.set.split(",")):
        key, val = kv.split("=")
        args.overrides[key.strip()] = int(val)
    if args.warmup < 3:
        log("warm-up raised to 3 steps")
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:  # the CPU reference arm runs on rank 0 only
            return 0
        if args.config == "router_micro":
            return run_router_micro_reference(args, world)
        return run_reference(args, shape_of(args.config, **args.overrides), world)

    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    gg = build_lib()
    torch.cuda.set_device(local)
    flush = Flusher(local)
    peaks, peak_kind = load_peaks()
    if args.config == "router_micro":
        m = measure_router_micro(gg, args.steps, args.warmup, world, rank, local, flush, args.overrides)
        result = router_micro_line(m, args, world, peaks, peak_kind)
    else:
        s = shape_of(args.config, **args.overrides)
        r = measure_layer(gg, s, args.steps, args.warmup, world, local, flush, seed=1234 + rank)
        rep = layer_report(s, r, peaks, peak_kind, world)
        result = {
            "metric": METRIC, "value": rep["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": rep["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": rep["dtype"],
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)", "config": config_block(s),
            "gemm_tflops": rep["gemm_tflops"], "gemm_frac_of_peak": rep["gemm_frac_of_peak"],
            "roofline": rep["roofline"], "kernels": rep["kernels"], "kernels_clocks": rep["kernels_clocks"],
            "e2e": rep["e2e"], "graph": rep["graph"],
            "gpu_launches": gg.forward_launches(make_cfg(gg, s)) * args.steps, "clocks": rep["clocks"],
            "expert_counts": rep["expert_counts"]}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(s, r["inp"])
        del r
        torch.cuda.empty_cache()
        names = []
        if args.workloads == "auto":
            if world == 1 and args.config == "mixtral" and not args.overrides:
                names = list(SIDE_WORKLOADS) + ["router_micro"]
        elif args.workloads != "none":
            names = [n for n in args.workloads.split(",") if n]
        side = {}
        for name in names:  # the other workloads, one after the other, each measured the same way
            if name == "router_micro":
                m = measure_router_micro(gg, args.steps, args.warmup, world, rank, local, flush, {})
                side[name] = router_micro_line(m, args, world, peaks, peak_kind, compact=True)
                continue
            ws_ = shape_of(name)
            rr = measure_layer(gg, ws_, args.steps, args.warmup, world, local, flush, seed=1234 + rank)
            side[name] = layer_report(ws_, rr, peaks, peak_kind, world)
            del rr
            torch.cuda.empty_cache()
        if side:
            result["workloads"] = side
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


# --------------------------------------------------------------------------- router microbenchmark
def router_micro_shape(overrides):
    return tuple(overrides.get(key, ROUTER_MICRO[key]) for key in ("N", "E", "k"))


ROUTER_MICRO_L2 = ("inputs larger than L2: each step reads its own copy of the logits, the copies together "
                   ">= 2x L2; the steps run back to back between one pair of events")


def router_micro_desc(N, E, k):
    return {"workload": f"router_micro: N={N} tokens, E={E} experts, top-{k}, fp16 logits ~ N(0,1)",
            "tokens_per_step": N, "seed": 1234, "l2": ROUTER_MICRO_L2}


def measure_router_micro(gg, steps, warmup, world, rank, dev, flush, overrides):
    """Softmax + top-k of N fp16 logits rows (moe_topk_logits), device-resident and host-buffered."""
    N, E, k = router_micro_shape(overrides)
    stream = torch.cuda.current_stream()
    logits = make_router_logits(N, E, seed=1234 + rank, device=dev)
    idx = torch.empty((N, k), dtype=torch.int32, device=dev)
    w = torch.empty((N, k), dtype=torch.float32, device=dev)

    copies = rotating_copies(logits, dev)  # the steps' inputs together exceed twice the L2 size

    def step_i(i):
        gg.topk_logits(copies[i % len(copies)], k, out_idx=idx, out_w=w)

    for i in range(warmup):
        step_i(i)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        # each bracket times exactly `steps` steps, one launch each on the next copy
        times = [time_back_to_back(step_i, steps, flush, stream) for _ in range(8)]
    ms = max_over_ranks(float(np.mean(times)), world, dev)
    del copies

    def step():
        gg.topk_logits(logits, k, out_idx=idx, out_w=w)

    lh = logits.cpu().pin_memory()
    ih = torch.empty((N, k), dtype=torch.int32).pin_memory()
    wh = torch.empty((N, k), dtype=torch.float32).pin_memory()

    def step_host():
        logits.copy_(lh, non_blocking=True)
        gg.topk_logits(logits, k, out_idx=idx, out_w=w)
        ih.copy_(idx, non_blocking=True)
        wh.copy_(w, non_blocking=True)

    e2e_ms = max_over_ranks(float(np.mean(time_steps(step_host, max(3, steps // 2), 2, flush, stream,
                                                     hold=False))), world, dev)
    return dict(N=N, E=E, k=k, ms=ms, e2e_ms=e2e_ms, clocks=clk.summary())


def router_micro_line(m, args, world, peaks, peak_kind, compact=False):
    N, E, k, ms = m["N"], m["E"], m["k"], m["ms"]
    bytes_per_step = N * E * 2 + N * k * 8
    achieved = bytes_per_step / (ms * 1e-3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "traffic": None,
            "kernel": "softmax + top-k of stored logits", "peak_kind": f"{peak_kind} HBM copy bandwidth",
            "algorithmic": {"bytes": bytes_per_step}}
    e2e = {"value": round(job_tokens_per_s(N, world, m["e2e_ms"]), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": N * E * 2, "d2h_bytes_per_step": N * k * 8}
    if compact:
        return {"workload": router_micro_desc(N, E, k)["workload"], "tokens_per_step": N, "dtype": "f16",
                "ms_per_step": round(ms, 5), "value": round(job_tokens_per_s(N, world, ms), 1),
                "unit": "tokens/s", "kernel_us": round(ms * 1e3, 2), "roofline": roof, "e2e": e2e,
                "clocks": m["clocks"]}
    return {"metric": METRIC, "value": round(job_tokens_per_s(N, world, ms), 1), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic", "config": router_micro_desc(N, E, k), "roofline": roof,
            "kernel_us": round(ms * 1e3, 2), "e2e": e2e, "gpu_launches": args.steps, "clocks": m["clocks"]}


def run_router_micro_reference(args, world):
    """The oracle's softmax + top-k on bounded row samples of the microbenchmark's logits."""
    import oracle
    N, E, k = router_micro_shape(args.overrides)
    logits = make_router_logits(N, E, seed=1234, device="cpu")
    lf = oracle.as_f64(logits)
    per_step = min(N, 4096)
    rng = np.random.default_rng(3)

    def step():
        rows = rng.choice(N, size=per_step, replace=False)
        oracle.gate_weights(oracle.softmax(lf[rows]), oracle.topk_select(lf[rows], k))

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = args.steps * per_step / dt
    print(json.dumps({"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "tokens/s",
                      "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                      "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
                      "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                      "config": router_micro_desc(N, E, k),
                      "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": blas_threads(),
                                       "kind": "oracle", "sample": f"{per_step} random rows of {N} per step",
                                       **host_cpu()},
                      "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                              "d2h_bytes_per_step": 0}}), flush=True)
    return 0


def run_reference(args, s, world):
    """The oracle (fp64, host cores) as the slow reference arm: each step is one
    of the cpu_baseline leg's token batches of the same workload."""
    inp = make_inputs(s, seed=1234, device="cuda" if torch.cuda.is_available() else "cpu")
    r = OracleRunner(s, inp)
    for _ in range(args.warmup):
        r.step()
    spent = sum(r.step() for _ in range(args.steps))
    value = args.steps * r.batch / spent
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(spent / args.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_block(s),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": r.describe(args.steps, spent), **host_cpu()},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
