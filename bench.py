"""Benchmark of the fused attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one forward over the workload (default: B=4 H=12 N=8192 d=64 fp16
causal, the worked sizing of inskillml Module 9).  Rank 0 prints one JSON line.
Metric: TFLOPS = 4*B*H*N^2*d / t, halved for causal, over all ranks (each rank
runs an independent replica: the forward has no exchange step).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import threading
import time
from typing import Optional

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from exact_attention_sdpa_b200.workloads import (WORKLOADS, algorithmic_bytes, alibi_slopes,  # noqa: E402
                                                 attention_flops, exponential_count, make_inputs)

METRIC = "attention fwd TFLOPS (4BHN²d, /2 causal) and % of B200 dense BF16/FP16 peak"
UNIT = "TFLOPS"
KERNEL_SOURCES = ["exact_attention_sdpa_b200/csrc/attn_fwd_kernel.cuh", "exact_attention_sdpa_b200/csrc/sm100.cuh",
                  "exact_attention_sdpa_b200/csrc/attn_api.cu"]


def kernel_source_hash() -> str:
    """First 16 hex digits of the SHA-256 of the kernel sources; ncu traffic is reported only
    for the hash it was captured on."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    """(peaks, source): the measured HBM copy rate and bf16 GEMM rates of this machine's GPUs when
    MEASURED_PEAKS.json exists, else the earlier measurements used as fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, \
        "fallback"


def load_traffic(workload: str):
    """Per-launch DRAM bytes from a committed ncu capture, if taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(workload)
    if not e or e.get("kernel_source_sha") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a background thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.0005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: report no samples
            self.nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(n_gpus: int, backend: Optional[str] = None):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE).  The process group
    carries only the barrier and the max-over-ranks timing: replicas exchange no data.
    NCCL on GPUs; gloo where no GPU is present (the CPU tests of this host logic)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def dist_max(x: float, world: int) -> float:
    """The maximum of x over all ranks (the slowest replica sets the job time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """All ranks' work (each replica runs the full workload) over the slowest rank's time."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def barrier(world: int):
    """A process-group barrier when more than one rank runs (no-op for a single process)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_reference(w, steps: int, warmup: int, rows_per_step: int = 1024):
    """The fp64 oracle, as it stands, on a bounded sample of the workload:
    each step computes `rows_per_step` full output rows of one (b, h) head.
    Returns (TFLOPS over the sampled work, description, cores, mean ms per timed step)."""
    import numpy as np

    from oracle import sdpa_rows
    if w.lengths is not None:                          # ragged: the longest sequence as one problem
        from exact_attention_sdpa_b200.workloads import make_varlen_inputs
        vi = make_varlen_inputs(w)
        b0 = int(np.argmax(w.lengths))
        r0, n = int(vi["cu_seqlens"][b0]), w.lengths[b0]
        inp = {x: vi[x][r0:r0 + n].transpose(0, 1).unsqueeze(0) for x in "qkv"}
        inp.update(bias=None, gate=None)
        w = w.with_(B=1, N=n, lengths=None)
    else:
        inp = make_inputs(w)
    q, k, v = inp["q"], inp["k"], inp["v"]
    rng = np.random.default_rng(0)
    flops, secs = 0.0, 0.0
    for step in range(warmup + steps):
        b, h = int(rng.integers(w.B)), int(rng.integers(w.H))
        r0 = max(0, w.N - rows_per_step)              # the heaviest rows of a causal head
        picks = [(b, h, i) for i in range(r0, w.N)]
        t0 = time.perf_counter()
        sdpa_rows(q, k, v, picks, bias=inp["bias"], gate=inp["gate"], causal=w.causal, scale=w.scale,
                  softcap=w.softcap, alibi_slopes=alibi_slopes(w), window_left=w.window_left)
        dt = time.perf_counter() - t0
        if step >= warmup:
            secs += dt
            nk, off = w.n_keys, w.n_keys - w.N
            # visible keys of row i: up to i + off (causal) or all, from i + off - window (left window)
            vis = sum(max(0, (min(nk, i + off + 1) if w.causal else nk) -
                          (max(0, i + off - w.window_left) if w.window_left >= 0 else 0))
                      for (_, _, i) in picks)
            flops += 4.0 * w.d * vis
    cores = len(os.sched_getaffinity(0))
    sample = f"{rows_per_step} query rows (the last, i.e. heaviest) of one random (b,h) head per step, {steps} steps"
    return flops / secs / 1e12, sample, cores, 1e3 * secs / max(steps, 1)


def run_e2e(args, w, inp_cpu, out, lse, stream, world, flops, slopes=None):
    """The same metric through the host-buffer entry point (fwd -> attn_fwd_host, or
    attn_fwd_host_ex with the workload's score modifications; ALiBi slopes stay on the device): every
    step copies the step's inputs from pinned host memory to the device, runs the kernel,
    and copies O and lse back to pinned host memory.  Steps alternate between two streams
    with their own staging and host output buffers, so one step's copies run under the
    previous step's kernel; the timed region spans both streams."""
    from exact_attention_sdpa_b200 import Staging, fwd
    host = {k: (None if t is None else t.pin_memory()) for k, t in inp_cpu.items()}
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    d2h = out.numel() * out.element_size() + lse.numel() * 4
    streams = [stream, torch.cuda.Stream()]
    stagings = [Staging(host["q"], host["k"], host["v"], host["bias"], host["gate"]) for _ in streams]
    outs = [(torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
             torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)) for _ in streams]

    def e2e_step(i):
        s = i % 2
        fwd(host["q"], host["k"], host["v"], bias=host["bias"], gate=host["gate"], causal=w.causal, scale=w.scale,
            out=outs[s][0], lse=outs[s][1], staging=stagings[s], stream=streams[s], sync=False,
            softcap=w.softcap, alibi_slopes=slopes, window_left=w.window_left)

    steps = max(4, min(args.steps, 20))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1, e_side = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    e0.record(streams[0])
    streams[1].wait_event(e0)
    for i in range(steps):
        e2e_step(i)
    e_side.record(streams[1])
    streams[0].wait_event(e_side)
    e1.record(streams[0])
    torch.cuda.synchronize()
    ms = dist_max(e0.elapsed_time(e1) / steps, world)
    return {"value": whole_job_tflops(world, flops, ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "api": "fwd() -> attn_fwd_host%s (C ABI, pinned host buffers), 2 streams" % ("_ex" if has_mods(w) else "")}


def has_mods(w) -> bool:
    """Whether the workload carries score modifications (ALiBi, softcap, left window)."""
    return w.softcap > 0 or bool(w.alibi) or w.window_left >= 0


def launch_percentiles(ms):
    """p10 / median / p90 of per-launch device times (nearest-rank on the sorted list)."""
    xs = sorted(ms)
    if not xs:
        return {"p10": None, "p50": None, "p90": None}
    pick = lambda q: xs[min(len(xs) - 1, max(0, int(round(q * (len(xs) - 1)))))]
    return {"p10": pick(0.10), "p50": pick(0.50), "p90": pick(0.90)}


# NVIDIA's B200 datasheet dense (no 2:4 sparsity) FP16/BF16 tensor-core rate, TFLOP/s
DATASHEET_DENSE_TFLOPS = 2250.0


def mufu_exp_peak(sm_mhz: float) -> float:
    """Exponentials per second of the special-function units: 148 SMs x 16 per clock."""
    return 148 * 16 * sm_mhz * 1e6


def peak_fractions(value_per_gpu: float, measured_tflops: float) -> dict:
    """The metric's percentage against the datasheet dense peak, and against the measured GEMM rate."""
    return {"pct_of_peak": 100.0 * value_per_gpu / DATASHEET_DENSE_TFLOPS,
            "pct_of_peak_basis": f"datasheet dense FP16/BF16 {DATASHEET_DENSE_TFLOPS:.0f} TFLOP/s",
            "pct_of_measured_gemm": 100.0 * value_per_gpu / measured_tflops}


def exp_bound(w, mean_launch_ms: float, sm_mhz: float) -> dict:
    """The special-function-unit bound of a launch: its exponentials at 16 per SM per clock."""
    n = exponential_count(w)
    peak = mufu_exp_peak(sm_mhz)
    return {"exponentials_per_launch": n, "mufu_only_ms": 1e3 * n / peak,
            "achieved_gexp_s": n / (mean_launch_ms * 1e-3) / 1e9, "peak_gexp_s": peak / 1e9,
            "frac": (n / (mean_launch_ms * 1e-3)) / peak}


def run_bwd(args, w, config):
    """The backward on one GPU: K timed attn_bwd calls (three kernels each: D = rowsum(dO * O),
    dK/dV, dQ) after W warm-ups, inputs, O, lse and dO resident.  FLOPs: the usual 2.5x the
    forward's (five N x N x d products against two); the kernels recompute S and dP in both
    the dK/dV and the dQ kernel, seven products in all, on the tensor cores."""
    from exact_attention_sdpa_b200 import attn_bwd, attn_fwd, load_library
    from exact_attention_sdpa_b200.workloads import make_grad_output
    load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = {k: (None if t is None else t.to(dev)) for k, t in make_inputs(w).items()}
    assert inp["bias"] is None and inp["gate"] is None, "the backward takes no bias or gate"
    do = make_grad_output(w).to(dev)
    out, lse = attn_fwd(inp["q"], inp["k"], inp["v"], causal=w.causal, scale=w.scale)
    stream = torch.cuda.current_stream(dev)

    def step():
        attn_bwd(inp["q"], inp["k"], inp["v"], out, lse, do, causal=w.causal, scale=w.scale, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    flops = 2.5 * attention_flops(w)
    value = flops / (ms * 1e-3) / 1e12
    cs = clocks.summary()
    peaks, peak_src = load_peaks()
    peak = peaks["bf16_tflops"]
    line = {"metric": "attention bwd TFLOPS (2.5 x forward FLOPs)", "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1) inputs and dO)",
            "config": dict(config, **{"pass": "backward"}),
            **peak_fractions(value, peak),
            "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s", "frac": value / peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "traffic": None, "kernel": "bwd_prep_kernel + bwd_dkdv_kernel + bwd_dq_kernel",
                         "algorithmic_flops_per_launch": flops},
            "gpu_launches": 3 * steps, "e2e": None, "clocks": cs}
    print(json.dumps(line), flush=True)


def run_fp8(args, w, config):
    """The forward on e4m3 inputs (attn_fwd_fp8) on one GPU: K timed launches after W warm-ups,
    inputs (q, k and V transposed) resident.  FLOPs as the 16-bit forward's; the roofline is the
    measured bf16 GEMM rate times the nominal e4m3 / bf16 ratio of the tensor cores (2)."""
    from exact_attention_sdpa_b200 import load_library
    from exact_attention_sdpa_b200 import _native as nat
    from exact_attention_sdpa_b200.workloads import make_e4m3_inputs
    assert not (w.bias or w.gate or w.softcap > 0 or w.alibi or w.window_left >= 0 or w.lengths), \
        "the FP8 forward takes the plain problem only"
    lib = load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = make_e4m3_inputs(w)
    q, k = inp["q"].to(dev), inp["k"].to(dev)
    B, H, Nk, d = inp["v"].shape
    vbuf = torch.zeros(B, H, d, (Nk + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    vbuf[..., :Nk] = inp["v"].view(torch.uint8).transpose(-1, -2).to(dev)
    vt = vbuf[..., :Nk].view(torch.float8_e4m3fn)
    out = torch.empty(q.shape, device=dev, dtype=torch.float16)
    lse = torch.empty(q.shape[:-1], device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)
    views = [nat.make_view(t) for t in (q, k, vt, out)]
    refs = [ctypes.byref(x) for x in views]
    status = []

    def step():
        r = lib.attn_fwd_fp8(refs[0], refs[1], refs[2], float(inp["q_scale"]), float(inp["k_scale"]),
                             float(inp["v_scale"]), int(w.causal), float(w.scale), refs[3], lse.data_ptr(),
                             stream.cuda_stream)
        if r != 0:
            status.append(r)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if status:
        raise RuntimeError(f"attn_fwd_fp8 returned status {status[0]}")
    ms = t0.elapsed_time(t1) / args.steps
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    mean_launch_ms = statistics.mean(launch_ms)
    flops = attention_flops(w)
    value = flops / (ms * 1e-3) / 1e12
    achieved = flops / (mean_launch_ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    peak = 2.0 * peaks["bf16_tflops"]
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic (seeded N(0,1) inputs as e4m3 codes with power-of-two scales)",
            "config": dict(config, dtype="e4m3 in, fp16 out", v_layout="transposed [B, H, d, Nk]"),
            "pct_of_peak": 100.0 * value / (2.0 * DATASHEET_DENSE_TFLOPS),
            "pct_of_peak_basis": f"datasheet dense FP8 {2.0 * DATASHEET_DENSE_TFLOPS:.0f} TFLOP/s",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst) x 2 (nominal e4m3 / bf16 ratio)",
                         "traffic": None, "kernel": "attn_fwd_kernel (e4m3)", "mean_launch_ms": mean_launch_ms,
                         "launch_ms_percentiles": launch_percentiles(launch_ms),
                         "algorithmic_flops_per_launch": flops},
            "gpu_launches": args.steps, "e2e": None, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


def run_varlen(args, w, config):
    """A ragged batch on one GPU: K timed attn_fwd_varlen calls (one kernel launch per
    sequence) after W warm-ups, packed inputs resident; the oracle times one sequence."""
    from exact_attention_sdpa_b200 import attn_fwd_varlen, load_library
    from exact_attention_sdpa_b200.workloads import make_varlen_inputs
    load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = make_varlen_inputs(w)
    q, k, v = (inp[n].to(dev) for n in "qkv")
    cu = inp["cu_seqlens"]
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[1], q.shape[0], device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)

    def step():
        attn_fwd_varlen(q, k, v, cu, cu, causal=w.causal, scale=w.scale, out=out, lse=lse, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clocks:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    flops = attention_flops(w)
    value = flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    peak = peaks["bf16_tflops"]
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded N(0,1) packed inputs)", "config": dict(config, lengths=list(w.lengths)),
            **peak_fractions(value, peak),
            "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s", "frac": value / peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst)", "traffic": None,
                         "kernel": "attn_fwd_kernel (one launch per sequence)", "algorithmic_flops_per_launch": flops},
            "gpu_launches": args.steps * sum(1 for n in w.lengths if n > 0), "e2e": None, "clocks": clocks.summary()}
    if not args.no_cpu_baseline:
        import numpy as np
        from oracle import sdpa_rows
        b = int(np.argmax(w.lengths))                 # the longest sequence, its last 1024 rows
        r0, n = int(cu[b]), w.lengths[b]
        qs, ks, vs = (inp[x][r0:r0 + n].transpose(0, 1).unsqueeze(0) for x in "qkv")
        picks = [(0, h, i) for h in range(1) for i in range(max(0, n - 1024), n)]
        t = time.perf_counter()
        sdpa_rows(qs, ks, vs, picks, causal=w.causal, scale=w.scale)
        dt = time.perf_counter() - t
        vis = sum(i + 1 for (_, _, i) in picks)
        line["cpu_baseline"] = {"value": 4.0 * w.d * vis / dt / 1e12, "unit": UNIT,
                                "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
                                "sample": f"the last 1024 query rows of one head of the longest sequence ({n} tokens)"}
    print(json.dumps(line), flush=True)


def main():
    """Parse the contract's arguments and print one JSON line (see the module docstring)."""
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="n8192_causal", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-steps", type=int, default=8)
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-staged end-to-end leg (profiling runs)")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward (attn_bwd) on the workload instead of the forward")
    ap.add_argument("--fp8", action="store_true",
                    help="time the e4m3 forward (attn_fwd_fp8) on the workload's shape instead")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    flops = attention_flops(w)
    config = {"workload": w.name, "description": w.description, "B": w.B, "H": w.H, "N": w.N, "Nk": w.n_keys,
              "d": w.d,
              "causal": w.causal, "bias": w.bias, "gate": w.gate, "dtype": w.dtype,
              "softcap": w.softcap, "alibi": w.alibi, "window_left": w.window_left,
              "inputs_bytes": algorithmic_bytes(w),
              "l2": "no flush: inputs+outputs larger than the 126 MB L2" if algorithmic_bytes(w) > 126e6
              else "inputs fit in L2 (not the benchmarked workload)",
              "parallelism": f"replicas x{args.gpus}"}

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        val, sample, cores, ms = cpu_reference(w, args.steps, args.warmup)
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
                "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if args.bwd:
        return run_bwd(args, w, config)
    if args.fp8:
        return run_fp8(args, w, config)
    if w.lengths is not None:
        return run_varlen(args, w, config)
    world, rank, local = dist_setup(args.gpus)
    from exact_attention_sdpa_b200 import attn_fwd, load_library
    load_library()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp_cpu = make_inputs(w)
    inp = {k: (None if t is None else t.to(dev)) for k, t in inp_cpu.items()}
    out = torch.empty_like(inp["q"])
    lse = torch.empty(inp["q"].shape[:-1], device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)

    slopes = alibi_slopes(w)
    slopes = None if slopes is None else slopes.to(dev)
    # The timed steps call the C entry point directly with views built once: for kernels
    # of a few tens of microseconds the per-call Python marshalling would otherwise take
    # longer than the kernel and the device would idle between launches.  The first call
    # goes through the Python binding (which checks the status).
    attn_fwd(inp["q"], inp["k"], inp["v"], bias=inp["bias"], gate=inp["gate"], causal=w.causal,
             scale=w.scale, out=out, lse=lse, stream=stream, softcap=w.softcap, alibi_slopes=slopes,
             window_left=w.window_left)
    from exact_attention_sdpa_b200 import _native as nat
    lib = load_library()
    views = [nat.make_view(t) for t in (inp["q"], inp["k"], inp["v"], inp["bias"], inp["gate"], out)]
    refs = [None if x is None else ctypes.byref(x) for x in views]
    mods_on = has_mods(w)
    mods = nat.AttnMods(None if slopes is None else slopes.data_ptr(), float(w.softcap), int(w.window_left))
    args_c = (refs[0], refs[1], refs[2], refs[3], refs[4], int(w.causal), float(w.scale))
    tail_c = (refs[5], lse.data_ptr(), stream.cuda_stream)
    status = []

    def step():
        if mods_on:
            r = lib.attn_fwd_ex(*args_c, ctypes.byref(mods), *tail_c)
        else:
            r = lib.attn_fwd(*args_c, *tail_c)
        if r != 0:
            status.append(r)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if status:
        raise RuntimeError(f"attn_fwd returned status {status[0]}")

    # ---- device-timed region: K launches, per-launch events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    if status:
        raise RuntimeError(f"attn_fwd returned status {status[0]}")
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    # host time of one C-ABI call (argument checks, tensor-map encoding, launch), outside the
    # timed region: calls enqueued back to back, the device left to drain afterwards
    n_host = 50
    h0 = time.perf_counter()
    for _ in range(n_host):
        step()
    host_us = 1e6 * (time.perf_counter() - h0) / n_host
    torch.cuda.synchronize()
    ms_per_step = dist_max(total_ms / args.steps, world)
    mean_launch_ms = statistics.mean(launch_ms)
    value = whole_job_tflops(world, flops, ms_per_step)

    # ---- end to end through the public API: pinned host inputs in, host outputs back, every step
    e2e = None if args.no_e2e else run_e2e(args, w, inp_cpu, out, lse, stream, world, flops, slopes)

    peaks, peak_src = load_peaks()
    peak = peaks["bf16_tflops"]            # burst figure: the kernel is timed alone; fp16 dense rate = bf16's
    achieved = flops / (mean_launch_ms * 1e-3) / 1e12
    cs = clocks.summary()
    sm_max = cs["sm_max_mhz"] or peaks.get("sm_max_mhz", 1965.0)
    nbytes = algorithmic_bytes(w)
    hbm = {"achieved_gbs": nbytes / (mean_launch_ms * 1e-3) / 1e9, "peak_gbs": peaks["hbm_gbs"],
           "frac": nbytes / (mean_launch_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
           "algorithmic_bytes_per_launch": nbytes, "peak_source": f"{peak_src} hbm_gbs"}
    exps = exp_bound(w, mean_launch_ms, sm_max)
    if w.d <= 32 and exps["mufu_only_ms"] > 1e3 * flops / (peak * 1e12):
        # short, narrow heads (the gated Evoformer row attention): the exponentials on the
        # special-function units bind before the tensor cores (every exponential on MUFU here)
        roofline = {"bound": "alu", "achieved": exps["achieved_gexp_s"], "peak": exps["peak_gexp_s"],
                    "unit": "Gexp/s", "frac": exps["frac"],
                    "peak_source": "MUFU: 148 SMs x 16 exponentials per clock x max SM clock",
                    "tensor": {"achieved_tflops": achieved, "peak_tflops": peak, "frac": achieved / peak}}
    else:
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "peak_source": f"{peak_src} bf16_tflops (burst)"}
    roofline.update({"traffic": load_traffic(w.name), "kernel": "attn_fwd_kernel",
                     "mean_launch_ms": mean_launch_ms, "launch_ms_percentiles": launch_percentiles(launch_ms),
                     "algorithmic_flops_per_launch": flops, "hbm": hbm, "exp": exps})
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1) inputs)", "config": config,
            **peak_fractions(value / world, peak),
            "roofline": roofline,
            "gpu_launches": args.steps,
            "host_us_per_call": host_us,
            "e2e": e2e,
            "clocks": cs}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, sample, cores, _ = cpu_reference(w, args.cpu_steps, 1)
        line["cpu_baseline"] = {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
