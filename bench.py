"""Benchmark of the sparse MoE FFN layer forward on B200 (sm_100a).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one moe_forward over a batch of T tokens of the named workload
(default: the Hy4-shape prefill layer, T=4096, H=6144, E=256 top-8 + 1 shared,
I=2048, bf16) with inputs resident in HBM.  Under torchrun each rank runs the
same layer on its own batch (data-parallel replicas, no collective on the data
path: weak scaling); the reported time is the max over ranks.

Printed (rank 0, one JSON line): tokens/s, the layer's roofline fraction, the
dominant kernel's roofline record (CUDA-event duration inside the timed
region), an end-to-end figure through host buffers, SM clocks sampled during
the timed region, our kernel launch count and the CPU oracle baseline.
``--impl reference`` times the CPU oracle instead (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_moe_layer_06_b200.workloads import CONFIGS, make_inputs, make_x, sample_tokens  # noqa

METRIC = "MoE-layer tokens/s and % of roofline (TFLOP/s or HBM GB/s) on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the expert GEMM kernels and their launch configuration (template arguments)
GEMM_SOURCES = ["sparse_moe_layer_06_b200/csrc/gemm_sm100.cuh",
                "sparse_moe_layer_06_b200/csrc/ptx.cuh",
                "sparse_moe_layer_06_b200/csrc/moe_api.cu"]


# ------------------------------------------------------------------ helpers

def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def layer_counts(cfg, idx_cpu, fp8=False):
    """Algorithmic FLOPs and bytes of one layer forward, from the actual routing
    (FP8: one byte per expert weight plus its fp32 channel scales)."""
    T, H, E, I, k, S = cfg.T, cfg.H, cfg.E, cfg.I, cfg.top_k, cfg.num_shared
    b = 2 if cfg.dtype == torch.bfloat16 else 4
    touched = int((torch.bincount(idx_cpu.reshape(-1).long(), minlength=E) > 0).sum())
    flops = T * (2 * H * E + (k + S) * 6 * H * I)
    wbytes = (touched + S) * ((3 * I * H) + (2 * I + H) * 4) if fp8 else \
        (touched + S) * 3 * I * H * b
    bytes_ = wbytes + E * H * b + 2 * T * H * b
    return flops, bytes_, touched


def gate_up_counts(cfg, touched, fp8=False):
    """Algorithmic FLOPs / bytes of one launch of the grouped gate/up GEMM, on
    the layer roofline's definition: the gate and up weights of every touched
    expert (+ the shared expert) and the token rows x, each read once (FP8:
    one byte per weight plus its fp32 row scales).  The permuted token copy and
    h are implementation traffic and are not credited."""
    T, H, I, k, S = cfg.T, cfg.H, cfg.I, cfg.top_k, cfg.num_shared
    rows = T * (k + S)
    flops = 2 * 2 * rows * H * I
    b = 2 if cfg.dtype == torch.bfloat16 else 4
    if fp8:
        bytes_ = (touched + S) * (2 * I * H + 2 * I * 4) + T * H * b
    else:
        bytes_ = (touched + S) * 2 * I * H * b + T * H * b
    return flops, bytes_


def down_counts(cfg, touched, scatter_add=False, fp8=False):
    """One launch of the grouped down GEMM, on the layer roofline's definition:
    the down weights of every touched expert (+ shared) read once and the
    layer output written once (FP8: one byte per weight plus its fp32 column
    scales).  h, the weighted rows and the fp32 accumulator are implementation
    traffic and are not credited."""
    T, H, I, k, S = cfg.T, cfg.H, cfg.I, cfg.top_k, cfg.num_shared
    rows = T * (k + S)
    flops = 2 * rows * H * I
    b = 2 if cfg.dtype == torch.bfloat16 else 4
    if fp8:
        bytes_ = (touched + S) * (I * H + H * 4) + T * H * b
    else:
        bytes_ = (touched + S) * I * H * b + T * H * b
    return flops, bytes_


def kernel_roofline(name, cfg, touched, fp8, ms_per_launch, hbm_peak, tf_peak):
    """Roofline record of one expert-GEMM launch: algorithmic work on the layer
    roofline's definition divided by its CUDA-event duration."""
    if name == "expert_down_combine_gemm":
        kf, kb = down_counts(cfg, touched, scatter_add=True)
    elif name in ("expert_down_gemm", "expert_down_gemm_fp8"):
        kf, kb = down_counts(cfg, touched, fp8=fp8)
    else:
        kf, kb = gate_up_counts(cfg, touched, fp8)
    t = ms_per_launch / 1e3
    if kb / (hbm_peak * 1e9) >= kf / (tf_peak * 1e12):
        r = {"bound": "hbm", "achieved": kb / t / 1e9, "peak": hbm_peak, "unit": "GB/s"}
    else:
        r = {"bound": "tensor", "achieved": kf / t / 1e12, "peak": tf_peak, "unit": "TFLOP/s"}
    r["frac"] = r["achieved"] / r["peak"]
    r["kernel"] = name
    r["ms_per_launch"] = ms_per_launch
    r["algorithmic"] = {"bytes": kb, "flops": kf}
    return r


def source_hash():
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture of this kernel
    (profiles/ncu_traffic.txt); None if absent or the kernel source changed."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    want = source_hash()
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("kernel") == kernel and f.get("workload") == workload and \
                f.get("source_hash") == want:
            return int(float(f["bytes_per_launch"]))
    return None


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of the GPU, sampled
    during the timed region.  Polls NVML every 10 ms from a thread (so even a
    timed region of a few tens of milliseconds gets samples); without NVML it
    falls back to `nvidia-smi -lms 50`.  summary() keeps only the samples
    taken inside a given wall-clock window.  Nothing here changes a setting."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    PERIOD_S = 0.010

    def __init__(self, gpu_index: int, device=None):
        self.gpu = gpu_index
        self.device = device
        self.proc = None
        self.samples = []  # (wall time, sm MHz, sm max MHz, power W, [reason names])
        self.thread = None
        self.stop_flag = threading.Event()
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.device is not None:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            for cand in (uuid, "GPU-" + uuid):
                try:
                    return pynvml, pynvml.nvmlDeviceGetHandleByUUID(cand)
                except pynvml.NVMLError:
                    pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:  # no NVML binding or device: use nvidia-smi
            return self._start_smi()
        self.source = "nvml, 10 ms"

        def poll():
            while not self.stop_flag.is_set():
                try:
                    sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((time.time(), sm, smax, pw,
                                         [k for k, b in bits.items() if r & b]))
                except Exception:
                    pass
                self.stop_flag.wait(self.PERIOD_S)
        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        return self

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.source = "nvidia-smi, 50 ms"

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        def read():
            for line in self.proc.stdout:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[0] == str(self.gpu):
                    reasons = [self.REASONS[i] for i in range(4)
                               if parts[5 + i].lower() in ("active", "1")]
                    self.samples.append((time.time(), num(parts[1]), num(parts[2]),
                                         num(parts[3]), reasons))
        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()
        return self

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        mine = [r for r in self.samples if t0 <= r[0] <= t1]
        if not mine:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples in window"],
                    "samples": 0, "source": self.source}
        sm = [r[1] for r in mine if r[1] is not None]
        smax = [r[2] for r in mine if r[2] is not None]
        pw = [r[3] for r in mine if r[3] is not None]
        reasons = sorted({x for r in mine for x in r[4]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(pw) if pw else None,
                "reasons": reasons, "samples": len(mine), "source": self.source}


# ------------------------------------------------------------------ ranks

def rank_token_seed(rank: int) -> int:
    """Seed of a rank's token batch: every rank holds the same weights (seeds
    1..3 of the workload recipe) and its own tokens."""
    return 1000 * rank


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The slowest rank's time: an all-reduce MAX over the process group (NCCL
    on GPUs, gloo on CPU), or the value itself on a single process."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, seconds: float) -> float:
    """Units all ranks processed divided by the (max over ranks) time."""
    return world * units_per_rank / seconds


# ------------------------------------------------------------------ CPU oracle baseline

def oracle_baseline(cfg, cpu_inp, budget_s=12.0, max_tokens=2048):
    """Time the CPU oracle (as it stands) on a seeded token sample of the same
    workload: batches of tokens until ~budget_s of work.  Returns a dict."""
    import oracle
    order = sample_tokens(cfg.T, min(cfg.T, max_tokens), seed=1)
    done = 0
    t0 = time.perf_counter()
    batch = max(1, oracle.num_threads())
    while done < len(order):
        toks = order[done:done + batch]
        oracle.forward(cpu_inp["x"], cpu_inp["gate_w"], cpu_inp["expert_w"], cpu_inp["shared_w"],
                       cfg.top_k, cfg.routed_scale, cfg.clip_limit,
                       logit_bias=cpu_inp["logit_bias"], tokens=toks)
        done += len(toks)
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{done} seeded tokens of the {cfg.name} batch (T={cfg.T}), "
                      f"full layer per token, fp64, {dt:.1f} s"}


def cpu_inputs(inp):
    return {k: (v.detach().cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


# ------------------------------------------------------------------ reference arm

def run_reference(args, cfg, rank, world):
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    torch.manual_seed(0)
    inp = make_inputs(cfg, seed=0, device="cpu") if cfg.T * cfg.H * cfg.E < 1 << 33 else None
    if inp is None:
        inp = cpu_inputs(make_inputs(cfg, seed=0, device="cuda"))
        torch.cuda.empty_cache()
    order = sample_tokens(cfg.T, cfg.T, seed=1)
    # calibrate tokens per step so that warmup+steps fit in ~150 s
    t0 = time.perf_counter()
    oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], inp["shared_w"], cfg.top_k,
                   cfg.routed_scale, cfg.clip_limit, logit_bias=inp["logit_bias"],
                   tokens=order[:1])
    per_tok = max(1e-6, time.perf_counter() - t0)
    n_steps = args.steps + args.warmup
    per_step = max(1, min(cfg.T, int(150.0 / n_steps / per_tok * max(1, oracle.num_threads()))))
    times = []
    cursor = 0
    for s in range(n_steps):
        toks = [order[(cursor + i) % cfg.T] for i in range(per_step)]
        cursor += per_step
        t0 = time.perf_counter()
        oracle.forward(inp["x"], inp["gate_w"], inp["expert_w"], inp["shared_w"], cfg.top_k,
                       cfg.routed_scale, cfg.clip_limit, logit_bias=inp["logit_bias"],
                       tokens=toks)
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = per_step * len(times) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "top_k": cfg.top_k,
                   "I": cfg.I, "num_shared": cfg.num_shared, "tokens_per_step": per_step},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{per_step} seeded tokens of the {cfg.name} batch per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ router statistics

def run_router_stats(args, cfg, local, world):
    """Time moe_router_stats (routing probabilities, selection shares, aux loss,
    EMA counts) over the workload's T tokens; one rank (an auxiliary line)."""
    from sparse_moe_layer_06_b200 import moe
    from sparse_moe_layer_06_b200.workloads import make_router_inputs
    if world != 1:
        raise SystemExit("--op router_stats runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    inp = make_router_inputs(cfg, seed=0, device=dev)
    p = moe.MoEProblem.from_config(cfg)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_ROUTER_STATS, device=dev)
    P = torch.empty(cfg.E, dtype=torch.float32, device=dev)
    f = torch.empty(cfg.E, dtype=torch.float32, device=dev)
    aux = torch.empty(1, dtype=torch.float32, device=dev)
    ema = torch.zeros(cfg.E, dtype=torch.float32, device=dev)
    ema_total = torch.zeros(1, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        moe.moe_router_stats(p, inp["x"], inp["gate_w"], inp["logit_bias"], P, f, aux, ema,
                             ema_total, 0.9, ws, stream)

    clocks = ClockSampler(0, dev).start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    moe.moe_profile_start(args.steps * 8 + 64)
    torch.cuda.synchronize(dev)
    launches0 = moe.moe_launch_count()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    ev1.synchronize()
    wall1 = time.time()
    launches = moe.moe_launch_count() - launches0
    kernel_times = moe.moe_profile_stop()
    clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    status = moe.moe_read_device_status(ws)
    peaks, peak_kind = read_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    b = 2 if cfg.dtype == torch.bfloat16 else 4
    bytes_ = cfg.T * cfg.H * b + cfg.E * cfg.H * b + cfg.T * cfg.E * 4
    flops = 2 * cfg.T * cfg.H * cfg.E
    dominant = max(kernel_times, key=lambda k: kernel_times[k][1])
    dom_ms = kernel_times[dominant][1] / max(1, kernel_times[dominant][0])
    line = {
        "metric": "router statistics tokens/s (moe_router_stats) on 1 B200",
        "value": cfg.T / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.006) router weights; random init)",
        "config": {"workload": f"{cfg.name}_router_stats", "T": cfg.T, "H": cfg.H, "E": cfg.E,
                   "top_k": cfg.top_k,
                   "l2": (f"x is {cfg.T * cfg.H * b / 1e6:.0f} MB, "
                          + ("larger than L2 (126 MB): streamed each step" if cfg.T * cfg.H * b > 126e6
                             else "smaller than L2 (126 MB): not a DRAM-bound measurement"))},
        "roofline": {"bound": "hbm", "achieved": bytes_ / (ms / 1e3) / 1e9, "peak": hbm_peak,
                     "unit": "GB/s", "frac": bytes_ / (ms / 1e3) / 1e9 / hbm_peak,
                     "traffic": None, "kernel": "whole call",
                     "algorithmic": {"bytes": bytes_, "flops": flops},
                     "peak_source": peak_kind},
        "kernels": {k: {"launches": v[0], "ms_per_launch": v[1] / max(1, v[0])}
                    for k, v in kernel_times.items()},
        "dominant_kernel_ms": dom_ms,
        "cpu_baseline": None,
        "clocks": clocks.summary(wall1 - ms * args.steps / 1e3, wall1),
        "e2e": None,
        "gpu_launches": launches,
        "device_status": status,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def time_steps(step, n, stream, dist=None, device=None):
    """Device time of n back-to-back steps (CUDA events on the launching
    stream, synchronised on both sides, max over ranks), in ms per step."""
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(n):
        step()
    ev1.record(stream)
    ev1.synchronize()
    return max_over_ranks(ev0.elapsed_time(ev1), dist, device) / n


def cool_down(seconds):
    """Let the GPU idle before the next pass, so that every pass starts from
    the same state: a pass that follows seconds of full load would otherwise
    run at the lower clock the 1 kW power limiter sets by then."""
    time.sleep(max(0.5, seconds))


def kernel_times(moe, step, n, device=None):
    """Per-kernel CUDA-event durations over n steps (the library records an
    event pair around each launch on its stream).  Those events also keep
    consecutive launches from overlapping, so this runs as its own pass after
    the timed region; returns {name: (launches, total ms)}."""
    torch.cuda.synchronize(device)
    moe.moe_profile_start(n * 16 + 64)
    for _ in range(n):
        step()
    torch.cuda.synchronize(device)
    return moe.moe_profile_stop()


def measure_workload(moe, cfg, inp, x, dev, stream, steps, warmup, fp8_weights=None):
    """Time one workload on weights already resident (a sub-record of the bench
    line): ms/step, tokens/s, layer roofline fraction and the dominant
    kernel's roofline record."""
    p = moe.MoEProblem.from_config(cfg)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD, device=dev)
    out = torch.empty(cfg.T, cfg.H, dtype=cfg.dtype, device=dev)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=dev)
    bias = inp["logit_bias"]

    def step():
        moe.moe_forward(p, x, inp["gate_w"], bias, inp["expert_w"], inp["shared_w"], out, idx, w,
                        ws, stream)
    for _ in range(warmup):
        step()
    cool_down(1.0)
    ms = time_steps(step, steps, stream, None, dev)
    cool_down(2 * ms * steps / 1e3)
    kt = kernel_times(moe, step, steps, dev)
    status = moe.moe_read_device_status(ws)
    peaks, _ = read_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    tf_peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    idx_cpu = idx.cpu()
    flops, bytes_, touched = layer_counts(cfg, idx_cpu)
    t_s = ms / 1e3
    roof_t = max(flops / (tf_peak * 1e12), bytes_ / (hbm_peak * 1e9))
    dom = max(kt, key=lambda k: kt[k][1])
    rec = {"workload": cfg.name, "T": cfg.T, "ms_per_step": ms, "tokens_per_s": cfg.T / t_s,
           "tflops": flops / t_s / 1e12, "layer_roofline_frac": roof_t / t_s,
           "layer_bound": "tensor" if flops / (tf_peak * 1e12) > bytes_ / (hbm_peak * 1e9)
           else "hbm",
           "touched_experts": touched,
           "dominant": kernel_roofline(dom, cfg, touched, False, kt[dom][1] / max(1, kt[dom][0]),
                                       hbm_peak, tf_peak),
           "kernels": {k: v[1] / max(1, v[0]) for k, v in kt.items()},
           "device_status": status}
    counts = torch.bincount(idx_cpu.reshape(-1).long(), minlength=cfg.E).float()
    rec["max_expert_share"] = float(counts.max() / cfg.T)
    del ws, out, idx, w
    torch.cuda.empty_cache()
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=600)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="hy4_prefill", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the decode / skewed sub-records of a Hy4 line")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="steps of the end-to-end measurement (default: --steps, so that "
                         "both run equally long under the power cap)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T of the workload (smaller cases for profiling)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E of the workload (smaller cases for profiling)")
    ap.add_argument("--op", default="forward", choices=["forward", "router_stats"],
                    help="router_stats: time moe_router_stats (the router's load-balancing "
                         "statistics) on the workload's tokens instead of the layer")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "fp8"],
                    help="expert weights as stored (fp8: E4M3 codes + power-of-two "
                         "channel scales, moe_forward_fp8)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.e2e_steps is None:
        args.e2e_steps = args.steps

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = CONFIGS[args.config]
    base_cfg = cfg
    if args.tokens is not None or args.experts is not None:
        from dataclasses import replace
        cfg = replace(cfg, T=args.tokens or cfg.T, E=args.experts or cfg.E,
                      name=f"{cfg.name}_T{args.tokens or cfg.T}_E{args.experts or cfg.E}")

    fp8 = args.weights == "fp8"
    if fp8:
        if cfg.dtype != torch.bfloat16:
            ap.error("--weights fp8 needs a bf16 workload")
        from dataclasses import replace
        cfg = replace(cfg, name=f"{cfg.name}_fp8")

    if args.impl == "reference":
        if fp8:
            ap.error("the reference arm times the fp64 oracle of the bf16 layer")
        return run_reference(args, cfg, rank, world)

    from sparse_moe_layer_06_b200 import moe
    if args.op == "router_stats":
        return run_router_stats(args, cfg, local, world)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    # identical weights on every rank, a different token batch per rank
    inp = make_inputs(cfg.with_tokens(1), seed=0, device=dev)
    inp["x"] = make_x(cfg, seed=rank_token_seed(rank), device=dev)
    if cfg.skew_bias:
        from sparse_moe_layer_06_b200.workloads import skew_logit_bias
        inp["logit_bias"] = skew_logit_bias(cfg.E).to(dev)
    p = moe.MoEProblem.from_config(cfg)
    ws = moe.alloc_workspace(p, moe.MOE_CALL_FORWARD_FP8 if fp8 else moe.MOE_CALL_FORWARD,
                             device=dev)
    out = torch.empty(cfg.T, cfg.H, dtype=cfg.dtype, device=dev)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    if fp8:
        # weights encoded once, outside the timed region (a load-time step)
        def quantize(wt):
            q = torch.empty(wt.shape, dtype=torch.uint8, device=dev)
            sg = torch.empty(wt.shape[0], 2, cfg.I, dtype=torch.float32, device=dev)
            sd = torch.empty(wt.shape[0], cfg.H, dtype=torch.float32, device=dev)
            moe.moe_quantize_weights_fp8(p, wt, q, sg, sd, stream)
            return q, sg, sd
        wq = quantize(inp["expert_w"])
        sq = quantize(inp["shared_w"].unsqueeze(0)) if inp["shared_w"] is not None else \
            (None, None, None)
        torch.cuda.synchronize(dev)
        del inp["expert_w"]
        torch.cuda.empty_cache()

    def forward(x_in, out_t, s):
        if fp8:
            moe.moe_forward_fp8(p, x_in, inp["gate_w"], inp["logit_bias"], *wq, *sq, out_t, idx,
                                w, ws, s)
        else:
            moe.moe_forward(p, x_in, inp["gate_w"], inp["logit_bias"], inp["expert_w"],
                            inp["shared_w"], out_t, idx, w, ws, s)

    def step():
        forward(inp["x"], out, stream)

    gpu_index = local if torch.cuda.device_count() > 1 else 0
    clocks = ClockSampler(gpu_index, dev).start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if moe.moe_read_device_status(ws) != 0:
        raise RuntimeError("device error word set during warm-up")

    # ---------------- timed region (device time, CUDA events, max over ranks)
    launches0 = moe.moe_launch_count()
    ms_per_step = time_steps(step, args.steps, stream, dist, dev)
    wall1 = time.time()
    launches = moe.moe_launch_count() - launches0
    clock_rec = clocks.summary(wall1 - ms_per_step * args.steps / 1e3, wall1)
    # per-kernel durations: the same number of steps again, with an event pair
    # around every launch (a separate pass: the events keep launches apart),
    # after an idle pause as long as the timed region ran, twice over
    cool_down(2 * ms_per_step * args.steps / 1e3)
    kt = kernel_times(moe, step, args.steps, dev)
    if dist:
        dist.barrier()
    status = moe.moe_read_device_status(ws)
    ms = ms_per_step * args.steps

    # ---------------- end to end: host buffers, copies inside the timed region.
    # Each step copies its tokens in from pinned host memory, runs the layer
    # and copies the output back.  As a serving loop would, steps are
    # pipelined over two device buffers and three streams (copy-in, compute,
    # copy-out) so the PCIe copies of one step overlap the layer of another.
    x_host = inp["x"].cpu().pin_memory()
    out_host = [torch.empty(cfg.T, cfg.H, dtype=cfg.dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(inp["x"]) for _ in range(2)]
    out_dev = [torch.empty_like(out) for _ in range(2)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    s_cmp = stream
    in_done = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        for i in range(n):
            b = i & 1
            if i >= 2:
                s_in.wait_event(cmp_done[b])  # the layer is done reading x_dev[b]
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host, non_blocking=True)
            in_done[b].record(s_in)
            s_cmp.wait_event(in_done[b])
            if i >= 2:
                s_cmp.wait_event(out_done[b])  # out_dev[b] was copied out
            forward(x_dev[b], out_dev[b], s_cmp)
            cmp_done[b].record(s_cmp)
            s_out.wait_event(cmp_done[b])
            with torch.cuda.stream(s_out):
                out_host[b].copy_(out_dev[b], non_blocking=True)
            out_done[b].record(s_out)

    e2e_steps(3)
    torch.cuda.synchronize(dev)
    cool_down(2 * ms_per_step * args.e2e_steps / 1e3)
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e2e_steps(args.e2e_steps)
    s_out.wait_event(cmp_done[(args.e2e_steps - 1) & 1])
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    if dist:
        dist.barrier()

    # ---------------- the other Hy4-shape workloads on the same weights
    # (decode: HBM-bound weight stream; skewed routing: tensor-bound), timed
    # the same way after the headline measurement, single GPU only
    workloads = None
    hy4 = ("hy4_prefill", "hy4_decode", "hy4_skew")
    if (world == 1 and not fp8 and not args.no_workloads and base_cfg.name in hy4
            and args.tokens is None and args.experts is None):
        workloads = {}
        from sparse_moe_layer_06_b200.workloads import skew_logit_bias
        for name in hy4:
            if name == base_cfg.name:
                continue
            c = CONFIGS[name]
            winp = dict(inp)
            winp["logit_bias"] = skew_logit_bias(c.E).to(dev) if c.skew_bias else None
            xw = make_x(c, seed=rank_token_seed(rank), device=dev)
            workloads[name] = measure_workload(moe, c, winp, xw, dev, stream, args.steps,
                                               args.warmup)
            del xw

    if rank != 0:
        clocks.stop()
        if dist:
            dist.destroy_process_group()
        return 0
    clocks.stop()

    # ---------------- derived numbers
    peaks, peak_kind = read_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    tf_peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    if fp8:
        tf_peak *= 2.0  # E4M3 dense peak: the bf16 measurement x the nominal 4.5/2.25 ratio
    idx_cpu = idx.cpu()
    flops, bytes_, touched = layer_counts(cfg, idx_cpu, fp8)
    t_s = ms_per_step / 1e3
    tokens_per_s = whole_job_rate(cfg.T, world, t_s)
    roof_t = max(flops / (tf_peak * 1e12), bytes_ / (hbm_peak * 1e9))
    layer_frac = roof_t / t_s
    roof_t_nominal = max(flops / 2250e12, bytes_ / 8000e9)

    per_kernel = {k: {"launches": v[0], "ms_per_launch": v[1] / max(1, v[0]),
                      "share": v[1] / max(1e-9, sum(x[1] for x in kt.values()))}
                  for k, v in kt.items()}
    dominant = max(kt, key=lambda k: kt[k][1])
    dom_ms = kt[dominant][1] / max(1, kt[dominant][0])
    roof = kernel_roofline(dominant, cfg, touched, fp8, dom_ms, hbm_peak, tf_peak)
    roof["traffic"] = ncu_traffic(dominant, cfg.name)
    roof["timing"] = ("CUDA events around each launch on its stream, over a pass of "
                      f"{args.steps} steps right after the timed region")
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" \
        else "fallback"
    if fp8 and roof["bound"] == "tensor":
        roof["peak_source"] += ", x2 for E4M3 (nominal ratio)"

    cpu_base = None
    # (the FP8 variant reports none: encoding the full weight set with the
    # CPU oracle alone takes minutes)
    if not args.no_cpu_baseline and world == 1 and not fp8:
        import oracle
        oracle.build()
        cpu_inp = cpu_inputs(inp)
        cpu_base = oracle_baseline(cfg, cpu_inp)

    h2d = cfg.T * cfg.H * x_host.element_size()
    d2h = cfg.T * cfg.H * out_host[0].element_size()
    line = {
        "metric": METRIC,
        "value": tokens_per_s,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3" if fp8 else ("bf16" if cfg.dtype == torch.bfloat16 else "f32"),
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.006) weights; random init)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E,
                   "top_k": cfg.top_k, "I": cfg.I, "num_shared": cfg.num_shared,
                   "global_batch": world * cfg.T, "parallelism": f"replicas x{world}",
                   "weights": args.weights,
                   "l2": "inputs larger than L2 (expert weights "
                         f"{cfg.E * 3 * cfg.I * cfg.H * (1 if fp8 else 2) / 1e9:.1f} GB "
                         "streamed each step)"},
        "tflops": flops / t_s / 1e12,
        "layer_roofline": {"frac": layer_frac, "frac_nominal_8tbs_2.25pf": roof_t_nominal / t_s,
                           "roofline_ms": roof_t * 1e3, "flops": flops, "bytes": bytes_,
                           "touched_experts": touched, "peak_source": peak_kind},
        "roofline": roof,
        "kernels": per_kernel,
        "workloads": workloads,
        "cpu_baseline": cpu_base,
        "clocks": clock_rec,
        "e2e": {"value": whole_job_rate(cfg.T * args.e2e_steps, world, e2e_ms / 1e3),
                "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "device_status": status,
    }
    print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
