#!/usr/bin/env python
"""Benchmark of the linear-attention hot path on B200.

One step = the whole path for one batch of synthetic input: S_0 = 0, the
chunkwise prefill of every sequence (la_prefill), then `decode_steps` decode
tokens per sequence (la_decode_step), all through the C ABI.  Default
workload: B=8 sequences x H=16 heads, T=8192 tokens, d_k=d_v=128, bf16
inputs with L2-normalised keys, 256 decode steps; the prefill runs the
library's default chunk (128), and a chunk sweep (16, 32, 64, 128) times the
prefill alone.  Also reported outside the timed step: decode with a cold
state, and the few-token prefill (8 tokens per unit from a saved state).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): units are independent, so every rank
runs its own batch (weak scaling, no data-path collective); the barrier and
the max-over-ranks time use NCCL.  Rank 0 prints one JSON line.

The reference arm (--impl reference) times the float64 CPU oracle (the
literal token-by-token recurrence) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s and % of bf16 tensor peak; decode tokens/s and % HBM BW (1×B200)"
DEFAULT_WORKLOAD = "b8h16_t8192_d128_knorm"
L2_BYTES_FALLBACK = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 HBM3e bandwidth as rated by NVIDIA (HGX figure), reported beside the
# fractions of the measured copy rate; the targets are judged on the measured one.
RATED_HBM_GBS = 7700.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--chunk", type=int, default=0, help="0 = the library's default for the shape")
    ap.add_argument("--sweep-chunks", default="16,32,64,128",
                    help="also time the prefill alone at these chunk sizes ('' = none)")
    ap.add_argument("--batch", type=int, default=0, help="override B (small profiling cases)")
    ap.add_argument("--e2e-steps", type=int, default=10, help="steps of the end-to-end run")
    ap.add_argument("--decode-steps", type=int, default=-1, help="-1 = the workload's count")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-short", action="store_true", help="skip the few-token prefill measurement")
    ap.add_argument("--short-only", default="", metavar="UNITS[,UNITS]",
                    help="only the few-token prefill measurement, on UNITS units (multiples of 32) of the workload's d")
    ap.add_argument("--no-cold-decode", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target wall time of the oracle sample")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- helpers --

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of one GPU
    every 20 ms through NVML (read-only queries) while the timed region runs."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nv = nv
            u = self.uuid if self.uuid is None or self.uuid.startswith("GPU-") else "GPU-" + self.uuid
            self._h = nv.nvmlDeviceGetHandleByUUID(u) if u else nv.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception as e:  # no NVML: report no samples
            self.error = repr(e)
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, mask))
            except Exception as e:
                self.error = repr(e)
            self._stop.wait(0.02)

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": self.error}
        nv = self._nv
        reasons = set()
        for _, mask in self.samples:
            for name, const in self.REASONS.items():
                if hasattr(nv, const) and mask & getattr(nv, const):
                    reasons.add(name)
        mhz = [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "sm_min_mhz": min(mhz),
                "reasons": sorted(reasons), "samples": len(mhz)}


def measured_traffic(kernel_key: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, or None
    when the kernel's sources changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic_b8h16_t8192_d128.json")
    try:
        with open(path) as f:
            entry = json.load(f)[kernel_key]
        for src, digest in entry["sources"].items():
            with open(os.path.join(ROOT, src), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        return int(entry["bytes_per_launch"])
    except Exception:
        return None


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------ multi-rank plumbing --

def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, units_per_step_per_rank: float, ms_max: float) -> float:
    """Weak scaling: every rank runs its own batch; the job's rate is all the
    ranks' work divided by the slowest rank's time."""
    return world * steps * units_per_step_per_rank / (ms_max * 1e-3)


# ------------------------------------------------------ algorithmic sizes --

def prefill_bytes(units, T, dk, dv, elem):
    """Q, K, V read and O written once, S_0 read and S_T written once."""
    return units * T * (2 * dk + 2 * dv) * elem + units * 2 * dk * dv * 4


def prefill_flops_dense(units, T, dk, dv, C):
    """Dense-tile tensor work: QK^T (2C d_k), PV (2C d_v), QS and K^T V (2 d_k d_v each) per token."""
    return units * T * (2 * C * dk + 2 * C * dv + 4 * dk * dv)


def decode_bytes(units, dk, dv, elem):
    """State read + written (fp32), q, k, v read and o written."""
    return units * (8 * dk * dv + elem * (2 * dk + 2 * dv))


# ----------------------------------------------------------- reference arm --

def _oracle_pass(wl, units, dsteps):
    """One pass of the whole path on `units` (sequence, head) units with the
    float64 oracle: full prefill, then `dsteps` decode tokens.  Returns seconds
    spent in the oracle (input generation excluded)."""
    import numpy as np
    from oracle import la_oracle as ora
    from recurrent_decode_la_b200 import inputs
    qkv = [inputs.unit_qkv(wl, u) for u in units]
    Q = np.stack([x[0].float().numpy() for x in qkv])[:, None]
    K = np.stack([x[1].float().numpy() for x in qkv])[:, None]
    V = np.stack([x[2].float().numpy() for x in qkv])[:, None]
    dec = [inputs.decode_token(wl, s, units=max(units) + 1) for s in range(dsteps)]
    t0 = time.perf_counter()
    _, S = ora.recurrent(Q, K, V)
    S = S.reshape(len(units), wl.d, wl.d)
    for dq, dk_, dv in dec:
        _, S = ora.decode_step(dq[units], dk_[units], dv[units], S)
    return time.perf_counter() - t0


def _oracle_units_for(wl, seconds, dsteps):
    """How many units make one oracle pass last about `seconds`."""
    from oracle import la_oracle as ora
    from recurrent_decode_la_b200 import inputs
    cores = ora.max_threads()
    n_units = inputs.n_units(wl)
    probe = list(range(min(cores, n_units)))
    t = _oracle_pass(wl, probe, wl.decode_steps and min(wl.decode_steps, dsteps))
    per_round = max(t, 1e-3)               # one unit per core in parallel
    rounds = max(1, int(seconds / per_round))
    return min(n_units, rounds * len(probe)), cores


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or "" if unknown."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


def run_reference(args, wl, world, rank):
    """The reference arm: the float64 CPU oracle (C recurrence over OpenMP
    threads) timed on a bounded sample of the same workload."""
    if rank != 0:
        return 0
    from recurrent_decode_la_b200 import inputs
    dsteps = wl.decode_steps if args.decode_steps < 0 else args.decode_steps
    n_units = inputs.n_units(wl)
    per_step = max(0.5, args.cpu_seconds / max(1, args.steps + args.warmup))
    units, cores = _oracle_units_for(wl, per_step, dsteps)
    sample = list(range(units))
    times = []
    for it in range(args.warmup + args.steps):
        t = _oracle_pass(wl, sample, dsteps)
        if it >= args.warmup:
            times.append(t)
    tot = sum(times)
    tokens = args.steps * units * (wl.T + dsteps) / wl.H   # a token carries H heads
    value = tokens / tot
    desc = (f"{units} of {n_units} (sequence, head) units per step: full T={wl.T} prefill + "
            f"{dsteps} decode tokens each, float64 recurrence; tokens = unit rows / H")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "T": wl.T, "d_k": wl.d, "d_v": wl.d,
                   "decode_steps": dsteps, "sample_units": units, "of_units": n_units},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline_sample(wl, seconds, dsteps):
    """The oracle on the host cores, one bounded pass (rank 0, N=1 only)."""
    from recurrent_decode_la_b200 import inputs
    units, cores = _oracle_units_for(wl, seconds, dsteps)
    t = _oracle_pass(wl, list(range(units)), dsteps)
    tokens = units * (wl.T + dsteps) / wl.H
    return {"value": tokens / t, "unit": "tokens/s", "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{units} of {inputs.n_units(wl)} (sequence, head) units: full T={wl.T} prefill + "
                      f"{dsteps} decode tokens each, float64 recurrence, {t:.1f} s; tokens = unit rows / H"}


# ------------------------------------------------------------------ our arm --

def run_ours(args, wl, world, rank, local):
    import torch
    import torch.distributed as dist

    import recurrent_decode_la_b200 as la
    from recurrent_decode_la_b200 import inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    la.load_library()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks, peak_src = load_peaks()
    B, H, T, d = wl.B, wl.H, wl.T, wl.d
    chunk = args.chunk or la.la_resolve_chunk(wl.torch_dtype, wl.d, wl.d, 0)
    dsteps = wl.decode_steps if args.decode_steps < 0 else args.decode_steps
    units = B * H
    elem = 2 if wl.dtype == "bf16" else 4
    dt = wl.torch_dtype

    # every rank runs its own batch of the same shape (weak scaling)
    q_h, k_h, v_h, _ = inputs.prefill_inputs(wl)
    dq_h, dk_h, dv_h = [], [], []
    for s in range(dsteps):
        a, b_, c = inputs.decode_token(wl, s, units=units)
        dq_h.append(a); dk_h.append(b_); dv_h.append(c)
    dq_h = torch.stack(dq_h).reshape(dsteps, B, H, d) if dsteps else torch.empty(0, B, H, d, dtype=dt)
    dk_h = torch.stack(dk_h).reshape(dsteps, B, H, d) if dsteps else torch.empty(0, B, H, d, dtype=dt)
    dv_h = torch.stack(dv_h).reshape(dsteps, B, H, d) if dsteps else torch.empty(0, B, H, d, dtype=dt)

    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    dq, dk_, dv = dq_h.to(dev), dk_h.to(dev), dv_h.to(dev)
    o = torch.empty_like(v)
    od = torch.empty_like(dv)
    state = torch.empty(units, d, d, dtype=torch.float32, device=dev)
    path = la.la_prefill_path(dt, d, d, chunk, q, k, v, o)
    ws_bytes = la.la_prefill_workspace_size(dt, B, H, T, d, d, 0, chunk)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None

    stream = torch.cuda.Stream(device=dev)

    def prefill_phase(s):
        la.la_state_init(state, None, stream=s)
        la.la_prefill(q, k, v, o, state, chunk=chunk, workspace=ws, stream=s)

    def decode_phase(s):
        for i in range(dsteps):
            la.la_decode_step(dq[i], dk_[i], dv[i], od[i], state, stream=s)

    # warm the launch path (sets kernel attributes) before capturing graphs
    with torch.cuda.stream(stream):
        prefill_phase(stream)
        decode_phase(stream)
    stream.synchronize()
    if la.la_device_status(stream) != la.LA_OK:
        raise RuntimeError("device status not ok after warm-up")

    g_pre = torch.cuda.CUDAGraph()
    g_dec = torch.cuda.CUDAGraph() if dsteps else None
    with torch.cuda.graph(g_pre, stream=stream):
        prefill_phase(torch.cuda.current_stream())
    if g_dec is not None:
        with torch.cuda.graph(g_dec, stream=stream):
            decode_phase(torch.cuda.current_stream())

    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            g_pre.replay()
            if g_dec is not None:
                g_dec.replay()
    stream.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(getattr(torch.cuda.get_device_properties(dev), "uuid", None) and
                      str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        with torch.cuda.stream(stream):
            t_start.record(stream)
            for i in range(args.steps):
                ev[i][0].record(stream)
                g_pre.replay()
                ev[i][1].record(stream)
                if g_dec is not None:
                    g_dec.replay()
                ev[i][2].record(stream)
            t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    status = la.la_device_status(stream)
    ms_total = t_start.elapsed_time(t_end)
    ms_pre = [e[0].elapsed_time(e[1]) for e in ev]
    ms_dec = [e[1].elapsed_time(e[2]) for e in ev]
    ms_total = max_over_ranks(ms_total, dev)

    tokens_step = B * T + B * dsteps              # sequence positions (all heads)
    value = whole_job_rate(world, args.steps, tokens_step, ms_total)
    pre_ms = statistics.mean(ms_pre)
    dec_ms = statistics.mean(ms_dec) if dsteps else 0.0
    pre_bytes = prefill_bytes(units, T, d, d, elem)
    pre_flops = prefill_flops_dense(units, T, d, d, chunk)
    dec_bytes = decode_bytes(units, d, d, elem)
    # prefill launch = state init + prefill kernel; the state init moves
    # units*d*d*4 bytes and is counted in its own launch below.
    pre_gbs = pre_bytes / (pre_ms * 1e-3) / 1e9
    dec_us = 1e3 * dec_ms / max(1, dsteps)
    dec_gbs = dec_bytes / (dec_us * 1e-6) / 1e9 if dsteps else 0.0
    pre_tflops = pre_flops / (pre_ms * 1e-3) / 1e12

    cold = None
    if not args.no_cold_decode and dsteps:
        cold = cold_decode(la, torch, dev, stream, wl, units, dq, dk_, dv, od, peaks, peak_src)
    # dominant kernel by device time within the step
    pre_share = pre_ms / (pre_ms + dec_ms) if (pre_ms + dec_ms) > 0 else 1.0
    default_shape = (wl.name == DEFAULT_WORKLOAD and chunk == 128)
    roof_pre = {"bound": "hbm", "kernel": f"prefill_{path}", "achieved": pre_gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": pre_gbs / peaks["hbm_gbs"], "frac_of_rated": pre_gbs / RATED_HBM_GBS,
                "traffic": measured_traffic("prefill_tc") if default_shape else None,
                "bytes_per_launch": pre_bytes, "share_of_step": pre_share,
                "peak_source": f"{peak_src} hbm_gbs"}
    dec_traffic = measured_traffic("decode_cols") if wl.name == DEFAULT_WORKLOAD else None
    if cold is not None:
        # the decode's HBM figure: the state is cold (rotating sets larger than L2)
        roof_dec = {"bound": "hbm", "kernel": "decode_cols", "achieved": cold["achieved_gbs"],
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": cold["hbm_frac"],
                    "frac_of_rated": cold["hbm_frac_of_rated"], "traffic": dec_traffic,
                    "traffic_note": "ncu capture with L2 flushed before the launch (cold state)",
                    "bytes_per_launch": dec_bytes, "share_of_step": 1 - pre_share,
                    "note": f"cold state: {cold['state_sets']} rotating state sets larger than L2, "
                            f"{cold['us_per_launch']:.3f} us per launch",
                    "peak_source": f"{peak_src} hbm_gbs"}
    else:
        roof_dec = {"bound": "l2", "kernel": "decode_cols", "achieved": dec_gbs, "peak": None, "unit": "GB/s",
                    "frac": None, "traffic": None, "bytes_per_launch": dec_bytes, "share_of_step": 1 - pre_share,
                    "note": "state L2-resident (stepped in place); no cold-state measurement in this run"}
    headline = {
        "prefill_tokens_per_s": B * T / (pre_ms * 1e-3),
        "prefill_tensor_frac_burst": pre_tflops / peaks["bf16_tflops"],
        "prefill_hbm_frac": pre_gbs / peaks["hbm_gbs"],
        "decode_tokens_per_s_cold": cold["tokens_per_s"] if cold else None,
        "decode_hbm_frac_cold": cold["hbm_frac"] if cold else None,
        "decode_tokens_per_s_in_step": B * dsteps / (dec_ms * 1e-3) if dsteps else 0.0,
        "note": "prefill at the library default C = %d; tensor fraction = dense-tile flops / burst bf16 peak; "
                "HBM fractions of the %s copy rate" % (chunk, peak_src),
    }
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "headline": headline, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "H": H, "T": T, "d_k": d, "d_v": d, "chunk": chunk,
                   "chunk_note": "the timed step runs C = %d (the library default); the workload lists C = %d, "
                                 "timed in chunk_sweep with the other sizes (C never changes the result)"
                                 % (chunk, wl.chunk),
                   "decode_steps": dsteps, "prefill_kernel": path, "workspace_bytes": ws_bytes,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (q/k/v %.0f MB per rank); decode state is the "
                         "prefill's output and stays L2-resident within a step" % (3 * q.numel() * elem / 1e6)},
        "value_note": "value = (B*T prefill + B*decode_steps decode) tokens per second of step time",
        "prefill": {"tokens_per_s": B * T / (pre_ms * 1e-3), "ms": pre_ms,
                    "achieved_gbs": pre_gbs, "hbm_frac": pre_gbs / peaks["hbm_gbs"],
                    "hbm_frac_of_rated": pre_gbs / RATED_HBM_GBS,
                    "dense_tflops": pre_tflops,
                    "tensor_frac_burst": pre_tflops / peaks["bf16_tflops"],
                    "tensor_frac_sustained": pre_tflops / peaks["bf16_tflops_sustained"]},
        "decode": {"tokens_per_s_in_step": B * dsteps / (dec_ms * 1e-3) if dsteps else 0.0,
                   "us_per_step_in_step": dec_us, "achieved_gbs_l2_resident": dec_gbs},
        "gpu_launches": args.steps * (2 + dsteps),
        "device_status": la.la_status_string(status),
        "peaks_source": peak_src, "rated_hbm_gbs": RATED_HBM_GBS,
    }
    result["roofline"] = roof_pre if pre_share >= 0.5 else roof_dec
    result["roofline_prefill"] = roof_pre
    result["roofline_decode"] = roof_dec
    result["clocks"] = clk.summary()

    if args.sweep_chunks:
        result["chunk_sweep"] = chunk_sweep(la, torch, stream, q, k, v, o, state, wl,
                                            [int(c) for c in args.sweep_chunks.split(",")], peaks, dev)
    if cold is not None:
        result["decode_cold"] = cold
    if not args.no_short and wl.dtype == "bf16":
        shapes = ((wl.B, wl.H), (256, 32))
        result["short_prefill"] = [short_prefill(la, torch, dev, stream, wl, B_, H_, 8, peaks, peak_src)
                                   for B_, H_ in shapes]
        if world == 1:
            for entry, ch in zip(result["short_prefill"], chunked_short_comparison(wl, shapes)):
                entry["chunked"] = ch

    if not args.no_e2e:
        result["e2e"] = e2e_run(args, la, torch, dev, stream, wl, chunk, dsteps, q_h, k_h, v_h, dq_h, dk_h, dv_h,
                                world)
    if world > 1:
        dist.barrier()
    del g_pre, g_dec
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline_sample(wl, args.cpu_seconds, dsteps)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def chunk_sweep(la, torch, stream, q, k, v, o, state, wl, chunks, peaks, dev):
    """Prefill alone at several chunk sizes (C never changes the result, only
    the cost): CUDA-event time of one launch, median of 20 after 3 warm-ups."""
    out = {}
    units, d = wl.B * wl.H, wl.d
    elem = 2 if wl.dtype == "bf16" else 4
    byts = prefill_bytes(units, wl.T, d, d, elem)
    for c in chunks:
        path = la.la_prefill_path(wl.torch_dtype, d, d, c, q, k, v, o)
        nb = la.la_prefill_workspace_size(wl.torch_dtype, wl.B, wl.H, wl.T, d, d, 0, c)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
        ts = []
        with torch.cuda.stream(stream):
            for i in range(23):
                la.la_state_init(state, None, stream=stream)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                la.la_prefill(q, k, v, o, state, chunk=c, workspace=ws, stream=stream)
                e1.record(stream)
                e1.synchronize()
                if i >= 3:
                    ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        flops = prefill_flops_dense(units, wl.T, d, d, c)
        out[str(c)] = {"kernel": path, "ms": ms, "tokens_per_s": wl.B * wl.T / (ms * 1e-3),
                       "hbm_frac": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                       "tensor_frac_burst_dense": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}
    return out


def run_varlen(args, wl, world, rank, local):
    """Packed variable-length workload: one step = prefill of every packed
    sequence (la_prefill with cu_seqlens), the prefilled states tiled
    decode_repeat times (la_state_init copies), then decode steps for all those
    states.  Same timing rules and JSON keys as the dense workload."""
    import concurrent.futures
    import torch
    import torch.distributed as dist

    import recurrent_decode_la_b200 as la
    from recurrent_decode_la_b200 import inputs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    la.load_library()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peaks, peak_src = load_peaks()
    H, d, N, rep = wl.H, wl.d, wl.num_seqs, wl.decode_repeat
    chunk = args.chunk or la.la_resolve_chunk(wl.torch_dtype, d, d, 0)
    dsteps = wl.decode_steps if args.decode_steps < 0 else args.decode_steps
    q_h, k_h, v_h, cu = inputs.prefill_inputs(wl)
    Ttot = q_h.shape[2]
    max_len = int((cu[1:] - cu[:-1]).max())
    units, dunits, bdec = N * H, inputs.decode_units(wl), N * rep
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        toks = list(ex.map(lambda s_: inputs.decode_token(wl, s_, units=dunits), range(dsteps)))
    q, k, v, cud = q_h.to(dev), k_h.to(dev), v_h.to(dev), cu.to(dev)
    shape = (dsteps, bdec, H, d)
    dq = torch.stack([t[0] for t in toks]).reshape(shape).to(dev) if dsteps else None
    dk_ = torch.stack([t[1] for t in toks]).reshape(shape).to(dev) if dsteps else None
    dv = torch.stack([t[2] for t in toks]).reshape(shape).to(dev) if dsteps else None
    del toks
    o = torch.empty_like(v)
    od = torch.empty_like(dv) if dsteps else None
    st_p = torch.empty(units, d, d, dtype=torch.float32, device=dev)
    st_d = torch.empty(dunits, d, d, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    # workspace for the longest-first order of the packed sequences
    ws_bytes = la.la_prefill_workspace_size(wl.torch_dtype, 1, H, Ttot, d, d, N, chunk)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    ordered = ws_bytes > 0 and units > torch.cuda.get_device_properties(dev).multi_processor_count

    def prefill_phase(s_):
        la.la_state_init(st_p, None, stream=s_)
        la.la_prefill(q, k, v, o, st_p, cu_seqlens=cud, max_seqlen=max_len, chunk=chunk, workspace=ws, stream=s_)
        for r in range(rep):
            la.la_state_init(st_d[r * units:(r + 1) * units], st_p, stream=s_)

    def decode_phase(s_):
        for i in range(dsteps):
            la.la_decode_step(dq[i], dk_[i], dv[i], od[i], st_d, stream=s_)

    with torch.cuda.stream(stream):
        prefill_phase(stream)
        if dsteps:
            decode_phase(stream)
    stream.synchronize()
    g_pre = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_pre, stream=stream):
        prefill_phase(torch.cuda.current_stream())
    g_dec = None
    if dsteps:
        g_dec = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_dec, stream=stream):
            decode_phase(torch.cuda.current_stream())
    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            g_pre.replay()
            if g_dec is not None:
                g_dec.replay()
    stream.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(str(torch.cuda.get_device_properties(dev).uuid)) as clk:
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                ev[i][0].record(stream)
                g_pre.replay()
                ev[i][1].record(stream)
                if g_dec is not None:
                    g_dec.replay()
                ev[i][2].record(stream)
        torch.cuda.synchronize()
    status = la.la_device_status(stream)
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    dec_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev) if dsteps else 0.0
    ms_total = max_over_ranks(ev[0][0].elapsed_time(ev[-1][2]), dev)
    tokens_step = Ttot + bdec * dsteps
    elem = 2 if wl.dtype == "bf16" else 4
    pre_bytes = Ttot * H * 4 * d * elem + units * 2 * d * d * 4
    dec_bytes = decode_bytes(dunits, d, d, elem)
    pre_gbs = pre_bytes / (pre_ms * 1e-3) / 1e9
    dec_us = 1e3 * dec_ms / max(1, dsteps)
    dec_gbs = dec_bytes / (dec_us * 1e-6) / 1e9 if dsteps else 0.0
    pre_share = pre_ms / (pre_ms + dec_ms) if (pre_ms + dec_ms) > 0 else 1.0
    roof_pre = {"bound": "hbm", "kernel": "prefill_" + la.la_prefill_path(wl.torch_dtype, d, d, chunk, q, k, v, o),
                "achieved": pre_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": pre_gbs / peaks["hbm_gbs"],
                "frac_of_rated": pre_gbs / RATED_HBM_GBS,
                "traffic": None, "bytes_per_launch": pre_bytes, "share_of_step": pre_share,
                "peak_source": f"{peak_src} hbm_gbs"}
    roof_dec = {"bound": "hbm", "kernel": "decode_cols", "achieved": dec_gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"], "frac_of_rated": dec_gbs / RATED_HBM_GBS,
                "traffic": None, "bytes_per_launch": dec_bytes,
                "share_of_step": 1 - pre_share, "note": "512 MiB of decode state: cold in every step",
                "peak_source": f"{peak_src} hbm_gbs"}
    headline = {"prefill_tokens_per_s": Ttot / (pre_ms * 1e-3), "prefill_hbm_frac": pre_gbs / peaks["hbm_gbs"],
                "decode_tokens_per_s_cold": bdec * dsteps / (dec_ms * 1e-3) if dsteps else None,
                "decode_hbm_frac_cold": dec_gbs / peaks["hbm_gbs"] if dsteps else None,
                "note": f"prefill at C = {chunk}; the decode state (512 MiB) is cold in every step"}
    result = {
        "metric": METRIC, "value": whole_job_rate(world, args.steps, tokens_step, ms_total), "unit": "tokens/s",
        "headline": headline, "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs": N, "H": H, "T_total": Ttot, "max_seqlen": max_len, "d_k": d,
                   "d_v": d, "chunk": chunk, "decode_units": dunits, "decode_steps": dsteps,
                   "workspace_bytes": ws_bytes, "schedule": "longest first" if ordered else "in order",
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs (%.1f GB) and decode state (512 MiB) larger than L2" % (3 * q.numel() * elem / 1e9)},
        "prefill": {"tokens_per_s": Ttot / (pre_ms * 1e-3), "ms": pre_ms, "achieved_gbs": pre_gbs,
                    "hbm_frac": pre_gbs / peaks["hbm_gbs"]},
        "decode": {"tokens_per_s": bdec * dsteps / (dec_ms * 1e-3) if dsteps else 0.0, "us_per_step": dec_us,
                   "achieved_gbs": dec_gbs, "hbm_frac": dec_gbs / peaks["hbm_gbs"] if dsteps else 0.0},
        "roofline": roof_pre if pre_share >= 0.5 else roof_dec, "roofline_prefill": roof_pre,
        "gpu_launches": args.steps * (2 + rep + dsteps + (1 if ordered else 0)),
        "device_status": la.la_status_string(status),
        "clocks": clk.summary(), "peaks_source": peak_src,
    }
    del g_pre, g_dec
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def cold_decode(la, torch, dev, stream, wl, units, dq, dk_, dv, od, peaks, peak_src):
    """Decode with a cold state: rotate over R state sets larger than L2 (as a
    stack of R layers would), one launch per set, timed with CUDA events.
    Beside it, the same rotation through a plain in-place read and write of
    every state set (torch's elementwise add, one launch per set): the
    streaming floor of moving these bytes on this GPU, for comparison."""
    d = wl.d
    try:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    except Exception:
        l2 = L2_BYTES_FALLBACK
    per = units * d * d * 4
    R = max(8, int(math.ceil(2.5 * l2 / per)))
    states = torch.zeros(R, units, d, d, dtype=torch.float32, device=dev)
    reps = 4

    def timed(body):
        with torch.cuda.stream(stream):
            for r in range(R):
                body(r, stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                for r in range(R):
                    body(r, torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        del g
        return 1e3 * e0.elapsed_time(e1) / (reps * R)

    n = dq.shape[0]
    us = timed(lambda r, s_: la.la_decode_step(dq[r % n], dk_[r % n], dv[r % n], od[0], states[r], stream=s_))
    floor_us = timed(lambda r, s_: states[r].add_(1.0))
    elem = 2 if wl.dtype == "bf16" else 4
    byts = decode_bytes(units, d, d, elem)
    gbs = byts / (us * 1e-6) / 1e9
    del states
    return {"us_per_launch": us, "units": units, "state_sets": R, "bytes_per_launch": byts,
            "achieved_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "hbm_frac_of_rated": gbs / RATED_HBM_GBS,
            "peak_source": f"{peak_src} hbm_gbs", "tokens_per_s": wl.B / (us * 1e-6),
            "copy_floor_us": floor_us, "kernel_over_floor": us / floor_us,
            "copy_floor": "torch in-place add over the same state sets (fp32 read + write, "
                          f"{units * d * d * 8} B per launch, no q/k/v/o)"}


def short_prefill(la, torch, dev, stream, wl, B, H, T, peaks, peak_src):
    """T tokens per unit from a saved state in one la_prefill call (the
    multi-token form of decode, e.g. speculative drafts), B*H units of the
    workload's d.  The state is cold: R state sets larger than L2 in
    rotation, one call per set.  Timed for the kernel the library picks in
    this process (the few-token kernel, unless the process started with
    LINATTN_SHORT=0)."""
    from recurrent_decode_la_b200 import inputs
    d = wl.d
    units = B * H
    try:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    except Exception:
        l2 = L2_BYTES_FALLBACK
    per = units * d * d * 4
    R = max(2, int(math.ceil(2.5 * l2 / per)))
    states = torch.zeros(R, units, d, d, dtype=torch.float32, device=dev)
    q, k, v = (x.to(dev) for x in inputs.random_qkv(4242, B, H, T, d, d, dtype=wl.torch_dtype))
    o = torch.empty_like(v)
    reps = max(1, 64 // R)
    kernel = la.la_prefill_kernel(wl.torch_dtype, T, d, d, 0, q, k, v, o, states[0])
    with torch.cuda.stream(stream):
        for r in range(R):
            la.la_prefill(q, k, v, o, states[r], stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(reps):
            for r in range(R):
                la.la_prefill(q, k, v, o, states[r], stream=torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    stream.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / (reps * R)
    del g, states
    elem = 2 if wl.dtype == "bf16" else 4
    byts = units * (2 * d * d * 4 + T * 4 * d * elem)
    gbs = byts / (us * 1e-6) / 1e9
    return {"T": T, "B": B, "H": H, "units": units, "state_sets": R, "kernel": kernel, "us_per_call": us,
            "tokens_per_s": B * T / (us * 1e-6), "bytes_per_call": byts, "achieved_gbs": gbs,
            "hbm_frac": gbs / peaks["hbm_gbs"], "hbm_frac_of_rated": gbs / RATED_HBM_GBS,
            "peak_source": f"{peak_src} hbm_gbs"}


def chunked_short_comparison(wl, shapes):
    """The same few-token calls with the few-token kernel switched off
    (LINATTN_SHORT=0 in a child process: the library reads its switches once
    per process), for comparison.  Returns one entry per (B, H) shape, or
    None entries when the child fails."""
    import subprocess
    spec = ",".join(f"{b}x{h}" for b, h in shapes)
    env = dict(os.environ, LINATTN_SHORT="0")
    try:
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--workload", wl.name, "--short-only", spec],
                           env=env, capture_output=True, text=True, timeout=900)
        res = json.loads(r.stdout.strip().splitlines()[-1])["short_prefill"]
        return [{"kernel": x["kernel"], "us_per_call": x["us_per_call"]} for x in res]
    except Exception as e:  # report, do not fail the benchmark
        return [{"error": repr(e)[:200]} for _ in shapes]


def e2e_run(args, la, torch, dev, stream, wl, chunk, dsteps, q_h, k_h, v_h, dq_h, dk_h, dv_h, world):
    """The same step through the public API with host buffers: pinned host ->
    device copies of every input and device -> host copies of every output,
    all inside the timed region.  Two forms are timed:

    - "batch" (the headline `e2e`): every input copied in, one la_prefill
      over the whole batch (the timed kernel's launch, same units and
      chunk), the decode steps, then the outputs copied back.  As in a
      serving loop, the copy-in of step i+1 (its own stream) overlaps the
      copy-out of step i (another stream); events order every reuse of a
      buffer, and the copy of o overlaps the decode steps.
    - "pipelined": sequences are independent, so the copy-in of sequence
      b+1 and the copy-out of sequence b-1 overlap the prefill of sequence b
      (la_prefill on that sequence's H units), then the decode steps."""
    B, H, T, d = wl.B, wl.H, wl.T, wl.d
    pins = [x.pin_memory() for x in (q_h, k_h, v_h, dq_h, dk_h, dv_h)]
    o_h = torch.empty_like(pins[2]).pin_memory()
    od_h = torch.empty_like(pins[5]).pin_memory()
    st_h = torch.empty(B * H, d, d, dtype=torch.float32).pin_memory()
    dev_bufs = [torch.empty_like(x, device=dev) for x in pins]
    o = torch.empty_like(dev_bufs[2])
    od = torch.empty_like(dev_bufs[5])
    st = torch.empty(B * H, d, d, dtype=torch.float32, device=dev)
    nb_seq = la.la_prefill_workspace_size(wl.torch_dtype, 1, H, T, d, d, 0, chunk)
    ws_seq = torch.empty(nb_seq, dtype=torch.uint8, device=dev) if nb_seq else None
    nb_all = la.la_prefill_workspace_size(wl.torch_dtype, B, H, T, d, d, 0, chunk)
    ws_all = torch.empty(nb_all, dtype=torch.uint8, device=dev) if nb_all else None
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def decode_and_copy_out():
        for i in range(dsteps):
            la.la_decode_step(dev_bufs[3][i], dev_bufs[4][i], dev_bufs[5][i], od[i], st, stream=stream)
        fin = torch.cuda.Event()
        fin.record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(fin)
            od_h.copy_(od, non_blocking=True)
            st_h.copy_(st, non_blocking=True)
        stream.wait_stream(s_out)

    carried = {}  # events of the previous batch step

    def step_batch():
        with torch.cuda.stream(s_in):
            if "inputs_read" in carried:  # the previous step's kernels are done with the inputs
                s_in.wait_event(carried["inputs_read"])
            for i in range(6):
                dev_bufs[i].copy_(pins[i], non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(s_in)
        stream.wait_event(copied)
        if "outputs_read" in carried:  # the previous step's o, od, state are on the host
            stream.wait_event(carried["outputs_read"])
        la.la_state_init(st, None, stream=stream)
        la.la_prefill(dev_bufs[0], dev_bufs[1], dev_bufs[2], o, st, chunk=chunk, workspace=ws_all, stream=stream)
        pre = torch.cuda.Event()
        pre.record(stream)
        for i in range(dsteps):
            la.la_decode_step(dev_bufs[3][i], dev_bufs[4][i], dev_bufs[5][i], od[i], st, stream=stream)
        fin = torch.cuda.Event()
        fin.record(stream)
        carried["inputs_read"] = fin
        with torch.cuda.stream(s_out):
            s_out.wait_event(pre)
            o_h.copy_(o, non_blocking=True)
            s_out.wait_event(fin)
            od_h.copy_(od, non_blocking=True)
            st_h.copy_(st, non_blocking=True)
            out = torch.cuda.Event()
            out.record(s_out)
        carried["outputs_read"] = out

    def step_pipelined():
        copied = [torch.cuda.Event() for _ in range(B)]
        done = [torch.cuda.Event() for _ in range(B)]
        with torch.cuda.stream(s_in):
            s_in.wait_stream(stream)
            for b in range(B):
                for i in range(3):
                    dev_bufs[i][b].copy_(pins[i][b], non_blocking=True)
                copied[b].record(s_in)
            for i in range(3, 6):
                dev_bufs[i].copy_(pins[i], non_blocking=True)
            dec_in = torch.cuda.Event()
            dec_in.record(s_in)
        for b in range(B):
            stream.wait_event(copied[b])
            sl = slice(b * H, (b + 1) * H)
            la.la_state_init(st[sl], None, stream=stream)
            la.la_prefill(dev_bufs[0][b:b + 1], dev_bufs[1][b:b + 1], dev_bufs[2][b:b + 1], o[b:b + 1], st[sl],
                          chunk=chunk, workspace=ws_seq, stream=stream)
            done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[b])
                o_h[b].copy_(o[b], non_blocking=True)
        stream.wait_event(dec_in)
        decode_and_copy_out()

    n_steps = max(1, min(args.steps, args.e2e_steps))
    h2d = sum(x.numel() * x.element_size() for x in pins)
    d2h = o_h.numel() * o_h.element_size() + od_h.numel() * od_h.element_size() + st_h.numel() * 4
    tokens = B * T + B * dsteps

    def timed(step):
        with torch.cuda.stream(stream):
            for _ in range(3):
                step()
            for x in (stream, s_in, s_out):
                x.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            s_in.wait_event(e0)  # the first copy-in starts inside the timed region
            for _ in range(n_steps):
                step()
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)  # the last copy-out ends inside it
            e1.record(stream)
        stream.synchronize()
        ms = e0.elapsed_time(e1)
        return {"value": world * n_steps * tokens / (ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / n_steps,
                "steps": n_steps, "h2d_gbs": h2d / (ms / n_steps * 1e-3) / 1e9}

    res = timed(step_batch)
    res["form"] = "batch: copy-in, one la_prefill over all units (the timed kernel's launch), decode, copy-out"
    pipe = timed(step_pipelined)
    res["pipelined"] = {"value": pipe["value"], "ms_per_step": pipe["ms_per_step"],
                        "form": "per sequence: copy-in / la_prefill on H units / copy-out on three streams"}
    return res


def run_short_only(args, wl):
    """Only the few-token prefill measurement (8 tokens per unit, cold
    state) on the (B, H) shapes of args.short_only ("BxH,..." or a unit count
    of 32 heads); prints one JSON line."""
    import torch

    import recurrent_decode_la_b200 as la
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    la.load_library()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    shapes = []
    for item in args.short_only.split(","):
        if "x" in item:
            b, h = item.split("x")
            shapes.append((int(b), int(h)))
        else:
            shapes.append((max(1, int(item) // 32), 32))
    res = [short_prefill(la, torch, dev, stream, wl, B, H, 8, peaks, peak_src) for B, H in shapes]
    print(json.dumps({"short_prefill": res, "device_status": la.la_status_string(la.la_device_status(stream))}))
    return 0


def main(argv=None):
    args = parse_args(argv)
    from recurrent_decode_la_b200 import inputs
    wl = inputs.WORKLOADS[args.workload]
    if args.batch > 0:
        import dataclasses
        wl = dataclasses.replace(wl, name=f"{wl.name}_b{args.batch}", B=args.batch)
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, wl, world, rank)
    if args.short_only:
        return run_short_only(args, wl)
    if wl.varlen:
        return run_varlen(args, wl, world, rank, local)
    return run_ours(args, wl, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
