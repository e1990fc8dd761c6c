#!/usr/bin/env python
"""Benchmark of the fused selective scan (S6) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole hot path over one batch of synthetic input: the forward
(softplus, zero-order-hold discretization, scan, C readout, D skip, SiLU gate,
store) and the recompute-based backward of sum(dy * y), on the bf16-I/O
workload of batch 8, 5120 channels, 2048 steps and N = 16 (fp32 state and
arithmetic).  Inputs are resident in HBM when the timed region starts and each
of u, delta, z, dy (168 MB) is larger than the 126 MB L2, so every step reads
them from DRAM.  Device time comes from CUDA events on the launching stream;
for N > 1 (torchrun, one process per GPU) every rank runs its own independent
batch (weak scaling, no data-path collective) and the step time is the max
over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle
on the host cores instead (bounded channel samples of the same workload).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_21_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = ("selective-scan fwd/bwd GB/s and token·channels/s vs B200 HBM roofline (1 GPU)")
UNIT = "token·channels/s"
DEFAULT_WORKLOAD = 2
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------- accounting

def fwd_bytes(w, last_state=False) -> int:
    """Algorithmic bytes of one forward: read u, delta, z and write y (4 s per
    token-channel), read the B and C rows, the parameters, and write
    last_state if asked."""
    s = w.io_bytes
    tc = w.token_channels
    b = 4 * s * tc + 2 * w.batch * w.N * w.L * s + 4 * (w.dim * w.N + 2 * w.dim)
    return b + (4 * w.batch * w.dim * w.N if last_state else 0)


def bwd_bytes(w) -> int:
    """Algorithmic bytes of one backward: read u, delta, z, dy and write du,
    ddelta, dz (7 s per token-channel), read B, C and write dB, dC, read A, D,
    bias and write dA, dD, dbias."""
    s = w.io_bytes
    tc = w.token_channels
    return 7 * s * tc + 4 * w.batch * w.N * w.L * s + 8 * (w.dim * w.N + 2 * w.dim)


# FP32 work per state element (b, d, t, n) of the method as the pages state it
# (Mamba paper, section 3 Algorithm 2 and the zero-order hold of eq. 4), with
# exp counted on the special-function unit, not here.  Forward: x = Delta A_n;
# Bbar u = (exp(x) - 1) * (B_n * (u / A_n)) as one FMA after two multiplies;
# h = Abar h + Bbar u; y0 += C_n h -> 6.  Backward (no saved states, so the
# forward's 5 state operations are redone): G = C_n dy0 + Abar' G'; Abar G;
# du += G Bbar (2 with forming Bbar); A_n h + B_n u; dDelta and A_n dA_n
# (Delta Abar G (A_n h + B_n u) - G Bbar u) -> 4; dB term G (exp(x) - 1) u / A_n
# and its sum over channels -> 4; dC term dy0 h and its sum -> 2: 5 + 15 = 20.
# Per-token work (softplus, gate, dz) is left out, so these are lower bounds.
FWD_FP32_OPS_PER_ELEMENT = 6
BWD_FP32_OPS_PER_ELEMENT = 20
# Nominal B200 figures, used only when the microbenchmark cannot run: 148 SMs
# x 128 FP32 lanes, one operation (an FMA counts as one) per lane per clock.
B200_SMS, FP32_LANES_PER_SM, B200_MAX_SM_MHZ = 148, 128, 1965

MICRO_KINDS = {"ffma": 0, "fma_f32x2": 1, "ex2": 2, "lg2": 3, "rcp": 4}
MICRO_ITERS = {"ffma": 1 << 17, "fma_f32x2": 1 << 16, "ex2": 1 << 14, "lg2": 1 << 14,
               "rcp": 1 << 14}


def fp32_peak_tops(sm_mhz=None) -> float:
    """Nominal FP32 operation peak of the whole GPU in Top/s at an SM clock."""
    return B200_SMS * FP32_LANES_PER_SM * float(sm_mhz or B200_MAX_SM_MHZ) * 1e6 / 1e12


def run_micro(device_index: int = 0) -> dict:
    """Instruction throughput measured on this GPU by libmambamicro.so (eight
    independent chains per thread, 2048 threads per SM): operations per second
    and per clock per SM at the SM clock NVML reports during each run."""
    import ctypes
    from selective_state_space_21_b200 import build
    lib = ctypes.CDLL(build.build_micro())
    lib.mamba_micro_run.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_double)]
    lib.mamba_micro_run.restype = ctypes.c_int
    sms = torch.cuda.get_device_properties(device_index).multi_processor_count
    out = {"sms": sms, "blocks_per_sm": 8, "threads_per_block": 256, "chains_per_thread": 8}
    for name, kind in MICRO_KINDS.items():
        ms, ops = ctypes.c_double(), ctypes.c_double()
        sampler = ClockSampler(device_index, period_s=0.002)
        with sampler:
            rc = lib.mamba_micro_run(kind, MICRO_ITERS[name], 8, ctypes.byref(ms), ctypes.byref(ops))
        if rc != 0:
            raise RuntimeError(f"microbenchmark {name} failed with CUDA error {rc}")
        clk = sampler.summary()
        rate = ops.value / (ms.value * 1e-3)
        mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz") or B200_MAX_SM_MHZ
        out[name] = {"ops_per_s": rate, "ms": round(ms.value, 3),
                     "per_clk_per_sm": round(rate / (mhz * 1e6) / sms, 2), "sm_mhz": mhz}
    return out


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_bytes_per_launch_bf16_b8_d5120_L2048_N16.txt")


def ncu_traffic(kernel_key: str):
    """Per-launch DRAM bytes of one call ("fwd_save", "bwd_saved", "fwd" or
    "bwd") from the committed ncu summary, only if it was taken on the current
    source of the staged kernels (else None).  Lines: <call> <bytes> <source
    digest> <launches>; # comments."""
    try:
        from selective_state_space_21_b200.build import STAGED_KERNEL_FILES, source_digest
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if not parts or parts[0].startswith("#") or parts[0] != kernel_key:
                    continue
                if parts[2] != source_digest(STAGED_KERNEL_FILES):
                    return None
                return {"bytes_per_launch": int(parts[1]), "source_digest": parts[2]}
    except Exception:
        return None
    return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            mask = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for name, bit in self.REASONS.items():
            if mask & bit and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._t is not None:
            self._stop.set()
            self._t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "source": "unavailable"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


# ------------------------------------------------------------- distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity with one rank)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling)."""
    return base_seed + 1000 * rank


def whole_job_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    return units_per_rank * world / max_seconds


# ------------------------------------------------------------- CPU oracle

def oracle_sample_rate(x_host: dict, w, seconds: float = 10.0, min_blocks: int = 1):
    """Time the fp64 oracle (forward + backward, as it stands) on channel
    blocks of batch row 0 until `seconds` elapse; returns (tc/s, threads,
    description)."""
    import oracle
    threads = oracle.default_threads()
    k = max(8, 2 * threads)
    done_tc = 0
    blocks = 0
    t0 = time.perf_counter()
    d0 = 0
    while True:
        ds = [(d0 + i) % w.dim for i in range(k)]
        d0 = (d0 + k) % w.dim
        idx = torch.tensor(ds)
        sub = {n: (x_host[n][0:1].index_select(1, idx).contiguous() if x_host[n] is not None
                   else None) for n in ("u", "delta", "z", "dy")}
        sub.update(B=x_host["B"][0:1].contiguous(), C=x_host["C"][0:1].contiguous(),
                   A=x_host["A"][idx].contiguous(),
                   D=None if x_host["D"] is None else x_host["D"][idx].contiguous(),
                   delta_bias=x_host["delta_bias"][idx].contiguous())
        oracle.s6_forward(sub["u"], sub["delta"], sub["A"], sub["B"], sub["C"],
                          sub["delta_bias"], sub["D"], sub["z"], nthreads=threads)
        oracle.s6_backward(sub["u"], sub["delta"], sub["A"], sub["B"], sub["C"], sub["dy"],
                           sub["delta_bias"], sub["D"], sub["z"], nthreads=threads)
        done_tc += k * w.L
        blocks += 1
        el = time.perf_counter() - t0
        if el >= seconds and blocks >= min_blocks:
            break
    desc = (f"forward + backward of {blocks} blocks of {k} channels of batch row 0 "
            f"(full L = {w.L}) of {w.name}: {blocks * k} of {w.batch * w.dim} channels, "
            f"{el:.1f} s on {threads} threads")
    return done_tc / el, threads, desc


# ------------------------------------------------------------------- arms

def workload_label(w, step: str) -> str:
    if step == "pair":
        return (f"{w.name} (training step: forward storing the 16-step states + backward "
                f"reading them)")
    return f"{w.name} (forward + recompute backward per step)"


def run_ours(args, world, rank, device):
    from selective_state_space_21_b200 import scan

    w = WORKLOADS[args.workload]
    if args.only == "cplx":  # the complex-A calls alone, for profiling
        if args.cplx_batch:
            w = dataclasses.replace(w, batch=args.cplx_batch)
        res = run_cplx(w, device, measured_peaks(), steps=args.steps, pair=args.step == "pair")
        return {"note": "--only cplx: a profiling run, not a benchmark result", "complex_A": res}
    if args.only == "dtproj":  # the projection calls alone, for profiling
        if args.cplx_batch:
            w = dataclasses.replace(w, batch=args.cplx_batch)
        xp = make_inputs(w.batch, w.dim, w.L, w.N, w.dtype, device=device, seed=1234 + args.workload,
                         has_z=w.has_z, has_D=w.has_D, with_dy=True)
        res = run_dtproj(w, xp, device, steps=args.steps, pair=args.step == "pair")
        return {"note": "--only dtproj: a profiling run, not a benchmark result", "dt_projection": res}
    x = make_inputs(w.batch, w.dim, w.L, w.N, w.dtype, device=device,
                    seed=shard_seed(1234 + args.workload, rank), has_z=w.has_z,
                    has_D=w.has_D, with_dy=True)
    y = torch.empty_like(x["u"])
    g = {"du": torch.empty_like(x["u"]), "ddelta": torch.empty_like(x["u"]),
         "dz": torch.empty_like(x["u"]),
         "dA": torch.empty(w.dim, w.N, device=device), "dB": torch.empty_like(x["B"]),
         "dC": torch.empty_like(x["C"]), "dD": torch.empty(w.dim, device=device),
         "dbias": torch.empty(w.dim, device=device)}

    # The training step: by default the pair whose forward stores the 16-step
    # states for its backward (mamba_scan_fwd_save / mamba_scan_bwd_saved);
    # --step recompute times the backward that re-runs the forward instead.
    pair = args.step == "pair"
    saved = None
    if pair:
        nsaved = scan.saved_bytes(w.batch, w.dim, w.L, w.N, w.dtype)
        saved = torch.empty(nsaved, device=device, dtype=torch.uint8) if nsaved else None

    def fwd():
        if pair:
            scan.mamba_scan_fwd_save(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                     x["D"], x["z"], y, None, saved)
        else:
            scan.mamba_scan_fwd(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                x["D"], x["z"], y, None)

    def bwd_recompute():
        scan.mamba_scan_bwd(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                            x["D"], x["z"], x["dy"], g["du"], g["ddelta"], g["dA"], g["dB"],
                            g["dC"], g["dD"], g["dz"], g["dbias"])

    def bwd():
        if pair:
            scan.mamba_scan_bwd_saved(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                      x["D"], x["z"], x["dy"], g["du"], g["ddelta"], g["dA"],
                                      g["dB"], g["dC"], g["dD"], g["dz"], g["dbias"], saved)
        else:
            bwd_recompute()

    do_fwd = args.only in (None, "fwd")
    do_bwd = args.only in (None, "bwd")
    if pair and do_bwd and not do_fwd:
        fwd()  # the backward reads what the forward saved
    for _ in range(args.warmup):
        if do_fwd:
            fwd()
        if do_bwd:
            bwd()
    torch.cuda.synchronize(device)
    if scan.mamba_scan_stream_status() != 0:
        raise RuntimeError("device error during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = scan.launch_count()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    barrier(device)
    torch.cuda.synchronize(device)
    with sampler:
        start.record()
        for k in range(K):
            ev[k][0].record()
            if do_fwd:
                fwd()
            ev[k][1].record()
            if do_bwd:
                bwd()
            ev[k][2].record()
        end.record()
        torch.cuda.synchronize(device)
    barrier(device)
    launches = scan.launch_count() - launches0
    status = scan.mamba_scan_stream_status()
    if status != 0:
        raise RuntimeError(f"device error in the timed region: {status}")
    total_ms = start.elapsed_time(end)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    step_ms_local = total_ms / K
    step_ms = max_over_ranks(step_ms_local, device)
    fwd_ms_max = max_over_ranks(fwd_ms, device)
    bwd_ms_max = max_over_ranks(bwd_ms, device)

    peaks = measured_peaks()
    peak = peaks["hbm_gbs"]
    fb, bb = fwd_bytes(w), bwd_bytes(w)

    def roof(name, nbytes, ms, kernels):
        ach = nbytes / (ms * 1e-3) / 1e9
        tr = ncu_traffic(name)
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                "frac": round(ach / peak, 4), "traffic": tr["bytes_per_launch"] if tr else None,
                "kernel": name, "launch_group": kernels, "bytes_per_launch": nbytes,
                "peak_source": f"{peaks['source']} hbm_gbs (copy bandwidth)",
                "ms_per_launch": round(ms, 4)}

    if pair:
        roof_fwd = roof("fwd_save", fb, fwd_ms_max, "mamba_scan_fwd_save call")
        roof_bwd = roof("bwd_saved", bb, bwd_ms_max, "mamba_scan_bwd_saved call")
    else:
        roof_fwd = roof("fwd", fb, fwd_ms_max, "mamba_scan_fwd call")
        roof_bwd = roof("bwd", bb, bwd_ms_max, "mamba_scan_bwd call")
    clocks = sampler.summary()
    elements = w.token_channels * w.N
    micro = None
    if not args.no_micro:
        try:
            micro = run_micro(device.index if device.index is not None else 0)
        except Exception as e:  # reported, and the nominal peak is used instead
            micro = {"unavailable": str(e)[:200]}
    if micro and "ffma" in micro:
        alu_peak = micro["ffma"]["ops_per_s"] / 1e12
        alu_src = (f"measured: fma.rn.f32 throughput of this GPU "
                   f"({micro['ffma']['per_clk_per_sm']} per clock per SM at "
                   f"{micro['ffma']['sm_mhz']} MHz; bench.py --micro)")
    else:
        alu_peak = fp32_peak_tops(clocks.get("sm_max_mhz"))
        alu_src = (f"nominal: {B200_SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x "
                   f"{clocks.get('sm_max_mhz') or B200_MAX_SM_MHZ} MHz (microbenchmark unavailable)")

    def roof_alu(name, ops_per_element, ms, hbm):
        ops = ops_per_element * elements
        ach = ops / (ms * 1e-3) / 1e12
        return {"bound": "alu", "achieved": round(ach, 2), "peak": round(alu_peak, 2),
                "unit": "Top/s (FP32, FMA = 1)", "frac": round(ach / alu_peak, 4),
                "traffic": hbm["traffic"], "kernel": name, "launch_group": hbm["launch_group"],
                "ops_per_launch": ops, "ops_per_element": ops_per_element,
                "peak_source": alu_src, "ms_per_launch": round(ms, 4), "hbm_frac": hbm["frac"]}

    alu_fwd = roof_alu(roof_fwd["kernel"], FWD_FP32_OPS_PER_ELEMENT, fwd_ms_max, roof_fwd)
    alu_bwd = roof_alu(roof_bwd["kernel"], BWD_FP32_OPS_PER_ELEMENT, bwd_ms_max, roof_bwd)
    # The metric is throughput against the HBM roofline, so the roofline of
    # record is the HBM fraction of the dominant call; its FP32 fraction
    # (against the measured FMA rate) stands beside it, since both calls are
    # bound by FP32 issue rather than by HBM.
    bwd_dominant = bwd_ms_max >= fwd_ms_max
    dominant = roof_bwd if bwd_dominant else roof_fwd
    dominant_alu = alu_bwd if bwd_dominant else alu_fwd

    tc_step = w.token_channels
    value = whole_job_rate(tc_step, world, step_ms * 1e-3)
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) u, delta, z, B, C, D, dy; log-uniform dt bias; "
                "A = -(n+1))",
        "config": {"workload": workload_label(w, args.step),
                   "batch": w.batch, "dim": w.dim, "L": w.L, "N": w.N,
                   "io_dtype": "bf16" if w.dtype == torch.bfloat16 else "fp32",
                   "state_dtype": "f32", "global_batch": w.batch * world,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (u, delta, z, dy 168 MB each; L2 126 MB)"},
        "gbs": round((fb + bb) / (step_ms * 1e-3) / 1e9 * world, 1),
        "fwd": {"ms": round(fwd_ms_max, 4), "tc_per_s": tc_step * world / (fwd_ms_max * 1e-3),
                "gbs": roof_fwd["achieved"], "frac_hbm": roof_fwd["frac"],
                "frac_alu": alu_fwd["frac"]},
        "bwd": {"ms": round(bwd_ms_max, 4), "tc_per_s": tc_step * world / (bwd_ms_max * 1e-3),
                "gbs": roof_bwd["achieved"], "frac_hbm": roof_bwd["frac"],
                "frac_alu": alu_bwd["frac"]},
        "roofline": dominant, "roofline_alu": dominant_alu,
        "roofline_fwd": roof_fwd, "roofline_fwd_alu": alu_fwd,
        "gpu_launches": launches, "clocks": clocks,
    }
    if micro:
        result["micro"] = micro
    if pair and not args.only:  # the recomputing backward, for context
        result["bwd_recompute"] = time_calls(bwd_recompute, device, args.conv_steps)
        result["bwd_recompute"]["call"] = "mamba_scan_bwd (re-runs the forward first)"

    if not args.only and not args.no_a_legs:
        result["structured_A"] = run_a_leg(w, x, device, peaks, "structured", steps=args.conv_steps)
        result["generic_A"] = run_a_leg(w, x, device, peaks, "generic", steps=args.conv_steps)
    if not args.only and not args.no_decode:
        result["decode"] = run_decode(w, x, device, peaks)
    if not args.only and not args.no_conv:
        result["conv_prologue"] = run_conv(w, x, device, peaks, steps=args.conv_steps,
                                           pair=args.step == "pair")
    if not args.only and not args.no_dtproj:
        result["dt_projection"] = run_dtproj(w, x, device, steps=args.conv_steps,
                                             pair=args.step == "pair")
    if not args.only and not args.no_cplx:
        result["complex_A"] = run_cplx(w, device, peaks, steps=3, pair=args.step == "pair")
    if args.only:
        result["note"] = f"--only {args.only}: a profiling run, not a benchmark result"
    if not args.no_e2e and not args.only:
        result["e2e"] = run_e2e(args, w, x, y, g, fwd, bwd, device, world, pair)

    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.only:
        xh = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in x.items()}
        rate, threads, desc = oracle_sample_rate(xh, w, seconds=args.cpu_seconds)
        result["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads,
                                  "kind": "oracle", "sample": desc}
    return result


def decode_bytes(w) -> int:
    """Algorithmic bytes of one decoding step: read and write the fp32 state
    (8 N bytes per channel), read u, delta, z and write y (4 s per channel),
    read the B and C rows and the parameters."""
    s = w.io_bytes
    ch = w.batch * w.dim
    return ch * (8 * w.N + 4 * s) + 2 * w.batch * w.N * s + 4 * (w.dim * w.N + 2 * w.dim)


def a_variant(dim: int, N: int, kind: str, device, seed: int = 4325) -> torch.Tensor:
    """A (dim, N) other than the S4D-Real initialisation A[d, n] = -(n + 1):
    'structured' scales each channel's row by a log-uniform factor in
    [1/2, 2] (A[d, n] = (n + 1) A[d, 0], the structured arithmetic);
    'generic' multiplies every entry by exp(N(0, 1/4)), as a trained A drifts
    from its initialisation (no structure: one exp per state element)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    base = -torch.arange(1, N + 1, dtype=torch.float32).repeat(dim, 1)
    if kind == "structured":
        s = torch.exp((torch.rand(dim, 1, generator=g) * 2.0 - 1.0) * math.log(2.0))
        A = base * s
    else:
        A = base * torch.exp(0.5 * torch.randn(dim, N, generator=g))
    return A.contiguous().to(device)


def run_a_leg(w, x, device, peaks, kind, steps=10):
    """The benchmark workload with another A (see a_variant): forward and
    backward timed per call with CUDA events."""
    from selective_state_space_21_b200 import scan

    A = a_variant(w.dim, w.N, kind, device)
    y = torch.empty_like(x["u"])
    g = {k: torch.empty_like(x[k]) for k in ("u", "delta", "z", "B", "C")}
    f32 = dict(device=device, dtype=torch.float32)
    dA, dD, db = torch.empty(w.dim, w.N, **f32), torch.empty(w.dim, **f32), torch.empty(w.dim, **f32)

    def fwd():
        scan.mamba_scan_fwd(x["u"], x["delta"], x["delta_bias"], A, x["B"], x["C"], x["D"],
                            x["z"], y, None)

    def bwd():
        scan.mamba_scan_bwd(x["u"], x["delta"], x["delta_bias"], A, x["B"], x["C"], x["D"],
                            x["z"], x["dy"], g["u"], g["delta"], dA, g["B"], g["C"], dD, g["z"],
                            db)

    for _ in range(3):
        fwd()
        bwd()
    torch.cuda.synchronize(device)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record()
        fwd()
        ev[k][1].record()
        bwd()
        ev[k][2].record()
    torch.cuda.synchronize(device)
    if scan.mamba_scan_stream_status() != 0:
        raise RuntimeError(f"device error in the {kind}-A run")
    fms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    bms = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
    fb, bb = fwd_bytes(w), bwd_bytes(w)
    hbm = peaks["hbm_gbs"]
    return {"fwd": {"ms": round(fms, 4), "gbs": round(fb / (fms * 1e-3) / 1e9, 1),
                    "frac_hbm": round(fb / (fms * 1e-3) / 1e9 / hbm, 4),
                    "tc_per_s": w.token_channels / (fms * 1e-3)},
            "bwd": {"ms": round(bms, 4), "gbs": round(bb / (bms * 1e-3) / 1e9, 1),
                    "frac_hbm": round(bb / (bms * 1e-3) / 1e9 / hbm, 4),
                    "tc_per_s": w.token_channels / (bms * 1e-3)},
            "A": {"structured": "A[d, n] = -(n + 1) s_d, s_d log-uniform in [1/2, 2]",
                  "generic": "A[d, n] = -(n + 1) exp(e_dn), e_dn ~ N(0, 1/4)"}[kind],
            "arithmetic": "structured (one expm1 per step)" if kind == "structured"
            else "generic (one exp per state element)",
            "steps": steps, "timing": "median of per-call CUDA events"}


def run_conv(w, x, device, peaks, steps=10, pair=True):
    """The same workload with the block's convolution prologue (width 4):
    the training pair mamba_conv_scan_fwd_save / _bwd_saved (pair=False: the
    plain calls) on x in place of u (u = SiLU(conv(x)) is made inside the
    scan kernels).  Times each call with CUDA events; the bytes are the
    algorithmic ones of the plain scan plus the filter."""
    from selective_state_space_21_b200 import scan
    from selective_state_space_21_b200.inputs import make_conv_params

    cp = make_conv_params(w.dim, 4, device=device, seed=4321)
    y = torch.empty_like(x["u"])
    g = {k: torch.empty_like(x[k]) for k in ("u", "delta", "z", "B", "C")}
    f32 = dict(device=device, dtype=torch.float32)
    dcw, dcb = torch.empty(w.dim, 4, **f32), torch.empty(w.dim, **f32)
    dA, dD, db = torch.empty(w.dim, w.N, **f32), torch.empty(w.dim, **f32), torch.empty(w.dim, **f32)
    nsaved = scan.conv_saved_bytes(w.batch, w.dim, w.L, w.N, 4, w.dtype) if pair else 0
    saved = torch.empty(nsaved, device=device, dtype=torch.uint8) if nsaved else None

    def fwd():
        if pair:
            scan.mamba_conv_scan_fwd_save(x["u"], cp["conv_w"], cp["conv_b"], x["delta"],
                                          x["delta_bias"], x["A"], x["B"], x["C"], x["D"], x["z"],
                                          y, None, saved)
        else:
            scan.mamba_conv_scan_fwd(x["u"], cp["conv_w"], cp["conv_b"], x["delta"],
                                     x["delta_bias"], x["A"], x["B"], x["C"], x["D"], x["z"], y,
                                     None)

    def bwd():
        if pair:
            scan.mamba_conv_scan_bwd_saved(x["u"], cp["conv_w"], cp["conv_b"], x["delta"],
                                           x["delta_bias"], x["A"], x["B"], x["C"], x["D"],
                                           x["z"], x["dy"], g["u"], dcw, dcb, g["delta"], dA,
                                           g["B"], g["C"], dD, g["z"], db, saved)
        else:
            scan.mamba_conv_scan_bwd(x["u"], cp["conv_w"], cp["conv_b"], x["delta"],
                                     x["delta_bias"], x["A"], x["B"], x["C"], x["D"], x["z"],
                                     x["dy"], g["u"], dcw, dcb, g["delta"], dA, g["B"], g["C"], dD,
                                     g["z"], db)

    for _ in range(3):
        fwd()
        bwd()
    torch.cuda.synchronize(device)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record()
        fwd()
        ev[k][1].record()
        bwd()
        ev[k][2].record()
    torch.cuda.synchronize(device)
    if scan.mamba_scan_stream_status() != 0:
        raise RuntimeError("device error in the convolution-prologue run")
    fms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    bms = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
    extra = 4 * (w.dim * 4 + w.dim)
    fb, bb = fwd_bytes(w) + extra, bwd_bytes(w) + 2 * extra
    hbm = peaks["hbm_gbs"]
    return {"fwd": {"ms": round(fms, 4), "gbs": round(fb / (fms * 1e-3) / 1e9, 1),
                    "frac_hbm": round(fb / (fms * 1e-3) / 1e9 / hbm, 4),
                    "tc_per_s": w.token_channels / (fms * 1e-3)},
            "bwd": {"ms": round(bms, 4), "gbs": round(bb / (bms * 1e-3) / 1e9, 1),
                    "frac_hbm": round(bb / (bms * 1e-3) / 1e9 / hbm, 4),
                    "tc_per_s": w.token_channels / (bms * 1e-3)},
            "steps": steps, "width": 4, "timing": "median of per-call CUDA events",
            "calls": ("mamba_conv_scan_fwd_save + mamba_conv_scan_bwd_saved" if pair
                      else "mamba_conv_scan_fwd + mamba_conv_scan_bwd"),
            "shape": f"x in place of u, batch {w.batch} x dim {w.dim} x L {w.L}, N {w.N}"}


def run_dtproj(w, x, device, steps=10, pair=True):
    """The same workload with the low-rank Delta projection of rank
    ceil(d_model / 16) = ceil(dim / 32): the training pair
    mamba_dtproj_scan_fwd_save / _bwd_saved (pair=False: mamba_dtproj_scan_fwd
    / _bwd) takes dt_low (batch, R, L) and W_dt (dim, R) in place of delta.
    Times each call with CUDA events; the projection's own share is the
    difference to the plain scan's calls of the same kind, timed alongside."""
    from selective_state_space_21_b200 import scan
    from selective_state_space_21_b200.inputs import make_dtproj_params

    R = -(-w.dim // 32)
    pp = make_dtproj_params(w.batch, w.dim, w.L, R, w.dtype, device=device, seed=4322)
    y = torch.empty_like(x["u"])
    g = {k: torch.empty_like(x[k]) for k in ("u", "z", "B", "C", "delta")}
    f32 = dict(device=device, dtype=torch.float32)
    ddl = torch.empty_like(pp["dt_low"])
    dW = torch.empty(w.dim, R, **f32)
    dA, dD, db = torch.empty(w.dim, w.N, **f32), torch.empty(w.dim, **f32), torch.empty(w.dim, **f32)

    def buf(n):
        return torch.empty(n, device=device, dtype=torch.uint8) if n else None

    psaved = buf(scan.dtproj_saved_bytes(w.batch, w.dim, w.L, w.N, R, w.dtype)) if pair else None
    ssaved = buf(scan.saved_bytes(w.batch, w.dim, w.L, w.N, w.dtype)) if pair else None

    def fwd():
        args = (x["u"], pp["dt_low"], pp["W_dt"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"],
                x["z"], y, None)
        if pair:
            scan.mamba_dtproj_scan_fwd_save(*args, psaved)
        else:
            scan.mamba_dtproj_scan_fwd(*args)

    def bwd():
        args = (x["u"], pp["dt_low"], pp["W_dt"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"],
                x["z"], x["dy"], g["u"], ddl, dW, dA, g["B"], g["C"], dD, g["z"], db)
        if pair:
            scan.mamba_dtproj_scan_bwd_saved(*args, psaved)
        else:
            scan.mamba_dtproj_scan_bwd(*args)

    def fwd_plain():
        args = (x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"], x["z"], y,
                None)
        if pair:
            scan.mamba_scan_fwd_save(*args, ssaved)
        else:
            scan.mamba_scan_fwd(*args)

    def bwd_plain():
        args = (x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"], x["D"], x["z"],
                x["dy"], g["u"], g["delta"], dA, g["B"], g["C"], dD, g["z"], db)
        if pair:
            scan.mamba_scan_bwd_saved(*args, ssaved)
        else:
            scan.mamba_scan_bwd(*args)

    def timed(fns):
        for _ in range(3):
            for f in fns:
                f()
        torch.cuda.synchronize(device)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
              for _ in range(steps)]
        for k in range(steps):
            for i, f in enumerate(fns):
                ev[k][i].record()
                f()
            ev[k][-1].record()
        torch.cuda.synchronize(device)
        return [statistics.median(e[i].elapsed_time(e[i + 1]) for e in ev)
                for i in range(len(fns))]

    fms, bms, fpl, bpl = timed([fwd, bwd, fwd_plain, bwd_plain])
    if scan.mamba_scan_stream_status() != 0:
        raise RuntimeError("device error in the projection run")
    calls = ("mamba_dtproj_scan_fwd_save + mamba_dtproj_scan_bwd_saved "
             "(plain: mamba_scan_fwd_save + mamba_scan_bwd_saved)" if pair
             else "mamba_dtproj_scan_fwd + mamba_dtproj_scan_bwd "
                  "(plain: mamba_scan_fwd + mamba_scan_bwd)")
    return {"rank": R, "fwd_ms": round(fms, 4), "bwd_ms": round(bms, 4),
            "plain_fwd_ms": round(fpl, 4), "plain_bwd_ms": round(bpl, 4),
            "projection_fwd_ms": round(fms - fpl, 4), "projection_bwd_ms": round(bms - bpl, 4),
            "fwd_tc_per_s": w.token_channels / (fms * 1e-3),
            "bwd_tc_per_s": w.token_channels / (bms * 1e-3), "steps": steps,
            "saved_bytes": psaved.numel() if psaved is not None else 0, "calls": calls,
            "timing": "median of per-call CUDA events",
            "shape": f"dt_low (batch {w.batch}, R {R}, L {w.L}), W_dt ({w.dim}, {R})"}


def run_cplx(w, device, peaks, steps=3, pair=True):
    """The workload's shape with a complex diagonal A (S4D-Lin) of N complex
    states, complex B and C: the training pair mamba_cplx_scan_fwd_save /
    _bwd_saved (pair=False: the plain calls), timed per call with CUDA events.
    Bytes: the real scan's plus the doubled B, C (and dB, dC) rows."""
    from selective_state_space_21_b200 import scan
    from selective_state_space_21_b200.inputs import make_cplx_inputs

    x = make_cplx_inputs(w.batch, w.dim, w.L, w.N, w.dtype, device=device, seed=4323,
                         with_dy=True)
    f32 = dict(device=device, dtype=torch.float32)
    y = torch.empty_like(x["u"])
    g = {k: torch.empty_like(x[k]) for k in ("u", "delta", "z", "B", "C")}
    dA = torch.empty(w.dim, 2 * w.N, **f32)
    dD, db = torch.empty(w.dim, **f32), torch.empty(w.dim, **f32)
    saved = (torch.empty(scan.cplx_saved_bytes(w.batch, w.dim, w.L, w.N, w.dtype), device=device,
                         dtype=torch.uint8) if pair else None)

    def fwd():
        if pair:
            scan.mamba_cplx_scan_fwd_save(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"],
                                          x["C"], x["D"], x["z"], y, None, saved)
        else:
            scan.mamba_cplx_scan_fwd(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                     x["D"], x["z"], y, None)

    def bwd():
        if pair:
            scan.mamba_cplx_scan_bwd_saved(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"],
                                           x["C"], x["D"], x["z"], x["dy"], g["u"], g["delta"], dA,
                                           g["B"], g["C"], dD, g["z"], db, saved)
        else:
            scan.mamba_cplx_scan_bwd(x["u"], x["delta"], x["delta_bias"], x["A"], x["B"], x["C"],
                                     x["D"], x["z"], x["dy"], g["u"], g["delta"], dA, g["B"],
                                     g["C"], dD, g["z"], db)

    fwd()
    bwd()
    torch.cuda.synchronize(device)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record()
        fwd()
        ev[k][1].record()
        bwd()
        ev[k][2].record()
    torch.cuda.synchronize(device)
    if scan.mamba_scan_stream_status() != 0:
        raise RuntimeError("device error in the complex-A run")
    fms = statistics.median(e[0].elapsed_time(e[1]) for e in ev)
    bms = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
    s_io = w.io_bytes
    bc = 2 * w.batch * (2 * w.N) * w.L * s_io
    fb = 4 * s_io * w.token_channels + bc + 4 * (w.dim * 2 * w.N + 2 * w.dim)
    bb = 7 * s_io * w.token_channels + 2 * bc + 8 * (w.dim * 2 * w.N + 2 * w.dim)
    hbm = peaks["hbm_gbs"]
    return {"fwd": {"ms": round(fms, 4), "gbs": round(fb / (fms * 1e-3) / 1e9, 1),
                    "frac_hbm": round(fb / (fms * 1e-3) / 1e9 / hbm, 4),
                    "tc_per_s": w.token_channels / (fms * 1e-3)},
            "bwd": {"ms": round(bms, 4), "gbs": round(bb / (bms * 1e-3) / 1e9, 1),
                    "frac_hbm": round(bb / (bms * 1e-3) / 1e9 / hbm, 4),
                    "tc_per_s": w.token_channels / (bms * 1e-3)},
            "steps": steps, "timing": "median of per-call CUDA events",
            "calls": ("mamba_cplx_scan_fwd_save + mamba_cplx_scan_bwd_saved" if pair
                      else "mamba_cplx_scan_fwd + mamba_cplx_scan_bwd"),
            "shape": f"batch {w.batch} x dim {w.dim} x L {w.L}, {w.N} complex states"}


def run_decode(w, x, device, peaks, steps=200):
    """One token per batch row through mamba_scan_step, repeated `steps` times
    on the workload's channels (a decoding loop after a prefill)."""
    from selective_state_space_21_b200 import scan

    tok = {k: x[k][:, :, 0].contiguous() for k in ("u", "delta", "z", "B", "C")}
    state = torch.zeros(w.batch, w.dim, w.N, device=device)
    y = torch.empty_like(tok["u"])

    def step():
        scan.mamba_scan_step(state, tok["u"], tok["delta"], x["delta_bias"], x["A"], tok["B"],
                             tok["C"], x["D"], tok["z"], y)

    for _ in range(10):
        step()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize(device)
    if scan.mamba_scan_stream_status() != 0:
        raise RuntimeError("device error in the decoding loop")
    ms = e0.elapsed_time(e1) / steps
    nb = decode_bytes(w)
    gbs = nb / (ms * 1e-3) / 1e9
    out = {"us_per_token_step": round(ms * 1e3, 3), "tokens_per_s": w.batch / (ms * 1e-3),
           "bytes_per_step": nb, "gbs": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
           "steps": steps, "launch": "eager (host-side argument checks every call)",
           "shape": f"batch {w.batch} x dim {w.dim} x N {w.N}, one token per row"}
    # The same loop through a decoding plan: the pointer checks are made once
    # when the plan is created, and each token is a single kernel launch.
    try:
        plan = scan.StepPlan(state, tok["u"], tok["delta"], x["delta_bias"], x["A"], tok["B"],
                             tok["C"], x["D"], tok["z"], y)
        for _ in range(10):
            plan.run()
        torch.cuda.synchronize(device)
        e0.record()
        for _ in range(steps):
            plan.run()
        e1.record()
        torch.cuda.synchronize(device)
        pms = e0.elapsed_time(e1) / steps
        plan.close()
        pgbs = nb / (pms * 1e-3) / 1e9
        out["plan"] = {"us_per_token_step": round(pms * 1e3, 3),
                       "tokens_per_s": w.batch / (pms * 1e-3), "gbs": round(pgbs, 1),
                       "frac_hbm": round(pgbs / peaks["hbm_gbs"], 4),
                       "launch": "eager, one launch per token (checks made once per plan)"}
    except Exception as e:
        out["plan"] = {"unavailable": str(e)[:200]}
    # The same loop replayed from a CUDA graph (how a decoding loop is usually
    # run): device time per step without the per-call host work.
    try:
        s_cap = torch.cuda.Stream(device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s_cap):
            step()
            torch.cuda.synchronize(device)
            with torch.cuda.graph(graph, stream=s_cap):
                for _ in range(steps):
                    step()
        graph.replay()
        torch.cuda.synchronize(device)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize(device)
        gms = e0.elapsed_time(e1) / steps
        ggbs = nb / (gms * 1e-3) / 1e9
        out["graph"] = {"us_per_token_step": round(gms * 1e3, 3),
                        "tokens_per_s": w.batch / (gms * 1e-3), "gbs": round(ggbs, 1),
                        "frac_hbm": round(ggbs / peaks["hbm_gbs"], 4)}
    except Exception as e:  # capture not possible here: report the eager loop only
        out["graph"] = {"unavailable": str(e)[:200]}
    return out


def time_calls(fn, device, steps=10) -> dict:
    """Median of per-call CUDA-event times of fn() after three warm-up calls."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize(device)
    times = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize(device)
        times.append(e0.elapsed_time(e1))
    return {"ms": round(statistics.median(times), 4), "steps": steps,
            "timing": "median of per-call CUDA events"}


def run_e2e(args, w, x, y, g, fwd, bwd, device, world, pair=False):
    """Same step through the public API with host buffers: each step copies its
    inputs from pinned host memory to the device and reads every result back.
    Steps are pipelined the way a user would: copy-in, compute and copy-out run
    on three streams over two device buffer sets, so step i+1's inputs travel
    while step i computes and step i-1's results come back (PCIe is
    full-duplex)."""
    from selective_state_space_21_b200 import scan

    names_in = ["u", "delta", "z", "B", "C", "A", "D", "delta_bias", "dy"]
    host_in = {k: x[k].cpu().pin_memory() for k in names_in}
    out_like = {"y": y, **g}
    host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                for k, v in out_like.items()}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    slots = [({k: torch.empty_like(x[k]) for k in names_in},
              {k: torch.empty_like(v) for k, v in out_like.items()}) for _ in range(2)]
    nsaved = scan.saved_bytes(w.batch, w.dim, w.L, w.N, w.dtype) if pair else 0
    saved = [torch.empty(nsaved, device=device, dtype=torch.uint8) if nsaved else None
             for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_ready = [ev(), ev()]
    comp_done = [ev(), ev()]
    out_done = [ev(), ev()]
    started = [False, False]

    def step(i):
        k = i % 2
        xi, oi = slots[k]
        with torch.cuda.stream(s_in):
            if started[k]:
                s_in.wait_event(comp_done[k])  # the kernels of step i-2 read this slot
            for n in names_in:
                xi[n].copy_(host_in[n], non_blocking=True)
            in_ready[k].record(s_in)
        s_comp.wait_event(in_ready[k])
        if started[k]:
            s_comp.wait_event(out_done[k])  # step i-2's results have left this slot
        if pair:
            scan.mamba_scan_fwd_save(xi["u"], xi["delta"], xi["delta_bias"], xi["A"], xi["B"],
                                     xi["C"], xi["D"], xi["z"], oi["y"], None, saved[k],
                                     stream=s_comp)
            scan.mamba_scan_bwd_saved(xi["u"], xi["delta"], xi["delta_bias"], xi["A"], xi["B"],
                                      xi["C"], xi["D"], xi["z"], xi["dy"], oi["du"], oi["ddelta"],
                                      oi["dA"], oi["dB"], oi["dC"], oi["dD"], oi["dz"], oi["dbias"],
                                      saved[k], stream=s_comp)
        else:
            scan.mamba_scan_fwd(xi["u"], xi["delta"], xi["delta_bias"], xi["A"], xi["B"],
                                xi["C"], xi["D"], xi["z"], oi["y"], None, stream=s_comp)
            scan.mamba_scan_bwd(xi["u"], xi["delta"], xi["delta_bias"], xi["A"], xi["B"],
                                xi["C"], xi["D"], xi["z"], xi["dy"], oi["du"], oi["ddelta"],
                                oi["dA"], oi["dB"], oi["dC"], oi["dD"], oi["dz"], oi["dbias"],
                                stream=s_comp)
        comp_done[k].record(s_comp)
        s_out.wait_event(comp_done[k])
        with torch.cuda.stream(s_out):
            for n, v in oi.items():
                host_out[n].copy_(v, non_blocking=True)
            out_done[k].record(s_out)
        started[k] = True

    for i in range(2):
        step(i)
    torch.cuda.synchronize(device)
    K = max(3, min(args.steps, 10))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    t0.record(s_in)
    for i in range(K):
        step(i)
    s_out.wait_event(comp_done[(K - 1) % 2])
    t1.record(s_out)  # after the last read-back
    torch.cuda.synchronize(device)
    barrier(device)
    if scan.mamba_scan_stream_status(s_comp) != 0:
        raise RuntimeError("device error in the end-to-end run")
    ms = max_over_ranks(t0.elapsed_time(t1) / K, device)
    return {"value": w.token_channels * world / (ms * 1e-3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "steps": K, "pipelined": "copy-in / compute / copy-out on three streams"}


def run_reference(args, world, rank):
    """The fp64 CPU oracle as it stands, on the host cores, over bounded channel
    samples of the same workload (one sample per step)."""
    import oracle
    w = WORKLOADS[args.workload]
    x = make_inputs(w.batch, w.dim, w.L, w.N, w.dtype, device="cpu",
                    seed=1234 + args.workload, has_z=w.has_z, has_D=w.has_D, with_dy=True)
    threads = args.cpu_threads or oracle.default_threads()
    k = max(8, 2 * threads)

    def step(d0):
        idx = torch.tensor([(d0 + i) % w.dim for i in range(k)])
        sub = {n: x[n][0:1].index_select(1, idx).contiguous() for n in ("u", "delta", "z", "dy")}
        A, D, bias = x["A"][idx].contiguous(), x["D"][idx].contiguous(), \
            x["delta_bias"][idx].contiguous()
        oracle.s6_forward(sub["u"], sub["delta"], A, x["B"][0:1], x["C"][0:1], bias, D,
                          sub["z"], nthreads=threads)
        oracle.s6_backward(sub["u"], sub["delta"], A, x["B"][0:1], x["C"][0:1], sub["dy"],
                           bias, D, sub["z"], nthreads=threads)

    for i in range(args.warmup):
        step(i * k)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step((args.warmup + i) * k)
    el = time.perf_counter() - t0
    per = el / args.steps
    value = k * w.L / per
    desc = (f"each step: forward + backward of {k} channels of batch row 0 (full L = {w.L}) "
            f"of {w.name}")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(w, args.step),
                   "batch": w.batch, "dim": w.dim, "L": w.L, "N": w.N,
                   "io_dtype": "bf16" if w.dtype == torch.bfloat16 else "fp32"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD,
                    help="index into the workload list (default: the bf16 2K-length one)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--step", choices=["pair", "recompute"], default="pair",
                    help="the training step: the pair whose forward saves the 16-step states for "
                         "its backward (default), or forward + the backward that re-runs it")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="threads of the oracle in the reference arm (0: all host cores)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-conv", action="store_true",
                    help="skip the convolution-prologue timing")
    ap.add_argument("--conv-steps", type=int, default=10,
                    help="timed calls of the convolution-prologue and projection legs")
    ap.add_argument("--no-dtproj", action="store_true",
                    help="skip the Delta-projection timing")
    ap.add_argument("--no-cplx", action="store_true", help="skip the complex-A timing")
    ap.add_argument("--no-a-legs", action="store_true",
                    help="skip the structured-A and generic-A timings")
    ap.add_argument("--no-micro", action="store_true",
                    help="skip the instruction-throughput microbenchmark (the FP32 roofline "
                         "then uses the nominal peak)")
    ap.add_argument("--micro", action="store_true",
                    help="run only the instruction-throughput microbenchmark and print it")
    ap.add_argument("--only", choices=["fwd", "bwd", "cplx", "dtproj"], default=None,
                    help="time one pass, or the complex-A or projection calls, only (for "
                         "profiling; not a benchmark result)")
    ap.add_argument("--cplx-batch", type=int, default=0,
                    help="batch of the calls with --only cplx / dtproj (0: the workload's)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world, rank, local = dist_env()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world, rank)), flush=True)
        return 0

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.micro:
        if rank == 0:
            print(json.dumps({"micro": run_micro(local)}), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    try:
        result = run_ours(args, world, rank, device)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
