"""FLARE forward throughput on B200 (tokens/s) with roofline and baselines.

One step = one FLARE forward (encode partials -> combine -> decode) over the
million-token workload: B=1, H=16, N=1,048,576, M=256, D=32, bf16 inputs,
float32 accumulation, scale 1/sqrt(D), synthetic N(0,1) inputs (seed = rank).
Inputs (3 GiB of K, V, Y) exceed the 126 MB L2, so no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 (torchrun, one process per GPU) each rank runs an independent
problem of the same size (weak scaling, no data-path collective); rank 0
prints one JSON line with the job-wide tokens/s over the max time across
ranks.  ``--impl reference`` times the double-precision CPU oracle (the only
reference available for this method) on a bounded sample of the workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from flare_inputs import WORKLOADS, make_inputs  # noqa: E402

WORKLOAD = WORKLOADS["c3_fwd_bf16_1M"]
METRIC = "FLARE fwd tokens/s at N=1M, M=256, H=16, D=32 bf16; % of roofline"

# The exponential ceilings come from the unit-rate probe the library carries
# (flare_probe_unit_rates, run at the start of every bench): MUFU ex2 results
# and packed fp32 FMAs per SM per clock, times the SM count and the max SM
# clock.  Nominal B200 figures (148 SMs, 16 ex2 and 128 FMAs per clock per
# SM) stand in only if the probe cannot run.  The HBM and tensor ceilings
# come from MEASURED_PEAKS.json.
NOMINAL_RATES = {"sms": 148, "ex2_per_clk_sm": 16.0, "fma_per_clk_sm": 128.0,
                 "fma2_per_clk_sm": 128.0}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}
# fp32 FMA-pipe operations per softmax weight, counted from the kernels'
# softmax loops: the scale-and-shift FMA and the row-sum add of every
# weight; a weight computed by the polynomial adds the three adds of its
# range reduction and the three FMAs of its Horner steps.  (The clamp, the
# exponent-field add and the bf16 packing run on the integer/ALU pipe.)
FMA_OPS_BASE = 2.0
FMA_OPS_POLY = 6.0

THROTTLE_BAD = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, out_path: str | None = None):
        self.gpu_index = gpu_index
        self.proc = None
        self.out_path = out_path

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        if self.out_path:
            with open(self.out_path, "w") as f:
                f.write(out)
        return self.parse(out)

    @staticmethod
    def parse(text: str):
        sms, maxes, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in text.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes),
                "reasons": sorted(reasons), "samples": len(sms)}


# ------------------------------------------------------------- distributed

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def dist_max(value: float, world: int, device) -> float:
    """Max of a host float over ranks (one tiny all-reduce; no data path)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_done(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# -------------------------------------------------------------- CPU oracle

def oracle_sample_rate(target_s: float, w=WORKLOAD, seed: int = 0):
    """Times the oracle's FLARE forward on a bounded sample of the workload:
    h_s of its heads with n_s of their N tokens each (same M, D, dtype
    rounding), sized so the timed run takes about target_s seconds (a whole
    head first, then more heads).  Returns (tokens/s of the full workload,
    description, cores, n_s, h_s).  A workload token carries H heads, so one
    head-token is 1/H of a token."""
    import oracle
    cores = oracle.num_threads()

    def run(h_s, n_s):
        x = make_inputs(1, h_s, n_s, w.M, w.D, dtype=w.torch_dtype, seed=seed)
        t0 = time.perf_counter()
        oracle.flare_fwd(x["Q"], x["K"], x["V"], w.scale)
        return time.perf_counter() - t0

    n_cal = 4096
    t_cal = max(run(1, n_cal), 1e-4)
    n_s = int(min(w.N, max(n_cal, n_cal * target_s / t_cal)))
    h_s = 1
    if n_s == w.N:
        h_s = int(max(1, min(w.B * w.H, target_s / (t_cal * w.N / n_cal))))
    t = run(h_s, n_s)
    rate = (h_s * n_s / w.H) / t
    desc = (f"oracle FLARE fwd (double, OpenMP) on {h_s} of {w.B * w.H} heads x {n_s} of "
            f"{w.N} tokens, M={w.M}, D={w.D}; {t:.2f} s; tokens/s counts 1/H token per "
            f"head-token")
    return rate, desc, cores, n_s, h_s


# ------------------------------------------------------------------ ours

def workload_from_args(args):
    """The headline workload, or a smaller one of the same per-head shape for
    profiling captures (--heads / --seq)."""
    import dataclasses
    w = WORKLOAD
    if args.heads or args.seq:
        w = dataclasses.replace(w, name=w.name + "_reduced", H=args.heads or w.H, N=args.seq or w.N)
    return w


def measure_unit_rates():
    """The library's unit-rate probe on the current device, or the nominal
    B200 figures (marked as such) if it fails."""
    import rank_latent_attention_flare_b200 as fl
    try:
        r = fl.probe_unit_rates()
        r["source"] = "flare_probe_unit_rates, this run"
        return r
    except Exception as e:   # noqa: BLE001 -- reported, nominal figures used instead
        r = dict(NOMINAL_RATES)
        r["source"] = f"nominal (probe failed: {str(e)[:120]})"
        return r


def exp_ceiling(exps: float, poly: float, rates: dict, clk_hz: float):
    """Time floor of `exps` softmax weights of which a share `poly` runs as
    the FMA-pipe polynomial and the rest on the MUFU: the slower of the two
    units at its measured rate.  Returns (seconds, binding unit)."""
    sms = rates["sms"]
    mufu = rates["ex2_per_clk_sm"] * sms * clk_hz
    fma = max(rates["fma_per_clk_sm"], rates["fma2_per_clk_sm"]) * sms * clk_hz
    t_mufu = exps * (1.0 - poly) / mufu
    t_fma = exps * (FMA_OPS_BASE + FMA_OPS_POLY * poly) / fma
    return (t_mufu, "mufu") if t_mufu >= t_fma else (t_fma, "fma")


def roofline_entry(kernel_ms: dict, peaks: dict, peak_kind: str, rates: dict, w=WORKLOAD):
    """Roofline of the dominant kernel (largest average duration), and of
    the whole forward.

    Both forward kernels are bound by exponentials: each computes B*H*N*M
    of them per launch (encode: softmax over tokens of every latent row;
    decode: softmax over latents of every token), a fixed share of them as
    a polynomial on the FMA pipe (flare_exp_split).  The ceiling is the
    combined MUFU + FMA one for that share (exp_ceiling), so moving
    exponentials to the polynomial cannot lift the fraction past 1; the
    MUFU-only figure and the tensor-pipe and HBM fractions are reported
    alongside.
    """
    import rank_latent_attention_flare_b200 as fl
    name = max(("encode", "decode"), key=lambda k: kernel_ms[k])
    exps = w.B * w.H * w.N * w.M
    clk = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    mufu_peak = rates["ex2_per_clk_sm"] * rates["sms"] * clk / 1e9   # Gexp/s
    ceil = {}
    for k, kid in (("encode", 0), ("decode", 1)):
        poly = fl.exp_split(kid, w.M, w.D, w.torch_dtype)
        t_c, unit = exp_ceiling(exps, poly, rates, clk)
        ceil[k] = {"poly_share": round(poly, 4), "t_ceiling_ms": round(t_c * 1e3, 4),
                   "binding_unit": unit, "peak_gexps": round(exps / t_c / 1e9, 1)}
    t = kernel_ms[name] / 1e3
    achieved = exps / t / 1e9
    peak = ceil[name]["peak_gexps"]
    flops = 4 * w.B * w.H * w.N * w.M * w.D
    hbm_bytes = 2 * w.B * w.H * w.N * w.D * 2   # encode: K and V read; decode: K read, Y written
    t_fwd = sum(kernel_ms.values()) / 1e3
    t_fwd_ceil = sum(c["t_ceiling_ms"] for c in ceil.values()) / 1e3
    # context: the share at which the two units bind together, whose floor no
    # split of the exponentials between them can beat
    mufu_r = rates["ex2_per_clk_sm"]
    fma_r = max(rates["fma_per_clk_sm"], rates["fma2_per_clk_sm"])
    phi_b = (fma_r - FMA_OPS_BASE * mufu_r) / (fma_r + FMA_OPS_POLY * mufu_r)
    t_b, _ = exp_ceiling(exps, phi_b, rates, clk)
    entry = {
        "bound": "alu", "kernel": f"flare_{name}", "achieved": round(achieved, 1),
        "peak": peak, "unit": "Gexp/s", "frac": round(achieved / peak, 4),
        "traffic": read_traffic(name),
        "peak_basis": (f"combined MUFU + FMA exponential ceiling at the kernel's polynomial share "
                       f"{ceil[name]['poly_share']:.4f}: max((1-share)/MUFU, "
                       f"({FMA_OPS_BASE:g} + {FMA_OPS_POLY:g} share)/FMA) per weight; MUFU "
                       f"{rates['ex2_per_clk_sm']:.2f} ex2/clk/SM, FMA "
                       f"{max(rates['fma_per_clk_sm'], rates['fma2_per_clk_sm']):.1f}/clk/SM "
                       f"({rates['source']}) x {rates['sms']} SMs x {clk / 1e6:.0f} MHz"),
        "mufu_only": {"peak": round(mufu_peak, 1), "frac": round(achieved / mufu_peak, 4)},
        "best_split": {"poly_share": round(phi_b, 4), "t_ceiling_ms": round(t_b * 1e3, 4),
                       "frac": round(t_b / t, 4),
                       "forward_frac": round(2 * t_b / t_fwd, 4)},
        "kernels": ceil,
        "forward": {"t_ms": round(t_fwd * 1e3, 4), "t_ceiling_ms": round(t_fwd_ceil * 1e3, 4),
                    "frac": round(t_fwd_ceil / t_fwd, 4)},
        "unit_rates": {k: (round(v, 3) if isinstance(v, float) else v) for k, v in rates.items()},
        "algorithmic": {"exps": exps, "tensor_flops": flops, "hbm_bytes": hbm_bytes},
        "other_ceilings": {
            "tensor_frac": round(flops / t / 1e12 / float(peaks["bf16_tflops"]), 4),
            "hbm_frac": round(hbm_bytes / t / 1e9 / float(peaks["hbm_gbs"]), 4),
            "peaks": f"{peak_kind}: bf16 {peaks['bf16_tflops']} TFLOP/s, "
                     f"HBM {peaks['hbm_gbs']} GB/s",
        },
    }
    return entry


def read_traffic(name: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        rec = d.get(name)
        if not rec:
            return None
        src = os.path.join(ROOT, rec["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if h != rec.get("source_sha256"):
            return None
        return rec["bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


def run_ours(args, rank, world, local):
    import torch

    import rank_latent_attention_flare_b200 as fl

    w = workload_from_args(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    rates = measure_unit_rates()
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=rank)
    g = {k: v.to(dev) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    Y = torch.empty_like(g["K"])
    st = torch.cuda.current_stream()

    def step(events=None):
        if events:
            events[0].record(st)
        fl.flare_encode(g["Q"], g["K"], g["V"], w.scale, workspace=ws)
        if events:
            events[1].record(st)
        fl.flare_combine(w.B, w.H, w.N, w.M, w.D, w.torch_dtype, workspace=ws)
        if events:
            events[2].record(st)
        fl.flare_decode(g["Q"], g["K"], w.scale, workspace=ws, out=Y)
        if events:
            events[3].record(st)

    # the clock sampler starts before the warm-up, so that no idle gap (while
    # nvidia-smi starts) separates the warm-up from the timed steps
    sampler = ClockSampler(local, os.path.join(args.out_dir, "clocks.csv") if args.out_dir else None) \
        if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.5)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fl.device_status(ws) != 0:
        raise RuntimeError("device wait ran out during warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    dist_barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(st)
    for i in range(args.steps):
        step(ev[i])
    t_end.record(st)
    torch.cuda.synchronize()
    dist_barrier(world)
    clocks = sampler.stop() if sampler else None
    if fl.device_status(ws) != 0:
        raise RuntimeError("device wait ran out in the timed region")

    ms_total = t_start.elapsed_time(t_end)
    ms_total = dist_max(ms_total, world, dev)
    kernel_ms = {
        "encode": statistics.mean(e[0].elapsed_time(e[1]) for e in ev),
        "combine": statistics.mean(e[1].elapsed_time(e[2]) for e in ev),
        "decode": statistics.mean(e[2].elapsed_time(e[3]) for e in ev),
    }
    tokens_per_step = w.B * w.N
    value = world * tokens_per_step * args.steps / (ms_total / 1e3)

    # End to end through the public API: pinned host inputs -> device ->
    # forward -> result back to pinned host memory, every step, by the
    # library's host-memory call (flare_fwd_host: the heads' copies in on a
    # second stream, overlapped with the compute and the copies out).
    e2e = None
    if not args.no_e2e:
        hx = {k: v.pin_memory() for k, v in x.items()}
        hY = torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True)
        dX = {k: torch.empty_like(v) for k, v in g.items()}
        bufs = {"Q": dX["Q"], "K": dX["K"], "V": dX["V"], "Y": Y}
        wsh = torch.empty(int(fl.load().flare_fwd_host_workspace_size(
            w.B, w.H, w.N, w.M, w.D,
            fl.FLARE_BF16 if w.torch_dtype == torch.bfloat16 else fl.FLARE_F32)),
            dtype=torch.uint8, device=dev)
        copy_stream = torch.cuda.Stream(device=dev)
        e2e_steps = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            fl.flare_fwd_host(hx["Q"], hx["K"], hx["V"], w.scale, out=hY, device_buffers=bufs,
                              workspace=wsh, device=dev, stream=st, copy_stream=copy_stream)

        e2e_step()
        torch.cuda.synchronize()
        dist_barrier(world)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(e2e_steps):
            e2e_step()
        b.record(st)
        torch.cuda.synchronize()
        e2e_ms = dist_max(a.elapsed_time(b), world, dev)
        h2d = sum(hx[k].numel() * hx[k].element_size() for k in ("Q", "K", "V"))
        e2e = {"value": world * tokens_per_step * e2e_steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hY.numel() * hY.element_size(),
               "steps": e2e_steps}
        del hx, hY, dX

    peaks, peak_kind = load_peaks()
    roof = roofline_entry(kernel_ms, peaks, peak_kind, rates, w)

    rows = None
    context = None
    if not args.no_rows:
        del Y, ws
        g.clear()
        torch.cuda.empty_cache()
        rows = time_other_rows(dev, peaks, peak_kind, seed=rank, rates=rates)
        try:
            context = time_sdpa_context(dev, seed=rank)
        except (RuntimeError, ValueError) as e:   # a torch build without a kernel for this shape
            context = {"what": "two torch scaled_dot_product_attention calls", "error": str(e)[:200]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, cores, _, _ = oracle_sample_rate(args.cpu_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": desc}

    path = fl.fwd_path(w.B, w.H, w.N, w.M, w.D, w.torch_dtype)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"FLARE fwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16, "
                               "fp32 accumulate, scale 1/sqrt(D), i.i.d. N(0,1)",
                   "global_batch": w.B * world, "seq_len": w.N, "heads": w.H, "latents": w.M,
                   "head_dim": w.D, "parallelism": f"independent problems x{world}",
                   "l2": "inputs 3 GiB > 126 MB L2: no flush",
                   "kernels": "tcgen05" if path == 1 else "cuda-core"},
        "kernel_ms": {k: round(v, 4) for k, v in kernel_ms.items()},
        "roofline": roof,
        "rows": rows,
        "context_sdpa": context,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 3 * args.steps * world,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------- the other rows

_ROW_RATES = dict(NOMINAL_RATES, source="nominal")


def _fwd_exp_floor(exps_per_stage: float, M: int, D: int, peaks: dict, stages=(0, 1)) -> float:
    """Seconds the forward's exponentials need at least: each stage (0 =
    an encode, 1 = the decode) computes exps_per_stage weights, a share of
    them on the FMA-pipe polynomial (flare_exp_split), at the combined
    MUFU + FMA ceiling of that share."""
    import torch

    import rank_latent_attention_flare_b200 as fl
    clk = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    return sum(exp_ceiling(exps_per_stage, fl.exp_split(k, M, D, torch.bfloat16), _ROW_RATES, clk)[0]
               for k in stages)


def _row_roofline(t_ms: float, exps: float, flops: float, hbm_bytes: float, peaks: dict,
                  peak_kind: str, fwd_exp_s: float = 0.0, fwd_exps: float = 0.0):
    """Roofline of a whole row: the slowest of the exponential, tensor and
    HBM limits (each at its peak) over the measured time.  The exponential
    limit takes the forward's fwd_exps weights at their combined MUFU + FMA
    floor fwd_exp_s (the kernels' polynomial shares) and the remaining
    exps - fwd_exps (the backward's, all on the MUFU) at the probe's
    measured MUFU rate."""
    clk = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    mufu = _ROW_RATES["ex2_per_clk_sm"] * _ROW_RATES["sms"] * clk   # exp/s
    lim = {"exp": fwd_exp_s + (exps - fwd_exps) / mufu,
           "tensor": flops / (float(peaks["bf16_tflops"]) * 1e12),
           "hbm": hbm_bytes / (float(peaks["hbm_gbs"]) * 1e9)}
    bound = max(lim, key=lim.get)
    t = t_ms / 1e3
    return {"bound": bound, "t_roof_ms": round(lim[bound] * 1e3, 4),
            "frac": round(lim[bound] / t, 4),
            "exp_frac": round(lim["exp"] / t, 4), "tensor_frac": round(lim["tensor"] / t, 4),
            "hbm_frac": round(lim["hbm"] / t, 4),
            "algorithmic": {"exps": exps, "tensor_flops": flops, "hbm_bytes": hbm_bytes},
            "peaks": f"MUFU {mufu / 1e9:.0f} Gexp/s ({_ROW_RATES['source']}), {peak_kind} bf16 "
                     f"{peaks['bf16_tflops']} TFLOP/s, {peak_kind} HBM {peaks['hbm_gbs']} GB/s"}


def time_other_rows(dev, peaks, peak_kind, iters: int = 20, seed: int = 0,
                    which=("flare_fwd_c2", "flare_fwd_m64", "flare_pp_fwd", "flare_fwd_bwd",
                           "flare_fwd_bwd_m256",
                           "flare_pp_fwd_bwd", "flare_strided", "flare_varlen"), rates=None):
    """Times the FLARE++ forward (B=2 H=8 N=262,144 M=256 D=32) and the
    forward + backward of B=8 H=8 N=16,384 M=128 D=32, both bf16, on the
    same device with CUDA events (median of `iters` launches after 3
    warm-ups, L2 flushed before each by writing 256 MB)."""
    import torch

    import rank_latent_attention_flare_b200 as fl

    st = torch.cuda.current_stream()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if rates is not None:
        _ROW_RATES.update(rates)

    def timed(fn):
        for _ in range(3):
            fn()
        pairs = []
        for _ in range(iters):
            flush_buf.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(st)
            fn()
            b.record(st)
            pairs.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in pairs)

    rows = {}
    if "flare_fwd_c2" in which:
        rows.update(_time_c2(dev, peaks, peak_kind, timed, seed))
    if "flare_fwd_m64" in which:
        rows.update(_time_c2(dev, peaks, peak_kind, timed, seed, M=64, row="flare_fwd_m64"))
    if "flare_pp_fwd" in which:
        rows.update(_time_pp(dev, peaks, peak_kind, timed, seed))
    if "flare_fwd_bwd" in which:
        rows.update(_time_fwd_bwd(dev, peaks, peak_kind, timed, seed))
    if "flare_fwd_bwd_m256" in which:
        rows.update(_time_fwd_bwd(dev, peaks, peak_kind, timed, seed, M=256,
                                  row="flare_fwd_bwd_m256"))
    if "flare_pp_fwd_bwd" in which:
        rows.update(_time_pp_fwd_bwd(dev, peaks, peak_kind, timed, seed))
    if "flare_strided" in which:
        rows.update(_time_strided(dev, peaks, peak_kind, timed, seed))
    if "flare_varlen" in which:
        rows.update(_time_varlen(dev, peaks, peak_kind, timed, seed))
    del flush_buf
    torch.cuda.empty_cache()
    return rows


def _time_c2(dev, peaks, peak_kind, timed, seed, M=None, row="flare_fwd_c2"):
    """FLARE forward on the 256x256-mesh workload: B=4 H=8 N=65,536 M=128
    D=16 bf16 (64 MiB per token tensor, so the L2 is flushed before each
    launch), or the same with another latent count M (the flare_fwd_m64
    row: 64 latents, padded to the kernels' 128-row latent tile).  Roofline
    as the headline's: the combined exponential ceilings of its encode and
    decode at their polynomial shares for the M latents of the workload,
    beside the tensor and HBM fractions."""
    import dataclasses

    import torch

    import rank_latent_attention_flare_b200 as fl
    w = WORKLOADS["c2_fwd_bf16_mesh256"]
    if M is not None:
        w = dataclasses.replace(w, M=M)
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed)
    g = {k: v.to(dev) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    Y = torch.empty_like(g["K"])
    ms = timed(lambda: fl.flare_fwd(g["Q"], g["K"], g["V"], w.scale, workspace=ws, out=Y))
    if fl.device_status(ws) != 0:
        raise RuntimeError("device wait ran out in the mesh-sized forward")
    u = w.B * w.H * w.N
    exps = u * w.M
    t_ceil = _fwd_exp_floor(exps, w.M, w.D, peaks)
    roof = _row_roofline(ms, 2.0 * exps, 8.0 * u * w.M * w.D, 4.0 * u * w.D * 2, peaks,
                         peak_kind, t_ceil, 2.0 * exps)
    return {row: {
        "workload": f"FLARE fwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16 (mesh 256x256)",
        "fwd_path": fl.fwd_path(w.B, w.H, w.N, w.M, w.D, w.torch_dtype),
        "ms": round(ms, 4), "tokens_per_s": w.B * w.N / (ms / 1e3), "l2": "flushed (256 MB)",
        "roofline": roof}}


def _time_pp(dev, peaks, peak_kind, timed, seed):
    import rank_latent_attention_flare_b200 as fl
    rows = {}
    w = WORKLOADS["c4_ppfwd_bf16_256k"]
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed)
    g = {k: v.to(dev) for k, v in x.items()}
    ws = fl.alloc_workspace(fl.FLARE_OP_PP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    ms = timed(lambda: fl.flare_pp_fwd(g["Q"], g["K"], g["V"], w.scale, workspace=ws))
    if fl.device_status(ws) != 0:
        raise RuntimeError("device wait ran out in the FLARE++ forward")
    u = w.B * w.H * w.N
    rows["flare_pp_fwd"] = {
        "workload": f"FLARE++ fwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16",
        "ms": round(ms, 4), "tokens_per_s": w.B * w.N / (ms / 1e3),
        "roofline": _row_roofline(ms, 3.0 * u * w.M, 12.0 * u * w.M * w.D,
                                  6.0 * u * w.D * 2, peaks, peak_kind,
                                  _fwd_exp_floor(u * w.M, w.M, w.D, peaks, (0, 0, 1)),
                                  3.0 * u * w.M)}
    return rows


def _time_fwd_bwd(dev, peaks, peak_kind, timed, seed, M=None, row="flare_fwd_bwd"):
    """FLARE forward + backward, B=8 H=8 N=16,384 D=32 bf16; M = 128 (the
    workload's) or, for the M = 256 row, the headline's latent count."""
    import dataclasses

    import rank_latent_attention_flare_b200 as fl
    rows = {}
    w = WORKLOADS["c5_fwdbwd_bf16_16k"]
    if M is not None:
        w = dataclasses.replace(w, M=M)
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed, with_dy=True)
    g = {k: v.to(dev) for k, v in x.items()}
    wsf = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    wsb = fl.alloc_workspace(fl.FLARE_OP_BWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    saved = {}

    def fwd():
        saved["out"] = fl.flare_fwd(g["Q"], g["K"], g["V"], w.scale, save=True, workspace=wsf)

    ms_f = timed(fwd)
    _, Z, lse = saved["out"]
    ms_b = timed(lambda: fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, w.scale,
                                      workspace=wsb))
    if fl.device_status(wsf) != 0 or fl.device_status(wsb) != 0:
        raise RuntimeError("device wait ran out in the forward + backward")
    u = w.B * w.H * w.N
    ms = ms_f + ms_b
    rows[row] = {
        "workload": f"FLARE fwd+bwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16",
        "ms": round(ms, 4), "fwd_ms": round(ms_f, 4), "bwd_ms": round(ms_b, 4),
        "tokens_per_s": w.B * w.N / (ms / 1e3),
        "roofline": _row_roofline(ms, 4.0 * u * w.M, 28.0 * u * w.M * w.D,
                                  9.0 * u * w.D * 2, peaks, peak_kind,
                                  _fwd_exp_floor(u * w.M, w.M, w.D, peaks), 2.0 * u * w.M),
        "bwd_roofline": _row_roofline(ms_b, 2.0 * u * w.M, 20.0 * u * w.M * w.D,
                                      5.0 * u * w.D * 2, peaks, peak_kind)}
    return rows


def _time_strided(dev, peaks, peak_kind, timed, seed):
    """Token tensors stored [B,N,H,D] (a fused projection's layout) and read
    in place: the headline forward (B=1: batch and head flatten, 3-D maps)
    and the forward + backward workload (B=8: 4-D maps), each beside the
    same call on contiguous [B,H,N,D] tensors.  Algorithmic work as in the
    contiguous rows."""
    import torch

    import rank_latent_attention_flare_b200 as fl

    def bnhd(t):
        return t.transpose(1, 2).contiguous().transpose(1, 2)

    out = {}
    w = WORKLOAD
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed)
    Q = x["Q"].to(dev)
    Kt, Vt = bnhd(x["K"].to(dev)), bnhd(x["V"].to(dev))
    Yt = torch.empty_like(Kt)
    ws = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    ms_t = timed(lambda: fl.flare_fwd(Q, Kt, Vt, w.scale, workspace=ws, out=Yt))
    del Kt, Vt, Yt
    K, V = x["K"].to(dev), x["V"].to(dev)
    Y = torch.empty_like(K)
    ms_c = timed(lambda: fl.flare_fwd(Q, K, V, w.scale, workspace=ws, out=Y))
    if fl.device_status(ws) != 0:
        raise RuntimeError("device wait ran out in the strided forward")
    del K, V, Y, ws
    u = w.B * w.H * w.N
    out["fwd_headline_bnhd"] = {
        "workload": f"FLARE fwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16, K/V/Y [B,N,H,D]",
        "ms": round(ms_t, 4), "contiguous_ms": round(ms_c, 4),
        "tokens_per_s": w.B * w.N / (ms_t / 1e3),
        "roofline": _row_roofline(ms_t, 2.0 * u * w.M, 8.0 * u * w.M * w.D, 4.0 * u * w.D * 2,
                                  peaks, peak_kind, _fwd_exp_floor(u * w.M, w.M, w.D, peaks),
                                  2.0 * u * w.M)}
    w = WORKLOADS["c5_fwdbwd_bf16_16k"]
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed, with_dy=True)
    Q = x["Q"].to(dev)
    t = {k: bnhd(x[k].to(dev)) for k in ("K", "V", "dY")}
    wsf = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    wsb = fl.alloc_workspace(fl.FLARE_OP_BWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    saved = {}

    def fwd():
        saved["out"] = fl.flare_fwd(Q, t["K"], t["V"], w.scale, save=True, workspace=wsf)

    ms_f = timed(fwd)
    _, Z, lse = saved["out"]
    ms_b = timed(lambda: fl.flare_bwd(Q, t["K"], t["V"], t["dY"], Z, lse, w.scale, workspace=wsb))
    if fl.device_status(wsf) != 0 or fl.device_status(wsb) != 0:
        raise RuntimeError("device wait ran out in the strided forward + backward")
    u = w.B * w.H * w.N
    ms = ms_f + ms_b
    out["fwd_bwd_bnhd"] = {
        "workload": f"FLARE fwd+bwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16, "
                    "K/V/dY/Y/dK/dV [B,N,H,D]",
        "ms": round(ms, 4), "fwd_ms": round(ms_f, 4), "bwd_ms": round(ms_b, 4),
        "tokens_per_s": w.B * w.N / (ms / 1e3),
        "roofline": _row_roofline(ms, 4.0 * u * w.M, 28.0 * u * w.M * w.D,
                                  9.0 * u * w.D * 2, peaks, peak_kind,
                                  _fwd_exp_floor(u * w.M, w.M, w.D, peaks), 2.0 * u * w.M)}
    return {"flare_strided": out}


def _time_varlen(dev, peaks, peak_kind, timed, seed):
    """Right-padded batches: the forward + backward workload (B=8 H=8
    N=16,384 M=128 D=32 bf16) with sequence lengths N - b N/16 (16,384 down
    to 9,216, 78% of the tokens valid), beside the same call without lengths
    (`vs_full_length` = the ratio of their times).  Throughput counts valid
    tokens; the roofline is that of the valid work."""
    import torch

    import rank_latent_attention_flare_b200 as fl
    w = WORKLOADS["c5_fwdbwd_bf16_16k"]
    lens_l = [w.N - b * (w.N // 16) for b in range(w.B)]
    lens = torch.tensor(lens_l, dtype=torch.int32, device=dev)
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed, with_dy=True)
    g = {k: v.to(dev) for k, v in x.items()}
    wsf = fl.alloc_workspace(fl.FLARE_OP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    wsb = fl.alloc_workspace(fl.FLARE_OP_BWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    saved = {}

    def fwd():
        saved["out"] = fl.flare_fwd(g["Q"], g["K"], g["V"], w.scale, save=True, workspace=wsf,
                                    seq_lens=lens)

    ms_f = timed(fwd)
    _, Z, lse = saved["out"]
    ms_b = timed(lambda: fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Z, lse, w.scale,
                                      workspace=wsb, seq_lens=lens))
    if fl.device_status(wsf) != 0 or fl.device_status(wsb) != 0:
        raise RuntimeError("device wait ran out in the variable-length forward + backward")

    # the same call without lengths (every token valid), for the ratio
    def fwd_full():
        saved["full"] = fl.flare_fwd(g["Q"], g["K"], g["V"], w.scale, save=True, workspace=wsf)

    ms_ff = timed(fwd_full)
    _, Zf, lsef = saved["full"]
    ms_fb = timed(lambda: fl.flare_bwd(g["Q"], g["K"], g["V"], g["dY"], Zf, lsef, w.scale,
                                       workspace=wsb))
    valid = sum(lens_l)
    u = w.H * valid
    ms = ms_f + ms_b
    return {"flare_varlen": {
        "workload": f"FLARE fwd+bwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16, "
                    f"seq_lens {lens_l[0]}..{lens_l[-1]} ({100 * valid / (w.B * w.N):.0f}% valid)",
        "ms": round(ms, 4), "fwd_ms": round(ms_f, 4), "bwd_ms": round(ms_b, 4),
        "full_length_ms": round(ms_ff + ms_fb, 4),
        "vs_full_length": round(ms / (ms_ff + ms_fb), 3),
        "valid_tokens_per_s": valid / (ms / 1e3),
        "roofline": _row_roofline(ms, 4.0 * u * w.M, 28.0 * u * w.M * w.D,
                                  9.0 * u * w.D * 2, peaks, peak_kind,
                                  _fwd_exp_floor(u * w.M, w.M, w.D, peaks), 2.0 * u * w.M)}}


def time_sdpa_context(dev, w=WORKLOAD, iters: int = 5, seed: int = 0):
    """Prior-art context, not a target: the pages' expression of FLARE as two
    stock attention calls (encode SDPA(Q, K, V), decode SDPA(K, Q, Z)) with
    torch.nn.functional.scaled_dot_product_attention on the same device and
    workload, CUDA-event timed (median of `iters` after 2 warm-ups)."""
    import torch
    import torch.nn.functional as F
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed)
    Q = x["Q"].to(dev).unsqueeze(0).expand(w.B, w.H, w.M, w.D).contiguous()
    K = x["K"].to(dev)
    V = x["V"].to(dev)
    st = torch.cuda.current_stream()

    def two_calls():
        Z = F.scaled_dot_product_attention(Q, K, V, scale=w.scale)
        return F.scaled_dot_product_attention(K, Q, Z, scale=w.scale)

    for _ in range(2):
        two_calls()
    times = []
    for _ in range(iters):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        two_calls()
        b.record(st)
        times.append((a, b))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in times)
    del Q, K, V
    torch.cuda.empty_cache()
    return {"what": "two torch scaled_dot_product_attention calls (prior art, context only)",
            "ms": round(ms, 4), "tokens_per_s": w.B * w.N / (ms / 1e3)}


def _time_pp_fwd_bwd(dev, peaks, peak_kind, timed, seed):
    """FLARE++ forward + backward on the forward + backward workload's shape
    (B=8 H=8 N=16,384 M=128 D=32 bf16).  Algorithmic work per token-head:
    forward 3 M exponentials, 12 M D tensor FLOPs, K read 3x, V 2x, Y written;
    backward 3 M exponentials (P_d, P_e of the second encode, P of the first),
    30 M D tensor FLOPs, K, V, dY read and dK, dV written once."""
    import rank_latent_attention_flare_b200 as fl
    w = WORKLOADS["c5_fwdbwd_bf16_16k"]
    x = make_inputs(w.B, w.H, w.N, w.M, w.D, dtype=w.torch_dtype, seed=seed, with_dy=True)
    g = {k: v.to(dev) for k, v in x.items()}
    wsf = fl.alloc_workspace(fl.FLARE_OP_PP_FWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    wsb = fl.alloc_workspace(fl.FLARE_OP_PP_BWD, w.B, w.H, w.N, w.M, w.D, w.torch_dtype, dev)
    saved = {}

    def fwd():
        saved["out"] = fl.flare_pp_fwd(g["Q"], g["K"], g["V"], w.scale, save=True, workspace=wsf)

    ms_f = timed(fwd)
    _, Qd, Z, lse = saved["out"]
    ms_b = timed(lambda: fl.flare_pp_bwd(g["Q"], g["K"], g["V"], g["dY"], Qd, Z, lse, w.scale,
                                         workspace=wsb))
    if fl.device_status(wsf) != 0 or fl.device_status(wsb) != 0:
        raise RuntimeError("device wait ran out in the FLARE++ forward + backward")
    u = w.B * w.H * w.N
    ms = ms_f + ms_b
    return {"flare_pp_fwd_bwd": {
        "workload": f"FLARE++ fwd+bwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16",
        "ms": round(ms, 4), "fwd_ms": round(ms_f, 4), "bwd_ms": round(ms_b, 4),
        "tokens_per_s": w.B * w.N / (ms / 1e3),
        "roofline": _row_roofline(ms, 6.0 * u * w.M, 42.0 * u * w.M * w.D,
                                  11.0 * u * w.D * 2, peaks, peak_kind,
                                  _fwd_exp_floor(u * w.M, w.M, w.D, peaks, (0, 0, 1)),
                                  3.0 * u * w.M),
        "bwd_roofline": _row_roofline(ms_b, 3.0 * u * w.M, 30.0 * u * w.M * w.D,
                                      5.0 * u * w.D * 2, peaks, peak_kind)}}


def run_row(args, rank, local):
    """One of the other workloads alone (FLARE++ forward, or forward +
    backward), e.g. for a profiler capture."""
    import torch
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    rows = time_other_rows(dev, peaks, peak_kind, iters=max(1, args.steps), seed=rank,
                           which=(args.row,), rates=measure_unit_rates())
    if rank == 0:
        print(json.dumps({"row": args.row, **rows[args.row]}), flush=True)


# ------------------------------------------------------------- reference

def run_reference(args, rank, world):
    """The oracle (double-precision CPU FLARE) timed per step on a bounded
    sample; rank 0 only."""
    if rank != 0:
        return
    w = WORKLOAD
    import oracle
    budget = max(1.0, args.ref_seconds)
    per_step = budget / (args.steps + args.warmup)
    _, _, cores, n_s, h_s = oracle_sample_rate(per_step)
    x = make_inputs(1, h_s, n_s, w.M, w.D, dtype=w.torch_dtype, seed=0)
    for _ in range(args.warmup):
        oracle.flare_fwd(x["Q"], x["K"], x["V"], w.scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.flare_fwd(x["Q"], x["K"], x["V"], w.scale)
    t = time.perf_counter() - t0
    value = args.steps * (h_s * n_s / w.H) / t
    sample = (f"per step: oracle FLARE fwd on {h_s} of {w.B * w.H} heads x {n_s} of {w.N} "
              f"tokens (M={w.M}, D={w.D}); tokens/s counts 1/H token per head-token")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"FLARE fwd B={w.B} H={w.H} N={w.N} M={w.M} D={w.D} bf16-rounded "
                               "inputs, scale 1/sqrt(D), i.i.d. N(0,1)",
                   "global_batch": w.B, "seq_len": w.N, "parallelism": "cpu (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true",
                    help="skip the FLARE++ and forward+backward timings")
    ap.add_argument("--row", choices=["flare_fwd_c2", "flare_fwd_m64", "flare_pp_fwd", "flare_fwd_bwd",
                                      "flare_fwd_bwd_m256",
                                      "flare_pp_fwd_bwd",
                                      "flare_strided", "flare_varlen"],
                    default=None,
                    help="time only this workload (one JSON line with its timing and roofline)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=120.0)
    ap.add_argument("--out-dir", default=None, help="where to write the clock samples")
    ap.add_argument("--heads", type=int, default=0, help="override H (profiling captures only)")
    ap.add_argument("--seq", type=int, default=0, help="override N (profiling captures only)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.row:
            run_row(args, rank, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        dist_done(world)


if __name__ == "__main__":
    main()
