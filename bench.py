#!/usr/bin/env python
"""Benchmark of the B200 GDN forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--T T] [--no-cpu-baseline] [--no-e2e]

A step is one whole GDN forward (prep, UT transform, scan, output) over the
workload with its inputs resident in HBM; the L2 cache is flushed (256 MiB
write) before every step, outside the timed interval.  Each step is timed
with CUDA events on the launching stream around the plain forward; per-kernel
times come from separate runs in which the library records events between its
launches (gdn_forward_timed), which serialises them.  With N > 1
(torchrun) every rank runs its own replica of the workload (the forward has
no cross-GPU exchange) and the time is the max over ranks.  Rank 0 prints one
JSON line.

--impl reference times the oracle (the plain fp64 CPU statement of the
method) on this host's cores, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import gdn_inputs  # noqa: E402

METRIC = "GDN fwd Mtokens/s at T=32760,H=12,d=128 bf16; % of tensor/HBM roofline"
UNIT = "Mtokens/s"
FLUSH_BYTES = 256 << 20
KERNELS_TENSOR_SEG = ("prep", "chunk", "transfer", "combine", "scan")
KERNELS_TENSOR_ONE = ("prep", "chunk", "scan")
KERNELS_FUSED_SEG = ("fused_transfer", "fused_combine", "fused_out")
KERNELS_FUSED_ONE = ("fused_out",)
KERNELS_SIMT = ("prep", "recurrence", "output")
KERNEL_SOURCES = {"prep": "gdn_prep.cu", "chunk": "gdn_chunk.cu", "transfer": "gdn_scan.cu",
                  "combine": "gdn_scan.cu", "scan": "gdn_scan.cu", "fused_transfer": "gdn_fused.cu",
                  "fused_combine": "gdn_fused.cu", "fused_out": "gdn_fused.cu", "recurrence": "gdn_simt.cu",
                  "output": "gdn_simt.cu"}


def kernel_names(plan, fused=False):
    if not plan.uses_tensor_path:
        return KERNELS_SIMT
    if fused:
        return KERNELS_FUSED_SEG if plan.segments > 1 else KERNELS_FUSED_ONE
    return KERNELS_TENSOR_SEG if plan.segments > 1 else KERNELS_TENSOR_ONE


def path_bytes_per_token_head(d, s_in, s_out):
    # q, k, v, z in; g, b fp32 in; y out (parameters negligible)
    return 4 * d * s_in + 8 + d * s_out


def path_flops_per_token_head(d, C=64):
    # five C x C x d block products counted as full tiles + three C x d x d products per chunk
    return 10 * C * d + 6 * d * d


def kernel_work_per_token_head(name, d, s_in, s_out):
    """HBM bytes each kernel itself must move, and the tensor-core flops it issues, per (token,
    head) of the token-heads it covers.

    Tensor path (d = 128, 128-token blocks, fp16 intermediates): prep writes q^, k^, v^; chunk
    builds W, U, Qt, Kt and the live 3/4 of Aqk; transfer runs each segment's [S | P] from W, U,
    Kt; combine moves per-segment states only; scan rebuilds Delta and writes y.
    Fused tensor path (64-token blocks, no intermediates in HBM): the transfer pass reads raw k, v
    and the gates and runs S and P side by side; the output pass reads raw q, k, v, z and the
    gates and writes y.  CUDA-core path: prep, recurrence and output kernels."""
    if name == "prep":      # q k v in; q^ k^ v^ fp16 out
        return 3 * d * s_in + 3 * d * 2, 0
    if name == "chunk":     # q^ k^ v^ + g b in; W U Qt Kt, 3/4 of Aqk, G beta log-alpha out; K K^T, Q K^T, W, U
        return 3 * d * 2 + 8 + 4 * 128 * 2 + 96 * 2 + 12, 4 * 2 * 128 * d
    if name == "transfer":  # W U Kt in; W [S|P]^T and Kt^T Delta with N = 2d
        return 3 * 128 * 2, 2 * 2 * 128 * 2 * d
    if name in ("combine", "fused_combine"):  # per-segment states only (negligible per token)
        return 0, 0
    if name == "scan":      # W U Qt Kt, 3/4 of Aqk, z in; y out; W S^T, Qt S^T, Kt^T Delta, Aqk Delta
        return 4 * 128 * 2 + 96 * 2 + d * s_in + d * s_out, 4 * 2 * 128 * d
    C = 64
    gram, wu = 2 * 128 * C * 128 // C, 2 * 2 * 128 * C * C // C          # [K;Q]K^T or KK^T; W^T and U^T
    step = 2 * 128 * C * d // C + 2 * 128 * 128 * C // C                # Delta^T, state update
    if name == "fused_transfer":
        return 2 * d * s_in + 8, gram + wu + 2 * step
    if name == "fused_out":    # Delta^T, O^T = N Qt^T, state, O^T += E Aqk^T
        return 4 * d * s_in + 8 + d * s_out, gram + wu + step + 2 * 128 * C * d // C + 2 * 128 * C * C // C
    if name == "output":    # o fp32 + z in; y out
        return d * 4 + d * s_in + d * s_out, 0
    if name == "recurrence":
        return 3 * d * 4 + 8 + d * 4, 6 * d * d
    raise KeyError(name)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm_gbs=float(j["hbm_gbs"]), bf16_tflops=float(j["bf16_tflops"]),
                    bf16_tflops_sustained=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def kernel_source_sha(name):
    with open(os.path.join(ROOT, "gated_deltanet_06_b200", "csrc", KERNEL_SOURCES[name]), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(name, workload):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    source is unchanged since the capture; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(name, {}).get(workload)
    if not e or e.get("source_sha") != kernel_source_sha(name):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.dev = device_index

    def start(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = self.dev
        if vis:
            try:
                idx = int(vis.split(",")[self.dev])
            except (ValueError, IndexError):
                idx = None
        sel = ["-i", str(idx)] if idx is not None else []
        self.err = os.devnull
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "100"] + sel, stdout=subprocess.PIPE,
                                         stderr=open(self.err, "w"), text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [[x.strip() for x in line.split(",")] for line in out.strip().splitlines() if line.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                s = float(r[1]); mx = float(r[2])
            except (ValueError, IndexError):
                continue
            sm.append(s)
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        loaded = [s for s in sm if mx and s >= 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def other_gpu_processes(device_index):
    """Compute processes other than this one on the GPU (another tenant time-slicing it would
    distort every timing), or None where NVML cannot tell."""
    try:
        import pynvml
        pynvml.nvmlInit()
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = int(vis.split(",")[device_index]) if vis else device_index
        h = pynvml.nvmlDeviceGetHandleByIndex(idx)
        procs = pynvml.nvmlDeviceGetComputeRunningProcesses(h)
        return sorted({p.pid for p in procs if p.pid != os.getpid()})
    except Exception:
        return None


def oracle_rate(w, T_sample, threads):
    import oracle
    inp = gdn_inputs.workload_inputs(w, T=T_sample)
    t0 = time.perf_counter()
    oracle.forward(inp, nthreads=threads)
    return time.perf_counter() - t0


def cpu_threads(w):
    return max(1, min(w.B * w.H, os.cpu_count() or 1))


def calibrate_oracle_T(w, seconds, threads):
    t_small = 256
    dt = oracle_rate(w, t_small, threads)
    per_tok = dt / t_small
    return int(max(256, min(w.T, seconds / max(per_tok, 1e-9))))


def sample_text(w, T_s):
    if T_s >= w.T:
        return f"the whole {w.name} workload (T={w.T})"
    return (f"{w.name} at T={T_s} instead of {w.T} (same seed, distributions, B and H; "
            f"cost is linear in T)")


def run_cpu_baseline(w, budget_s=12.0):
    threads = cpu_threads(w)
    T_s = calibrate_oracle_T(w, budget_s, threads)
    dt = oracle_rate(w, T_s, threads)
    return {"value": w.B * T_s / dt / 1e6, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{sample_text(w, T_s)}: fp64 sequential recurrence, {threads} threads, {dt:.1f} s"}


def reference_arm(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    threads = cpu_threads(w)
    per_step = max(0.2, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    T_s = calibrate_oracle_T(w, per_step, threads)
    times = []
    for i in range(args.warmup + args.steps):
        dt = oracle_rate(w, T_s, threads)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = w.B * T_s * len(times) / total / 1e6
    sample = f"{sample_text(w, T_s)} per step: fp64 sequential recurrence, {threads} threads"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(w, args.out_dtype, max(1, args.gpus)), "sample_T": T_s,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def ranks_max(x, world, dist=None, device=None):
    """The max of x over the ranks (every rank gets it); x itself with one rank."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_rank, ms_per_step):
    """Whole-job Mtokens/s: every rank processes its own replica of the workload per step."""
    return world * tokens_per_rank / (ms_per_step / 1e3) / 1e6


def out_name_of(w, out_dtype=None):
    return out_dtype or ("bf16" if w.dtype == "bf16" else "f32")


def workload_config(w, out_dtype, world):
    """The JSON line's config object: the workload's name, shape, types and input recipe."""
    return {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "d": w.d, "in_dtype": w.dtype,
            "out_dtype": out_name_of(w, out_dtype), "g_mean": w.g_mean, "seed": w.seed,
            "l2": "flushed before every step (256 MiB write, outside the timed interval)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def path_roofline(w, s_in, s_out, ms_per_step, peaks):
    """The method's whole-path roofline: 1288 B and 180,224 chunk flops per (token, head) at d = 128
    bf16, t_roof = max(bytes / HBM bandwidth, flops / bf16 tensor peak)."""
    units = w.B * w.T * w.H
    pb = path_bytes_per_token_head(w.d, s_in, s_out)
    pf = path_flops_per_token_head(w.d)
    t_roof = max(pb * units / (peaks["hbm_gbs"] * 1e9), pf * units / (peaks["bf16_tflops"] * 1e12))
    return {"bytes_per_token_head": pb, "flops_per_token_head": pf, "roofline_ms": t_roof * 1e3,
            "roofline_Mtokens_s": w.B * w.T / t_roof / 1e6, "frac": (t_roof * 1e3) / ms_per_step,
            "bound": "hbm" if pb * units / peaks["hbm_gbs"] >= pf * units / (peaks["bf16_tflops"] * 1e3) else "tensor"}


def launch_units(name, w, plan):
    """Token-heads one launch of a kernel covers: a transfer pass runs every segment but the last
    (segments of Ls blocks of 128 tokens on the tensor path, of 64 on the fused path)."""
    if name in ("transfer", "fused_transfer"):
        C = 64 if name == "fused_transfer" else 128
        ns = plan.segments
        nb = -(-w.T // C)
        ls = -(-nb // ns)
        return w.B * w.H * min((ns - 1) * ls * C, w.T)
    return w.B * w.H * w.T


def device_tensors(inp, w, dev):
    import torch
    tens = {}
    for n in ("q", "k", "v", "z"):
        if w.dtype == "bf16":
            tens[n] = torch.from_numpy(inp[n + "_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
        else:
            tens[n] = torch.from_numpy(inp[n]).to(dev)
    for n in ("g", "b", "conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w"):
        tens[n] = torch.from_numpy(np.ascontiguousarray(inp[n], dtype=np.float32)).to(dev)
    return tens


def time_steps(run, flush, stream, steps):
    """CUDA-event times (ms) of `steps` calls of run(), the L2 flushed before each, outside the interval."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for k in range(steps):
        flush.zero_()
        ev[k][0].record(stream)
        run()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def bench_other_config(w, dev, flush, stream, steps, cpu_budget_s):
    """One of the other seeded workloads: the same step, flush and event timing as the headline, the
    path roofline, and the oracle on a bounded sample as its baseline."""
    import torch

    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.workload_inputs(w)
    tens = device_tensors(inp, w, dev)
    del inp
    in_code = gdn.DTYPE_BF16 if w.dtype == "bf16" else gdn.DTYPE_F32
    out_name = out_name_of(w)
    out_t = {"bf16": torch.bfloat16, "f32": torch.float32}[out_name]
    plan = gdn.Plan(w.B, w.T, w.H, w.d, in_code, gdn.DTYPE_BF16 if out_name == "bf16" else gdn.DTYPE_F32)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
    y = torch.empty((w.B, w.T, w.H, w.d), dtype=out_t, device=dev)
    ptrs = gdn.tensor_ptrs(tens)
    s = stream.cuda_stream
    run = lambda: plan.forward_raw(ptrs, y.data_ptr(), ws.data_ptr(), s)  # noqa: E731
    for _ in range(3):
        run()
    ms = time_steps(run, flush, stream, steps)
    st = plan.device_status(ws.data_ptr(), s)
    if st != gdn.OK:
        raise SystemExit(f"device status, {w.name}: {gdn.status_string(st)}")
    ms_step = statistics.mean(ms)
    s_in = 2 if w.dtype == "bf16" else 4
    s_out = 2 if out_name == "bf16" else 4
    out = {"value": w.B * w.T / (ms_step / 1e3) / 1e6, "unit": UNIT, "ms_per_step": ms_step, "steps": steps,
           "config": workload_config(w, None, 1), "tensor_path": plan.uses_tensor_path,
           "segments": plan.segments, "launches_per_step": plan.launches,
           "path_roofline": path_roofline(w, s_in, s_out, ms_step, load_peaks()),
           "step_ms": {"min": min(ms), "median": statistics.median(ms), "max": max(ms)}}
    del tens, ws, y
    torch.cuda.empty_cache()
    if cpu_budget_s > 0:
        out["cpu_baseline"] = run_cpu_baseline(w, cpu_budget_s)
    return out


def block_flops(w, D):
    """Tensor-core flops of the two projections per layer: 2 M N K each."""
    M, Hd = w.B * w.T, w.H * w.d
    return 2 * M * (4 * Hd + 2 * w.H) * D, 2 * M * D * Hd


def bench_block(w, dev, flush, stream, steps, world, dist):
    """gdn_block_forward on this workload's shape with D = H * d: step time, per-kernel times and the
    projections' tensor-core throughput against the measured bf16 peak."""
    import torch

    import gated_deltanet_06_b200 as gdn
    D = w.H * w.d
    inp = gdn_inputs.make_block_inputs(w.B, w.T, w.H, w.d, D, seed=w.seed)
    t = {}
    for n in ("x", "w_in", "w_out"):
        t[n] = torch.from_numpy(inp[n + "_bits"].view(np.int16)).view(torch.bfloat16).to(dev)
    for n in ("conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w"):
        t[n] = torch.from_numpy(np.ascontiguousarray(inp[n], dtype=np.float32)).to(dev)
    del inp
    bp = gdn.BlockPlan(w.B, w.T, w.H, w.d, D, gdn.DTYPE_BF16)
    ws = torch.empty(bp.workspace_bytes, dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, w.T, D), dtype=torch.bfloat16, device=dev)
    ptrs = {n: v.data_ptr() for n, v in t.items()}
    s = stream.cuda_stream
    run = lambda: bp.forward_raw(ptrs, out.data_ptr(), ws.data_ptr(), s)  # noqa: E731
    for _ in range(3):
        run()
    ms = time_steps(run, flush, stream, steps)
    st = bp.device_status(ws.data_ptr(), s)
    if st != gdn.OK:
        raise SystemExit(f"device status after the block forward: {gdn.status_string(st)}")
    m = ranks_max(sum(ms), world, dist, dev) / steps
    L = bp.launches
    names = ["bf16_to_f16", "proj_in", "chunk"] + (["transfer", "combine"] if L == 7 else []) + ["scan", "proj_out"]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(L + 1)] for _ in range(3)]
    for row in evs:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    for k in range(3):
        flush.zero_()
        bp.forward_timed_raw(ptrs, out.data_ptr(), ws.data_ptr(), s, [e.cuda_event for e in evs[k]])
    torch.cuda.synchronize()
    km = {names[i]: statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(3)) for i in range(L)}
    f_in, f_out = block_flops(w, D)
    peak = load_peaks()["bf16_tflops"]
    res = {"ms_per_step": m, "value": job_throughput(world, w.B * w.T, m), "unit": UNIT, "steps": steps, "D": D,
           "launches_per_step": L, "kernels_ms": km,
           "proj_in": {"flops": f_in, "tflops": f_in / (km["proj_in"] / 1e3) / 1e12,
                       "frac_of_bf16_peak": f_in / (km["proj_in"] / 1e3) / 1e12 / peak},
           "proj_out": {"flops": f_out, "tflops": f_out / (km["proj_out"] / 1e3) / 1e12,
                        "frac_of_bf16_peak": f_out / (km["proj_out"] / 1e3) / 1e12 / peak},
           "step_ms": {"min": min(ms), "median": statistics.median(ms), "max": max(ms)}}
    del ws, out, t
    torch.cuda.empty_cache()
    return res


def backward_kernel_names(launches: int):
    """Names of gdn_backward's launches in order: the tensor-core backward (12 launches, or 8 with
    one segment per sequence) or the fp32 CUDA-core backward (6)."""
    if launches == 6:
        return ("prep_f32", "fwd_rows", "out_bwd", "core_bwd", "tokens_bwd", "params")
    if launches == 12:
        return ("prep", "ut_keep", "transfer", "combine", "scan_out_o", "out_bwd", "bwd_transfer", "bwd_combine",
                "bwd_scan", "bwd_grad", "tokens_bwd", "params")
    if launches == 8:
        return ("prep", "ut_keep", "scan_out_o", "out_bwd", "bwd_scan", "bwd_grad", "tokens_bwd", "params")
    raise ValueError(launches)


def backward_grad_flops(bh: int, blocks: int) -> float:
    """FLOPs of the block-gradient kernel: 16 products of 128 x 128 x 128 per 128-token block."""
    return 16 * 2.0 * 128 ** 3 * bh * blocks


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=gdn_inputs.HEADLINE.name)
    ap.add_argument("--T", type=int, default=None, help="override the sequence length (profiling runs)")
    ap.add_argument("--out-dtype", default=None, choices=[None, "bf16", "f16", "f32"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-state", action="store_true", help="skip the carried-state timing")
    ap.add_argument("--no-reverse", action="store_true", help="skip the reverse-scan timing")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward timing")
    ap.add_argument("--no-configs", action="store_true", help="skip the other four seeded workloads")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--no-block", action="store_true", help="skip the layer-with-projections timing")
    ap.add_argument("--fused", action="store_true", help="time the fused forward (FLAG_FUSED) as the main path")
    ap.add_argument("--no-fused", action="store_true", help="skip the fused-forward timing beside the main path")
    ap.add_argument("--load-seconds", type=float, default=1.5)
    args = ap.parse_args()
    w = gdn_inputs.by_name(args.workload)
    if args.T:
        w = gdn_inputs.Workload(w.name + f"_T{args.T}", w.B, w.H, args.T, w.d, w.dtype, w.g_mean, w.seed, w.note)
    if args.impl == "reference":
        return reference_arm(args, w)

    import torch
    import torch.distributed as dist

    import gated_deltanet_06_b200 as gdn

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    inp = gdn_inputs.workload_inputs(w, T=args.T)
    tens = device_tensors(inp, w, dev)
    del inp
    in_code = gdn.DTYPE_BF16 if w.dtype == "bf16" else gdn.DTYPE_F32
    out_name = args.out_dtype or ("bf16" if w.dtype == "bf16" else "f32")
    out_code = {"bf16": gdn.DTYPE_BF16, "f16": gdn.DTYPE_F16, "f32": gdn.DTYPE_F32}[out_name]
    out_t = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[out_name]
    base_flags = gdn.FLAG_FUSED if args.fused else 0
    plan = gdn.Plan(w.B, w.T, w.H, w.d, in_code, out_code, flags=base_flags)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
    y = torch.empty((w.B, w.T, w.H, w.d), dtype=out_t, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    ptrs = gdn.tensor_ptrs(tens)
    L = plan.launches
    names = kernel_names(plan, args.fused)
    assert len(names) == L

    for _ in range(args.warmup):
        plan.forward_raw(ptrs, y.data_ptr(), ws.data_ptr(), s)
    torch.cuda.synchronize()
    # untimed load phase so that the clock samples see the GPU busy with this work
    others_before = other_gpu_processes(local)
    sampler = ClockSampler(local)
    sampler.start()
    t_end = time.perf_counter() + args.load_seconds
    while time.perf_counter() < t_end:
        for _ in range(20):
            plan.forward_raw(ptrs, y.data_ptr(), ws.data_ptr(), s)
        torch.cuda.synchronize()

    # timed steps: the plain forward (consecutive kernels overlap their launch and prologue with
    # the previous kernel's tail), one event pair per step around it
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.zero_()
        ev_step[k][0].record(stream)
        plan.forward_raw(ptrs, y.data_ptr(), ws.data_ptr(), s)
        ev_step[k][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    others_after = other_gpu_processes(local)
    st = plan.device_status(ws.data_ptr(), s)
    if st != gdn.OK:
        raise SystemExit(f"device status after timing: {gdn.status_string(st)}")
    step_ms = [a.elapsed_time(b) for a, b in ev_step]
    # each forward clears the device status word, so the check above sees only the last step:
    # repeat the steps untimed, reading the status after every one (a bounded device wait that ran
    # out in any of them would show here)
    for _ in range(args.steps):
        flush.zero_()
        plan.forward_raw(ptrs, y.data_ptr(), ws.data_ptr(), s)
        st = plan.device_status(ws.data_ptr(), s)
        if st != gdn.OK:
            raise SystemExit(f"device status in the per-step check: {gdn.status_string(st)}")

    # the same forward captured once in a CUDA graph and replayed (launch overhead out of the step);
    # the flush stays outside the graph and outside the timed interval
    graph = None
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            torch.cuda.synchronize()
            with torch.cuda.graph(g):
                plan.forward_raw(ptrs, y.data_ptr(), ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
            for _ in range(3):
                g.replay()
            g_ms = time_steps(g.replay, flush, stream, args.steps)
            st = plan.device_status(ws.data_ptr(), s)
            if st != gdn.OK:
                raise SystemExit(f"device status after the graph replays: {gdn.status_string(st)}")
            gm = ranks_max(sum(g_ms), world, dist, dev) / args.steps
            graph = {"ms_per_step": gm, "value": job_throughput(world, w.B * w.T, gm), "unit": UNIT,
                     "steps": args.steps, "step_ms": {"min": min(g_ms), "median": statistics.median(g_ms),
                                                      "max": max(g_ms)}}
            del g
        except RuntimeError as e:  # capture refused by the runtime: reported, not fatal
            graph = {"unavailable": str(e).splitlines()[0][:200]}

    # per-kernel breakdown (not part of the timed steps): the library records an event before each
    # launch and after the last one (gdn_forward_timed), which also serialises the launches
    n_kt = max(3, min(args.steps, 10))
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(L + 1)] for _ in range(n_kt)]
    for row in events:  # torch creates the underlying cudaEvent_t on first record
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    for k in range(n_kt):
        flush.zero_()
        plan.forward_timed_raw(ptrs, y.data_ptr(), ws.data_ptr(), s, [e.cuda_event for e in events[k]])
    torch.cuda.synchronize()
    kern_ms = {names[i]: statistics.mean(events[k][i].elapsed_time(events[k][i + 1]) for k in range(n_kt))
               for i in range(L)}
    total_ms = ranks_max(sum(step_ms), world, dist, dev)
    ms_per_step = total_ms / args.steps
    tokens = w.B * w.T
    value = job_throughput(world, tokens, ms_per_step)

    # the same forward with the recurrent state carried in and out (gdn_forward_state): an initial
    # state read and the final state written, [B][H][d][d] fp32 each
    state_io = None
    if not args.no_state:
        s0 = torch.randn((w.B, w.H, w.d, w.d), dtype=torch.float32, device=dev).mul_(0.5)
        s_end = torch.empty_like(s0)
        n_st = max(3, min(args.steps, 10))
        for _ in range(2):
            plan.forward_state_raw(ptrs, s0.data_ptr(), y.data_ptr(), s_end.data_ptr(), ws.data_ptr(), s)
        ev_st = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_st)]
        torch.cuda.synchronize()
        for k in range(n_st):
            flush.zero_()
            ev_st[k][0].record(stream)
            plan.forward_state_raw(ptrs, s0.data_ptr(), y.data_ptr(), s_end.data_ptr(), ws.data_ptr(), s)
            ev_st[k][1].record(stream)
        torch.cuda.synchronize()
        st_ms = ranks_max(sum(a.elapsed_time(b) for a, b in ev_st), world, dist, dev) / n_st
        state_io = {"ms_per_step": st_ms, "value": job_throughput(world, w.B * w.T, st_ms), "unit": UNIT,
                    "state_bytes_per_step": 2 * w.B * w.H * w.d * w.d * 4, "steps": n_st}

    # the reverse (anti-causal) scan of the same workload, its own plan and workspace
    reverse = None
    if not args.no_reverse:
        plan_r = gdn.Plan(w.B, w.T, w.H, w.d, in_code, out_code, flags=gdn.FLAG_REVERSE | base_flags)
        ws_r = torch.empty(plan_r.workspace_bytes, dtype=torch.uint8, device=dev)
        n_r = max(3, min(args.steps, 10))
        for _ in range(2):
            plan_r.forward_raw(ptrs, y.data_ptr(), ws_r.data_ptr(), s)
        ev_r = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_r)]
        torch.cuda.synchronize()
        for k in range(n_r):
            flush.zero_()
            ev_r[k][0].record(stream)
            plan_r.forward_raw(ptrs, y.data_ptr(), ws_r.data_ptr(), s)
            ev_r[k][1].record(stream)
        torch.cuda.synchronize()
        st = plan_r.device_status(ws_r.data_ptr(), s)
        if st != gdn.OK:
            raise SystemExit(f"device status after the reverse scan: {gdn.status_string(st)}")
        r_ms = ranks_max(sum(a.elapsed_time(b) for a, b in ev_r), world, dist, dev) / n_r
        reverse = {"ms_per_step": r_ms, "value": job_throughput(world, w.B * w.T, r_ms), "unit": UNIT,
                   "steps": n_r}
        del ws_r

    # the backward (gradient of sum(y * dy) w.r.t. every input and parameter) of the same workload
    bwd = None
    if not args.no_backward:
        ws_b = torch.empty(plan.backward_workspace_bytes, dtype=torch.uint8, device=dev)
        dy = torch.randn((w.B, w.T, w.H, w.d), device=dev).to(out_t)
        f32 = dict(dtype=torch.float32, device=dev)
        gr = {n: torch.empty((w.B, w.T, w.H, w.d), **f32) for n in ("dq", "dk", "dv", "dz")}
        gr.update(dg=torch.empty((w.B, w.T, w.H), **f32), db=torch.empty((w.B, w.T, w.H), **f32),
                  dA_log=torch.empty(w.H, **f32), ddt_bias=torch.empty(w.H, **f32), dnorm_w=torch.empty(w.d, **f32))
        for n in ("dconv_q", "dconv_k", "dconv_v"):
            gr[n] = torch.empty((w.H * w.d, 4), **f32)
        gp = {n: gr[n].data_ptr() for n in gdn.GRAD_NAMES}
        n_b = 3
        torch.cuda.nvtx.range_push("gdn_backward")  # the first call, for a profiler's launch list (--nvtx)
        plan.backward_raw(ptrs, dy.data_ptr(), gp, ws_b.data_ptr(), s)
        torch.cuda.nvtx.range_pop()
        ev_b = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_b)]
        torch.cuda.synchronize()
        for k in range(n_b):
            flush.zero_()
            ev_b[k][0].record(stream)
            plan.backward_raw(ptrs, dy.data_ptr(), gp, ws_b.data_ptr(), s)
            ev_b[k][1].record(stream)
        torch.cuda.synchronize()
        st = plan.device_status(ws_b.data_ptr(), s)
        if st != gdn.OK:
            raise SystemExit(f"device status after the backward: {gdn.status_string(st)}")
        b_ms = ranks_max(sum(a.elapsed_time(b) for a, b in ev_b), world, dist, dev) / n_b
        # per-kernel breakdown (events between the launches, one more run)
        LB = plan.backward_launches
        evk = [torch.cuda.Event(enable_timing=True) for _ in range(LB + 1)]
        for e in evk:
            e.record(stream)
        torch.cuda.synchronize()
        flush.zero_()
        plan.backward_timed_raw(ptrs, dy.data_ptr(), gp, ws_b.data_ptr(), s, [e.cuda_event for e in evk])
        torch.cuda.synchronize()
        bnames = backward_kernel_names(LB)
        kms = {bnames[i]: evk[i].elapsed_time(evk[i + 1]) for i in range(LB)}
        bwd = {"ms_per_step": b_ms, "value": job_throughput(world, w.B * w.T, b_ms), "unit": UNIT,
               "steps": n_b, "launches_per_step": LB,
               "precision": ("fp16 tensor-core operands, fp32 accumulation" if LB != 6 else "fp32 CUDA cores"),
               "vs_forward": b_ms / ms_per_step, "kernels_ms": kms}
        if "bwd_grad" in kms:  # the block-gradient kernel: 16 products of 128 x 128 x 128 per block
            fl = backward_grad_flops(w.B * w.H, -(-w.T // 128))
            bwd["bwd_grad_tflops"] = fl / (kms["bwd_grad"] / 1e3) / 1e12
            pk = load_peaks()
            if pk and pk.get("bf16_tflops"):  # fp16 and bf16 run at the same dense rate
                bwd["bwd_grad_frac_of_tensor_peak"] = bwd["bwd_grad_tflops"] / pk["bf16_tflops"]
        del ws_b, gr, dy

    # end to end through the public host-buffer entry point (gdn_forward_host: every input copied from
    # pinned host memory, the forward, y copied back), first on one stream, then on two streams that
    # take alternate steps with their own staging, workspace and host output, so that one step's
    # host-to-device copies overlap the previous step's compute and device-to-host copy
    e2e = None
    if not args.no_e2e:
        host = {n: tens[n].cpu().pin_memory() for n in tens}
        hptrs = gdn.tensor_ptrs(host)
        n_e2e = max(4, min(args.steps, 10))
        y_hosts = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
        stagings = [torch.empty(plan.staging_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        wss = [ws, torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)]
        streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]

        def run_e2e(nstreams):
            for i in range(nstreams):  # warm-up
                plan.forward_host_raw(hptrs, y_hosts[i].data_ptr(), stagings[i].data_ptr(), wss[i].data_ptr(),
                                      streams[i].cuda_stream)
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            for i in range(nstreams):
                streams[i].wait_event(ev0)
            for k in range(n_e2e):
                i = k % nstreams
                plan.forward_host_raw(hptrs, y_hosts[i].data_ptr(), stagings[i].data_ptr(), wss[i].data_ptr(),
                                      streams[i].cuda_stream)
            for i in range(nstreams):
                ev = torch.cuda.Event()
                ev.record(streams[i])
                stream.wait_event(ev)
            ev1.record(stream)
            torch.cuda.synchronize()
            for i in range(nstreams):
                st = plan.device_status(wss[i].data_ptr(), streams[i].cuda_stream)
                if st != gdn.OK:
                    raise SystemExit(f"device status after the end-to-end steps: {gdn.status_string(st)}")
            return ranks_max(ev0.elapsed_time(ev1) / n_e2e, world, dist, dev)

        serial_ms = run_e2e(1)
        te_ms = run_e2e(2)
        if not torch.equal(y_hosts[0], y_hosts[1]):
            raise SystemExit("the two streams' end-to-end outputs differ")
        h2d = sum(host[n].numel() * host[n].element_size() for n in host)
        d2h = y_hosts[0].numel() * y_hosts[0].element_size()
        e2e = {"value": job_throughput(world, tokens, te_ms), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n_e2e,
               "streams": 2, "ms_per_step": te_ms,
               "one_stream": {"value": job_throughput(world, tokens, serial_ms), "ms_per_step": serial_ms}}
        del wss[1], stagings

    # the fused forward (FLAG_FUSED) of the same workload beside the main path: step time, its
    # per-kernel breakdown and its roofline figures
    fused = None
    if not args.fused and not args.no_fused and plan.uses_tensor_path:
        plan_f = gdn.Plan(w.B, w.T, w.H, w.d, in_code, out_code, flags=gdn.FLAG_FUSED)
        ws_f = torch.empty(plan_f.workspace_bytes, dtype=torch.uint8, device=dev)
        run_f = lambda: plan_f.forward_raw(ptrs, y.data_ptr(), ws_f.data_ptr(), s)  # noqa: E731
        for _ in range(3):
            run_f()
        n_f = max(5, min(args.steps, 20))
        f_ms = ranks_max(sum(time_steps(run_f, flush, stream, n_f)), world, dist, dev) / n_f
        st = plan_f.device_status(ws_f.data_ptr(), s)
        if st != gdn.OK:
            raise SystemExit(f"device status after the fused forward: {gdn.status_string(st)}")
        fnames = kernel_names(plan_f, True)
        evf = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fnames) + 1)] for _ in range(3)]
        for row in evf:
            for e in row:
                e.record(stream)
        torch.cuda.synchronize()
        for k in range(3):
            flush.zero_()
            plan_f.forward_timed_raw(ptrs, y.data_ptr(), ws_f.data_ptr(), s, [e.cuda_event for e in evf[k]])
        torch.cuda.synchronize()
        fk = {fnames[i]: statistics.mean(evf[k][i].elapsed_time(evf[k][i + 1]) for k in range(3))
              for i in range(len(fnames))}
        s_in_f = 2 if w.dtype == "bf16" else 4
        s_out_f = {"bf16": 2, "f16": 2, "f32": 4}[out_name]
        fused = {"ms_per_step": f_ms, "value": job_throughput(world, w.B * w.T, f_ms), "unit": UNIT,
                 "steps": n_f, "launches_per_step": plan_f.launches, "kernels_ms": fk,
                 "workspace_bytes": plan_f.workspace_bytes,
                 "path_frac": path_roofline(w, s_in_f, s_out_f, f_ms, load_peaks())["frac"]}
        del ws_f

    # the layer with its projections (gdn_block_forward) at this workload's shape, model width
    # D = H * d (the Wan2.1-1.3B / Wan2.2-5B widths): input projection with the fused conv / SiLU /
    # L2 epilogue, the tensor path, output projection
    block = None
    if not args.no_block and plan.uses_tensor_path and w.H % 2 == 0:
        block = bench_block(w, dev, flush, stream, max(5, min(args.steps, 20)), world, dist)

    # the other four seeded workloads (rank 0 alone, 1 GPU): same step, flush and event timing
    configs = None
    if world == 1 and not args.no_configs and not args.T:
        configs = {}
        del ws, y
        torch.cuda.empty_cache()
        for wo in gdn_inputs.WORKLOADS:
            if wo.name != w.name:
                configs[wo.name] = bench_other_config(wo, dev, flush, stream, max(5, min(args.steps, 20)),
                                                      0.0 if args.no_cpu_baseline else 5.0)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    peaks = load_peaks()
    s_in = 2 if w.dtype == "bf16" else 4
    s_out = {"bf16": 2, "f16": 2, "f32": 4}[out_name]
    tokens = w.B * w.T
    path_roof = path_roofline(w, s_in, s_out, ms_per_step, peaks)
    # the dominant kernel against the method's roofline (the per-unit figures of the whole path,
    # 1288 B and 180,224 flops per token-head, times the token-heads the launch covers); the
    # kernel's own HBM bytes beside them
    top = max(kern_ms, key=kern_ms.get)
    units = launch_units(top, w, plan)
    pb, pf = path_roof["bytes_per_token_head"], path_roof["flops_per_token_head"]
    t_top = kern_ms[top] / 1e3
    ach_gbs = pb * units / t_top / 1e9
    ach_tfs = pf * units / t_top / 1e12
    kb, kf = kernel_work_per_token_head(top, w.d, s_in, s_out)
    traffic = ncu_traffic(top, w.name)
    # the whole forward's DRAM bytes (every kernel's capture, while all their sources are unchanged)
    path_traffic = None
    kt = [ncu_traffic(n, w.name) for n in names]
    if all(x is not None for x in kt):
        path_traffic = {"bytes_per_step": int(sum(kt)), "per_kernel": {n: int(x) for n, x in zip(names, kt)},
                        "algorithmic_bytes_per_step": int(path_bytes_per_token_head(w.d, s_in, s_out) * w.B * w.T * w.H),
                        "ratio": sum(kt) / (path_bytes_per_token_head(w.d, s_in, s_out) * w.B * w.T * w.H)}
    roof = {"bound": "hbm", "achieved": ach_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": ach_gbs / peaks["hbm_gbs"], "traffic": traffic,
            "peak_source": ("measured (MEASURED_PEAKS.json)" if peaks["source"] == "measured" else "fallback"),
            "kernel": top, "avg_launch_ms": kern_ms[top], "units_per_launch": units,
            "algorithmic_bytes_per_launch": pb * units, "algorithmic_flops_per_launch": pf * units,
            "tensor_frac": ach_tfs / peaks["bf16_tflops"], "kernel_bytes_per_launch": kb * units,
            "kernel_mma_flops_per_launch": kf * units, "path_frac": path_roof["frac"]}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(w)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16-mma/f32" if plan.uses_tensor_path else "f32", "data": "synthetic",
            "config": workload_config(w, args.out_dtype, world),
            "path": "fused tensor (FLAG_FUSED)" if args.fused else ("tensor" if plan.uses_tensor_path else "CUDA-core fp32"),
            "roofline": roof, "path_roofline": path_roof, "path_roofline_frac": path_roof["frac"],
            "path_traffic": path_traffic,
            "kernels_ms": kern_ms,
            "segments": plan.segments, "cpu_baseline": cpu, "e2e": e2e, "state_io": state_io,
            "reverse": reverse, "backward": bwd, "fused": fused, "graph": graph, "block": block,
            "configs": configs,
            "clocks": clocks, "gpu_launches": L * args.steps,
            "step_ms": {"min": min(step_ms), "median": statistics.median(step_ms), "max": max(step_ms)},
            "other_gpu_processes": None if others_before is None or others_after is None
            else sorted(set(others_before) | set(others_after)),
            "gpu": torch.cuda.get_device_name(dev)}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
