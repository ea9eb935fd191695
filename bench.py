"""Benchmark of the Mixtral sparse-MoE block forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole hot path (router + TopK + softmax, permute, both expert GEMMs,
gated combine; for stacked workloads RMSNorm and the residual add, in every block) over one
batch of seeded synthetic input of the workload's shapes.  Default workload: the largest
single-GPU configuration, 32 stacked Mixtral MoE blocks (RMSNorm -> MoE -> residual,
attention omitted) on T=8192 tokens, d=4096, F=14336, n=8, K=2, bf16, ~90 GB of weights.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a device
synchronisation, timed with CUDA events on the launching stream, max over ranks.  The expert
weights (2.8 GB per layer) exceed the 126 MB L2, so no flush is needed between steps.
  value   tokens/s of all ranks with inputs resident in HBM (moe_forward / moe_stack_forward);
  e2e     the same through the host-I/O entry points (moe_forward_host_io /
          moe_stack_forward_host_io) with pinned host x / out, host<->device copies and a
          per-step synchronisation inside the timed region;
  roofline  the dominant kernel (the gate/up expert GEMM), its duration from events the
          library records on its own stream around each stage (of every block);
  parity  the benched workload's GPU result against the oracle on the CPU-baseline leg's
          token sample (for the stack: block 1 on the GPU's own input).
With N > 1 (torchrun) every rank runs an independent replica on its own batch (the block
has no exchange step on one node's data-parallel path): weak scaling.

--impl reference times the CPU oracle (plain C, fp64, OpenMP) on the host cores on the same
workload's metric, each step a bounded sample of tokens (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import moe_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s and TFLOP/s (bf16, top-2 of 8) as % of B200 roofline"
DEFAULT_WORKLOAD = "stack32_t8192"

# DRAM bytes (read + write) of one launch of the dominant kernel (G13), from one ncu capture
# of that kernel on the workload's shapes (for the stack: one T=8192 block), valid only for
# the kernel source it was taken on (hash of csrc/gemm_tc.cu + csrc/common.cuh).
TRAFFIC = {
    "stack32_t8192": {"bytes": 2961393408, "src": "f189b48f7381"},
    "decode_t16": {"bytes": 1885246976, "src": "f189b48f7381"},
    "decode_t16 mxfp8": {"bytes": 971478528, "src": "f189b48f7381"},
    "experts8_top2_t512": {"bytes": 1894018304, "src": "f189b48f7381"},
    # experts8_top2_t512's capture (the same 128 rows per expert) scaled by 8 to n = 64
    "experts64_top2_t4096": {"bytes": 15152146432, "src": "f189b48f7381"},
}


def kernel_source_hash() -> str:
    """Hash of the GEMM kernels' code (csrc/gemm_tc.cu + csrc/common.cuh) with comments and
    blank lines removed, so that the traffic figures stay tied to the code they were taken on
    but survive edits to comments."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "common.cuh"):
        with open(os.path.join(ROOT, "sparse_mixture_experts_18_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
        h.update(code.encode())
    return h.hexdigest()[:12]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"],
                "bf16_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0,
                "source": "fallback"}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return False
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) >= 9:
                self.rows.append(f)
        return False

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4)
                          if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if smax and s > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(self.rows)}


def replica_workload(w, rank: int):
    """Each rank's independent replica: its own seeded batch and weights."""
    return w.replace(seed=w.seed + 7919 * rank)


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings (identity on one rank)."""
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def _flops_per_token(w):
    # routed work: 2 FLOPs per multiply-add; K experts x 3 d-by-F matrices + router d*n
    return w.K * 3 * 2 * w.d * w.F + 2 * w.d * w.n


def run_gpu(args, w):
    import torch.distributed as dist

    import sparse_mixture_experts_18_b200 as moe

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=300))
    peaks = _peaks()
    # per-rank replica: its own batch (seed offset by rank), its own copy of the weights
    wr = replica_workload(w, rank)
    x = moe_inputs.make_x(wr, device=dev)
    layers = [moe_inputs.make_layer(wr, layer=l, device=dev) for l in range(w.layers)]
    layer = layers[0]
    stream = torch.cuda.Stream(device=dev)
    plan = moe.moe_plan_info(w.T, w.d, w.F, w.n, w.K)
    small_batch, s13, s2, launches = (plan["small_batch"], plan["split13"], plan["split2"],
                                      plan["launches"])
    stacked = w.layers > 1
    out = torch.empty_like(x)
    if stacked:  # x is the residual stream: every step restarts from the same input
        ws = moe.alloc_workspace(moe.moe_stack_workspace_bytes(w.T, w.d, w.F, w.n, w.K), dev,
                                 stream)
        # each block: the MoE block and its input's RMSNorm, which the previous block's K = 2
        # combine writes on the large-batch tilings (only the first block launches it then)
        fused_norm = not small_batch and w.T >= 1024 and w.K == 2
        launches = w.layers * launches + (1 if fused_norm else w.layers)
    else:
        ws = moe.alloc_workspace(moe.moe_workspace_bytes(w.T, w.d, w.F, w.n, w.K,
                                                         torch.bfloat16), dev, stream)

    def step():
        if stacked:
            with torch.cuda.stream(stream):
                out.copy_(x, non_blocking=True)
            moe.moe_stack_forward(out, layers, w.K, workspace=ws, stream=stream)
        else:
            moe.moe_forward(x, layer["Wg"], layer["W1"], layer["W3"], layer["W2"], w.K, out=out,
                            workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    # routing of the (first) block on this batch, for the report and the roofline bytes
    ws1 = moe.alloc_workspace(moe.moe_workspace_bytes(w.T, w.d, w.F, w.n, w.K, torch.bfloat16),
                              dev, stream)
    _, idx, _, counts, _, _ = moe.moe_forward_debug(x, layer["Wg"], layer["W1"], layer["W3"],
                                                    layer["W2"], w.K, workspace=ws1,
                                                    stream=stream)
    del ws1
    torch.cuda.synchronize(dev)
    counts = counts.cpu().tolist()
    n_active = sum(1 for c in counts if c > 0)

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        # ---- value: device-resident inputs
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        barrier()
        ms = ev0.elapsed_time(ev1)
        # ---- per-stage durations from events recorded by the library on its stream
        # (stacked: six per block); stage_ms[i] lists (route, G13, reduce, G2, combine) per block
        nev = 6 * w.layers
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)]
               for _ in range(args.steps)]
        for i in range(args.steps):
            for e in evs[i]:
                e.record(stream)  # creates the cudaEvent_t; the library re-records it
            if stacked:
                with torch.cuda.stream(stream):
                    out.copy_(x, non_blocking=True)
                moe.moe_stack_forward_profiled(out, layers, w.K, evs[i], workspace=ws,
                                               stream=stream)
            else:
                moe.moe_forward_profiled(x, layer["Wg"], layer["W1"], layer["W3"], layer["W2"],
                                         w.K, evs[i], out=out, workspace=ws, stream=stream)
        barrier()
        stage_ms = [[evs[i][6 * b + j].elapsed_time(evs[i][6 * b + j + 1]) for j in range(5)]
                    for i in range(args.steps) for b in range(w.layers)]
        del evs
        # ---- e2e: pinned host x in, host out back, every step, through the C-ABI host-I/O
        # entry points
        xh = x.cpu().pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        xd, od = torch.empty_like(x), torch.empty_like(x)

        def e2e_step():
            if stacked:
                moe.moe_stack_forward_host_io(xh, xd, layers, w.K, oh, workspace=ws,
                                              stream=stream)
            else:
                moe.moe_forward_host_io(xh, xd, layer["Wg"], layer["W1"], layer["W3"],
                                        layer["W2"], w.K, od, oh, ws, stream=stream)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            e2e_step()
            stream.synchronize()
        ev1.record(stream)
        barrier()
        e2e_ms = ev0.elapsed_time(ev1)
    code, raw = moe.moe_workspace_status(ws, stream)
    if code != 0:
        raise RuntimeError(f"device status {code} ({raw:#x})")

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None

    ms_step = ms / args.steps
    tok_s = world * w.T * args.steps / (ms / 1e3)
    tflops = tok_s * w.layers * _flops_per_token(w) / 1e12
    g13 = statistics.mean(st[1] for st in stage_ms)       # gate/up GEMM (dominant kernel)
    stage_avg = [statistics.mean(st[j] for st in stage_ms) for j in range(5)]
    es = 2
    timed_s = ms / 1e3
    bf16_peak = peaks["bf16_sustained"] if timed_s > 1.0 else peaks["bf16"]
    # The bound of each is the larger of its two floors: algorithmic bytes at the measured HBM
    # copy rate, algorithmic FLOPs at the measured bf16 GEMM rate.
    rows = w.T * w.K
    bytes13 = n_active * 2 * w.F * w.d * es + rows * w.d * es + rows * w.F * es
    flops13 = 4 * w.d * w.F * rows
    if bytes13 / (peaks["hbm_gbs"] * 1e9) >= flops13 / (bf16_peak * 1e12):
        bound, unit, peak = "hbm", "GB/s", peaks["hbm_gbs"]
        achieved = bytes13 / (g13 / 1e3) / 1e9
    else:
        bound, unit, peak = "tensor", "TFLOP/s", bf16_peak
        achieved = flops13 / (g13 / 1e3) / 1e12
    step_bytes = (w.layers * (n_active * 3 * w.F * w.d * es + w.d * w.n * 4)
                  + 2 * w.T * w.d * es)
    step_hbm = step_bytes / (peaks["hbm_gbs"] * 1e9) >= tflops * ms_step / 1e3 / bf16_peak
    step_frac = (step_bytes / (ms_step / 1e3) / 1e9 / peaks["hbm_gbs"] if step_hbm
                 else tflops / bf16_peak)
    tiling = (f"small-batch swap-AB split-K {s13}/{s2}" if small_batch else
              "CTA-pair 256-row tiles" if plan["pair"] else
              "weight-stationary tiles (128 weight rows x up to 256 token rows)" if plan["mid"]
              else "128-row tiles")
    cap = TRAFFIC.get(w.name)
    traffic = cap["bytes"] if cap and cap["src"] == kernel_source_hash() else None
    workload = workload_label(w)
    line = {
        "metric": METRIC, "value": round(tok_s, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations, RMS-normalised; N(0,1/fan_in) weights)",
        "config": {"workload": workload,
                   "tokens_per_rank": w.T, "l2": "inputs larger than L2 "
                   f"({w.layers * 3 * w.n * w.F * w.d * es / 1e9:.2f} GB of expert weights)",
                   "parallelism": f"replicas x{world}",
                   "tiling": tiling + (", A rows gathered from x" if args.gather_x and plan["pair"]
                                       else ""),
                   "active_experts": n_active, "expert_counts": counts},
        "tflops": round(tflops, 3),
        "pct_roofline": {"bound": "hbm" if step_hbm else "tensor",
                         "frac": round(step_frac, 4),
                         "basis": "unique expert-weight bytes of selected experts per step / "
                                  "measured HBM copy GB/s" if step_hbm else
                                  "routed FLOPs per step / measured bf16 GEMM TFLOP/s"
                                  + (" (sustained)" if bf16_peak == peaks["bf16_sustained"]
                                     else " (burst)")},
        "roofline": {"bound": bound,
                     "kernel": ("tc_pair_gemm" if plan["pair"] else "tc_grouped_gemm")
                               + " G13 (gate/up + SwiGLU)"
                               + (f", every block of {w.layers}" if stacked else ""),
                     "achieved": round(achieved, 2), "peak": peak, "unit": unit,
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": peaks["source"]
                     + (" (sustained)" if unit == "TFLOP/s" and peak == peaks["bf16_sustained"]
                        else " (burst)" if unit == "TFLOP/s" else ""),
                     "launch_ms": round(g13, 5),
                     "launches_timed": len(stage_ms)},
        "stage_ms": {"route": round(stage_avg[0], 5), "gemm13": round(stage_avg[1], 5),
                     "splitk_reduce": round(stage_avg[2], 5), "gemm2": round(stage_avg[3], 5),
                     "combine": round(stage_avg[4], 5)},
        "e2e": {"value": round(world * w.T * args.steps / (e2e_ms / 1e3), 2),
                "unit": "tokens/s", "h2d_bytes_per_step": w.T * w.d * es,
                "d2h_bytes_per_step": w.T * w.d * es,
                "api": "moe_stack_forward_host_io" if stacked else "moe_forward_host_io"},
        "gpu_launches": launches * args.steps,
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline:
        # GPU result the CPU-baseline leg checks its oracle sample against: the first block
        if stacked:
            gpu1 = x.clone()
            moe.moe_stack_forward(gpu1, layers[:1], w.K, workspace=ws, stream=stream)
        else:
            gpu1 = out
        torch.cuda.synchronize(dev)
        line["cpu_baseline"], line["parity"] = cpu_baseline(
            w, x.cpu(), {k: v.cpu() for k, v in layer.items()}, args.cpu_tokens,
            gpu_out=gpu1.float().cpu())
    del layers
    print(json.dumps(line), flush=True)
    return line


def workload_label(w) -> str:
    """config.workload string, shared by both arms of the benchmark."""
    return (f"{w.name}: T={w.T} d={w.d} F={w.F} n={w.n} K={w.K} bf16"
            + (f", {w.layers} x (RMSNorm -> MoE -> residual)" if w.layers > 1 else ""))


def run_gpu_fp8(args, w):
    """The FP8-weight variant (MXFP8 expert weights: E4M3 codes, an E8M0 scale per 32
    elements) on a small-batch workload:
    same step, timing and JSON line as run_gpu, one GPU (replicas as run_gpu for N > 1)."""
    import torch.distributed as dist

    import sparse_mixture_experts_18_b200 as moe

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=300))
    peaks = _peaks()
    wr = replica_workload(w, rank)
    x = moe_inputs.make_x(wr, device=dev)
    layer = moe_inputs.make_layer(wr, device=dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        q = {k: moe.moe_quantize_mx_e4m3(layer[k], stream=stream) for k in ("W1", "W3", "W2")}
    Wg = layer["Wg"]
    del layer
    args_q = (q["W1"][0], q["W3"][0], q["W2"][0], q["W1"][1], q["W3"][1], q["W2"][1])
    nbytes = moe.moe_workspace_bytes_fp8(w.T, w.d, w.F, w.n, w.K)
    if nbytes == 0:
        raise SystemExit(f"{w.name}: the FP8-weight block covers small-batch shapes only")
    ws = moe.alloc_workspace(nbytes, dev, stream)
    out = torch.empty_like(x)
    plan = moe.moe_plan_info(w.T, w.d, w.F, w.n, w.K)

    def step():
        moe.moe_forward_fp8(x, Wg, *args_q, w.K, out=out, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        barrier()
        ms = ev0.elapsed_time(ev1)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)]
               for _ in range(args.steps)]
        for i in range(args.steps):
            for e in evs[i]:
                e.record(stream)
            moe.moe_forward_fp8(x, Wg, *args_q, w.K, out=out, workspace=ws, stream=stream,
                                events=evs[i])
        barrier()
        stage_ms = [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(5)]
                    for i in range(args.steps)]
        xh = x.cpu().pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        xd = torch.empty_like(x)

        def e2e_step():  # pinned host x in, the block, host out back
            with torch.cuda.stream(stream):
                xd.copy_(xh, non_blocking=True)
            moe.moe_forward_fp8(xd, Wg, *args_q, w.K, out=out, workspace=ws, stream=stream)
            with torch.cuda.stream(stream):
                oh.copy_(out, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        barrier()
        ev0.record(stream)
        for _ in range(args.steps):
            e2e_step()
            stream.synchronize()
        ev1.record(stream)
        barrier()
        e2e_ms = ev0.elapsed_time(ev1)
    code, raw = moe.moe_workspace_status(ws, stream)
    if code != 0:
        raise RuntimeError(f"device status {code} ({raw:#x})")
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None
    # active experts of this batch, from the bf16 router on the host (routing is shared)
    l = x.float().cpu() @ Wg.float().cpu()
    n_active = int(torch.unique(torch.topk(l, w.K, dim=1).indices).numel())
    ms_step = ms / args.steps
    tok_s = world * w.T * args.steps / (ms / 1e3)
    g13 = statistics.mean(st[1] for st in stage_ms)
    stage_avg = [statistics.mean(st[j] for st in stage_ms) for j in range(5)]
    # E4M3 codes plus one E8M0 scale byte per 32 of them
    bytes13 = n_active * 2 * w.F * w.d * 33 // 32 + w.T * w.K * w.d * 33 // 32
    step_bytes = n_active * 3 * w.F * w.d * 33 // 32 + w.d * w.n * 4 + 2 * w.T * w.d * 2
    achieved = bytes13 / (g13 / 1e3) / 1e9
    cap = TRAFFIC.get(w.name + " mxfp8")
    traffic = cap["bytes"] if cap and cap["src"] == kernel_source_hash() else None
    line = {
        "metric": METRIC + " -- FP8 (MXFP8) expert-weight variant", "value": round(tok_s, 2),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "mxfp8 (e4m3 + e8m0 per 32) weights and activations, fp32 accumulate, bf16 out",
        "data": "synthetic (seeded N(0,1) activations, RMS-normalised; N(0,1/fan_in) weights "
                "quantised to MXFP8 on the device)",
        "config": {"workload": f"{w.name}: T={w.T} d={w.d} F={w.F} n={w.n} K={w.K}, "
                               "MXFP8 expert weights",
                   "tokens_per_rank": w.T,
                   "l2": f"inputs larger than L2 ({3 * w.n * w.F * w.d / 1e9:.2f} GB of E4M3 "
                         "expert-weight codes)",
                   "parallelism": f"replicas x{world}",
                   "tiling": f"small-batch swap-AB split-K {plan['split13']}/{plan['split2']}, "
                             "tcgen05 kind::mxf8f6f4 block_scale", "active_experts": n_active},
        "pct_roofline": {"bound": "hbm", "frac": round(step_bytes / (ms_step / 1e3) / 1e9 /
                                                       peaks["hbm_gbs"], 4),
                         "basis": "E4M3 weight bytes (+ block scales) of selected experts per "
                                  "step / measured HBM copy GB/s"},
        "roofline": {"bound": "hbm", "kernel": "tc_grouped_gemm G13 (MXFP8)",
                     "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": traffic, "peak_source": peaks["source"],
                     "launch_ms": round(g13, 5)},
        "stage_ms": {"route": round(stage_avg[0], 5), "gemm13": round(stage_avg[1], 5),
                     "swiglu_quantize": round(stage_avg[2], 5),
                     "gemm2": round(stage_avg[3], 5), "combine": round(stage_avg[4], 5)},
        "e2e": {"value": round(world * w.T * args.steps / (e2e_ms / 1e3), 2),
                "unit": "tokens/s", "h2d_bytes_per_step": w.T * w.d * 2,
                "d2h_bytes_per_step": w.T * w.d * 2},
        "gpu_launches": 5 * args.steps,
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    return line


NVLINK_GBS = 770.0  # measured peer copy per direction per GPU on this kind of node (GB/s)


def run_ep_emulation(args, w):
    """Expert parallelism over R ranks, emulated on one GPU.  Every virtual rank routes its own
    batch (the workload with its own seed).  Experts are placed contiguously (n / R per rank),
    or with --ep-slots C > n / R hot experts are replicated (ep.ExpertPlacement.balanced over
    the global loads) and each source splits a replicated expert's rows evenly over its
    replicas.  The ranks' GPU stages run one after another on this GPU and are timed with CUDA
    events: moe_route (and the row gather into destination order when experts are
    replicated) per rank; moe_experts_forward per rank on the rows it receives from every
    source; the row gather back into grouped order and moe_combine per rank.  The two
    all-to-alls are not run (one GPU): their time is modelled from the bytes each rank sends
    and receives at the peer-copy rate NVLINK_GBS.  The modelled step is the slowest rank's
    route + dispatch + slowest experts stage + return + slowest combine, nothing overlapped."""
    import sparse_mixture_experts_18_b200 as moe
    from sparse_mixture_experts_18_b200 import ep

    R = args.ep_emulate
    if w.n % R:
        raise SystemExit(f"{w.name}: n = {w.n} experts do not split over {R} ranks")
    slots = args.ep_slots or w.n // R
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    layer = moe_inputs.make_layer(w, device=dev)
    xs = [moe_inputs.make_x(replica_workload(w, r), device=dev) for r in range(R)]
    Wg = layer["Wg"]
    es = xs[0].element_size()
    dt = 1 if xs[0].dtype == torch.bfloat16 else 0
    lib = moe.lib()
    ws_route = [moe.alloc_workspace(int(lib.moe_route_workspace_bytes(w.T, w.d, w.n, w.K, dt)),
                                    dev) for _ in range(R)]
    routed = [moe.moe_route(xs[r], Wg, w.K, workspace=ws_route[r]) for r in range(R)]
    all_counts = torch.stack([r[3] for r in routed]).cpu()
    loads = all_counts.sum(dim=0)
    if slots == w.n // R:
        pl = ep.ExpertPlacement.contiguous(w.n, R)
    else:
        pl = ep.ExpertPlacement.balanced(loads, R, slots)
    plans = [pl.send_order(all_counts[s]) for s in range(R)]
    ident = [order == list(range(len(order))) for order, _ in plans]
    perms = [torch.tensor(o, dtype=torch.int32, device=dev) for o, _ in plans]
    invs = []
    for pm in perms:
        inv = torch.empty_like(pm)
        inv[pm.long()] = torch.arange(len(pm), dtype=torch.int32, device=dev)
        invs.append(inv)
    starts = [[sum(plans[s][1][:q]) for q in range(R + 1)] for s in range(R)]
    segs = [torch.tensor(pl.recv_counts(all_counts, q), dtype=torch.int32, device=dev)
            for q in range(R)]
    rows_q = [int(sg.sum()) for sg in segs]
    local = []
    for q in range(R):
        idx = torch.tensor(pl.local_experts(q), device=dev)
        local.append({k: layer[k][idx].contiguous() for k in ("W1", "W3", "W2")})
    del layer
    ws_exp = [moe.alloc_workspace(int(lib.moe_experts_workspace_bytes(
        max(rows_q[q], 1), w.d, w.F, len(pl.local_experts(q)), dt)), dev) for q in range(R)]
    outs = [torch.empty_like(x) for x in xs]
    t_route = [[] for _ in range(R)]
    t_exp = [[] for _ in range(R)]
    t_comb = [[] for _ in range(R)]

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        res = fn()
        e1.record()
        return res, (e0, e1)

    for it in range(args.warmup + args.steps):
        ev = []
        x_send = [None] * R
        for r in range(R):
            def route_stage(r=r):
                routed[r] = moe.moe_route(xs[r], Wg, w.K, workspace=ws_route[r])
                return routed[r][0] if ident[r] else moe.moe_gather_rows(routed[r][0], perms[r])
            x_send[r], e = timed(route_stage)
            ev.append(("route", r, e))
        # the dispatch, by slicing (untimed): rank q receives its slice of every source
        x_recv = [torch.cat([x_send[s][starts[s][q]:starts[s][q + 1]] for s in range(R)])
                  for q in range(R)]
        y_recv = []
        for q in range(R):
            y, e = timed(lambda q=q: moe.moe_experts_forward(
                x_recv[q], segs[q], local[q]["W1"], local[q]["W3"], local[q]["W2"],
                workspace=ws_exp[q]))
            y_recv.append(y)
            ev.append(("experts", q, e))
        for s in range(R):  # the return, by slicing (untimed)
            parts_s = []
            for q in range(R):
                off = int(segs[q][:s].sum())
                parts_s.append(y_recv[q][off:off + int(segs[q][s].sum())])
            y_send_back = torch.cat(parts_s)

            def combine_stage(s=s, y_send_back=y_send_back):
                y_back = y_send_back if ident[s] else moe.moe_gather_rows(y_send_back, invs[s])
                moe.moe_combine(y_back, routed[s][4], routed[s][2], outs[s])
            _, e = timed(combine_stage)
            ev.append(("combine", s, e))
        torch.cuda.synchronize()
        if it >= args.warmup:
            for kind, r, (e0, e1) in ev:
                {"route": t_route, "experts": t_exp, "combine": t_comb}[kind][r].append(
                    e0.elapsed_time(e1))
    for wsp in ws_route + ws_exp:
        code, raw = moe.moe_workspace_status(wsp)
        if code != 0:
            raise RuntimeError(f"device status {code} ({raw:#x})")
    med = statistics.median
    route_ms = [med(t) for t in t_route]
    exp_ms = [med(t) for t in t_exp]
    comb_ms = [med(t) for t in t_comb]
    # rows that cross NVLink (parts for other ranks only): dispatch bf16 rows, return fp32
    out_rows = [sum(plans[s][1][q] for q in range(R) if q != s) for s in range(R)]
    in_rows = [sum(int(segs[q][s].sum()) for s in range(R) if s != q) for q in range(R)]
    worst = max(max(o, i) for o, i in zip(out_rows, in_rows))
    disp, ret = worst * w.d * es, worst * w.d * 4
    t_disp = disp / (NVLINK_GBS * 1e9) * 1e3
    t_ret = ret / (NVLINK_GBS * 1e9) * 1e3
    step = max(route_ms) + t_disp + max(exp_ms) + t_ret + max(comb_ms)
    flops = 2.0 * 3 * w.d * w.F * w.K * w.T * R
    line = {
        "metric": "expert-parallel MoE block, emulated on one GPU (modelled step)",
        "value": round(R * w.T / (step / 1e3), 2), "unit": "tokens/s", "n_gpus": 1,
        "ranks_emulated": R, "expert_slots_per_rank": slots, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step_modelled": round(step, 5),
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded per rank)",
        "config": {"workload": f"{workload_label(w)}, {R} ranks x {w.T} tokens, "
                               f"{slots} expert slots per rank", "global_batch": R * w.T},
        "placement": [list(r) for r in pl.replicas],
        "stage_ms_per_rank": {"route": [round(v, 5) for v in route_ms],
                              "experts": [round(v, 5) for v in exp_ms],
                              "combine": [round(v, 5) for v in comb_ms]},
        "rows_per_rank": rows_q,
        "exchange": {"dispatch_bytes_max": disp, "return_bytes_max": ret,
                     "dispatch_ms_modelled": round(t_disp, 5),
                     "return_ms_modelled": round(t_ret, 5), "link_GBps": NVLINK_GBS},
        "tflops_modelled": round(flops / (step / 1e3) / 1e12, 1),
        "note": "GPU stages measured one rank after another on one GPU; all-to-alls modelled "
                "at the peer-copy rate, not run",
    }
    print(json.dumps(line), flush=True)
    return line


def _oracle_block(oracle, w, x, layer, toks):
    """The oracle's result for token rows `toks` of the workload's (first) block, rounded to
    bf16 as the GPU's output is: the MoE block, or for stacked workloads one whole block
    x + MoE(RMSNorm(x)).  Also the oracle's router logits of those rows."""
    import numpy as np
    xs = x[toks]
    if w.layers > 1:
        xin = xs.double().numpy()
        ref, _, _ = oracle.block_forward(xin, layer["Wg"], layer["W1"], layer["W3"], layer["W2"],
                                         w.n, w.K, 1e-5)
        xn = torch.from_numpy(oracle.rmsnorm(xin, 1e-5, oracle.BF16)).to(torch.bfloat16)
        logits, _, _ = oracle.route(xn, layer["Wg"], w.n, w.K)
        return ref, logits
    y, _, _ = oracle.moe_forward(x, layer["Wg"], layer["W1"], layer["W3"], layer["W2"], w.n, w.K,
                                 tokens=np.asarray(toks, np.int64))
    logits, _, _ = oracle.route(xs, layer["Wg"], w.n, w.K)
    return oracle.round_array(y, oracle.BF16), logits


def cpu_baseline(w, x, layer, ntok, seconds: float = 10.0, gpu_out=None):
    """The oracle as it stands on the host cores, on a bounded sample of the workload: calls
    of max(ntok, threads) tokens (cycling through the batch) repeated for about `seconds`;
    for stacked workloads the oracle runs one whole block and the rate is divided by the
    number of blocks.  Returns (baseline dict, parity dict): the parity dict compares the
    oracle's results for the tokens it evaluated with gpu_out (the GPU's result of the same
    block on the same input) -- max-abs and relative L2 error over the tokens whose K-th and
    (K+1)-th oracle logits are more than 1e-4 apart (relative), and the count of those that
    are not (exempt near-ties, whose expert set either way is correct)."""
    import numpy as np

    import oracle
    oracle.build()
    threads = _omp_threads()
    chunk = max(1, min(max(ntok, threads), w.T))
    done, start = 0, 0
    refs = {}
    t0 = time.perf_counter()
    while True:
        toks = [(start + j) % w.T for j in range(chunk)]
        ref, logits = _oracle_block(oracle, w, x, layer, toks)
        for j, t in enumerate(toks):
            refs.setdefault(t, (ref[j], logits[j]))
        done += chunk
        start = (start + chunk) % w.T
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    blocks = f", one whole block of the {w.layers} (rate divided by {w.layers})" \
        if w.layers > 1 else ""
    base = {"value": round(done / dt / w.layers, 4), "unit": "tokens/s",
            "cores": min(chunk, threads), "kind": "oracle",
            "sample": f"{done} token evaluations in calls of {chunk} (cycling over the {w.T} "
                      f"tokens of {w.name}){blocks}, {dt:.1f} s (fp64 C, OpenMP over tokens)"}
    if gpu_out is None:
        return base, None
    toks = sorted(refs)
    exempt, err, refn = 0, [], []
    for t in toks:
        r, l = refs[t]
        srt = np.sort(l)[::-1]
        a, b = srt[w.K - 1], srt[w.K] if w.K < w.n else -np.inf
        if w.K < w.n and abs(a - b) <= 1e-4 * max(abs(a), abs(b)):
            exempt += 1
            continue
        err.append(gpu_out[t].double().numpy() - r)
        refn.append(r)
    err, refn = np.array(err), np.array(refn)
    max_abs = float(np.max(np.abs(err))) if err.size else 0.0
    rel_l2 = float(np.linalg.norm(err) / max(np.linalg.norm(refn), 1e-300)) if err.size else 0.0
    allow = 2e-2 + (2.0 ** -7 * np.abs(refn) if w.layers > 1 else 0.0)
    par = {"what": ("block 1 of the stack (RMSNorm -> MoE -> residual) on the GPU's input"
                    if w.layers > 1 else "the block's output") + ", oracle in fp64",
           "tokens": len(toks), "exempt": exempt, "max_abs": max_abs, "rel_l2": rel_l2,
           "ok": bool(err.size == 0 or (np.all(np.abs(err) <= allow) and rel_l2 <= 5e-3)),
           "bars": "max-abs 2e-2" + (" + 2^-7 |ref|" if w.layers > 1 else "")
                   + ", rel-L2 5e-3; exempt: 2nd-vs-3rd logit gap <= 1e-4 relative"}
    return base, par


def _omp_threads():
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else (len(os.sched_getaffinity(0))
                                             if hasattr(os, "sched_getaffinity")
                                             else os.cpu_count())


def run_reference(args, w):
    """Reference arm: the CPU oracle timed on the host cores (rank 0 only), on the same
    workload, metric and unit as the GPU arm; each step a bounded sample of tokens of the
    (first) block, for stacked workloads one whole block with the rate divided by the number
    of blocks."""
    world, rank, _ = _dist()
    if rank != 0:
        return None
    import oracle
    oracle.build()
    x = moe_inputs.make_x(w)
    layer = moe_inputs.make_layer(w)
    threads = _omp_threads()
    per_step = min(w.T, max(args.cpu_tokens, threads))  # a token for every host thread
    for i in range(args.warmup):
        _oracle_block(oracle, w, x, layer, [i % w.T])
    t0 = time.perf_counter()
    for i in range(args.steps):
        toks = [(i * per_step + j) % w.T for j in range(per_step)]
        _oracle_block(oracle, w, x, layer, toks)
    dt = time.perf_counter() - t0
    v = per_step * args.steps / dt / w.layers
    sample = (f"{per_step} of {w.T} tokens of {w.name} per step "
              "(fp64 C oracle, OpenMP over tokens)"
              + (f"; one whole block, rate divided by {w.layers} blocks" if w.layers > 1 else ""))
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_label(w)},
            "cpu_baseline": {"value": round(v, 4), "unit": "tokens/s",
                             "cores": min(per_step, threads), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return line


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(moe_inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=4,
                    help="tokens per oracle sample (CPU baseline / reference arm)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "e4m3"],
                    help="e4m3: the FP8 expert-weight variant (small-batch workloads)")
    ap.add_argument("--layers", type=int, default=None,
                    help="run only the first N blocks of a stacked workload (N=1: one MoE "
                         "block of its shape), e.g. for an ncu capture of a few GB")
    ap.add_argument("--ep-emulate", type=int, default=0, metavar="R",
                    help="expert parallelism over R ranks emulated on one GPU: measured GPU "
                         "stages per rank, all-to-alls modelled from their bytes")
    ap.add_argument("--ep-slots", type=int, default=0, metavar="C",
                    help="with --ep-emulate: expert slots per rank; more than n / R replicates "
                         "the hot experts (balanced placement over the measured loads)")
    ap.add_argument("--gather-x", action="store_true",
                    help="CTA-pair path: gather G13's A rows from x (TMA gather4) instead of "
                         "X_perm, gates applied in G2 (sets MOE_GATHER_X=1)")
    args = ap.parse_args(argv)
    if args.gather_x:
        os.environ["MOE_GATHER_X"] = "1"
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = moe_inputs.WORKLOADS[args.workload]
    if args.layers is not None:
        if not 1 <= args.layers <= w.layers:
            ap.error(f"--layers must be in 1..{w.layers} for {w.name}")
        w = w.replace(layers=args.layers)
    if w.dtype != "bf16":
        ap.error("the bench measures the bf16 path")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.ep_emulate:
        return run_ep_emulation(args, w)
    if args.weights == "e4m3":
        return run_gpu_fp8(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    main()
