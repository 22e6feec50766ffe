#!/usr/bin/env python
"""Benchmark of the quantization hot path on B200: one JSON line on stdout.

A *step* is one pass of every hot-path kernel over the 70B-class W4A16 layer
(28672x8192 up and 8192x28672 down fp16 weights, N(0, 0.015), activations with
0.5% outlier channels x100) and the W8A8 SmoothQuant layer (X [2048, 8192] with
64 outlier channels x60, W [8192, 8192]):

  INT4 group quantizer on both weights          (fresh outputs)
  W4A16 GEMV, batch 1, on both weights          (the headline: HBM GB/s)
  W4A16 tensor-core GEMM, batch 16 and 64, on both weights
  INT8 per-channel quantizer on both weights + W8A16 GEMV, batch 1
  SmoothQuant factors, INT8 per-channel (W*s) and per-token (X/s) quantizers
  W8A8 INT8 tensor-core GEMM                    (the second headline: TOPS)

Every input lives in HBM before the timed region; the matmuls read packed
weights that no kernel of the step has touched since the previous step, and
the step streams several GB, so no kernel reads its operands from L2.  Kernel
times come from CUDA events on the launching stream.  `value` is the batch-1
W4A16 GEMV's algorithmic bytes / its device time over all ranks; the W8A8
GEMM's INT8 TOPS ride along in `w8a8`.

--impl reference times the CPU oracle (single-threaded C) on a bounded sample
of the same workload instead.  With torchrun (N > 1) every rank runs an
independent replica (the path has no exchange step); rank 0 prints.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W4A16 GEMV achieved HBM GB/s (% of peak) + W8A8 GEMM INT8 TOPS (% of peak)"
WORKLOAD = "llama70b_class_w4a16_layer+w8a8_smoothquant_2048x8192x8192"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
UP, DOWN = (28672, 8192), (8192, 28672)
W8A8_SHAPE = (2048, 8192, 8192)
LLM_THRESHOLD, LLM_CAP = 6.0, 64      # LLM.int8(): outlier threshold and carved-column capacity
# nominal dense tensor throughput relative to bf16 (FP8/INT8 2x, FP4 4x)
TENSOR_RATIO = {"gemm_w8a8": 2.0, "gemm_fp8": 2.0, "gemm_llm_int8": 2.0, "gemm_mxfp4": 4.0, "gemm_nvfp4": 4.0}


# ----------------------------------------------------------------------------- peaks
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ----------------------------------------------------------------------------- algorithmic work
def packed_bytes(N, K, g=128):
    return N * K // 2 + 2 * N * (K // g) + 4 * N * ((K // g + 7) // 8)


def work_table():
    """Algorithmic bytes (HBM) and ops per launch of each kernel in a step."""
    t = {}
    for tag, (N, K) in (("up", UP), ("down", DOWN)):
        t[f"quant_int4_{tag}"] = {"bytes": 2 * N * K + packed_bytes(N, K), "ops": 0}
        t[f"gemv_w4a16_b1_{tag}"] = {"bytes": packed_bytes(N, K) + 2 * K + 2 * N, "ops": 2 * N * K}
        for M in (16, 64):
            t[f"gemm_w4a16_m{M}_{tag}"] = {"bytes": packed_bytes(N, K) + 2 * M * K + 2 * M * N, "ops": 2 * M * N * K}
        t[f"quant_int8_pc_{tag}"] = {"bytes": 3 * N * K + 4 * N, "ops": 0}
        t[f"gemv_w8a16_b1_{tag}"] = {"bytes": N * K + 4 * N + 2 * K + 2 * N, "ops": 2 * N * K}
    M, N, K = W8A8_SHAPE
    # FP8 E4M3 W8A8 (per-token X, per-channel W), LLM.int8() and block-scaled FP4 on the same layer
    t["quant_fp8_w"] = {"bytes": 3 * N * K + 4 * N, "ops": 0}
    t["quant_fp8_x"] = {"bytes": 3 * M * K + 4 * M, "ops": 0}
    t["gemm_fp8"] = {"bytes": M * K + N * K + 4 * (M + N) + 2 * M * N, "ops": 2 * M * N * K}
    t["llm_outlier_columns"] = {"bytes": 2 * M * K + 4 * K, "ops": 0}
    t["llm_quant_x"] = {"bytes": 3 * M * K + 4 * M + 4 * K, "ops": 0}
    t["llm_gather"] = {"bytes": 4 * (M + N) * LLM_CAP + 4 * LLM_CAP, "ops": 0}
    t["gemm_llm_int8"] = {"bytes": M * K + N * K + 4 * (M + N) + 2 * (M + N) * LLM_CAP + 2 * M * N,
                          "ops": 2 * M * N * (K + LLM_CAP)}
    for fmt, bs in (("mxfp4", 32), ("nvfp4", 16)):
        t[f"quant_{fmt}_w"] = {"bytes": 2 * N * K + N * K // 2 + N * K // bs, "ops": 0}
        t[f"quant_{fmt}_x"] = {"bytes": 2 * M * K + M * K // 2 + M * K // bs, "ops": 0}
        t[f"gemm_{fmt}"] = {"bytes": (M + N) * (K // 2 + K // bs) + 2 * M * N, "ops": 2 * M * N * K}
    t["smooth"] = {"bytes": 2 * (M + N) * K + 4 * K, "ops": 0}
    t["quant_int8_pc_smooth"] = {"bytes": 3 * N * K + 4 * N + 4 * K, "ops": 0}
    t["quant_int8_pt_smooth"] = {"bytes": 3 * M * K + 4 * M + 4 * K, "ops": 0}
    t["gemm_w8a8"] = {"bytes": M * K + N * K + 4 * (M + N) + 2 * M * N, "ops": 2 * M * N * K}
    return t


def roofline_for(name, us, work, peaks):
    """Achieved rate against the kernel's binding roofline (measured peaks)."""
    hbm = peaks["hbm_gbs"]
    f16 = peaks["bf16_tflops"]                 # fp16 dense = bf16
    b, ops = work["bytes"], work["ops"]
    if name in TENSOR_RATIO:
        peak = TENSOR_RATIO[name] * peaks["bf16_tflops"]
        ach = ops / (us * 1e-6) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TOPS", "frac": ach / peak}
    if name.startswith("gemm_w4a16"):
        t_mem, t_tc = b / (hbm * 1e9), ops / (f16 * 1e12)
        if t_tc > t_mem:
            ach = ops / (us * 1e-6) / 1e12
            return {"bound": "tensor", "achieved": ach, "peak": f16, "unit": "TFLOP/s", "frac": ach / f16}
    ach = b / (us * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, period_ms=20):
        self.index, self.period_ms, self.rows, self.proc = index, period_ms, [], None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = [r for (t, r) in self.rows if t0 - 0.05 <= t <= t1 + 0.05 and len(r) >= 9]
        if not rows:
            rows = [r for (_, r) in self.rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- distributed
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def reduce_max(values, world, device=None):
    """Element-wise max over ranks (identity for world == 1)."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_value(bytes_per_rank_step, steps, world, max_time_s):
    """Whole-job GB/s: units all ranks processed / max-over-ranks time."""
    return bytes_per_rank_step * steps * world / max_time_s / 1e9


# ----------------------------------------------------------------------------- GPU arm
def make_inputs(torch, dev):
    import workloads
    ins = {}
    for tag, (N, K), si in (("up", UP, 0), ("down", DOWN, 1)):
        w = workloads.config_weight("llama70b_class", si)
        ins[f"w_{tag}"] = torch.from_numpy(w).to(dev)
        del w
        for B in (1, 16, 64):
            ins[f"x{B}_{tag}"] = torch.from_numpy(workloads.config_activations("llama70b_class", B, K)).to(dev)
    M, N, K = W8A8_SHAPE
    ins["x_w8a8"] = torch.from_numpy(workloads.config_activations("w8a8_smoothquant", M, K)).to(dev)
    ins["w_w8a8"] = torch.from_numpy(workloads.config_weight("w8a8_smoothquant")).to(dev)
    return ins


class Step:
    """Buffers and launches of one hot-path step, with per-kernel CUDA events."""

    def __init__(self, torch, wq, ins):
        self.torch, self.wq, self.ins = torch, wq, ins
        self.names = []
        # read-side packed weights (previous "model state"), never written inside a step
        self.qB = {t: wq.quantize_group_int4(ins[f"w_{t}"], 128) for t in ("up", "down")}
        self.q8B = {t: wq.quantize_int8_per_channel(ins[f"w_{t}"]) for t in ("up", "down")}
        self.w8_plain = wq.quantize_int8_per_channel(ins["w_w8a8"])  # LLM.int8() weights (no smoothing)
        torch.cuda.synchronize()
        self.ws = torch.empty(wq.smooth_workspace_bytes(W8A8_SHAPE[2]), dtype=torch.uint8, device=ins["x_w8a8"].device)
        self.out = {}

    def launches(self):
        """The step's kernels, ordered so that no matmul finds its operands in L2: the batch-1
        GEMVs run after the 470 MB INT8 weight stream of the W8A16 GEMVs (clean lines), and
        every packed weight read was last touched a full step earlier or before that stream."""
        wq, ins, qB, q8B = self.wq, self.ins, self.qB, self.q8B
        L = []
        for t in ("up", "down"):
            L.append((f"quant_int4_{t}", lambda t=t: wq.quantize_group_int4(ins[f"w_{t}"], 128)))

        def smooth():
            self.out["s"] = wq.smooth(ins["x_w8a8"], ins["w_w8a8"], 0.5, workspace=self.ws)

        def q_w():
            self.out["wq_w8a8"] = wq.quantize_int8_per_channel(ins["w_w8a8"], self.out["s"])

        def q_x():
            self.out["xq_w8a8"] = wq.quantize_int8_per_token(ins["x_w8a8"], self.out["s"])

        def w8a8():
            xq, sx = self.out["xq_w8a8"]
            w8, sw = self.out["wq_w8a8"]
            self.out["y5"] = wq.gemm_w8a8(xq, sx, w8, sw)

        L += [("smooth", smooth), ("quant_int8_pc_smooth", q_w), ("quant_int8_pt_smooth", q_x), ("gemm_w8a8", w8a8)]
        X, W = ins["x_w8a8"], ins["w_w8a8"]
        o = self.out

        # FP8 E4M3 W8A8: W first, so that its 200 MB stream evicts X from L2 before X is read
        def fp8_w():
            o["fp8_w"] = wq.quantize_fp8_e4m3(W, per_row=True)

        def fp8_x():
            o["fp8_x"] = wq.quantize_fp8_e4m3(X, per_row=True)

        def fp8_gemm():
            o["y_fp8"] = wq.gemm_fp8(o["fp8_x"][0], o["fp8_x"][1], o["fp8_w"][0], o["fp8_w"][1])

        # LLM.int8(): weights are the plain per-channel INT8 codes of W (model state, made once)
        def llm_cols():
            o["llm_cols"] = wq.outlier_columns(X, LLM_THRESHOLD, LLM_CAP)

        def llm_qx():
            o["llm_x"] = wq.quantize_int8_per_channel(X, o["llm_cols"][2])

        def llm_gather():
            idx, count, _ = o["llm_cols"]
            o["llm_16"] = wq.gather_outliers(X, self.w8_plain[0], idx, count, LLM_CAP)

        def llm_gemm():
            xq, sx = o["llm_x"]
            o["y_llm"] = wq.gemm_w8a8_outliers(xq, sx, self.w8_plain[0], self.w8_plain[1], *o["llm_16"])

        L += [("quant_fp8_w", fp8_w), ("quant_fp8_x", fp8_x), ("gemm_fp8", fp8_gemm), ("llm_outlier_columns", llm_cols),
              ("llm_quant_x", llm_qx), ("llm_gather", llm_gather), ("gemm_llm_int8", llm_gemm)]
        for fmt in ("mxfp4", "nvfp4"):
            qf = wq.quantize_mxfp4 if fmt == "mxfp4" else wq.quantize_nvfp4

            def q_w(qf=qf, fmt=fmt):
                o[f"{fmt}_w"] = qf(W)

            def q_x(qf=qf, fmt=fmt):
                o[f"{fmt}_x"] = qf(X)

            def mm(fmt=fmt):
                a, b = o[f"{fmt}_x"], o[f"{fmt}_w"]
                o[f"y_{fmt}"] = wq.gemm_fp4(a[0], a[1], b[0], b[1], *((a[2], b[2]) if fmt == "nvfp4" else ()))

            L += [(f"quant_{fmt}_w", q_w), (f"quant_{fmt}_x", q_x), (f"gemm_{fmt}", mm)]
        for t in ("up", "down"):
            L.append((f"quant_int8_pc_{t}", lambda t=t: wq.quantize_int8_per_channel(ins[f"w_{t}"])))
        for M in (16, 64):
            for t in ("up", "down"):
                L.append((f"gemm_w4a16_m{M}_{t}", lambda t=t, M=M: wq.gemm_w4a16(ins[f"x{M}_{t}"], *qB[t], 128)))
        for t in ("up", "down"):
            L.append((f"gemv_w8a16_b1_{t}", lambda t=t: wq.gemv_w8a16(ins[f"x1_{t}"], *q8B[t])))
        for t in ("up", "down"):
            L.append((f"gemv_w4a16_b1_{t}", lambda t=t: wq.gemv_w4a16(ins[f"x1_{t}"], *qB[t], 128)))
        return L


def run_gpu(args):
    import torch
    import bit_gemv_gemm_group_b200 as wq

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    ins = make_inputs(torch, dev)
    step = Step(torch, wq, ins)
    launches = step.launches()
    names = [n for n, _ in launches]
    work = work_table()
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[dev.index])
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        for _, fn in launches:
            fn()
    barrier()
    if wq.device_status() != 0:
        raise RuntimeError("a kernel reported a wait timeout during warm-up")

    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in launches]
           for _ in range(args.steps)]
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    barrier()
    t_wall0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # A 50 ms spin (before the timed region) lets the host queue the step's launches ahead of the
    # GPU, so the per-kernel events bracket device work rather than host launch gaps.
    torch.cuda._sleep(int(0.05 * 1.9e9))
    start.record(stream)
    for k in range(args.steps):
        for (name, fn), (e0, e1) in zip(launches, evs[k]):
            e0.record(stream)
            fn()
            e1.record(stream)
    end.record(stream)
    barrier()
    t_wall1 = time.time()
    sampler.stop()
    if wq.device_status() != 0:
        raise RuntimeError("a kernel reported a wait timeout in the timed region")
    total_ms = start.elapsed_time(end)
    per_kernel_us = {n: [] for n in names}
    for k in range(args.steps):
        for n, (e0, e1) in zip(names, evs[k]):
            per_kernel_us[n].append(e0.elapsed_time(e1) * 1e3)
    mean_us = {n: statistics.median(v) for n, v in per_kernel_us.items()}  # median device time per launch

    # max over ranks of the timed region and of each kernel's summed time
    red = reduce_max([total_ms] + [sum(per_kernel_us[n]) for n in names], world, dev)
    total_ms_max, kernel_tot_us_max = red[0], dict(zip(names, red[1:]))

    gemv = [n for n in names if n.startswith("gemv_w4a16_b1")]
    gemv_bytes = sum(work[n]["bytes"] for n in gemv)
    gemv_time_s = sum(kernel_tot_us_max[n] for n in gemv) * 1e-6
    value = aggregate_value(gemv_bytes, args.steps, world, gemv_time_s)
    w8a8_s = kernel_tot_us_max["gemm_w8a8"] * 1e-6
    w8a8_tops = work["gemm_w8a8"]["ops"] * args.steps * world / w8a8_s / 1e12

    kernels = []
    for n in names:
        r = roofline_for(n, mean_us[n], work[n], peaks)
        kernels.append({"name": n, "us": round(mean_us[n], 2), "achieved": round(r["achieved"], 1),
                        "unit": r["unit"], "bound": r["bound"], "frac": round(r["frac"], 4)})
    dom = dominant_kernel(names, mean_us)
    rdom = roofline_for(dom, mean_us[dom], work[dom], peaks)
    traffic = load_traffic(dom)
    gemv_roof = roofline_for("gemv_w4a16_b1_up", 1.0, {"bytes": 1, "ops": 0}, peaks)

    # e2e: the GEMV through the public API with the activations copied in from pinned host
    # memory and the result read back, every step
    e2e = run_e2e(torch, wq, step, args.steps, stream)

    clocks = sampler.summary(t_wall0, t_wall1)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int4 weights x fp16 activations; int8 x int8",
        "data": "synthetic (seeded; shapes and outlier structure of the pages' workloads)",
        "config": arm_config(world),
        "value_frac_of_hbm_peak": round(value / world / peaks["hbm_gbs"], 4),
        "w8a8": {"value": round(w8a8_tops, 1), "unit": "TOPS", "peak": 2.0 * peaks["bf16_tflops"],
                 "frac": round(w8a8_tops / world / (2.0 * peaks["bf16_tflops"]), 4),
                 "peak_note": "INT8 dense = 2 x measured bf16 burst (nominal ratio)"},
        "roofline": {"kernel": dom, "bound": rdom["bound"], "achieved": round(rdom["achieved"], 1),
                     "peak": rdom["peak"], "unit": rdom["unit"], "frac": round(rdom["frac"], 4),
                     "traffic": traffic, "peak_source": peaks["source"]},
        "gemv_roofline": {"bound": "hbm", "achieved": round(value / world, 1), "peak": gemv_roof["peak"],
                          "unit": "GB/s", "frac": round(value / world / gemv_roof["peak"], 4),
                          "traffic": load_traffic("gemv_w4a16_b1_up")},
        "kernels": kernels,
        "e2e": e2e,
        "gpu_launches": len(launches) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[dev.index])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def arm_config(world):
    """The workload both arms report (the reference arm times a bounded sample of it)."""
    return {"workload": WORKLOAD, "w4a16_shapes": [list(UP), list(DOWN)], "gemv_batch": 1,
            "gemm_batches": [16, 64], "group_size": 128, "w8a8": list(W8A8_SHAPE), "alpha": 0.5,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2; matmul operands untouched since the previous step"}


def run_e2e(torch, wq, step, steps, stream):
    """Both batch-1 GEMVs through the public API, with the step's activations copied in from
    pinned host memory (one copy) and both results read back (one copy) every step.

    The step is timed twice: launched call by call from Python (`eager_value`), and as one
    CUDA graph captured from the same calls and replayed each step (`value`), which is how a
    decode loop issues it; the graph removes the per-call host overhead, not any work."""
    ins, qB = step.ins, step.qB
    kx = {"up": UP[1], "down": DOWN[1]}
    ny = {"up": UP[0], "down": DOWN[0]}
    hx = torch.cat([ins["x1_up"].reshape(-1), ins["x1_down"].reshape(-1)]).cpu().pin_memory()
    hy = torch.empty(ny["up"] + ny["down"], dtype=torch.float16).pin_memory()
    dx = torch.empty_like(hx, device=ins["x_w8a8"].device)
    dy = torch.empty(hy.numel(), dtype=torch.float16, device=ins["x_w8a8"].device)
    xv = {"up": dx[:kx["up"]].view(1, -1), "down": dx[kx["up"]:].view(1, -1)}
    yv = {"up": dy[:ny["up"]].view(1, -1), "down": dy[ny["up"]:].view(1, -1)}

    def one():
        dx.copy_(hx, non_blocking=True)
        for t in ("up", "down"):
            wq.gemv_w4a16(xv[t], *qB[t], 128, out=yv[t])
        hy.copy_(dy, non_blocking=True)

    def timed(fn, s):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(steps):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e-3

    w = work_table()
    byts = w["gemv_w4a16_b1_up"]["bytes"] + w["gemv_w4a16_b1_down"]["bytes"]
    t_eager = timed(one, stream)
    graph, graph_value = None, None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            one()
        graph_value = round(byts * steps / timed(graph.replay, stream) / 1e9, 1)
    except Exception:  # capture unsupported: only the call-by-call number
        graph_value = None
    finally:
        del graph
    return {"value": round(byts * steps / t_eager / 1e9, 1), "unit": "GB/s", "h2d_bytes_per_step": hx.numel() * 2,
            "d2h_bytes_per_step": hy.numel() * 2, "graph_value": graph_value,
            "launch": "call by call from Python (value); the same calls replayed as one CUDA graph (graph_value)",
            "what": "batch-1 W4A16 GEMV on both weights via the Python/C API, x copied from pinned host memory "
                    "and y read back each step (one copy each way)"}


def dominant_kernel(names, mean_us):
    """The kernel whose launches (on both projections: `_up` and `_down`) take the largest share
    of the step; returns its first launch, whose roofline the bench line reports and whose DRAM
    traffic comes from a committed ncu capture."""
    def family(n):
        return n.rsplit("_", 1)[0] if n.endswith(("_up", "_down")) else n
    share = {}
    for n in names:
        share[family(n)] = share.get(family(n), 0.0) + mean_us[n]
    top = max(share, key=share.get)
    return next(n for n in names if family(n) == top)


def load_traffic(kernel):
    """Per-launch DRAM bytes for `kernel` from the committed ncu summary, if any."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    return None if e is None else e.get("bytes_per_launch")


# ----------------------------------------------------------------------------- CPU oracle
_ORACLE_INPUTS = {}


def _oracle_inputs(rows=4096):
    """Oracle-side copy of the first rows of the up-projection, quantized by the oracle."""
    if rows not in _ORACLE_INPUTS:
        import oracle
        import workloads
        w = workloads.config_weight("llama70b_class", 0, shape=(rows, UP[1]))
        _ORACLE_INPUTS[rows] = (oracle.quantize_group_int4(w, 128), workloads.config_activations("llama70b_class", 1, UP[1]))
    return _ORACLE_INPUTS[rows]


def cpu_baseline(seconds=12.0):
    """The oracle's fp64 W4A16 GEMV on a bounded sample of the workload's rows (one core)."""
    import oracle
    (qw, sc, qz), x = _oracle_inputs()
    K = UP[1]
    t0 = time.perf_counter()
    oracle.matmul_w4a16_ref(x, qw[:64], sc[:64], qz[:64], K, 128)
    per_row = (time.perf_counter() - t0) / 64
    passes = max(1, int(round(seconds / max(per_row * qw.shape[0], 1e-9))))
    t0 = time.perf_counter()
    for _ in range(passes):
        oracle.matmul_w4a16_ref(x, qw, sc, qz, K, 128)
    dt = time.perf_counter() - t0
    rows = qw.shape[0] * passes
    byts = passes * (packed_bytes(qw.shape[0], K) + 2 * K + 2 * qw.shape[0])
    return {"value": float(f"{byts / dt / 1e9:.4g}"), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"fp64 oracle W4A16 GEMV, batch 1, the first {qw.shape[0]} rows of the 28672x8192 "
                      f"up-projection x {passes} passes ({rows} rows, {dt:.1f} s)",
            "host_cores_total": os.cpu_count()}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    _oracle_inputs()
    for _ in range(args.warmup):
        cpu_baseline(0.1)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_baseline(per_step))
    dt = time.perf_counter() - t0
    v = statistics.median([b["value"] for b in vals])
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp64 (oracle)", "data": "synthetic (seeded)",
            "config": arm_config(world), "impl": "reference",
            "cpu_baseline": {"value": v, "unit": "GB/s", "kind": "oracle", "cores": 1, "sample": vals[-1]["sample"]},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """Runs one named kernel of the step `--profile-launches` times on the step's inputs and
    prints nothing: the command that ncu captures for the per-kernel summaries."""
    import torch
    import bit_gemv_gemm_group_b200 as wq

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    step = Step(torch, wq, make_inputs(torch, dev))
    launches = dict(step.launches())
    if args.profile_case not in launches:
        raise SystemExit(f"unknown kernel {args.profile_case!r}; one of {sorted(launches)}")
    # producers of a profiled kernel's operands run first (in step order), then the kernel itself
    names = [n for n, _ in step.launches()]
    producers = {"quant_int8_pc_smooth": ["smooth"], "quant_int8_pt_smooth": ["smooth"],
                 "gemm_w8a8": ["smooth", "quant_int8_pc_smooth", "quant_int8_pt_smooth"],
                 "gemm_fp8": ["quant_fp8_w", "quant_fp8_x"], "llm_quant_x": ["llm_outlier_columns"],
                 "llm_gather": ["llm_outlier_columns"],
                 "gemm_llm_int8": ["llm_outlier_columns", "llm_quant_x", "llm_gather"],
                 "gemm_mxfp4": ["quant_mxfp4_w", "quant_mxfp4_x"], "gemm_nvfp4": ["quant_nvfp4_w", "quant_nvfp4_x"]}
    for name in names:
        if name in producers.get(args.profile_case, []):
            launches[name]()
    torch.cuda.synchronize()
    for _ in range(args.profile_launches):
        launches[args.profile_case]()
    torch.cuda.synchronize()
    if wq.device_status() != 0:
        raise RuntimeError("a kernel reported a wait timeout")


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["wq", "reference"], default="wq")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="size of the CPU oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", default=None,
                    help="run only this kernel of the step (e.g. gemv_w4a16_b1_up) for an ncu capture; no output")
    ap.add_argument("--profile-launches", type=int, default=3)
    args = ap.parse_args(argv)
    if args.profile_case:
        run_profile_case(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
