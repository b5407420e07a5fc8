#!/usr/bin/env python
"""Throughput of the EfficientQAT fake-quantized linear hot path on B200.

One step = one pass of the whole path over one batch of synthetic tokens, on the
Llama-2-7B q_proj workload (M = 4096 tokens, W [4096, 4096] bf16, w2g64), in the
order of a training step (the backward reuses the W-hat its forward left in the
workspace):

  init      min-max init (s, z)                       HBM-bound, 1 kernel
  fq_fwd    Block-AP forward  Y = X W-hat^T           quantizer prepass + tcgen05 GEMM
  fq_bwd    Block-AP backward dX = dY W-hat and       one grouped tcgen05 launch; the
            dW, ds, dz from dY^T X                    dW-hat tiles run the fused
                                                      straight-through epilogue
  pack      2-bit codes + zq                          HBM-bound, 1 kernel
  dq_fwd    E2E-QP forward Y = X ((W_q - z) s)^T      dequant prepass + tcgen05 GEMM
  dq_bwd    E2E-QP backward dX and ds                 one grouped tcgen05 launch

value = (6 M N K for Block-AP + 6 M N K for E2E-QP) / step time, in TFLOP/s.
L2 is flushed (a 512 MiB write) before every timed step.  Under torchrun (N > 1)
every rank runs the same step on its own token batch (weak scaling) and the
weight gradients dW, ds, dz and the E2E ds are summed over ranks with NCCL
all-reduce inside the step (data-parallel training).

--impl reference times the CPU oracle (the only other arm: the pages hold no
code to run) on a bounded sample of the same workload.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import weight_quantization_aware_b200 as eqat  # noqa: E402
from weight_quantization_aware_b200 import dp, synthetic  # noqa: E402

WORKLOAD = synthetic.WORKLOADS[2]
METRIC = "fake-quant linear fwd+bwd TFLOP/s & % bf16 peak (w2g64); init/pack HBM GB/s"
PHASES = ["init", "fq_fwd", "fq_bwd", "pack", "dq_fwd", "dq_bwd"]
LAUNCHES_PER_STEP = {"init": 1, "fq_fwd": 2, "fq_bwd": 1, "pack": 1, "dq_fwd": 2, "dq_bwd": 1}
# One launch: the grouped backward GEMM (dY W-hat tiles and dY^T X tiles with the
# fused straight-through epilogue), 4 M N K flops.
DOMINANT = "fq_bwd"
DOMINANT_KERNEL_SOURCES = ["weight_quantization_aware_b200/csrc/eqat_gemm_tc.cu",
                           "weight_quantization_aware_b200/csrc/eqat_ptx.cuh",
                           "weight_quantization_aware_b200/csrc/eqat_qmath.cuh"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in DOMINANT_KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_traffic():
    """dram bytes per launch of the dominant kernel from the committed ncu summary,
    if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "gemm_bwd_grouped_fused_ste_llama2-7b-q_proj_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        else:
            self.lines = []

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------ our arm

class Step:
    """Holds the device buffers of one rank and runs the hot path through the C ABI."""

    def __init__(self, wl, rank, bits, group, dev):
        lin = wl.linears[0]
        self.M, self.N, self.K = wl.m, lin.n, lin.k
        self.bits, self.group = bits, group
        d = dp.rank_batch(wl, 0, rank)  # each data-parallel rank sees its own tokens; W is shared
        self.host = {k: v.pin_memory() for k, v in d.items()}
        self.X = self.host["X"].to(dev)
        self.W = self.host["W"].to(dev)
        self.dY = self.host["dY"].to(dev)
        M, N, K, G = self.M, self.N, self.K, self.K // group
        bf = torch.bfloat16
        self.ws = eqat.workspace(M, N, K, bits, group, bf, dev)
        self.s = torch.empty((N, G), dtype=torch.float32, device=dev)
        self.z = torch.empty_like(self.s)
        self.Y = torch.empty((M, N), dtype=bf, device=dev)
        self.dX = torch.empty((M, K), dtype=bf, device=dev)
        self.dW = torch.empty((N, K), dtype=bf, device=dev)
        self.ds = torch.empty_like(self.s)
        self.dz = torch.empty_like(self.s)
        self.codes = torch.empty((N, eqat.packed_row_bytes(K, bits)), dtype=torch.uint8, device=dev)
        self.zq = torch.empty((N, G), dtype=torch.uint8, device=dev)
        self.Y2 = torch.empty_like(self.Y)
        self.dX2 = torch.empty_like(self.dX)
        self.ds2 = torch.empty_like(self.s)

    def outputs(self):
        return [self.s, self.z, self.Y, self.dX, self.dW, self.ds, self.dz, self.codes, self.zq,
                self.Y2, self.dX2, self.ds2]

    def run(self, events=None, allreduce=None):
        b, g = self.bits, self.group

        def mark(i):
            if events is not None:
                events[i].record()

        mark(0)
        eqat.minmax_init(self.W, b, g, s=self.s, z=self.z)
        mark(1)
        eqat.fq_linear_fwd(self.X, self.W, self.s, self.z, b, g, ws=self.ws, Y=self.Y)
        mark(2)
        eqat.fq_linear_bwd(self.X, self.W, self.s, self.z, self.dY, b, g, ws=self.ws,
                           out=(self.dX, self.dW, self.ds, self.dz), w_hat_in_ws=True)
        mark(3)
        eqat.pack_codes(self.W, self.s, self.z, b, g, codes=self.codes, zq=self.zq)
        mark(4)
        eqat.dq_linear_fwd(self.X, self.codes, self.zq, self.s, b, g, ws=self.ws, Y=self.Y2)
        mark(5)
        eqat.dq_linear_bwd_s(self.X, self.codes, self.zq, self.s, self.dY, b, g, ws=self.ws,
                             out=(self.dX2, self.ds2), w_hat_in_ws=True)
        mark(6)
        if allreduce is not None:
            allreduce([self.dW, self.ds, self.dz, self.ds2])


def phase_bytes(M, N, K, bits, group):
    """Algorithmic HBM bytes of the two HBM-bound phases (bf16 W)."""
    G = K // group
    init = N * K * 2 + 8 * N * G
    pack = N * K * 2 + 8 * N * G + N * K * bits // 8 + N * G
    if bits == 3:
        pack = N * K * 2 + 8 * N * G + N * K + N * G
    return init, pack


def flush_l2(buf):
    buf.zero_()


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    eqat.load_library()
    wl = WORKLOAD
    step = Step(wl, rank, wl.bits, wl.group, dev)
    M, N, K = step.M, step.N, step.K
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    allreduce = None
    if dist is not None:
        def allreduce(ts):
            dp.allreduce_weight_grads(ts, dist)

    for _ in range(args.warmup):
        flush_l2(flush)
        step.run(allreduce=allreduce)
    torch.cuda.synchronize()
    if eqat.device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    nph = len(PHASES)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nph + 2)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush_l2(flush)
            step.run(events=ev[i], allreduce=allreduce)
            ev[i][nph + 1].record()
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if eqat.device_error() != 0:
        raise RuntimeError("device error word set during the timed region")

    step_ms = [ev[i][0].elapsed_time(ev[i][nph + 1]) for i in range(args.steps)]
    phase_ms = {p: [ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)] for j, p in enumerate(PHASES)}
    total_ms = sum(step_ms)
    if dist is not None:
        t = torch.tensor([total_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    flops_step = 12 * M * N * K
    value = flops_step * world / (ms_per_step * 1e-3) / 1e12

    peaks = load_peaks()
    mean = {p: sum(v) / len(v) for p, v in phase_ms.items()}
    dom_ms = mean[DOMINANT]
    dom_flops = 4 * M * N * K
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    init_b, pack_b = phase_bytes(M, N, K, wl.bits, wl.group)
    traffic = load_traffic()
    clocks = clk.summary()

    # --------------------------------------------------------------------- e2e (host buffers)
    # Every step copies its inputs (X, W, dY) from pinned host memory and reads its
    # result back: the gradients of the quantization parameters (ds, dz of Block-AP,
    # ds of E2E-QP) and the packed model (codes, zq).  Y, dX and dW stay on the device,
    # where the next layer consumes them.  The input copies of step i+1 run on a copy
    # stream into the second of two input buffers while step i computes; the read of
    # step i's result runs on a second copy stream and ends before step i+1 writes it.
    e2e = None
    if not args.no_e2e:
        res = [step.ds, step.dz, step.ds2, step.codes, step.zq]
        host_res = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in res] for _ in range(2)]
        host_in = [step.host["X"], step.host["W"], step.host["dY"]]
        bufs = [[step.X, step.W, step.dY], [torch.empty_like(step.X), torch.empty_like(step.W),
                                            torch.empty_like(step.dY)]]
        h2d = sum(h.numel() * h.element_size() for h in host_in)
        d2h = sum(t.numel() * t.element_size() for t in res)
        n_e2e = max(3, min(args.steps, 20))
        comp = torch.cuda.current_stream(dev)
        s_in = torch.cuda.Stream(device=dev)
        s_out = torch.cuda.Stream(device=dev)

        def e2e_run(n):
            in_ready = [torch.cuda.Event(), torch.cuda.Event()]
            in_free = [torch.cuda.Event(), torch.cuda.Event()]
            out_done = [torch.cuda.Event(), torch.cuda.Event()]
            with torch.cuda.stream(s_in):
                for h, d in zip(host_in, bufs[0]):
                    d.copy_(h, non_blocking=True)
                in_ready[0].record(s_in)
            for it in range(n):
                b = it % 2
                if it + 1 < n:  # next step's inputs, into the other buffer
                    with torch.cuda.stream(s_in):
                        if it >= 1:
                            s_in.wait_event(in_free[1 - b])
                        for h, d in zip(host_in, bufs[1 - b]):
                            d.copy_(h, non_blocking=True)
                        in_ready[1 - b].record(s_in)
                comp.wait_event(in_ready[b])
                if it >= 1:
                    comp.wait_event(out_done[1 - b])  # step it-1's result read out before it is overwritten
                step.X, step.W, step.dY = bufs[b]
                step.run(allreduce=allreduce)
                in_free[b].record(comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_stream(comp)
                    for d, h in zip(res, host_res[b]):
                        h.copy_(d, non_blocking=True)
                    out_done[b].record(s_out)
            comp.wait_stream(s_out)
            comp.wait_stream(s_in)

        e2e_run(3)  # warm
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        e2e_run(n_e2e)
        e1.record(comp)
        torch.cuda.synchronize()
        step.X, step.W, step.dY = bufs[0]
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        if dist is not None:
            t = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        e2e = {"value": round(flops_step * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
               "steps": n_e2e,
               "note": "inputs X, W, dY copied in every step (double-buffered, overlapping the previous step); "
                       "result read back every step: ds, dz, ds2, codes, zq"}

    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations and gradients, N(0,0.02) weights with 0.1% x10 outliers)",
        "config": {"workload": wl.name, "M": M, "N": N, "K": K, "bits": wl.bits, "group": wl.group,
                   "flops_per_step": flops_step, "l2": "flushed before every step (512 MiB write)",
                   "parallelism": f"dp{world}" if world > 1 else "single-gpu",
                   "step": "+".join(PHASES)},
        "roofline": {"bound": "tensor",
                     "kernel": "k_gemm_tc2 grouped backward on CTA pairs: dY W-hat + dY^T X with the fused "
                               "straight-through epilogue",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": f"bf16 dense, sustained, {peaks['source']}",
                     "frac_of_burst_peak": round(achieved / peaks["bf16_tflops"], 4)},
        "phases_ms": {p: round(v, 4) for p, v in mean.items()},
        "phase_rates": {
            "init_GBps": round(init_b / (mean["init"] * 1e-3) / 1e9, 1),
            "pack_GBps": round(pack_b / (mean["pack"] * 1e-3) / 1e9, 1),
            "init_frac_hbm": round(init_b / (mean["init"] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "pack_frac_hbm": round(pack_b / (mean["pack"] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "blockap_fwd_bwd_TFLOPs": round(6 * M * N * K / ((mean["fq_fwd"] + mean["fq_bwd"]) * 1e-3) / 1e12, 2),
            "e2e_fwd_bwd_TFLOPs": round(6 * M * N * K / ((mean["dq_fwd"] + mean["dq_bwd"]) * 1e-3) / 1e12, 2),
            "hbm_peak_GBps": peaks["hbm_gbs"],
        },
        "gpu_launches": sum(LAUNCHES_PER_STEP.values()) * args.steps,
        "clocks": clocks,
        "wall_s_timed": round(t_wall, 3),
        "e2e": e2e,
    }
    if not args.no_initpack70b:
        ip = initpack_70b_block(dev)
        ip["init_frac_hbm"] = round(ip["init_GBps"] / peaks["hbm_gbs"], 4)
        ip["pack_frac_hbm"] = round(ip["pack_GBps"] / peaks["hbm_gbs"], 4)
        line["initpack_70b_block"] = ip
    if not args.no_variants:
        line["variants"] = quantizer_variants(step, dev)
    if not args.no_gemv:
        line["decode_gemv"] = decode_gemv(dev, peaks)
    if not args.no_blockap:
        line["blockap_block"] = blockap_block(dev, peaks)
    if not args.no_configs:
        line["per_config"] = per_config(dev, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(target_s=args.cpu_seconds)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def quantizer_variants(step, dev, reps=50):
    """Backward throughput of the quantizer variants on the step's workload, each
    beside its default (same buffers, W-hat reused from the workspace, L2 flushed
    before every call): the all-pass clamp gradient of the Block-AP backward, and
    the E2E-QP backward with dz and fp32 / fp16 step sizes.  TFLOP/s = 4MNK / event
    time of the call."""
    b, g = step.bits, step.group
    M, N, K = step.M, step.N, step.K
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    s16 = step.s.to(torch.float16)
    dz2 = torch.empty_like(step.ds2)
    eqat.fq_linear_fwd(step.X, step.W, step.s, step.z, b, g, ws=step.ws, Y=step.Y)
    calls = {
        "fq_bwd": lambda: eqat.fq_linear_bwd(step.X, step.W, step.s, step.z, step.dY, b, g, ws=step.ws,
                                             out=(step.dX, step.dW, step.ds, step.dz), w_hat_in_ws=True),
        "fq_bwd_clamp_pass": lambda: eqat.fq_linear_bwd(step.X, step.W, step.s, step.z, step.dY, b, g,
                                                        ws=step.ws, out=(step.dX, step.dW, step.ds, step.dz),
                                                        w_hat_in_ws=True, clamp_pass=True),
    }
    e2e = {
        "dq_bwd_ds": lambda s_: eqat.dq_linear_bwd(step.X, step.codes, step.zq, s_, step.dY, b, g, ws=step.ws,
                                                   out=(step.dX2, step.ds2, None), w_hat_in_ws=True),
        "dq_bwd_ds_dz": lambda s_: eqat.dq_linear_bwd(step.X, step.codes, step.zq, s_, step.dY, b, g, ws=step.ws,
                                                     out=(step.dX2, step.ds2, dz2), w_hat_in_ws=True),
    }

    def timed(fn):
        tot = 0.0
        for r in range(reps + 3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush.zero_()
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if r >= 3:
                tot += e0.elapsed_time(e1)
        return tot / reps

    out = {}
    for name, fn in calls.items():
        out[name + "_TFLOPs"] = round(4 * M * N * K / (timed(fn) * 1e-3) / 1e12, 1)
    for sname, s_ in (("s32", step.s), ("s16", s16)):
        eqat.dq_linear_fwd(step.X, step.codes, step.zq, s_, b, g, ws=step.ws, Y=step.Y2)
        for name, fn in e2e.items():
            out[f"{name}_{sname}_TFLOPs"] = round(4 * M * N * K / (timed(lambda: fn(s_)) * 1e-3) / 1e12, 1)
    out["note"] = "4MNK per backward call, L2 flushed before each call, W-hat reused from the forward"
    return out


def per_config(dev, peaks, reps=10):
    """Fake-quant linear forward + backward throughput per linear and per config, for the
    bf16 workloads (Llama-2 7B q_proj; 7B MLP w3g128; 13B E2E-QP w2g64 on packed codes;
    70B block w2g64).  Block-AP: fq_linear_fwd then fq_linear_bwd (dX, dW, ds, dz, W-hat
    reused); E2E-QP: dq_linear_fwd then dq_linear_bwd_s (dX, ds).  6 M N K per linear;
    CUDA events around `reps` back-to-back fwd+bwd pairs after 2 warm ones.  Inputs are
    drawn on the device (seeded); the per-linear bytes exceed L2 for all but the smallest."""
    out = {}
    gen = torch.Generator(device=dev)
    for idx in (2, 3, 4, 5):
        wl = synthetic.WORKLOADS[idx]
        M, b, g = wl.m, wl.bits, wl.group
        lines, tot_flops, tot_ms = {}, 0, 0.0
        for lin in wl.linears:
            N, K = lin.n, lin.k
            gen.manual_seed(4000 + 10 * idx + len(lines))
            X = torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16)
            W = (torch.randn(N, K, generator=gen, device=dev) * wl.sigma).to(torch.bfloat16)
            dY = torch.randn(M, N, generator=gen, device=dev).to(torch.bfloat16)
            s, z = eqat.minmax_init(W, b, g)
            ws = eqat.workspace(M, N, K, b, g, torch.bfloat16, dev)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            if wl.mode == "e2e_qp":
                codes, zq = eqat.pack_codes(W, s, z, b, g)
                out_b = (torch.empty_like(X), torch.empty_like(s))

                def fb():
                    eqat.dq_linear_fwd(X, codes, zq, s, b, g, ws=ws, Y=Y)
                    eqat.dq_linear_bwd_s(X, codes, zq, s, dY, b, g, ws=ws, out=out_b, w_hat_in_ws=True)
            else:
                out_b = (torch.empty_like(X), torch.empty_like(W), torch.empty_like(s), torch.empty_like(s))

                def fb():
                    eqat.fq_linear_fwd(X, W, s, z, b, g, ws=ws, Y=Y)
                    eqat.fq_linear_bwd(X, W, s, z, dY, b, g, ws=ws, out=out_b, w_hat_in_ws=True)
            fb(); fb()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                fb()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            fl = 6 * M * N * K
            lines[lin.name] = {"N": N, "K": K, "us": round(ms * 1e3, 1),
                               "TFLOPs": round(fl / (ms * 1e-3) / 1e12, 1),
                               "frac_bf16_sustained": round(fl / (ms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"], 3)}
            tot_flops += fl
            tot_ms += ms
            del X, W, dY, ws, Y, out_b
            torch.cuda.empty_cache()
        out[wl.name] = {"M": M, "bits": b, "group": g, "mode": wl.mode, "linears": lines,
                        "TFLOPs": round(tot_flops / (tot_ms * 1e-3) / 1e12, 1),
                        "frac_bf16_sustained": round(tot_flops / (tot_ms * 1e-3) / 1e12 /
                                                     peaks["bf16_tflops_sustained"], 3)}
    out["note"] = "6 M N K per linear (forward + dX + dW-hat), prepasses included; no L2 flush between calls"
    return out


def blockap_block(dev, peaks, steps=5):
    """Block-AP step over the seven linears of one Llama-2-7B decoder block (q, k, v, o
    4096x4096; gate, up 11008x4096; down 4096x11008), 2-bit g64, 4096 tokens (batch 2 x
    2048): per linear the fake-quant forward with the fused MSE epilogue against the
    full-precision output and the straight-through backward (dW, ds, dz; no dX: the
    inputs are the step's data), then one AdamW launch over all 21 tensors.  Synthetic
    seeded inputs; targets = X W_fp^T.  The weights and optimizer state (2.8 GB) exceed L2,
    so no flush.  TFLOP/s = sum 4 M N K / step time; AdamW GB/s = its algorithmic bytes
    (28 per weight, 32 per s/z entry) / its own event time."""
    from weight_quantization_aware_b200.blockap import BlockAPConfig, QuantLinearState, blockap_step
    M = 4096
    shapes = {"q_proj": (4096, 4096), "k_proj": (4096, 4096), "v_proj": (4096, 4096), "o_proj": (4096, 4096),
              "gate_proj": (11008, 4096), "up_proj": (11008, 4096), "down_proj": (4096, 11008)}
    cfg = BlockAPConfig(bits=2, group=64, total_steps=4096)
    gen = torch.Generator(device=dev)
    gen.manual_seed(3007)
    X_in = {K: torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16) for K in (4096, 11008)}
    lin, Xs, Ts = [], [], []
    flops = 0
    for name, (N, K) in shapes.items():
        W = torch.randn(N, K, generator=gen, device=dev) * 0.02
        L = QuantLinearState.from_weight(W, cfg.bits, cfg.group, M)
        X = X_in[K]
        Ts.append(torch.matmul(X, W.to(torch.bfloat16).t()))  # the full-precision output
        lin.append(L)
        Xs.append(X)
        flops += 4 * M * N * K
        del W
    losses = torch.empty(len(lin), dtype=torch.float64, device=dev)
    blockap_step(lin, Xs, Ts, cfg, 1, losses)
    torch.cuda.synchronize()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    e[0].record()
    for t in range(2, 2 + steps):
        blockap_step(lin, Xs, Ts, cfg, t, losses)
    e[1].record()
    torch.cuda.synchronize()
    step_ms = e[0].elapsed_time(e[1]) / steps
    # AdamW alone, same tensors and gradients
    groups = [dict(lr=cfg.lr_w, weight_decay=0.0), dict(lr=cfg.lr_q, weight_decay=0.0)]
    entries = []
    nw = nq = 0
    for L in lin:
        _, dW, ds, dz = L.grads
        entries += [(L.W_master, dW, *L.moments["W"], L.W, 0), (L.s, ds, *L.moments["s"], None, 1),
                    (L.z, dz, *L.moments["z"], None, 1)]
        nw += L.W_master.numel()
        nq += L.s.numel() + L.z.numel()
    ea = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    eqat.adamw_step(entries, groups, 10)
    ea[0].record()
    for t in range(3):
        eqat.adamw_step(entries, groups, 11 + t)
    ea[1].record()
    torch.cuda.synchronize()
    adamw_ms = ea[0].elapsed_time(ea[1]) / 3
    adamw_bytes = 28 * nw + 32 * nq
    out = {"workload": "llama2-7b-block-blockap-w2g64-m4096 (7 linears, 202.4 M weights)",
           "step_ms": round(step_ms, 3), "TFLOPs": round(flops / (step_ms * 1e-3) / 1e12, 1),
           "flops_per_step": flops, "adamw_ms": round(adamw_ms, 3),
           "adamw_GBps": round(adamw_bytes / (adamw_ms * 1e-3) / 1e9, 1),
           "adamw_frac_hbm": round(adamw_bytes / (adamw_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
           "loss_first_linear": float(losses[0].item()),
           "launches_per_step": 7 * 2 + 7 + 1,
           "note": "fq prepass + MSE-epilogue forward + grouped STE backward per linear, one AdamW launch"}
    del lin, Xs, Ts, X_in
    torch.cuda.empty_cache()
    return out


def decode_gemv(dev, peaks, budget_bytes=300_000_000):
    """Batch-1 inference on frozen 2-, 3- and 4-bit codes (eqat_dq_linear_fwd at
    M = 1, the decode-size path), against a bf16 matvec (torch.matmul) of the same
    shape.
    Back-to-back calls over enough distinct layers that their bytes exceed L2,
    captured in a CUDA graph so that host launch cost is excluded; CUDA events
    around three replays.  GB/s = algorithmic bytes (codes + s + zq + X + Y) /
    time per call."""
    out = {}
    side = torch.cuda.Stream(device=dev)
    for name, N, K, b, g in (("llama2-70b-gate_proj", 28672, 8192, 2, 64), ("llama2-7b-q_proj", 4096, 4096, 2, 64),
                             ("llama2-7b-mlp-gate_proj-w3g128", 11008, 4096, 3, 128),
                             ("llama2-70b-gate_proj-w4g64", 28672, 8192, 4, 64)):
        M = 1
        G = K // g
        cb = K * b // 8 if b != 3 else K  # code bytes per row (3-bit: one code per byte)
        per = N * cb + N * G * 5
        L = max(2, -(-budget_bytes // per))
        gen = torch.Generator(device=dev)
        gen.manual_seed(2000 + N)
        layers = [(torch.randint(0, 256 if b != 3 else 8, (N, cb), generator=gen, device=dev, dtype=torch.uint8),
                   torch.randint(0, 1 << b, (N, G), generator=gen, device=dev, dtype=torch.uint8),
                   torch.rand(N, G, generator=gen, device=dev) * 0.01 + 1e-3) for _ in range(L)]
        X = torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16)
        ws = eqat.workspace(M, N, K, b, g, torch.bfloat16, dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

        def timed_graph(fn, n_calls):
            fn()
            torch.cuda.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=side):
                fn()
            gr.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(3):
                gr.replay()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) * 1e3 / (3 * n_calls)

        def run():
            for c, z, s_ in layers:
                eqat.dq_linear_fwd(X, c, z, s_, b, g, ws=ws, Y=Y)

        t = timed_graph(run, L)
        del layers
        Lb = max(2, -(-budget_bytes // (N * K * 2)))
        Ws = [torch.randn(N, K, generator=gen, device=dev).to(torch.bfloat16) for _ in range(Lb)]

        def runb():
            for W in Ws:
                torch.matmul(X, W.t(), out=Y)

        tb = timed_graph(runb, Lb)
        del Ws
        torch.cuda.empty_cache()
        byts = per + M * K * 2 + M * N * 2
        gbs = byts / (t * 1e-6) / 1e9
        out[name] = {"N": N, "K": K, "M": M, "bits": b, "group": g, "us": round(t, 2), "GBps": round(gbs, 1),
                     "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "bf16_matvec_us": round(tb, 2),
                     "speedup_vs_bf16_matvec": round(tb / t, 2), "layers_cycled": L}
    out["note"] = ("GPU time per call from a CUDA graph of back-to-back calls (the streaming kernel and the partial "
                   "sum; for layers above the build-mode size also the X-fragment kernel); bf16 matvec = "
                   "torch.matmul on bf16 weights, same method")
    return out


def initpack_70b_block(dev, reps=5):
    """HBM throughput of min-max init and pack over all seven linears of the
    Llama-2-70B block (855.6 M bf16 weights, w2g64): algorithmic bytes / event time.
    Before each launch L2 is flushed by a 512 MiB write and then a 256 MiB read of
    another buffer, so that the kernel starts on clean lines instead of first
    writing back the flush's dirty ones.  Weights are seeded N(0, 0.015) with 0.1%
    x10 outliers, drawn on the device."""
    wl = synthetic.WORKLOADS[5]
    gen = torch.Generator(device=dev)
    gen.manual_seed(1005)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    clean = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush_clean():
        flush.zero_()
        clean.amax()
    t_init = t_pack = 0.0
    b_init = b_pack = 0
    for lin in wl.linears:
        N, K = lin.n, lin.k
        W = torch.randn(N, K, generator=gen, device=dev).mul_(wl.sigma)
        idx = torch.randint(0, N * K, ((N * K) // 1000,), generator=gen, device=dev)
        W.view(-1)[idx] *= 10.0
        W = W.to(torch.bfloat16)
        G = K // wl.group
        s = torch.empty((N, G), dtype=torch.float32, device=dev)
        z = torch.empty_like(s)
        codes = torch.empty((N, eqat.packed_row_bytes(K, wl.bits)), dtype=torch.uint8, device=dev)
        zq = torch.empty((N, G), dtype=torch.uint8, device=dev)
        bi, bp = phase_bytes(1, N, K, wl.bits, wl.group)
        for r in range(reps + 1):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            flush_clean()
            e[0].record()
            eqat.minmax_init(W, wl.bits, wl.group, s=s, z=z)
            e[1].record()
            flush_clean()
            e[2].record()
            eqat.pack_codes(W, s, z, wl.bits, wl.group, codes=codes, zq=zq)
            e[3].record()
            torch.cuda.synchronize()
            if r:  # first round is warm-up
                t_init += e[0].elapsed_time(e[1]) / reps
                t_pack += e[2].elapsed_time(e[3]) / reps
        b_init += bi
        b_pack += bp
        del W, s, z, codes, zq
    return {"workload": wl.name + " (init+pack of all 7 linears, 855.6 M weights)",
            "init_GBps": round(b_init / (t_init * 1e-3) / 1e9, 1),
            "pack_GBps": round(b_pack / (t_pack * 1e-3) / 1e9, 1),
            "init_ms": round(t_init, 4), "pack_ms": round(t_pack, 4),
            "init_bytes": b_init, "pack_bytes": b_pack,
            "l2": "flushed by a 512 MiB write, then a 256 MiB read of another buffer, before each launch"}


# ------------------------------------------------------------------------------ oracle arm

def oracle_sample(rows: int):
    """The oracle's hot path on a bounded sample of the workload: min-max init and
    pack of the whole W; Block-AP and E2E-QP forward (Y rows), input gradient (dX
    rows) and weight-side gradients (dW, ds, dz / ds rows) for `rows` token rows
    and `rows` weight rows.  Returns (seconds, flops, description)."""
    import oracle
    wl = WORKLOAD
    lin = wl.linears[0]
    d = synthetic.workload_linear(wl, 0)
    X, W, dY = (synthetic.as_f32_numpy(d[k]) for k in ("X", "W", "dY"))
    M, N, K = wl.m, lin.n, lin.k
    b, g = wl.bits, wl.group
    rng = np.random.default_rng(5)
    r = np.sort(rng.choice(M, rows, replace=False))
    wr = np.sort(rng.choice(N, rows, replace=False))
    t0 = time.perf_counter()
    s, z = oracle.minmax_init(W, b, g)
    oracle.fq_linear_fwd(X, W, s, z, b, g, rows=r)
    oracle.fq_linear_bwd(X, W, s, z, dY, b, g, rows=r, wrows=wr)
    packed, zq = oracle.pack(W, s, z, b, g)
    oracle.dq_linear_fwd(X, packed, zq, s, b, g, rows=r)
    oracle.dq_linear_bwd_s(X, packed, zq, s, dY, b, g, rows=r, wrows=wr)
    dt = time.perf_counter() - t0
    flops = 2 * (2 * rows * N * K + 2 * rows * N * K + 2 * rows * M * K)  # per mode: Y, dX rows; dW-hat rows
    desc = (f"{wl.name}: init+pack of all {N}x{K} weights; fwd and dX for {rows} of {M} token rows; "
            f"dW-hat/dW/ds/dz for {rows} of {N} weight rows; both Block-AP and E2E-QP")
    return dt, flops, desc


def calibrate_rows(target_s: float) -> int:
    """Rows of the sample so that one oracle_sample() takes about target_s seconds:
    the cost is a fixed part (init, pack, W-hat) plus a part linear in the rows."""
    t4, _, _ = oracle_sample(4)
    t20, _, _ = oracle_sample(20)
    per_row = max((t20 - t4) / 16, 1e-5)
    fixed = max(t4 - 4 * per_row, 0.0)
    return int(max(4, min(WORKLOAD.m, (target_s - fixed) / per_row)))


def cpu_model() -> str:
    """The host CPU's model name (first entry of /proc/cpuinfo), for the baseline's record."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(target_s: float = 15.0):
    import oracle
    rows = calibrate_rows(target_s)
    dt, flops, desc = oracle_sample(rows)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "cpu": cpu_model(), "kind": "oracle", "sample": desc, "seconds": round(dt, 2)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    wl = WORKLOAD
    lin = wl.linears[0]
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    rows = calibrate_rows(per_step)
    for _ in range(args.warmup):
        oracle_sample(rows)
    times, flops, desc = [], 0, ""
    for _ in range(args.steps):
        dt, flops, desc = oracle_sample(rows)
        times.append(dt)
    sec = sum(times) / len(times)
    value = flops / sec / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "M": wl.m, "N": lin.n, "K": lin.k, "bits": wl.bits, "group": wl.group},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "cpu": cpu_model(), "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="eqat", choices=["eqat", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-initpack70b", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-gemv", action="store_true")
    ap.add_argument("--gemv-only", action="store_true")
    ap.add_argument("--gemv-layer", default="70b-gate_proj", choices=["70b-gate_proj", "7b-q_proj"])
    ap.add_argument("--no-blockap", action="store_true")
    ap.add_argument("--blockap-only", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--configs-only", action="store_true")
    ap.add_argument("--initpack70b-only", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # timing rule: at least 3 untimed warm-up steps
    if args.configs_only:  # the per-config table alone
        torch.cuda.set_device(0)
        eqat.load_library()
        print(json.dumps(per_config(torch.device("cuda", 0), load_peaks())), flush=True)
        return
    if args.blockap_only:  # profiling aid: the Block-AP block step measurement alone
        torch.cuda.set_device(0)
        eqat.load_library()
        print(json.dumps(blockap_block(torch.device("cuda", 0), load_peaks(), steps=2)), flush=True)
        return
    if args.gemv_only:  # profiling aid: four plain decode GEMV calls at M = 1, w2g64
        torch.cuda.set_device(0)
        eqat.load_library()
        dev = torch.device("cuda", 0)
        # Llama-2-70B gate_proj (fragment mode), or Llama-2-7B q_proj (build mode)
        N, K, b, g = (4096, 4096, 2, 64) if args.gemv_layer == "7b-q_proj" else (28672, 8192, 2, 64)
        gen = torch.Generator(device=dev)
        gen.manual_seed(2000 + N)
        c = torch.randint(0, 256, (N, K * b // 8), generator=gen, device=dev, dtype=torch.uint8)
        z = torch.randint(0, 1 << b, (N, K // g), generator=gen, device=dev, dtype=torch.uint8)
        s_ = torch.rand(N, K // g, generator=gen, device=dev) * 0.01 + 1e-3
        X = torch.randn(1, K, generator=gen, device=dev).to(torch.bfloat16)
        ws = eqat.workspace(1, N, K, b, g, torch.bfloat16, dev)
        for _ in range(4):
            eqat.dq_linear_fwd(X, c, z, s_, b, g, ws=ws)
        torch.cuda.synchronize()
        if eqat.device_error() != 0:
            raise RuntimeError("device error word set")
        print(json.dumps({"gemv_only": "ok"}), flush=True)
        return
    if args.initpack70b_only:  # profiling aid: just the 70B-block init/pack measurement
        torch.cuda.set_device(0)
        eqat.load_library()
        print(json.dumps(initpack_70b_block(torch.device("cuda", 0), reps=1)), flush=True)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
