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

CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, read (never set) through NVML by
    a background thread every `period_s`, with a wall-clock stamp per sample, so that
    the samples inside a short timed region can be picked out afterwards.  mark()
    records the wall clock of the region's ends.  If NVML is unavailable it falls
    back to `nvidia-smi -lms 200`, which sees only regions longer than its period."""

    def __init__(self, device: torch.device, period_s: float = 0.0005):
        self.device = device
        self.period = period_s
        self.samples = []  # (t, sm_mhz, reasons set)
        self.marks = {}
        self.sm_max = None
        self._stop = None
        self._thread = None
        self._smi = None
        self.source = "none"

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:  # noqa: BLE001 - fall back to the CUDA ordinal
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            self._stop = threading.Event()

            def loop():
                while not self._stop.is_set():
                    t = time.perf_counter()
                    try:
                        mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    except Exception:  # noqa: BLE001
                        break
                    self.samples.append((t, mhz, {n for n, b in bits.items() if r & b}))
                    self._stop.wait(self.period)
            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
            self.source = "nvml"
        except Exception:  # noqa: BLE001 - no NVML: nvidia-smi's own sampler
            fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                      "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                      "clocks_event_reasons.sw_power_cap")
            try:
                self._smi = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.device.index or 0}", f"--query-gpu={fields}",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self._t0 = time.perf_counter()
                self.source = "nvidia-smi"
            except OSError:
                self._smi = None
        return self

    def mark(self, name):
        self.marks[name] = time.perf_counter()

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._smi is not None:
            self._smi.terminate()
            try:
                out, _ = self._smi.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._smi.kill()
                out, _ = self._smi.communicate()
            # nvidia-smi gives no timestamps here: treat its samples as spread evenly
            lines = [l for l in out.splitlines() if l.strip()]
            t1 = time.perf_counter()
            for i, l in enumerate(lines):
                f = [x.strip() for x in l.split(",")]
                try:
                    mhz, self.sm_max = float(f[0]), float(f[1])
                except (ValueError, IndexError):
                    continue
                rs = {n for n, v in zip(CLOCK_REASONS, f[2:6]) if v.lower().startswith("active")}
                self.samples.append((self._t0 + (t1 - self._t0) * (i + 0.5) / max(1, len(lines)), mhz, rs))

    def summary(self, start="start", end="end"):
        """Samples inside [mark start, mark end], plus the last sample before the
        region and the first after it (the region is often shorter than a few ms)."""
        t0, t1 = self.marks.get(start), self.marks.get(end)
        inside = [x for x in self.samples if t0 is not None and t1 is not None and t0 <= x[0] <= t1]
        before = [x for x in self.samples if t0 is not None and x[0] < t0][-1:]
        after = [x for x in self.samples if t1 is not None and x[0] > t1][:1]
        use = inside or (before + after)
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": ["unsampled"], "samples": 0,
                    "source": self.source}
        reasons = set()
        for x in use:
            reasons |= x[2]
        return {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": self.sm_max,
                "reasons": sorted(reasons), "samples": len(inside),
                "sm_mhz_before": before[0][1] if before else None, "sm_mhz_after": after[0][1] if after else None,
                "region_ms": round((t1 - t0) * 1e3, 3) if t0 is not None and t1 is not None else None,
                "source": self.source}


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
        """One step; `events` maps phase boundaries (0 = before init ... 6 = after the
        E2E-QP backward) to CUDA events recorded there."""
        b, g = self.bits, self.group

        def mark(i):
            if events is not None and events.get(i) is not None:
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


def code_bytes(N, K, bits):
    """Bytes of the packed codes: 2-bit 4 per byte, 4-bit 2 per byte, 3-bit one per byte."""
    return N * K // 4 if bits == 2 else N * K // 2 if bits == 4 else N * K


def hbm_bytes(kernel, N, K, bits, group, wbytes=2):
    """Algorithmic HBM bytes of one launch of an HBM-bound kernel over an [N, K]
    weight: every input read once and every output written once.
      init     W, then s and z (fp32)
      pack     W, s, z, then the codes and zq (uint8)
      prepass  W, s, z, then W-hat (the weight's dtype)
      dequant  codes, zq, s, then W-hat"""
    G = K // group
    if kernel == "init":
        return N * K * wbytes + 8 * N * G
    if kernel == "pack":
        return N * K * wbytes + 8 * N * G + code_bytes(N, K, bits) + N * G
    if kernel == "prepass":
        return 2 * N * K * wbytes + 8 * N * G
    if kernel == "dequant":
        return code_bytes(N, K, bits) + 5 * N * G + N * K * wbytes
    raise ValueError(kernel)


def phase_bytes(M, N, K, bits, group):
    """Algorithmic HBM bytes of the two HBM-bound phases of the step (bf16 W)."""
    return hbm_bytes("init", N, K, bits, group), hbm_bytes("pack", N, K, bits, group)


class L2Flush:
    """Leaves L2 holding none of the next kernel's data and no dirty lines: a write
    of 512 MiB (4x L2), then a read of 256 MiB of another buffer, so the next kernel
    neither hits in L2 nor first writes back the flush's own dirty lines."""

    def __init__(self, dev):
        self.w = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.amax()


def bench_config(world):
    """The `config` of both arms' JSON lines (the reference arm prints the same dict)."""
    wl = WORKLOAD
    lin = wl.linears[0]
    return {"workload": wl.name, "M": wl.m, "N": lin.n, "K": lin.k, "bits": wl.bits, "group": wl.group,
            "flops_per_step": 12 * wl.m * lin.n * lin.k,
            "l2": "flushed before every step (512 MiB write, then a 256 MiB read of another buffer)",
            "parallelism": f"dp{world}" if world > 1 else "single-gpu",
            "step": "+".join(PHASES)}


def choose_gemm_peak(peaks, region_s):
    """The measured bf16 peak that matches how long the kernel ran back to back: the
    burst figure for a region under a second (the GPU does not reach its power-capped
    clock in that time), the sustained one for a longer region."""
    if region_s < 1.0:
        return peaks["bf16_tflops"], f"bf16 dense, burst (timed region {region_s * 1e3:.1f} ms < 1 s), {peaks['source']}"
    return peaks["bf16_tflops_sustained"], f"bf16 dense, sustained (timed region {region_s:.1f} s), {peaks['source']}"


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
    flush = L2Flush(dev)

    allreduce = None
    if dist is not None:
        def allreduce(ts):
            dp.allreduce_weight_grads(ts, dist)

    nph = len(PHASES)
    dom = PHASES.index(DOMINANT)

    def new_events(bounds):
        return {j: torch.cuda.Event(enable_timing=True) for j in bounds}

    # Timed region: events at the step's ends and around the dominant launch only.
    # An event between two launches costs about 2.7 us of a 0.54 ms step on B200
    # (it also stops the next kernel from starting before the previous one ends),
    # so the phase breakdown comes from a second pass with an event at every
    # boundary, after the timed region.
    ev = [new_events((0, dom, dom + 1, nph)) for _ in range(args.steps)]
    with ClockSampler(dev) as clk:
        for _ in range(args.warmup):
            flush()
            step.run(allreduce=allreduce)
        torch.cuda.synchronize()
        if eqat.device_error() != 0:
            raise RuntimeError("device error word set during warm-up")
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        clk.mark("start")
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush()
            step.run(events=ev[i], allreduce=allreduce)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
        clk.mark("end")
        time.sleep(0.01)  # one more sample after the region
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if eqat.device_error() != 0:
        raise RuntimeError("device error word set during the timed region")
    step_ms = [ev[i][0].elapsed_time(ev[i][nph]) for i in range(args.steps)]
    dom_in_region = [ev[i][dom].elapsed_time(ev[i][dom + 1]) for i in range(args.steps)]
    # phase breakdown: the same steps again, an event at every boundary
    evp = [new_events(range(nph + 1)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush()
        step.run(events=evp[i], allreduce=allreduce)
    torch.cuda.synchronize()
    phase_ms = {p: [evp[i][j].elapsed_time(evp[i][j + 1]) for i in range(args.steps)] for j, p in enumerate(PHASES)}
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
    dom_ms = sum(dom_in_region) / len(dom_in_region)
    dom_flops = 4 * M * N * K
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    peak, peak_kind = choose_gemm_peak(peaks, t_wall)
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

    # HBM-bound kernels: each timed alone after a clean flush, on the step's layer and
    # over the seven linears of the Llama-2-70B block
    hbm = hbm_kernels(step, dev, peaks, flush) if not args.no_hbm else {}
    ip = initpack_70b_block(dev, peaks) if not args.no_initpack70b else None
    if ip is not None:
        for k in ("init", "pack", "prepass", "dequant"):
            hbm.setdefault(k, {})["llama2-70b-block"] = ip[k]
        for k in ("init", "pack"):
            hbm[k]["llama2-70b-block_per_layer"] = ip[k + "_per_layer"]
    for k, ms, b in (("init", mean["init"], init_b), ("pack", mean["pack"], pack_b)):
        gbs = b / (ms * 1e-3) / 1e9
        hbm.setdefault(k, {})["in_step"] = {"GBps": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4),
                                            "bytes": b, "us": round(ms * 1e3, 2)}
    hbm["peak_GBps"] = peaks["hbm_gbs"]
    hbm["peak_kind"] = f"copy bandwidth, {peaks['source']}"
    hbm["note"] = ("algorithmic bytes (each input read once, each output written once) / CUDA-event time; "
                   "'in_step' inside the timed step, the others alone after a clean L2 flush")

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
        "config": bench_config(world),
        "roofline": {"bound": "tensor",
                     "kernel": "k_gemm_tc2 grouped backward on CTA pairs: dY W-hat + dY^T X with the fused "
                               "straight-through epilogue",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": peak_kind,
                     "frac_of_sustained_peak": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "hbm": hbm},
        "gpu_launches": sum(LAUNCHES_PER_STEP.values()) * args.steps,
        "clocks": clocks,
        "wall_s_timed": round(t_wall, 3),
        "e2e": e2e,
        "phases_ms": {p: round(v, 4) for p, v in mean.items()},
        "phases_note": ("a second pass of the same number of steps after the timed region, with an event at "
                        "every phase boundary (events between launches cost a few us each, so the timed region "
                        "has them only at the step's ends and around the dominant launch)"),
        "phase_rates": {
            "blockap_fwd_bwd_TFLOPs": round(6 * M * N * K / ((mean["fq_fwd"] + mean["fq_bwd"]) * 1e-3) / 1e12, 2),
            "e2e_fwd_bwd_TFLOPs": round(6 * M * N * K / ((mean["dq_fwd"] + mean["dq_bwd"]) * 1e-3) / 1e12, 2),
        },
    }
    if not args.no_variants:
        line["variants"] = quantizer_variants(step, dev)
    if not args.no_gemv:
        line["decode_gemv"] = decode_gemv(dev, peaks)
    if not args.no_blockap:
        line["blockap_block"] = blockap_block(dev, peaks)
    if not args.no_cfg1:
        line["cfg1_latency"] = cfg1_latency(dev)
    if not args.no_configs:
        line["per_config"] = per_config(dev, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(target_s=args.cpu_seconds, plan=not args.no_oracle_plan)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def timed_alone(fn, flush, reps):
    """Median CUDA-event time (ms) of fn() over `reps` calls, each after a clean L2 flush."""
    out = []
    for r in range(reps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush()
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        if r >= 2:
            out.append(e0.elapsed_time(e1))
    return statistics.median(out)


def hbm_kernels(step, dev, peaks, flush, reps=20):
    """The four HBM-bound quantizer kernels on the step's layer, each launched alone
    after a clean L2 flush: min-max init, pack, the Block-AP prepass (eqat_fake_quant
    writing W-hat only: the kernel inside eqat_fq_linear_fwd) and the E2E-QP
    dequantization (eqat_dequant_codes)."""
    b, g, N, K = step.bits, step.group, step.N, step.K
    wh = torch.empty_like(step.W)
    calls = {
        "init": lambda: eqat.minmax_init(step.W, b, g, s=step.s, z=step.z),
        "pack": lambda: eqat.pack_codes(step.W, step.s, step.z, b, g, codes=step.codes, zq=step.zq),
        "prepass": lambda: eqat.fake_quant(step.W, step.s, step.z, b, g, want_code=False, want_mask=False, W_hat=wh),
        "dequant": lambda: eqat.dequant_codes(step.codes, step.zq, step.s, K, b, g, out=wh),
    }
    out = {}
    for k, fn in calls.items():
        ms = timed_alone(fn, flush, reps)
        byts = hbm_bytes(k, N, K, b, g)
        gbs = byts / (ms * 1e-3) / 1e9
        out[k] = {step_layer_name(): {"GBps": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4),
                                      "bytes": byts, "us": round(ms * 1e3, 2)}}
    return out


def step_layer_name():
    return "llama2-7b-q_proj"


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


def fused_linears(wl):
    """The linears of a workload as they are launched: k_proj and v_proj of the 70B
    block read the same X and have the same K, so their weights are stored as one
    [N_k + N_v, K] matrix (k's rows, then v's) and run as one linear, the usual fused
    k/v projection.  Groups never cross rows, so s, z and the codes of the fused
    layer are the row-concatenations of the two layers', and every output element is
    the one the separate layers give (Y_k, Y_v are the column blocks of Y_kv).
    Returns (name, N, K, [member names])."""
    lins = list(wl.linears)
    names = [l.name for l in lins]
    out = []
    for l in lins:
        if l.name == "v_proj" and "k_proj" in names:
            continue
        if l.name == "k_proj" and "v_proj" in names:
            v = lins[names.index("v_proj")]
            if v.k == l.k:
                out.append(("kv_proj", l.n + v.n, l.k, ["k_proj", "v_proj"]))
                continue
        out.append((l.name, l.n, l.k, [l.name]))
    return out


def per_config(dev, peaks, reps=10):
    """Fake-quant linear forward + backward throughput per linear and per config, for the
    bf16 workloads (Llama-2 7B q_proj; 7B MLP w3g128; 13B E2E-QP w2g64 on packed codes;
    70B block w2g64, k_proj and v_proj as one fused kv linear).  Block-AP: fq_linear_fwd
    then fq_linear_bwd (dX, dW, ds, dz, W-hat reused); E2E-QP: dq_linear_fwd then
    dq_linear_bwd_s (dX, ds).  6 M N K per linear; CUDA events around `reps`
    back-to-back fwd+bwd pairs after 2 warm ones, so each linear's timed region is a
    few ms and its fraction is of the burst bf16 peak.  Inputs are drawn on the device
    (seeded); the per-linear bytes exceed L2 for all but the smallest."""
    out = {}
    gen = torch.Generator(device=dev)
    peak = peaks["bf16_tflops"]
    for idx in (2, 3, 4, 5):
        wl = synthetic.WORKLOADS[idx]
        M, b, g = wl.m, wl.bits, wl.group
        lines, tot_flops, tot_ms = {}, 0, 0.0
        for name, N, K, members in fused_linears(wl):
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
            lines[name] = {"N": N, "K": K, "us": round(ms * 1e3, 1),
                           "TFLOPs": round(fl / (ms * 1e-3) / 1e12, 1),
                           "frac_bf16_burst": round(fl / (ms * 1e-3) / 1e12 / peak, 3)}
            if len(members) > 1:
                lines[name]["fused"] = "+".join(members)
            tot_flops += fl
            tot_ms += ms
            del X, W, dY, ws, Y, out_b
            torch.cuda.empty_cache()
        out[wl.name] = {"M": M, "bits": b, "group": g, "mode": wl.mode, "linears": lines,
                        "TFLOPs": round(tot_flops / (tot_ms * 1e-3) / 1e12, 1),
                        "frac_bf16_burst": round(tot_flops / (tot_ms * 1e-3) / 1e12 / peak, 3)}
    out["peak_TFLOPs"] = peak
    out["note"] = ("6 M N K per linear (forward + dX + dW-hat), prepasses included; no L2 flush between calls; "
                   "fractions of the measured burst bf16 peak (each linear's timed region is a few ms)")
    return out


def cfg1_latency(dev, reps=50):
    """The fp32 parity workload (one linear, M = 128, W [512, 256], w2g64), which is
    latency-bound: median CUDA-event time of each call of the step, alone (each
    call synchronised), and of the whole step issued back to back."""
    wl = synthetic.WORKLOADS[1]
    d = synthetic.workload_linear(wl, 0)
    X, W, dY = (d[k].to(dev) for k in ("X", "W", "dY"))
    M, N, K = X.shape[0], W.shape[0], W.shape[1]
    b, g = wl.bits, wl.group
    ws = eqat.workspace(M, N, K, b, g, torch.float32, dev)
    s, z = eqat.minmax_init(W, b, g)
    codes, zq = eqat.pack_codes(W, s, z, b, g)
    bufs = dict(Y=torch.empty(M, N, device=dev), out=(torch.empty(M, K, device=dev), torch.empty(N, K, device=dev),
                                                     torch.empty_like(s), torch.empty_like(s)),
                out2=(torch.empty(M, K, device=dev), torch.empty_like(s)))
    calls = {
        "init": lambda: eqat.minmax_init(W, b, g, s=s, z=z),
        "fq_fwd": lambda: eqat.fq_linear_fwd(X, W, s, z, b, g, ws=ws, Y=bufs["Y"]),
        "fq_bwd": lambda: eqat.fq_linear_bwd(X, W, s, z, dY, b, g, ws=ws, out=bufs["out"], w_hat_in_ws=True),
        "pack": lambda: eqat.pack_codes(W, s, z, b, g, codes=codes, zq=zq),
        "dq_fwd": lambda: eqat.dq_linear_fwd(X, codes, zq, s, b, g, ws=ws, Y=bufs["Y"]),
        "dq_bwd": lambda: eqat.dq_linear_bwd_s(X, codes, zq, s, dY, b, g, ws=ws, out=bufs["out2"], w_hat_in_ws=True),
    }
    res = {}
    for name, fn in calls.items():
        fn()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        res[name + "_us"] = round(statistics.median(ts), 2)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for fn in calls.values():
            fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    res["step_us"] = round(statistics.median(ts), 2)
    res.update(workload=wl.name, dtype="f32", note="median CUDA-event time; each call alone, then the six "
               "calls issued back to back (host launch cost included: the layer is latency-bound)")
    return res


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
    out["note"] = ("GPU time per call from a CUDA graph of back-to-back calls: one kernel for layers with few row "
                   "tiles (clusters sum the partials on chip), else the streaming kernel and the partial sum, and "
                   "above the build-mode size also the X-fragment kernel; bf16 matvec = torch.matmul on bf16 "
                   "weights, same method")
    return out


def initpack_70b_block(dev, peaks, reps=5):
    """HBM throughput of the four quantizer kernels over all seven linears of the
    Llama-2-70B block (855.6 M bf16 weights, w2g64): min-max init, pack, the Block-AP
    prepass (W-hat only) and the E2E-QP dequantization of the packed codes.

    Init and pack of the block are one call each (eqat_minmax_init_multi,
    eqat_pack_codes_multi: the sweep initialises and packs all seven linears
    together); they are also timed layer by layer ("<kernel>_per_layer": sum of the
    seven single-layer calls).  The prepass and dequant run once per linear inside
    the training step, so they are timed layer by layer only.  GB/s = algorithmic
    bytes / median CUDA-event time, each call alone after a clean L2 flush (a 512 MiB
    write, then a 256 MiB read of another buffer, so the kernel starts on clean lines
    instead of first writing back the flush's dirty ones).  Weights are seeded
    N(0, 0.015) with 0.1% x10 outliers, drawn on the device."""
    wl = synthetic.WORKLOADS[5]
    gen = torch.Generator(device=dev)
    gen.manual_seed(1005)
    flush = L2Flush(dev)
    b, g = wl.bits, wl.group
    Ws, ss, zs, codes, zqs = [], [], [], [], []
    for lin in wl.linears:
        N, K = lin.n, lin.k
        W = torch.randn(N, K, generator=gen, device=dev).mul_(wl.sigma)
        idx = torch.randint(0, N * K, ((N * K) // 1000,), generator=gen, device=dev)
        W.view(-1)[idx] *= 10.0
        Ws.append(W.to(torch.bfloat16))
        del W, idx
        G = K // g
        ss.append(torch.empty((N, G), dtype=torch.float32, device=dev))
        zs.append(torch.empty((N, G), dtype=torch.float32, device=dev))
        codes.append(torch.empty((N, eqat.packed_row_bytes(K, b)), dtype=torch.uint8, device=dev))
        zqs.append(torch.empty((N, G), dtype=torch.uint8, device=dev))
    wh = torch.empty(max(W.numel() for W in Ws), dtype=torch.bfloat16, device=dev)
    kinds = ("init", "pack", "prepass", "dequant")
    t = dict.fromkeys(kinds, 0.0)
    nbytes = dict.fromkeys(kinds, 0)
    for i, lin in enumerate(wl.linears):
        N, K = lin.n, lin.k
        W, s, z = Ws[i], ss[i], zs[i]
        whi = wh[:N * K].view(N, K)
        calls = {
            "init": lambda: eqat.minmax_init(W, b, g, s=s, z=z),
            "pack": lambda: eqat.pack_codes(W, s, z, b, g, codes=codes[i], zq=zqs[i]),
            "prepass": lambda: eqat.fake_quant(W, s, z, b, g, want_code=False, want_mask=False, W_hat=whi),
            "dequant": lambda: eqat.dequant_codes(codes[i], zqs[i], s, K, b, g, out=whi),
        }
        for k in kinds:  # in this order: pack and dequant read what init and pack wrote
            t[k] += timed_alone(calls[k], flush, reps)
            nbytes[k] += hbm_bytes(k, N, K, b, g)
    block = {
        "init": timed_alone(lambda: eqat.minmax_init_multi(Ws, b, g, ss, zs), flush, reps),
        "pack": timed_alone(lambda: eqat.pack_codes_multi(Ws, ss, zs, b, g, codes, zqs), flush, reps),
    }
    del Ws, ss, zs, codes, zqs, wh
    torch.cuda.empty_cache()

    def entry(ms, byts, how):
        gbs = byts / (ms * 1e-3) / 1e9
        return {"GBps": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes": byts,
                "us": round(ms * 1e3, 1), "how": how}

    out = {}
    for k in ("init", "pack"):
        out[k] = entry(block[k], nbytes[k], "one call for the seven linears")
        out[k + "_per_layer"] = entry(t[k], nbytes[k], "seven single-layer calls")
    for k in ("prepass", "dequant"):
        out[k] = entry(t[k], nbytes[k], "seven single-layer calls")
    out["workload"] = wl.name + " (all 7 linears, 855.6 M weights)"
    return out


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


def cpu_baseline(target_s: float = 15.0, plan: bool = True):
    import oracle
    rows = calibrate_rows(target_s)
    dt, flops, desc = oracle_sample(rows)
    out = {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
           "cpu": cpu_model(), "kind": "oracle", "sample": desc, "seconds": round(dt, 2)}
    if plan:
        out["configs"] = oracle_plan()
    return out


def oracle_step_cfg1(reps=5):
    """Median seconds of the oracle's whole step on the fp32 parity workload (one
    linear, M = 128, W [512, 256], w2g64): init, Block-AP forward and backward, pack,
    E2E-QP forward and backward, every row."""
    import oracle
    wl = synthetic.WORKLOADS[1]
    d = synthetic.workload_linear(wl, 0)
    X, W, dY = (synthetic.as_f32_numpy(d[k]) for k in ("X", "W", "dY"))
    b, g = wl.bits, wl.group
    ts = []
    for _ in range(reps + 1):
        t0 = time.perf_counter()
        s, z = oracle.minmax_init(W, b, g)
        oracle.fq_linear_fwd(X, W, s, z, b, g)
        oracle.fq_linear_bwd(X, W, s, z, dY, b, g)
        packed, zq = oracle.pack(W, s, z, b, g)
        oracle.dq_linear_fwd(X, packed, zq, s, b, g)
        oracle.dq_linear_bwd_s(X, packed, zq, s, dY, b, g)
        ts.append(time.perf_counter() - t0)
    return statistics.median(ts[1:]), oracle.num_threads()


def oracle_linear_times(wl, li, frac, rng):
    """Seconds of the oracle on one linear of a workload with a `frac` of the token
    rows (Y, dX) and of the weight rows (dW-hat and the per-group gradients): init
    and pack of all weights are timed on their own, the rest in one call chain."""
    import oracle
    d = synthetic.workload_linear(wl, li)
    X, W, dY = (synthetic.as_f32_numpy(d[k]) for k in ("X", "W", "dY"))
    del d
    M, N = X.shape[0], W.shape[0]
    b, g = wl.bits, wl.group
    r = np.sort(rng.choice(M, max(1, int(round(M * frac))), replace=False))
    wr = np.sort(rng.choice(N, max(1, int(round(N * frac))), replace=False))
    t0 = time.perf_counter()
    s, z = oracle.minmax_init(W, b, g)
    t1 = time.perf_counter()
    packed, zq = oracle.pack(W, s, z, b, g)
    t2 = time.perf_counter()
    if wl.mode == "e2e_qp":
        oracle.dq_linear_fwd(X, packed, zq, s, b, g, rows=r)
        oracle.dq_linear_bwd_s(X, packed, zq, s, dY, b, g, rows=r, wrows=wr)
    else:
        oracle.fq_linear_fwd(X, W, s, z, b, g, rows=r)
        oracle.fq_linear_bwd(X, W, s, z, dY, b, g, rows=r, wrows=wr)
    t3 = time.perf_counter()
    return t1 - t0, t2 - t1, t3 - t2


def oracle_plan(budget_s: float = 120.0):
    """The oracle's time on the other workloads: the fp32 parity workload in full, on
    all host threads and on one; the three large bf16 workloads on a sample, with the
    full problem's time extrapolated.  For each linear the contraction part is timed
    at two sample fractions f and 2f of the token and weight rows; its cost is a
    fixed part (W-hat) plus a part linear in f, so the full time is the straight line
    through the two points at f = 1.  Init and pack run on every weight.  Workloads
    that would exceed `budget_s` seconds in all are left out and say so."""
    out = {}
    t_all, nthr = oracle_step_cfg1()
    one = None
    try:
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--oracle-cfg1-only"],
                           env=dict(os.environ, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES=""),
                           capture_output=True, text=True, timeout=300)
        one = json.loads(r.stdout.strip().splitlines()[-1]) if r.returncode == 0 else None
    except (subprocess.TimeoutExpired, ValueError, IndexError):
        one = None
    out[synthetic.WORKLOADS[1].name] = {
        "what": "whole step, every row (init, Block-AP fwd+bwd, pack, E2E-QP fwd+bwd)",
        "threads_all": {"ms": round(t_all * 1e3, 3), "threads": nthr},
        "threads_1": {"ms": round(one["seconds"] * 1e3, 3), "threads": one["threads"]} if one else None,
        "label": "measured"}
    t_begin = time.perf_counter()
    rng = np.random.default_rng(11)
    for idx, f in ((3, 1 / 256), (4, 1 / 256), (5, 1 / 256)):
        wl = synthetic.WORKLOADS[idx]
        if time.perf_counter() - t_begin > budget_s:
            out[wl.name] = {"label": "not run (time budget of the baseline spent)"}
            continue
        t0 = time.perf_counter()
        full = 0.0
        init_pack = 0.0
        for li in range(len(wl.linears)):
            ti, tp, tc1 = oracle_linear_times(wl, li, f, rng)
            _, _, tc2 = oracle_linear_times(wl, li, 2 * f, rng)
            slope = max((tc2 - tc1) / f, 0.0)
            fixed = max(tc1 - slope * f, 0.0)
            full += ti + tp + fixed + slope
            init_pack += ti + tp
        out[wl.name] = {"seconds_full": round(full, 2), "label": "extrapolated",
                        "init_pack_seconds": round(init_pack, 2),
                        "seconds_spent": round(time.perf_counter() - t0, 2),
                        "sample": f"per linear: init+pack of every weight; fwd, dX and weight-side gradients on "
                                  f"{f:.5f} and {2 * f:.5f} of the token and weight rows, extrapolated to all rows",
                        "flops_full": wl.flops_per_step(),
                        "TFLOPs_extrapolated": round(wl.flops_per_step() / full / 1e12, 6),
                        "threads": nthr}
    return out


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
            "config": bench_config(args.gpus),
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
    ap.add_argument("--quant-multi-only", action="store_true")
    ap.add_argument("--quant-gate-only", action="store_true")
    ap.add_argument("--dq-only", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-hbm", action="store_true")
    ap.add_argument("--no-cfg1", action="store_true")
    ap.add_argument("--no-oracle-plan", action="store_true")
    ap.add_argument("--oracle-cfg1-only", action="store_true")
    args = ap.parse_args()
    if args.oracle_cfg1_only:  # the oracle's fp32 parity step, in a process of its own (its thread count)
        sec, thr = oracle_step_cfg1()
        print(json.dumps({"seconds": sec, "threads": thr}), flush=True)
        return
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
    if args.dq_only:  # profiling aid: one E2E-QP forward and backward on the step's workload
        torch.cuda.set_device(0)
        eqat.load_library()
        dev = torch.device("cuda", 0)
        step = Step(WORKLOAD, 0, WORKLOAD.bits, WORKLOAD.group, dev)
        b, g = step.bits, step.group
        eqat.minmax_init(step.W, b, g, s=step.s, z=step.z)
        eqat.pack_codes(step.W, step.s, step.z, b, g, codes=step.codes, zq=step.zq)
        eqat.dq_linear_fwd(step.X, step.codes, step.zq, step.s, b, g, ws=step.ws, Y=step.Y2)
        eqat.dq_linear_bwd_s(step.X, step.codes, step.zq, step.s, step.dY, b, g, ws=step.ws,
                             out=(step.dX2, step.ds2), w_hat_in_ws=True)
        torch.cuda.synchronize()
        if eqat.device_error() != 0:
            raise RuntimeError("device error word set")
        print(json.dumps({"dq_only": "ok"}), flush=True)
        return
    if args.quant_gate_only:  # profiling aid: init, prepass, pack, dequant once each on the 70B gate_proj
        torch.cuda.set_device(0)
        eqat.load_library()
        dev = torch.device("cuda", 0)
        gen = torch.Generator(device=dev)
        gen.manual_seed(1008)
        W = (torch.randn(28672, 8192, generator=gen, device=dev) * 0.015).to(torch.bfloat16)
        s_, z_ = eqat.minmax_init(W, 2, 64)
        wh = torch.empty_like(W)
        eqat.fake_quant(W, s_, z_, 2, 64, want_code=False, want_mask=False, W_hat=wh)
        codes, zq = eqat.pack_codes(W, s_, z_, 2, 64)
        eqat.dequant_codes(codes, zq, s_, 8192, 2, 64, out=wh)
        torch.cuda.synchronize()
        if eqat.device_error() != 0:
            raise RuntimeError("device error word set")
        print(json.dumps({"quant_gate_only": "ok"}), flush=True)
        return
    if args.quant_multi_only:  # profiling aid: block-wide init and pack once each, Llama-2-7B block shapes
        torch.cuda.set_device(0)
        eqat.load_library()
        dev = torch.device("cuda", 0)
        gen = torch.Generator(device=dev)
        gen.manual_seed(1007)
        shapes = [(4096, 4096)] * 4 + [(11008, 4096), (11008, 4096), (4096, 11008)]
        Ws = [(torch.randn(N, K, generator=gen, device=dev) * 0.02).to(torch.bfloat16) for N, K in shapes]
        ss, zs = eqat.minmax_init_multi(Ws, 2, 64)
        eqat.pack_codes_multi(Ws, ss, zs, 2, 64)
        torch.cuda.synchronize()
        if eqat.device_error() != 0:
            raise RuntimeError("device error word set")
        print(json.dumps({"quant_multi_only": "ok", "weights": sum(N * K for N, K in shapes)}), flush=True)
        return
    if args.initpack70b_only:  # profiling aid: just the 70B-block init/pack measurement
        torch.cuda.set_device(0)
        eqat.load_library()
        print(json.dumps(initpack_70b_block(torch.device("cuda", 0), load_peaks(), reps=1)), flush=True)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
