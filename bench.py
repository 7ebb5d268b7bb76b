#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear hot path on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]

Default workload (the training-shape configuration the headline metric is quoted on): all 7
projections of one LLaMA-7B-shaped layer (h = 4096, FFN 11008) as packed NF4 (block 64,
double-quantized scales), LoRA r = 64, s = 0.25, 4096 tokens (batch 4 x seq 1024), bf16,
upstream gradient dY ~ N(0,1). One step = forward (qlora_linear_fwd) and backward
(qlora_linear_bwd) of all 7 linears; the weights are quantized once at load, as the frozen
base is never re-quantized. With N > 1 ranks every rank runs its own 4096 tokens (weak
scaling) and the adapter gradients are summed over ranks (NCCL all-reduce) inside the step.

Printed: one JSON line (rank 0) with the headline tokens/s, the roofline of the dominant
kernel (the fused NF4 tcgen05 GEMM), the CPU oracle baseline, the end-to-end figure through
the C ABI with host buffers, clocks, and the secondary legs (decode GEMV packed-weight GB/s,
quantize and dequantize GB/s).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

METRIC = "QLoRA NF4 linear fwd+bwd tokens/s"
UNIT = "tokens/s"
WORKLOAD = "llama7b_layer_7_linears_fwd_bwd_t4096_r64"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------------------
# setup helpers
# ------------------------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# the sources the fused NF4 GEMM is compiled from (its DRAM counters stay valid while these
# files are unchanged)
GEMM_SOURCES = ("nf4_gemm.cuh", "nf4_codec.cuh", "qlora_common.cuh")


def kernel_source_hash() -> str:
    csrc = os.path.join(ROOT, "bit_quantized_lora_03_b200", "csrc")
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel sources (else None: the counters no longer describe this code)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash():
        return None
    entry = d.get("kernels", {}).get(kernel)
    return None if entry is None else entry.get("dram_bytes_per_launch_full_size")


class ClockSampler:
    """SM clock, power and clock-event reasons of GPU `index` during a timed region: read
    through NVML every 5 ms by a background thread (a 0.1 s region still gets about twenty
    samples); where NVML cannot be used, `nvidia-smi -lms 50` in the background instead."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    NVML_PERIOD_S = 0.005

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.nvml = None
        self.rows = []              # NVML samples: (sm MHz, power W, set of reason names)
        self.max_mhz = None
        self.stop = None
        self.thread = None

    def _start_nvml(self):
        import threading
        import pynvml as nv
        nv.nvmlInit()
        try:
            h = nv.nvmlDeviceGetHandleByIndex(self.index)   # the index nvidia-smi --id takes
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}

            def sample():
                mask = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                return (float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                        nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                        {n for n, b in bits.items() if mask & b})
            self.rows.append(sample())          # one sample before the region starts
        except Exception:
            nv.nvmlShutdown()
            raise
        self.nvml = nv
        self.stop = threading.Event()

        def loop():
            try:
                while not self.stop.wait(self.NVML_PERIOD_S):
                    self.rows.append(sample())
            except Exception:
                pass
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def __enter__(self):
        try:
            self._start_nvml()
            return self
        except Exception:
            self.nvml, self.rows = None, []
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.nvml is not None:
            self.stop.set()
            self.thread.join(timeout=2.0)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        if self.nvml is not None:
            rows = list(self.rows)
            if not rows:
                return None
            return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": self.max_mhz,
                    "samples": len(rows),
                    "reasons": sorted({n for r in rows for n in r[2]}),
                    "power_w_max": max(r[1] for r in rows), "source": "nvml, every 5 ms"}
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        reasons = sorted({n for r in rows for n, v in zip(self.REASONS, r[5:9])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]), "samples": len(rows), "reasons": reasons,
                "power_w_max": max((num(r[3]) or 0.0) for r in rows),
                "source": "nvidia-smi, every 50 ms"}


# ------------------------------------------------------------------------------------------
# the workload on the GPU
# ------------------------------------------------------------------------------------------
class Layer:
    """One adapted linear resident on the device: packed W, adapters, inputs, outputs."""

    def __init__(self, i: int, dev, t: int, r: int, s: float):
        from bit_quantized_lora_03_b200 import binding as B
        from bit_quantized_lora_03_b200 import inputs
        li = inputs.training_linear(i, t=t, r=r, s=s)
        self.name, self.h, self.o, self.t, self.r, self.s = li.name, li.h, li.o, t, r, s
        self.p = B.nf4_quantize(li.Wt.to(dev))
        self.X, self.dY = li.X.to(dev), li.dY.to(dev)
        self.L1, self.L2 = li.L1.to(dev), li.L2.to(dev)
        self.Y = torch.empty(t, self.o, dtype=torch.bfloat16, device=dev)
        self.sT = torch.empty(t, r, dtype=torch.bfloat16, device=dev)
        self.dX = torch.empty(t, self.h, dtype=torch.bfloat16, device=dev)
        self.dL1 = torch.empty(self.h, r, dtype=torch.float32, device=dev)
        self.dL2 = torch.empty(r, self.o, dtype=torch.float32, device=dev)
        self.wsf = torch.empty(B.fwd_workspace_bytes(t, self.h, self.o, r), dtype=torch.uint8, device=dev)
        self.wsb = torch.empty(B.bwd_workspace_bytes(t, self.h, self.o, r), dtype=torch.uint8, device=dev)
        self.X_cpu, self.dY_cpu = li.X, li.dY

    def step(self):
        from bit_quantized_lora_03_b200 import binding as B
        B.qlora_linear_fwd(self.X, self.p, self.L1, self.L2, self.s, Y=self.Y, sT=self.sT, ws=self.wsf)
        B.qlora_linear_bwd(self.dY, self.X, self.p, self.L1, self.L2, self.s, sT=self.sT,
                           dX=self.dX, dL1=self.dL1, dL2=self.dL2, ws=self.wsb)

    def step_dropout(self, p: float, seed: int):
        """The same step with LoRA dropout on the adapter input (workspaces made on first use)."""
        from bit_quantized_lora_03_b200 import binding as B
        if not hasattr(self, "wsfd"):
            dev = self.X.device
            lib = B.lib()
            self.wsfd = torch.empty(lib.qlora_fwd_dropout_workspace_bytes(self.t, self.h, self.o, self.r),
                                    dtype=torch.uint8, device=dev)
            self.wsbd = torch.empty(lib.qlora_bwd_dropout_workspace_bytes(self.t, self.h, self.o, self.r),
                                    dtype=torch.uint8, device=dev)
            self.mask = torch.empty(B.dropout_mask_bytes(self.t, self.h), dtype=torch.uint8, device=dev)
        B.qlora_linear_fwd_dropout(self.X, self.p, self.L1, self.L2, self.s, p, seed, Y=self.Y,
                                   sT=self.sT, mask=self.mask, ws=self.wsfd)
        B.qlora_linear_bwd_dropout(self.dY, self.X, self.p, self.L1, self.L2, self.s, p, seed,
                                   sT=self.sT, mask=self.mask, dX=self.dX, dL1=self.dL1,
                                   dL2=self.dL2, ws=self.wsbd)

    def free_dropout(self):
        for k in ("wsfd", "wsbd", "mask"):
            if hasattr(self, k):
                delattr(self, k)


def step_all(layers, world, streams=None, one=None):
    """One step: fwd+bwd of every linear (`one(L)`, default L.step()). The linears are
    independent, so with `streams` they run round-robin on those streams (joined back to the
    caller's stream), letting one linear's kernels fill the SMs another's last wave leaves idle."""
    from bit_quantized_lora_03_b200 import dp
    one = one or (lambda L: L.step())
    if not streams:
        for L in layers:
            one(L)
    else:
        cur = torch.cuda.current_stream()
        go = torch.cuda.Event()
        go.record(cur)
        for st in streams:
            st.wait_event(go)
        for i, L in enumerate(layers):
            with torch.cuda.stream(streams[i % len(streams)]):
                one(L)
        for st in streams:
            done = torch.cuda.Event()
            done.record(st)
            cur.wait_event(done)
    if world > 1:
        dp.allreduce_adapter_grads([g for L in layers for g in (L.dL1, L.dL2)])


QUEUE_SLEEP_CYCLES = 40_000_000   # ~20 ms at 1.965 GHz: time for the host to queue a loop


def timed(fn, steps, warmup, world, dev):
    """Device time of `steps` calls of fn (after `warmup`), max over ranks, in ms."""
    from bit_quantized_lora_03_b200 import dp
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        fn()
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return dp.max_over_ranks(start.elapsed_time(end), dev)


def queued_ms(fn, reps, warmup):
    """Device time of `reps` calls of fn queued behind a device-side sleep, so that the events
    time back-to-back GPU work rather than the host's launch rate (single GPU legs)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    torch.cuda._sleep(QUEUE_SLEEP_CYCLES)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(reps):
        fn()
    end.record()
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def fused_gemm_flops(layers):
    """Algorithmic flops of the fused NF4 GEMM launches of one step: forward X.W' + sT.L2 and
    backward dY.W'^T + sU.L1^T, per linear."""
    f = 0
    for L in layers:
        f += 2 * L.t * L.h * L.o + 2 * L.t * L.r * L.o      # forward kernel
        f += 2 * L.t * L.o * L.h + 2 * L.t * L.r * L.h      # backward kernel
    return f


def step_flops(layers):
    """All algorithmic flops of one fwd+bwd step: 4 t h o + 6 t r (h + o) per linear."""
    return sum(4 * L.t * L.h * L.o + 6 * L.t * L.r * (L.h + L.o) for L in layers)


# ------------------------------------------------------------------------------------------
# secondary legs: decode GEMV, quantize, dequantize (HBM-bound)
# ------------------------------------------------------------------------------------------
def gemv_leg(dev, peaks, l2_bytes):
    from bit_quantized_lora_03_b200 import binding as B
    from bit_quantized_lora_03_b200 import inputs
    out = []
    for name, Wt in inputs.decode_gemv_weights():
        o, h = Wt.shape
        p0 = B.nf4_quantize(Wt.to(dev))
        del Wt
        ncopy = max(2, -(-4 * l2_bytes // p0.nbytes))      # rotate over >= 4x L2 of weights
        copies = [p0]
        for _ in range(ncopy - 1):
            q = B.PackedNF4(o, h, dev)
            q.codes.copy_(p0.codes)
            q.absmax_q8.copy_(p0.absmax_q8)
            q.absmax_s2.copy_(p0.absmax_s2)
            copies.append(q)
        L1, L2 = (a.to(dev) for a in inputs.decode_gemv_adapters(h, o, 16))
        for t in (1, 4, 16):
            X = inputs.decode_gemv_activations(h, t).to(dev)
            Y = torch.empty(t, o, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(B.fwd_workspace_bytes(t, h, o, 16), dtype=torch.uint8, device=dev)
            it = [0]

            def call():
                q = copies[it[0] % ncopy]
                it[0] += 1
                B.qlora_linear_fwd(X, q, L1, L2, 2.0, Y=Y, want_sT=False, ws=ws)
            reps = 4 * ncopy
            host_ms = timed(call, reps, ncopy, 1, dev) / reps
            # queued behind a device-side sleep, so that the events time the GPU work of
            # back-to-back calls rather than the host's launch rate
            torch.cuda.synchronize()
            torch.cuda._sleep(QUEUE_SLEEP_CYCLES)
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record()
            for _ in range(reps):
                call()
            end.record()
            torch.cuda.synchronize()
            ms = start.elapsed_time(end) / reps
            with B.KernelProfile() as prof:
                torch.cuda._sleep(QUEUE_SLEEP_CYCLES)
                for _ in range(reps):
                    call()
            k_ms = prof.ms["nf4_gemv_kernel"] / max(1, prof.launches["nf4_gemv_kernel"])
            call_kernels = sum(prof.launches.values()) // reps
            packed = p0.nbytes
            out.append({
                "weight": name, "t": t, "packed_bytes": packed,
                "call_us": round(ms * 1e3, 2),
                "host_bound_call_us": round(host_ms * 1e3, 2),
                "call_packed_gbs": round(packed / (ms * 1e-3) / 1e9, 1),
                "gemv_kernel_us": round(k_ms * 1e3, 2),
                "gemv_kernel_packed_gbs": round(packed / (k_ms * 1e-3) / 1e9, 1),
                "gemv_kernel_frac_hbm": round(packed / (k_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
                "kernels_per_call": call_kernels,
                "rotating_copies": ncopy})
        del copies, p0
        torch.cuda.empty_cache()
    return out


def codec_leg(dev, peaks):
    from bit_quantized_lora_03_b200 import binding as B
    from bit_quantized_lora_03_b200 import inputs
    W = [w.to(dev) for _, w in inputs.llama7b_quant_weights(with_outliers=True)]
    packs = [B.PackedNF4(w.shape[0], w.shape[1], dev) for w in W]
    outs = [torch.empty(w.shape, dtype=torch.bfloat16, device=dev) for w in W]
    n = sum(w.numel() for w in W)
    packed = sum(p.nbytes for p in packs)

    def quant():
        for w, p in zip(W, packs):
            B.nf4_quantize(w, out=p)

    def deq():
        for p, o_ in zip(packs, outs):
            B.nf4_dequantize(p, out=o_)
    qms = queued_ms(quant, 5, 2) / 5
    dms = queued_ms(deq, 5, 2) / 5
    qbytes = 4 * n + packed
    dbytes = packed + 2 * n
    res = {
        "weights": n,
        "quantize_ms": round(qms, 4), "quantize_gbs": round(qbytes / (qms * 1e-3) / 1e9, 1),
        "quantize_frac_hbm": round(qbytes / (qms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
        "dequantize_ms": round(dms, 4), "dequantize_gbs": round(dbytes / (dms * 1e-3) / 1e9, 1),
        "dequantize_frac_hbm": round(dbytes / (dms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
        "algorithmic_bytes": {"quantize": qbytes, "dequantize": dbytes},
    }
    del W, packs, outs
    torch.cuda.empty_cache()
    # one launch long enough for its steady rate: the layer's launches above cover 17-45 M
    # weights each (6-17 us at the copy bandwidth), where each launch's start and drain
    # (~2-3 us) weigh in; the 28672 x 8192 decode weight (235 M weights) is one launch
    o, h = 28672, 8192
    Wb = inputs.weight_f32(o, h, 301).to(dev)   # the decode recipe's seed for this shape
    pb = B.PackedNF4(o, h, dev)
    ob = torch.empty(o, h, dtype=torch.bfloat16, device=dev)
    qms = queued_ms(lambda: B.nf4_quantize(Wb, out=pb), 5, 2) / 5
    dms = queued_ms(lambda: B.nf4_dequantize(pb, out=ob), 5, 2) / 5
    qbytes, dbytes = 4 * o * h + pb.nbytes, pb.nbytes + 2 * o * h
    res["one_launch_28672x8192"] = {
        "quantize_ms": round(qms, 4),
        "quantize_frac_hbm": round(qbytes / (qms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
        "dequantize_ms": round(dms, 4),
        "dequantize_frac_hbm": round(dbytes / (dms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}
    del Wb, pb, ob
    torch.cuda.empty_cache()
    return res


def stack65b_leg(dev, peaks, steps: int = 2, warmup: int = 1):
    """The 65B-shaped stack (80 layers x 7 linears, 33.4 GB packed, t = 2048, r = 64): device
    time of full fwd+bwd steps through all 560 linears."""
    from bit_quantized_lora_03_b200 import binding as B
    from bit_quantized_lora_03_b200.stack65b import Stack65B
    import time as _time
    t0 = _time.time()
    st = Stack65B(dev)
    setup_s = _time.time() - t0
    ms = timed(st.step, steps, warmup, 1, dev)
    status = B.last_status()
    flops = st.flops_per_step()
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    res = {
        "workload": "llama65b_stack_80x7_linears_fwd_bwd_t2048_r64",
        "tokens_per_s": round(st.t * steps / (ms * 1e-3), 1),
        "ms_per_step": round(ms / steps, 2), "steps": steps, "warmup": warmup,
        "packed_weight_bytes": st.packed_bytes,
        "tflop_per_step": round(flops / 1e12, 2),
        "tflops": round(flops * steps / (ms * 1e-3) / 1e12, 1),
        "frac_of_sustained_bf16": round(flops * steps / (ms * 1e-3) / 1e12 / peak, 4),
        "launches_per_step": 6 * len(st.lin),
        "setup_s": round(setup_s, 1), "device_status": status,
    }
    del st
    torch.cuda.empty_cache()
    return res


def codebook_leg(dev):
    """The pages' format comparison on the LLaMA-7B-shaped layer's weights: relative
    reconstruction error (sum of squared errors / sum of squares) of NF4, FP4 and INT4 packing
    (same blocks and double-quantized scales), and of NF4 with the block scales in signed int8
    (/127) and FP8 E4M3 instead of unsigned 8-bit, on N(0, 0.02) weights with the 1% outliers
    at 8 sigma of the quantization workload and without them, and the quantizer's time for each."""
    from bit_quantized_lora_03_b200 import binding as B
    from bit_quantized_lora_03_b200 import inputs
    res = {}
    variants = (("nf4", B.CODEBOOK_NF4, B.SCALES_U8), ("fp4", B.CODEBOOK_FP4, B.SCALES_U8),
                ("int4", B.CODEBOOK_INT4, B.SCALES_U8),
                ("nf4_scales_s8", B.CODEBOOK_NF4, B.SCALES_S8),
                ("nf4_scales_e4m3", B.CODEBOOK_NF4, B.SCALES_E4M3))
    for tag, outl in (("with_outliers", True), ("gaussian", False)):
        W = [w.to(dev) for _, w in inputs.llama7b_quant_weights(with_outliers=outl)]
        res[tag] = {}
        for name, cb, fmt in variants:
            packs = [B.PackedNF4(w.shape[0], w.shape[1], dev) for w in W]

            def quant():
                for w, p in zip(W, packs):
                    B.nf4_quantize(w, out=p, codebook_id=cb, scale_format=fmt)
            ms = queued_ms(quant, 3, 1) / 3
            se, ss = 0.0, 0.0
            for w, p in zip(W, packs):
                d = B.nf4_dequantize(p, codebook_id=cb, scale_format=fmt).float()
                se += float((d - w).pow(2).sum())
                ss += float(w.pow(2).sum())
            res[tag][name] = {"rel_mse": round(se / ss, 6), "quantize_ms": round(ms, 4)}
            del packs
        del W
        torch.cuda.empty_cache()
    res["device_status"] = B.last_status()
    return res


def adamw_leg(dev, peaks, r: int = 64):
    """The adapters' update for the 7-linear layer (L1 and L2 of every linear: sum r (h + o) =
    4.997 M parameters): device time of one fused AdamW step over all 14 adapters with the
    state in device memory, with it in unified memory resident on the GPU, and with it in
    unified memory paged out to the host first (the paged optimizer's spike path)."""
    import ctypes
    from bit_quantized_lora_03_b200 import binding as B
    from bit_quantized_lora_03_b200 import inputs
    from cuda.bindings import runtime as rt
    sizes = [n for _, h, o in inputs.LLAMA7B_LINEARS for n in (h * r, r * o)]
    total = sum(sizes)
    p = [torch.randn(n, device=dev) * 0.01 for n in sizes]
    g = [torch.randn(n, device=dev) * 0.01 for n in sizes]
    p16 = [torch.empty(n, dtype=torch.bfloat16, device=dev) for n in sizes]
    md = [torch.zeros(n, device=dev) for n in sizes]
    vd = [torch.zeros(n, device=dev) for n in sizes]
    mu, vu = [], []
    for n in sizes:
        for lst in (mu, vu):
            err, ptr = rt.cudaMallocManaged(4 * n, rt.cudaMemAttachGlobal)
            assert err == rt.cudaError_t.cudaSuccess
            ctypes.memset(int(ptr), 0, 4 * n)
            lst.append(int(ptr))
    step = [0]

    def ptrs(xs):
        return [x if isinstance(x, int) else x.data_ptr() for x in xs]

    def run(ms, vs, flags=0):
        """All 14 adapters in one multi-tensor launch."""
        step[0] += 1
        B.adamw_step_multi_ptr(ptrs(p), ptrs(p16), ptrs(g), ptrs(ms), ptrs(vs), sizes, 1e-4, 0.9,
                               0.999, 1e-8, 0.0, step[0], flags)

    def run_each(ms, vs):
        """The same step as 14 single-tensor launches."""
        step[0] += 1
        for i, n in enumerate(sizes):
            B.adamw_step_ptr(p[i].data_ptr(), p16[i].data_ptr(), g[i].data_ptr(), ms[i].data_ptr(),
                             vs[i].data_ptr(), n, 1e-4, 0.9, 0.999, 1e-8, 0.0, step[0], 0)

    def paged_in(flags):
        """One step after the state was moved to host memory."""
        torch.cuda.synchronize()
        for ptr, n in zip(mu + vu, sizes + sizes):
            rt.cudaMemPrefetchAsync(ptr, 4 * n, rt.cudaCpuDeviceId, 0)
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        run(mu, vu, flags)
        end.record()
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    dev_ms = queued_ms(lambda: run(md, vd), 5, 2) / 5
    each_ms = queued_ms(lambda: run_each(md, vd), 5, 2) / 5
    uni_ms = queued_ms(lambda: run(mu, vu), 5, 2) / 5
    uni_pf_ms = queued_ms(lambda: run(mu, vu, B.ADAMW_PREFETCH), 5, 2) / 5
    paged_fault_ms = paged_in(0)
    paged_pf_ms = paged_in(B.ADAMW_PREFETCH)
    status = B.last_status()
    for ptr in mu + vu:
        rt.cudaFree(ptr)
    nbytes = 30 * total   # read p, g, m, v; write p, m, v (fp32) and the bf16 copy
    return {"params": total, "bytes_per_step": nbytes,
            "device_state_ms": round(dev_ms, 4),
            "device_state_gbs": round(nbytes / (dev_ms * 1e-3) / 1e9, 1),
            "device_state_frac_hbm": round(nbytes / (dev_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
            "device_state_14_launches_ms": round(each_ms, 4),
            "unified_state_resident_ms": round(uni_ms, 4),
            "unified_state_resident_prefetch_ms": round(uni_pf_ms, 4),
            "unified_state_paged_out_first_touch_ms": round(paged_fault_ms, 4),
            "unified_state_paged_out_prefetch_ms": round(paged_pf_ms, 4),
            "device_status": status}


def merge_leg(dev, peaks, r: int = 64, s: float = 0.25):
    """Adapter merge over the 7 linears of the LLaMA-7B-shaped layer: GB/s of the merge
    (write 4 B + read 0.516 B per weight) and of the re-quantization, and the output drift of
    one linear (up_proj, 4096 tokens) merged two ways against the unmerged layer: into the
    dequantized base then re-quantized to NF4, and into a 16-bit copy of the original base."""
    from bit_quantized_lora_03_b200 import binding as B
    from bit_quantized_lora_03_b200 import inputs
    lins = [inputs.training_linear(i, r=r, s=s) for i in range(7)]
    packs = [B.nf4_quantize(li.Wt.to(dev)) for li in lins]
    L1s = [li.L1.to(dev) for li in lins]
    L2s = [li.L2.to(dev) for li in lins]
    outs = [torch.empty(li.o, li.h, dtype=torch.float32, device=dev) for li in lins]
    reqs = [B.PackedNF4(li.o, li.h, dev) for li in lins]
    n = sum(li.o * li.h for li in lins)

    def merge():
        for p, a, b, o_ in zip(packs, L1s, L2s, outs):
            B.merge_adapters(p, a, b, s, out=o_)

    def requant():
        for o_, q in zip(outs, reqs):
            B.nf4_quantize(o_, out=q)
    mms = queued_ms(merge, 5, 2) / 5
    qms = queued_ms(requant, 5, 2) / 5
    mbytes = 4 * n + sum(p.nbytes for p in packs) + sum(2 * (a.numel() + b.numel()) for a, b in zip(L1s, L2s))
    # drift of up_proj
    li, p, pm = lins[5], packs[5], reqs[5]
    X = li.X.to(dev)
    Yu, _ = B.qlora_linear_fwd(X, p, L1s[5], L2s[5], s, want_sT=False)
    zero1, zero2 = torch.zeros_like(L1s[5]), torch.zeros_like(L2s[5])
    Ym, _ = B.qlora_linear_fwd(X, pm, zero1, zero2, 0.0, want_sT=False)
    W16 = (li.Wt.to(dev) + s * (L1s[5].float() @ L2s[5].float()).t()).to(torch.bfloat16)
    Y16 = X @ W16.t()   # a plain bf16 library GEMM, for the report only
    torch.cuda.synchronize()

    def rel(a, b):
        return round(float((a.float() - b.float()).pow(2).mean().sqrt() / b.float().pow(2).mean().sqrt()), 5)
    res = {
        "weights": n, "r": r, "s": s,
        "merge_ms": round(mms, 4), "merge_gbs": round(mbytes / (mms * 1e-3) / 1e9, 1),
        "merge_frac_hbm": round(mbytes / (mms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
        "requantize_ms": round(qms, 4),
        "drift_up_proj_t4096": {
            "merged_into_dequantized_then_nf4_vs_unmerged_rel_rms": rel(Ym, Yu),
            "merged_into_16bit_original_vs_unmerged_rel_rms": rel(Y16, Yu)},
        "device_status": B.last_status(),
    }
    del packs, outs, reqs, L1s, L2s
    torch.cuda.empty_cache()
    return res


def dropout_leg(dev, peaks, layers, streams, base_ms_step, steps: int = 30, p: float = 0.05):
    """The headline step with LoRA dropout p on every linear's adapter input (the mask drawn in
    the forward's kernels, a fresh seed per linear and step, and handed to the backward as
    bits): tokens/s against the same step without dropout, and the mask kernels' bandwidth
    (read 2 B + write 2 B per input element, + 1/8 B of mask bits)."""
    from bit_quantized_lora_03_b200 import binding as B
    t = layers[0].t
    counter = [0]

    def one(L):
        counter[0] += 1
        L.step_dropout(p, 0xD00D_0000 + counter[0])
    ms = timed(lambda: step_all(layers, 1, streams, one), steps, 3, 1, dev) / steps
    with B.KernelProfile() as prof:
        for _ in range(5):
            step_all(layers, 1, None, one)
    kname = "dropout_apply_kernel"
    n_mask = prof.launches.get(kname, 0)
    mask_ms = prof.ms.get(kname, 0.0) / max(1, n_mask)
    # each linear's fwd and bwd apply the mask to its t x h input once
    elems = sum(L.t * L.h for L in layers) * 2 * 5 / max(1, n_mask)
    gbs = 4.125 * elems / (mask_ms * 1e-3) / 1e9 if mask_ms else None
    tc_ms = prof.ms.get("tc_gemm_kernel", 0.0) / 5
    res = {"p": p, "tokens_per_s": round(t / (ms * 1e-3), 1), "ms_per_step": round(ms, 4),
           "vs_no_dropout_ms_per_step": round(base_ms_step, 4),
           "overhead": round(ms / base_ms_step - 1.0, 4),
           "mask_kernel_avg_ms": round(mask_ms, 4),
           "mask_kernel_gbs": round(gbs, 1) if gbs else None,
           "mask_kernel_frac_hbm": round(gbs / peaks["hbm_gbs"], 3) if gbs else None,
           "tc_gemm_ms_per_step": round(tc_ms, 4),
           "device_status": B.last_status()}
    for L in layers:
        L.free_dropout()
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ------------------------------------------------------------------------------------------
def oracle_sample(sample_tokens: int, prepared=None):
    """Oracle fwd+bwd of `sample_tokens` tokens for one linear of each shape class of the
    7-linear layer (q_proj 4096->4096 x4, up_proj 4096->11008 x2, down_proj 11008->4096 x1),
    including the per-step dequantization of W, scaled to the 7 linears.
    Returns (tokens_per_s, seconds_for_one_step_equivalent, prepared)."""
    from bit_quantized_lora_03_b200 import inputs
    from oracle import nf4_oracle as O
    classes = [(0, 4), (5, 2), (6, 1)]
    if prepared is None:
        prepared = []
        for i, mult in classes:
            li = inputs.training_linear(i)
            packed = O.nf4_quantize(li.Wt.numpy())
            f = lambda x: x[:sample_tokens].float().numpy()  # noqa: E731
            prepared.append((packed, f(li.X), f(li.dY), li.L1.float().numpy(),
                             li.L2.float().numpy(), li.s, mult))
    total = 0.0
    for packed, X, dY, L1, L2, s, mult in prepared:
        t0 = time.perf_counter()
        Wdq = O.nf4_dequantize(packed)
        O.qlora_linear_fwd(X, Wdq, L1, L2, s)
        O.qlora_linear_bwd(dY, X, Wdq, L1, L2, s)
        total += (time.perf_counter() - t0) * mult
    return sample_tokens / total, total, prepared


def oracle_sample_one_core(sample_tokens: int, prepared):
    """The same oracle sample with the BLAS pool limited to one thread (the oracle's other
    steps are single-threaded numpy already). None if the pool cannot be limited."""
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return None
    with threadpool_limits(limits=1):
        tps, sec, _ = oracle_sample(sample_tokens, prepared)
    return {"value": round(tps, 3), "unit": UNIT, "cores": 1, "seconds": round(sec, 2)}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------------------------------
# main
# ------------------------------------------------------------------------------------------
def oracle_linear_prep(i: int, sample_tokens: int):
    """The oracle's own packing of linear i of the layer and its first `sample_tokens` tokens
    (inputs and upstream gradients), for timing one linear per step (set-up, untimed)."""
    from bit_quantized_lora_03_b200 import inputs
    from oracle import nf4_oracle as O
    li = inputs.training_linear(i)
    f = lambda x: x[:sample_tokens].float().numpy()  # noqa: E731
    return (li.name, O.nf4_quantize(li.Wt.numpy()), f(li.X), f(li.dY),
            li.L1.float().numpy(), li.L2.float().numpy(), li.s)


def oracle_linear_step(entry) -> float:
    """Seconds of one oracle fwd+bwd of one linear on the sampled tokens, W dequantized first."""
    from oracle import nf4_oracle as O
    _, packed, X, dY, L1, L2, s = entry
    t0 = time.perf_counter()
    Wdq = O.nf4_dequantize(packed)
    O.qlora_linear_fwd(X, Wdq, L1, L2, s)
    O.qlora_linear_bwd(dY, X, Wdq, L1, L2, s)
    return time.perf_counter() - t0


def run_reference(args, rank):
    """The oracle on the host cores: step k is the fwd+bwd of linear k mod 7 of the layer on
    `--cpu-sample-tokens` tokens (its weight dequantized in the step). The layer's throughput
    is the sampled tokens over the sum of the 7 linears' mean step times; ms_per_step is the
    wall time the timed steps actually took."""
    if rank != 0:
        return 0
    from bit_quantized_lora_03_b200 import inputs
    sample = args.cpu_sample_tokens
    n = len(inputs.LLAMA7B_LINEARS)
    prep = {i: oracle_linear_prep(i, sample) for i in sorted({k % n for k in range(args.warmup + args.steps)})}
    for k in range(args.warmup):
        oracle_linear_step(prep[k % n])
    per = [[] for _ in range(n)]
    t_run = time.perf_counter()
    for k in range(args.steps):
        per[k % n].append(oracle_linear_step(prep[k % n]))
    wall = time.perf_counter() - t_run
    names = [nm for nm, _, _ in inputs.LLAMA7B_LINEARS]
    # a linear the timed steps did not reach takes the mean of its shape class
    shape = [(1 if i < 4 else 2 if i < 6 else 3) for i in range(n)]
    mean = [statistics.mean(v) if v else None for v in per]
    for i in range(n):
        if mean[i] is None:
            same = [mean[j] for j in range(n) if shape[j] == shape[i] and mean[j] is not None]
            mean[i] = statistics.mean(same) if same else max(m for m in mean if m is not None)
    layer_s = sum(mean)
    value = sample / layer_s
    desc = (f"oracle fwd+bwd of {sample} of the 4096 tokens, one linear of the layer per step in "
            f"rotation (W dequantized in the step); the layer's time is the sum of the 7 linears' "
            f"mean step times ({layer_s:.2f} s)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * wall / max(1, args.steps), 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens_per_step": sample, "r": 64, "s": 0.25},
            "timed_wall_s": round(wall, 2), "layer_seconds": round(layer_s, 3),
            "linear_step_s": {names[i]: round(mean[i], 3) for i in range(n)},
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cpu_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def oracle_legs():
    """The oracle timed on the host cores beside the secondary configurations, each on a bounded
    sample (stated), with the rate in the GPU leg's unit."""
    from bit_quantized_lora_03_b200 import inputs
    from oracle import nf4_oracle as O
    cores = cpu_threads()
    res = {}
    # configuration 1, in full: quantize, dequantize, forward of 16 tokens
    li = inputs.single_linear_1024()
    t0 = time.perf_counter()
    pk = O.nf4_quantize(li.Wt.numpy())
    Wdq = O.nf4_dequantize(pk)
    O.qlora_linear_fwd(li.X.float().numpy(), Wdq, li.L1.float().numpy(), li.L2.float().numpy(), li.s)
    sec = time.perf_counter() - t0
    res["single_linear_1024"] = {"value": round(sec * 1e6, 1), "unit": "us per quantize+dequantize+fwd",
                                 "cores": cores, "kind": "oracle", "sample": "the whole configuration"}
    # configuration 2: quantize and dequantize of q_proj (16.8 M of the 202.4 M weights)
    _, Wt = next(iter(inputs.llama7b_quant_weights(with_outliers=True)))
    n = Wt.numel()
    t0 = time.perf_counter()
    pk = O.nf4_quantize(Wt.numpy())
    tq = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.nf4_dequantize(pk)
    td = time.perf_counter() - t0
    packed = O.packed_bytes(n)
    res["codec_llama7b_layer"] = {
        "quantize_gbs": round((4 * n + packed) / tq / 1e9, 3),
        "dequantize_gbs": round((packed + 2 * n) / td / 1e9, 3), "unit": "GB/s",
        "cores": cores, "kind": "oracle",
        "sample": f"q_proj alone (16.8 M of the 202.4 M weights): {tq:.1f} s quantize, {td:.1f} s dequantize"}
    # configuration 3: 256 rows of the 4096 x 11008 weight (the scale groups covering them
    # quantized), forward at t = 1 and 16; packed bytes of those rows per second
    name, Wt = inputs.decode_gemv_weights()[0]
    o, h = Wt.shape
    rows = np.arange(0, o, o // 256)[:256]
    Wn = Wt.numpy()
    L1, L2 = (a.float().numpy() for a in inputs.decode_gemv_adapters(h, o, 16))
    out = {}
    for t in (1, 16):
        X = inputs.decode_gemv_activations(h, t).float().numpy()
        t0 = time.perf_counter()
        deq = []
        nbr = h // 64
        flat = Wn.reshape(-1)
        for j in rows:
            g0, g1 = j * nbr // 256, ((j + 1) * nbr - 1) // 256 + 1
            lo, hi = g0 * 256 * 64, min(g1 * 256 * 64, flat.size)
            d = O.nf4_dequantize(O.nf4_quantize(flat[lo:hi].reshape(1, -1))).reshape(-1)
            deq.append(d[j * h - lo:(j + 1) * h - lo])
        Wr = np.stack(deq).astype(np.float64)
        _ = X.astype(np.float64) @ Wr.T + 2.0 * ((X.astype(np.float64) @ L1) @ L2[:, rows])
        sec = time.perf_counter() - t0
        out[f"t{t}"] = round(O.packed_bytes(len(rows) * h) / sec / 1e9, 4)
    res["decode_gemv"] = {"packed_gbs": out, "unit": "GB/s (packed bytes of the sampled rows)",
                          "cores": cores, "kind": "oracle",
                          "sample": f"256 of the 11008 rows of {name} (quantize of their scale groups, "
                                    "dequantize, forward)"}
    # configuration 5: 64 rows of one 8192 x 8192 linear at 2048 tokens, forward and the rows'
    # share of the backward, extrapolated to the 560 linears of the stack
    Wq = inputs.weight_f32(64, 8192, 7).numpy()
    X = inputs.normal_bf16((inputs.STACK65B_TOKENS, 8192), 1.0, inputs._gen(510)).float().numpy()
    dY = inputs.normal_bf16((inputs.STACK65B_TOKENS, 64), 1.0, inputs._gen(520)).float().numpy()
    t0 = time.perf_counter()
    Wr = O.nf4_dequantize(O.nf4_quantize(Wq)).astype(np.float64)
    _ = X.astype(np.float64) @ Wr.T
    _ = dY.astype(np.float64) @ Wr
    sec = time.perf_counter() - t0
    stack_w = inputs.STACK65B_LAYERS * sum(hh * oo for _, hh, oo in inputs.LLAMA65B_LINEARS)
    step_s = sec * stack_w / (64 * 8192)
    res["stack65b"] = {"value": round(inputs.STACK65B_TOKENS / step_s, 6), "unit": UNIT,
                       "cores": cores, "kind": "oracle", "extrapolated": True,
                       "sample": f"64 rows of an 8192 x 8192 linear, 2048 tokens, base product fwd and "
                                 f"bwd ({sec:.1f} s), scaled by weights to the 64.76 G of the stack "
                                 f"(adapter terms left out)"}
    return res


def decode_case(B, dev, t, wi):
    """A short decode run for one capture: the third GEMV launch is the steady state."""
    from bit_quantized_lora_03_b200 import inputs
    name, Wt = inputs.decode_gemv_weights()[wi]
    o, h = Wt.shape
    p = B.nf4_quantize(Wt.to(dev))
    del Wt
    L1, L2 = (a.to(dev) for a in inputs.decode_gemv_adapters(h, o, 16))
    X = inputs.decode_gemv_activations(h, t).to(dev)
    for _ in range(3):
        B.qlora_linear_fwd(X, p, L1, L2, 2.0, want_sT=False)
    torch.cuda.synchronize()
    status = B.last_status()
    print(json.dumps({"case": f"decode {name} o={o} h={h} t={t}", "device_status": status}),
          flush=True)
    return 0 if status == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=900)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--tokens", type=int, default=4096)
    ap.add_argument("--cpu-sample-tokens", type=int, default=32)
    ap.add_argument("--quick", action="store_true", help="skip the secondary legs and the CPU baseline")
    ap.add_argument("--streams", type=int, default=2,
                    help="streams the 7 independent linears of a step are spread over")
    ap.add_argument("--single-linear", type=int, default=None, metavar="I",
                    help="profiling case: only linear I of the layer, fwd+bwd, no extras")
    ap.add_argument("--dropout", type=float, default=0.0, metavar="P",
                    help="with --single-linear: LoRA dropout P on the adapter input")
    ap.add_argument("--gemv-only", action="store_true",
                    help="run only the decode GEMV leg (configuration 3) and print it")
    ap.add_argument("--codec-only", action="store_true",
                    help="only the quantize / dequantize leg (the 7B layer's weights, then one long launch)")
    ap.add_argument("--codebooks-only", action="store_true",
                    help="run only the codebook / scale-format comparison leg and print it")
    ap.add_argument("--dropout-only", action="store_true",
                    help="after the headline, run only the LoRA-dropout leg (no other legs, no CPU baseline)")
    ap.add_argument("--decode-case", type=int, nargs=2, default=None, metavar=("T", "I"),
                    help="profiling case: quantize decode weight I, then three forward calls "
                         "at T tokens")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)

    from bit_quantized_lora_03_b200 import binding as B
    from bit_quantized_lora_03_b200 import build as _build
    _build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks, peak_src = load_peaks()
    props = torch.cuda.get_device_properties(dev)
    l2_bytes = getattr(props, "L2_cache_size", 126 * 2**20)

    if args.decode_case is not None:
        return decode_case(B, dev, *args.decode_case)
    if args.codebooks_only:
        print(json.dumps(codebook_leg(dev)), flush=True)
        return 0
    if args.codec_only:
        print(json.dumps(codec_leg(dev, peaks)), flush=True)
        return 0
    if args.gemv_only:
        with ClockSampler(local) as clk:
            res = gemv_leg(dev, peaks, l2_bytes)
        print(json.dumps({"decode_gemv": res, "clocks": clk.summary(),
                          "device_status": B.last_status()}), flush=True)
        return 0
    t, r, s = args.tokens, 64, 0.25
    if args.single_linear is not None:
        L = Layer(args.single_linear, dev, t, r, s)
        fn = (lambda: L.step_dropout(args.dropout, 1234)) if args.dropout > 0 else L.step
        ms = timed(fn, args.steps, args.warmup, 1, dev)
        print(json.dumps({"case": f"single linear {L.name} h={L.h} o={L.o} t={t} r={r} "
                                  f"dropout={args.dropout}",
                          "ms_per_fwd_bwd": round(ms / args.steps, 4),
                          "tflops": round(step_flops([L]) * args.steps / (ms * 1e-3) / 1e12, 1),
                          "device_status": B.last_status()}), flush=True)
        return 0
    layers = [Layer(i, dev, t, r, s) for i in range(7)]
    names = [L.name for L in layers]
    torch.cuda.synchronize()
    assert B.last_status() == 0

    # headline: device-timed steps with inputs resident in HBM
    with ClockSampler(local) as clk:
        streams = [torch.cuda.Stream(dev) for _ in range(args.streams)] if args.streams > 1 else None
        ms_total = timed(lambda: step_all(layers, world, streams), args.steps, args.warmup, world, dev)
    clocks = clk.summary()
    ms_step = ms_total / args.steps
    value = world * t * args.steps / (ms_total * 1e-3)
    status = B.last_status()

    # per-kernel device time over the same steps (events around each launch)
    with B.KernelProfile() as prof:
        for _ in range(args.steps):
            step_all(layers, world)
    launches_per_step = sum(prof.launches.values()) / args.steps
    gemm_ms = prof.ms["nf4_gemm_kernel<fwd>"] + prof.ms["nf4_gemm_kernel<bwd>"]
    gemm_launches = prof.launches["nf4_gemm_kernel<fwd>"] + prof.launches["nf4_gemm_kernel<bwd>"]
    gemm_flops_step = fused_gemm_flops(layers)
    achieved = gemm_flops_step * args.steps / (gemm_ms * 1e-3) / 1e12
    # a timed region shorter than a second runs below the power cap: the burst peak applies;
    # a seconds-long one settles at the cap: the sustained peak
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    timed_s = ms_total * 1e-3
    peak = burst if timed_s < 1.0 else sustained
    peak_kind = "bf16_tflops (burst)" if timed_s < 1.0 else "bf16_tflops_sustained"
    traffic = ncu_traffic("nf4_gemm_kernel")
    kernel_table = {k: {"ms_per_step": round(v / args.steps, 4),
                        "launches_per_step": prof.launches[k] / args.steps,
                        "share": round(v / max(1e-9, sum(prof.ms.values())), 4)}
                    for k, v in prof.ms.items() if prof.launches[k]}

    # end to end through the C ABI with host buffers
    e2e = None
    if rank == 0 or world > 1:
        hX = [L.X_cpu.pin_memory() for L in layers]
        hdY = [L.dY_cpu.pin_memory() for L in layers]
        hg = [(torch.empty(L.h, r, dtype=torch.float32).pin_memory(),
               torch.empty(r, L.o, dtype=torch.float32).pin_memory()) for L in layers]

        # host->device copies on one stream, device->host on another, the linears on the
        # compute stream: linear i+1's inputs cross the host link while linear i computes,
        # and each linear's adapter gradients go back as soon as they exist
        h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        freed = [torch.cuda.Event() for _ in layers]   # compute is done with L.X, L.dY
        for ev in freed:
            ev.record()

        def e2e_step():
            comp = torch.cuda.current_stream(dev)
            arrived = []
            with torch.cuda.stream(h2d_stream):
                for L, x, dy, fr in zip(layers, hX, hdY, freed):
                    h2d_stream.wait_event(fr)
                    L.X.copy_(x, non_blocking=True)
                    L.dY.copy_(dy, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d_stream)
                    arrived.append(ev)
            for L, ev, fr in zip(layers, arrived, freed):
                comp.wait_event(ev)
                L.step()
                fr.record(comp)
            if world > 1:
                from bit_quantized_lora_03_b200 import dp
                dp.allreduce_adapter_grads([g for L in layers for g in (L.dL1, L.dL2)])
                reduced = torch.cuda.Event()
                reduced.record(comp)
            with torch.cuda.stream(d2h_stream):
                for L, (g1, g2), fr in zip(layers, hg, freed):
                    d2h_stream.wait_event(reduced if world > 1 else fr)
                    g1.copy_(L.dL1, non_blocking=True)
                    g2.copy_(L.dL2, non_blocking=True)
                back = torch.cuda.Event()
                back.record(d2h_stream)
            comp.wait_event(back)   # a step ends when its gradients are on the host
        e2e_steps = max(3, args.steps // 2)
        e_ms = timed(e2e_step, e2e_steps, 1, world, dev)
        h2d = sum(x.numel() * 2 + dy.numel() * 2 for x, dy in zip(hX, hdY))
        d2h = sum(g1.numel() * 4 + g2.numel() * 4 for g1, g2 in hg)
        e2e = {"value": round(world * t * e2e_steps / (e_ms * 1e-3), 1), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(e_ms / e2e_steps, 3)}

    legs = {}
    cpu = None
    if rank == 0 and world == 1 and not args.quick:
        dstreams = [torch.cuda.Stream(dev) for _ in range(args.streams)] if args.streams > 1 else None
        legs["dropout_llama7b_layer"] = dropout_leg(dev, peaks, layers, dstreams, ms_step)
    if rank == 0 and world == 1 and not args.quick and not args.dropout_only:
        del layers
        torch.cuda.empty_cache()
        legs["decode_gemv"] = gemv_leg(dev, peaks, l2_bytes)
        legs["codec_llama7b_layer"] = codec_leg(dev, peaks)
        legs["stack65b"] = stack65b_leg(dev, peaks)
        legs["merge_llama7b_layer"] = merge_leg(dev, peaks)
        legs["codebooks_llama7b_layer"] = codebook_leg(dev)
        legs["adamw_llama7b_adapters"] = adamw_leg(dev, peaks)
        for leg, cb in oracle_legs().items():
            if isinstance(legs.get(leg), dict):
                legs[leg]["cpu_baseline"] = cb
            else:
                legs[leg + "_cpu_baseline"] = cb
        tps, sec, prepared = oracle_sample(args.cpu_sample_tokens)
        cpu = {"value": round(tps, 3), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": (f"fwd+bwd of {args.cpu_sample_tokens} of the 4096 tokens, one linear per "
                          "shape class (q 4096x4096 x4, up 4096x11008 x2, down 11008x4096 x1), "
                          f"incl. per-step W dequant; {sec:.1f} s of CPU work")}
        one = oracle_sample_one_core(args.cpu_sample_tokens, prepared)
        if one is not None:
            cpu["one_core"] = one

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens_per_gpu": t, "global_tokens": world * t,
                       "linears": names,
                       "h": 4096, "ffn": 11008, "r": r, "s": s, "weights": "NF4 blk64 + DQ",
                       "parallelism": f"dp{world}", "streams": args.streams,
                       "l2": "inputs larger than L2: ~1.3 GB of activations and gradients "
                             "touched per step vs 126 MB L2"},
            "step_tflops": round(step_flops_value(t, r) / (ms_step * 1e-3) / 1e12, 1),
            "roofline": {"kernel": "nf4_gemm_kernel (fwd+bwd, fused dequant + LoRA fold)",
                         "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic,
                         "peak_source": f"{peak_src} {peak_kind}: the timed region lasted "
                                        f"{timed_s:.3f} s",
                         "frac_of_burst": round(achieved / burst, 4),
                         "frac_of_sustained": round(achieved / sustained, 4),
                         "algorithmic_flops_per_launch": round(gemm_flops_step / (gemm_launches / args.steps)),
                         "avg_launch_ms": round(gemm_ms / gemm_launches, 4)},
            "kernels": kernel_table,
            "gpu_launches": int(round(launches_per_step * args.steps)),
            "device_status": status,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clocks,
            "legs": legs,
            "gpu": props.name,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def step_flops_value(t, r):
    from bit_quantized_lora_03_b200 import inputs
    return sum(4 * t * h * o + 6 * t * r * (h + o) for _, h, o in inputs.LLAMA7B_LINEARS)


if __name__ == "__main__":
    sys.exit(main())
