#!/usr/bin/env python
"""Benchmark of the W4/W2 weight-only decode path on a Llama-3-8B-shaped stack.

One step = one decode forward through all 32 layers x 7 projections
(q, k, v, o 4096x4096 / 1024x4096; gate, up 14336x4096; down 4096x14336)
for each batch size M in {1, 4, 16}.  Projections that read the same input
run as one linear over their weights concatenated along N, as an inference
engine runs a layer: qkv 6144x4096, o, gate_up 28672x4096, down; 4 bq_linear
calls per layer, 384 per step, replayed from one CUDA graph.  Weights are synthetic fp16 N(0, 0.02) (seed 1000*layer + module),
quantized on the GPU by bq_quantize (INT4 group 128 by default); activations
are bf16 N(0, 1).  The packed stack (3.76 GB at INT4) is far larger than the
126 MB L2, so every pass streams the weights from HBM; no flush is needed.

Printed: ONE JSON line (rank 0).  ``value`` = effective weight GB/s of the
whole job = (packed codes + scales + zeros + x + y bytes of every linear of
the step, over all ranks) / max-over-ranks step time.  Extra fields report
per-M numbers, per-shape numbers, the quantizer over the whole ~7B-weight
stack and on one 8192x49152 matrix (with the fused fake-quantization pass),
the prefill GEMM (tcgen05 path, M = 2048 and 8192 tokens against the
14336x4096, 4096x14336, 49152x8192 and 8192x49152 weights at INT4 and INT2)
in TFLOP/s, the end-to-end host-buffer path, the roofline of the dominant
kernel (the decode GEMV) and the CPU oracle baseline.

Multi-GPU (torchrun): every rank runs its own replica of the stack on its own
GPU with its own inputs (independent batches, no data-path collective);
``scaling`` is "weak".

``--impl reference`` times the CPU oracle (the plain C reference of the same
computation) on a bounded sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_gemm_group_b200 import bq, synth  # noqa: E402

MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
M_SET = (1, 4, 16)
# DRAM bytes (read + write) per algorithmic byte of the decode kernel, from
# one ncu capture of gemv_kernel on the gate_up 28672x4096 INT4 linear at
# M = 1 (63,343,360 bytes read + 155,392 written for 63,373,312 algorithmic
# bytes); the kernel reads every weight byte once, so traffic scales with
# the bytes.
GEMV_DRAM_PER_ALGO_BYTE = (63343360 + 155392) / 63373312
METRIC = "W4/W2 dequant-GEMV weight GB/s (M<=16) & GEMM TFLOP/s (M>=2048) vs roofline"


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def weight_bytes(N, K, bits, group, scale_bytes=4):
    """Algorithmic bytes of one decode linear's weights: codes + scale (fp32, or
    binary16) + u8 zero per group."""
    return N * K * bits // 8 + N * (K // group) * (scale_bytes + 1)


def linear_bytes(N, K, bits, group, M, scale_bytes=4):
    return weight_bytes(N, K, bits, group, scale_bytes) + 2 * M * K + 2 * M * N


def peaks():
    try:
        with open(MEASURED_PEAKS) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if not self.path or not os.path.exists(self.path):
            return out
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if sm:
            busy = [s for s in sm if s > 0.5 * max(sm)] or sm
            out = {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                   "samples": len(sm)}
        return out


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def stack_shapes(layers):
    return [(l, mi, name, N, K) for l in range(layers) for mi, (name, N, K) in enumerate(synth.LLAMA3_8B_LINEARS)]


def fused_shapes(layers):
    """(layer, name, N, K, module indices): the linears of the decode step,
    q/k/v and gate/up each as one linear over their concatenated weights."""
    L = synth.LLAMA3_8B_LINEARS
    return [(l, fname, sum(L[m][1] for m in mods), L[mods[0]][2], mods)
            for l in range(layers) for fname, mods in synth.LLAMA3_8B_FUSED]


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class Stack:
    """The quantized decode stack resident in HBM, plus per-M activations."""

    def __init__(self, layers, bits, group, seed_offset, dist_kind, quant_time=True, scheme="asymmetric"):
        self.layers, self.bits, self.group = layers, bits, group
        self.scheme = scheme
        self.scale_bytes = 2 if scheme == "asymmetric_f16_scale" else 4
        self.shapes = stack_shapes(layers)
        dev = "cuda"
        # fp16 weights for the whole stack (~14 GB at 32 layers) so the
        # quantizer can be timed over all of it, then dropped.
        Ws = []
        for (l, mi, name, N, K) in self.shapes:
            seed = synth.weight_seed(l, mi) + seed_offset
            if dist_kind == "t4":
                Ws.append(synth.student_t4((N, K), 0.02, seed, "f16", dev, outlier_frac=0.001))
            else:
                Ws.append(synth.normal((N, K), 0.02, seed, "f16", dev))
        # fused linears: one packed / scales / zeros buffer each; every module
        # is quantized into its slice (the interleaved layout is 128-row-block
        # major, so stacking whole blocks along N concatenates the buffers)
        self.fused = fused_shapes(layers)
        self.fq = []
        self.q = [None] * len(self.shapes)
        nlin = len(synth.LLAMA3_8B_LINEARS)
        for (l, fname, N, K, mods) in self.fused:
            pk = torch.empty(bq.bq_packed_bytes(N, K, bits), dtype=torch.uint8, device=dev)
            sc = torch.empty(N * (K // group), dtype=torch.float16 if self.scale_bytes == 2 else torch.float32,
                             device=dev)
            ze = torch.empty(N * (K // group), dtype=torch.uint8, device=dev)
            self.fq.append((pk, sc, ze))
            r0 = 0
            for m in mods:
                Nm = synth.LLAMA3_8B_LINEARS[m][1]
                cb, gb = bq.bq_packed_bytes(r0, K, bits), r0 * (K // group)
                ce, ge = bq.bq_packed_bytes(r0 + Nm, K, bits), (r0 + Nm) * (K // group)
                self.q[l * nlin + m] = (pk[cb:ce], sc[gb:ge], ze[gb:ge])
                r0 += Nm
        for W, (l, mi, name, N, K), out in zip(Ws, self.shapes, self.q):
            bq.bq_quantize(W, bits, group, "interleaved", out=out, scheme=scheme)
        torch.cuda.synchronize()
        if bq.bq_device_status() != bq.BQ_OK:
            raise RuntimeError("quantizer reported a device error")
        self.quant = None
        if quant_time:
            self.quant = self._time_quantizer(Ws)
        del Ws
        torch.cuda.empty_cache()

    def _time_quantizer(self, Ws, reps=3):
        """Quantize the whole stack (all ~7B weights) from one CUDA graph."""
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for W, out in zip(Ws, self.q):            # warm
                bq.bq_quantize(W, self.bits, self.group, "interleaved", out=out, stream=s, scheme=self.scheme)
            s.synchronize()
            with torch.cuda.graph(g, stream=s):
                for W, out in zip(Ws, self.q):
                    bq.bq_quantize(W, self.bits, self.group, "interleaved", out=out, stream=s, scheme=self.scheme)
        torch.cuda.current_stream().wait_stream(s)
        g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            times.append(a.elapsed_time(b) / 1e3)
        t = min(times)
        weights = sum(N * K for (_, _, _, N, K) in self.shapes)
        byts = sum(N * K * 2 + weight_bytes(N, K, self.bits, self.group, self.scale_bytes)
                   for (_, _, _, N, K) in self.shapes)
        del g
        return {"weights": weights, "seconds": t, "weights_per_s": weights / t, "GBps": byts / t / 1e9,
                "bytes": byts, "launches": len(self.shapes)}

    def make_graph(self, Ms, xs, ys, stream):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for M in Ms:                                  # warm / lazy init outside capture
                for i, (l, fname, N, K, mods) in enumerate(self.fused):
                    pk, sc, ze = self.fq[i]
                    bq.bq_linear(xs[M][i], pk, sc, ze, N, self.bits, self.group, out=ys[M][i], stream=stream)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for M in Ms:
                    for i, (l, fname, N, K, mods) in enumerate(self.fused):
                        pk, sc, ze = self.fq[i]
                        bq.bq_linear(xs[M][i], pk, sc, ze, N, self.bits, self.group, out=ys[M][i], stream=stream)
        return g

    def step_bytes(self, Ms):
        return sum(linear_bytes(N, K, self.bits, self.group, M, self.scale_bytes)
                   for M in Ms for (_, _, N, K, _) in self.fused)


def time_graph(g, steps, warmup, stream, world, profile=False):
    """Replay `g` warmup + steps times; the steps are timed with CUDA events on
    `stream`.  profile=True brackets the timed replays with cudaProfilerStart/
    Stop so an external profiler started with --profile-from-start off records
    exactly the timed launches."""
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if profile:
        torch.cuda.cudart().cudaProfilerStart()
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(steps):
            g.replay()
        b.record(stream)
    b.synchronize()
    if profile:
        torch.cuda.cudart().cudaProfilerStop()
    torch.cuda.synchronize()
    barrier(world)
    return a.elapsed_time(b) / 1e3


def per_shape_numbers(stack, M, stream, reps=20):
    """Each distinct shape alone: one graph of 8 rotating weight copies x reps."""
    res = {}
    seen = {}
    for i, (l, name, N, K, mods) in enumerate(stack.fused):
        if name not in seen:
            seen[name] = i
    for name, i in seen.items():
        (_, _, N, K, _) = stack.fused[i]
        idx = [j for j, s in enumerate(stack.fused) if s[1] == name][:8]
        x = synth.activations(M, K, seed=5, device="cuda")
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    for j in idx:
                        pk, sc, ze = stack.fq[j]
                        bq.bq_linear(x, pk, sc, ze, N, stack.bits, stack.group, out=y, stream=stream)
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        t = a.elapsed_time(b) / 1e3 / (reps * len(idx))
        byts = linear_bytes(N, K, stack.bits, stack.group, M)
        res[f"{name} {N}x{K}"] = {"us": round(t * 1e6, 2), "GBps": round(byts / t / 1e9, 1)}
        del g
    return res


def grad_numbers(stack, Ms, hbm, reps=5):
    """Input gradient dx = dy . dequant(W) (bq_linear_grad_input) over the
    whole decode stack -- every fused projection of every layer, one CUDA
    graph per token count; dy bf16 N(0,1).  GB/s of algorithmic bytes (packed
    weights + metadata + dy + dx), CUDA-event median."""
    res = {}
    for M in Ms:
        dys, dxs = {}, {}
        for (_, _, N, K, _) in stack.fused:
            if (N, K) not in dys:
                dys[(N, K)] = synth.activations(M, N, seed=9, device="cuda")
                dxs[(N, K)] = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for j, (_, _, N, K, _) in enumerate(stack.fused):
                    pk, sc, ze = stack.fq[j]
                    bq.bq_linear_grad_input(dys[(N, K)], pk, sc, ze, K, stack.bits, stack.group, out=dxs[(N, K)],
                                            stream=s)
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        t = statistics.median(ts)
        byts = sum(linear_bytes(N, K, stack.bits, stack.group, M) for (_, _, N, K, _) in stack.fused)
        res[str(M)] = {"ms": round(t * 1e3, 4), "GBps": round(byts / t / 1e9, 1),
                       "frac_of_measured_hbm": round(byts / t / 1e9 / hbm, 4), "launches": len(stack.fused)}
        del g
    if bq.bq_device_status() != bq.BQ_OK:
        raise RuntimeError("input-gradient kernel reported a device error")
    return res


def mixed_numbers(layers, Ms, hbm, reps=5):
    """Decode stack with per-128-row-block widths (4 bits -> group 128, 2 bits
    -> group 64): Layer-mix (one width per layer, 8 of 32 layers at 4 bits)
    and Channel-mix (25% of the blocks of every matrix at 4 bits).  Weights
    fp16 N(0, 0.02), one fused matrix per linear; x bf16 N(0, 1).  GB/s of
    algorithmic bytes (each block's codes + metadata, x, y) over one CUDA
    graph per token count, CUDA-event median."""
    res = {}
    lmap = synth.layer_mix_map(layers)
    for kind in ("layer_mix", "channel_mix"):
        mods = []
        for i, (l, _, N, K, _) in enumerate(fused_shapes(layers)):
            W = synth.normal((N, K), 0.02, seed=500000 + i, dtype="f16", device="cuda")
            if kind == "layer_mix":
                bmap = [lmap[l]] * (N // 128)
            else:
                bmap = synth.channel_mix_map(N, seed=600000 + i).tolist()
            pk, sc, ze, bm = bq.bq_quantize_mixed(W, bmap, "interleaved")
            del W
            wb = sum(weight_bytes(128, K, b, 128 if b == 4 else 64) for b in bmap)
            mods.append((N, K, pk, sc, ze, bm, wb, 128 * K * bmap.count(4)))
        torch.cuda.synchronize()
        if bq.bq_device_status() != bq.BQ_OK:
            raise RuntimeError("mixed quantizer reported a device error")
        weights4 = sum(m[7] for m in mods)
        weights = sum(N * K for (N, K, *_rest) in mods)
        per_m = {}
        for M in Ms:
            xs = {K: synth.activations(M, K, seed=7, device="cuda") for K in {m[1] for m in mods}}
            ys = {N: torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for N in {m[0] for m in mods}}
            s = torch.cuda.Stream()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    for (N, K, pk, sc, ze, bm, *_rest) in mods:
                        bq.bq_linear(xs[K], pk, sc, ze, N, bit_map_dev=bm, out=ys[N], stream=s)
            g.replay()
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                g.replay()
                b.record()
                b.synchronize()
                ts.append(a.elapsed_time(b) / 1e3)
            t = statistics.median(ts)
            byts = sum(m[6] + 2 * M * m[1] + 2 * M * m[0] for m in mods)
            per_m[str(M)] = {"ms": round(t * 1e3, 4), "GBps": round(byts / t / 1e9, 1),
                             "frac_of_measured_hbm": round(byts / t / 1e9 / hbm, 4)}
            del g
            # the input gradient dx = dy . dequant(W) of the same linears
            dys = {N: synth.activations(M, N, seed=8, device="cuda") for N in {m[0] for m in mods}}
            dxs = {K: torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for K in {m[1] for m in mods}}
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s):
                for (N, K, pk, sc, ze, bm, *_rest) in mods[:4]:   # lazy init outside the capture
                    bq.bq_linear_grad_input(dys[N], pk, sc, ze, K, out=dxs[K], stream=s, bit_map_dev=bm)
                s.synchronize()
                with torch.cuda.graph(g, stream=s):
                    for (N, K, pk, sc, ze, bm, *_rest) in mods:
                        bq.bq_linear_grad_input(dys[N], pk, sc, ze, K, out=dxs[K], stream=s, bit_map_dev=bm)
            g.replay()
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                g.replay()
                b.record()
                b.synchronize()
                ts.append(a.elapsed_time(b) / 1e3)
            t = statistics.median(ts)
            per_m[str(M)]["grad_input"] = {"ms": round(t * 1e3, 4), "GBps": round(byts / t / 1e9, 1),
                                           "frac_of_measured_hbm": round(byts / t / 1e9 / hbm, 4)}
            del g
        if bq.bq_device_status() != bq.BQ_OK:
            raise RuntimeError("mixed linear reported a device error")
        res[kind] = {"bpw_codes": round((4 * weights4 + 2 * (weights - weights4)) / weights, 4), "launches": len(mods),
                     "per_M": per_m}
        del mods
        torch.cuda.empty_cache()
    return res


def stack_per_m(stack, Ms, hbm, steps, world):
    """Decode numbers of one stack: one CUDA graph per token count."""
    xs = {M: [synth.activations(M, K, seed=20000 * M + i, device="cuda")
              for i, (_, _, N, K, _) in enumerate(stack.fused)] for M in Ms}
    ys = {M: [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for (_, _, N, K, _) in stack.fused]
          for M in Ms}
    stream = torch.cuda.Stream()
    per_m = {}
    for M in Ms:
        g = stack.make_graph((M,), xs, ys, stream)
        tm = max_over_ranks(time_graph(g, steps, 1, stream, world) / steps, world)
        bm = stack.step_bytes((M,))
        per_m[str(M)] = {"ms": round(tm * 1e3, 4), "GBps": round(bm / tm / 1e9, 1),
                         "frac_of_measured_hbm": round(bm / tm / 1e9 / hbm, 4), "tokens_per_s": round(M / tm, 1)}
        del g
    return per_m


def e2e_numbers(stack, Ms, steps, warmup, world):
    """Same metric through the C ABI with host buffers: every step copies all
    activations from pinned host memory to the device and all outputs back.
    The copies are pipelined with the compute: the inputs of the next batch
    size go up while the current one computes, and its outputs come down
    while the next computes (separate copy streams, events between them)."""
    xs_h, ys_h, xs_d, ys_d = {}, {}, {}, {}
    h2d = d2h = 0
    for M in Ms:
        tot_x = sum(M * K for (_, _, N, K, _) in stack.fused)
        tot_y = sum(M * N for (_, _, N, K, _) in stack.fused)
        xs_h[M] = torch.empty(tot_x, dtype=torch.bfloat16, pin_memory=True)
        xs_h[M].copy_(synth.normal((tot_x,), 1.0, seed=900 + M, dtype="bf16"))
        ys_h[M] = torch.empty(tot_y, dtype=torch.bfloat16, pin_memory=True)
        xs_d[M] = torch.empty(tot_x, dtype=torch.bfloat16, device="cuda")
        ys_d[M] = torch.empty(tot_y, dtype=torch.bfloat16, device="cuda")
        h2d += tot_x * 2
        d2h += tot_y * 2
    comp, up, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    x_ready = {M: torch.cuda.Event() for M in Ms}     # inputs on the device
    x_free = {M: torch.cuda.Event() for M in Ms}      # compute done reading them
    y_ready = {M: torch.cuda.Event() for M in Ms}     # outputs written
    y_free = {M: torch.cuda.Event() for M in Ms}      # outputs copied down
    for M in Ms:
        x_free[M].record(comp)
        y_free[M].record(down)

    def one_step():
        for M in Ms:
            with torch.cuda.stream(up):
                up.wait_event(x_free[M])
                xs_d[M].copy_(xs_h[M], non_blocking=True)
                x_ready[M].record(up)
        for M in Ms:
            with torch.cuda.stream(comp):
                comp.wait_event(x_ready[M])
                comp.wait_event(y_free[M])
                ox = oy = 0
                for i, (l, fname, N, K, mods) in enumerate(stack.fused):
                    pk, sc, ze = stack.fq[i]
                    bq.bq_linear(xs_d[M][ox:ox + M * K].view(M, K), pk, sc, ze, N, stack.bits, stack.group,
                                 out=ys_d[M][oy:oy + M * N].view(M, N), stream=comp)
                    ox += M * K
                    oy += M * N
                x_free[M].record(comp)
                y_ready[M].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(y_ready[M])
                ys_h[M].copy_(ys_d[M], non_blocking=True)
                y_free[M].record(down)

    for _ in range(warmup):
        one_step()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(up)
    for _ in range(steps):
        one_step()
    for M in Ms:
        up.wait_event(y_free[M])       # the last outputs are on the host
    b.record(up)
    b.synchronize()
    barrier(world)
    t = a.elapsed_time(b) / 1e3 / steps
    return t, h2d, d2h


def quant_shape_numbers(hbm, reps=10):
    """Quantizer and fused fake-quantization on one 8192x49152 fp16 matrix
    (N(0, 0.02)): GB/s of algorithmic bytes (read 2 B per weight; write
    codes + scales + zeros, or 2 B per weight for the fake-quantized output)."""
    N, K = 8192, 49152
    W = synth.normal((N, K), 0.02, seed=5, dtype="f16", device="cuda")
    res = {}

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        return statistics.median(ts)

    for bits, group in ((4, 128), (2, 64)):
        out = bq.bq_quantize(W, bits, group, "interleaved")
        t = timed(lambda: bq.bq_quantize(W, bits, group, "interleaved", out=out))
        byts = N * K * 2 + weight_bytes(N, K, bits, group)
        res[f"quantize {N}x{K} INT{bits} g{group}"] = {"us": round(t * 1e6, 1), "GBps": round(byts / t / 1e9, 1),
                                                       "frac_of_measured_hbm": round(byts / t / 1e9 / hbm, 4)}
        del out
    out = bq.bq_quantize(W, 4, 128, "interleaved", scheme="symmetric")
    t = timed(lambda: bq.bq_quantize(W, 4, 128, "interleaved", out=out, scheme="symmetric"))
    byts = N * K * 2 + weight_bytes(N, K, 4, 128)
    res[f"quantize_symmetric {N}x{K} INT4 g128"] = {"us": round(t * 1e6, 1), "GBps": round(byts / t / 1e9, 1),
                                                   "frac_of_measured_hbm": round(byts / t / 1e9 / hbm, 4)}
    del out
    out = bq.bq_quantize(W, 2, 64, "interleaved", scheme="asymmetric_f16_scale")
    t = timed(lambda: bq.bq_quantize(W, 2, 64, "interleaved", out=out, scheme="asymmetric_f16_scale"))
    byts = N * K * 2 + weight_bytes(N, K, 2, 64, scale_bytes=2)
    res[f"quantize_f16_scales {N}x{K} INT2 g64"] = {"us": round(t * 1e6, 1), "GBps": round(byts / t / 1e9, 1),
                                                   "frac_of_measured_hbm": round(byts / t / 1e9 / hbm, 4)}
    del out
    fq = torch.empty_like(W)
    t = timed(lambda: bq.bq_fake_quantize(W, 4, 128, out=fq))
    byts = N * K * 4
    res[f"fake_quantize {N}x{K} INT4 g128 fp16->fp16"] = {"us": round(t * 1e6, 1), "GBps": round(byts / t / 1e9, 1),
                                                          "frac_of_measured_hbm": round(byts / t / 1e9 / hbm, 4)}
    del W, fq
    torch.cuda.empty_cache()
    if bq.bq_device_status() != bq.BQ_OK:
        raise RuntimeError("quantizer reported a device error")
    return res


GEMM_SHAPES = ((14336, 4096), (4096, 14336), (49152, 8192), (8192, 49152))
GEMM_M = (2048, 4096, 8192)


def medium_m_numbers(reps=20):
    """Medium token counts (the prefill of short prompts, batched decode):
    bq_linear at M = 32 (two 16-token decode passes) and M = 64 .. 256 (the
    tensor-core kernel, split over K through bq_linear_ws's workspace where
    the plan splits), INT4 g128 on Llama-3-8B shapes, one CUDA graph of 8
    calls per point, CUDA-event median; TFLOP/s = 2 M N K / time."""
    res = {}
    s = torch.cuda.Stream()
    for (N, K) in ((4096, 4096), (6144, 4096), (28672, 4096), (4096, 14336)):
        W = synth.normal((N, K), 0.02, seed=N + 3 * K, dtype="f16", device="cuda")
        pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
        del W
        for M in (32, 64, 128, 256):
            x = synth.activations(M, K, seed=M + 1, device="cuda")
            y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            wsb = bq.bq_linear_workspace_bytes(M, N, K, 4)
            ws = torch.empty(wsb, dtype=torch.uint8, device="cuda") if wsb else None
            with torch.cuda.stream(s):
                bq.bq_linear(x, pk, sc, ze, N, 4, 128, out=y, stream=s, workspace=ws)
                s.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=s):
                    for _ in range(8):
                        bq.bq_linear(x, pk, sc, ze, N, 4, 128, out=y, stream=s, workspace=ws)
            with torch.cuda.stream(s):
                g.replay()
            s.synchronize()
            ts = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(s):
                    a.record(s)
                    g.replay()
                    b.record(s)
                b.synchronize()
                ts.append(a.elapsed_time(b) / 1e3 / 8)
            t = statistics.median(ts)
            path = "decode passes" if M < 64 else (f"tensor cores, split-K ({wsb // 1024} KB workspace)" if wsb
                                                   else "tensor cores")
            res[f"{N}x{K} M{M}"] = {"us": round(t * 1e6, 1), "TFLOPs": round(2.0 * M * N * K / t / 1e12, 1),
                                    "path": path}
            del g, x, y, ws
        del pk, sc, ze
        torch.cuda.empty_cache()
    if bq.bq_device_status() != bq.BQ_OK:
        raise RuntimeError("linear reported a device error")
    return res


def gemm_numbers(Ms, bf16, bf16_sus, reps=10):
    """Prefill weight-only GEMM (tcgen05 path of bq_linear) at the prefill
    shapes: bf16 x N(0,1) [M, K] against INT4 g128 / INT2 g64 weights
    N(0, 0.015).  TFLOP/s = 2 M N K / CUDA-event time per call (median)."""
    res = {}
    for (N, K) in GEMM_SHAPES:
        W = synth.normal((N, K), 0.015, seed=N + K, dtype="f16", device="cuda")
        for bits, group in ((4, 128), (2, 64)):
            pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
            for M in Ms:
                x = synth.activations(M, K, seed=M, device="cuda")
                y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
                for _ in range(3):
                    bq.bq_linear(x, pk, sc, ze, N, bits, group, out=y)
                torch.cuda.synchronize()
                ts = []
                for _ in range(reps):
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    bq.bq_linear(x, pk, sc, ze, N, bits, group, out=y)
                    b.record()
                    b.synchronize()
                    ts.append(a.elapsed_time(b) / 1e3)
                t = statistics.median(ts)
                tf = 2.0 * M * N * K / t / 1e12
                res[f"{N}x{K} INT{bits} M{M}"] = {"us": round(t * 1e6, 1), "TFLOPs": round(tf, 1),
                                                  "frac_of_measured_bf16_burst": round(tf / bf16, 4),
                                                  "frac_of_measured_bf16_sustained": round(tf / bf16_sus, 4)}
                del x, y
            del pk, sc, ze
        del W
        torch.cuda.empty_cache()
    # Channel-mix (25% of the 128-row blocks at 4 bits, the rest at 2 bits)
    # through the same tensor-core path
    N, K = 14336, 4096
    W = synth.normal((N, K), 0.015, seed=N + K, dtype="f16", device="cuda")
    bmap = synth.channel_mix_map(N, seed=77).tolist()
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bmap, "interleaved")
    del W
    for M in Ms[:1]:
        x = synth.activations(M, K, seed=M, device="cuda")
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            bq.bq_linear(x, pk, sc, ze, N, bit_map_dev=bm, out=y)
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            bq.bq_linear(x, pk, sc, ze, N, bit_map_dev=bm, out=y)
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        t = statistics.median(ts)
        tf = 2.0 * M * N * K / t / 1e12
        res[f"{N}x{K} Channel-mix 2.5 bpw M{M}"] = {"us": round(t * 1e6, 1), "TFLOPs": round(tf, 1),
                                                    "frac_of_measured_bf16_burst": round(tf / bf16, 4),
                                                    "frac_of_measured_bf16_sustained": round(tf / bf16_sus, 4)}
    del pk, sc, ze, bm
    torch.cuda.empty_cache()
    if bq.bq_device_status() != bq.BQ_OK:
        raise RuntimeError("GEMM reported a device error")
    return res


def split_numbers(layers, bits, group, Ms, steps, world, rank, hbm):
    """The decode stack split over the ranks by output channels (not measured
    on more than one GPU here): each rank quantizes and keeps whole 128-row
    blocks of every fused linear (shard.block_ranges), computes its rows of y,
    and one NCCL all-gather per linear assembles y on every rank.  Eager
    launches, timed with CUDA events over whole steps, max over ranks; value
    is the whole stack's bytes (all ranks together) per step time.  With one
    rank the gather is skipped."""
    from quantized_gemm_group_b200 import shard
    L = synth.LLAMA3_8B_LINEARS
    fused = fused_shapes(layers)
    lins = []
    for (l, fname, N, K, mods) in fused:
        parts = [synth.normal((L[m][1], K), 0.02, synth.weight_seed(l, m), "f16", "cuda") for m in mods]
        W = torch.cat(parts) if len(parts) > 1 else parts[0]
        lins.append(shard.ShardedLinear(W, bits, group, rank, world))
        del W, parts
    torch.cuda.synchronize()
    if bq.bq_device_status() != bq.BQ_OK:
        raise RuntimeError("quantizer reported a device error")
    xs = {M: [synth.activations(M, K, seed=20000 * M + i, device="cuda") for i, (_, _, N, K, _) in enumerate(fused)]
          for M in Ms}

    def step(M):
        for sl, x in zip(lins, xs[M]):
            y = sl.local(x)
            if world > 1:
                shard.gather_rows(y, sl.ranges, rank)

    res = {}
    for M in Ms:
        for _ in range(2):
            step(M)
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            step(M)
        b.record()
        b.synchronize()
        t = max_over_ranks(a.elapsed_time(b) / 1e3 / steps, world)
        byts = sum(linear_bytes(N, K, bits, group, M) for (_, _, N, K, _) in fused)
        res[str(M)] = {"ms": round(t * 1e3, 4), "GBps": round(byts / t / 1e9, 1),
                       "frac_of_measured_hbm_per_gpu": round(byts / t / 1e9 / hbm / world, 4)}
    if bq.bq_device_status() != bq.BQ_OK:
        raise RuntimeError("device error in the split stack")
    del lins
    torch.cuda.empty_cache()
    return {"per_M": res, "ranks": world, "collective": "NCCL all_gather of y per linear" if world > 1 else "none",
            "launches": "eager", "measured_on_hardware": "1 GPU only" if world == 1 else f"{world} GPUs"}


def workload_config(args):
    """The workload both arms report (the reference arm times a bounded sample of it)."""
    bits = args.bits
    group = 128 if bits == 4 else 64
    return {"workload": f"Llama-3-8B-shaped decode stack, {args.layers} layers x 7 projections "
                        f"(q/k/v and gate/up fused along N: 4 linears per layer), "
                        f"INT{bits} g{group} weight-only, M in {{1,4,16}} per step",
            "layers": args.layers, "bits": bits, "group": group, "M": list(M_SET)}


def run_gpu(args, world, rank, local):
    hbm, bf16, bf16_sus, peak_kind = peaks()
    bits, group = args.bits, (128 if args.bits == 4 else 64)
    dist_kind = "t4" if args.bits == 2 else "normal"
    stack = Stack(args.layers, bits, group, seed_offset=rank * 100000, dist_kind=dist_kind,
                  quant_time=not args.no_quant)
    torch.cuda.synchronize()
    bq.bq_set_option(bq.BQ_OPT_LINEAR_OVERLAP, args.overlap)
    Ms = M_SET
    xs = {M: [synth.activations(M, K, seed=10000 * M + i + rank * 7, device="cuda")
              for i, (_, _, N, K, _) in enumerate(stack.fused)] for M in Ms}
    ys = {M: [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for (_, _, N, K, _) in stack.fused]
          for M in Ms}
    stream = torch.cuda.Stream()
    g = stack.make_graph(Ms, xs, ys, stream)
    torch.cuda.synchronize()

    with ClockSampler(local) as clk:
        t_total = time_graph(g, args.steps, args.warmup, stream, world, profile=True)
    t_step = max_over_ranks(t_total / args.steps, world)
    clocks = clk.summary()

    # per-M graphs (same kernels) for the breakdown
    per_m = {}
    for M in Ms:
        gm = stack.make_graph((M,), xs, ys, stream)
        tm = time_graph(gm, max(2, args.steps), 1, stream, world) / max(2, args.steps)
        tm = max_over_ranks(tm, world)
        bm = stack.step_bytes((M,))
        per_m[str(M)] = {"ms": round(tm * 1e3, 4), "GBps": round(bm / tm / 1e9, 1),
                         "frac_of_measured_hbm": round(bm / tm / 1e9 / hbm, 4),
                         "tokens_per_s": round(M / tm, 1)}
        del gm
    shapes = {str(M): per_shape_numbers(stack, M, stream) for M in Ms} if not args.quick else {}

    step_bytes = stack.step_bytes(Ms)
    value = world * step_bytes / t_step / 1e9
    launches_per_step = len(Ms) * len(stack.fused)
    packed_gb = sum(weight_bytes(N, K, bits, group) for (_, _, N, K, _) in stack.fused) / 1e9

    # end to end through the C ABI with host buffers
    t_e2e, h2d, d2h = e2e_numbers(stack, Ms, max(1, args.steps // 2), 2, world)
    t_e2e = max_over_ranks(t_e2e, world)

    achieved = step_bytes / t_step / 1e9   # per-GPU: the GEMV is the only kernel in the step
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4),
                "traffic": round(GEMV_DRAM_PER_ALGO_BYTE * step_bytes / launches_per_step) if bits == 4 else None,
                "traffic_note": "bytes per launch: ncu DRAM bytes per algorithmic byte of one capture of the "
                                "kernel (gate_up 28672x4096, M = 1) x this step's algorithmic bytes per launch",
                "kernel": "gemv_kernel (decode dequant-GEMV, mma.sync bf16)",
                "peak_kind": peak_kind + " (copy burst)",
                "frac_of_nominal_8TBps": round(achieved / 8000.0, 4),
                "bytes_per_launch_avg": round(step_bytes / launches_per_step),
                "us_per_launch_avg": round(t_step / launches_per_step * 1e6, 3)}

    def quant_summary(qz):
        return {"weights": qz["weights"], "ms": round(qz["seconds"] * 1e3, 3),
                "weights_per_s": round(qz["weights_per_s"], 1), "GBps": round(qz["GBps"], 1),
                "frac_of_measured_hbm": round(qz["GBps"] / hbm, 4), "launches": qz["launches"]}

    extra = {"per_M": per_m, "per_shape": shapes, "quantizer_stack": None}
    if not args.no_grad:
        extra["grad_input_stack"] = grad_numbers(stack, Ms, hbm)
    if not args.no_gemm:
        del g
    if stack.quant:
        extra["quantizer_stack"] = quant_summary(stack.quant)
    if not args.no_other_width:
        # the other width's stack (INT2 g64 on heavy-tailed weights with
        # outlier columns, or INT4 g128 on N(0, 0.02)): quantizer over all of
        # its weights and the decode numbers per token count
        obits = 2 if bits == 4 else 4
        del stack
        torch.cuda.empty_cache()
        other = Stack(args.layers, obits, 128 if obits == 4 else 64, seed_offset=rank * 100000 + 7,
                      dist_kind="t4" if obits == 2 else "normal", quant_time=not args.no_quant)
        extra[f"int{obits}_stack"] = {
            "weights": "fp16 Student-t4 std 0.02 + 0.1% x10 outlier cols" if obits == 2 else "fp16 N(0,0.02)",
            "group": 128 if obits == 4 else 64, "per_M": stack_per_m(other, Ms, hbm, max(2, args.steps), world),
            "quantizer_stack": quant_summary(other.quant) if other.quant else None}
        del other
        torch.cuda.empty_cache()
    if not args.no_f16_scale:
        # the INT2 g64 stack again with binary16 group scales (3 instead of 5
        # metadata bytes per group): quantizer and decode numbers
        f16s = Stack(args.layers, 2, 64, seed_offset=rank * 100000 + 7, dist_kind="t4",
                     quant_time=not args.no_quant, scheme="asymmetric_f16_scale")
        extra["int2_stack_f16_scales"] = {
            "weights": "fp16 Student-t4 std 0.02 + 0.1% x10 outlier cols", "group": 64,
            "bytes_per_weight": round(0.25 + 3 / 64, 5),
            "per_M": stack_per_m(f16s, Ms, hbm, max(2, args.steps), world),
            "quantizer_stack": quant_summary(f16s.quant) if f16s.quant else None}
        del f16s
        torch.cuda.empty_cache()
    if not args.no_mixed:
        extra["mixed_stack"] = mixed_numbers(args.layers, (1, 16), hbm)
    if args.split:
        extra["split_stack"] = split_numbers(args.layers, bits, group, Ms, max(2, args.steps), world, rank, hbm)
    if not args.no_quant:
        extra["quantizer_8192x49152"] = quant_shape_numbers(hbm)
    if not args.no_gemm:
        extra["prefill_gemm"] = gemm_numbers(GEMM_M if not args.quick else (2048,), bf16, bf16_sus or bf16)
        extra["medium_m"] = medium_m_numbers()
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_step * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": f"bf16 x int{bits} -> fp32 acc", "data": "synthetic",
        "config": {**workload_config(args),
                   "weights": "fp16 N(0,0.02)" if bits == 4 else "fp16 Student-t4 std 0.02 + 0.1% x10 outlier cols",
                   "activations": "bf16 N(0,1)", "l2": "inputs larger than L2 (packed stack %.2f GB)" % packed_gb,
                   "graph": "one CUDA graph per step", "overlap": args.overlap,
                   "parallelism": f"replicas x{world} (independent batches)"},
        "roofline": roofline,
        "clocks": clocks,
        "e2e": {"value": round(world * step_bytes / t_e2e / 1e9, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(t_e2e * 1e3, 4)},
        "gpu_launches": launches_per_step * args.steps,
        "extra": extra,
    }
    return out


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def oracle_prepare(threads: int, layers_sample: int = 1, bits=4):
    """Quantize (with the oracle) the first `layers_sample` layers' linears of
    the stack on the host, q/k/v and gate/up each sharing their input."""
    from oracle import oracle as O  # test infrastructure, CPU baseline only
    group = 128 if bits == 4 else 64
    prep = []
    for (l, fname, N, K, mods) in fused_shapes(layers_sample):
        quant = []
        for m in mods:
            Nm = synth.LLAMA3_8B_LINEARS[m][1]
            W = synth.normal((Nm, K), 0.02, synth.weight_seed(l, m), "f16", "cpu")
            quant.append(O.quantize(synth.bits16(W), "f16", bits, group, threads=threads))
        prep.append((N, K, mods, quant))
    return prep, bits, group


def oracle_sample(threads: int, prep, Ms=M_SET):
    """Time the CPU oracle's linear layer over prepared linears at every M of
    the step: (GB/s of weight traffic, seconds, bytes)."""
    from oracle import oracle as O  # test infrastructure, CPU baseline only
    lins, bits, group = prep
    total_bytes = 0
    t_lin = 0.0
    for (N, K, mods, quant) in lins:
        for M in Ms:
            x = O.decode_f64(synth.bits16(synth.activations(M, K, seed=M + mods[0], device="cpu")), "bf16")
            t0 = time.perf_counter()
            for codes, scales, zeros in quant:
                O.linear_f64(x, codes, scales, zeros, group, threads=threads)
            t_lin += time.perf_counter() - t0
            total_bytes += linear_bytes(N, K, bits, group, M)
    return total_bytes / t_lin / 1e9, t_lin, total_bytes


def parity_sample(O, W, xt, y_ref, bits, group):
    """The baseline's own oracle product (256 tokens `xt` x the first layer's
    q weight `W`, both host tensors) against the library's on the GPU: the
    decode kernel on the first token and the tensor-core kernel on all 256.
    Per-token relative L2 error (the 2e-3 tolerance metric) and, for context,
    the element-wise max of |y - y_ref| / max|y_ref|, both maxed over tokens.
    Plain launches: the linear reads weights the quantizer has just written."""
    yr = O.bf16_bits_to_f64(O.to_bf16_bits(y_ref))
    mode = bq.bq_get_option(bq.BQ_OPT_LINEAR_OVERLAP)
    bq.bq_set_option(bq.BQ_OPT_LINEAR_OVERLAP, 0)
    pk, sc, ze = bq.bq_quantize(W.to("cuda"), bits, group, "interleaved")
    x = xt.to("cuda")
    out = {}
    for name, xs, ref in (("decode_M1", x[:1], yr[:1]), ("prefill_M256", x, yr)):
        y = bq.bq_linear(xs, pk, sc, ze, W.shape[0], bits, group).double().cpu().numpy()
        l2 = float(np.max(np.linalg.norm(y - ref, axis=1) / np.linalg.norm(ref, axis=1)))
        elem = float(np.max(np.max(np.abs(y - ref), axis=1) / np.max(np.abs(ref), axis=1)))
        out[name] = {"rel_l2_max_over_tokens": float(f"{l2:.3e}"), "elementwise_max_rel": float(f"{elem:.3e}")}
    assert bq.bq_device_status() == bq.BQ_OK
    bq.bq_set_option(bq.BQ_OPT_LINEAR_OVERLAP, mode)
    out["shape"] = f"{W.shape[0]}x{W.shape[1]} INT{bits} g{group}"
    return out


def cpu_baseline(args):
    """The CPU oracle as it stands, on bounded samples of the workloads (about
    half a minute of CPU work): the decode linear on all host cores (the
    headline `value`) and on one core, the quantizer on all cores and on one,
    and the prefill product on 256 tokens, extrapolated per multiply-add to
    the largest prefill shape."""
    from oracle import oracle as O  # test infrastructure, CPU baseline only
    threads = os.cpu_count() or 1
    bits, group = args.bits, (128 if args.bits == 4 else 64)
    prep = oracle_prepare(threads, args.oracle_layers, bits)
    gbps, secs, byts = oracle_sample(threads, prep)
    prep1 = (prep[0][:4], prep[1], prep[2])
    gbps1, secs1, byts1 = oracle_sample(1, prep1, Ms=(1,))
    del prep, prep1
    # quantizer: the first layer's seven weight matrices
    Ws = [synth.normal((N, K), 0.02, synth.weight_seed(0, m), "f16", "cpu")
          for m, (_, N, K) in enumerate(synth.LLAMA3_8B_LINEARS)]
    nweights = sum(W.numel() for W in Ws)
    t0 = time.perf_counter()
    for W in Ws:
        O.quantize(synth.bits16(W), "f16", bits, group, threads=threads)
    tq = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.quantize(synth.bits16(Ws[0]), "f16", bits, group, threads=1)
    tq1 = time.perf_counter() - t0
    qbytes = nweights * 2 + sum(weight_bytes(W.shape[0], W.shape[1], bits, group) for W in Ws)
    # prefill: 256 tokens against a 4096x4096 weight, per multiply-add
    W = Ws[0]
    c, sc, ze = O.quantize(synth.bits16(W), "f16", bits, group, threads=threads)
    xt = synth.activations(256, W.shape[1], seed=3, device="cpu")
    x = O.decode_f64(synth.bits16(xt), "bf16")
    t0 = time.perf_counter()
    y_ref = O.linear_f64(x, c, sc, ze, group, threads=threads)
    tg = time.perf_counter() - t0
    macs_per_s = 256 * W.shape[0] * W.shape[1] / tg
    big = 8192 * 49152 * 8192
    parity = parity_sample(O, W, xt, y_ref, bits, group)
    return {"value": round(gbps, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"first {args.oracle_layers} layer(s) x 4 linears (qkv, o, gate_up, down) x M in {{1,4,16}} "
                      f"({byts / 1e6:.1f} MB of weight traffic, {secs:.1f} s); fp64 linear over dequantized weights",
            "single_core": {"value": round(gbps1, 4), "unit": "GB/s", "cores": 1,
                            "sample": f"first layer's 4 linears at M = 1 ({byts1 / 1e6:.1f} MB, {secs1:.1f} s)"},
            "quantizer": {"weights_per_s": round(nweights / tq, 1), "GBps": round(qbytes / tq / 1e9, 4),
                          "cores": threads, "weights_per_s_single_core": round(Ws[0].numel() / tq1, 1),
                          "sample": f"first layer's 7 weight matrices ({nweights / 1e6:.0f} M weights, {tq:.1f} s; "
                                    f"one core: q 4096x4096, {tq1:.1f} s), INT{bits} g{group}"},
            "parity_sample": parity,
            "prefill_extrapolated": {"TFLOPs": round(2 * macs_per_s / 1e12, 6), "cores": threads,
                                     "seconds_8192x49152_M8192": round(big / macs_per_s, 1),
                                     "sample": f"256 tokens x 4096x4096 fp64 ({tg:.1f} s), extrapolated per "
                                               "multiply-add (not measured at full size)"}}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    threads = os.cpu_count() or 1
    times = []
    byts_step = None
    prep = oracle_prepare(threads, args.reference_layers, args.bits)
    for _ in range(args.warmup):
        oracle_sample(threads, prep, Ms=(1,))
    for _ in range(max(1, args.steps)):
        gbps, secs, byts = oracle_sample(threads, prep)
        times.append(secs)
        byts_step = byts
    t = statistics.median(times)
    value = byts_step / t / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"first {args.reference_layers} layer(s) x 4 linears (qkv, o, gate_up, down) "
                                   f"x M in {{1,4,16}} per step (quantized once, outside the timed steps)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--bits", type=int, default=4, choices=[2, 4])
    ap.add_argument("--layers", type=int, default=synth.LLAMA3_8B_LAYERS)
    ap.add_argument("--oracle-layers", type=int, default=16,
                    help="layers in the CPU baseline's timed oracle sample (about 10 s of CPU work)")
    ap.add_argument("--reference-layers", type=int, default=1,
                    help="layers per step of the reference arm (the oracle)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quant", action="store_true")
    ap.add_argument("--quick", action="store_true", help="skip the per-shape breakdown")
    ap.add_argument("--no-gemm", action="store_true", help="skip the prefill GEMM numbers")
    ap.add_argument("--no-grad", action="store_true", help="skip the input-gradient (backward) numbers")
    ap.add_argument("--no-mixed", action="store_true", help="skip the Layer-mix / Channel-mix decode stacks")
    ap.add_argument("--no-f16-scale", action="store_true", help="skip the INT2 stack with binary16 scales")
    ap.add_argument("--no-other-width", action="store_true",
                    help="skip the second stack at the other width (INT2 g64 when timing INT4)")
    ap.add_argument("--split", action="store_true",
                    help="also time the decode stack split over the ranks by output channels, y all-gathered")
    ap.add_argument("--overlap", type=int, default=2, choices=[0, 1, 2],
                    help="bq_linear launch overlap: 0 plain, 1 programmatic dependent launch, "
                         "2 PDL + weight streaming before the wait (weights are static here)")
    args = ap.parse_args()

    world, rank, local = dist_setup()
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    if args.impl == "reference":
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
    else:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py: a CUDA GPU is required for the GPU arm")
        bq.lib()  # fail loudly if the CUDA library is missing
        out = run_gpu(args, world, rank, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(args)
            print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
