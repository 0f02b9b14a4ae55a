"""Single-kernel cases for profiling (ncu) and timing: one shape, a few
launches, then a device-status check.

    python -m quantized_gemm_group_b200.cases gemv  M N K BITS    # decode linear, M <= 16
    python -m quantized_gemm_group_b200.cases gemm  M N K BITS    # prefill linear, M >= 64
    python -m quantized_gemm_group_b200.cases quant N K BITS      # quantizer, interleaved layout
    python -m quantized_gemm_group_b200.cases grad  M N K BITS    # input gradient dx = dy . dequant(W)

Weights are synthetic fp16 N(0, 0.02) (N(0, 0.015) for the prefill case),
activations (and dy) bf16 N(0, 1); INT4 uses group 128, INT2 group 64.  Each case runs
its kernel 4 times (3 for the prefill case), so a profiler can skip the first
launches.
"""
from __future__ import annotations

import sys

import torch

from . import bq, synth


def main(argv):
    which = argv[0]
    if which in ("gemv", "gemm"):
        M, N, K, bits = (int(v) for v in argv[1:5])
        g = 128 if bits == 4 else 64
        W = synth.normal((N, K), 0.02 if which == "gemv" else 0.015, seed=1, dtype="f16", device="cuda")
        pk, sc, ze = bq.bq_quantize(W, bits, g, "interleaved")
        x = synth.activations(M, K, seed=2, device="cuda")
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        for _ in range(4 if which == "gemv" else 3):
            bq.bq_linear(x, pk, sc, ze, N, bits, g, out=y)
    elif which == "grad":
        M, N, K, bits = (int(v) for v in argv[1:5])
        g = 128 if bits == 4 else 64
        W = synth.normal((N, K), 0.02, seed=1, dtype="f16", device="cuda")
        pk, sc, ze = bq.bq_quantize(W, bits, g, "interleaved")
        dy = synth.activations(M, N, seed=2, device="cuda")
        dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        for _ in range(4):
            bq.bq_linear_grad_input(dy, pk, sc, ze, K, bits, g, out=dx)
    elif which == "quant":
        N, K, bits = (int(v) for v in argv[1:4])
        g = 128 if bits == 4 else 64
        W = synth.normal((N, K), 0.02, seed=1, dtype="f16", device="cuda")
        out = bq.bq_quantize(W, bits, g, "interleaved")
        for _ in range(3):
            bq.bq_quantize(W, bits, g, "interleaved", out=out)
    else:
        raise SystemExit(__doc__)
    torch.cuda.synchronize()
    status = bq.bq_device_status()
    if status != bq.BQ_OK:
        raise SystemExit(f"device status {bq.status_string(status)}")
    print("ok")


if __name__ == "__main__":
    main(sys.argv[1:])
