"""GPU parity of the symmetric abs-max quantizer (bq_quantize_symmetric) with
the CPU oracle: packed codes, scales and zeros bit-exact in both layouts;
the weight-only linear consumes its output unchanged (within the linear
tolerance of the oracle's fp64 product)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_gemm_group_b200 import bq, synth

from .test_linear_gpu import check

pytestmark = pytest.mark.gpu

DEV = "cuda"


def oracle_sym(W, bits, group, layout):
    wt = "f16" if W.dtype == torch.float16 else "bf16"
    codes, scales, zeros = O.quantize(synth.bits16(W), wt, bits, group, threads=8, scheme="symmetric")
    ms, mz = O.pack_meta(scales, zeros, layout)
    return O.pack(codes, bits, layout), ms, mz, codes, scales, zeros


@pytest.mark.parametrize("layout", ["canonical", "interleaved"])
@pytest.mark.parametrize("wdt", ["f16", "bf16"])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64), (4, 32)])
def test_symmetric_bit_exact(layout, wdt, bits, group):
    W = synth.student_t4((272, 1024), 0.02, seed=bits + group, dtype=wdt, device=DEV, outlier_frac=0.01)
    W[5, :group] = 0.0                                  # an all-zero group
    pk, sc, ze = bq.bq_quantize(W, bits, group, layout, scheme="symmetric")
    assert bq.bq_device_status() == bq.BQ_OK
    rpk, rsc, rze, codes, _, _ = oracle_sym(W, bits, group, layout)
    assert (sc.cpu().numpy().reshape(-1).view(np.uint32) == rsc.view(np.uint32)).all(), "scales differ"
    assert (ze.cpu().numpy().reshape(-1) == rze).all(), "zeros differ"
    assert (pk.cpu().numpy() == rpk).all(), "packed codes differ"
    assert (ze.cpu().numpy() == (1 << (bits - 1))).all()


@pytest.mark.parametrize("M", [1, 16, 128])
def test_symmetric_linear(M):
    N, K = 512, 2048
    W = synth.normal((N, K), 0.02, seed=M, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=M + 1, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved", scheme="symmetric")
    y = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    codes, scales, zeros = O.quantize(synth.bits16(W), "f16", 4, 128, threads=8, scheme="symmetric")
    xf = O.decode_f64(synth.bits16(x), "bf16")
    check(y, O.linear_f64(xf, codes, scales, zeros, 128, threads=8), torch.bfloat16)
