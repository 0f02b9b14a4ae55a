"""GPU parity of the binary16-scale format (bq_quantize_f16s / bq_linear_f16s)
with the CPU oracle's "asymmetric_f16_scale" scheme: packed codes, binary16
scales and zeros bit-exact in both layouts (including scales in the binary16
subnormal range); the linear layer on those weights within the linear
tolerance of the oracle's fp64 product, and bit-identical to bq_linear given
the same scale values as fp32."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_gemm_group_b200 import bq, synth

from .test_linear_gpu import check

pytestmark = pytest.mark.gpu

DEV = "cuda"
SCHEME = "asymmetric_f16_scale"


def oracle_f16s(W, bits, group, layout):
    wt = "f16" if W.dtype == torch.float16 else "bf16"
    codes, scales, zeros = O.quantize(synth.bits16(W), wt, bits, group, threads=8, scheme=SCHEME)
    ms, mz = O.pack_meta(scales, zeros, layout)
    return O.pack(codes, bits, layout), ms, mz, codes, scales, zeros


@pytest.mark.parametrize("layout", ["canonical", "interleaved"])
@pytest.mark.parametrize("wdt", ["f16", "bf16"])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_f16_scale_bit_exact(layout, wdt, bits, group):
    W = synth.student_t4((272, 1024), 0.02, seed=bits + group, dtype=wdt, device=DEV, outlier_frac=0.01)
    W[5, :group] = 0.0                                     # an all-zero group
    W[6, group:2 * group] *= 1e-4                          # scales in the binary16 subnormals
    W[7, :group] *= 1e-7                                   # scales below the binary16 range (-> 2^-24)
    pk, sc, ze = bq.bq_quantize(W, bits, group, layout, scheme=SCHEME)
    assert sc.dtype == torch.float16
    assert bq.bq_device_status() == bq.BQ_OK
    rpk, rsc, rze, codes, _, _ = oracle_f16s(W, bits, group, layout)
    want = O.f32_to_f16_bits(rsc)
    assert (want.view(np.float16).astype(np.float32) == rsc).all()  # every oracle scale is a binary16 value
    got = sc.cpu().numpy().reshape(-1).view(np.uint16)
    assert (got == want.reshape(-1)).all(), "scales differ"
    assert (ze.cpu().numpy().reshape(-1) == rze).all(), "zeros differ"
    assert (pk.cpu().numpy() == rpk).all(), "packed codes differ"


def test_f16_scale_overflow_sets_nonfinite():
    # bf16 weights whose group range needs a scale above 65504
    W = synth.normal((16, 128), 1.0, seed=3, dtype="bf16", device=DEV)
    W[2, :] *= 1e6
    bq.bq_quantize(W, 4, 128, "interleaved", scheme=SCHEME)
    assert bq.bq_device_status() == bq.BQ_ERR_NONFINITE
    assert bq.bq_device_status() == bq.BQ_OK


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
@pytest.mark.parametrize("M", [1, 5, 16, 64, 300])
@pytest.mark.parametrize("xdt", ["bf16", "f16"])
def test_f16_scale_linear(bits, group, M, xdt):
    N, K = 640, 2048
    W = synth.student_t4((N, K), 0.02, seed=10 * bits + M, dtype="f16", device=DEV, outlier_frac=0.001)
    x = synth.activations(M, K, seed=M + 1, dtype=xdt, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved", scheme=SCHEME)
    y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
    assert bq.bq_device_status() == bq.BQ_OK
    codes, scales, zeros = O.quantize(synth.bits16(W), "f16", bits, group, threads=8, scheme=SCHEME)
    xf = O.decode_f64(synth.bits16(x), xdt)
    check(y, O.linear_f64(xf, codes, scales, zeros, group, threads=8),
          torch.bfloat16 if xdt == "bf16" else torch.float16)
    # the same weights with the scale values in fp32 through bq_linear: the
    # binary16 scale is exact in fp32, so every output is identical
    y32 = bq.bq_linear(x, pk, sc.float(), ze, N, bits, group)
    assert torch.equal(y, y32)


def test_f16_scale_rejects_other_groups_and_maps():
    W = synth.normal((128, 1024), 0.02, seed=1, dtype="f16", device=DEV)
    with pytest.raises(bq.BQError):
        bq.bq_quantize(W, 4, 64, "interleaved", scheme=SCHEME)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved", scheme=SCHEME)
    x = synth.activations(1, 1024, seed=2, device=DEV)
    with pytest.raises(bq.BQError):
        bq.bq_linear(x, pk, sc, ze, 128, 4, 64)
