"""GPU parity of the fused fake-quantization pass (bq_fake_quantize) with
the CPU oracle: W_out must equal the oracle's dequant(quant(W)) -- codes,
scales and zeros from the oracle quantizer, (q - z) * s in fp32, rounded once
to the output type -- bit for bit, and equal bq_dequantize(bq_quantize(W))."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_gemm_group_b200 import bq, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def oracle_fake(W: torch.Tensor, bits: int, group: int, out_dtype) -> np.ndarray:
    wt = "f16" if W.dtype == torch.float16 else "bf16"
    codes, scales, zeros = O.quantize(synth.bits16(W), wt, bits, group, threads=8)
    w32 = O.dequant_f32(codes, scales, zeros, group)
    if out_dtype == torch.float32:
        return w32.view(np.uint32)
    if out_dtype == torch.float16:
        return w32.astype(np.float16).view(np.uint16)
    return O.to_bf16_bits(w32.astype(np.float64))


@pytest.mark.parametrize("wdt", ["f16", "bf16"])
@pytest.mark.parametrize("odt", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64), (4, 32), (2, 8)])
def test_fake_quant_bit_exact(wdt, odt, bits, group):
    # 37 rows x 256 columns: several 256-weight warp steps and a ragged tail
    W = synth.student_t4((37, 256), 0.02, seed=bits * 100 + group, dtype=wdt, device=DEV, outlier_frac=0.01)
    out = bq.bq_fake_quantize(W, bits, group, out_dtype=odt)
    assert bq.bq_device_status() == bq.BQ_OK
    if odt == torch.float32:
        got = out.view(torch.int32).cpu().numpy().view(np.uint32)
    else:
        got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert (got == oracle_fake(W, bits, group, odt)).all()


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_fake_quant_equals_quantize_then_dequantize(bits, group):
    W = synth.normal((1024, 4096), 0.02, seed=3, dtype="bf16", device=DEV)
    fused = bq.bq_fake_quantize(W, bits, group, out_dtype=torch.bfloat16)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "canonical")
    two_pass = bq.bq_dequantize(pk, sc, ze, 1024, 4096, bits, group, "canonical", out_dtype=torch.bfloat16)
    assert torch.equal(fused.view(torch.int16), two_pass.view(torch.int16))


def test_fake_quant_nonfinite_flag():
    W = synth.normal((16, 256), 0.02, seed=4, dtype="f16", device=DEV)
    W[3, 17] = float("inf")
    bq.bq_fake_quantize(W, 4, 128)
    assert bq.bq_device_status() == bq.BQ_ERR_NONFINITE
    assert bq.bq_device_status() == bq.BQ_OK
