"""GPU parity of the split-K plan of the tensor-core kernel (bq_linear_ws):
y against the oracle's fp64 product at token counts where the output tiles
do not fill the GPU, identical across repeated calls on the same workspace
(fixed rank order of the partial sums; counters reset by the library), and
bq_linear's result when the workspace is too small to split."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_gemm_group_b200 import bq, synth

from .test_linear_gpu import check

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ws(M, N, K, bits, mixed=False):
    n = bq.bq_linear_workspace_bytes(M, N, K, bits, mixed)
    return n, torch.empty(max(n, 256), dtype=torch.uint8, device=DEV)


@pytest.mark.parametrize("N,K,bits", [(4096, 4096, 4), (6144, 4096, 4), (4096, 14336, 4), (1024, 4096, 2),
                                      (2048, 2048, 4)])
@pytest.mark.parametrize("M", [64, 100, 256, 300])
def test_split_k_matches_oracle(N, K, bits, M):
    group = 128 if bits == 4 else 64
    W = synth.normal((N, K), 0.02, seed=N + K + M, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=M, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    n, ws = _ws(M, N, K, bits)
    tiles = (N // 128) * ((M + 255) // 256)
    if 2 * tiles <= torch.cuda.get_device_properties(0).multi_processor_count:
        assert n > 0, "the plan should split this shape"
    y1 = bq.bq_linear(x, pk, sc, ze, N, bits, group, workspace=ws)
    y2 = bq.bq_linear(x, pk, sc, ze, N, bits, group, workspace=ws)
    assert bq.bq_device_status() == bq.BQ_OK
    assert torch.equal(y1, y2)
    codes, scales, zeros = O.quantize(synth.bits16(W), "f16", bits, group, threads=8)
    check(y1, O.linear_f64(O.decode_f64(synth.bits16(x), "bf16"), codes, scales, zeros, group, threads=8),
          torch.bfloat16)
    y0 = bq.bq_linear(x, pk, sc, ze, N, bits, group)
    d = (y1.float() - y0.float()).abs().max().item()
    assert d <= 2e-2 * y0.float().abs().max().item()


def test_split_k_fp16_and_small_workspace():
    N, K, M = 4096, 4096, 128
    W = synth.normal((N, K), 0.02, seed=5, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=6, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    n, ws = _ws(M, N, K, 4)
    y = bq.bq_linear(x, pk, sc, ze, N, 4, 128, workspace=ws)
    codes, scales, zeros = O.quantize(synth.bits16(W), "f16", 4, 128, threads=8)
    check(y, O.linear_f64(O.decode_f64(synth.bits16(x), "f16"), codes, scales, zeros, 128, threads=8),
          torch.float16)
    small = torch.empty(n // 2, dtype=torch.uint8, device=DEV)
    assert torch.equal(bq.bq_linear(x, pk, sc, ze, N, 4, 128, workspace=small), bq.bq_linear(x, pk, sc, ze, N, 4, 128))
    assert bq.bq_device_status() == bq.BQ_OK


@pytest.mark.parametrize("M", [64, 200])
def test_split_k_channel_mix(M):
    N, K = 1024, 4096
    bit_map = synth.channel_mix_map(N, seed=M)
    bit_map[0], bit_map[1] = 4, 2
    W = synth.normal((N, K), 0.02, seed=M + 1, dtype="f16", device=DEV)
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map)
    x = synth.activations(M, K, seed=M + 2, device=DEV)
    n, ws = _ws(M, N, K, 4, mixed=True)
    assert n > 0
    y = bq.bq_linear(x, pk, sc, ze, N, bit_map_dev=bm, workspace=ws)
    assert bq.bq_device_status() == bq.BQ_OK
    _, _, _, blocks = O.quantize_mixed(synth.bits16(W), "f16", bit_map, "interleaved", threads=8)
    check(y, O.linear_mixed_f64(O.decode_f64(synth.bits16(x), "bf16"), blocks, bit_map, threads=8), torch.bfloat16)


def test_workspace_alignment_and_large_shapes():
    # a shape whose tiles fill the GPU plans no split
    assert bq.bq_linear_workspace_bytes(4096, 28672, 4096, 4) == 0
    assert bq.bq_linear_workspace_bytes(16, 4096, 4096, 4) == 0        # decode kernel, no workspace
    W = synth.normal((1024, 4096), 0.02, seed=9, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    x = synth.activations(64, 4096, seed=10, device=DEV)
    ws = torch.empty(bq.bq_linear_workspace_bytes(64, 1024, 4096, 4) + 512, dtype=torch.uint8, device=DEV)
    with pytest.raises(bq.BQError):
        bq.bq_linear(x, pk, sc, ze, 1024, 4, 128, workspace=ws[1:])     # not 256-byte aligned
