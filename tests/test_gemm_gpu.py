"""GPU parity of the tensor-core prefill path of the weight-only linear layer
(taken by bq_linear for 64 tokens or more, uniform width, whole 128-row
blocks) with the CPU oracle.

Same tolerance as the decode path: per-token relative L2 error of the 16-bit
output against the oracle's fp64 product rounded to the output type, at most
2e-3."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_gemm_group_b200 import bq, synth

from .test_linear_gpu import check, oracle_y

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("M", [64, 100, 256, 300, 512])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_prefill_small(M, bits, group):
    N, K = 256, 1024
    W = synth.normal((N, K), 0.02, seed=M + bits, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=200 + M, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
    assert bq.bq_device_status() == bq.BQ_OK
    check(y, oracle_y(x, W, bits, group), torch.bfloat16)


@pytest.mark.parametrize("bits,group", [(4, 64), (4, 256), (2, 128), (2, 256)])
def test_prefill_other_groups(bits, group):
    N, K, M = 384, 2048, 200
    W = synth.normal((N, K), 0.02, seed=group + bits, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=5, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
    check(y, oracle_y(x, W, bits, group), torch.bfloat16)


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_prefill_fp16(bits, group):
    N, K, M = 256, 1536 if bits == 4 else 2048, 160
    W = synth.normal((N, K), 0.02, seed=11, dtype="f16", device=DEV)
    x = synth.normal((M, K), 1.0, seed=12, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
    assert y.dtype == torch.float16
    check(y, oracle_y(x, W, bits, group), torch.float16)


def test_prefill_heavy_tailed_int2():
    N, K, M = 512, 4096, 384
    W = synth.student_t4((N, K), 0.02, seed=21, dtype="bf16", device=DEV, outlier_frac=0.001)
    x = synth.activations(M, K, seed=22, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 2, 64, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, 2, 64)
    check(y, oracle_y(x, W, 2, 64), torch.bfloat16)


def test_prefill_matches_decode_blocks():
    """The same product through the tensor-core path (all tokens at once) and
    through 16-token decode passes (token slices of 16) agrees to rounding."""
    N, K, M = 256, 2048, 128
    W = synth.normal((N, K), 0.02, seed=31, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=32, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    y_gemm = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    y_dec = torch.cat([bq.bq_linear(x[m:m + 16].contiguous(), pk, sc, ze, N, 4, 128) for m in range(0, M, 16)])
    d = (y_gemm.float() - y_dec.float()).norm(dim=1) / y_dec.float().norm(dim=1)
    assert float(d.max()) < 2e-3


def test_prefill_deterministic():
    N, K, M = 1024, 4096, 512
    W = synth.normal((N, K), 0.02, seed=41, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=42, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    y1 = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    y2 = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("name,N,K,bits,M", [
    ("q", 4096, 4096, 4, 2048), ("gate", 14336, 4096, 4, 2048), ("down", 4096, 14336, 4, 2048),
    ("down", 4096, 14336, 2, 2048), ("gate", 14336, 4096, 2, 8192), ("qwen_up", 49152, 8192, 4, 2048),
    ("qwen_up", 49152, 8192, 2, 2048), ("qwen_down", 8192, 49152, 4, 2048), ("qwen_down", 8192, 49152, 2, 8192),
    ("gate", 14336, 4096, 4, 4096), ("qwen_down", 8192, 49152, 4, 4096),
])
def test_prefill_full_size_sampled(name, N, K, bits, M):
    """Prefill shapes at the bench's token counts; the oracle checks a sample
    of output channels and tokens (rows and tokens are independent)."""
    group = 128 if bits == 4 else 64
    W = synth.normal((N, K), 0.02, seed=51, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=52, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
    rng = np.random.default_rng(N + K + bits)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.choice(N, 60, replace=False)]))
    toks = np.unique(np.concatenate([[0, 255, 256, M - 1], rng.choice(M, 60, replace=False)]))
    r_t, t_t = torch.from_numpy(rows).to(DEV), torch.from_numpy(toks).to(DEV)
    y_ref = oracle_y(x[t_t].contiguous(), W, bits, group, rows=r_t)
    check(y[t_t][:, r_t], y_ref, torch.bfloat16)


def test_prefill_mixed_small_full():
    """A width map on the tensor-core path: every output against the oracle
    (each 128-row block quantized with its own width)."""
    N, K, M = 768, 1024, 100
    W = synth.normal((N, K), 0.02, seed=61, dtype="f16", device=DEV)
    bit_map = [4, 2, 2, 4, 2, 4]
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map, "interleaved")
    x = synth.activations(M, K, seed=62, device=DEV)
    y = bq.bq_linear(x, pk, sc, ze, N, bit_map_dev=bm)
    assert bq.bq_device_status() == bq.BQ_OK
    _, _, _, blocks = O.quantize_mixed(synth.bits16(W), "f16", bit_map, "interleaved", threads=8)
    y_ref = O.linear_mixed_f64(O.decode_f64(synth.bits16(x), "bf16"), blocks, bit_map, threads=8)
    check(y, y_ref, torch.bfloat16)


def test_prefill_layer_mix_equals_uniform():
    """A constant map runs the same arithmetic as the uniform call: equal bits."""
    N, K, M = 512, 2048, 300
    W = synth.normal((N, K), 0.02, seed=63, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=64, device=DEV)
    for bits, group in ((4, 128), (2, 64)):
        pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
        y_uni = bq.bq_linear(x, pk, sc, ze, N, bits, group)
        pk2, sc2, ze2, bm = bq.bq_quantize_mixed(W, [bits] * (N // 128), "interleaved")
        y_mix = bq.bq_linear(x, pk2, sc2, ze2, N, bit_map_dev=bm)
        assert torch.equal(y_uni, y_mix)


@pytest.mark.parametrize("M", [64, 256, 2048])
def test_prefill_channel_mix_llama_sampled(M):
    """Channel-mix (25% of the 128-row blocks at 4 bits) on a Llama-3-8B
    gate shape through the tensor-core path; sampled rows of both widths and
    sampled tokens against the oracle."""
    from .test_linear_gpu import oracle_y_mixed_rows
    N, K = 14336, 4096
    W = synth.normal((N, K), 0.015, seed=65, dtype="f16", device=DEV)
    bit_map = synth.channel_mix_map(N, seed=66).tolist()
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map, "interleaved")
    x = synth.activations(M, K, seed=67, device=DEV)
    y = bq.bq_linear(x, pk, sc, ze, N, bit_map_dev=bm)
    assert bq.bq_device_status() == bq.BQ_OK
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.choice(N, 40, replace=False)]))
    toks = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(M, 24), replace=False)]))
    t_t = torch.from_numpy(toks).to(DEV)
    y_ref = oracle_y_mixed_rows(x[t_t].contiguous(), W, bit_map, rows)
    check(y[t_t][:, torch.from_numpy(rows).to(DEV)], y_ref, torch.bfloat16)
