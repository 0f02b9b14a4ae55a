"""GPU parity of the weight-only linear layer with the CPU oracle.

Tolerance (the reading of "max relative error 2e-3" on bf16 outputs): for
every token m, ||y_m - bf16(y_ref,m)||_2 / ||bf16(y_ref,m)||_2 <= 2e-3, where
y_ref is the oracle's fp64 product over the dequantized weights and bf16() its
round-to-nearest (fp16 outputs likewise with fp16).  An elementwise ratio is
unattainable for any implementation: one output that straddles a bf16
rounding boundary already differs by one ulp (2^-8 relative)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_gemm_group_b200 import bq, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = 2e-3


def oracle_y(x: torch.Tensor, W: torch.Tensor, bits, group, rows=None):
    """fp64 oracle output for the given output rows (all rows by default)."""
    wt = "f16" if W.dtype == torch.float16 else "bf16"
    Wr = W if rows is None else W[rows]
    codes, scales, zeros = O.quantize(synth.bits16(Wr), wt, bits, group, threads=8)
    xt = "f16" if x.dtype == torch.float16 else "bf16"
    xf = O.decode_f64(synth.bits16(x), xt)
    return O.linear_f64(xf, codes, scales, zeros, group, threads=8)


def round_ref(y_ref: np.ndarray, dtype) -> np.ndarray:
    if dtype == torch.bfloat16:
        return O.bf16_bits_to_f64(O.to_bf16_bits(y_ref))
    return y_ref.astype(np.float16).astype(np.float64)


def rel_err(y_gpu: torch.Tensor, y_ref: np.ndarray, dtype):
    yr = round_ref(y_ref, dtype)
    yg = y_gpu.double().cpu().numpy()
    num = np.linalg.norm(yg - yr, axis=1)
    den = np.linalg.norm(yr, axis=1)
    return float(np.max(num / np.maximum(den, 1e-300))), yg, yr


def check(y_gpu, y_ref, dtype, tol=TOL):
    err, yg, yr = rel_err(y_gpu, y_ref, dtype)
    assert np.isfinite(yg).all()
    assert err <= tol, f"max per-token relative L2 error {err:.3e} > {tol}"
    return err


def test_config1_fp16():
    W = synth.normal((1024, 1024), 0.02, seed=0, dtype="f16", device=DEV)
    x = synth.normal((1, 1024), 1.0, seed=1, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, 1024, 4, 128)
    err = check(y, oracle_y(x, W, 4, 128), torch.float16)
    assert err < 2e-4


@pytest.mark.parametrize("M", [1, 2, 4, 7, 8, 9, 12, 16])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_decode_shapes_bf16(M, bits, group):
    N, K = 1024, 4096
    W = synth.normal((N, K), 0.02, seed=M + bits, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=100 + M, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
    check(y, oracle_y(x, W, bits, group), torch.bfloat16)


@pytest.mark.parametrize("bits,group", [(4, 32), (4, 64), (4, 256), (2, 32), (2, 128), (2, 256)])
def test_other_groups(bits, group):
    N, K = 272, 1024
    W = synth.normal((N, K), 0.02, seed=group, dtype="f16", device=DEV)
    x = synth.activations(5, K, seed=3, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
    check(y, oracle_y(x, W, bits, group), torch.bfloat16)


@pytest.mark.parametrize("N,K", [(16, 256), (48, 512), (16, 4096), (32, 14336), (112, 1536), (144, 1024),
                                 (400, 2560)])
def test_small_and_ragged(N, K):
    """Shapes with one row tile, partial 128-row blocks, odd block counts."""
    W = synth.normal((N, K), 0.02, seed=N, dtype="f16", device=DEV)
    x = synth.activations(3, K, seed=K, device=DEV)
    for bits, group in ((4, 128), (2, 64)):
        if K % (256 if bits == 4 else 512):
            continue
        pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
        y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
        check(y, oracle_y(x, W, bits, group), torch.bfloat16)


def test_heavy_tailed_int2_outliers():
    N, K = 1024, 4096
    W = synth.student_t4((N, K), 0.02, seed=31, dtype="f16", device=DEV, outlier_frac=0.001)
    x = synth.activations(16, K, seed=32, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 2, 64, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, 2, 64)
    check(y, oracle_y(x, W, 2, 64), torch.bfloat16)


def test_more_than_16_tokens():
    N, K = 528, 1024
    W = synth.normal((N, K), 0.02, seed=41, dtype="f16", device=DEV)
    x = synth.activations(40, K, seed=42, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    check(y, oracle_y(x, W, 4, 128), torch.bfloat16)


def test_deterministic():
    N, K = 4096, 4096
    W = synth.normal((N, K), 0.02, seed=51, dtype="f16", device=DEV)
    x = synth.activations(16, K, seed=52, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    y1 = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    y2 = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("M", [1, 16])
def test_channel_mix(M):
    N, K = 1024, 4096
    W = synth.normal((N, K), 0.02, seed=61, dtype="f16", device=DEV)
    x = synth.activations(M, K, seed=62, device=DEV)
    bit_map = synth.channel_mix_map(N, seed=7)
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map, "interleaved")
    y = bq.bq_linear(x, pk, sc, ze, N, bit_map_dev=bm)
    _, _, _, blocks = O.quantize_mixed(synth.bits16(W), "f16", bit_map, "interleaved", threads=8)
    xf = O.decode_f64(synth.bits16(x), "bf16")
    y_ref = O.linear_mixed_f64(xf, blocks, bit_map, threads=8)
    check(y, y_ref, torch.bfloat16)


def test_layer_mix_is_uniform_map():
    """Layer-mix assigns one width per layer: a constant map must equal the
    uniform call."""
    N, K = 512, 2048
    W = synth.normal((N, K), 0.02, seed=71, dtype="f16", device=DEV)
    x = synth.activations(4, K, seed=72, device=DEV)
    for bits, group in ((4, 128), (2, 64)):
        pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
        y_uni = bq.bq_linear(x, pk, sc, ze, N, bits, group)
        pk2, sc2, ze2, bm = bq.bq_quantize_mixed(W, [bits] * (N // 128), "interleaved")
        assert torch.equal(pk, pk2) and torch.equal(sc.reshape(-1), sc2) and torch.equal(ze.reshape(-1), ze2)
        y_mix = bq.bq_linear(x, pk2, sc2, ze2, N, bit_map_dev=bm)
        assert torch.equal(y_uni, y_mix)


@pytest.mark.parametrize("name,N,K,bits", [
    ("gate", 14336, 4096, 4), ("down", 4096, 14336, 4), ("q", 4096, 4096, 2), ("down", 4096, 14336, 2),
])
def test_full_size_sampled_rows(name, N, K, bits):
    """Llama-3-8B shapes at the bench's launch geometry; the oracle checks a
    sample of output channels (rows quantize independently)."""
    group = 128 if bits == 4 else 64
    if bits == 4:
        W = synth.normal((N, K), 0.02, seed=81, dtype="f16", device=DEV)
    else:
        W = synth.student_t4((N, K), 0.02, seed=82, dtype="f16", device=DEV, outlier_frac=0.001)
    x = synth.activations(16, K, seed=83, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    for M in (1, 4, 16):
        y = bq.bq_linear(x[:M].contiguous(), pk, sc, ze, N, bits, group)
        rng = np.random.default_rng(N + M)
        rows = np.sort(np.concatenate([[0, N - 1], rng.choice(N, 62, replace=False)]))
        rows = np.unique(rows)
        y_ref = oracle_y(x[:M].contiguous(), W, bits, group, rows=torch.from_numpy(rows).to(DEV))
        check(y[:, torch.from_numpy(rows).to(DEV)], y_ref, torch.bfloat16)


def test_fused_projections():
    """q/k/v quantized into consecutive slices of one buffer equal the
    quantized concatenation, and one linear over it matches the oracle."""
    K = 2048
    Ws = [synth.normal((n, K), 0.02, seed=90 + i, dtype="f16", device=DEV) for i, n in enumerate((512, 128, 128))]
    Wc = torch.cat(Ws)
    N = Wc.shape[0]
    pk, sc, ze = bq.bq_quantize(Wc, 4, 128, "interleaved")
    pk2, sc2, ze2 = torch.empty_like(pk), torch.empty_like(sc), torch.empty_like(ze)
    r0 = 0
    for W in Ws:
        n = W.shape[0]
        cb, ce = bq.bq_packed_bytes(r0, K, 4), bq.bq_packed_bytes(r0 + n, K, 4)
        gb, ge = r0 * (K // 128), (r0 + n) * (K // 128)
        bq.bq_quantize(W, 4, 128, "interleaved", out=(pk2[cb:ce], sc2[gb:ge], ze2[gb:ge]))
        r0 += n
    assert torch.equal(pk, pk2) and torch.equal(sc, sc2) and torch.equal(ze, ze2)
    x = synth.activations(4, K, seed=93, device=DEV)
    y = bq.bq_linear(x, pk2, sc2, ze2, N, 4, 128)
    check(y, oracle_y(x, Wc, 4, 128), torch.bfloat16)


def oracle_y_mixed_rows(x: torch.Tensor, W: torch.Tensor, bit_map, rows: np.ndarray):
    """fp64 oracle output of a mixed-width matrix for the given rows: each row
    quantized with its 128-row block's width (rows quantize independently)."""
    xf = O.decode_f64(synth.bits16(x), "bf16")
    cols = []
    for n in rows:
        b = int(bit_map[int(n) // 128])
        g = O.GROUP_OF_BITS[b]
        c, s_, z = O.quantize(synth.bits16(W[int(n):int(n) + 1]), "f16", b, g)
        cols.append(O.linear_f64(xf, c, s_, z, g)[:, 0])
    return np.stack(cols, axis=1)


@pytest.mark.parametrize("kind,N,K", [("channel", 14336, 4096), ("channel", 4096, 14336),
                                      ("layer4", 14336, 4096), ("layer2", 4096, 14336)])
def test_mixed_llama_sized_sampled(kind, N, K):
    """Llama-3-8B-sized Channel-mix (25% of the 128-row blocks at 4 bits) and
    Layer-mix (one width for the whole matrix) at M = 1 and 16, through the
    mixed launch; the oracle checks sampled output channels of every width."""
    W = synth.normal((N, K), 0.02, seed=N + 3, dtype="f16", device=DEV)
    if kind == "channel":
        bit_map = synth.channel_mix_map(N, seed=N + 5).tolist()
    else:
        bit_map = [4 if kind == "layer4" else 2] * (N // 128)
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map, "interleaved")
    rng = np.random.default_rng(N)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.choice(N, 44, replace=False)]))
    x = synth.activations(16, K, seed=K + 9, device=DEV)
    for M in (1, 16):
        y = bq.bq_linear(x[:M].contiguous(), pk, sc, ze, N, bit_map_dev=bm)
        y_ref = oracle_y_mixed_rows(x[:M].contiguous(), W, bit_map, rows)
        check(y[:, torch.from_numpy(rows).to(DEV)], y_ref, torch.bfloat16)
    assert bq.bq_device_status() == bq.BQ_OK


def test_decode_split_blocks_many_shapes():
    """The persistent decode kernel splits 128-row blocks between CTAs at
    unit boundaries that depend on the shape; sweep shapes whose blocks are
    split in different places (and a last partial block) against the oracle."""
    for N, K in ((144, 4096), (1040, 2048), (3072, 1536), (256, 14336)):
        W = synth.normal((N, K), 0.02, seed=N + K, dtype="f16", device=DEV)
        for bits, group in ((4, 128), (2, 64)):
            if K % (256 if bits == 4 else 512):
                continue
            pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
            for M in (1, 16):
                x = synth.activations(M, K, seed=M + N, device=DEV)
                y = bq.bq_linear(x, pk, sc, ze, N, bits, group)
                check(y, oracle_y(x, W, bits, group), torch.bfloat16)
