"""GPU parity of the input gradient of the weight-only linear layer,
dx = dy . dequant(W) (bq_linear_grad_input), with the CPU oracle.

Tolerance: per-token relative L2 error of the 16-bit dx against the oracle's
fp64 result rounded to the output type, at most 2e-3 -- the bound of the
forward product.  The kernel's one rounding before its fp32 accumulation is
dy * s to tf32 (relative 2^-11); the smoke case measures about 1.1e-3."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_gemm_group_b200 import bq, synth

from .test_linear_gpu import check

pytestmark = pytest.mark.gpu

DEV = "cuda"


def oracle_dx(dy: torch.Tensor, W: torch.Tensor, bits, group, scheme="asymmetric", groups=None):
    """fp64 oracle dx for the given groups of columns (all by default)."""
    wt = "f16" if W.dtype == torch.float16 else "bf16"
    if groups is not None:
        cols = torch.cat([torch.arange(j * group, (j + 1) * group) for j in groups]).to(W.device)
        W = W[:, cols]
    codes, scales, zeros = O.quantize(synth.bits16(W), wt, bits, group, threads=8, scheme=scheme)
    dt = "f16" if dy.dtype == torch.float16 else "bf16"
    dyf = O.decode_f64(synth.bits16(dy), dt)
    return O.linear_grad_input_f64(dyf, codes, scales, zeros, group, threads=8)


@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_grad_small(M, bits, group):
    N, K = 512, 1024
    W = synth.normal((N, K), 0.02, seed=M + bits, dtype="f16", device=DEV)
    dy = synth.activations(M, N, seed=300 + M, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bits, group)
    assert bq.bq_device_status() == bq.BQ_OK
    assert dx.shape == (M, K) and dx.dtype == dy.dtype
    check(dx, oracle_dx(dy, W, bits, group), torch.bfloat16)


@pytest.mark.parametrize("bits,group", [(4, 32), (4, 64), (4, 256), (2, 32), (2, 128), (2, 256)])
def test_grad_other_groups(bits, group):
    N, K, M = 384, 2048, 12
    W = synth.normal((N, K), 0.02, seed=group + bits, dtype="f16", device=DEV)
    dy = synth.activations(M, N, seed=7, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bits, group)
    check(dx, oracle_dx(dy, W, bits, group), torch.bfloat16)


@pytest.mark.parametrize("N", [16, 144, 272, 1040])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_grad_partial_row_block(N, bits, group):
    """N not a multiple of 128: the last row block holds N % 128 rows."""
    K, M = 512, 5
    W = synth.normal((N, K), 0.02, seed=N, dtype="f16", device=DEV)
    dy = synth.activations(M, N, seed=N + 1, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bits, group)
    check(dx, oracle_dx(dy, W, bits, group), torch.bfloat16)


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_grad_fp16(bits, group):
    N, K, M = 256, 1536, 16
    W = synth.normal((N, K), 0.02, seed=11, dtype="bf16", device=DEV)
    dy = synth.normal((M, N), 1.0, seed=12, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bits, group)
    assert dx.dtype == torch.float16
    check(dx, oracle_dx(dy, W, bits, group), torch.float16)


def test_grad_many_tokens():
    """More than 16 tokens run in 16-token passes."""
    N, K, M = 256, 1024, 40
    W = synth.normal((N, K), 0.02, seed=21, dtype="f16", device=DEV)
    dy = synth.activations(M, N, seed=22, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, 4, 128)
    check(dx, oracle_dx(dy, W, 4, 128), torch.bfloat16)


def test_grad_heavy_tailed_int2():
    N, K, M = 512, 4096, 16
    W = synth.student_t4((N, K), 0.02, seed=31, dtype="bf16", device=DEV, outlier_frac=0.001)
    dy = synth.activations(M, N, seed=32, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 2, 64, "interleaved")
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, 2, 64)
    check(dx, oracle_dx(dy, W, 2, 64), torch.bfloat16)


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_grad_symmetric_weights(bits, group):
    N, K, M = 256, 1024, 4
    W = synth.normal((N, K), 0.02, seed=41, dtype="f16", device=DEV)
    dy = synth.activations(M, N, seed=42, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved", scheme="symmetric")
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bits, group)
    check(dx, oracle_dx(dy, W, bits, group, scheme="symmetric"), torch.bfloat16)


def test_grad_edge_cases():
    W = synth.normal((256, 512), 0.02, seed=51, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    # no tokens: nothing to do
    dx = bq.bq_linear_grad_input(torch.empty((0, 256), dtype=torch.bfloat16, device=DEV), pk, sc, ze, 512, 4, 128)
    assert dx.shape == (0, 512)
    # no output channels: an empty sum, dx = 0
    dx = torch.full((3, 512), 7.0, dtype=torch.bfloat16, device=DEV)
    bq.bq_linear_grad_input(torch.empty((3, 0), dtype=torch.bfloat16, device=DEV), pk[:0], sc, ze, 512, 4, 128,
                            out=dx)
    assert (dx == 0).all()
    # an all-zero dy gives exactly zero
    dx = bq.bq_linear_grad_input(torch.zeros((4, 256), dtype=torch.bfloat16, device=DEV), pk, sc, ze, 512, 4, 128)
    assert (dx == 0).all()
    # bad shape comes back as an error
    with pytest.raises(bq.BQError):
        bq.bq_linear_grad_input(torch.zeros((4, 256), dtype=torch.bfloat16, device=DEV), pk, sc, ze, 448, 4, 64)
    assert bq.bq_device_status() == bq.BQ_OK


def test_grad_one_hot_selects_dequantized_rows():
    """dy = one-hot rows picks rows of dequant(W): within the tf32 rounding
    of s and the bf16 rounding of dx (2^-11 + 2^-9 < 2^-8 relative), and
    exactly zero where q = z."""
    N, K = 384, 1024
    W = synth.normal((N, K), 0.02, seed=61, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    picks = [0, 5, 127, 128, 200, N - 1]
    dy = torch.zeros((len(picks), N), dtype=torch.bfloat16, device=DEV)
    for m, n in enumerate(picks):
        dy[m, n] = 1.0
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, 4, 128)
    Wd = bq.bq_dequantize(pk, sc, ze, N, K, 4, 128, "interleaved", out_dtype=torch.float32)[picks]
    assert ((dx.float() - Wd).abs() <= Wd.abs() * 2.0 ** -8).all()
    assert ((Wd == 0) == (dx == 0)).all()


def test_grad_adjoint_of_forward():
    """<dy, bq_linear(x)> = <bq_linear_grad_input(dy), x> up to the rounding of
    both 16-bit outputs, at a decode shape."""
    N, K, M = 6144, 4096, 8
    W = synth.normal((N, K), 0.02, seed=71, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    x = synth.activations(M, K, seed=72, device=DEV)
    dy = synth.activations(M, N, seed=73, device=DEV)
    y = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, 4, 128)
    lhs = (dy.double() * y.double()).sum(dim=1)
    rhs = (dx.double() * x.double()).sum(dim=1)
    scale = (dy.double().norm(dim=1) * y.double().norm(dim=1))
    assert float(((lhs - rhs).abs() / scale).max()) < 4e-3


def test_grad_deterministic():
    N, K, M = 4096, 4096, 16
    W = synth.normal((N, K), 0.02, seed=81, dtype="f16", device=DEV)
    dy = synth.activations(M, N, seed=82, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    d1 = bq.bq_linear_grad_input(dy, pk, sc, ze, K, 4, 128)
    d2 = bq.bq_linear_grad_input(dy, pk, sc, ze, K, 4, 128)
    assert torch.equal(d1, d2)


@pytest.mark.parametrize("name,N,K,bits,M", [
    ("qkv", 6144, 4096, 4, 16), ("gate_up", 28672, 4096, 4, 16), ("down", 4096, 14336, 4, 1),
    ("down", 4096, 14336, 2, 16), ("gate_up", 28672, 4096, 2, 4), ("o", 4096, 4096, 4, 4),
])
def test_grad_full_size_sampled(name, N, K, bits, M):
    """Decode-stack shapes (the backward of each fused projection); the oracle
    checks a sample of whole groups of columns (groups are independent along K)."""
    group = 128 if bits == 4 else 64
    W = synth.normal((N, K), 0.02, seed=91, dtype="f16", device=DEV)
    dy = synth.activations(M, N, seed=92, device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bits, group)
    G = K // group
    rng = np.random.default_rng(N + K + bits)
    groups = sorted(set([0, G - 1] + rng.choice(G, 4, replace=False).tolist()))
    cols = torch.cat([torch.arange(j * group, (j + 1) * group) for j in groups]).to(DEV)
    check(dx[:, cols], oracle_dx(dy, W, bits, group, groups=groups), torch.bfloat16)


# ---------------------------------------------------------------------------
# width maps (Layer-mix / Channel-mix)
# ---------------------------------------------------------------------------

def oracle_dx_mixed(dy: torch.Tensor, W: torch.Tensor, bit_map):
    """fp64 oracle dx of a mixed matrix: the sum over its 128-row blocks of
    each block's input gradient (the block's own width and group)."""
    _, _, _, blocks = O.quantize_mixed(synth.bits16(W), "f16", bit_map, "interleaved", threads=8)
    dt = "f16" if dy.dtype == torch.float16 else "bf16"
    dyf = O.decode_f64(synth.bits16(dy), dt)
    ref = None
    for i, ((c, s, z), b) in enumerate(zip(blocks, bit_map)):
        part = O.linear_grad_input_f64(dyf[:, 128 * i:128 * (i + 1)], c, s, z, O.GROUP_OF_BITS[int(b)], threads=8)
        ref = part if ref is None else ref + part
    return ref


@pytest.mark.parametrize("M", [1, 9, 16, 40])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_grad_channel_mix(M, dt):
    N, K = 1280, 1024
    bit_map = synth.channel_mix_map(N, seed=M + 5)
    bit_map[1] = 4                       # both widths present whatever the draw
    bit_map[2] = 2
    W = synth.student_t4((N, K), 0.02, seed=M, dtype="f16", device=DEV, outlier_frac=0.001)
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map)
    dy = synth.activations(M, N, seed=M + 11, dtype=dt, device=DEV)
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bit_map_dev=bm)
    assert bq.bq_device_status() == bq.BQ_OK
    check(dx, oracle_dx_mixed(dy, W, bit_map), torch.bfloat16 if dt == "bf16" else torch.float16)


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("M", [1, 16])
def test_grad_layer_mix_equals_uniform(bits, M):
    """A map of one width runs the same arithmetic as the uniform kernel of
    that width (power-of-two bookkeeping only), so dx is identical."""
    N, K = 1024, 2048
    group = 128 if bits == 4 else 64
    W = synth.normal((N, K), 0.02, seed=bits, dtype="f16", device=DEV)
    bit_map = np.full(N // 128, bits, dtype=np.uint8)
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map)
    dy = synth.activations(M, N, seed=M, device=DEV)
    dxm = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bit_map_dev=bm)
    pku, scu, zeu = bq.bq_quantize(W, bits, group, "interleaved")
    dxu = bq.bq_linear_grad_input(dy, pku, scu, zeu, K, bits, group)
    assert bq.bq_device_status() == bq.BQ_OK
    assert torch.equal(dxm, dxu)


def test_grad_mixed_llama_sized_sampled():
    """Channel-mix on the 14336x4096 gate (dx of the down projection's input
    side shape) at M = 4, sampled input columns against the oracle."""
    N, K, M = 14336, 4096, 4
    bit_map = synth.channel_mix_map(N, seed=77)
    W = synth.normal((N, K), 0.02, seed=78, dtype="f16", device=DEV)
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map)
    dy = synth.activations(M, N, seed=79, device=DEV)
    dx = bq.bq_linear_grad_input(dy, pk, sc, ze, K, bit_map_dev=bm)
    assert bq.bq_device_status() == bq.BQ_OK
    cols = np.array([0, 1, 127, 128, 1000, 2049, 4095])
    _, _, _, blocks = O.quantize_mixed(synth.bits16(W), "f16", bit_map, "interleaved", threads=8)
    dyf = O.decode_f64(synth.bits16(dy), "bf16")
    ref = np.zeros((M, cols.size))
    for i, ((c, s, z), b) in enumerate(zip(blocks, bit_map)):
        deq = O.dequant_f64(c, s, z, O.GROUP_OF_BITS[int(b)])   # the block's weights, [128, K]
        ref += dyf[:, 128 * i:128 * (i + 1)] @ deq[:, cols]
    check(dx[:, torch.as_tensor(cols, device=DEV)], ref, torch.bfloat16)
