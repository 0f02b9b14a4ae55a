"""GPU parity of the quantizer and dequantizer with the CPU oracle: packed
codes, scales and zeros bit-exact, on the workloads' shapes and distributions
and on edge cases.  Every call goes through the C ABI (libbq.so)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import oracle as O
from quantized_gemm_group_b200 import bq, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def oracle_quant(W: torch.Tensor, bits, group, layout, threads=8):
    """Oracle codes packed in `layout`, scales / zeros in the layout's metadata order."""
    wt = "f16" if W.dtype == torch.float16 else "bf16"
    codes, scales, zeros = O.quantize(synth.bits16(W), wt, bits, group, threads=threads)
    ms, mz = O.pack_meta(scales, zeros, layout)
    return O.pack(codes, bits, layout), ms, mz, codes, scales, zeros


def gpu_quant(W, bits, group, layout):
    pk, sc, ze = bq.bq_quantize(W, bits, group, layout)
    assert bq.bq_device_status() == bq.BQ_OK
    return pk.cpu().numpy(), sc.cpu().numpy().reshape(-1), ze.cpu().numpy().reshape(-1)


def assert_same(gpu, ref):
    pk, sc, ze = gpu
    rpk, rsc, rze = ref[:3]
    assert pk.shape == rpk.shape
    assert (sc.view(np.uint32) == rsc.view(np.uint32)).all(), "scales differ"
    assert (ze == rze).all(), "zeros differ"
    if not (pk == rpk).all():
        bad = np.nonzero(pk != rpk)[0]
        raise AssertionError(f"{bad.size} packed bytes differ, first at {bad[:8]}")


# --------------------------------------------------------------------------
# config 1 and distributions of the workloads
# --------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["interleaved", "canonical"])
def test_config1_int4_g128(layout):
    W = synth.normal((1024, 1024), 0.02, seed=0, dtype="f16", device=DEV)
    assert_same(gpu_quant(W, 4, 128, layout), oracle_quant(W, 4, 128, layout))


@pytest.mark.parametrize("layout", ["interleaved", "canonical"])
def test_int2_g64_heavy_tailed_outliers(layout):
    W = synth.student_t4((512, 4096), 0.02, seed=3, dtype="f16", device=DEV, outlier_frac=0.001)
    assert_same(gpu_quant(W, 2, 64, layout), oracle_quant(W, 2, 64, layout))


@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
@pytest.mark.parametrize("layout", ["interleaved", "canonical"])
def test_bf16_weights(bits, group, layout):
    W = synth.normal((256, 2048), 0.015, seed=11, dtype="bf16", device=DEV)
    assert_same(gpu_quant(W, bits, group, layout), oracle_quant(W, bits, group, layout))


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("group", [16, 32, 64, 128, 256])
def test_tiled_groups(bits, group):
    W = synth.normal((48, 768), 0.02, seed=group + bits, dtype="f16", device=DEV)
    assert_same(gpu_quant(W, bits, group, "interleaved"), oracle_quant(W, bits, group, "interleaved"))


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("group", [8, 16, 32, 64, 128, 256])
def test_canonical_groups(bits, group):
    W = synth.normal((7, 1024), 0.02, seed=group * 3 + bits, dtype="f16", device=DEV)
    assert_same(gpu_quant(W, bits, group, "canonical"), oracle_quant(W, bits, group, "canonical"))


@pytest.mark.parametrize("shape", [(16, 128), (32, 256), (16, 3072), (1, 256), (3, 512)])
def test_small_and_ragged_shapes(shape):
    W = synth.normal(shape, 0.02, seed=sum(shape), dtype="f16", device=DEV)
    if shape[0] % 16 == 0:
        assert_same(gpu_quant(W, 4, 128, "interleaved"), oracle_quant(W, 4, 128, "interleaved"))
        assert_same(gpu_quant(W, 2, 64, "interleaved"), oracle_quant(W, 2, 64, "interleaved"))
    assert_same(gpu_quant(W, 4, 128, "canonical"), oracle_quant(W, 4, 128, "canonical"))
    assert_same(gpu_quant(W, 2, 64, "canonical"), oracle_quant(W, 2, 64, "canonical"))


def special_matrix(dtype):
    """Rows of special groups: all zero, constants, one-signed, subnormals,
    the fp16 extremes, exact ties, +-0, a single non-zero."""
    rng = np.random.default_rng(5)
    K = 256
    rows = []
    rows.append(np.zeros(K))
    rows.append(np.full(K, 0.75))
    rows.append(np.full(K, -3.0))
    rows.append(np.abs(rng.normal(0, 1, K)) + 0.5)
    rows.append(-np.abs(rng.normal(0, 1, K)) - 0.5)
    rows.append(rng.integers(-4, 5, K) * 2.0 ** -24)                      # fp16 subnormals
    rows.append(np.where(rng.random(K) < 0.5, 65504.0, -65504.0))          # fp16 extremes
    rows.append(rng.integers(-16, 17, K) * 0.25)                           # dyadic: ties
    r = np.zeros(K); r[5] = 1e-3; rows.append(r)                           # single non-zero
    r = -np.zeros(K); r[::2] = 0.0; rows.append(r)                         # +-0
    rows.append(rng.normal(0, 1e-6, K))                                    # tiny values
    rows.append(np.tile([-7.5, 7.5, 0, 1], K // 4))                        # the clamp case
    while len(rows) < 16:
        rows.append(rng.standard_t(2, K))
    W = np.stack(rows)
    if dtype == torch.bfloat16:
        W[6] = np.where(W[6] > 0, 3.0e38, -1.0e30)                          # bf16: huge but finite range
    return torch.tensor(W, dtype=torch.float32).to(dtype).to(DEV)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64), (4, 32)])
@pytest.mark.parametrize("layout", ["interleaved", "canonical"])
def test_special_groups(dtype, bits, group, layout):
    W = special_matrix(dtype)
    assert_same(gpu_quant(W, bits, group, layout), oracle_quant(W, bits, group, layout))


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
@pytest.mark.parametrize("layout", ["interleaved", "canonical"])
def test_nonfinite_sets_status(bad, layout):
    W = synth.normal((32, 256), 0.02, seed=1, dtype="f16", device=DEV)
    W[17, 99] = bad
    bq.bq_quantize(W, 4, 128, layout)
    assert bq.bq_device_status() == bq.BQ_ERR_NONFINITE
    assert bq.bq_device_status() == bq.BQ_OK          # cleared by the read
    # the other rows are still exact
    ref = oracle_quant(W[:16].contiguous(), 4, 128, layout)
    got = gpu_quant(W[:16].contiguous(), 4, 128, layout)
    assert_same(got, ref)


def test_bf16_scale_overflow_sets_status():
    W = torch.zeros((16, 128), dtype=torch.bfloat16, device=DEV)
    W[3, 0] = 3.0e38
    W[3, 1] = -3.0e38
    bq.bq_quantize(W, 4, 128, "interleaved")
    assert bq.bq_device_status() == bq.BQ_ERR_NONFINITE


# --------------------------------------------------------------------------
# full-size shapes, sampled 16-row blocks (rows quantize independently)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("shape,bits,dist", [
    ((14336, 4096), 4, "normal"),
    ((4096, 14336), 2, "t4"),
    ((8192, 49152), 4, "normal015"),
])
def test_full_size_sampled_blocks(shape, bits, dist):
    N, K = shape
    group = 128 if bits == 4 else 64
    if dist == "normal":
        W = synth.normal(shape, 0.02, seed=7, dtype="f16", device=DEV)
    elif dist == "normal015":
        W = synth.normal(shape, 0.015, seed=9, dtype="f16", device=DEV)
    else:
        W = synth.student_t4(shape, 0.02, seed=8, dtype="f16", device=DEV, outlier_frac=0.001)
    pk, sc, ze = bq.bq_quantize(W, bits, group, "interleaved")
    assert bq.bq_device_status() == bq.BQ_OK
    # a 128-row block is contiguous in the interleaved layout (codes and metadata)
    blk_bytes = 128 * K * bits // 8
    G = K // group
    rng = np.random.default_rng(N + K)
    for b in sorted(set([0, N // 128 - 1] + rng.integers(0, N // 128, 3).tolist())):
        Wb = W[b * 128:(b + 1) * 128].contiguous()
        rpk, rsc, rze = oracle_quant(Wb, bits, group, "interleaved")[:3]
        got = (pk[b * blk_bytes:(b + 1) * blk_bytes].cpu().numpy(),
               sc[b * 128 * G:(b + 1) * 128 * G].cpu().numpy(), ze[b * 128 * G:(b + 1) * 128 * G].cpu().numpy())
        assert_same(got, (rpk, rsc, rze))
    del W, pk, sc, ze
    torch.cuda.empty_cache()


# --------------------------------------------------------------------------
# mixed precision (Layer-mix / Channel-mix maps)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["interleaved", "canonical"])
def test_channel_mix_quantize(layout):
    N, K = 1024, 1024
    W = synth.normal((N, K), 0.02, seed=21, dtype="f16", device=DEV)
    bit_map = synth.channel_mix_map(N, seed=5)
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map, layout)
    assert bq.bq_device_status() == bq.BQ_OK
    rpk, rsc, rze, _ = O.quantize_mixed(synth.bits16(W), "f16", bit_map, layout, threads=8)
    assert (pk.cpu().numpy() == rpk).all()
    assert (sc.cpu().numpy().view(np.uint32) == rsc.view(np.uint32)).all()
    assert (ze.cpu().numpy() == rze).all()


def test_mixed_bad_map_sets_status():
    W = synth.normal((256, 256), 0.02, seed=2, dtype="f16", device=DEV)
    bq.bq_quantize_mixed(W, [4, 2], "interleaved")
    assert bq.bq_device_status() == bq.BQ_OK
    bm = torch.tensor([4, 3], dtype=torch.uint8, device=DEV)
    pk = torch.empty(256 * 256 // 2, dtype=torch.uint8, device=DEV)
    sc = torch.empty(256 * 4, dtype=torch.float32, device=DEV)
    ze = torch.empty(256 * 4, dtype=torch.uint8, device=DEV)
    st = bq.lib().bq_quantize_mixed(bq._ptr(W), bq.BQ_F16, 256, 256, bq._ptr(bm), 1, bq._ptr(pk),
                                    bq._ptr(sc), bq._ptr(ze), bq._stream())
    assert st == bq.BQ_OK
    assert bq.bq_device_status() == bq.BQ_ERR_UNSUPPORTED


# --------------------------------------------------------------------------
# dequantize
# --------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["interleaved", "canonical"])
@pytest.mark.parametrize("bits,group", [(4, 128), (2, 64)])
def test_dequantize_f32_bit_exact(layout, bits, group):
    W = synth.normal((64, 1024), 0.02, seed=4, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, bits, group, layout)
    got = bq.bq_dequantize(pk, sc, ze, 64, 1024, bits, group, layout, torch.float32).cpu().numpy()
    codes, rsc, rze = oracle_quant(W, bits, group, layout)[3:]
    ref = O.dequant_f32(codes, rsc, rze, group)
    assert (got.view(np.uint32) == ref.view(np.uint32)).all()
    # 16-bit outputs: the fp32 value rounded once
    for dt in (torch.float16, torch.bfloat16):
        got16 = bq.bq_dequantize(pk, sc, ze, 64, 1024, bits, group, layout, dt).cpu()
        assert torch.equal(got16, torch.from_numpy(ref).to(dt))


@pytest.mark.parametrize("layout", ["interleaved", "canonical"])
def test_dequantize_mixed(layout):
    N, K = 512, 512
    W = synth.normal((N, K), 0.02, seed=6, dtype="f16", device=DEV)
    bit_map = [4, 2, 2, 4]
    pk, sc, ze, bm = bq.bq_quantize_mixed(W, bit_map, layout)
    got = bq.bq_dequantize(pk, sc, ze, N, K, layout=layout, out_dtype=torch.float32, bit_map_dev=bm).cpu().numpy()
    _, _, _, blocks = O.quantize_mixed(synth.bits16(W), "f16", bit_map, layout)
    ref = np.concatenate([O.dequant_f32(c, s, z, O.GROUP_OF_BITS[b]) for (c, s, z), b in zip(blocks, bit_map)])
    assert (got.view(np.uint32) == ref.view(np.uint32)).all()
