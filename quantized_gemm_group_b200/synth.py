"""Seeded synthetic inputs for tests and benchmarks.

This module holds no quantization or linear-layer arithmetic: it only draws
random tensors with the shapes and distributions of the workloads (normal
weights, heavy-tailed Student-t weights with outlier input channels, normal
activations, Layer-mix / Channel-mix width maps).  Both the CUDA path's tests
and the CPU oracle's tests take their inputs from here.

Every draw comes from a ``torch.Generator`` seeded explicitly, on the device
the tensor is made on.  A tensor drawn on the GPU is copied to the host
before the oracle sees it, so both sides always see identical bits.
"""
from __future__ import annotations

import math

import numpy as np
import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std: float, seed: int, dtype: str = "f16", device="cpu",
           chunk_rows: int = 4096) -> torch.Tensor:
    """N(0, std^2) drawn in fp32, scaled, then rounded to fp16/bf16 (nearest-even).

    Large matrices are drawn in row chunks to bound the fp32 temporary."""
    shape = tuple(int(s) for s in shape)
    g = _gen(seed, device)
    out = torch.empty(shape, dtype=DTYPES[dtype], device=device)
    if len(shape) == 1 or shape[0] <= chunk_rows:
        out.copy_(torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(std))
        return out
    for r in range(0, shape[0], chunk_rows):
        rows = min(chunk_rows, shape[0] - r)
        t = torch.randn((rows,) + shape[1:], generator=g, device=device, dtype=torch.float32)
        out[r:r + rows].copy_(t.mul_(std))
    return out


def outlier_columns(cols: int, seed: int, frac: float = 0.001, device="cpu") -> torch.Tensor:
    """A seeded choice of floor(frac * cols) distinct input channels."""
    n = int(math.floor(frac * cols))
    g = _gen(seed, device)
    return torch.randperm(cols, generator=g, device=device)[:n].sort().values


def student_t4(shape, std: float, seed: int, dtype: str = "f16", device="cpu",
               outlier_frac: float = 0.0, outlier_gain: float = 10.0,
               chunk_rows: int = 2048) -> torch.Tensor:
    """Student-t with nu = 4, scaled to standard deviation `std`.

    t = Z / sqrt(V / 4) with V ~ chi^2_4 = 2 (E1 + E2), E = -ln U, so
    t = Z / sqrt((E1 + E2) / 2).  The standard deviation of t_4 is sqrt(2), so
    t is multiplied by std / sqrt(2).  Optionally floor(outlier_frac * cols)
    seeded input columns are multiplied by `outlier_gain` (in fp32, before the
    final rounding)."""
    shape = tuple(int(s) for s in shape)
    rows, cols = shape
    g = _gen(seed, device)
    out = torch.empty(shape, dtype=DTYPES[dtype], device=device)
    gain = None
    if outlier_frac > 0:
        idx = outlier_columns(cols, seed + 7919, outlier_frac, device=device)
        gain = torch.ones(cols, dtype=torch.float32, device=device)
        gain[idx] = outlier_gain
    scale = std / math.sqrt(2.0)
    for r in range(0, rows, chunk_rows):
        n = min(chunk_rows, rows - r)
        z = torch.randn((n, cols), generator=g, device=device, dtype=torch.float32)
        u1 = 1.0 - torch.rand((n, cols), generator=g, device=device, dtype=torch.float32)
        u2 = 1.0 - torch.rand((n, cols), generator=g, device=device, dtype=torch.float32)
        v_half = (-(torch.log(u1) + torch.log(u2))) * 0.5
        t = z / torch.sqrt(v_half) * scale
        if gain is not None:
            t *= gain
        out[r:r + n].copy_(t)
        del z, u1, u2, v_half, t
    return out


def activations(M: int, K: int, seed: int, dtype: str = "bf16", device="cpu") -> torch.Tensor:
    """x ~ N(0, 1), [M, K]."""
    return normal((M, K), 1.0, seed, dtype, device)


def bits16(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of an fp16/bf16 tensor, on the host."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------
# Llama-3-8B-shaped decode stack and the Qwen1.5-110B-shaped prefill shapes
# --------------------------------------------------------------------------

#: (name, rows N = output channels, cols K = input channels) of one layer
LLAMA3_8B_LINEARS = (
    ("q", 4096, 4096),
    ("k", 1024, 4096),
    ("v", 1024, 4096),
    ("o", 4096, 4096),
    ("gate", 14336, 4096),
    ("up", 14336, 4096),
    ("down", 4096, 14336),
)
LLAMA3_8B_LAYERS = 32
# Projections that read the same input, run as one linear over their weights
# concatenated along N (indices into LLAMA3_8B_LINEARS).
LLAMA3_8B_FUSED = (
    ("qkv", (0, 1, 2)),
    ("o", (3,)),
    ("gate_up", (4, 5)),
    ("down", (6,)),
)

PREFILL_SHAPES = ((14336, 4096), (4096, 14336), (49152, 8192), (8192, 49152))


def weight_seed(layer: int, module: int) -> int:
    return 1000 * layer + module


def layer_mix_map(layers: int = LLAMA3_8B_LAYERS, int4_layers: int = 8, seed: int = 4242):
    """Layer-mix: a seeded choice of `int4_layers` layers at 4 bits, the rest at 2 bits.
    Returns a list of widths per layer."""
    g = _gen(seed, "cpu")
    pick = set(torch.randperm(layers, generator=g)[:int4_layers].tolist())
    return [4 if l in pick else 2 for l in range(layers)]


def channel_mix_map(rows: int, seed: int, int4_frac: float = 0.25, block: int = 128):
    """Channel-mix: a seeded 25% of the 128-row output blocks of one matrix at 4 bits."""
    nb = rows // block
    n4 = int(round(int4_frac * nb))
    g = _gen(seed, "cpu")
    pick = set(torch.randperm(nb, generator=g)[:n4].tolist())
    return np.array([4 if i in pick else 2 for i in range(nb)], dtype=np.uint8)
