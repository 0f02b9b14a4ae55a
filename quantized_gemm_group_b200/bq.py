"""Thin Python binding of the C ABI in ``include/bq.h`` (``libbq.so``).

Argument marshalling only: every step of the quantizer and the linear layer
runs in the library's CUDA kernels.  Tensors are torch CUDA tensors used as
plain device buffers; outputs are allocated here with torch and their
pointers passed down.  There is no fallback: if the library is missing or a
call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

LIB_PATH = _build.LIB

# enums, mirrored from include/bq.h
BQ_OK, BQ_ERR_NULL, BQ_ERR_SHAPE, BQ_ERR_ALIGN, BQ_ERR_UNSUPPORTED = 0, 1, 2, 3, 4
BQ_ERR_WORKSPACE, BQ_ERR_NONFINITE, BQ_ERR_TIMEOUT, BQ_ERR_CUDA = 5, 6, 7, 8
BQ_F16, BQ_BF16, BQ_F32 = 0, 1, 2
BQ_LAYOUT_CANONICAL, BQ_LAYOUT_INTERLEAVED = 0, 1

LAYOUTS = {"canonical": BQ_LAYOUT_CANONICAL, "interleaved": BQ_LAYOUT_INTERLEAVED}
DTYPE_CODE = {torch.float16: BQ_F16, torch.bfloat16: BQ_BF16, torch.float32: BQ_F32}
CODE_DTYPE = {v: k for k, v in DTYPE_CODE.items()}
GROUP_OF_BITS = {4: 128, 2: 64}

#: every symbol include/bq.h declares
EXPORTS = (
    "bq_packed_bytes", "bq_group_count", "bq_mixed_offsets", "bq_quantize", "bq_quantize_symmetric",
    "bq_quantize_mixed",
    "bq_dequantize", "bq_fake_quantize", "bq_linear", "bq_linear_grad_input", "bq_check_division",
    "bq_check_const_division", "bq_quantize_f16s", "bq_linear_f16s", "bq_linear_workspace_bytes", "bq_linear_ws",
    "bq_selftest_bounded_wait", "bq_set_option", "bq_get_option", "bq_device_status",
    "bq_status_string", "bq_version",
)
BQ_OPT_LINEAR_OVERLAP = 0


class BQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)}")


_lib = None


def lib(path: str | None = None):
    """Load libbq.so (raises if it is missing; build it with build.build())."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise FileNotFoundError(f"{p} is missing: build the CUDA library first "
                                "(python -m quantized_gemm_group_b200.build)")
    L = ctypes.CDLL(p)
    i64, i32, vp, u8p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p
    L.bq_packed_bytes.argtypes = [i64, i64, i32]
    L.bq_packed_bytes.restype = ctypes.c_size_t
    L.bq_group_count.argtypes = [i64, i64, i32]
    L.bq_group_count.restype = ctypes.c_size_t
    L.bq_mixed_offsets.argtypes = [u8p, i64, i64, vp, vp]
    L.bq_mixed_offsets.restype = i32
    L.bq_quantize.argtypes = [vp, i32, i64, i64, i32, i32, i32, vp, vp, vp, vp]
    L.bq_quantize.restype = i32
    L.bq_quantize_symmetric.argtypes = [vp, i32, i64, i64, i32, i32, i32, vp, vp, vp, vp]
    L.bq_quantize_symmetric.restype = i32
    L.bq_quantize_f16s.argtypes = [vp, i32, i64, i64, i32, i32, i32, vp, vp, vp, vp]
    L.bq_quantize_f16s.restype = i32
    L.bq_quantize_mixed.argtypes = [vp, i32, i64, i64, vp, i32, vp, vp, vp, vp]
    L.bq_quantize_mixed.restype = i32
    L.bq_dequantize.argtypes = [vp, vp, vp, vp, i32, i32, i64, i64, i32, vp, i32, vp]
    L.bq_dequantize.restype = i32
    L.bq_fake_quantize.argtypes = [vp, i32, i64, i64, i32, i32, vp, i32, vp]
    L.bq_fake_quantize.restype = i32
    L.bq_linear.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp, i32, i32, i64, i32, vp, vp]
    L.bq_linear.restype = i32
    L.bq_linear_f16s.argtypes = [vp, i32, i64, i64, vp, vp, vp, i32, i32, i64, i32, vp, vp]
    L.bq_linear_f16s.restype = i32
    L.bq_linear_workspace_bytes.argtypes = [i64, i64, i64, i32, i32]
    L.bq_linear_workspace_bytes.restype = ctypes.c_size_t
    L.bq_linear_ws.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp, i32, i32, i64, i32, vp, vp, ctypes.c_size_t, vp]
    L.bq_linear_ws.restype = i32
    L.bq_linear_grad_input.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp, i32, i32, i64, i32, vp, vp]
    L.bq_linear_grad_input.restype = i32
    L.bq_check_division.argtypes = [ctypes.c_uint32, ctypes.c_uint32, i32, vp, vp]
    L.bq_check_division.restype = i32
    L.bq_check_const_division.argtypes = [i32, ctypes.c_uint32, ctypes.c_uint32, vp, vp]
    L.bq_check_const_division.restype = i32
    L.bq_selftest_bounded_wait.argtypes = [ctypes.c_uint32, vp]
    L.bq_selftest_bounded_wait.restype = i32
    L.bq_set_option.argtypes = [i32, i32]
    L.bq_set_option.restype = i32
    L.bq_get_option.argtypes = [i32]
    L.bq_get_option.restype = i32
    L.bq_device_status.argtypes = [vp]
    L.bq_device_status.restype = i32
    L.bq_status_string.argtypes = [i32]
    L.bq_status_string.restype = ctypes.c_char_p
    L.bq_version.argtypes = []
    L.bq_version.restype = ctypes.c_char_p
    if path is None:
        _lib = L
    return L


def status_string(status: int) -> str:
    return lib().bq_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != BQ_OK:
        raise BQError(fn, status)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------------------
# size queries
# ---------------------------------------------------------------------------

def bq_packed_bytes(rows: int, cols: int, bits: int) -> int:
    return int(lib().bq_packed_bytes(rows, cols, bits))


def bq_group_count(rows: int, cols: int, group: int) -> int:
    return int(lib().bq_group_count(rows, cols, group))


def bq_mixed_offsets(bit_map, rows: int, cols: int):
    bm = np.ascontiguousarray(np.asarray(bit_map, dtype=np.uint8))
    nb = rows // 128
    co = np.zeros(nb + 1, dtype=np.int64)
    go = np.zeros(nb + 1, dtype=np.int64)
    _check("bq_mixed_offsets", lib().bq_mixed_offsets(bm.ctypes.data_as(ctypes.c_void_p), rows, cols,
                                                      co.ctypes.data_as(ctypes.c_void_p),
                                                      go.ctypes.data_as(ctypes.c_void_p)))
    return co, go


# ---------------------------------------------------------------------------
# quantize / dequantize / linear
# ---------------------------------------------------------------------------

def bq_quantize(W: torch.Tensor, bits: int, group: int | None = None, layout: str = "interleaved",
                out=None, stream=None, scheme: str = "asymmetric"):
    """Quantize W [N, K] (fp16/bf16, CUDA) with the asymmetric MinMax scheme (default), the
    symmetric abs-max one, or the MinMax scheme with binary16 scales ("asymmetric_f16_scale").
    Returns (packed u8, scales, zeros u8): scales f32 (f16 for the binary16 format) / zeros are
    [N, K/g] in the canonical layout and flat (128-row-block-major order) in the interleaved one."""
    group = group or GROUP_OF_BITS[bits]
    N, K = W.shape
    s16 = scheme == "asymmetric_f16_scale"
    if out is None:
        packed = torch.empty(max(1, bq_packed_bytes(N, K, bits)), dtype=torch.uint8, device=W.device)
        mshape = (N, K // group) if layout == "canonical" else (N * (K // group),)
        scales = torch.empty(mshape, dtype=torch.float16 if s16 else torch.float32, device=W.device)
        zeros = torch.empty(mshape, dtype=torch.uint8, device=W.device)
    else:
        packed, scales, zeros = out
    fn = {"symmetric": lib().bq_quantize_symmetric, "asymmetric_f16_scale": lib().bq_quantize_f16s,
          "asymmetric": lib().bq_quantize}[scheme]
    st = fn(_ptr(W), DTYPE_CODE[W.dtype], N, K, bits, group, LAYOUTS[layout],
            _ptr(packed), _ptr(scales), _ptr(zeros), _stream(stream))
    _check("bq_quantize", st)
    return packed, scales, zeros


def mixed_sizes(bit_map, rows: int, cols: int):
    co, go = bq_mixed_offsets(bit_map, rows, cols)
    return int(co[-1]), int(go[-1])


def bq_quantize_mixed(W: torch.Tensor, bit_map, layout: str = "interleaved", stream=None):
    """Per-128-row-block width (4 -> group 128, 2 -> group 64).  bit_map: host sequence.
    Returns (packed, scales, zeros, bit_map_dev)."""
    N, K = W.shape
    code_bytes, groups = mixed_sizes(bit_map, N, K)
    bm = torch.as_tensor(np.asarray(bit_map, dtype=np.uint8)).to(W.device)
    packed = torch.empty(max(1, code_bytes), dtype=torch.uint8, device=W.device)
    scales = torch.empty(max(1, groups), dtype=torch.float32, device=W.device)
    zeros = torch.empty(max(1, groups), dtype=torch.uint8, device=W.device)
    st = lib().bq_quantize_mixed(_ptr(W), DTYPE_CODE[W.dtype], N, K, _ptr(bm), LAYOUTS[layout],
                                 _ptr(packed), _ptr(scales), _ptr(zeros), _stream(stream))
    _check("bq_quantize_mixed", st)
    return packed, scales, zeros, bm


def bq_dequantize(packed, scales, zeros, rows: int, cols: int, bits: int = 4, group: int | None = None,
                  layout: str = "interleaved", out_dtype=torch.float32, bit_map_dev=None, stream=None):
    group = group or GROUP_OF_BITS.get(bits, 0)
    out = torch.empty((rows, cols), dtype=out_dtype, device=packed.device)
    st = lib().bq_dequantize(_ptr(packed), _ptr(scales), _ptr(zeros), _ptr(bit_map_dev), bits, group,
                             rows, cols, LAYOUTS[layout], _ptr(out), DTYPE_CODE[out_dtype], _stream(stream))
    _check("bq_dequantize", st)
    return out


def bq_fake_quantize(W: torch.Tensor, bits: int, group: int | None = None, out_dtype=None, out=None, stream=None):
    """dequant(quant(W)) in one pass (codes, scales, zeros not stored); out in W's dtype by default."""
    group = group or GROUP_OF_BITS[bits]
    N, K = W.shape
    o = out if out is not None else torch.empty((N, K), dtype=out_dtype or W.dtype, device=W.device)
    st = lib().bq_fake_quantize(_ptr(W), DTYPE_CODE[W.dtype], N, K, bits, group, _ptr(o), DTYPE_CODE[o.dtype],
                                _stream(stream))
    _check("bq_fake_quantize", st)
    return o


def bq_linear_workspace_bytes(M: int, N: int, K: int, bits: int = 4, mixed: bool = False) -> int:
    """Device workspace bytes that let bq_linear(..., workspace=...) split K (0: no split)."""
    return int(lib().bq_linear_workspace_bytes(M, N, K, bits, 1 if mixed else 0))


def bq_linear(x: torch.Tensor, packed, scales, zeros, N: int, bits: int = 4, group: int | None = None,
              bit_map_dev=None, layout: str = "interleaved", out=None, stream=None, workspace=None):
    """y [M, N] = x [M, K] . dequant(W)^T, y in x's dtype.  fp16 `scales` (from the binary16
    scale format) select bq_linear_f16s; a device `workspace` (uint8, from
    bq_linear_workspace_bytes) selects bq_linear_ws."""
    group = group or GROUP_OF_BITS.get(bits, 0)
    M, K = x.shape
    y = out if out is not None else torch.empty((M, N), dtype=x.dtype, device=x.device)
    if scales.dtype == torch.float16:
        if bit_map_dev is not None:
            raise ValueError("binary16 scales take no width map")
        st = lib().bq_linear_f16s(_ptr(x), DTYPE_CODE[x.dtype], M, K, _ptr(packed), _ptr(scales), _ptr(zeros),
                                  bits, group, N, LAYOUTS[layout], _ptr(y), _stream(stream))
        _check("bq_linear_f16s", st)
        return y
    if workspace is not None:
        st = lib().bq_linear_ws(_ptr(x), DTYPE_CODE[x.dtype], M, K, _ptr(packed), _ptr(scales), _ptr(zeros),
                                _ptr(bit_map_dev), bits, group, N, LAYOUTS[layout], _ptr(y), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream))
        _check("bq_linear_ws", st)
        return y
    st = lib().bq_linear(_ptr(x), DTYPE_CODE[x.dtype], M, K, _ptr(packed), _ptr(scales), _ptr(zeros),
                         _ptr(bit_map_dev), bits, group, N, LAYOUTS[layout], _ptr(y), _stream(stream))
    _check("bq_linear", st)
    return y


def bq_linear_grad_input(dy: torch.Tensor, packed, scales, zeros, K: int, bits: int = 4, group: int | None = None,
                         layout: str = "interleaved", out=None, stream=None, bit_map_dev=None):
    """dx [M, K] = dy [M, N] . dequant(W), dx in dy's dtype (the input
    gradient of bq_linear); bit_map_dev: a width map's device copy, as for bq_linear."""
    group = group or GROUP_OF_BITS.get(bits, 0)
    M, N = dy.shape
    dx = out if out is not None else torch.empty((M, K), dtype=dy.dtype, device=dy.device)
    st = lib().bq_linear_grad_input(_ptr(dy), DTYPE_CODE[dy.dtype], M, N, _ptr(packed), _ptr(scales), _ptr(zeros),
                                    _ptr(bit_map_dev), bits, group, K, LAYOUTS[layout], _ptr(dx), _stream(stream))
    _check("bq_linear_grad_input", st)
    return dx


def bq_check_division(s_bits_begin: int, s_bits_end: int, refinements: int = 2, stream=None):
    """Returns (mismatches, pairs checked, first bad divisor bits, first bad fp16 numerator bits)."""
    res = torch.zeros(4, dtype=torch.int64, device="cuda")
    _check("bq_check_division", lib().bq_check_division(s_bits_begin, s_bits_end, refinements, _ptr(res),
                                                        _stream(stream)))
    torch.cuda.synchronize()
    return tuple(int(v) for v in res.cpu())


def bq_check_const_division(divisor: int, x_bits_begin: int, x_bits_end: int, stream=None):
    """Returns (mismatches, values checked, first bad x bits, its divisor)."""
    res = torch.zeros(4, dtype=torch.int64, device="cuda")
    _check("bq_check_const_division", lib().bq_check_const_division(divisor, x_bits_begin, x_bits_end, _ptr(res),
                                                                    _stream(stream)))
    torch.cuda.synchronize()
    return tuple(int(v) for v in res.cpu())


def bq_selftest_bounded_wait(limit: int, stream=None):
    _check("bq_selftest_bounded_wait", lib().bq_selftest_bounded_wait(limit, _stream(stream)))


def bq_set_option(option: int, value: int):
    _check("bq_set_option", lib().bq_set_option(option, value))


def bq_get_option(option: int) -> int:
    return int(lib().bq_get_option(option))


def bq_device_status(stream=None) -> int:
    return int(lib().bq_device_status(_stream(stream)))


def bq_version() -> str:
    return lib().bq_version().decode()


# ---------------------------------------------------------------------------
# host-buffer path (end-to-end: pinned host in, host out, through the C ABI)
# ---------------------------------------------------------------------------

def bq_linear_host(x_host: torch.Tensor, packed, scales, zeros, N: int, bits: int = 4, group=None,
                   bit_map_dev=None, x_dev=None, y_dev=None, y_host=None, stream=None):
    """Copy x from (pinned) host memory, run bq_linear, copy y back to host."""
    s = stream or torch.cuda.current_stream()
    if x_dev is None:
        x_dev = torch.empty(x_host.shape, dtype=x_host.dtype, device="cuda")
    x_dev.copy_(x_host, non_blocking=True)
    y_dev = bq_linear(x_dev, packed, scales, zeros, N, bits, group, bit_map_dev, out=y_dev, stream=s)
    if y_host is None:
        y_host = torch.empty(y_dev.shape, dtype=y_dev.dtype, pin_memory=True)
    y_host.copy_(y_dev, non_blocking=True)
    return y_host
