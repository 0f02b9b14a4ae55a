"""Python access to the CPU oracle (``bq_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  The product package never
imports it and has no fallback to it.

The C file holds all of the method's arithmetic; this module only marshals
numpy arrays, splits rows across threads, and assembles mixed-precision
matrices block by block.  Page citations for each step are in the C file's
header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bq_oracle.c")
_SO = os.path.join(_HERE, "_build", "libbq_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/libbq_oracle.so`` with gcc."""
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            L = ctypes.CDLL(path)
            i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
            L.bqo_f16_to_f32.argtypes = [ctypes.c_uint16]
            L.bqo_f16_to_f32.restype = ctypes.c_float
            L.bqo_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.bqo_bf16_to_f32.restype = ctypes.c_float
            L.bqo_quantize_group.argtypes = [vp, i32, i32, vp, vp, vp]
            L.bqo_quantize_group.restype = i32
            L.bqo_quantize.argtypes = [vp, i32, i64, i64, i32, i32, i64, i64, vp, vp, vp]
            L.bqo_quantize.restype = i32
            L.bqo_quantize_scheme.argtypes = [vp, i32, i64, i64, i32, i32, i32, i64, i64, vp, vp, vp]
            L.bqo_quantize_scheme.restype = i32
            L.bqo_quantize_group_sym.argtypes = [vp, i32, i32, vp, vp, vp]
            L.bqo_quantize_group_sym.restype = i32
            L.bqo_quantize_group_s16.argtypes = [vp, i32, i32, vp, vp, vp]
            L.bqo_quantize_group_s16.restype = i32
            L.bqo_f32_to_f16.argtypes = [ctypes.c_float]
            L.bqo_f32_to_f16.restype = ctypes.c_uint16
            L.bqo_code_position.argtypes = [i32, i64, i64, i64, i64, i32, vp, vp]
            L.bqo_code_position.restype = None
            L.bqo_pack.argtypes = [vp, i64, i64, i32, i32, vp]
            L.bqo_pack.restype = i32
            L.bqo_unpack.argtypes = [vp, i64, i64, i32, i32, vp]
            L.bqo_unpack.restype = i32
            L.bqo_dequant_f64.argtypes = [vp, vp, vp, i64, i64, i32, i64, i64, vp]
            L.bqo_dequant_f64.restype = None
            L.bqo_dequant_f32.argtypes = [vp, vp, vp, i64, i64, i32, vp]
            L.bqo_dequant_f32.restype = None
            L.bqo_linear_f64.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i64, i64, vp, vp]
            L.bqo_linear_f64.restype = None
            L.bqo_linear_grad_input_f64.argtypes = [vp, i64, i64, vp, vp, vp, i64, i32, i64, i64, vp, vp]
            L.bqo_linear_grad_input_f64.restype = None
            L.bqo_decode_f64.argtypes = [vp, i32, i64, vp]
            L.bqo_decode_f64.restype = None
            L.bqo_meta_index.argtypes = [i32, i64, i64, i64, i64]
            L.bqo_meta_index.restype = i64
            L.bqo_pack_meta_f32.argtypes = [vp, i64, i64, i32, vp]
            L.bqo_pack_meta_f32.restype = None
            L.bqo_pack_meta_u8.argtypes = [vp, i64, i64, i32, vp]
            L.bqo_pack_meta_u8.restype = None
            L.bqo_f64_to_bf16.argtypes = [ctypes.c_double]
            L.bqo_f64_to_bf16.restype = ctypes.c_uint16
            _lib = L
    return _lib


class OracleError(RuntimeError):
    pass


class using_library:
    """Temporarily route every call through another build of the oracle
    (used by the tests that plant mistakes in a copy of the C file)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        lib()
        self._saved = _lib
        with _lock:
            _lib = None
        saved_build = globals()["build"]
        globals()["build"] = lambda force=False: self.path
        try:
            lib()
        finally:
            globals()["build"] = saved_build
        return self

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self._saved
        return False


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


WTYPE = {"f16": 0, "bf16": 1}
LAYOUT = {"canonical": 0, "interleaved": 1}
GROUP_OF_BITS = {4: 128, 2: 64}


def _row_chunks(rows: int, threads: int):
    threads = max(1, min(threads, rows))
    step = (rows + threads - 1) // threads
    return [(r, min(rows, r + step)) for r in range(0, rows, step)]


# ---------------------------------------------------------------------------
# quantizer
# ---------------------------------------------------------------------------

def quantize_group(x: np.ndarray, bits: int, scheme: str = "asymmetric"):
    """One group of fp32 values -> (s, z, q)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    q = np.zeros(x.size, dtype=np.uint8)
    s = ctypes.c_float()
    z = ctypes.c_int()
    fn = {"symmetric": lib().bqo_quantize_group_sym,
          "asymmetric_f16_scale": lib().bqo_quantize_group_s16}.get(scheme, lib().bqo_quantize_group)
    rc = fn(_p(x), x.size, bits, ctypes.byref(s), ctypes.byref(z), _p(q))
    if rc:
        raise OracleError(f"bqo_quantize_group rc={rc}")
    return float(np.float32(s.value)), int(z.value), q


def f32_to_f16_bits(values) -> np.ndarray:
    """binary32 values -> binary16 bit patterns (round to nearest, ties to even)."""
    v = np.ascontiguousarray(values, dtype=np.float32).ravel()
    L = lib()
    return np.array([L.bqo_f32_to_f16(float(a)) for a in v], dtype=np.uint16).reshape(np.shape(values))


SCHEMES = {"asymmetric": 0, "symmetric": 1, "asymmetric_f16_scale": 2}


def quantize(w_bits: np.ndarray, wtype: str, bits: int, group: int, threads: int = 1, scheme: str = "asymmetric"):
    """Quantize W (uint16 bit patterns of fp16/bf16, shape [N, K]) with the
    asymmetric MinMax scheme (default) or the symmetric abs-max scheme.

    Returns unpacked codes u8 [N, K], scales f32 [N, K/group], zeros u8 [N, K/group].
    """
    w_bits = np.ascontiguousarray(w_bits, dtype=np.uint16)
    N, K = w_bits.shape
    if K % group:
        raise OracleError("cols % group != 0")
    G = K // group
    codes = np.empty((N, K), dtype=np.uint8)
    scales = np.empty((N, G), dtype=np.float32)
    zeros = np.empty((N, G), dtype=np.uint8)
    L = lib()

    def run(r):
        return L.bqo_quantize_scheme(_p(w_bits), WTYPE[wtype], N, K, bits, group, SCHEMES[scheme], r[0], r[1],
                                     _p(codes), _p(scales), _p(zeros))

    if threads <= 1:
        rcs = [run((0, N))]
    else:
        with ThreadPoolExecutor(threads) as ex:
            rcs = list(ex.map(run, _row_chunks(N, threads)))
    if any(rcs):
        raise OracleError(f"bqo_quantize rc={max(rcs)}")
    return codes, scales, zeros


# ---------------------------------------------------------------------------
# packing
# ---------------------------------------------------------------------------

def code_position(layout: str, n: int, k: int, rows: int, cols: int, bits: int):
    b = ctypes.c_int64()
    o = ctypes.c_int()
    lib().bqo_code_position(LAYOUT[layout], n, k, rows, cols, bits, ctypes.byref(b), ctypes.byref(o))
    return int(b.value), int(o.value)


def pack(codes: np.ndarray, bits: int, layout: str) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    out = np.empty(N * K * bits // 8, dtype=np.uint8)
    rc = lib().bqo_pack(_p(codes), N, K, bits, LAYOUT[layout], _p(out))
    if rc:
        raise OracleError(f"bqo_pack rc={rc}")
    return out


def unpack(packed: np.ndarray, N: int, K: int, bits: int, layout: str) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    codes = np.empty((N, K), dtype=np.uint8)
    rc = lib().bqo_unpack(_p(packed), N, K, bits, LAYOUT[layout], _p(codes))
    if rc:
        raise OracleError(f"bqo_unpack rc={rc}")
    return codes


def meta_index(layout: str, n: int, g: int, rows: int, G: int) -> int:
    return int(lib().bqo_meta_index(LAYOUT[layout], n, g, rows, G))


def pack_meta(scales: np.ndarray, zeros: np.ndarray, layout: str):
    """Scales / zeros [rows, G] -> the layout's flat storage order."""
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    zeros = np.ascontiguousarray(zeros, dtype=np.uint8)
    rows, G = scales.shape
    s = np.empty(rows * G, dtype=np.float32)
    z = np.empty(rows * G, dtype=np.uint8)
    lib().bqo_pack_meta_f32(_p(scales), rows, G, LAYOUT[layout], _p(s))
    lib().bqo_pack_meta_u8(_p(zeros), rows, G, LAYOUT[layout], _p(z))
    return s, z


# ---------------------------------------------------------------------------
# dequant / linear
# ---------------------------------------------------------------------------

def dequant_f64(codes, scales, zeros, group: int) -> np.ndarray:
    N, K = codes.shape
    out = np.empty((N, K), dtype=np.float64)
    lib().bqo_dequant_f64(_p(codes), _p(scales), _p(zeros), N, K, group, 0, N, _p(out))
    return out


def dequant_f32(codes, scales, zeros, group: int) -> np.ndarray:
    N, K = codes.shape
    out = np.empty((N, K), dtype=np.float32)
    lib().bqo_dequant_f32(_p(codes), _p(scales), _p(zeros), N, K, group, _p(out))
    return out


def decode_f64(bits16: np.ndarray, wtype: str) -> np.ndarray:
    bits16 = np.ascontiguousarray(bits16, dtype=np.uint16)
    out = np.empty(bits16.shape, dtype=np.float64)
    lib().bqo_decode_f64(_p(bits16), WTYPE[wtype], bits16.size, _p(out))
    return out


def linear_f64(x_f64: np.ndarray, codes, scales, zeros, group: int, threads: int = 1) -> np.ndarray:
    """y = x . dequant(W)^T in fp64 (k ascending).  x_f64: [M, K] float64."""
    x_f64 = np.ascontiguousarray(x_f64, dtype=np.float64)
    M, K = x_f64.shape
    N = codes.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    L = lib()

    def run(r):
        scratch = np.empty(K, dtype=np.float64)
        L.bqo_linear_f64(_p(x_f64), M, K, _p(codes), _p(scales), _p(zeros), N, group,
                         r[0], r[1], _p(scratch), _p(y))

    if threads <= 1:
        run((0, N))
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, _row_chunks(N, threads)))
    return y


def linear_grad_input_f64(dy_f64: np.ndarray, codes, scales, zeros, group: int, threads: int = 1) -> np.ndarray:
    """dx = dy . dequant(W) in fp64 (n ascending).  dy_f64: [M, N] float64;
    codes / scales / zeros as returned by quantize (row-major)."""
    dy_f64 = np.ascontiguousarray(dy_f64, dtype=np.float64)
    M, N = dy_f64.shape
    K = codes.shape[1]
    assert codes.shape[0] == N
    dx = np.empty((M, K), dtype=np.float64)
    L = lib()

    def run(c):
        scratch = np.empty(N, dtype=np.float64)
        L.bqo_linear_grad_input_f64(_p(dy_f64), M, N, _p(codes), _p(scales), _p(zeros), K, group,
                                    c[0], c[1], _p(scratch), _p(dx))

    if threads <= 1:
        run((0, K))
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, _row_chunks(K, threads)))
    return dx


def to_bf16_bits(y: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    L = lib()
    flat = np.asarray(y, dtype=np.float64).reshape(-1)
    out = np.fromiter((L.bqo_f64_to_bf16(float(v)) for v in flat), dtype=np.uint16, count=flat.size)
    return out.reshape(np.shape(y))


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return decode_f64(b, "bf16")


# ---------------------------------------------------------------------------
# mixed precision ([GB]: Layer-mix / Channel-mix over 128-row blocks)
# ---------------------------------------------------------------------------

MIX_BLOCK = 128


def mixed_offsets(bit_map, K: int):
    """Byte offset of each 128-row block's codes and index of its first group,
    as running sums over the blocks in order (block sizes follow from its width)."""
    code_off, group_off = [0], [0]
    for b in bit_map:
        b = int(b)
        code_off.append(code_off[-1] + MIX_BLOCK * K * b // 8)
        group_off.append(group_off[-1] + MIX_BLOCK * (K // GROUP_OF_BITS[b]))
    return code_off, group_off


def quantize_mixed(w_bits: np.ndarray, wtype: str, bit_map, layout: str, threads: int = 1):
    """Per 128-row block: quantize with (bits, group) = (4, 128) or (2, 64), pack,
    and concatenate.  Returns (packed u8, scales f32, zeros u8, per-block unpacked codes)."""
    N, K = w_bits.shape
    assert N % MIX_BLOCK == 0 and len(bit_map) == N // MIX_BLOCK
    packed, scales, zeros, codes_blocks = [], [], [], []
    for i, b in enumerate(bit_map):
        b = int(b)
        blk = w_bits[i * MIX_BLOCK:(i + 1) * MIX_BLOCK]
        c, s, z = quantize(blk, wtype, b, GROUP_OF_BITS[b], threads)
        packed.append(pack(c, b, layout))
        ms, mz = pack_meta(s, z, layout)
        scales.append(ms)
        zeros.append(mz)
        codes_blocks.append((c, s, z))
    return (np.concatenate(packed), np.concatenate(scales), np.concatenate(zeros), codes_blocks)


def linear_mixed_f64(x_f64: np.ndarray, codes_blocks, bit_map, threads: int = 1) -> np.ndarray:
    ys = []
    for (c, s, z), b in zip(codes_blocks, bit_map):
        ys.append(linear_f64(x_f64, c, s, z, GROUP_OF_BITS[int(b)], threads))
    return np.concatenate(ys, axis=1)
