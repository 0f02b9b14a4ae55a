"""Argument-validation cases with fake device pointers.

Never collected directly: tests/test_abi_host.py runs this file in a child
process with CUDA_VISIBLE_DEVICES set to empty, so even a validation bug can
only return an error code and can never touch a device.  Every fake-pointer
case below expects an error status; the only BQ_OK cases pass NULL pointers
with an empty shape."""
from __future__ import annotations

import ctypes
import os

import pytest

from quantized_gemm_group_b200 import bq

assert os.environ.get("CUDA_VISIBLE_DEVICES") == "", "run only through tests/test_abi_host.py"


@pytest.fixture(scope="module")
def L():
    return bq.lib()


FAKE = ctypes.c_void_p(0x7F0000001000)       # 16-byte aligned, never dereferenced
FAKE_MIS = ctypes.c_void_p(0x7F0000001004)   # misaligned


def q(L, W=FAKE, wt=bq.BQ_F16, rows=16, cols=128, bits=4, group=128, layout=1, pk=FAKE, sc=FAKE, ze=FAKE):
    return L.bq_quantize(W, wt, rows, cols, bits, group, layout, pk, sc, ze, None)


def test_quantize_validation(L):
    assert q(L, rows=-1) == bq.BQ_ERR_SHAPE
    assert q(L, bits=3) == bq.BQ_ERR_UNSUPPORTED
    assert q(L, bits=8) == bq.BQ_ERR_UNSUPPORTED
    assert q(L, wt=bq.BQ_F32) == bq.BQ_ERR_UNSUPPORTED
    assert q(L, layout=7) == bq.BQ_ERR_UNSUPPORTED
    assert q(L, group=48) == bq.BQ_ERR_UNSUPPORTED
    assert q(L, group=8) == bq.BQ_ERR_UNSUPPORTED          # interleaved needs >= 16
    assert q(L, cols=192) == bq.BQ_ERR_SHAPE               # cols % group
    assert q(L, rows=24) == bq.BQ_ERR_SHAPE                # rows % 16 (interleaved)
    assert q(L, bits=2, group=64, cols=64) == bq.BQ_ERR_SHAPE   # 2-bit tile is 128 wide
    assert q(L, W=None) == bq.BQ_ERR_NULL
    assert q(L, pk=None) == bq.BQ_ERR_NULL
    assert q(L, W=FAKE_MIS) == bq.BQ_ERR_ALIGN
    assert q(L, pk=FAKE_MIS) == bq.BQ_ERR_ALIGN
    assert q(L, rows=0, W=None) == bq.BQ_OK                # empty: nothing to do
    assert q(L, layout=0, rows=3, cols=24, group=8, bits=2) == bq.BQ_ERR_SHAPE  # 24*2 % 32
    assert q(L, layout=0, rows=3, cols=0, group=8, W=None) == bq.BQ_OK


def test_quantize_symmetric_validation(L):
    f = L.bq_quantize_symmetric
    assert f(FAKE, bq.BQ_F16, 16, 128, 3, 128, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_UNSUPPORTED
    assert f(FAKE, bq.BQ_F32, 16, 128, 4, 128, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_UNSUPPORTED
    assert f(FAKE, bq.BQ_F16, 20, 128, 4, 128, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_SHAPE   # rows % 16
    assert f(FAKE, bq.BQ_F16, 16, 192, 4, 128, 0, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_SHAPE   # cols % group
    assert f(None, bq.BQ_F16, 16, 128, 4, 128, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_NULL
    assert f(FAKE_MIS, bq.BQ_F16, 16, 128, 4, 128, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_ALIGN
    assert f(None, bq.BQ_F16, 0, 128, 4, 128, 1, None, None, None, None) == bq.BQ_OK


def test_quantize_mixed_validation(L):
    f = L.bq_quantize_mixed
    assert f(FAKE, bq.BQ_F16, 200, 256, FAKE, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_SHAPE
    assert f(FAKE, bq.BQ_F16, 256, 192, FAKE, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_SHAPE
    assert f(FAKE, bq.BQ_F16, 256, 128, FAKE, 0, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_SHAPE  # canonical: 256
    assert f(FAKE, bq.BQ_F16, 256, 256, None, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_NULL
    assert f(FAKE_MIS, bq.BQ_F16, 256, 256, FAKE, 1, FAKE, FAKE, FAKE, None) == bq.BQ_ERR_ALIGN
    assert f(None, bq.BQ_F16, 0, 256, None, 1, None, None, None, None) == bq.BQ_OK


def lin(L, x=FAKE, xt=bq.BQ_BF16, M=1, K=4096, pk=FAKE, sc=FAKE, ze=FAKE, bm=None, bits=4, group=128,
        N=4096, layout=1, y=FAKE):
    return L.bq_linear(x, xt, M, K, pk, sc, ze, bm, bits, group, N, layout, y, None)


def test_linear_validation(L):
    assert lin(L, M=-1) == bq.BQ_ERR_SHAPE
    assert lin(L, xt=bq.BQ_F32) == bq.BQ_ERR_UNSUPPORTED
    assert lin(L, layout=0) == bq.BQ_ERR_UNSUPPORTED       # linear reads the interleaved layout
    assert lin(L, bits=3) == bq.BQ_ERR_UNSUPPORTED
    assert lin(L, group=16) == bq.BQ_ERR_UNSUPPORTED
    assert lin(L, N=24) == bq.BQ_ERR_SHAPE
    assert lin(L, K=4032) == bq.BQ_ERR_SHAPE
    assert lin(L, K=4224) == bq.BQ_ERR_SHAPE                # 4-bit needs K % 256
    assert lin(L, K=4352, bits=2, group=64) == bq.BQ_ERR_SHAPE   # 2-bit needs K % 512
    assert lin(L, bm=FAKE, N=4096, K=4352) == bq.BQ_ERR_SHAPE    # mixed needs K % 512
    assert lin(L, sc=FAKE_MIS) == bq.BQ_ERR_ALIGN          # bulk copies need 16-byte metadata
    assert lin(L, bm=FAKE, N=4000) == bq.BQ_ERR_SHAPE      # mixed needs N % 128
    assert lin(L, x=None) == bq.BQ_ERR_NULL
    assert lin(L, pk=None) == bq.BQ_ERR_NULL
    assert lin(L, x=FAKE_MIS) == bq.BQ_ERR_ALIGN
    assert lin(L, y=FAKE_MIS) == bq.BQ_ERR_ALIGN
    assert lin(L, M=0, x=None, y=None) == bq.BQ_OK


def grad(L, dy=FAKE, dt=bq.BQ_BF16, M=1, N=4096, pk=FAKE, sc=FAKE, ze=FAKE, bm=None, bits=4, group=128,
         K=4096, layout=1, dx=FAKE):
    return L.bq_linear_grad_input(dy, dt, M, N, pk, sc, ze, bm, bits, group, K, layout, dx, None)


def test_linear_grad_input_validation(L):
    assert grad(L, M=-1) == bq.BQ_ERR_SHAPE
    assert grad(L, dt=bq.BQ_F32) == bq.BQ_ERR_UNSUPPORTED
    assert grad(L, layout=0) == bq.BQ_ERR_UNSUPPORTED       # reads the interleaved layout
    assert grad(L, bm=FAKE, N=4000) == bq.BQ_ERR_SHAPE      # a width map needs whole 128-row blocks
    assert grad(L, bm=FAKE, K=4160) == bq.BQ_ERR_SHAPE      # 128-column slices
    assert grad(L, bits=3) == bq.BQ_ERR_UNSUPPORTED
    assert grad(L, group=16) == bq.BQ_ERR_UNSUPPORTED
    assert grad(L, N=24) == bq.BQ_ERR_SHAPE                 # row tiles of 16
    assert grad(L, K=4160) == bq.BQ_ERR_SHAPE               # 128-column slices
    assert grad(L, K=4224, group=256) == bq.BQ_ERR_SHAPE    # K % group
    assert grad(L, dy=None) == bq.BQ_ERR_NULL
    assert grad(L, ze=None) == bq.BQ_ERR_NULL
    assert grad(L, dx=None) == bq.BQ_ERR_NULL
    assert grad(L, dy=FAKE_MIS) == bq.BQ_ERR_ALIGN
    assert grad(L, dx=FAKE_MIS) == bq.BQ_ERR_ALIGN
    assert grad(L, sc=FAKE_MIS) == bq.BQ_ERR_ALIGN
    assert grad(L, M=0, dy=None, dx=None) == bq.BQ_OK
    assert grad(L, K=0, dy=None, dx=None) == bq.BQ_OK


def test_fake_quantize_validation(L):
    f = L.bq_fake_quantize
    assert f(FAKE, bq.BQ_F32, 16, 128, 4, 128, FAKE, bq.BQ_BF16, None) == bq.BQ_ERR_UNSUPPORTED  # W must be 16-bit
    assert f(FAKE, bq.BQ_F16, 16, 128, 4, 128, FAKE, 7, None) == bq.BQ_ERR_UNSUPPORTED
    assert f(FAKE, bq.BQ_F16, 16, 128, 3, 128, FAKE, bq.BQ_F32, None) == bq.BQ_ERR_UNSUPPORTED
    assert f(FAKE, bq.BQ_F16, 16, 128, 4, 96, FAKE, bq.BQ_F32, None) == bq.BQ_ERR_UNSUPPORTED
    assert f(FAKE, bq.BQ_F16, 16, 192, 4, 128, FAKE, bq.BQ_F32, None) == bq.BQ_ERR_SHAPE   # cols % group
    assert f(FAKE, bq.BQ_F16, -1, 128, 4, 128, FAKE, bq.BQ_F32, None) == bq.BQ_ERR_SHAPE
    assert f(None, bq.BQ_F16, 16, 128, 4, 128, FAKE, bq.BQ_F32, None) == bq.BQ_ERR_NULL
    assert f(FAKE_MIS, bq.BQ_F16, 16, 128, 4, 128, FAKE, bq.BQ_F32, None) == bq.BQ_ERR_ALIGN
    assert f(FAKE, bq.BQ_F16, 16, 128, 4, 128, FAKE_MIS, bq.BQ_F32, None) == bq.BQ_ERR_ALIGN
    assert f(None, bq.BQ_F16, 0, 128, 4, 128, None, bq.BQ_F32, None) == bq.BQ_OK


def test_dequant_validation(L):
    f = L.bq_dequantize
    assert f(FAKE, FAKE, FAKE, None, 4, 128, 16, 128, 1, FAKE, 7, None) == bq.BQ_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, None, 3, 128, 16, 128, 1, FAKE, 2, None) == bq.BQ_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, None, 4, 100, 16, 128, 1, FAKE, 2, None) == bq.BQ_ERR_SHAPE
    assert f(None, FAKE, FAKE, None, 4, 128, 16, 128, 1, FAKE, 2, None) == bq.BQ_ERR_NULL
    assert f(FAKE, FAKE, FAKE, None, 4, 128, 16, 128, 1, FAKE_MIS, 2, None) == bq.BQ_ERR_ALIGN


