"""GPU checks of the C ABI's options and the host-buffer path.

* BQ_OPT_LINEAR_OVERLAP (0 plain launches, 1 programmatic dependent launch,
  2 weights streamed before the wait) changes launch order only: results
  are identical for back-to-back linears, decode and prefill.
* bq_linear_host (pinned host x in, host y out) equals the device call.
* Degenerate shapes: M = 0 and N = 0 are no-ops; K = 0 gives y = 0.
"""
from __future__ import annotations

import pytest
import torch

from quantized_gemm_group_b200 import bq, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("M", [1, 16, 40, 256])
def test_overlap_modes_identical(M):
    N, K = 1024, 2048
    W = synth.normal((N, K), 0.02, seed=7, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    xs = [synth.activations(M, K, seed=8 + i, device=DEV) for i in range(3)]
    old = bq.bq_get_option(bq.BQ_OPT_LINEAR_OVERLAP)
    outs = {}
    try:
        for mode in (0, 1, 2):
            bq.bq_set_option(bq.BQ_OPT_LINEAR_OVERLAP, mode)
            ys = [bq.bq_linear(x, pk, sc, ze, N, 4, 128) for x in xs]   # back to back on one stream
            torch.cuda.synchronize()
            outs[mode] = torch.stack(ys)
    finally:
        bq.bq_set_option(bq.BQ_OPT_LINEAR_OVERLAP, old)
    assert bq.bq_device_status() == bq.BQ_OK
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_set_option_rejects_unknown():
    with pytest.raises(bq.BQError):
        bq.bq_set_option(bq.BQ_OPT_LINEAR_OVERLAP, 3)
    with pytest.raises(bq.BQError):
        bq.bq_set_option(99, 0)


def test_host_buffer_path_matches_device():
    N, K, M = 512, 4096, 4
    W = synth.normal((N, K), 0.02, seed=11, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    x = synth.activations(M, K, seed=12, device=DEV)
    x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    x_host.copy_(x.cpu())
    y_host = bq.bq_linear_host(x_host, pk, sc, ze, N, 4, 128)
    torch.cuda.synchronize()
    y_dev = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    assert torch.equal(y_host, y_dev.cpu())


def test_degenerate_shapes():
    N, K = 256, 1024
    W = synth.normal((N, K), 0.02, seed=13, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    y0 = bq.bq_linear(torch.empty((0, K), dtype=torch.bfloat16, device=DEV), pk, sc, ze, N, 4, 128)
    assert y0.shape == (0, N)
    # K = 0: an empty sum, y = 0
    yk = torch.full((3, N), 7.0, dtype=torch.bfloat16, device=DEV)
    bq.bq_linear(torch.empty((3, 0), dtype=torch.bfloat16, device=DEV), pk, sc, ze, N, 4, 128, out=yk)
    torch.cuda.synchronize()
    assert torch.count_nonzero(yk) == 0
    # N = 0 is a no-op
    yn = bq.bq_linear(synth.activations(2, K, seed=14, device=DEV), pk, sc, ze, 0, 4, 128)
    assert yn.shape == (2, 0)
    assert bq.bq_device_status() == bq.BQ_OK


def test_bounded_wait_gives_up_and_reports_timeout():
    """The kernels' bounded wait, driven to expiry on a barrier phase nothing
    completes: the kernel returns, the status reports BQ_ERR_TIMEOUT once,
    and the context keeps working."""
    assert bq.bq_device_status() == bq.BQ_OK
    bq.bq_selftest_bounded_wait(256)
    assert bq.bq_device_status() == bq.BQ_ERR_TIMEOUT
    assert bq.bq_device_status() == bq.BQ_OK          # read and cleared
    N, K = 256, 1024
    W = synth.normal((N, K), 0.02, seed=11, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    x = synth.activations(2, K, seed=12, device=DEV)
    y1 = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    y2 = bq.bq_linear(x, pk, sc, ze, N, 4, 128)
    torch.cuda.synchronize()
    assert bq.bq_device_status() == bq.BQ_OK
    assert torch.equal(y1, y2)
    with pytest.raises(bq.BQError):
        bq.bq_selftest_bounded_wait(0)


def test_two_host_threads_two_streams():
    """Two host threads call the library at once, each on its own stream:
    results equal the sequential ones (kernel attributes are set per device
    and kernel, options are atomic)."""
    import threading
    N, K = 2048, 4096
    W = synth.normal((N, K), 0.02, seed=31, dtype="f16", device=DEV)
    pk, sc, ze = bq.bq_quantize(W, 4, 128, "interleaved")
    xs = [synth.activations(m, K, seed=40 + m, device=DEV) for m in (1, 16)]
    ref = [bq.bq_linear(x, pk, sc, ze, N, 4, 128) for x in xs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in xs]
    got = [None, None]
    errs = []

    def run(t):
        try:
            with torch.cuda.stream(streams[t]):
                ys = [bq.bq_linear(xs[t], pk, sc, ze, N, 4, 128, stream=streams[t]) for _ in range(20)]
            streams[t].synchronize()
            got[t] = ys
        except Exception as e:  # noqa: BLE001
            errs.append(e)

    th = [threading.Thread(target=run, args=(t,)) for t in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    assert bq.bq_device_status() == bq.BQ_OK
    for t in range(2):
        for y in got[t]:
            assert torch.equal(y, ref[t])
