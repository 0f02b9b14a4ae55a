"""Splitting a weight-only linear by output channels over ranks (host logic,
CPU only): the partition into whole 128-row blocks, and two gloo ranks whose
gathered per-rank oracle products equal the oracle's product of the whole
matrix.  The product on each rank is the CPU oracle here; on GPUs it is
bq_linear (bench.py --split)."""
from __future__ import annotations

import os
import socket
import subprocess
import sys
import textwrap

import numpy as np
import pytest

from quantized_gemm_group_b200 import shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N", [128, 1024, 4096, 6144, 14336, 28672, 400, 16, 0])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_block_ranges_cover_whole_blocks(N, world):
    rs = shard.block_ranges(N, world)
    assert len(rs) == world
    assert rs[0][0] == 0 and rs[-1][1] == N
    for (a0, a1), (b0, b1) in zip(rs, rs[1:]):
        assert a1 == b0 and a0 <= a1
    for r0, r1 in rs:
        assert (r0 % 128 == 0 or r0 == N) and (r1 % 128 == 0 or r1 == N)
    nblk = (N + 127) // 128
    if nblk >= world:   # balanced to within one block
        sizes = [(r1 - r0 + 127) // 128 for r0, r1 in rs]
        assert max(sizes) - min(sizes) <= 1


def test_block_ranges_balance_bytes_of_a_width_map():
    bit_map = [4] * 8 + [2] * 24          # Channel-mix-like: 4-bit blocks weigh twice
    rs = shard.block_ranges(32 * 128, 2, bit_map)
    w = [sum(bit_map[r0 // 128:r1 // 128]) for r0, r1 in rs]
    assert abs(w[0] - w[1]) <= 4
    assert rs[0][1] // 128 < 16           # the heavy blocks come first: rank 0 takes fewer


CHILD = textwrap.dedent("""
    import os, sys
    sys.path.insert(0, os.environ["BQ_ROOT"])
    import numpy as np, torch, torch.distributed as dist
    from oracle import oracle as O
    from quantized_gemm_group_b200 import shard, synth
    dist.init_process_group("gloo")
    rank, world = dist.get_rank(), dist.get_world_size()
    N, K, M = int(os.environ["N"]), 512, 3
    W = synth.normal((N, K), 0.02, seed=7, dtype="f16", device="cpu")
    x = synth.activations(M, K, seed=8, device="cpu")
    xf = O.decode_f64(synth.bits16(x), "bf16")
    ranges = shard.block_ranges(N, world)
    r0, r1 = ranges[rank]
    if r1 > r0:
        c, s, z = O.quantize(synth.bits16(W[r0:r1]), "f16", 4, 128)
        y_local = torch.from_numpy(O.linear_f64(xf, c, s, z, 128))
    else:
        y_local = torch.zeros((M, 0), dtype=torch.float64)
    y = shard.gather_rows(y_local, ranges, rank)
    c, s, z = O.quantize(synth.bits16(W), "f16", 4, 128)
    y_ref = O.linear_f64(xf, c, s, z, 128)
    assert y.shape == (M, N), y.shape
    assert np.array_equal(y.numpy(), y_ref), np.abs(y.numpy() - y_ref).max()
    dist.destroy_process_group()
    print("ok", rank)
""")


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("N", [1024, 400, 128])
def test_two_gloo_ranks_gathered_product_equals_whole(N):
    port = free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, BQ_ROOT=ROOT, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", N=str(N),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=300) for p in procs]
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e[-3000:]
        assert o.startswith("ok")
