"""Host logic of bench.py's multi-GPU path (one process per GPU) on CPU:
two gloo ranks on 127.0.0.1 check that the timing reduction takes the
maximum over ranks and that the barrier and the rank-0-only output behave."""
from __future__ import annotations

import os
import socket
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import os, sys, json
    sys.path.insert(0, os.environ["BQ_ROOT"])
    import bench
    world, rank, local = bench.dist_setup()
    assert world == 2 and rank in (0, 1)
    bench.barrier(world)
    t = bench.max_over_ranks(1.0 + rank, world)      # rank 1 is the slow one
    assert t == 2.0, t
    args = type("A", (), {"steps": 1, "warmup": 0, "oracle_layers": 1, "reference_layers": 1, "bits": 4})()
    out = bench.run_reference(args, world, rank) if rank == 1 else None
    assert out is None                               # only rank 0 runs the reference arm
    import torch.distributed as dist
    dist.destroy_process_group()
    print(json.dumps({"rank": rank, "max": t}))
""")


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_max_over_ranks():
    port = free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, BQ_ROOT=ROOT, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=180) for p in procs]
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e[-2000:]
        assert '"max": 2.0' in o
