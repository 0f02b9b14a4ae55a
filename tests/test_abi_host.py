"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments synchronously.  No GPU needed: every
call below returns before any CUDA work is enqueued (fake pointers are never
dereferenced because validation fails first)."""
from __future__ import annotations

import os
import re
import subprocess
import sys

import numpy as np
import pytest

from quantized_gemm_group_b200 import bq, build
from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return bq.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "bq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bq_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert names, "no declarations found"
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(bq.EXPORTS), set(names) ^ set(bq.EXPORTS)


def test_sizes(L):
    assert bq.bq_packed_bytes(4096, 4096, 4) == 4096 * 4096 // 2
    assert bq.bq_packed_bytes(14336, 4096, 2) == 14336 * 4096 // 4
    assert bq.bq_packed_bytes(16, 128, 3) == 0
    assert bq.bq_group_count(4096, 4096, 128) == 4096 * 32
    assert bq.bq_group_count(16, 100, 64) == 0


def test_mixed_offsets_match_oracle(L):
    rng = np.random.default_rng(0)
    for K in (256, 4096, 14336):
        bm = rng.choice([2, 4], size=24).astype(np.uint8)
        co, go = bq.bq_mixed_offsets(bm, 24 * 128, K)
        oco, ogo = O.mixed_offsets(bm, K)
        assert co.tolist() == oco and go.tolist() == ogo


def test_mixed_offsets_errors(L):
    with pytest.raises(bq.BQError) as e:
        bq.bq_mixed_offsets([4, 3], 256, 256)
    assert e.value.status == bq.BQ_ERR_UNSUPPORTED
    with pytest.raises(bq.BQError) as e:
        bq.bq_mixed_offsets([4], 100, 256)
    assert e.value.status == bq.BQ_ERR_SHAPE


def test_validation_cases_without_a_device():
    """Run the fake-pointer validation cases in a child with no visible GPU."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "abi_cases.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


def test_status_strings(L):
    for s in range(9):
        assert bq.status_string(s).startswith("BQ_")
    assert "unknown" in bq.status_string(99)
    assert "sm_100a" in bq.bq_version()
