"""The debug build of the library (libtlc_debug.so: the same sources with
-DTLC_DEBUG) runs a subset of the GPU parity tests in a child process: the
cases that stress indices (every ragged tail, zero runs across tile edges,
the deferred placement, the indexed decode on both tilings, the fused
accumulate, random payloads), with every bounds check recorded instead of
faulting and canaries around every scratch allocation.  Each test of the
subset also requires that no check failed (tests/conftest.py)."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

from conftest import ROOT

torch = pytest.importorskip("torch")

SUBSET = ("ragged or every_tail or runs_across or deferred or fuzz or density_sweep or "
          "tile_edges or fused_accumulate or unaligned_payload or large_plan or indexed_plan")


@pytest.mark.gpu
@pytest.mark.timeout(1200)
def test_debug_build_subset_with_no_failed_check():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gradient_traffic_compression_b200 import build
    build.ensure_built(debug=True)
    env = dict(os.environ, TLC_LIB="debug")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "gpu",
           "-k", SUBSET, "tests/test_gpu_parity.py", "tests/test_gpu_indexed.py",
           "tests/test_gpu_batch.py"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1100)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail
