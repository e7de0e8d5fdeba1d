"""Shared test setup: markers, paths, fixture parsing."""
from __future__ import annotations

import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200)")
    config.addinivalue_line("markers", "slow: full-size cases (minutes)")


def _floats(tokens):
    return np.array([np.float32(float(t)) for t in tokens], dtype=np.float32)


def load_quantizer_cases():
    """Parse tests/golden/quantizer_cases.txt into a list of dicts."""
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "quantizer_cases.txt")) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case "):
                cur = {"name": line[5:].strip()}
                continue
            if line == "end":
                cases.append(cur)
                cur = None
                continue
            key, _, val = line.partition("=")
            key, toks = key.strip(), val.split()
            if key == "s":
                cur["s"] = float(toks[0])
            elif key in ("x", "err", "err_out"):
                cur[key] = _floats(toks)
            elif key == "q":
                cur["q"] = np.array([int(t) for t in toks], np.int8)
            elif key == "status":
                cur["status"] = int(toks[0])
            elif key == "stream":
                cur["stream"] = np.array([int(t, 16) for t in toks], np.uint8)
    return cases


def load_zre_runs():
    out = []
    with open(os.path.join(GOLDEN, "zre_runs.txt")) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            t = line.split()
            out.append((int(t[0]), [int(v, 16) for v in t[1:]]))
    return out


def load_quartic_anchors():
    out = []
    with open(os.path.join(GOLDEN, "quartic_anchors.txt")) as f:
        for raw in f:
            line = raw.strip()
            if not line or line.startswith("#"):
                continue
            t = [int(v) for v in line.split()]
            out.append((t[:5], t[5]))
    return out


@pytest.fixture(autouse=True)
def _debug_build_checks(request):
    """Under TLC_LIB=debug (the debug build of the library), every GPU test
    also requires that no bounds check or scratch canary failed."""
    yield
    if os.environ.get("TLC_LIB") != "debug" or request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    import gradient_traffic_compression_b200 as g
    assert g.tlc_debug_build(), "TLC_LIB=debug but the release library is loaded"
    fault = g.tlc_debug_fault(reset=True)
    assert fault == 0, f"debug check failed at line {fault & 0xFFFF} of file id {fault >> 16}"


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
