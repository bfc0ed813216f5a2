"""The library's per-token softmax + top-k routine (every router entry point uses it), compiled
as host C++ and checked against the oracle on inputs full of exact ties: expert ids bit-exact
(ties to the lower index), gate weights within float32 rounding."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import moe_oracle as mo

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path_factory.mktemp("route") / "route_serial")
    subprocess.run([cxx, "-O2", "-std=c++17", os.path.join(HERE, "host", "route_serial_driver.cpp"),
                    "-o", exe], check=True)
    return exe


def _run(exe, L, k, gate_norm):
    T, E = L.shape
    txt = f"{T} {E} {k} {gate_norm}\n" + "\n".join(" ".join(repr(float(v)) for v in r) for r in L)
    out = subprocess.run([exe], input=txt, capture_output=True, text=True, check=True).stdout
    rows = [list(map(float, line.split())) for line in out.strip().splitlines()]
    a = np.array(rows)
    return a[:, :k].astype(np.int64), a[:, k:]


@pytest.mark.parametrize("gate_norm", [0, 1])
@pytest.mark.parametrize("E,k", [(4, 1), (6, 2), (8, 8), (13, 3), (64, 6), (256, 8)])
def test_route_serial_matches_oracle_with_ties(driver, E, k, gate_norm):
    rng = np.random.default_rng(E * 10 + k)
    # values on a coarse grid so that exact ties are everywhere; exactly representable in fp32
    L = (rng.integers(-4, 5, size=(300, E)) * 0.25).astype(np.float32)
    idx, w = _run(driver, L, k, gate_norm)
    L64 = L.astype(np.float64)
    assert np.array_equal(idx, mo.select_topk(L64, k))
    assert np.allclose(w, mo.gate_weights(L64, idx, gate_norm), rtol=2e-6, atol=1e-7)
