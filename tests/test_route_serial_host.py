"""The library's per-token softmax + top-k routine (every router entry point uses it), compiled
as host C++ and checked against the oracle on inputs full of exact ties: expert ids bit-exact
(ties to the lower index), gate weights within float32 rounding.  Both slot counts are checked:
8 slots (the CUDA-core routers) and the fewest slots for k (the tensor-core router), which must give
the same ids and weights."""
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


def _run(exe, L, k, gate_norm, slots="8"):
    T, E = L.shape
    txt = f"{T} {E} {k} {gate_norm}\n" + "\n".join(" ".join(repr(float(v)) for v in r) for r in L)
    args = [exe] + (["kslots"] if slots == "k" else [])
    out = subprocess.run(args, input=txt, capture_output=True, text=True, check=True).stdout
    rows = [list(map(float, line.split())) for line in out.strip().splitlines()]
    a = np.array(rows)
    return a[:, :k].astype(np.int64), a[:, k:]


@pytest.mark.parametrize("slots", ["8", "k"])
@pytest.mark.parametrize("gate_norm", [0, 1])
@pytest.mark.parametrize("E,k", [(4, 1), (6, 2), (8, 8), (13, 3), (16, 4), (40, 5), (64, 6),
                                 (70, 7), (256, 8)])
def test_route_serial_matches_oracle_with_ties(driver, E, k, gate_norm, slots):
    rng = np.random.default_rng(E * 10 + k)
    # values on a coarse grid so that exact ties are everywhere; exactly representable in fp32
    L = (rng.integers(-4, 5, size=(300, E)) * 0.25).astype(np.float32)
    idx, w = _run(driver, L, k, gate_norm, slots)
    L64 = L.astype(np.float64)
    assert np.array_equal(idx, mo.select_topk(L64, k))
    assert np.allclose(w, mo.gate_weights(L64, idx, gate_norm), rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("E,k,gate_norm", [(8, 2, 1), (64, 6, 0), (24, 3, 0), (256, 5, 1)])
def test_slot_counts_agree_bitwise(driver, E, k, gate_norm):
    """The tensor-core router keeps only the slots k needs and the CUDA-core routers keep 8: the
    same logits must give the same ids and bitwise the same weights, so that every entry point
    routes alike."""
    rng = np.random.default_rng(7 * E + k)
    L = np.concatenate([rng.standard_normal((200, E)),
                        rng.integers(-3, 4, size=(100, E)) * 0.5]).astype(np.float32)
    i8, w8 = _run(driver, L, k, gate_norm, "8")
    ik, wk = _run(driver, L, k, gate_norm, "k")
    assert np.array_equal(i8, ik)
    assert np.array_equal(w8, wk)
