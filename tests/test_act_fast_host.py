"""The bf16 epilogues' GELU, GELU' and sigmoid (Abramowitz & Stegun 7.1.26 erf), compiled as
host C++, against scipy's erf and the normal pdf: the published bound (|erf error| <= 1.5e-7)
carries over to absolute errors of a few 1e-7 here, far below bf16 resolution (2^-8)."""
import os
import shutil
import subprocess

import numpy as np
import pytest
from scipy.special import erf, expit

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = str(tmp_path_factory.mktemp("act") / "act")
    subprocess.run([cxx, "-O2", "-std=c++17", os.path.join(HERE, "host", "act_driver.cpp"),
                    "-o", exe], check=True)
    return exe


def test_fast_activations_within_published_bound(driver):
    u = np.concatenate([np.linspace(-9, 9, 4001), [0.0, -0.0, 1e-6, -1e-6, 30.0, -30.0]])
    u32 = u.astype(np.float32)
    txt = "\n".join(repr(float(v)) for v in u32)
    out = subprocess.run([driver], input=txt, capture_output=True, text=True, check=True).stdout
    got = np.array([list(map(float, l.split())) for l in out.strip().splitlines()])
    x = u32.astype(np.float64)
    phi_cdf = 0.5 * (1 + erf(x / np.sqrt(2)))
    gelu = x * phi_cdf
    gelu_grad = phi_cdf + x * np.exp(-0.5 * x * x) / np.sqrt(2 * np.pi)
    # erf error 1.5e-7 -> GELU error <= 0.5 |u| 1.5e-7 (+ float32 rounding of the pieces)
    assert np.all(np.abs(got[:, 0] - gelu) <= 1e-7 * np.abs(x) + 2e-6 * np.abs(gelu) + 1e-7)
    assert np.max(np.abs(got[:, 1] - gelu_grad)) <= 1e-6
    assert np.max(np.abs(got[:, 2] - expit(x))) <= 1e-6
