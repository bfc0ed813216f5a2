"""Host-side checks of the C ABI that need no GPU: the library builds and loads, exports every
symbol include/moe.h declares, and validates arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_23_b200 import build as moe_build
from mixture_experts_layer_23_b200.configs import (BF16, DROPLESS, FP32, LAYERS, PARITY_FP32,
                                                   PARITY_SMALL, LayerShape)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    moe_build.build()
    from mixture_experts_layer_23_b200 import moe as m
    return m


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = _declared_functions()
    for required in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine",
                     "moe_layer_fwd", "moe_layer_bwd"):
        assert required in names


def test_library_exports_every_declared_symbol(moe):
    lib = ctypes.CDLL(moe.lib_path())
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(moe.EXPORTS) == set(_declared_functions())


def test_layout_capacity_matches_the_capacity_rule(moe):
    from oracle import moe_oracle as mo
    for s in LAYERS + PARITY_SMALL + PARITY_FP32:
        L = moe.get_layout(moe.make_config(s))
        C = mo.capacity(s.capacity_factor, s.k, s.T, s.E)
        assert L.capacity == (DROPLESS if C is None else C), s.name
        assert L.T_pad % 128 == 0 and L.T_pad >= s.T
        assert L.routed_row0 == s.n_shared * L.T_pad
        # the row space holds the worst-case routing with every segment padded to 128
        kmax = s.T if C is None else min(C, s.T)
        worst = min(s.T * s.k, s.E * kmax)
        assert L.rows - L.routed_row0 >= worst
        assert L.ctx_bytes > 0 and L.scratch_bytes > 0
        for f in ("ctx_logits", "ctx_topk_idx", "ctx_Xd", "ctx_Gu", "ctx_H", "ctx_O"):
            assert getattr(L, f) % 256 == 0


def test_named_capacities(moe):
    want = {"switch_tiny": 80, "gpt2_gshard": 640, "bert_large_skew": 512,
            "mixtral_dropless": DROPLESS, "deepseek_v2": 2304}
    for s in LAYERS:
        assert moe.get_layout(moe.make_config(s)).capacity == want[s.name]


@pytest.mark.parametrize("field,value,status", [
    ("k", 0, 1), ("k", 5, 1), ("T", 0, 1), ("d", 12, 2), ("E", 300, 2), ("act", 7, 1),
    ("gate_norm", 2, 1), ("dtype", 3, 1), ("n_shared", 9, 2),
])
def test_invalid_configs_rejected(moe, field, value, status):
    s = LayerShape("t", T=64, d=64, E=4, k=2, d_ff=64, dtype=BF16)
    cfg = moe.make_config(s)
    setattr(cfg, field, value)
    L = moe.Layout()
    assert moe.lib().moe_get_layout(ctypes.byref(cfg), ctypes.byref(L)) == status


def test_bad_capacity_factor_rejected(moe):
    s = LayerShape("t", T=64, d=64, E=4, k=2, d_ff=64, dtype=BF16)
    cfg = moe.make_config(s)
    cfg.capacity_factor = -1.0
    L = moe.Layout()
    assert moe.lib().moe_get_layout(ctypes.byref(cfg), ctypes.byref(L)) == 1


@pytest.mark.parametrize("coef", [-0.5, float("nan"), float("inf")])
def test_bad_aux_loss_coef_rejected(moe, coef):
    s = LayerShape("t", T=64, d=64, E=4, k=2, d_ff=64, dtype=BF16)
    cfg = moe.make_config(s)
    cfg.aux_loss_coef = coef
    L = moe.Layout()
    assert moe.lib().moe_get_layout(ctypes.byref(cfg), ctypes.byref(L)) == 1


def test_bad_drop_order_rejected(moe):
    s = LayerShape("t", T=64, d=64, E=4, k=2, d_ff=64, dtype=BF16)
    cfg = moe.make_config(s)
    cfg.drop_order = 2
    L = moe.Layout()
    assert moe.lib().moe_get_layout(ctypes.byref(cfg), ctypes.byref(L)) == 1


def test_choice_major_scratch_holds_k_histogram_layers(moe):
    base = LayerShape("t", T=1000, d=64, E=16, k=4, d_ff=64, dtype=BF16)
    from dataclasses import replace
    a = moe.get_layout(moe.make_config(base)).scratch_bytes
    b = moe.get_layout(moe.make_config(replace(base, choice_major=True))).scratch_bytes
    assert b >= a + 3 * 4 * 16 * 4 - 256   # (k - 1) more layers of ceil(T/256) x E int32


def test_aux_loss_layout_and_argument_checks(moe):
    s = LayerShape("t", T=300, d=64, E=6, k=2, d_ff=64, dtype=BF16, aux_loss_coef=0.01)
    cfg = moe.make_config(s)
    L = moe.get_layout(cfg)
    assert L.ctx_aux_loss % 256 == 0 and L.ctx_aux_loss + 4 <= L.ctx_bytes
    lib = moe.lib()
    good = 0x10000
    assert lib.moe_aux_loss(ctypes.byref(cfg), good, good, None, good, None) == 1
    assert lib.moe_aux_loss(ctypes.byref(cfg), good, good + 4, good, good, None) == 3


def test_pointer_checks_happen_before_any_cuda_call(moe):
    s = LayerShape("t", T=64, d=64, E=4, k=2, d_ff=64, dtype=BF16)
    cfg = moe.make_config(s)
    lib = moe.lib()
    good = 0x10000
    # null pointer -> invalid argument
    assert lib.moe_route(ctypes.byref(cfg), None, good, None, good, good, good, None) == 1
    # misaligned pointer -> misaligned
    assert lib.moe_route(ctypes.byref(cfg), good + 4, good, None, good, good, good, None) == 3
    assert lib.moe_combine(ctypes.byref(cfg), good, good, good + 8, good, None) == 3
    assert lib.moe_layer_fwd(ctypes.byref(cfg), good, good, None, good, None, good, good, good,
                             good + 1, None) == 3
    # SwiGLU needs W3
    s2 = s.with_(act=1)
    cfg2 = moe.make_config(s2)
    assert lib.moe_layer_fwd(ctypes.byref(cfg2), good, good, None, good, None, good, good, good,
                             good, None) == 1


def test_fused_forward_rejects_large_layers_before_any_cuda_call(moe):
    s = [l for l in LAYERS if l.name == "gpt2_gshard"][0]
    cfg = moe.make_config(s)
    good = 0x10000
    lib = moe.lib()
    assert lib.moe_layer_fwd_fused(ctypes.byref(cfg), good, good, None, good, None, good, good,
                                   None, None, None, None) == 2
    # routing outputs are all-or-none
    t = [l for l in LAYERS if l.name == "switch_tiny"][0]
    assert lib.moe_layer_fwd_fused(ctypes.byref(moe.make_config(t)), good, good, None, good, None,
                                   good, good, good, None, None, None) == 1


def test_ctypes_structs_match_the_header(moe, tmp_path):
    """The binding's ctypes mirrors of moe_config_t and moe_layout_t have the C compiler's layout:
    the same size, and every field at the same offset with the same size."""
    import subprocess
    exe = tmp_path / "abi_layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "host", "abi_layout.c"), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    structs = {"moe_config_t": moe.Config, "moe_layout_t": moe.Layout}
    seen = {name: set() for name in structs}
    for line in filter(None, out):
        parts = line.split()
        S = structs[parts[0]]
        if parts[1] == "sizeof":
            assert ctypes.sizeof(S) == int(parts[2]), parts[0]
            continue
        field = getattr(S, parts[1])
        assert (field.offset, field.size) == (int(parts[2]), int(parts[3])), line
        seen[parts[0]].add(parts[1])
    for name, S in structs.items():
        assert seen[name] == {f for f, _ in S._fields_}, name


def test_status_strings(moe):
    for code in range(7):
        assert moe.lib().moe_status_string(code)
    assert moe.lib().moe_status_string(99) == b"unknown status"


def test_wait_hooks_validate_their_arguments(moe):
    """The bounded-wait settings are host-only setters: out-of-range values are refused, valid
    ones accepted (and the defaults put back)."""
    lib = moe.lib()
    assert lib.moe_set_wait_budget_ns(0) == 1
    assert lib.moe_set_wait_budget_ns(999) == 1
    assert lib.moe_set_wait_budget_ns(61 * 10**9) == 1
    assert lib.moe_set_wait_stall(2) == 1
    assert lib.moe_set_wait_stall(-1) == 1
    assert lib.moe_set_wait_budget_ns(1000) == 0
    assert lib.moe_set_wait_stall(1) == 0
    assert lib.moe_set_wait_stall(0) == 0
    assert lib.moe_set_wait_budget_ns(2 * 10**9) == 0
