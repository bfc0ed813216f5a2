"""Seeded synthetic inputs for an MoE layer.

This module is the one piece the CUDA path and the CPU oracle share.  It draws random numbers
and rounds them to the storage dtype; it holds none of the layer's arithmetic.

Recipe (per tensor, one NumPy PCG64 stream spawned from the seed, in the fixed order
x, W_g, bias, W1, W3, W2, dy):
  x  ~ N(0, 1)            [T, d]
  Wg ~ N(0, 1/d)          [E, d]       (gate logits then have unit variance: "gain 1.0")
  W1 ~ N(0, 1/d)          [E_tot, F, d]
  W3 ~ N(0, 1/d)          [E_tot, F, d]  (SwiGLU only)
  W2 ~ N(0, 1/F)          [E_tot, d, F]
  dy ~ N(0, 1)            [T, d]       (upstream gradient)
  bias (fp32, [E]):  "zipf":   b_e = 2.0 * (pi(e) + 1) ** -1.2, pi a random permutation of experts
                     "normal": b_e ~ N(0, 0.5)
The second argument of N(.,.) is the variance.  Values are drawn in float32 and, for bf16
layers, rounded once to bf16 (round to nearest even); both sides then read identical bytes.
bf16 arrays are stored as uint16 bit patterns.
"""
from __future__ import annotations

import numpy as np

from .configs import BF16, SWIGLU, LayerShape

_ORDER = ("x", "Wg", "bias", "W1", "W3", "W2", "dy")


def round_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> 16) & 1
    return ((u + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(rng: np.random.Generator, shape, var: float) -> np.ndarray:
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if var != 1.0:
        out *= np.float32(np.sqrt(var))
    return out


def make_inputs(shape: LayerShape, seed: int = 0, *, with_dy: bool = True) -> dict:
    """All inputs of one layer, in storage form (float32, or uint16 bf16 bits)."""
    ss = np.random.SeedSequence(seed)
    rngs = dict(zip(_ORDER, [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(len(_ORDER))]))
    T, d, E, F, Et = shape.T, shape.d, shape.E, shape.d_ff, shape.E_tot
    raw = {
        "x": _normal(rngs["x"], (T, d), 1.0),
        "Wg": _normal(rngs["Wg"], (E, d), 1.0 / d),
        "W1": _normal(rngs["W1"], (Et, F, d), 1.0 / d),
        "W3": _normal(rngs["W3"], (Et, F, d), 1.0 / d) if shape.act == SWIGLU else None,
        "W2": _normal(rngs["W2"], (Et, d, F), 1.0 / F),
        "dy": _normal(rngs["dy"], (T, d), 1.0) if (with_dy and not shape.fwd_only) else None,
    }
    if shape.bias == "zipf":
        perm = rngs["bias"].permutation(E)
        bias = (2.0 * (perm.astype(np.float64) + 1.0) ** -1.2).astype(np.float32)
    elif shape.bias == "normal":
        bias = _normal(rngs["bias"], (E,), 0.5)
    else:
        bias = None
    out = {"bias": bias}
    for name, v in raw.items():
        if v is None:
            out[name] = None
        elif shape.dtype == BF16:
            out[name] = round_to_bf16_bits(v)
        else:
            out[name] = v
    return out


def to_f64(a, dtype: int):
    """Storage form -> float64 (exact: every bf16 / fp32 value is a float64)."""
    if a is None:
        return None
    if dtype == BF16 and a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)
