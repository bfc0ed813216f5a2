"""Shared machinery of the GPU parity tests: run the layer through the C ABI, run the oracle on
the same seeded inputs, and compare (bit-exact for routing and dispatch, the stated float
tolerance for everything else)."""
from __future__ import annotations

import numpy as np

from mixture_experts_layer_23_b200.configs import BF16, SWIGLU, LayerShape
from mixture_experts_layer_23_b200.synth import bf16_bits_to_f32, make_inputs, to_f64
from oracle import moe_oracle as mo

ROW_ALIGN = 128


def tol_for(shape: LayerShape) -> float:
    """max-abs error bound, relative to max|ref|, per tensor: 1e-4 (fp32) / 2e-2 (bf16)."""
    return 2e-2 if shape.dtype == BF16 else 1e-4


def assert_close(name, got, ref, rel):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert err <= rel * scale + 1e-30, f"{name}: max|err| {err:.3e} > {rel:.0e} * max|ref| {scale:.3e}"
    return err / scale if scale else 0.0


class LazyF64:
    """Per-expert float64 view of a large storage-form weight (converted on use; kept for reuse
    unless keep=False)."""

    def __init__(self, a, dtype, keep=True):
        self.a, self.dtype, self.cache, self.keep = a, dtype, {}, keep
        self.shape = a.shape

    def __getitem__(self, e):
        if not self.keep:
            return to_f64(self.a[e], self.dtype)
        if e not in self.cache:
            self.cache[e] = to_f64(self.a[e], self.dtype)
        return self.cache[e]


def act_to_np(t):
    import torch
    return t.detach().to(torch.float32).cpu().numpy()


def run_gpu(shape: LayerShape, inp: dict, *, capacity=None, backward=True):
    """Forward (+ backward) through moe_layer_fwd / moe_layer_bwd; returns host arrays."""
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import MoELayer, to_device
    dev = {k: to_device(v, shape) for k, v in inp.items() if k != "bias"}
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
    layer = MoELayer(shape, capacity=capacity)
    layer.forward(dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"])
    if backward and not shape.fwd_only:
        layer.backward(dev["dy"], dev["x"], dev["Wg"], dev["W1"], dev["W3"], dev["W2"])
    st = layer.status()
    assert st == moe.MOE_OK, moe.STATUS_NAMES.get(st, st)
    out = {n: layer.view(n).cpu().numpy() for n in
           ("logits", "topk_idx", "topk_w", "counts", "kept", "offsets", "slot", "row_token")}
    out["Xd_bits"] = layer.view("Xd").contiguous().view(
        __import__("torch").int16 if shape.dtype == BF16 else __import__("torch").int32).cpu().numpy()
    out["y"] = act_to_np(layer.y)
    if shape.aux_loss_coef:
        out["aux_loss"] = float(layer.view("aux_loss").cpu().numpy()[0])
    out["C"] = layer.L.capacity
    out["routed_row0"] = layer.L.routed_row0
    out["rows"] = layer.L.rows
    if backward and not shape.fwd_only:
        out["dx"] = act_to_np(layer.dx)
        out["dWg"] = layer.dWg.cpu().numpy()
        out["dW1"] = layer.dW1.cpu().numpy()
        out["dW2"] = layer.dW2.cpu().numpy()
        out["dW3"] = None if layer.dW3 is None else layer.dW3.cpu().numpy()
        out["dg"] = layer.scratch_view("dg").cpu().numpy()
    del layer
    return out


def check_routing(shape: LayerShape, gpu: dict, ol: np.ndarray):
    """Top-k bit-exact on the GPU's own logits; against the oracle's logits only near-ties
    (|difference| <= 1e-5) may differ.  Returns the GPU's expert ids (int64)."""
    gl = gpu["logits"].astype(np.float64)
    assert_close("logits", gl, ol, 1e-4)
    gidx = gpu["topk_idx"].astype(np.int64)
    assert np.array_equal(mo.select_topk(gl, shape.k), gidx), "top-k differs on identical logits"
    oidx = mo.select_topk(ol, shape.k)
    bad = np.nonzero(np.any(oidx != gidx, axis=1))[0]
    for t in bad:
        a = ol[t, oidx[t]]
        b = ol[t, gidx[t]]
        assert np.max(np.abs(a - b)) <= 1e-5, f"token {t}: routing differs outside a near-tie"
    return gidx


def check_dispatch(shape: LayerShape, gpu: dict, gidx: np.ndarray, x_bits: np.ndarray, C):
    """counts, kept, slot map and drop mask bit-exact against the oracle's dispatch of the same
    expert ids; the dispatched buffer holds exact copies of the token rows, padding rows zero."""
    counts, kept, pos = mo.dispatch(gidx, shape.E, C, choice_major=shape.choice_major)
    assert np.array_equal(gpu["counts"], counts)
    assert np.array_equal(gpu["kept"], kept)
    off = gpu["offsets"].astype(np.int64)
    assert off[0] == gpu["routed_row0"]
    seg = ((kept + ROW_ALIGN - 1) // ROW_ALIGN) * ROW_ALIGN
    assert np.array_equal(np.diff(off), seg)
    assert off[-1] <= gpu["rows"]
    slot = gpu["slot"].astype(np.int64)
    gpos = np.where(slot >= 0, slot - off[gidx], -1)
    assert np.array_equal(gpos, pos), "slot map / drop mask differs"
    rt = gpu["row_token"]
    T = shape.T
    kept_mask = slot >= 0
    tt = np.repeat(np.arange(T)[:, None], shape.k, axis=1)
    assert np.array_equal(rt[slot[kept_mask]], tt[kept_mask])
    Xd = gpu["Xd_bits"]
    assert np.array_equal(Xd[slot[kept_mask]], x_bits[tt[kept_mask]]), "dispatched rows not exact"
    for e in range(shape.E):
        r0, r1 = off[e] + kept[e], off[e + 1]
        assert np.all(rt[r0:r1] == -1)
        assert not np.any(Xd[r0:r1]), "padding rows must be zero"
    return C, counts, kept, pos


def x_bits_of(shape, inp):
    x = inp["x"]
    return x.view(np.int16) if shape.dtype == BF16 else x.view(np.int32)


def oracle_capacity(shape, capacity=None):
    from mixture_experts_layer_23_b200.configs import DROPLESS
    if capacity is None:
        return mo.capacity(shape.capacity_factor, shape.k, shape.T, shape.E)
    return None if capacity == DROPLESS else capacity


def full_compare(shape: LayerShape, seed=0, *, inp=None, capacity=None):
    """Whole-layer comparison (every output element) for shapes the oracle runs in seconds.
    capacity: an explicit C passed to the library (None: the capacity factor's)."""
    inp = make_inputs(shape, seed) if inp is None else inp
    gpu = run_gpu(shape, inp, capacity=capacity)
    dt = shape.dtype
    x, Wg = to_f64(inp["x"], dt), to_f64(inp["Wg"], dt)
    W1, W3, W2 = to_f64(inp["W1"], dt), to_f64(inp["W3"], dt), to_f64(inp["W2"], dt)
    ol = mo.gate_logits(x, Wg, inp["bias"])
    gidx = check_routing(shape, gpu, ol)
    C = oracle_capacity(shape, capacity)
    check_dispatch(shape, gpu, gidx, x_bits_of(shape, inp), C)
    f = mo.layer_forward(x, Wg, inp["bias"], W1, W3, W2, k=shape.k, act=shape.act,
                         gate_norm=shape.gate_norm, capacity_factor=shape.capacity_factor,
                         n_shared=shape.n_shared, idx_override=gidx, capacity_override=C,
                         aux_loss_coef=shape.aux_loss_coef, choice_major=shape.choice_major)
    rel = tol_for(shape)
    errs = {"topk_w": assert_close("topk_w", gpu["topk_w"], f["g"], rel),
            "y": assert_close("y", gpu["y"], f["y"], rel)}
    if shape.aux_loss_coef:
        # a scalar from fp32 softmax sums of fp32 logits: relative 1e-5
        want = f["aux_loss"]
        assert abs(gpu["aux_loss"] - want) <= 1e-5 * abs(want), (gpu["aux_loss"], want)
        errs["aux_loss"] = abs(gpu["aux_loss"] - want)
    if not shape.fwd_only:
        dy = to_f64(inp["dy"], dt)
        g = mo.layer_backward(f, x, Wg, W1, W3, W2, dy)
        for n in ("dx", "dWg", "dW1", "dW2", "dg"):
            errs[n] = assert_close(n, gpu[n], g[n], rel)
        if shape.act == SWIGLU:
            errs["dW3"] = assert_close("dW3", gpu["dW3"], g["dW3"], rel)
    return gpu, errs


def large_compare(shape: LayerShape, seed=0, *, full_dx=True, n_tok=24, n_f=3, experts=None):
    """Full-size layers.  Routing and dispatch in full (bit-exact).  y, dg and dWg in full, and
    dx in full when full_dx, from the oracle's one-expert-at-a-time form of the whole layer;
    otherwise dx on sampled tokens.  Rows of dW1/dW3 and columns of dW2 on sampled experts (each
    an exact sum over all of the expert's rows).  Returns the GPU outputs and the oracle's CPU
    seconds."""
    import time
    inp = make_inputs(shape, seed)
    gpu = run_gpu(shape, inp)
    dt = shape.dtype
    x, Wg = to_f64(inp["x"], dt), to_f64(inp["Wg"], dt)
    W1, W2 = LazyF64(inp["W1"], dt, keep=False), LazyF64(inp["W2"], dt, keep=False)
    W3 = None if inp["W3"] is None else LazyF64(inp["W3"], dt, keep=False)
    dy = None if shape.fwd_only else to_f64(inp["dy"], dt)
    r = mo.route(x, Wg, inp["bias"], k=shape.k, gate_norm=shape.gate_norm,
                 capacity_factor=shape.capacity_factor, choice_major=shape.choice_major)
    gidx = check_routing(shape, gpu, r["logits"])
    check_dispatch(shape, gpu, gidx, x_bits_of(shape, inp), r["C"])
    # downstream comparisons use the GPU's expert ids (identical unless a near-tie flipped)
    r["idx"] = gidx
    r["g"] = mo.gate_weights(r["logits"], gidx, shape.gate_norm)
    r["counts"], r["kept"], r["pos"] = mo.dispatch(gidx, shape.E, r["C"],
                                                   choice_major=shape.choice_major)
    rel = tol_for(shape)
    assert_close("topk_w", gpu["topk_w"], r["g"], rel)
    assert not shape.fwd_only
    t0 = time.perf_counter()
    f = mo.layer_by_expert(x, Wg, inp["bias"], W1, W3, W2, dy, k=shape.k, act=shape.act,
                           gate_norm=shape.gate_norm, capacity_factor=shape.capacity_factor,
                           n_shared=shape.n_shared, idx_override=gidx,
                           choice_major=shape.choice_major, aux_loss_coef=shape.aux_loss_coef,
                           with_dx=full_dx)
    cpu_s = time.perf_counter() - t0
    assert np.array_equal(f["pos"], r["pos"])
    assert_close("y", gpu["y"], f["y"], rel)
    assert_close("dg", gpu["dg"], f["dg"], rel)
    assert_close("dWg", gpu["dWg"], f["dWg"], rel)
    rng = np.random.default_rng(seed + 1)
    if full_dx:
        assert_close("dx", gpu["dx"], f["dx"], rel)
    else:
        dropped_tok = np.nonzero(np.any(r["pos"] < 0, axis=1))[0]
        picks = [0, shape.T - 1] + list(rng.choice(shape.T, n_tok, replace=False))
        if len(dropped_tok):
            picks += list(rng.choice(dropped_tok, min(4, len(dropped_tok)), replace=False))
        toks = sorted(set(int(t) for t in picks))
        _, dx, _ = mo.token_forward_backward(toks, r, x, Wg, W1, W3, W2, dy, act=shape.act,
                                             gate_norm=shape.gate_norm, n_shared=shape.n_shared)
        assert_close("dx[sampled]", gpu["dx"][toks], dx, rel)
    exps = experts if experts is not None else sorted(set([0, shape.E - 1, shape.E_tot - 1]))
    for e in exps:
        fs = sorted(set([0, shape.d_ff - 1] + list(rng.choice(shape.d_ff, n_f, replace=False))))
        a, b, c = mo.expert_weight_grad_rows(e, fs, r, x, W1, W3, W2, dy, act=shape.act,
                                             n_shared=shape.n_shared)
        assert_close(f"dW1[{e}][fs]", gpu["dW1"][e][fs], a, rel)
        assert_close(f"dW2[{e}][:,fs]", gpu["dW2"][e][:, fs], c, rel)
        if b is not None:
            assert_close(f"dW3[{e}][fs]", gpu["dW3"][e][fs], b, rel)
    return gpu, cpu_s
