"""Time the layer's step entry points alone, on a named layer's shapes.

    python -m mixture_experts_layer_23_b200.kernel_bench [--workload NAME] [--T T] [--E E]
        [--step route|dispatch|combine|experts|experts_bwd|all] [--iters N] [--warmup W]

Each step runs on the buffers it needs and nothing else (a few hundred MB for the HBM-bound steps
of the largest layer), so one launch can be captured with a profiler without the whole layer on
the device:
  route        moe_route on x                     (reads x and Wg, writes logits and the routing)
  dispatch     moe_dispatch_noalloc on x          (reads x, writes the dispatched rows)
  combine      moe_combine on random expert rows  (reads the kept and shared rows, writes y)
  experts      moe_expert_ffn on the dispatched rows (the up- and down-projection GEMMs)
  experts_bwd  moe_expert_ffn_bwd after it (activation-, input- and weight-gradient GEMMs)
--T and --E shrink the layer (fewer tokens or experts) to bound the device memory of the GEMM
steps.  The routing comes from moe_route on the workload's seeded inputs; the expert rows fed to
the combine and the output gradients fed to the backward are random (their values do not change
the cost).  Each timed launch is
bracketed by CUDA events on the launching stream, with an L2 flush between launches (a 256 MiB
write, then a 256 MiB read of a second buffer, so that L2 holds no dirty lines whose write-back
the next launch would pay for).  Prints one JSON line per step: average microseconds per launch, the step's algorithmic bytes
and the resulting GB/s.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import moe
from .configs import BY_NAME
from .layer import act_dtype, to_device
from .synth import make_inputs


class L2Flush:
    """256 MiB write, then 256 MiB read of another buffer: L2 ends up holding clean lines only."""

    def __init__(self):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(64 << 20, dtype=torch.int32, device="cuda")

    def __call__(self):
        self.w.zero_()
        torch.amax(self.r)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="mixtral_dropless")
    ap.add_argument("--step", default="all",
                    choices=["all", "route", "dispatch", "combine", "experts", "experts_bwd",
                             "layer"])
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--E", type=int, default=None)
    ap.add_argument("--F", type=int, default=None)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args(argv)
    shape = BY_NAME[a.workload]
    if a.T or a.E or a.F:
        shape = shape.with_(name=shape.name + "_reduced", T=a.T or shape.T, E=a.E or shape.E,
                            k=min(shape.k, a.E or shape.E), d_ff=a.F or shape.d_ff)
    if a.step == "layer":
        return run_layer(shape, a)
    gemm = a.step in ("experts", "experts_bwd")
    inp = make_inputs(shape, 0, with_dy=False)
    if not gemm:
        inp["W1"] = inp["W3"] = inp["W2"] = None
    cfg = moe.make_config(shape)
    L = moe.get_layout(cfg)
    T, d, E, k, R = shape.T, shape.d, shape.E, shape.k, L.rows
    dt = act_dtype(shape)
    b = 2 if shape.dtype == 1 else 4
    x, Wg = to_device(inp["x"], shape), to_device(inp["Wg"], shape)
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
    i32 = dict(dtype=torch.int32, device="cuda")
    logits = torch.empty(T, E, device="cuda")
    idx = torch.empty(T, k, **i32)
    w = torch.empty(T, k, device="cuda")
    counts, kept = torch.empty(E, **i32), torch.empty(E, **i32)
    offsets, slot = torch.empty(E + 1, **i32), torch.empty(T, k, **i32)
    row_token = torch.empty(R, **i32)
    flush = L2Flush()
    stream = torch.cuda.current_stream()

    def route():
        moe.route(cfg, x, Wg, bias, logits, idx, w)

    route()
    Xd = torch.empty(R, d, dtype=dt, device="cuda")

    def dispatch():
        moe.dispatch_noalloc(cfg, x, idx, counts, kept, offsets, slot, row_token, Xd)

    dispatch()
    torch.cuda.synchronize()
    n_kept = int(kept.sum().item())
    del Xd
    O = torch.randn(R, d, device="cuda").to(dt)
    y = torch.empty(T, d, dtype=dt, device="cuda")

    def combine():
        moe.combine(cfg, O, slot, w, y)

    Td, Nd = T * d * b, n_kept * d * b
    F, Et, S = shape.d_ff, shape.E_tot, shape.n_shared
    g = 2 if shape.act == 1 else 1
    rows = n_kept + S * T
    if gemm:
        W1, W2 = to_device(inp["W1"], shape), to_device(inp["W2"], shape)
        W3 = to_device(inp["W3"], shape)
        del O
        Xd = torch.empty(R, d, dtype=dt, device="cuda")
        dispatch()
        Gu, H = (torch.empty(R, F, dtype=dt, device="cuda") for _ in range(2))
        Gv = torch.empty(R, F, dtype=dt, device="cuda") if W3 is not None else None
        O = torch.empty(R, d, dtype=dt, device="cuda")
        scratch = torch.zeros(L.scratch_bytes, dtype=torch.uint8, device="cuda")

        def experts():
            moe.expert_ffn(cfg, Xd, x, offsets, W1, W3, W2, Gu, Gv, H, O, scratch)

        experts()
        dO = (0.1 * torch.randn(R, d, device="cuda")).to(dt)
        dy = (0.1 * torch.randn(T, d, device="cuda")).to(dt)
        dXd = torch.empty(R, d, dtype=dt, device="cuda")
        dW1 = torch.empty(Et, F, d, device="cuda")
        dW3 = torch.empty(Et, F, d, device="cuda") if W3 is not None else None
        dW2 = torch.empty(Et, d, F, device="cuda")

        def experts_bwd():
            moe.expert_ffn_bwd(cfg, dO, dy, Xd, x, offsets, W1, W3, W2, Gu, Gv, H, dXd, dW1, dW3,
                               dW2, scratch)
    else:
        experts = experts_bwd = None
    steps = {
        "route": (route, Td + E * d * b + T * E * 4 + T * k * 8),
        "dispatch": (dispatch, Td + Nd + T * k * 8),
        "combine": (combine, Nd + shape.n_shared * Td + Td + T * k * 8),
        "experts": (experts, 2.0 * rows * d * F * (g + 1)),
        "experts_bwd": (experts_bwd, 2.0 * rows * d * F * (2 * g + 2)),
    }
    if a.step in ("dispatch", "all") and not gemm:
        Xd = torch.empty(R, d, dtype=dt, device="cuda")   # for the dispatch runs below
    scratch_status = (lambda: moe.read_status(scratch)) if gemm else None
    for name, (fn, nbytes) in steps.items():
        if a.step not in ("all", name) or fn is None:
            continue
        for _ in range(a.warmup):
            fn()
            flush()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(a.iters)]
        torch.cuda.synchronize()
        for s, e in ev:
            s.record(stream)
            fn()
            e.record(stream)
            flush()
        torch.cuda.synchronize()
        us = 1e3 * sum(s.elapsed_time(e) for s, e in ev) / a.iters
        line = {"workload": shape.name, "step": name, "us_per_launch": us,
                "kept_assignments": n_kept}
        if name in ("experts", "experts_bwd"):
            line.update(flops=nbytes, tflops=nbytes / (us * 1e-6) / 1e12)
        else:
            line.update(algorithmic_bytes=nbytes, gbs=nbytes / (us * 1e-6) / 1e9)
        if scratch_status is not None:
            line["status"] = scratch_status()
        print(json.dumps(line), flush=True)


def run_layer(shape, a):
    """The whole layer, forward + backward (MoELayer), on the given shape: for captures of the
    backward's HBM-bound kernels on a layer whose experts are shrunk (--F) to bound memory."""
    from .layer import MoELayer
    inp = make_inputs(shape, 0)
    dev = {k: to_device(v, shape) for k, v in inp.items() if k != "bias"}
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
    layer = MoELayer(shape)
    flush = L2Flush()

    def step():
        layer.forward(dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"])
        layer.backward(dev["dy"], dev["x"], dev["Wg"], dev["W1"], dev["W3"], dev["W2"])

    for _ in range(a.warmup):
        step()
        flush()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(a.iters)]
    torch.cuda.synchronize()
    for s_, e_ in ev:
        s_.record()
        step()
        e_.record()
        flush()
    torch.cuda.synchronize()
    us = 1e3 * sum(s_.elapsed_time(e_) for s_, e_ in ev) / a.iters
    print(json.dumps({"workload": shape.name, "step": "layer", "us_per_step": us,
                      "status": layer.status()}), flush=True)


if __name__ == "__main__":
    main()
