"""Device-side convenience around the C ABI: workspace allocation (torch), uploads of host
inputs and typed views of the saved forward state.  Marshalling only; the layer's arithmetic
is all in libmoe.so."""
from __future__ import annotations

import numpy as np
import torch

from . import moe
from .configs import BF16, SWIGLU, LayerShape

INT32 = torch.int32


def act_dtype(shape: LayerShape):
    return torch.bfloat16 if shape.dtype == BF16 else torch.float32


def to_device(a, shape: LayerShape, device="cuda", pin=False):
    """Storage-form numpy array (float32 or bf16 bits) -> torch tensor on `device`."""
    if a is None:
        return None
    if a.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    if pin:
        return t.pin_memory()
    return t.to(device)


class MoELayer:
    """One layer's workspaces on one device."""

    def __init__(self, shape: LayerShape, device="cuda", capacity=None):
        self.shape = shape
        self.cfg = moe.make_config(shape, capacity)
        self.L = moe.get_layout(self.cfg)
        self.device = torch.device(device)
        self.dt = act_dtype(shape)
        self.ctx = torch.empty(self.L.ctx_bytes, dtype=torch.uint8, device=self.device)
        self.scratch = torch.zeros(self.L.scratch_bytes, dtype=torch.uint8, device=self.device)
        T, d, E, F, Et = shape.T, shape.d, shape.E, shape.d_ff, shape.E_tot
        self.y = torch.empty(T, d, dtype=self.dt, device=self.device)
        self.dx = torch.empty(T, d, dtype=self.dt, device=self.device)
        self.dWg = torch.empty(E, d, dtype=torch.float32, device=self.device)
        self.dW1 = torch.empty(Et, F, d, dtype=torch.float32, device=self.device)
        self.dW3 = (torch.empty(Et, F, d, dtype=torch.float32, device=self.device)
                    if shape.act == SWIGLU else None)
        self.dW2 = torch.empty(Et, d, F, dtype=torch.float32, device=self.device)

    # typed views into ctx
    def _view(self, off, dtype, shape):
        n = int(np.prod(shape))
        esz = torch.tensor([], dtype=dtype).element_size()
        return self.ctx[off: off + n * esz].view(dtype).view(*shape)

    def view(self, name):
        s, L = self.shape, self.L
        R = L.rows
        table = {
            "logits": (L.ctx_logits, torch.float32, (s.T, s.E)),
            "topk_idx": (L.ctx_topk_idx, INT32, (s.T, s.k)),
            "topk_w": (L.ctx_topk_w, torch.float32, (s.T, s.k)),
            "counts": (L.ctx_counts, INT32, (s.E,)),
            "kept": (L.ctx_kept, INT32, (s.E,)),
            "offsets": (L.ctx_offsets, INT32, (s.E + 1,)),
            "slot": (L.ctx_slot, INT32, (s.T, s.k)),
            "row_token": (L.ctx_row_token, INT32, (R,)),
            "Xd": (L.ctx_Xd, self.dt, (R, s.d)),
            "Gu": (L.ctx_Gu, self.dt, (R, s.d_ff)),
            "Gv": (L.ctx_Gv, self.dt, (R, s.d_ff)),
            "H": (L.ctx_H, self.dt, (R, s.d_ff)),
            "O": (L.ctx_O, self.dt, (R, s.d)),
            "aux_loss": (L.ctx_aux_loss, torch.float32, (1,)),
        }
        off, dt, shp = table[name]
        return self._view(off, dt, shp)

    def scratch_view(self, name):
        dg_off, dl_off = moe.scratch_grad_offsets(self.cfg)
        s = self.shape
        if name == "dg":
            return self.scratch[dg_off: dg_off + s.T * s.k * 4].view(torch.float32).view(s.T, s.k)
        if name == "dlogits":
            return self.scratch[dl_off: dl_off + s.T * s.E * 4].view(torch.float32).view(s.T, s.E)
        raise KeyError(name)

    def forward(self, x, Wg, bias, W1, W3, W2, stream=None):
        moe.layer_fwd(self.cfg, x, Wg, bias, W1, W3, W2, self.y, self.ctx, self.scratch, stream)
        return self.y

    def backward(self, dy, x, Wg, W1, W3, W2, stream=None):
        moe.layer_bwd(self.cfg, self.ctx, dy, x, Wg, W1, W3, W2, self.dx, self.dWg, self.dW1,
                      self.dW3, self.dW2, self.scratch, stream)
        return self.dx

    def status(self, stream=None) -> int:
        return moe.read_status(self.scratch, stream)


class MoEFunction(torch.autograd.Function):
    """torch.autograd wrapper around one MoELayer: forward through moe_layer_fwd, backward through
    moe_layer_bwd.  Convenience only: the returned y is a copy of the layer's output buffer, and
    weight gradients (fp32 in the library) are cast to each weight's dtype, as autograd requires.
    The logit bias is a constant (no gradient).  Usage: y = MoEFunction.apply(x, Wg, W1, W3, W2,
    layer, bias) with W3 None for GELU layers."""

    @staticmethod
    def forward(ctx, x, Wg, W1, W3, W2, layer, bias):
        x = x.contiguous()
        y = layer.forward(x, Wg, bias, W1, W3, W2).clone()
        ctx.layer = layer
        ctx.has_w3 = W3 is not None
        ctx.save_for_backward(x, Wg, W1, W3 if W3 is not None else x.new_empty(0), W2)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, Wg, W1, W3, W2 = ctx.saved_tensors
        W3 = W3 if ctx.has_w3 else None
        L = ctx.layer
        L.backward(dy.contiguous(), x, Wg, W1, W3, W2)
        return (L.dx.clone(), L.dWg.to(Wg.dtype), L.dW1.to(W1.dtype),
                None if W3 is None else L.dW3.to(W3.dtype), L.dW2.to(W2.dtype), None, None)


class MoEStepGraph:
    """One forward (+ backward) of a MoELayer captured into a CUDA graph and replayed.

    The library's launches, their programmatic-dependent-launch edges included, are recorded once
    from the current torch stream; replay() re-issues them with one call, without the host cost of
    each launch.  Every buffer is fixed at capture: to run a new batch, copy it into the same x and
    dy tensors before replay().  Outputs land in the layer's buffers (layer.y, layer.dx, layer.dWg,
    ...), as with direct calls."""

    def __init__(self, layer, x, Wg, bias, W1, W3, W2, dy=None):
        self.layer = layer
        args = (x, Wg, bias, W1, W3, W2)

        def run():
            layer.forward(*args)
            if dy is not None:
                layer.backward(dy, x, Wg, W1, W3, W2)

        side = torch.cuda.Stream(device=layer.device)
        side.wait_stream(torch.cuda.current_stream(layer.device))
        with torch.cuda.stream(side):   # one eager pass first: one-time host set-up stays out of the graph
            run()
        torch.cuda.current_stream(layer.device).wait_stream(side)
        torch.cuda.synchronize(layer.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            run()

    def replay(self):
        self.graph.replay()
