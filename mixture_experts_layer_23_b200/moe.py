"""Python binding of libmoe.so: argument marshalling only.

Every function here forwards torch tensors (device pointers) and the current CUDA stream to the
C entry point of the same name in include/moe.h.  All arithmetic runs in the library's CUDA
kernels; there is no fallback.  If libmoe.so is missing or fails to load, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os

from .configs import BF16, DROPLESS, LayerShape

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_MISALIGNED", 4: "MOE_ERR_WORKSPACE_TOO_SMALL", 5: "MOE_ERR_CUDA",
                6: "MOE_ERR_DEVICE_TIMEOUT"}

# Every symbol include/moe.h declares.
EXPORTS = ("moe_get_layout", "moe_workspace_size", "moe_route", "moe_route_from_logits",
           "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_layer_fwd", "moe_layer_bwd",
           "moe_scratch_grad_offsets", "moe_read_status", "moe_status_string", "moe_gemm_engine",
           "moe_kernel_launches", "moe_set_profile_events", "moe_dispatch_noalloc",
           "moe_last_cuda_error", "moe_aux_loss", "moe_layer_fwd_fused",
           "moe_set_wait_budget_ns", "moe_set_wait_stall", "moe_combine_bwd",
           "moe_expert_ffn_bwd", "moe_router_bwd", "moe_layer_step_host")

FWD_PHASES = ("router", "dispatch", "expert_up", "expert_down", "combine")
BWD_PHASES = ("combine_bwd", "router_bwd", "dgrad_h", "dgrad_x", "wgrad_w1", "wgrad_w2",
              "undispatch")


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = _lib.moe_status_string(status).decode()
        if status == 5:
            detail += "; " + _lib.moe_last_cuda_error().decode()
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({detail})")


class Config(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("act", ctypes.c_int32), ("gate_norm", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("capacity", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("has_bias", ctypes.c_int32),
                ("aux_loss_coef", ctypes.c_float), ("drop_order", ctypes.c_int32)]


class Layout(ctypes.Structure):
    _fields_ = [("capacity", ctypes.c_int64), ("T_pad", ctypes.c_int64), ("rows", ctypes.c_int64),
                ("routed_row0", ctypes.c_int64), ("max_group_rows", ctypes.c_int64)] + [
        (n, ctypes.c_size_t) for n in (
            "ctx_logits", "ctx_topk_idx", "ctx_topk_w", "ctx_counts", "ctx_kept", "ctx_offsets",
            "ctx_slot", "ctx_row_token", "ctx_Xd", "ctx_Gu", "ctx_Gv", "ctx_H", "ctx_O",
            "ctx_bytes", "scratch_bytes", "ctx_aux_loss")]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libmoe.so not built ({_LIB_PATH}); run "
                          "`python -m mixture_experts_layer_23_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    CP = ctypes.POINTER(Config)
    sig = {
        "moe_get_layout": [CP, ctypes.POINTER(Layout)],
        "moe_workspace_size": [CP, ctypes.POINTER(SZ), ctypes.POINTER(SZ)],
        "moe_route": [CP, P, P, P, P, P, P, P],
        "moe_route_from_logits": [CP, P, P, P, P],
        "moe_aux_loss": [CP, P, P, P, P, P],
        "moe_layer_fwd_fused": [CP, P, P, P, P, P, P, P, P, P, P, P],
        "moe_dispatch": [CP, P, P, P, P, P, P, P, P, P, P],
        "moe_dispatch_noalloc": [CP, P, P, P, P, P, P, P, P, P],
        "moe_expert_ffn": [CP, P, P, P, P, P, P, P, P, P, P, P, P],
        "moe_combine": [CP, P, P, P, P, P],
        "moe_layer_fwd": [CP, P, P, P, P, P, P, P, P, P, P],
        "moe_layer_bwd": [CP, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "moe_scratch_grad_offsets": [CP, ctypes.POINTER(SZ), ctypes.POINTER(SZ)],
        "moe_read_status": [P, P],
        "moe_status_string": [I32],
        "moe_gemm_engine": [CP],
        "moe_kernel_launches": [],
        "moe_set_profile_events": [P, P],
        "moe_last_cuda_error": [],
        "moe_set_wait_budget_ns": [ctypes.c_uint64],
        "moe_set_wait_stall": [I32],
        "moe_combine_bwd": [CP, P, P, P, P, P],
        "moe_expert_ffn_bwd": [CP, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P],
        "moe_router_bwd": [CP, P, P, P, P, P, P, P, P],
        "moe_layer_step_host": [CP] + [P] * 20,
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = I32
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_kernel_launches.restype = ctypes.c_int64
    lib.moe_last_cuda_error.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib():
    return _lib


def lib_path() -> str:
    return _LIB_PATH


# ----------------------------------------------------------------------------- helpers

def make_config(shape: LayerShape, capacity: int | None = None) -> Config:
    """The C config of a LayerShape.  capacity None: derived from the capacity factor (or
    dropless when the shape has none)."""
    if capacity is None:
        capacity = DROPLESS if shape.dropless else -1
    return Config(T=shape.T, d=shape.d, E=shape.E, k=shape.k, d_ff=shape.d_ff,
                  n_shared=shape.n_shared, act=shape.act, gate_norm=shape.gate_norm,
                  capacity_factor=0.0 if shape.dropless else float(shape.capacity_factor),
                  capacity=capacity, dtype=shape.dtype, has_bias=int(shape.bias != "none"),
                  aux_loss_coef=float(shape.aux_loss_coef), drop_order=int(shape.choice_major))


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoEError(st, where)


def get_layout(cfg: Config) -> Layout:
    L = Layout()
    _check(_lib.moe_get_layout(ctypes.byref(cfg), ctypes.byref(L)), "moe_get_layout")
    return L


def workspace_size(cfg: Config):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(a), ctypes.byref(b)),
           "moe_workspace_size")
    return a.value, b.value


def scratch_grad_offsets(cfg: Config):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.moe_scratch_grad_offsets(ctypes.byref(cfg), ctypes.byref(a), ctypes.byref(b)),
           "moe_scratch_grad_offsets")
    return a.value, b.value


def gemm_engine(cfg: Config) -> int:
    return _lib.moe_gemm_engine(ctypes.byref(cfg))


def route(cfg, x, Wg, bias, logits, topk_idx, topk_w, stream=None):
    _check(_lib.moe_route(ctypes.byref(cfg), _p(x), _p(Wg), _p(bias), _p(logits), _p(topk_idx),
                          _p(topk_w), _stream(stream)), "moe_route")


def layer_fwd_fused(cfg, x, Wg, bias, W1, W3, W2, y, topk_idx=None, topk_w=None, counts=None,
                    stream=None):
    _check(_lib.moe_layer_fwd_fused(ctypes.byref(cfg), _p(x), _p(Wg), _p(bias), _p(W1), _p(W3),
                                    _p(W2), _p(y), _p(topk_idx), _p(topk_w), _p(counts),
                                    _stream(stream)), "moe_layer_fwd_fused")


def aux_loss(cfg, logits, counts, loss, scratch, stream=None):
    _check(_lib.moe_aux_loss(ctypes.byref(cfg), _p(logits), _p(counts), _p(loss), _p(scratch),
                             _stream(stream)), "moe_aux_loss")


def route_from_logits(cfg, logits, topk_idx, topk_w, stream=None):
    _check(_lib.moe_route_from_logits(ctypes.byref(cfg), _p(logits), _p(topk_idx), _p(topk_w),
                                      _stream(stream)), "moe_route_from_logits")


def dispatch(cfg, x, topk_idx, counts, kept, offsets, slot, row_token, Xd, scratch, stream=None):
    _check(_lib.moe_dispatch(ctypes.byref(cfg), _p(x), _p(topk_idx), _p(counts), _p(kept),
                             _p(offsets), _p(slot), _p(row_token), _p(Xd), _p(scratch),
                             _stream(stream)), "moe_dispatch")


def dispatch_noalloc(cfg, x, topk_idx, counts, kept, offsets, slot, row_token, Xd, stream=None):
    """moe_dispatch without a scratch argument (for callers that cannot allocate; see moe.h)."""
    _check(_lib.moe_dispatch_noalloc(ctypes.byref(cfg), _p(x), _p(topk_idx), _p(counts), _p(kept),
                                     _p(offsets), _p(slot), _p(row_token), _p(Xd),
                                     _stream(stream)), "moe_dispatch_noalloc")


def expert_ffn(cfg, Xd, x, offsets, W1, W3, W2, Gu, Gv, H, O, scratch, stream=None):
    _check(_lib.moe_expert_ffn(ctypes.byref(cfg), _p(Xd), _p(x), _p(offsets), _p(W1), _p(W3),
                               _p(W2), _p(Gu), _p(Gv), _p(H), _p(O), _p(scratch), _stream(stream)),
           "moe_expert_ffn")


def combine(cfg, O, slot, topk_w, y, stream=None):
    _check(_lib.moe_combine(ctypes.byref(cfg), _p(O), _p(slot), _p(topk_w), _p(y),
                            _stream(stream)), "moe_combine")


def layer_fwd(cfg, x, Wg, bias, W1, W3, W2, y, ctx, scratch, stream=None):
    _check(_lib.moe_layer_fwd(ctypes.byref(cfg), _p(x), _p(Wg), _p(bias), _p(W1), _p(W3), _p(W2),
                              _p(y), _p(ctx), _p(scratch), _stream(stream)), "moe_layer_fwd")


def layer_bwd(cfg, ctx, dy, x, Wg, W1, W3, W2, dx, dWg, dW1, dW3, dW2, scratch, stream=None):
    _check(_lib.moe_layer_bwd(ctypes.byref(cfg), _p(ctx), _p(dy), _p(x), _p(Wg), _p(W1), _p(W3),
                              _p(W2), _p(dx), _p(dWg), _p(dW1), _p(dW3), _p(dW2), _p(scratch),
                              _stream(stream)), "moe_layer_bwd")


def combine_bwd(cfg, ctx, dy, dO, scratch, stream=None):
    _check(_lib.moe_combine_bwd(ctypes.byref(cfg), _p(ctx), _p(dy), _p(dO), _p(scratch),
                                _stream(stream)), "moe_combine_bwd")


def expert_ffn_bwd(cfg, dO, dy, Xd, x, offsets, W1, W3, W2, Gu, Gv, H, dXd, dW1, dW3, dW2,
                   scratch, stream=None):
    _check(_lib.moe_expert_ffn_bwd(ctypes.byref(cfg), _p(dO), _p(dy), _p(Xd), _p(x), _p(offsets),
                                   _p(W1), _p(W3), _p(W2), _p(Gu), _p(Gv), _p(H), _p(dXd),
                                   _p(dW1), _p(dW3), _p(dW2), _p(scratch), _stream(stream)),
           "moe_expert_ffn_bwd")


def router_bwd(cfg, ctx, x, Wg, dXd, dx, dWg, scratch, stream=None):
    _check(_lib.moe_router_bwd(ctypes.byref(cfg), _p(ctx), _p(x), _p(Wg), _p(dXd), _p(dx),
                               _p(dWg), _p(scratch), _stream(stream)), "moe_router_bwd")


def layer_step_host(cfg, x_host, dy_host, y_host, dx_host, x_dev, dy_dev, Wg, bias, W1, W3, W2,
                    y_dev, dx_dev, dWg, dW1, dW3, dW2, ctx, scratch, stream=None):
    """One forward + backward from pinned host x, dy to host y, dx (moe_layer_step_host)."""
    _check(_lib.moe_layer_step_host(ctypes.byref(cfg), _p(x_host), _p(dy_host), _p(y_host),
                                    _p(dx_host), _p(x_dev), _p(dy_dev), _p(Wg), _p(bias), _p(W1),
                                    _p(W3), _p(W2), _p(y_dev), _p(dx_dev), _p(dWg), _p(dW1),
                                    _p(dW3), _p(dW2), _p(ctx), _p(scratch), _stream(stream)),
           "moe_layer_step_host")


def read_status(scratch, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status (MOE_OK when clean)."""
    return _lib.moe_read_status(_stream(stream), _p(scratch))


def kernel_launches() -> int:
    """Kernels libmoe.so has launched in this process so far."""
    return int(_lib.moe_kernel_launches())


def set_profile_events(fwd_events=None, bwd_events=None):
    """Install (or clear, with None) per-phase CUDA events for moe_layer_fwd / moe_layer_bwd.
    Each is a list of torch.cuda.Event (timing enabled) or None (boundary not recorded),
    len(phases) + 1 long; the arrays are kept alive on this module until cleared."""
    global _prof_keep

    def arr(evs, n):
        if evs is None:
            return None
        assert len(evs) == n + 1
        for e in evs:
            if e is not None and not e.cuda_event:  # torch creates the event on first record
                e.record()
        return (ctypes.c_void_p * (n + 1))(*[None if e is None else e.cuda_event for e in evs])
    a, b = arr(fwd_events, len(FWD_PHASES)), arr(bwd_events, len(BWD_PHASES))
    _prof_keep = (a, b, fwd_events, bwd_events)
    _check(_lib.moe_set_profile_events(a, b), "moe_set_profile_events")


_prof_keep = None


def set_wait_budget_ns(budget_ns: int) -> None:
    _check(_lib.moe_set_wait_budget_ns(int(budget_ns)), "moe_set_wait_budget_ns")


def set_wait_stall(on: bool) -> None:
    _check(_lib.moe_set_wait_stall(1 if on else 0), "moe_set_wait_stall")
