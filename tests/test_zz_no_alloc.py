"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device memory.

Some callers cannot hand the library a scratch buffer (a framework that owns all device memory
through its own pool, a deployment whose memory is budgeted once at start-up, a loop that cannot
afford an allocation).  For them the library keeps the dispatch's only scratch, the per-CTA
expert histograms, in a fixed array of its own.  This file checks, through the C ABI, that the
no-allocation call gives exactly what moe_dispatch gives (dispatch outputs are integers and
copied rows: bit-exact), on two calls in a row, and that configs beyond the array's size are
refused.  It is collected last and passes both alone and after the other tests.
"""
import ctypes

import numpy as np
import pytest

from mixture_experts_layer_23_b200.configs import BF16, FP32, LayerShape
from mixture_experts_layer_23_b200.synth import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    from mixture_experts_layer_23_b200 import build
    build.build()
    yield


def _dispatch_both(shape, seed):
    """Route once, then dispatch with moe_dispatch (caller scratch) and with moe_dispatch_noalloc;
    output buffers start from different fill values so every compared element was written."""
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import act_dtype, to_device
    inp = make_inputs(shape, seed, with_dy=False)
    cfg = moe.make_config(shape)
    L = moe.get_layout(cfg)
    T, E, k, d, R = shape.T, shape.E, shape.k, shape.d, L.rows
    x, Wg = to_device(inp["x"], shape), to_device(inp["Wg"], shape)
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
    logits = torch.empty(T, E, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, device="cuda")
    moe.route(cfg, x, Wg, bias, logits, idx, w)

    def outputs(fill):
        i32 = dict(dtype=torch.int32, device="cuda")
        return dict(counts=torch.full((E,), fill, **i32), kept=torch.full((E,), fill, **i32),
                    offsets=torch.full((E + 1,), fill, **i32), slot=torch.full((T, k), fill, **i32),
                    row_token=torch.full((R,), fill, **i32),
                    Xd=torch.full((R, d), float(fill), dtype=act_dtype(shape), device="cuda"))

    ref, got = outputs(-7), outputs(11)
    scratch = torch.zeros(L.scratch_bytes, dtype=torch.uint8, device="cuda")
    moe.dispatch(cfg, x, idx, ref["counts"], ref["kept"], ref["offsets"], ref["slot"],
                 ref["row_token"], ref["Xd"], scratch)
    moe.dispatch_noalloc(cfg, x, idx, got["counts"], got["kept"], got["offsets"], got["slot"],
                         got["row_token"], got["Xd"])
    torch.cuda.synchronize()
    return L, ref, got


def _assert_same(L, ref, got, E):
    import torch
    for name in ("counts", "kept", "offsets", "slot"):
        assert torch.equal(ref[name], got[name]), name
    end = int(ref["offsets"][E].item())
    r0 = int(L.routed_row0)
    # the rows the dispatch defines: shared rows' row_token, every routed row and its tokens
    assert torch.equal(ref["row_token"][:end], got["row_token"][:end])
    assert torch.equal(ref["Xd"][r0:end].view(torch.int16 if ref["Xd"].element_size() == 2
                                              else torch.int32),
                       got["Xd"][r0:end].view(torch.int16 if got["Xd"].element_size() == 2
                                              else torch.int32))


SHAPES = [
    # a large call first, so the second call runs over a fuller array than it needs
    LayerShape("noalloc_big", T=8192, d=256, E=64, k=6, d_ff=64, n_shared=1, capacity_factor=1.0,
               dtype=BF16, bias="zipf"),
    LayerShape("noalloc_small", T=700, d=64, E=8, k=2, d_ff=64, capacity_factor=1.25,
               dtype=FP32),
    # choice-major drops keep one histogram layer per choice index in the array
    LayerShape("noalloc_choice_major", T=2000, d=64, E=32, k=4, d_ff=64, capacity_factor=0.7,
               dtype=BF16, bias="normal", choice_major=True),
]


def test_noalloc_dispatch_matches_dispatch_on_two_calls_in_a_row():
    for i, shape in enumerate(SHAPES):
        L, ref, got = _dispatch_both(shape, seed=10 + i)
        _assert_same(L, ref, got, shape.E)


def test_noalloc_dispatch_repeated_call_same_shape():
    shape = SHAPES[0].with_(name="noalloc_repeat", T=3000, E=32, k=4)
    for seed in (1, 2):
        L, ref, got = _dispatch_both(shape, seed=seed)
        _assert_same(L, ref, got, shape.E)


def _refused(shape):
    from mixture_experts_layer_23_b200 import moe
    cfg = moe.make_config(shape)
    fake = 1 << 20  # aligned, never dereferenced: the size check comes before any CUDA call
    st = moe.lib().moe_dispatch_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake,
                                        fake, fake, None)
    return st == 4  # MOE_ERR_WORKSPACE_TOO_SMALL


# ceil(T / 256) * E = 256 * 256 = 65536 histogram entries: exactly the array in token order
AT_LIMIT = LayerShape("noalloc_at_limit", T=65536, d=64, E=256, k=2, d_ff=64,
                      capacity_factor=1.0, dtype=BF16)


def test_noalloc_dispatch_refuses_configs_beyond_its_array():
    assert _refused(LayerShape("too_big", T=1 << 20, d=64, E=256, k=2, d_ff=64, dtype=BF16))
    # the same size in token order fits exactly; choice-major needs k layers of it, which do not
    assert _refused(AT_LIMIT.with_(name="at_limit_choice_major", choice_major=True))
    assert _refused(AT_LIMIT.with_(name="one_block_more", T=65536 + 1))


def test_noalloc_dispatch_at_its_size_limit():
    L, ref, got = _dispatch_both(AT_LIMIT, seed=21)
    _assert_same(L, ref, got, AT_LIMIT.E)
