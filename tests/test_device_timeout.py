"""Failure detection on the GPU without a fault: a bounded device wait that runs out.

Every wait of the tensor-core kernels on a barrier is bounded; when one runs out the CTA stops,
lets its own copies and MMAs in flight land, frees its tensor memory and sets a status word that
moe_read_status reports as MOE_ERR_DEVICE_TIMEOUT.  Here the library's test hook makes each
tensor-core kernel wait first on a barrier that nothing arrives on (a flag nothing sets), with a
2 ms budget, so the whole forward and backward pass takes that path.  The test checks that the
timeout is reported, that reading the status clears it, and that the same context, the same
layer object and the same buffers then give the oracle's results again.
"""
import numpy as np
import pytest

from mixture_experts_layer_23_b200.configs import BF16, SWIGLU, LayerShape
from mixture_experts_layer_23_b200.synth import make_inputs

pytestmark = pytest.mark.gpu

# bf16 with d and F multiples of 64: the router, the expert GEMMs and both router-backward
# contractions all run on the tcgen05 kernels that carry bounded waits
SHAPE = LayerShape("timeout_path", T=700, d=128, E=8, k=2, d_ff=192, n_shared=1, act=SWIGLU,
                   capacity_factor=1.0, dtype=BF16, bias="normal")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    from mixture_experts_layer_23_b200 import build
    build.build()
    yield


def test_wait_that_runs_out_is_reported_and_the_layer_recovers():
    import torch
    import parity
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import MoELayer, to_device
    assert moe.gemm_engine(moe.make_config(SHAPE)) == 1
    inp = make_inputs(SHAPE, 11)
    dev = {k: to_device(v, SHAPE) for k, v in inp.items() if k != "bias"}
    bias = torch.from_numpy(inp["bias"]).cuda()
    args = (dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"])
    layer = MoELayer(SHAPE)

    def step():
        layer.forward(*args)
        layer.backward(dev["dy"], dev["x"], dev["Wg"], dev["W1"], dev["W3"], dev["W2"])

    step()
    assert layer.status() == moe.MOE_OK
    y_ok, dx_ok = layer.y.clone(), layer.dx.clone()
    dW1_ok = layer.dW1.clone()

    moe.set_wait_budget_ns(2_000_000)
    moe.set_wait_stall(True)
    try:
        step()
        st = layer.status()
    finally:
        moe.set_wait_stall(False)
        moe.set_wait_budget_ns(2_000_000_000)
    assert st == 6, moe.STATUS_NAMES.get(st, st)       # MOE_ERR_DEVICE_TIMEOUT
    assert layer.status() == moe.MOE_OK                # the read cleared the status word
    # the aborted router wrote the placeholder routing (experts 0..k-1), so the rest of the
    # pass stayed in bounds
    assert torch.equal(layer.view("topk_idx").cpu(),
                       torch.arange(SHAPE.k, dtype=torch.int32).repeat(SHAPE.T, 1))

    # same context, same layer object, same buffers: a normal pass again
    step()
    assert layer.status() == moe.MOE_OK
    assert torch.equal(layer.y, y_ok)
    assert torch.equal(layer.dx, dx_ok)
    assert torch.equal(layer.dW1, dW1_ok)
    # and a fresh layer in the same context matches the oracle element by element
    parity.full_compare(SHAPE, seed=11, inp=inp)


def test_expert_ffn_alone_reports_the_timeout():
    """moe_expert_ffn (the grouped GEMMs of step 3, paired-CTA kernels) takes the same path."""
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import MoELayer, act_dtype, to_device
    inp = make_inputs(SHAPE, 12)
    dev = {k: to_device(v, SHAPE) for k, v in inp.items() if k != "bias"}
    bias = torch.from_numpy(inp["bias"]).cuda()
    layer = MoELayer(SHAPE)
    layer.forward(dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"])
    assert layer.status() == moe.MOE_OK
    R, F, d = layer.L.rows, SHAPE.d_ff, SHAPE.d
    dt = act_dtype(SHAPE)
    Gu, Gv, H = (torch.empty(R, F, dtype=dt, device="cuda") for _ in range(3))
    O = torch.empty(R, d, dtype=dt, device="cuda")
    moe.set_wait_budget_ns(1_000_000)
    moe.set_wait_stall(True)
    try:
        moe.expert_ffn(layer.cfg, layer.view("Xd"), dev["x"], layer.view("offsets"), dev["W1"],
                       dev["W3"], dev["W2"], Gu, Gv, H, O, layer.scratch)
        st = layer.status()
    finally:
        moe.set_wait_stall(False)
        moe.set_wait_budget_ns(2_000_000_000)
    assert st == 6, moe.STATUS_NAMES.get(st, st)
    moe.expert_ffn(layer.cfg, layer.view("Xd"), dev["x"], layer.view("offsets"), dev["W1"],
                   dev["W3"], dev["W2"], Gu, Gv, H, O, layer.scratch)
    assert layer.status() == moe.MOE_OK
    off = layer.view("offsets").cpu().numpy()
    rows = np.r_[np.arange(0, SHAPE.T), np.arange(off[0], off[-1])]
    assert torch.equal(O[rows], layer.view("O")[rows])
