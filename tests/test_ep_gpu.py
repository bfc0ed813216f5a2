"""Expert parallelism on one GPU: N ranks emulated in one process (ep.step_local), every step
through the library's kernels and every exchange a device-to-device copy of the same row blocks
the distributed exchange moves.

Each rank's y and dx must equal, bit for bit, the single-device layer run on that rank's own
batch (the expert GEMMs compute each row the same way wherever its block sits); each expert's
weight gradient, which sums rows from every rank in one GEMM, and the router gradient summed over
ranks are compared with the oracle within the bf16 tolerance.
"""
import numpy as np
import pytest

from mixture_experts_layer_23_b200.configs import BF16, GELU, SWIGLU, LayerShape
from mixture_experts_layer_23_b200.synth import make_inputs, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    from mixture_experts_layer_23_b200 import build
    build.build()
    yield


CASES = [
    # (shape of one rank's batch, ranks, chunks)
    (LayerShape("ep_swiglu", T=600, d=128, E=8, k=2, d_ff=192, act=SWIGLU, capacity_factor=1.0,
                dtype=BF16, bias="normal"), 2, 1),
    (LayerShape("ep_gelu_chunks", T=500, d=256, E=8, k=2, d_ff=128, act=GELU,
                capacity_factor=0.8, dtype=BF16, bias="zipf"), 4, 2),
    (LayerShape("ep_dropless_renorm", T=333, d=64, E=16, k=4, d_ff=64, act=SWIGLU, gate_norm=1,
                capacity_factor=None, dtype=BF16), 4, 4),
]


@pytest.mark.parametrize("shape,world,chunks", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_ep_matches_single_device_layers(shape, world, chunks):
    import torch
    import parity
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.ep import EPRank, step_local
    from mixture_experts_layer_23_b200.layer import MoELayer, to_device
    from oracle import moe_oracle as mo
    El = shape.E // world
    base = make_inputs(shape, 0)          # weights shared by every rank
    batches = [make_inputs(shape, 100 + q) for q in range(world)]   # each rank's x and dy
    dev = lambda a: to_device(a, shape)
    Wg, W1, W3, W2 = dev(base["Wg"]), dev(base["W1"]), dev(base["W3"]), dev(base["W2"])
    bias = None if base["bias"] is None else torch.from_numpy(base["bias"]).cuda()
    xs = [dev(b["x"]) for b in batches]
    dys = [dev(b["dy"]) for b in batches]
    Wl = [(W1[q * El:(q + 1) * El], None if W3 is None else W3[q * El:(q + 1) * El],
           W2[q * El:(q + 1) * El]) for q in range(world)]
    F, d = shape.d_ff, shape.d
    grads = [(torch.empty(El, F, d, device="cuda"),
              torch.empty(El, F, d, device="cuda") if W3 is not None else None,
              torch.empty(El, d, F, device="cuda")) for _ in range(world)]
    ranks = [EPRank(shape, q, world, chunks=chunks) for q in range(world)]
    ys, dxs, dWg = step_local(ranks, xs, Wg, bias, Wl, dys, grads)
    torch.cuda.synchronize()
    for r in ranks:
        assert r.status() == moe.MOE_OK
    # each rank against the single-device layer on its own batch
    dW_sum = {n: 0 for n in ("dW1", "dW3", "dW2")}
    dWg_ref = 0
    for q in range(world):
        one = MoELayer(shape)
        one.forward(xs[q], Wg, bias, W1, W3, W2)
        one.backward(dys[q], xs[q], Wg, W1, W3, W2)
        assert one.status() == moe.MOE_OK
        assert torch.equal(ys[q], one.y), q
        assert torch.equal(dxs[q], one.dx), q
        assert torch.equal(ranks[q].tok.view("slot"), one.view("slot"))
    # expert and router weight gradients against the oracle, summed over the ranks' batches
    f64 = lambda a: to_f64(a, shape.dtype)
    x64 = [f64(b["x"]) for b in batches]
    for q in range(world):
        f = mo.layer_forward(x64[q], f64(base["Wg"]), base["bias"], f64(base["W1"]),
                             f64(base["W3"]), f64(base["W2"]), k=shape.k, act=shape.act,
                             gate_norm=shape.gate_norm, capacity_factor=shape.capacity_factor,
                             idx_override=ranks[q].tok.view("topk_idx").cpu().numpy())
        g = mo.layer_backward(f, x64[q], f64(base["Wg"]), f64(base["W1"]), f64(base["W3"]),
                              f64(base["W2"]), f64(batches[q]["dy"]))
        for n in dW_sum:
            if g[n] is not None:
                dW_sum[n] = dW_sum[n] + g[n]
        dWg_ref = dWg_ref + g["dWg"]
    rel = parity.tol_for(shape)
    for n, i in (("dW1", 0), ("dW3", 1), ("dW2", 2)):
        if grads[0][i] is None:
            continue
        got = torch.cat([grads[q][i] for q in range(world)]).cpu().numpy()
        parity.assert_close(n, got, dW_sum[n], rel)
    parity.assert_close("dWg", dWg.cpu().numpy(), dWg_ref, rel)
