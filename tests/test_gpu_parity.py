"""CUDA path vs the CPU oracle, through the C ABI, on a B200.

Routing ids, per-expert counts, kept counts, the slot map / drop mask and the dispatched rows
must match bit-exactly; every float output and gradient must sit within max-abs error
<= 1e-4 * max|ref| (fp32 layers) or 2e-2 * max|ref| (bf16 layers), per tensor.
"""
import numpy as np
import pytest

from mixture_experts_layer_23_b200.configs import (BF16, DROPLESS, FP32, GELU, LAYERS,
                                                   PARITY_FP32, PARITY_SMALL, SWIGLU, LayerShape)
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


def _parity():
    import parity
    return parity


@pytest.mark.parametrize("shape", PARITY_SMALL + PARITY_FP32, ids=lambda s: s.name)
def test_small_layers_match_oracle(shape):
    _parity().full_compare(shape, seed=0)


@pytest.mark.parametrize("shape", [s for s in LAYERS if s.name in
                                   ("switch_tiny", "gpt2_gshard", "bert_large_skew")],
                         ids=lambda s: s.name)
def test_full_size_layers_match_oracle(shape):
    """The three smaller named layers at full size, every element compared."""
    _assert_engine(shape)
    _parity().full_compare(shape, seed=0)


def _assert_engine(shape):
    """bf16 layers with d, F multiples of 64 must run on the tcgen05 engine, fp32 on CUDA cores."""
    from mixture_experts_layer_23_b200 import moe
    want = 1 if (shape.dtype == BF16 and shape.d % 64 == 0 and shape.d_ff % 64 == 0) else 0
    assert moe.gemm_engine(moe.make_config(shape)) == want


@pytest.mark.parametrize("shape", [s for s in LAYERS if s.name in
                                   ("mixtral_dropless", "deepseek_v2")], ids=lambda s: s.name)
def test_full_size_large_layers(shape):
    """The two large named layers at full size: routing and dispatch in full; y, dg and dWg in
    full; dx in full on the DeepSeek-style layer (its oracle runs in well under a minute) and on
    sampled tokens on the Mixtral-style one (whose full input gradient would double the oracle's
    ~11.5 TFLOP of float64 forward work); expert weight gradients on sampled rows."""
    _assert_engine(shape)
    _, cpu_s = _parity().large_compare(shape, seed=0, full_dx=shape.name == "deepseek_v2")
    print(f"{shape.name}: float64 oracle {cpu_s:.1f} s")


EDGE = [
    LayerShape("one_token", T=1, d=64, E=4, k=2, d_ff=64, dtype=BF16),
    LayerShape("single_expert_dense", T=130, d=64, E=1, k=1, d_ff=128, capacity_factor=1.0,
               dtype=BF16),
    LayerShape("k_equals_E", T=200, d=32, E=4, k=4, d_ff=48, gate_norm=1, capacity_factor=None,
               act=SWIGLU, dtype=BF16),
    LayerShape("ragged_bf16", T=333, d=40, E=5, k=2, d_ff=24, capacity_factor=0.9, dtype=BF16,
               bias="zipf"),
    LayerShape("ragged_fp32", T=129, d=12, E=3, k=2, d_ff=20, capacity_factor=1.1, dtype=FP32),
    LayerShape("max_k_many_experts", T=300, d=32, E=256, k=8, d_ff=32, capacity_factor=2.0,
               dtype=BF16, n_shared=1, act=SWIGLU, bias="normal"),
    LayerShape("fp32_shared_only_top1", T=77, d=16, E=2, k=1, d_ff=8, n_shared=2,
               capacity_factor=0.5, dtype=FP32),
    # tensor-core router at its widest (E = 256 experts, N = 256 accumulator columns), k = 8
    LayerShape("wide_router_tc", T=300, d=64, E=256, k=8, d_ff=64, capacity_factor=2.0,
               dtype=BF16, bias="normal"),
    # tensor-core router (more than 32 experts) with E not a multiple of 16 and a ragged last
    # token tile
    LayerShape("odd_experts_tc", T=517, d=128, E=45, k=3, d_ff=128, capacity_factor=1.1,
               dtype=BF16, bias="zipf"),
    # warp-per-token router and un-dispatch at their widest (32 experts, every lane holds a
    # logit), d not a multiple of 64 (so not the tensor-core router) nor of the warp's 256-column
    # stride, k = 8
    LayerShape("warp_router_e32", T=333, d=136, E=32, k=8, d_ff=64, capacity_factor=1.5,
               dtype=BF16, bias="normal"),
    LayerShape("warp_router_fp32", T=301, d=100, E=24, k=3, d_ff=36, n_shared=1,
               capacity_factor=1.2, dtype=FP32, bias="zipf"),
    # router backward on the tensor cores: E = 72 is not a multiple of the
    # 64-wide K block, T not a multiple of the token chunk, with shared experts and SwiGLU
    LayerShape("router_bwd_tc_shared", T=700, d=192, E=72, k=6, d_ff=128, n_shared=2,
               capacity_factor=1.5, act=SWIGLU, dtype=BF16, bias="normal"),
]


@pytest.mark.parametrize("shape", EDGE, ids=lambda s: s.name)
def test_edge_shapes(shape):
    _parity().full_compare(shape, seed=3)


EDGE_ROUTER = [
    # router token tiles of 16 rows (44 CTAs), ragged last tile
    LayerShape("router_ragged_tiles", T=700, d=1024, E=8, k=2, d_ff=64, capacity_factor=1.0,
               dtype=BF16, bias="normal"),
    # fewer tokens than a 128-row tile: 16-row router tiles, the last one ragged
    LayerShape("router_fewer_tokens_than_a_tile", T=100, d=2048, E=16, k=2, d_ff=64,
               capacity_factor=2.0, dtype=BF16),
    # two waves of router tiles (72 rows each, 264 CTAs), ragged last tile
    LayerShape("router_two_waves", T=18945, d=64, E=8, k=2, d_ff=32, capacity_factor=1.25,
               dtype=BF16, bias="normal"),
    # 64 experts (the widest row staged in shared memory), 6 routed + 2 shared rows gathered per
    # token by the un-dispatch epilogue, router weight gradient with N = 64
    LayerShape("router_e64_shared_gathers", T=1111, d=512, E=64, k=6, d_ff=64, n_shared=2,
               act=SWIGLU, capacity_factor=1.25, dtype=BF16, bias="normal"),
    # 200 experts (whole-d router), k = 8 with 8 shared experts: 16 gathered rows per token;
    # router weight gradient with N = 256 and d = 192 (its second 128-column tile half outside d)
    LayerShape("wide_e_max_gathers", T=600, d=192, E=200, k=8, d_ff=128, n_shared=8,
               capacity_factor=2.0, dtype=BF16, bias="normal"),
]


# rows too long for the dispatch's shared-memory row buffers (8 warps x 2 rows of 13 KB), which
# take the 16-byte register copies instead of bulk copies
EDGE_LONG_ROWS = [
    LayerShape("dispatch_long_rows_bf16", T=300, d=6656, E=4, k=2, d_ff=64, capacity_factor=1.25,
               dtype=BF16, bias="normal"),
    LayerShape("dispatch_long_rows_fp32", T=200, d=3328, E=4, k=2, d_ff=32, capacity_factor=1.0,
               dtype=FP32),
]


@pytest.mark.parametrize("shape", EDGE_LONG_ROWS, ids=lambda s: s.name)
def test_dispatch_long_rows(shape):
    _parity().full_compare(shape, seed=6)


# layers with at least 2048 routed rows per expert on average, whose weight gradients read Xd^T and
# dO^T (and x^T, dy^T for shared experts) K-major from transposed copies: a shared expert with a
# ragged token count (T_pad columns, zeros past T), and a GELU top-1 layer
EDGE_WGRAD = [
    LayerShape("kmajor_wgrad_shared_ragged", T=2500, d=128, E=2, k=2, d_ff=192, n_shared=1,
               act=SWIGLU, capacity_factor=1.25, dtype=BF16, bias="normal"),
    LayerShape("kmajor_wgrad_gelu_top1", T=4200, d=192, E=2, k=1, d_ff=128, act=GELU,
               capacity_factor=None, dtype=BF16),
    # F ending in a partial tile of at most 128 columns with d a multiple of 256: dW1 and dW3 are
    # computed transposed (stored through the transposing epilogue) with N = 128 edge tiles; with
    # the K-major operand and a shared expert, and without
    LayerShape("transposed_dw1_kmajor_shared", T=2100, d=256, E=2, k=2, d_ff=320, n_shared=1,
               act=SWIGLU, capacity_factor=1.25, dtype=BF16, bias="normal"),
    LayerShape("transposed_dw1_gelu", T=300, d=512, E=4, k=2, d_ff=64, act=GELU,
               capacity_factor=1.0, dtype=BF16),
]


@pytest.mark.parametrize("shape", EDGE_WGRAD, ids=lambda s: s.name)
def test_kmajor_weight_gradient_shapes(shape):
    _parity().full_compare(shape, seed=5)


@pytest.mark.parametrize("shape", EDGE_ROUTER, ids=lambda s: s.name)
def test_router_tiles_and_fused_backward_shapes(shape):
    _parity().full_compare(shape, seed=4)


AUX = [
    # load-balancing loss on: its value, and its gradient through dlogits into dx and dWg
    LayerShape("aux_gelu_drops", T=700, d=64, E=8, k=2, d_ff=96, capacity_factor=0.9,
               dtype=BF16, bias="zipf", aux_loss_coef=0.05),
    LayerShape("aux_swiglu_renorm_shared", T=333, d=128, E=12, k=3, d_ff=64, n_shared=1,
               gate_norm=1, act=SWIGLU, capacity_factor=None, dtype=BF16, aux_loss_coef=0.5),
    LayerShape("aux_many_experts_tc", T=520, d=192, E=72, k=6, d_ff=128, capacity_factor=1.25,
               act=SWIGLU, dtype=BF16, bias="normal", aux_loss_coef=0.01),
    LayerShape("aux_fp32", T=150, d=48, E=5, k=2, d_ff=40, capacity_factor=1.0, dtype=FP32,
               aux_loss_coef=1.0),
]


@pytest.mark.parametrize("shape", AUX, ids=lambda s: s.name)
def test_aux_loss_layers_match_oracle(shape):
    _parity().full_compare(shape, seed=5)


def test_aux_loss_entry_point_matches_the_layer():
    """moe_aux_loss on the layer's own logits and counts reproduces the forward's value bitwise."""
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import MoELayer, to_device
    shape = AUX[0]
    inp = make_inputs(shape, 7)
    dev = {k: to_device(v, shape) for k, v in inp.items() if k != "bias"}
    bias = torch.from_numpy(inp["bias"]).cuda()
    layer = MoELayer(shape)
    layer.forward(dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"])
    loss = torch.zeros(4, dtype=torch.float32, device="cuda")
    scratch = torch.zeros(layer.L.scratch_bytes, dtype=torch.uint8, device="cuda")
    moe.aux_loss(layer.cfg, layer.view("logits"), layer.view("counts"), loss, scratch)
    torch.cuda.synchronize()
    assert loss[0].item() == layer.view("aux_loss")[0].item()
    assert layer.status() == moe.MOE_OK


CHOICE_MAJOR = [
    # choice-major drop priority (all first choices before any second choice) with drops: the
    # slot map must match the oracle's bit for bit
    LayerShape("cm_gelu_tc", T=1500, d=128, E=8, k=2, d_ff=128, capacity_factor=0.6,
               dtype=BF16, bias="zipf", choice_major=True),
    LayerShape("cm_swiglu_shared_k6", T=900, d=64, E=24, k=6, d_ff=64, n_shared=1,
               act=SWIGLU, capacity_factor=0.8, dtype=BF16, bias="normal", choice_major=True),
    LayerShape("cm_fp32_k3", T=301, d=36, E=5, k=3, d_ff=20, capacity_factor=0.7, dtype=FP32,
               choice_major=True, aux_loss_coef=0.2),
]


@pytest.mark.parametrize("shape", CHOICE_MAJOR, ids=lambda s: s.name)
def test_choice_major_layers_match_oracle(shape):
    gpu, _ = _parity().full_compare(shape, seed=6)
    assert np.any(gpu["slot"] < 0), "the case must drop assignments"


def test_choice_major_full_size():
    from dataclasses import replace
    from mixture_experts_layer_23_b200.configs import BY_NAME
    _parity().large_compare(replace(BY_NAME["bert_large_skew"], choice_major=True), seed=0)


FUSED = [
    # the one-launch forward: the tiny Switch layer at full size, and bf16 shapes with shared
    # experts, drops, renormalised gates and choice-major priority
    [l for l in LAYERS if l.name == "switch_tiny"][0],
    LayerShape("fused_bf16_swiglu_shared", T=300, d=64, E=8, k=2, d_ff=96, n_shared=1,
               act=SWIGLU, capacity_factor=0.8, dtype=BF16, bias="normal"),
    LayerShape("fused_choice_major_renorm", T=500, d=32, E=6, k=3, d_ff=48, gate_norm=1,
               capacity_factor=0.7, dtype=BF16, choice_major=True),
]


@pytest.mark.parametrize("shape", FUSED, ids=lambda s: s.name)
def test_fused_small_forward_matches_oracle(shape):
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import act_dtype, to_device
    from mixture_experts_layer_23_b200.synth import to_f64
    from oracle import moe_oracle as mo
    P = _parity()
    inp = make_inputs(shape, 9)
    dev = {k: to_device(v, shape) for k, v in inp.items() if k != "bias"}
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
    cfg = moe.make_config(shape)
    y = torch.empty(shape.T, shape.d, dtype=act_dtype(shape), device="cuda")
    idx = torch.empty(shape.T, shape.k, dtype=torch.int32, device="cuda")
    w = torch.empty(shape.T, shape.k, dtype=torch.float32, device="cuda")
    counts = torch.empty(shape.E, dtype=torch.int32, device="cuda")
    moe.layer_fwd_fused(cfg, dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"], y,
                        idx, w, counts)
    torch.cuda.synchronize()
    dt = shape.dtype
    x, Wg = to_f64(inp["x"], dt), to_f64(inp["Wg"], dt)
    W1, W3, W2 = to_f64(inp["W1"], dt), to_f64(inp["W3"], dt), to_f64(inp["W2"], dt)
    ol = mo.gate_logits(x, Wg, inp["bias"])
    gidx = idx.cpu().numpy().astype(np.int64)
    oidx = mo.select_topk(ol, shape.k)
    for t in np.nonzero(np.any(oidx != gidx, axis=1))[0]:   # only near-ties may differ
        assert np.max(np.abs(ol[t, oidx[t]] - ol[t, gidx[t]])) <= 1e-5, t
    C = P.oracle_capacity(shape)
    f = mo.layer_forward(x, Wg, inp["bias"], W1, W3, W2, k=shape.k, act=shape.act,
                         gate_norm=shape.gate_norm, capacity_factor=shape.capacity_factor,
                         n_shared=shape.n_shared, idx_override=gidx, capacity_override=C,
                         choice_major=shape.choice_major)
    assert np.array_equal(counts.cpu().numpy(), f["counts"])
    rel = P.tol_for(shape)
    P.assert_close("topk_w", w.cpu().numpy(), f["g"], rel)
    P.assert_close("y", P.act_to_np(y), f["y"], rel)
    if shape.capacity_factor is not None and shape.name != "switch_tiny":
        assert np.any(f["pos"] < 0), "the case must drop assignments"


def test_autograd_function_matches_the_c_abi():
    """MoEFunction gives the same y and gradients as calling moe_layer_fwd / moe_layer_bwd."""
    import torch
    from mixture_experts_layer_23_b200.layer import MoEFunction, MoELayer, to_device
    shape = LayerShape("autograd", T=300, d=64, E=6, k=2, d_ff=128, n_shared=1, act=SWIGLU,
                       capacity_factor=1.0, dtype=BF16, bias="normal")
    inp = make_inputs(shape, 8)
    dev = {k: to_device(v, shape) for k, v in inp.items() if k != "bias"}
    bias = torch.from_numpy(inp["bias"]).cuda()
    ref = MoELayer(shape)
    y_ref = ref.forward(dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"]).clone()
    ref.backward(dev["dy"], dev["x"], dev["Wg"], dev["W1"], dev["W3"], dev["W2"])
    leaves = {n: dev[n].clone().requires_grad_(True) for n in ("x", "Wg", "W1", "W3", "W2")}
    y = MoEFunction.apply(leaves["x"], leaves["Wg"], leaves["W1"], leaves["W3"], leaves["W2"],
                          MoELayer(shape), bias)
    y.backward(dev["dy"])
    assert torch.equal(y, y_ref)
    assert torch.equal(leaves["x"].grad, ref.dx)
    for n, g in (("Wg", ref.dWg), ("W1", ref.dW1), ("W3", ref.dW3), ("W2", ref.dW2)):
        assert torch.equal(leaves[n].grad, g.to(leaves[n].dtype)), n


def test_step_graph_replays_the_layer_bitwise():
    """A CUDA graph of one forward + backward gives the eager results bit for bit, and a new
    batch copied into the captured input buffers is picked up by the next replay."""
    import torch
    from mixture_experts_layer_23_b200.layer import MoELayer, MoEStepGraph, to_device
    shape = LayerShape("graph", T=700, d=128, E=8, k=2, d_ff=192, capacity_factor=1.0, dtype=BF16,
                       bias="zipf")
    inp, inp2 = make_inputs(shape, 10), make_inputs(shape, 11)
    dev = {k: to_device(v, shape) for k, v in inp.items() if k != "bias"}
    bias = torch.from_numpy(inp["bias"]).cuda()
    eager = MoELayer(shape)

    def run_eager(x, dy):
        eager.forward(x, dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"])
        eager.backward(dy, x, dev["Wg"], dev["W1"], dev["W3"], dev["W2"])
        return eager.y.clone(), eager.dx.clone(), eager.dWg.clone(), eager.dW1.clone()

    layer = MoELayer(shape)
    x, dy = dev["x"].clone(), dev["dy"].clone()
    g = MoEStepGraph(layer, x, dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"], dy)
    for src in (inp, inp2):
        x.copy_(to_device(src["x"], shape))
        dy.copy_(to_device(src["dy"], shape))
        g.replay()
        want = run_eager(x, dy)
        got = (layer.y, layer.dx, layer.dWg, layer.dW1)
        for a, b in zip(got, want):
            assert torch.equal(a, b)


def test_zero_capacity_drops_everything():
    s = LayerShape("cap0", T=100, d=32, E=4, k=2, d_ff=32, n_shared=1, dtype=FP32)
    gpu, _ = _parity().full_compare(s, seed=1, capacity=0)
    assert np.all(gpu["slot"] == -1)
    assert np.all(gpu["dW1"][:4] == 0) and np.all(gpu["dW2"][:4] == 0)


def test_explicit_dropless_capacity():
    s = LayerShape("dropless_explicit", T=150, d=32, E=4, k=2, d_ff=32, dtype=BF16)
    gpu, _ = _parity().full_compare(s, seed=2, capacity=DROPLESS)
    assert np.all(gpu["slot"] >= 0)


def test_one_expert_takes_every_token():
    s = LayerShape("hot_expert", T=400, d=64, E=8, k=2, d_ff=64, capacity_factor=1.0, dtype=BF16,
                   bias="normal")
    inp = make_inputs(s, 0)
    inp["bias"] = np.zeros(8, np.float32)
    inp["bias"][5] = 1000.0           # expert 5 is every token's first choice
    gpu, _ = _parity().full_compare(s, inp=inp)
    assert gpu["counts"][5] == 400 and gpu["kept"][5] == 100


def test_exact_logit_ties_go_to_lower_index():
    """Identical gate rows make exact logit ties: the lower expert index must win."""
    s = LayerShape("ties", T=256, d=32, E=6, k=2, d_ff=32, capacity_factor=2.0, dtype=BF16)
    inp = make_inputs(s, 4)
    inp["Wg"][3] = inp["Wg"][1]
    inp["Wg"][4] = inp["Wg"][1]
    gpu, _ = _parity().full_compare(s, inp=inp)
    idx = gpu["topk_idx"]
    assert np.array_equal(gpu["logits"][:, 1], gpu["logits"][:, 3])
    assert not np.any(idx == 4)                              # a tied higher index never wins
    has3 = np.any(idx == 3, axis=1)
    assert np.all(np.any(idx == 1, axis=1)[has3])            # 3 only ever beside its tie 1


@pytest.mark.parametrize("shape", [PARITY_SMALL[1], PARITY_SMALL[4], PARITY_FP32[1]],
                         ids=lambda s: s.name)
def test_bitwise_deterministic(shape):
    p = _parity()
    inp = make_inputs(shape, 5)
    a = p.run_gpu(shape, inp)
    b = p.run_gpu(shape, inp)
    for k in ("logits", "topk_idx", "topk_w", "slot", "y", "dx", "dWg", "dW1", "dW2", "dg"):
        assert np.array_equal(a[k], b[k]), k
    # the row space is sized for the worst routing: rows past the last routed segment are never
    # written (their contents are whatever the workspace held), so compare the written rows only
    end = int(a["offsets"][-1])
    assert end == int(b["offsets"][-1])
    assert np.array_equal(a["Xd_bits"][:end], b["Xd_bits"][:end]), "Xd"


def test_route_and_route_from_logits_agree():
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import to_device
    s = PARITY_SMALL[2]
    inp = make_inputs(s, 0)
    cfg = moe.make_config(s)
    x, Wg = to_device(inp["x"], s), to_device(inp["Wg"], s)
    bias = torch.from_numpy(inp["bias"]).cuda()
    logits = torch.empty(s.T, s.E, device="cuda")
    i1 = torch.empty(s.T, s.k, dtype=torch.int32, device="cuda")
    w1 = torch.empty(s.T, s.k, device="cuda")
    i2, w2 = torch.empty_like(i1), torch.empty_like(w1)
    moe.route(cfg, x, Wg, bias, logits, i1, w1)
    moe.route_from_logits(cfg, logits, i2, w2)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(w1, w2)


def test_step_entry_points_compose_to_the_layer():
    """route -> dispatch -> expert_ffn -> combine equals moe_layer_fwd bit for bit."""
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import MoELayer, to_device
    s = PARITY_SMALL[4]
    inp = make_inputs(s, 0)
    dev = {k: to_device(v, s) for k, v in inp.items() if k != "bias"}
    bias = torch.from_numpy(inp["bias"]).cuda()
    layer = MoELayer(s)
    y_ref = layer.forward(dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"]).clone()
    cfg, L = layer.cfg, layer.L
    R = L.rows
    dt = layer.dt
    T, E, k, d, F = s.T, s.E, s.k, s.d, s.d_ff
    logits = torch.empty(T, E, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    kept, offsets = torch.empty_like(counts), torch.empty(E + 1, dtype=torch.int32, device="cuda")
    slot = torch.empty(T, k, dtype=torch.int32, device="cuda")
    row_token = torch.empty(R, dtype=torch.int32, device="cuda")
    Xd = torch.empty(R, d, dtype=dt, device="cuda")
    U, V, H = (torch.empty(R, F, dtype=dt, device="cuda") for _ in range(3))
    O = torch.empty(R, d, dtype=dt, device="cuda")
    y = torch.empty(T, d, dtype=dt, device="cuda")
    scratch = torch.zeros(L.scratch_bytes, dtype=torch.uint8, device="cuda")
    moe.route(cfg, dev["x"], dev["Wg"], bias, logits, idx, w)
    moe.dispatch(cfg, dev["x"], idx, counts, kept, offsets, slot, row_token, Xd, scratch)
    moe.expert_ffn(cfg, Xd, dev["x"], offsets, dev["W1"], dev["W3"], dev["W2"], U, V, H, O, scratch)
    moe.combine(cfg, O, slot, w, y)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert torch.equal(slot, layer.view("slot"))


@pytest.mark.parametrize("shape", [PARITY_SMALL[4], PARITY_SMALL[1], PARITY_FP32[1]],
                         ids=lambda s: s.name)
def test_backward_steps_compose_to_the_layer(shape):
    """combine_bwd -> expert_ffn_bwd -> router_bwd on the forward's ctx equals moe_layer_bwd bit
    for bit (tensor-core and CUDA-core paths, with and without shared experts)."""
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import MoELayer, to_device
    inp = make_inputs(shape, 2)
    dev = {k: to_device(v, shape) for k, v in inp.items() if k != "bias"}
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
    layer = MoELayer(shape)
    layer.forward(dev["x"], dev["Wg"], bias, dev["W1"], dev["W3"], dev["W2"])
    layer.backward(dev["dy"], dev["x"], dev["Wg"], dev["W1"], dev["W3"], dev["W2"])
    assert layer.status() == moe.MOE_OK
    cfg, L, dt = layer.cfg, layer.L, layer.dt
    R, T, d, E, F, Et = L.rows, shape.T, shape.d, shape.E, shape.d_ff, shape.E_tot
    dO = torch.zeros(R, d, dtype=dt, device="cuda")
    dXd = torch.zeros(R, d, dtype=dt, device="cuda")
    dx = torch.empty(T, d, dtype=dt, device="cuda")
    dWg = torch.empty(E, d, device="cuda")
    dW1, dW2 = torch.empty(Et, F, d, device="cuda"), torch.empty(Et, d, F, device="cuda")
    dW3 = torch.empty(Et, F, d, device="cuda") if shape.act == SWIGLU else None
    scratch = torch.zeros(L.scratch_bytes, dtype=torch.uint8, device="cuda")
    gv = layer.view("Gv") if shape.act == SWIGLU else None
    moe.combine_bwd(cfg, layer.ctx, dev["dy"], dO, scratch)
    moe.expert_ffn_bwd(cfg, dO, dev["dy"], layer.view("Xd"), dev["x"], layer.view("offsets"),
                       dev["W1"], dev["W3"], dev["W2"], layer.view("Gu"), gv, layer.view("H"), dXd,
                       dW1, dW3, dW2, scratch)
    moe.router_bwd(cfg, layer.ctx, dev["x"], dev["Wg"], dXd, dx, dWg, scratch)
    assert moe.read_status(scratch) == moe.MOE_OK
    assert torch.equal(dx, layer.dx)
    assert torch.equal(dWg, layer.dWg)
    assert torch.equal(dW1, layer.dW1) and torch.equal(dW2, layer.dW2)
    if dW3 is not None:
        assert torch.equal(dW3, layer.dW3)


def test_step_from_host_buffers_matches_the_layer():
    """moe_layer_step_host (host x, dy in; host y, dx out) gives moe_layer_fwd + moe_layer_bwd's
    results bit for bit, on two calls in a row on one stream."""
    import torch
    from mixture_experts_layer_23_b200 import moe
    from mixture_experts_layer_23_b200.layer import MoELayer, to_device
    s = PARITY_SMALL[3]
    ref = MoELayer(s)
    got = MoELayer(s)
    for seed in (4, 5):
        inp = make_inputs(s, seed)
        dev = {k: to_device(v, s) for k, v in inp.items() if k != "bias"}
        ref.forward(dev["x"], dev["Wg"], None, dev["W1"], dev["W3"], dev["W2"])
        ref.backward(dev["dy"], dev["x"], dev["Wg"], dev["W1"], dev["W3"], dev["W2"])
        x_h = dev["x"].cpu().pin_memory()
        dy_h = dev["dy"].cpu().pin_memory()
        y_h = torch.empty_like(x_h).pin_memory()
        dx_h = torch.empty_like(x_h).pin_memory()
        x_d, dy_d = torch.empty_like(dev["x"]), torch.empty_like(dev["dy"])
        moe.layer_step_host(got.cfg, x_h, dy_h, y_h, dx_h, x_d, dy_d, dev["Wg"], None, dev["W1"],
                            dev["W3"], dev["W2"], got.y, got.dx, got.dWg, got.dW1, got.dW3,
                            got.dW2, got.ctx, got.scratch)
        torch.cuda.synchronize()
        assert got.status() == moe.MOE_OK and ref.status() == moe.MOE_OK
        assert torch.equal(y_h, ref.y.cpu()) and torch.equal(dx_h, ref.dx.cpu())
        assert torch.equal(got.dWg, ref.dWg) and torch.equal(got.dW1, ref.dW1)
        assert torch.equal(got.dW2, ref.dW2) and torch.equal(got.dW3, ref.dW3)
