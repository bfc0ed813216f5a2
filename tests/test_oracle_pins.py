"""Pins of the CPU oracle against things other than itself.

Brute force on tiny inputs, hand-worked fixtures, closed forms, library special cases,
invariants and float64 central finite differences.  The planted-mistake tests at the end
swap a plausible error into the oracle (on the CPU) and check that some pin here fails.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import expit
from scipy.stats import norm

from oracle import brute
from oracle import moe_oracle as mo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- pin helpers
# Each returns True when the oracle passes; the planted-mistake tests expect False.

def pin_topk_brute(seed=0):
    rng = np.random.default_rng(seed)
    for E, k in [(4, 1), (5, 2), (8, 3), (16, 6), (6, 6)]:
        # few distinct values so exact ties are frequent
        L = rng.integers(-3, 4, size=(60, E)).astype(np.float64) * 0.25
        idx = mo.select_topk(L, k)
        for t in range(L.shape[0]):
            if list(idx[t]) != brute.topk_brute(list(L[t]), k):
                return False
    return True


def pin_ties_golden():
    for c in _golden("ties.json")["cases"]:
        got = mo.select_topk(np.array([c["logits"]]), c["k"])[0]
        if list(got) != c["idx"]:
            return False
    return True


def pin_dispatch_brute(seed=0):
    rng = np.random.default_rng(seed)
    for T, E, k, cf in [(40, 4, 1, 1.0), (64, 5, 2, 0.8), (50, 8, 3, 1.25), (30, 3, 2, None)]:
        L = rng.standard_normal((T, E)) + np.linspace(0, 1.5, E)[None, :]
        idx = mo.select_topk(L, k)
        C = mo.capacity(cf, k, T, E)
        for cm in (False, True):
            counts, kept, pos = mo.dispatch(idx, E, C, choice_major=cm)
            bc, bk, bp = brute.dispatch_brute(idx.tolist(), E, C, choice_major=cm)
            if list(counts) != bc or list(kept) != bk or pos.tolist() != bp:
                return False
    return True


def pin_hand_dispatch(name="hand_dispatch.json"):
    g = _golden(name)
    L = np.array(g["logits"])
    idx = mo.select_topk(L, g["k"])
    C = mo.capacity(g["capacity_factor"], g["k"], g["T"], g["E"])
    counts, kept, pos = mo.dispatch(idx, g["E"], C, choice_major=g.get("choice_major", False))
    ex = g["expect"]
    return (C == ex["C"] and idx.tolist() == ex["idx"] and counts.tolist() == ex["counts"]
            and kept.tolist() == ex["kept"] and pos.tolist() == ex["pos"])


def pin_gate_bias_golden():
    """The hand-worked gate with a per-expert logit bias: the bias flips every token's top-1 and
    sets the softmax weights (exact fractions), for the full and the top-k softmax."""
    g = _golden("hand_gate_bias.json")
    x, Wg, b = np.array(g["x"]), np.array(g["Wg"]), np.array(g["bias"])
    logits = mo.gate_logits(x, Wg, b)
    if mo.select_topk(mo.gate_logits(x, Wg, None), 1).tolist() != g["without_bias_top1"]:
        return False
    for c in g["cases"]:
        idx = mo.select_topk(logits, c["k"])
        want = np.array([[n / m for n, m in row] for row in c["w_frac"]])
        if idx.tolist() != c["idx"]:
            return False
        if not np.allclose(mo.gate_weights(logits, idx, c["gate_norm"]), want, rtol=0,
                           atol=1e-12):
            return False
        # the same through the layer: identity experts, nothing dropped -> y_t = sum_j w_tj x_t
        f = mo.layer_forward(x, Wg, b, None, None, None, k=c["k"], act=mo.GELU,
                             gate_norm=c["gate_norm"], capacity_factor=None,
                             identity_experts=True)
        if f["idx"].tolist() != c["idx"]:
            return False
        if not np.allclose(f["y"], want.sum(axis=1, keepdims=True) * x, rtol=0, atol=1e-12):
            return False
    return True


def pin_choice_major_priority(seed=3):
    """Choice-major invariant: at every expert, once a choice index j has a dropped assignment,
    no assignment with a later choice index is kept; and the kept counts equal token order's."""
    rng = np.random.default_rng(seed)
    for T, E, k, cf in [(60, 4, 2, 0.7), (45, 6, 3, 0.5), (33, 3, 3, 1.0)]:
        idx = mo.select_topk(rng.standard_normal((T, E)), k)
        C = mo.capacity(cf, k, T, E)
        counts, kept, pos = mo.dispatch(idx, E, C, choice_major=True)
        c0, k0, _ = mo.dispatch(idx, E, C)
        if not (np.array_equal(counts, c0) and np.array_equal(kept, k0)):
            return False
        for e in range(E):
            worst_kept = -1
            best_dropped = k
            for t in range(T):
                for j in range(k):
                    if idx[t, j] != e:
                        continue
                    if pos[t, j] >= 0:
                        worst_kept = max(worst_kept, j)
                    else:
                        best_dropped = min(best_dropped, j)
            if worst_kept > best_dropped:
                return False
    return True


def pin_gelu_values():
    phi = _golden("normal_cdf.json")["Phi"]
    u = np.array([float(s) for s in phi])
    want = np.array([float(s) * v for s, v in phi.items()])
    ok = np.allclose(mo.gelu(u), want, rtol=0, atol=1e-15)
    z = np.linspace(-6, 6, 101)
    ok &= np.allclose(mo.gelu(z), z * norm.cdf(z), rtol=1e-13, atol=1e-15)
    ok &= np.allclose(mo.silu(z), z * expit(z), rtol=1e-13, atol=1e-15)
    return bool(ok)


def pin_activation_derivatives():
    z = np.linspace(-5, 5, 41)
    h = 1e-6
    fd_g = (mo.gelu(z + h) - mo.gelu(z - h)) / (2 * h)
    fd_s = (mo.silu(z + h) - mo.silu(z - h)) / (2 * h)
    return (np.allclose(mo.gelu_grad(z), fd_g, rtol=0, atol=1e-8)
            and np.allclose(mo.silu_grad(z), fd_s, rtol=0, atol=1e-8))


def _tiny_layer(seed, *, T=8, d=4, E=3, k=2, F=5, act=mo.GELU, gate_norm=0, cf=0.75,
                n_shared=0, bias=True, min_gap=1e-3, aux=0.0):
    """Random float64 layer whose top-k sets sit at least min_gap from a logit tie."""
    rng = np.random.default_rng(seed)
    for _ in range(1000):
        x = rng.standard_normal((T, d))
        Wg = rng.standard_normal((E, d)) / math.sqrt(d)
        b = rng.standard_normal(E) * 0.3 if bias else None
        L = mo.gate_logits(x, Wg, b)
        s = np.sort(L, axis=1)[:, ::-1]
        if k < E and np.min(s[:, k - 1] - s[:, k]) < min_gap:
            continue
        Et = E + n_shared
        W1 = rng.standard_normal((Et, F, d)) / math.sqrt(d)
        W3 = rng.standard_normal((Et, F, d)) / math.sqrt(d) if act == mo.SWIGLU else None
        W2 = rng.standard_normal((Et, d, F)) / math.sqrt(F)
        dy = rng.standard_normal((T, d))
        return dict(x=x, Wg=Wg, bias=b, W1=W1, W3=W3, W2=W2, dy=dy,
                    kw=dict(k=k, act=act, gate_norm=gate_norm, capacity_factor=cf, n_shared=n_shared,
                            aux_loss_coef=aux))
    raise RuntimeError("no tie-free draw")


def _loss(p, **over):
    q = {**p, **over}
    f = mo.layer_forward(q["x"], q["Wg"], q["bias"], q["W1"], q["W3"], q["W2"], **p["kw"])
    return float(np.sum(f["y"] * p["dy"])) + f["aux_loss"]


def pin_backward_fd(p, h=1e-6, tol=1e-6):
    f = mo.layer_forward(p["x"], p["Wg"], p["bias"], p["W1"], p["W3"], p["W2"], **p["kw"])
    g = mo.layer_backward(f, p["x"], p["Wg"], p["W1"], p["W3"], p["W2"], p["dy"])
    pairs = [("x", "dx"), ("Wg", "dWg"), ("W1", "dW1"), ("W2", "dW2")]
    if p["W3"] is not None:
        pairs.append(("W3", "dW3"))
    for name, gname in pairs:
        base = p[name]
        fd = np.zeros_like(base)
        for i in np.ndindex(base.shape):
            a = base.copy(); a[i] += h
            b = base.copy(); b[i] -= h
            fd[i] = (_loss(p, **{name: a}) - _loss(p, **{name: b})) / (2 * h)
        err = np.max(np.abs(fd - g[gname]))
        if not err <= tol * max(1.0, np.max(np.abs(fd))):
            return False
    return True


FD_CASES = {
    "gelu_softmax_drops": dict(seed=1, act=mo.GELU, gate_norm=0, cf=0.75),
    "swiglu_shared": dict(seed=2, act=mo.SWIGLU, gate_norm=0, cf=1.0, n_shared=1),
    "swiglu_renorm_dropless": dict(seed=3, act=mo.SWIGLU, gate_norm=1, cf=None),
    "gelu_top1": dict(seed=4, act=mo.GELU, gate_norm=0, k=1, cf=1.0),
    # the load-balancing loss added to <y, dy>: its gradient reaches dx and dWg through dlogits
    "gelu_aux_drops": dict(seed=5, act=mo.GELU, gate_norm=0, cf=0.75, aux=0.3),
    "swiglu_renorm_aux": dict(seed=6, act=mo.SWIGLU, gate_norm=1, cf=None, n_shared=1, aux=0.3),
}


# ----------------------------------------------------------------------------- tests

def test_topk_matches_brute_force_with_ties():
    assert pin_topk_brute()


def test_topk_tie_fixtures():
    assert pin_ties_golden()


def test_dispatch_matches_brute_force():
    assert pin_dispatch_brute()


def test_hand_worked_dispatch():
    assert pin_hand_dispatch()


def test_hand_worked_gate_bias():
    assert pin_gate_bias_golden()


def test_hand_worked_choice_major_dispatch():
    assert pin_hand_dispatch("hand_dispatch_choice_major.json")


def test_choice_major_priority_invariant():
    assert pin_choice_major_priority()


def test_gelu_silu_values():
    assert pin_gelu_values()


def test_activation_derivatives_fd():
    assert pin_activation_derivatives()


def test_capacity_values():
    # cf*k*T/E is an integer at every capped workload: 80, 640, 512, 2304
    assert mo.capacity(1.25, 1, 256, 4) == 80
    assert mo.capacity(1.25, 2, 4096, 16) == 640
    assert mo.capacity(1.0, 2, 8192, 32) == 512
    assert mo.capacity(1.5, 6, 16384, 64) == 2304
    assert mo.capacity(None, 2, 16384, 8) is None
    assert mo.capacity(1.0, 1, 5, 2) == 3            # rounds up


def test_softmax_closed_forms():
    rng = np.random.default_rng(0)
    L = rng.standard_normal((50, 2)) * 3
    p = mo.softmax(L)
    assert np.allclose(p[:, 0], expit(L[:, 0] - L[:, 1]), rtol=0, atol=1e-15)
    L = rng.standard_normal((40, 5))
    assert np.allclose(mo.softmax(L).sum(1), 1.0, atol=1e-15)
    # softmax over the k chosen with k = E is the full softmax, reordered
    idx = mo.select_topk(L, 5)
    g1 = mo.gate_weights(L, idx, 1)
    g0 = mo.gate_weights(L, idx, 0)
    assert np.allclose(g1, g0, rtol=0, atol=1e-15)
    # invariance to a constant shift of the logits (large values do not overflow)
    assert np.allclose(mo.softmax(L + 700.0), mo.softmax(L), atol=1e-15)
    # for any k, the softmax over the k chosen logits is the full softmax at the chosen experts
    # renormalised over them (GShard-style renormalised top-k is gate_norm 1)
    for k in (1, 2, 3):
        idx = mo.select_topk(L, k)
        p = np.take_along_axis(mo.softmax(L), idx, axis=1)
        assert np.allclose(mo.gate_weights(L, idx, 1), p / p.sum(1, keepdims=True), rtol=0,
                           atol=1e-15)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_routing_invariants(seed):
    rng = np.random.default_rng(seed)
    T, E, k = 500, 8, 2
    L = rng.standard_normal((T, E)) + 2.0 * (np.arange(E) + 1.0) ** -1.2
    idx = mo.select_topk(L, k)
    assert all(len(set(r)) == k for r in idx.tolist())          # k distinct experts per token
    for cf in [0.5, 1.0, 1.25]:
        C = mo.capacity(cf, k, T, E)
        counts, kept, pos = mo.dispatch(idx, E, C)
        assert counts.sum() == T * k
        assert np.all(kept <= C) and np.all(kept == np.minimum(counts, C))
        assert kept.sum() + np.sum(pos < 0) == T * k
        for e in range(E):
            r = np.sort(pos[(idx == e) & (pos >= 0)])
            assert np.array_equal(r, np.arange(kept[e]))             # slots injective, dense
            # the kept ones are the earliest tokens of that expert
            toks = np.nonzero((idx == e).any(1))[0]
            kept_toks = np.nonzero(((idx == e) & (pos >= 0)).any(1))[0]
            assert np.array_equal(kept_toks, toks[:kept[e]])
    # capacity >= T: nothing drops
    C = mo.capacity(E / k, k, T, E)
    _, _, pos = mo.dispatch(idx, E, C)
    assert np.all(pos >= 0)


def test_identity_experts_give_weighted_sum_of_x():
    rng = np.random.default_rng(5)
    T, d, E, k = 64, 6, 5, 2
    x = rng.standard_normal((T, d))
    Wg = rng.standard_normal((E, d))
    f = mo.layer_forward(x, Wg, None, None, None, None, k=k, act=mo.GELU, gate_norm=0,
                         capacity_factor=0.8, identity_experts=True)
    wsum = np.where(f["pos"] >= 0, f["g"], 0.0).sum(1)
    assert np.allclose(f["y"], wsum[:, None] * x, rtol=0, atol=1e-14)
    assert np.any(f["pos"] < 0)
    # k = E, renormalised over the chosen, dropless: the layer is the identity
    f = mo.layer_forward(x, Wg, None, None, None, None, k=E, act=mo.GELU, gate_norm=1,
                         capacity_factor=None, identity_experts=True)
    assert np.allclose(f["y"], x, rtol=0, atol=1e-14)


@pytest.mark.parametrize("act", [mo.GELU, mo.SWIGLU])
def test_single_expert_is_a_dense_mlp(act):
    rng = np.random.default_rng(7)
    T, d, F = 9, 5, 7
    x = rng.standard_normal((T, d))
    Wg = rng.standard_normal((1, d))
    W1 = rng.standard_normal((1, F, d))
    W3 = rng.standard_normal((1, F, d)) if act == mo.SWIGLU else None
    W2 = rng.standard_normal((1, d, F))
    f = mo.layer_forward(x, Wg, None, W1, W3, W2, k=1, act=act, gate_norm=0, capacity_factor=1.0)
    for t in range(T):
        want = brute.dense_mlp_brute(list(x[t]), W1[0].tolist(),
                                     None if W3 is None else W3[0].tolist(), W2[0].tolist(), act)
        assert np.allclose(f["y"][t], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("case", list(FD_CASES))
def test_backward_matches_finite_differences(case):
    c = dict(FD_CASES[case])
    p = _tiny_layer(c.pop("seed"), **c)
    f = mo.layer_forward(p["x"], p["Wg"], p["bias"], p["W1"], p["W3"], p["W2"], **p["kw"])
    if case == "gelu_softmax_drops":
        assert np.any(f["pos"] < 0), "this case must exercise capacity drops"
    assert pin_backward_fd(p)


def pin_aux_loss_closed_forms():
    """Closed forms of the load-balancing loss: an even routing with uniform probabilities gives
    coef; every token sent to one expert with (numerically) certain probability gives coef * E;
    E = 2 reduces to coef * 2 * (f0 * mean sigmoid(l0 - l1) + f1 * mean sigmoid(l1 - l0))."""
    coef, T, E, k = 0.7, 12, 4, 2
    ok = math.isclose(mo.aux_loss(np.zeros((T, E)), np.full(E, T * k // E), k, coef), coef,
                      rel_tol=1e-15)
    L = np.zeros((T, E)); L[:, 0] = 200.0
    ok &= math.isclose(mo.aux_loss(L, np.array([T, 0, 0, 0]), 1, coef), coef * E, rel_tol=1e-12)
    rng = np.random.default_rng(11)
    L2 = rng.standard_normal((T, 2))
    cnt = np.array([7, 5])
    p0 = expit(L2[:, 0] - L2[:, 1])
    want = coef * 2 * (7 / T * p0.mean() + 5 / T * (1 - p0).mean())
    ok &= math.isclose(mo.aux_loss(L2, cnt, 1, coef), want, rel_tol=1e-12)
    return bool(ok)


def pin_aux_grad_fd(h=1e-6):
    """The gradient of the load-balancing loss against central differences of the loss itself
    (counts held fixed: they do not depend continuously on the logits)."""
    rng = np.random.default_rng(12)
    T, E, k, coef = 6, 5, 2, 0.4
    L = rng.standard_normal((T, E))
    cnt = rng.integers(0, 5, size=E)
    g = mo.aux_loss_grad(L, cnt, k, coef)
    fd = np.zeros_like(L)
    for i in np.ndindex(L.shape):
        a = L.copy(); a[i] += h
        b = L.copy(); b[i] -= h
        fd[i] = (mo.aux_loss(a, cnt, k, coef) - mo.aux_loss(b, cnt, k, coef)) / (2 * h)
    return bool(np.max(np.abs(fd - g)) <= 1e-8)


def test_aux_loss_closed_forms():
    assert pin_aux_loss_closed_forms()


def test_aux_loss_gradient_matches_finite_differences():
    assert pin_aux_grad_fd()


@pytest.mark.parametrize("case", [
    dict(act=1, gate_norm=0, cf=1.0, n_shared=1, bias="normal", choice_major=False, aux=0.0),
    dict(act=0, gate_norm=0, cf=0.7, n_shared=0, bias="zipf", choice_major=True, aux=0.3),
    dict(act=1, gate_norm=1, cf=None, n_shared=2, bias="none", choice_major=False, aux=0.0),
])
def test_by_expert_form_equals_full_layer(case):
    """layer_by_expert (one expert's intermediates at a time) gives layer_forward's y and
    layer_backward's dg, dlogits, dWg and dx; expert_input_grad gives expert_backward's dX."""
    from mixture_experts_layer_23_b200.configs import LayerShape
    from mixture_experts_layer_23_b200.synth import make_inputs, to_f64
    sh = LayerShape("s", T=150, d=16, E=7, k=3, d_ff=24, n_shared=case["n_shared"],
                    act=case["act"], gate_norm=case["gate_norm"], capacity_factor=case["cf"],
                    dtype=1, bias=case["bias"])
    inp = make_inputs(sh, 4)
    x, Wg, W1, W3, W2, dy = (to_f64(inp[n], 1) for n in ("x", "Wg", "W1", "W3", "W2", "dy"))
    kw = dict(k=sh.k, act=sh.act, gate_norm=sh.gate_norm, capacity_factor=sh.capacity_factor,
              n_shared=sh.n_shared, choice_major=case["choice_major"],
              aux_loss_coef=case["aux"])
    f = mo.layer_forward(x, Wg, inp["bias"], W1, W3, W2, **kw)
    g = mo.layer_backward(f, x, Wg, W1, W3, W2, dy)
    s = mo.layer_by_expert(x, Wg, inp["bias"], W1, W3, W2, dy, **kw)
    if case["cf"] is not None:
        assert np.any(s["pos"] < 0)
    for n in ("idx", "counts", "kept", "pos"):
        assert np.array_equal(s[n], f[n]), n
    assert np.allclose(s["y"], f["y"], rtol=0, atol=1e-12)
    for n in ("dg", "dlogits", "dWg", "dx"):
        assert np.allclose(s[n], g[n], rtol=0, atol=1e-12), n
    s2 = mo.layer_by_expert(x, Wg, inp["bias"], W1, W3, W2, dy, with_dx=False, **kw)
    assert s2["dx"] is None and np.array_equal(s2["dWg"], s["dWg"])
    for e, (tt, jj, X, U, V, H, O) in f["cache"].items():
        dO = dy[tt] if jj is None else f["g"][tt, jj][:, None] * dy[tt]
        w3 = None if W3 is None else W3[e]
        want = mo.expert_backward(X, U, V, H, dO, W1[e], w3, W2[e], sh.act)[0]
        got = mo.expert_input_grad(X, U, V, H, dO, W1[e], w3, W2[e], sh.act)
        assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_sampled_forms_equal_full_layer():
    from mixture_experts_layer_23_b200.configs import LayerShape, SWIGLU as SW
    from mixture_experts_layer_23_b200.synth import make_inputs, to_f64
    sh = LayerShape("s", T=120, d=16, E=6, k=3, d_ff=24, n_shared=1, act=SW, gate_norm=0,
                    capacity_factor=1.0, dtype=1, bias="normal")
    inp = make_inputs(sh, 3)
    x, Wg, W1, W3, W2, dy = (to_f64(inp[n], 1) for n in ("x", "Wg", "W1", "W3", "W2", "dy"))
    kw = dict(k=sh.k, act=sh.act, gate_norm=sh.gate_norm, capacity_factor=sh.capacity_factor,
              n_shared=sh.n_shared)
    f = mo.layer_forward(x, Wg, inp["bias"], W1, W3, W2, **kw)
    g = mo.layer_backward(f, x, Wg, W1, W3, W2, dy)
    r = mo.route(x, Wg, inp["bias"], k=sh.k, gate_norm=sh.gate_norm,
                 capacity_factor=sh.capacity_factor)
    toks = [0, 5, 77, 119]
    y, dx, dg = mo.token_forward_backward(toks, r, x, Wg, W1, W3, W2, dy, act=sh.act,
                                          gate_norm=sh.gate_norm, n_shared=sh.n_shared)
    assert np.allclose(y, f["y"][toks], atol=1e-12)
    assert np.allclose(dx, g["dx"][toks], atol=1e-12)
    assert np.allclose(dg, g["dg"][toks], atol=1e-12)
    for e in [0, 3, 6]:
        fs = [0, 7, 23]
        a, b, c = mo.expert_weight_grad_rows(e, fs, r, x, W1, W3, W2, dy, act=sh.act,
                                             n_shared=sh.n_shared)
        assert np.allclose(a, g["dW1"][e][fs], atol=1e-12)
        assert np.allclose(b, g["dW3"][e][fs], atol=1e-12)
        assert np.allclose(c, g["dW2"][e][:, fs], atol=1e-12)


# ----------------------------------------------------------------------------- planted mistakes

def _planted(monkeypatch, name, fn):
    monkeypatch.setattr(mo, name, fn)


def test_planted_gate_bias_dropped_is_caught(monkeypatch):
    _planted(monkeypatch, "gate_logits", lambda x, Wg, bias: x @ Wg.T)   # forgets the bias
    assert not pin_gate_bias_golden()


def test_planted_gate_bias_misapplied_is_caught(monkeypatch):
    def per_token(x, Wg, bias):          # adds b[t] to token t's logits instead of b[e] to e's
        l = x @ Wg.T
        return l if bias is None else l + np.asarray(bias)[:x.shape[0], None]

    def subtracted(x, Wg, bias):
        l = x @ Wg.T
        return l if bias is None else l - np.asarray(bias)[None, :]
    _planted(monkeypatch, "gate_logits", per_token)
    assert not pin_gate_bias_golden()
    _planted(monkeypatch, "gate_logits", subtracted)
    assert not pin_gate_bias_golden()


def test_planted_gelu_grad_missing_term_is_caught(monkeypatch):
    Phi = lambda u: 0.5 * (1.0 + __import__("scipy.special", fromlist=["erf"]).erf(u / math.sqrt(2)))
    _planted(monkeypatch, "gelu_grad", Phi)              # drops the u * phi(u) term
    assert not pin_activation_derivatives()
    p = _tiny_layer(1, act=mo.GELU, cf=0.75)
    assert not pin_backward_fd(p)


def test_planted_silu_grad_error_is_caught(monkeypatch):
    _planted(monkeypatch, "silu_grad", mo.sigmoid)       # forgets the product rule
    p = _tiny_layer(2, act=mo.SWIGLU, cf=1.0, n_shared=1)
    assert not pin_backward_fd(p)


def test_planted_router_sign_error_is_caught(monkeypatch):
    orig = mo.router_backward
    _planted(monkeypatch, "router_backward", lambda *a: -orig(*a))
    assert not pin_backward_fd(_tiny_layer(1, act=mo.GELU, cf=0.75))


def test_planted_renorm_router_error_is_caught(monkeypatch):
    def wrong(logits, idx, g, dg, gate_norm):      # treats the renormalised gate like the full one
        return mo.__dict__["_orig_rb"](logits, idx, g, dg, 0)
    monkeypatch.setitem(mo.__dict__, "_orig_rb", mo.router_backward)
    _planted(monkeypatch, "router_backward", wrong)
    assert not pin_backward_fd(_tiny_layer(3, act=mo.SWIGLU, gate_norm=1, cf=None))


def test_planted_tie_toward_higher_index_is_caught(monkeypatch):
    def wrong(logits, k):
        E = logits.shape[1]
        rev = np.argsort(-logits[:, ::-1], axis=1, kind="stable")
        return (E - 1 - rev)[:, :k]
    _planted(monkeypatch, "select_topk", wrong)
    assert not pin_ties_golden()
    assert not pin_topk_brute()


def test_planted_choice_major_drop_order_is_caught(monkeypatch):
    def wrong(idx, E, C, choice_major=False):            # always all first choices first
        T, k = idx.shape
        counts = np.zeros(E, dtype=np.int64)
        pos = np.full((T, k), -1, dtype=np.int64)
        for j in range(k):
            for t in range(T):
                e = idx[t, j]
                if C is None or counts[e] < C:
                    pos[t, j] = counts[e]
                counts[e] += 1
        kept = counts.copy() if C is None else np.minimum(counts, C)
        return counts, kept, pos
    _planted(monkeypatch, "dispatch", wrong)
    assert not pin_dispatch_brute()


def test_planted_aux_loss_without_expert_count_is_caught(monkeypatch):
    def wrong(logits, counts, k, coef):                  # forgets the factor E
        T, E = logits.shape
        f = np.asarray(counts, dtype=np.float64) / (T * k)
        return float(coef * np.sum(f * mo.softmax(logits).mean(axis=0)))
    _planted(monkeypatch, "aux_loss", wrong)
    assert not pin_aux_loss_closed_forms()


def test_planted_aux_grad_missing_centering_is_caught(monkeypatch):
    def wrong(logits, counts, k, coef):                  # drops the -<p, f> term
        T, E = logits.shape
        f = np.asarray(counts, dtype=np.float64) / (T * k)
        return coef * E / T * mo.softmax(logits) * f[None, :]
    _planted(monkeypatch, "aux_loss_grad", wrong)
    assert not pin_aux_grad_fd()


def test_planted_aux_grad_left_out_of_backward_is_caught(monkeypatch):
    _planted(monkeypatch, "aux_loss_grad", lambda logits, counts, k, coef: np.zeros(logits.shape))
    c = dict(FD_CASES["gelu_aux_drops"])
    p = _tiny_layer(c.pop("seed"), **c)
    assert not pin_backward_fd(p)


def test_planted_dropped_term_in_dx_is_caught(monkeypatch):
    orig = mo.expert_backward

    def wrong(X, U, V, H, dO, W1e, W3e, W2e, act):
        dX, dW1, dW3, dW2 = orig(X, U, V, H, dO, W1e, W3e, W2e, act)
        if V is not None:
            dX = dX - (dO @ W2e) * mo.silu(U) @ W3e      # loses the dV . W3 branch
        return dX, dW1, dW3, dW2
    _planted(monkeypatch, "expert_backward", wrong)
    assert not pin_backward_fd(_tiny_layer(2, act=mo.SWIGLU, cf=1.0, n_shared=1))


def test_planted_transposed_weight_is_caught(monkeypatch):
    def wrong(X, W1e, W3e, W2e, act):                    # uses W2 untransposed (square case)
        U = X @ W1e.T
        H = mo.gelu(U)
        return U, None, H, H @ W2e
    _planted(monkeypatch, "expert_forward", wrong)
    rng = np.random.default_rng(7)
    T, d = 5, 4
    x = rng.standard_normal((T, d))
    W1 = rng.standard_normal((1, d, d)); W2 = rng.standard_normal((1, d, d))
    f = mo.layer_forward(x, rng.standard_normal((1, d)), None, W1, None, W2, k=1, act=mo.GELU,
                         gate_norm=0, capacity_factor=1.0)
    want = np.array([brute.dense_mlp_brute(list(x[t]), W1[0].tolist(), None, W2[0].tolist(), 0)
                     for t in range(T)])
    assert not np.allclose(f["y"], want, rtol=1e-12, atol=1e-12)
