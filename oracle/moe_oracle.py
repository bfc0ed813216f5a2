"""CPU oracle for one Mixture-of-Experts layer, forward and backward, in float64.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plainly written definition that the CUDA
library is checked against.  Only the tests, the package smoke check and the benchmark's CPU
baseline leg may import it; the library itself never does, and it shares no code with the
CUDA path (the seeded input generator is the one shared module, and it holds no layer
arithmetic).

What the layer computes comes from the pages' prose:
  * Ch.4 "分布式训练" (MoE distributed-training tutorial), section "专家并行", part 二 (the
    four-step expert-parallel workflow table): (1) a small replicated router gates each local
    token, (2) tokens travel to the experts they were routed to, (3) each expert processes the
    tokens it received, (4) results come back and the token order is restored.
  * same page, section "专家并行与数据并行的结合", part 三 (forward / backward walk-through):
    the backward pass routes gradients back along the same path and expert weight gradients
    are computed where the experts live.
  * same page, section "All-to-All 通信模式", part 二: the gate g(x) picks each token's target
    expert; device i sends the subset S_ik of its tokens to the device holding expert k.
  * same page, section "框架", Tutel usage (gate_type {'type': 'top', 'k': 2}) and section
    "实践", part 四 model config (top_k: 2): a top-k gate.
  * Piper news digest, section "方法论" 1 (resource model): "expert capacity" is an input of the
    model; no formula is given.
The pages give no formula for the softmax, the top-k tie rule, the capacity, the drop order or
the expert activation.  Each reading taken here is marked "Reading:" where it is used.

Everything is float64, computed from the exact values the GPU also sees (bf16 inputs are
widened exactly).  Library primitives used as single steps: matrix products (numpy @), a stable
argsort, scipy's erf.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

GELU = 0
SWIGLU = 1


# ----------------------------------------------------------------------------- router

def gate_logits(x: np.ndarray, Wg: np.ndarray, bias: np.ndarray | None) -> np.ndarray:
    """l[t, e] = sum_i x[t, i] * Wg[e, i] + b[e].

    The router is one linear map of the token (Ch.4 "专家并行" 二, step 1: local gating with a
    replicated router; "All-to-All 通信模式" 二: g(x)).  Reading: b is a constant per-expert
    logit offset (the synthetic workloads' "logit bias"); it shifts both selection and softmax
    and has no gradient.
    """
    l = x @ Wg.T
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def select_topk(logits: np.ndarray, k: int) -> np.ndarray:
    """The k experts with the largest logits, best first; equal logits go to the lower index.

    Top-k gate: Ch.4 "框架" (Tutel gate_type top, k=2) and "实践" 四 (top_k).  Reading: the
    selection is made on logits (softmax is monotone, and rounding can make distinct logits'
    probabilities equal); ties are broken toward the lower expert index, i.e. experts are
    ordered by the key (-logit, index).  A stable sort of -logit gives exactly that order.
    """
    assert np.all(np.isfinite(logits)), "non-finite logits are outside the contract"
    order = np.argsort(-logits, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def softmax(z: np.ndarray) -> np.ndarray:
    z = z - z.max(axis=-1, keepdims=True)
    ez = np.exp(z)
    return ez / ez.sum(axis=-1, keepdims=True)


def gate_weights(logits: np.ndarray, idx: np.ndarray, gate_norm: int) -> np.ndarray:
    """Combine weight g[t, j] of token t's j-th chosen expert.

    gate_norm 0: g = softmax over all E logits, read at the chosen experts (not renormalised).
    gate_norm 1: g = softmax over the k chosen logits only (the Mixtral-style layer).
    Reading: the pages say only "gate"; these are the two plain forms the workloads name.
    Weights are fixed before any capacity drop; a dropped assignment keeps its weight but
    contributes nothing.
    """
    if gate_norm == 0:
        p = softmax(logits)
        return np.take_along_axis(p, idx, axis=1)
    sel = np.take_along_axis(logits, idx, axis=1)
    return softmax(sel)


# ----------------------------------------------------------------------------- dispatch

def capacity(capacity_factor, k: int, T: int, E: int):
    """Per-expert capacity C = ceil(cf * k * T / E), or None for dropless routing.

    Piper digest, "方法论" 1, names expert capacity as a resource-model input without a
    formula.  Reading: capacity factor times the fair share k*T/E, rounded up; evaluated in
    double precision from the float32 capacity factor, left to right.
    """
    if capacity_factor is None:
        return None
    cf = float(np.float32(capacity_factor))
    return int(math.ceil(cf * k * T / E))


def dispatch(idx: np.ndarray, E: int, C, choice_major: bool = False):
    """Rank each expert's assignments by token index and keep rank < C.

    Ch.4 "All-to-All 通信模式" 二: device i sends subset S_ik of its tokens to the device of
    expert k; on one device this is the permutation of token rows into expert-contiguous
    buffers.  Reading ("drop by token order", position priority): within expert e the
    assignments are ordered by token index (a token chooses an expert at most once, so this is
    a total order); the first C are kept.

    choice_major (a routing variant; FSMoE summary: several routing functions): all first
    choices in token order, then all second choices, and so on, so a token's j-th choice is only
    dropped after every token's earlier choices at that expert were placed.

    Returns counts[e] (demand before the drop), kept[e] = min(counts[e], C) and pos[t, j] (the
    rank of assignment (t, j) within its expert, -1 when dropped).
    """
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    pos = np.full((T, k), -1, dtype=np.int64)
    order = ([(t, j) for j in range(k) for t in range(T)] if choice_major
             else [(t, j) for t in range(T) for j in range(k)])   # token order
    for t, j in order:
        e = idx[t, j]
        r = counts[e]
        counts[e] += 1
        if C is None or r < C:
            pos[t, j] = r
    kept = counts.copy() if C is None else np.minimum(counts, C)
    return counts, kept, pos


def expert_rows(idx: np.ndarray, pos: np.ndarray, e: int):
    """Token ids and slots (t, j) of expert e's kept assignments, in rank order."""
    tt, jj = np.nonzero((idx == e) & (pos >= 0))
    order = np.argsort(pos[tt, jj], kind="stable")
    return tt[order], jj[order]


# ----------------------------------------------------------------------------- experts

def gelu(u):
    """GELU, erf form: u * Phi(u).  Reading: the pages name no activation; the erf form is the
    exact one (the tanh approximation differs by up to ~1e-3)."""
    return 0.5 * u * (1.0 + _erf(u / math.sqrt(2.0)))


def gelu_grad(u):
    """d/du [u Phi(u)] = Phi(u) + u phi(u)."""
    Phi = 0.5 * (1.0 + _erf(u / math.sqrt(2.0)))
    phi = np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)
    return Phi + u * phi


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    return z * sigmoid(z)


def silu_grad(z):
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def expert_forward(X, W1e, W3e, W2e, act: int):
    """One expert FFN on the rows X: (U, V, H, O).

    Each expert is an MLP (Ch.4 "专家并行" 一: each expert is a large MLP; 二 step 3: each
    device runs its local experts on the tokens it received).  Reading: no biases;
    GELU: H = gelu(X W1^T); SwiGLU: H = silu(X W1^T) * (X W3^T); O = H W2^T.
    """
    U = X @ W1e.T
    if act == GELU:
        V = None
        H = gelu(U)
    else:
        V = X @ W3e.T
        H = silu(U) * V
    O = H @ W2e.T
    return U, V, H, O


def expert_backward(X, U, V, H, dO, W1e, W3e, W2e, act: int):
    """Chain rule through one expert: (dX, dW1, dW3, dW2) given dO = dL/dO."""
    dW2 = dO.T @ H
    dH = dO @ W2e
    if act == GELU:
        dU = dH * gelu_grad(U)
        dV = None
    else:
        dU = dH * V * silu_grad(U)
        dV = dH * silu(U)
    dW1 = dU.T @ X
    dX = dU @ W1e
    dW3 = None
    if dV is not None:
        dW3 = dV.T @ X
        dX = dX + dV @ W3e
    return dX, dW1, dW3, dW2


# ----------------------------------------------------------------------------- load balancing

def aux_loss(logits, counts, k: int, coef: float) -> float:
    """Auxiliary load-balancing loss.

    Ch.4 "分布式训练": section "框架" (DeepSpeed config: `loss_coef`, the load-balancing loss
    coefficient), section "实践" part 四 (model config `aux_loss_factor`) and part 七.3 (the
    auxiliary loss should sit near 0 with experts chosen evenly).  The pages give no formula.
    Reading: coef * E * sum_e f_e * P_e, with f_e = counts[e] / (T k) the share of the T k
    assignments routed to expert e (before the capacity drop) and P_e the mean over tokens of
    the full softmax probability of e.  At a perfectly even routing with uniform probabilities
    it equals coef, so with the pages' small coefficients it stays near 0; it grows to coef * E
    when every token goes to one expert with certainty.
    """
    T, E = logits.shape
    f = np.asarray(counts, dtype=np.float64) / (T * k)
    P = softmax(logits).mean(axis=0)
    return float(coef * E * np.sum(f * P))


def aux_loss_grad(logits, counts, k: int, coef: float) -> np.ndarray:
    """dL_aux / dlogits.  f is piecewise constant in the logits (no gradient through the
    selection); dP_e / dl[t, :] = (1/T) p_t * (onehot_e - p_t), so
    dl[t] = coef * E / T * p_t * (f - <p_t, f>)."""
    T, E = logits.shape
    f = np.asarray(counts, dtype=np.float64) / (T * k)
    p = softmax(logits)
    return coef * E / T * p * (f[None, :] - (p @ f)[:, None])


# ----------------------------------------------------------------------------- whole layer

def layer_forward(x, Wg, bias, W1, W3, W2, *, k: int, act: int, gate_norm: int,
                  capacity_factor, n_shared: int = 0, identity_experts: bool = False,
                  idx_override: np.ndarray | None = None, capacity_override=None,
                  aux_loss_coef: float = 0.0, choice_major: bool = False):
    """Forward of the layer: route, dispatch under capacity, run experts, combine.

    Combine (Ch.4 "专家并行" 二 step 4: results return and sequence order is restored):
    y_t = sum over t's kept assignments j of g[t, j] * o_tj, plus each shared expert's output
    on t with weight 1.  A token whose assignments were all dropped gets 0 from the routed part.
    Reading: the residual connection is outside the layer.

    identity_experts: every expert returns its input (o = x), a pin of dispatch + combine.
    idx_override: route with these expert ids instead of re-selecting (used to compare against a
    device whose logits differ from the oracle's inside a near-tie).
    capacity_override: an explicit capacity C instead of the one the capacity factor gives.
    aux_loss_coef: weight of the load-balancing loss (aux_loss); 0 leaves it out.
    choice_major: the drop priority of dispatch (default: token order).
    """
    T, d = x.shape
    E = Wg.shape[0]
    logits = gate_logits(x, Wg, bias)
    idx = select_topk(logits, k) if idx_override is None else np.asarray(idx_override, np.int64)
    g = gate_weights(logits, idx, gate_norm)
    C = capacity(capacity_factor, k, T, E) if capacity_override is None else capacity_override
    counts, kept, pos = dispatch(idx, E, C, choice_major)
    y = np.zeros((T, d))
    cache = {}
    for e in range(E):
        tt, jj = expert_rows(idx, pos, e)
        if len(tt) == 0:
            continue
        X = x[tt]
        if identity_experts:
            U = V = H = None
            O = X.copy()
        else:
            U, V, H, O = expert_forward(X, W1[e], None if W3 is None else W3[e], W2[e], act)
        np.add.at(y, tt, g[tt, jj][:, None] * O)
        cache[e] = (tt, jj, X, U, V, H, O)
    for s in range(n_shared):
        e = E + s
        if identity_experts:
            U = V = H = None
            O = x.copy()
        else:
            U, V, H, O = expert_forward(x, W1[e], None if W3 is None else W3[e], W2[e], act)
        y = y + O
        cache[e] = (np.arange(T), None, x, U, V, H, O)
    aux = aux_loss(logits, counts, k, aux_loss_coef) if aux_loss_coef else 0.0
    return {"logits": logits, "idx": idx, "g": g, "C": C, "counts": counts, "kept": kept,
            "pos": pos, "y": y, "cache": cache, "k": k, "act": act, "gate_norm": gate_norm,
            "E": E, "n_shared": n_shared, "aux_loss": aux, "aux_loss_coef": aux_loss_coef}


def router_backward(logits, idx, g, dg, gate_norm: int):
    """dL/dlogits from dL/dg.  Selection and drops are piecewise constant: no gradient flows
    through the chosen indices.

    gate_norm 0: dp[e] = sum_j [idx_j = e] dg_j; dl = p * (dp - <p, dp>) over all E.
    gate_norm 1: dl at the chosen experts = w * (dg - <w, dg>); 0 elsewhere.
    """
    T, E = logits.shape
    dl = np.zeros((T, E))
    if gate_norm == 0:
        p = softmax(logits)
        dp = np.zeros((T, E))
        np.add.at(dp, (np.repeat(np.arange(T), idx.shape[1]), idx.reshape(-1)), dg.reshape(-1))
        dl = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    else:
        dsel = g * (dg - (g * dg).sum(axis=1, keepdims=True))
        np.put_along_axis(dl, idx, dsel, axis=1)
    return dl


def layer_backward(fwd: dict, x, Wg, W1, W3, W2, dy):
    """Backward of the layer for the scalar L = <y, dy> (+ the load-balancing loss when the
    forward had a coefficient).

    Ch.4 "专家并行与数据并行的结合" 三.3: gradients are routed back to the experts, whose weight
    gradients are computed locally; the router and the token rows receive theirs on the way back.
    Returns dx, dWg, dW1, dW3 (None for GELU), dW2 and dg (dL/dg, 0 at dropped assignments).
    """
    T, d = x.shape
    E, k, act = fwd["E"], fwd["k"], fwd["act"]
    idx, g = fwd["idx"], fwd["g"]
    dx = np.zeros_like(x)
    dg = np.zeros_like(g)
    dW1 = np.zeros_like(W1)
    dW2 = np.zeros_like(W2)
    dW3 = None if W3 is None else np.zeros_like(W3)
    for e, (tt, jj, X, U, V, H, O) in fwd["cache"].items():
        if e < E:
            dg[tt, jj] = np.einsum("rd,rd->r", dy[tt], O)
            dO = g[tt, jj][:, None] * dy[tt]
        else:
            dO = dy
        dX, dW1e, dW3e, dW2e = expert_backward(X, U, V, H, dO, W1[e],
                                               None if W3 is None else W3[e], W2[e], act)
        np.add.at(dx, tt, dX)
        dW1[e] = dW1e
        dW2[e] = dW2e
        if dW3 is not None:
            dW3[e] = dW3e
    dl = router_backward(fwd["logits"], idx, g, dg, fwd["gate_norm"])
    if fwd.get("aux_loss_coef"):
        dl = dl + aux_loss_grad(fwd["logits"], fwd["counts"], k, fwd["aux_loss_coef"])
    dWg = dl.T @ x
    dx = dx + dl @ Wg
    return {"dx": dx, "dWg": dWg, "dW1": dW1, "dW3": dW3, "dW2": dW2, "dg": dg, "dlogits": dl}


# ----------------------------------------------------------------------------- sampled forms
# The same definitions restricted to a few tokens / weight rows, for layers too large to run
# whole on the CPU.  Each is the full-layer formula evaluated on a subset; nothing is
# approximated.

def route(x, Wg, bias, *, k, gate_norm, capacity_factor, choice_major=False):
    """Router + dispatch for all tokens (cheap: T*d*E multiply-adds)."""
    T = x.shape[0]
    E = Wg.shape[0]
    logits = gate_logits(x, Wg, bias)
    idx = select_topk(logits, k)
    g = gate_weights(logits, idx, gate_norm)
    C = capacity(capacity_factor, k, T, E)
    counts, kept, pos = dispatch(idx, E, C, choice_major)
    return {"logits": logits, "idx": idx, "g": g, "C": C, "counts": counts, "kept": kept, "pos": pos}


def token_forward_backward(tokens, r, x, Wg, W1, W3, W2, dy, *, act, gate_norm, n_shared):
    """y_t, dg_t and dx_t for the listed tokens, from the routing r of `route`.

    Per token: the same expert forward / backward formulas as `layer_forward` and
    `layer_backward`, evaluated on that token's rows only.
    """
    E = Wg.shape[0]
    k = r["idx"].shape[1]
    out_y, out_dx, out_dg = [], [], []
    for t in tokens:
        xt = x[t:t + 1]
        yt = np.zeros((1, x.shape[1]))
        dxt = np.zeros((1, x.shape[1]))
        dgt = np.zeros(k)
        for j in range(k):
            if r["pos"][t, j] < 0:
                continue
            e = r["idx"][t, j]
            w3 = None if W3 is None else W3[e]
            U, V, H, O = expert_forward(xt, W1[e], w3, W2[e], act)
            yt += r["g"][t, j] * O
            if dy is not None:
                dgt[j] = float(O[0] @ dy[t])
                dX, _, _, _ = expert_backward(xt, U, V, H, r["g"][t, j] * dy[t:t + 1],
                                              W1[e], w3, W2[e], act)
                dxt += dX
        for s in range(n_shared):
            e = E + s
            w3 = None if W3 is None else W3[e]
            U, V, H, O = expert_forward(xt, W1[e], w3, W2[e], act)
            yt += O
            if dy is not None:
                dX, _, _, _ = expert_backward(xt, U, V, H, dy[t:t + 1], W1[e], w3, W2[e], act)
                dxt += dX
        if dy is not None:
            dl = router_backward(r["logits"][t:t + 1], r["idx"][t:t + 1], r["g"][t:t + 1],
                                 dgt[None, :], gate_norm)
            dxt += dl @ Wg
        out_y.append(yt[0])
        out_dx.append(dxt[0])
        out_dg.append(dgt)
    return np.array(out_y), np.array(out_dx), np.array(out_dg)


def expert_weight_grad_rows(e, fs, r, x, W1, W3, W2, dy, *, act, n_shared):
    """Rows fs of dW1[e] and dW3[e] and columns fs of dW2[e] (each an exact sum over all of
    expert e's rows).  Restricting the inner dimension F to fs is exact: U[:, f], V[:, f],
    H[:, f] and dH[:, f] depend only on weight row / column f."""
    E = W1.shape[0] - n_shared
    if e < E:
        tt, jj = expert_rows(r["idx"], r["pos"], e)
        X = x[tt]
        dO = r["g"][tt, jj][:, None] * dy[tt]
    else:
        X = x
        dO = dy
    fs = np.asarray(fs)
    U = X @ W1[e][fs].T
    dH = dO @ W2[e][:, fs]
    if act == GELU:
        H = gelu(U)
        dU = dH * gelu_grad(U)
        dV = None
    else:
        V = X @ W3[e][fs].T
        H = silu(U) * V
        dU = dH * V * silu_grad(U)
        dV = dH * silu(U)
    dW1_rows = dU.T @ X
    dW3_rows = None if dV is None else dV.T @ X
    dW2_cols = dO.T @ H           # [d, len(fs)]
    return dW1_rows, dW3_rows, dW2_cols


def expert_input_grad(X, U, V, H, dO, W1e, W3e, W2e, act: int):
    """dX of one expert alone: the input-gradient part of `expert_backward` (same chain rule,
    without the weight gradients), for layers whose weight gradients are checked elsewhere."""
    dH = dO @ W2e
    if act == GELU:
        return (dH * gelu_grad(U)) @ W1e
    dU = dH * V * silu_grad(U)
    dV = dH * silu(U)
    return dU @ W1e + dV @ W3e


def layer_by_expert(x, Wg, bias, W1, W3, W2, dy, *, k: int, act: int, gate_norm: int,
                    capacity_factor, n_shared: int = 0, idx_override=None,
                    choice_major: bool = False, aux_loss_coef: float = 0.0,
                    with_dx: bool = True):
    """y, dg, dlogits, dWg and (with_dx) dx of the whole layer, one expert at a time.

    The same formulas as `layer_forward` followed by `layer_backward` (routing, dispatch, each
    expert's FFN, combine; dg = <dy, o> at kept assignments, the router backward, dWg = dl^T x,
    dx = the experts' input gradients + dl Wg), evaluated expert by expert so that no expert's
    activations are kept once its rows are done: a layer with large experts then needs only one
    expert's intermediates in memory.  W1, W3, W2 may be anything indexable by expert id.
    Weight gradients of the experts are not formed (see expert_weight_grad_rows).
    """
    T, d = x.shape
    E = Wg.shape[0]
    logits = gate_logits(x, Wg, bias)
    idx = select_topk(logits, k) if idx_override is None else np.asarray(idx_override, np.int64)
    g = gate_weights(logits, idx, gate_norm)
    C = capacity(capacity_factor, k, T, E)
    counts, kept, pos = dispatch(idx, E, C, choice_major)
    y = np.zeros((T, d))
    dx = np.zeros((T, d)) if with_dx else None
    dg = np.zeros((T, k))
    for e in range(E + n_shared):
        if e < E:
            tt, jj = expert_rows(idx, pos, e)
            if len(tt) == 0:
                continue
            X = x[tt]
        else:
            tt, jj, X = np.arange(T), None, x
        W1e, W2e = W1[e], W2[e]
        W3e = None if W3 is None else W3[e]
        U, V, H, O = expert_forward(X, W1e, W3e, W2e, act)
        if e < E:
            np.add.at(y, tt, g[tt, jj][:, None] * O)
            dg[tt, jj] = np.einsum("rd,rd->r", dy[tt], O)
            dO = g[tt, jj][:, None] * dy[tt]
        else:
            y += O
            dO = dy
        if with_dx:
            np.add.at(dx, tt, expert_input_grad(X, U, V, H, dO, W1e, W3e, W2e, act))
        del U, V, H, O, dO
    dl = router_backward(logits, idx, g, dg, gate_norm)
    if aux_loss_coef:
        dl = dl + aux_loss_grad(logits, counts, k, aux_loss_coef)
    dWg = dl.T @ x
    if with_dx:
        dx += dl @ Wg
    return {"logits": logits, "idx": idx, "g": g, "C": C, "counts": counts, "kept": kept,
            "pos": pos, "y": y, "dg": dg, "dlogits": dl, "dWg": dWg, "dx": dx}
