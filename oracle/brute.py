"""Brute-force restatements of the routing steps and a loop-level dense MLP, for tiny inputs.

TEST INFRASTRUCTURE ONLY (same rule as moe_oracle: tests, smoke and the CPU baseline only).
Pure Python on lists of floats: no NumPy in the arithmetic, written independently of
moe_oracle so the two can pin each other on tiny cases.
"""
from __future__ import annotations

import math


def topk_brute(row, k):
    """Sort every expert by (-logit, index) and take the first k."""
    return [e for _, e in sorted(((-v, e) for e, v in enumerate(row)))][:k]


def dispatch_brute(idx_rows, E, C, choice_major=False):
    """For each expert, list its assignments in priority order -- token order, or with
    choice_major by (choice index, token) -- then cut the list at C.

    Returns (counts, kept, pos) with pos[t][j] = -1 for dropped assignments."""
    per_expert = [[] for _ in range(E)]
    for t, row in enumerate(idx_rows):
        for j, e in enumerate(row):
            per_expert[e].append((t, j))
    if choice_major:
        per_expert = [sorted(lst, key=lambda tj: (tj[1], tj[0])) for lst in per_expert]
    pos = [[-1] * len(row) for row in idx_rows]
    counts = [len(lst) for lst in per_expert]
    kept = []
    for e in range(E):
        lst = per_expert[e]
        n = len(lst) if C is None else min(len(lst), C)
        kept.append(n)
        for r in range(n):
            t, j = lst[r]
            pos[t][j] = r
    return counts, kept, pos


def normal_cdf(u):
    return 0.5 * (1.0 + math.erf(u / math.sqrt(2.0)))


def dense_mlp_brute(x_row, W1, W3, W2, act):
    """o = W2 . act(W1 x) with loops; act 0 = GELU (u * Phi(u)), 1 = SwiGLU."""
    F = len(W1)
    d_out = len(W2)
    h = []
    for f in range(F):
        u = sum(W1[f][i] * x_row[i] for i in range(len(x_row)))
        if act == 0:
            h.append(u * normal_cdf(u))
        else:
            v = sum(W3[f][i] * x_row[i] for i in range(len(x_row)))
            h.append(u / (1.0 + math.exp(-u)) * v)
    return [sum(W2[o][f] * h[f] for f in range(F)) for o in range(d_out)]
