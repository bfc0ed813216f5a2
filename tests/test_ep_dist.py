"""Expert parallelism's host-side logic on CPU: gloo ranks, no GPU.

Each rank holds its own tokens and E/N experts.  The test builds every rank's dispatched row
space from the oracle's routing and capacity drop (the layout moe_dispatch writes: expert
segments in expert order, kept rows in rank order, each segment padded to 128 rows), runs the
plan and the exchanges of mixture_experts_layer_23_b200.ep over torch.distributed (gloo), lets
the oracle play the experts on the rows each rank received, and checks that every rank ends
with the oracle's single-device results on its own batch: y, dx and dg; that each expert's
weight gradient, summed over ranks, equals the oracle's; and that the received rows are exactly
the expected expert-major blocks.  Runs for world sizes 2 and 4, with one and several chunks.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

D, F, K = 8, 12, 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch(rank, E, T, seed=0):
    """Rank `rank`'s tokens, dy and the shared weights, drawn from fixed seeds (every rank can
    regenerate every other rank's batch)."""
    g = np.random.default_rng(1000 * seed + rank)
    x = g.standard_normal((T, D))
    dy = g.standard_normal((T, D))
    w = np.random.default_rng(seed)
    Wg = w.standard_normal((E, D)) / np.sqrt(D)
    W1 = w.standard_normal((E, F, D)) / np.sqrt(D)
    W3 = w.standard_normal((E, F, D)) / np.sqrt(D)
    W2 = w.standard_normal((E, D, F)) / np.sqrt(F)
    bias = w.standard_normal(E) * 0.7   # skew the routing so the capacity cut drops rows
    return x, dy, Wg, bias, W1, W3, W2


def _row_space(r, kept, E):
    """Dispatch layout of one rank's assignments: (row of each kept assignment, total rows)."""
    seg = (kept + 127) // 128 * 128
    off = np.concatenate([[0], np.cumsum(seg)])
    rows = np.full(r["idx"].shape, -1)
    keep = r["pos"] >= 0
    rows[keep] = off[r["idx"][keep]] + r["pos"][keep]
    return rows, int(off[-1]), off


def _rank_main(rank, world, port, E, T, cf, chunks, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from mixture_experts_layer_23_b200.ep import DistExchange, EPPlan
    from oracle import moe_oracle as mo
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ex = DistExchange()
        El = E // world
        kw = dict(k=K, act=mo.SWIGLU, gate_norm=0, capacity_factor=cf)
        x, dy, Wg, bias, W1, W3, W2 = _batch(rank, E, T)
        r = mo.route(x, Wg, bias, k=K, gate_norm=0, capacity_factor=cf)
        kept = torch.tensor(r["kept"], dtype=torch.int32)
        kept_all = ex.all_gather_kept(kept)
        plan = EPPlan(kept_all, rank, world, 0, chunks)
        rows, R, off = _row_space(r, r["kept"], E)
        assert np.array_equal(plan.send_off, off)
        # token side: the dispatched rows (float64 so every comparison below is exact)
        Xd = torch.zeros(max(R, 1), D, dtype=torch.float64)
        keep = rows >= 0
        tt = np.repeat(np.arange(T)[:, None], K, axis=1)
        Xd[rows[keep]] = torch.from_numpy(x[tt[keep]])
        Xr = torch.zeros(max(int(plan.recv_off[-1]), 1), D, dtype=torch.float64)
        works = [ex.move(Xd, Xr, *plan.blocks_to_experts(c)) for c in range(chunks)]
        for w in works:
            ex.wait(w)
        # expected receive space: expert-major, source ranks in order, token order inside
        want = torch.zeros_like(Xr)
        for l in range(El):
            e = rank * El + l
            at = int(plan.recv_off[l])
            for src in range(world):
                xs = _batch(src, E, T)[0]
                rs = mo.route(xs, Wg, bias, k=K, gate_norm=0, capacity_factor=cf)
                tok, _ = mo.expert_rows(rs["idx"], rs["pos"], e)
                want[at:at + len(tok)] = torch.from_numpy(xs[tok])
                at += len(tok)
            assert at == plan.recv_off[l] + plan.recv_n[l]
        assert torch.equal(Xr, want)
        # the oracle plays this rank's experts on the received rows
        Or = torch.zeros_like(Xr)
        cache = {}
        for l in range(El):
            e = rank * El + l
            a, b = int(plan.recv_off[l]), int(plan.recv_off[l] + plan.recv_n[l])
            if b > a:
                U, V, H, O = mo.expert_forward(Xr[a:b].numpy(), W1[e], W3[e], W2[e], mo.SWIGLU)
                Or[a:b] = torch.from_numpy(O)
                cache[l] = (a, b, U, V, H)
        O = torch.zeros_like(Xd)
        for c in range(chunks):
            ex.wait(ex.move(Or, O, *plan.blocks_back(c)))
        # combine on the token side, as moe_combine does
        y = np.zeros((T, D))
        for t in range(T):
            for j in range(K):
                if rows[t, j] >= 0:
                    y[t] += r["g"][t, j] * O[rows[t, j]].numpy()
        f = mo.layer_forward(x, Wg, bias, W1, W3, W2, **kw)
        g = mo.layer_backward(f, x, Wg, W1, W3, W2, dy)
        assert np.allclose(y, f["y"], rtol=0, atol=1e-12)
        # backward: dg and dO on the token side, dO to the experts, dX back
        dg = np.zeros((T, K))
        dO = torch.zeros_like(Xd)
        for t in range(T):
            for j in range(K):
                if rows[t, j] >= 0:
                    dg[t, j] = float(dy[t] @ O[rows[t, j]].numpy())
                    dO[rows[t, j]] = torch.from_numpy(r["g"][t, j] * dy[t])
        assert np.allclose(dg, g["dg"], rtol=0, atol=1e-12)
        dOr = torch.zeros_like(Xr)
        for c in range(chunks):
            ex.wait(ex.move(dO, dOr, *plan.blocks_to_experts(c)))
        dXr = torch.zeros_like(Xr)
        dW = {n: np.zeros((E,) + a.shape[1:]) for n, a in (("W1", W1), ("W3", W3), ("W2", W2))}
        for l, (a, b, U, V, H) in cache.items():
            e = rank * El + l
            dX, d1, d3, d2 = mo.expert_backward(Xr[a:b].numpy(), U, V, H, dOr[a:b].numpy(), W1[e],
                                                W3[e], W2[e], mo.SWIGLU)
            dXr[a:b] = torch.from_numpy(dX)
            dW["W1"][e], dW["W3"][e], dW["W2"][e] = d1, d3, d2
        dXd = torch.zeros_like(Xd)
        for c in range(chunks):
            ex.wait(ex.move(dXr, dXd, *plan.blocks_back(c)))
        dl = mo.router_backward(r["logits"], r["idx"], r["g"], dg, 0)
        dx = dl @ Wg
        for t in range(T):
            for j in range(K):
                if rows[t, j] >= 0:
                    dx[t] += dXd[rows[t, j]].numpy()
        assert np.allclose(dx, g["dx"], rtol=0, atol=1e-12)
        # expert weight gradients: summed over ranks, each expert's equals the sum of the oracle's
        # per-rank gradients (one process owns each expert, the others contribute zeros)
        for n in dW:
            t = torch.from_numpy(dW[n])
            ex.all_reduce_sum(t)
            ref = torch.from_numpy(g["d" + n])
            ex.all_reduce_sum(ref)
            assert torch.allclose(t, ref, rtol=0, atol=1e-10), n
        dWg = torch.from_numpy(dl.T @ x)
        ex.all_reduce_sum(dWg)
        out[rank] = (int(plan.recv_n.sum()), float(dWg.abs().sum()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E,chunks", [(2, 4, 1), (2, 4, 2), (4, 8, 2)])
def test_ep_exchange_gives_each_rank_the_single_device_layer(world, E, chunks):
    T, cf = 60, 0.8
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, E, T, cf, chunks, out), nprocs=world, join=True)
        got = dict(out)
    assert sorted(got) == list(range(world))
    # every kept assignment of every rank reached exactly one expert owner
    sys.path.insert(0, ROOT)
    from oracle import moe_oracle as mo
    total = 0
    for q in range(world):
        x, _, Wg, bias, *_ = _batch(q, E, T)
        total += int(mo.route(x, Wg, bias, k=K, gate_norm=0, capacity_factor=cf)["kept"].sum())
    assert sum(v[0] for v in got.values()) == total
    # the router gradient sum is the same on every rank
    assert len({round(v[1], 9) for v in got.values()}) == 1


def test_plan_layouts():
    """EPPlan on a hand-made count table: send offsets follow the dispatch layout, receive
    blocks stack source ranks inside each expert, segments are padded to 128 rows, and both
    directions list the same blocks."""
    sys.path.insert(0, ROOT)
    from mixture_experts_layer_23_b200.ep import EPPlan
    kept_all = np.array([[5, 0, 130, 7], [1, 2, 3, 200]])
    p = EPPlan(kept_all, rank=1, world=2, routed_row0=256, chunks=2)
    assert list(p.send_off) == [256, 384, 512, 640, 896]
    assert p.El == 2 and list(p.recv_n) == [133, 207]
    assert list(p.recv_off) == [0, 256, 512]
    assert p.recv_start.tolist() == [[0, 256], [130, 263]]
    sends, recvs = p.blocks_to_experts()
    assert sends == [(0, 0, 256, 1), (0, 1, 384, 2), (1, 2, 512, 3), (1, 3, 640, 200)]
    assert recvs == [(0, 2, 0, 130), (1, 2, 130, 3), (0, 3, 256, 7), (1, 3, 263, 200)]
    assert p.blocks_back() == (recvs, sends)
    s0, r0 = p.blocks_to_experts(0)
    s1, r1 = p.blocks_to_experts(1)
    assert sorted(s0 + s1) == sorted(sends) and sorted(r0 + r1) == sorted(recvs)
    with pytest.raises(ValueError):
        EPPlan(np.zeros((2, 3), int), 0, 2)
