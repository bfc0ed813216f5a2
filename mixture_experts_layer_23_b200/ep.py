"""Expert parallelism: one MoE layer spread over N GPUs, each GPU owning E/N of the experts.

The pages' four-step expert-parallel workflow (Ch.4 "分布式训练", section "专家并行", part 二):
every rank gates its own tokens with the replicated router (step 1), sends each token row to the
rank that owns the chosen expert (step 2: the all-to-all of section "All-to-All 通信模式", part
二, where device i sends the subset S_ik of its tokens to expert k's device), runs its own experts
on the rows it received (step 3) and sends the results back to be combined in token order
(step 4).  The backward pass runs the same exchanges in reverse (section "专家并行与数据并行的结合",
part 三.3): output gradients go to the experts, input gradients come back, expert weight
gradients stay where the experts live and the replicated router's gradient is summed over ranks.
Section "通信优化" overlaps the exchange with expert compute on separate streams, and the FlowMoE
notes pipeline it in R micro-batches: `chunks` below splits each rank's experts into R groups
whose exchange and compute overlap.

Placement: rank q owns experts [q E/N, (q+1) E/N) (contiguous, so the dispatch's expert-contiguous
buffer is already ordered by destination rank).  Capacity is applied by each rank to its own
tokens (C = ceil(cf k T_rank / E)), so every rank's result is the single-device layer on that
rank's batch, and each expert's weight gradient is the sum of its gradients over the ranks'
batches.  Layers with shared experts are not supported here (shared experts are replicated
compute and belong to data parallelism).

Data plane: only kept rows travel, as one point-to-point message per (peer, expert) block,
grouped into one batch per exchange (NCCL ncclSend/ncclRecv through torch.distributed for real
ranks).  Senders read their blocks in place from the dispatch buffer; receivers write them in
place into an expert-major row space (per local expert: the rows of source rank 0, then rank 1,
..., padded to 128 rows), which is exactly the layout moe_expert_ffn and moe_expert_ffn_bwd take,
so no pack or unpack kernel runs.  All compute is the library's kernels; this module only plans
and moves buffers.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch

from . import moe
from .configs import DROPLESS, LayerShape
from .layer import MoELayer, act_dtype

ROW_ALIGN = 128


def _round_up(a, b):
    return (np.asarray(a, dtype=np.int64) + b - 1) // b * b


class EPPlan:
    """Host-side bookkeeping of one exchange, from every rank's kept counts.

    kept_all[src, e] = rows rank `src` keeps for expert e after its own capacity drop.
    Sender side (moe_dispatch's layout): rank r holds expert e's kept rows at
    [send_off[e], send_off[e] + kept_all[r, e]), send_off[e] = routed_row0 + sum over e' < e of
    roundup(kept_all[r, e'], 128).
    Receiver side: rank q stacks, for local expert l (global q El + l), the blocks of source ranks
    0..N-1 in order from recv_off[l], and pads the expert to a multiple of 128 rows.
    """

    def __init__(self, kept_all, rank: int, world: int, routed_row0: int = 0, chunks: int = 1):
        kept_all = np.asarray(kept_all, dtype=np.int64)
        N, E = kept_all.shape
        if N != world or E % world != 0:
            raise ValueError(f"{E} experts cannot be split evenly over {world} ranks")
        El = E // world
        if not 1 <= chunks <= El:
            raise ValueError(f"chunks must lie in [1, {El}]")
        self.rank, self.world, self.E, self.El, self.chunks = rank, world, E, El, chunks
        self.kept_all = kept_all
        seg = _round_up(kept_all[rank], ROW_ALIGN)
        self.send_off = routed_row0 + np.concatenate([[0], np.cumsum(seg)])
        mine = kept_all[:, rank * El:(rank + 1) * El]            # [src, l]
        self.recv_count = mine
        self.recv_n = mine.sum(axis=0)                            # rows per local expert
        self.recv_off = np.concatenate([[0], np.cumsum(_round_up(self.recv_n, ROW_ALIGN))])
        below = np.concatenate([np.zeros((1, El), np.int64), np.cumsum(mine, axis=0)[:-1]])
        self.recv_start = self.recv_off[:-1][None, :] + below     # [src, l]
        # experts of chunk c: [bounds[c], bounds[c + 1]) (local indices, as equal as possible)
        self.bounds = [int(round(c * El / chunks)) for c in range(chunks + 1)]

    def owner(self, e: int) -> int:
        return e // self.El

    def chunk_of(self, l: int) -> int:
        for c in range(self.chunks):
            if self.bounds[c] <= l < self.bounds[c + 1]:
                return c
        raise IndexError(l)

    def blocks_to_experts(self, chunk: int | None = None):
        """(sends, recvs) of the exchange towards the experts, as lists of
        (peer, expert, first row, rows): sends index this rank's dispatch buffer, recvs its
        receive buffer.  Blocks with no rows are left out; blocks to itself are included (the
        caller copies them).  Between any two ranks, blocks travel in expert order on both
        sides, so messages pair up in posting order.  chunk: only the experts of that chunk."""
        sends, recvs = [], []
        for e in range(self.E):
            q, l = self.owner(e), e % self.El
            if chunk is not None and self.chunk_of(l) != chunk:
                continue
            n = int(self.kept_all[self.rank, e])
            if n:
                sends.append((q, e, int(self.send_off[e]), n))
        for l in range(self.El):
            if chunk is not None and self.chunk_of(l) != chunk:
                continue
            e = self.rank * self.El + l
            for src in range(self.world):
                n = int(self.recv_count[src, l])
                if n:
                    recvs.append((src, e, int(self.recv_start[src, l]), n))
        return sends, recvs

    def blocks_back(self, chunk: int | None = None):
        """The return exchange: every receive block goes back to its source, every send block
        comes back to where it left."""
        sends, recvs = self.blocks_to_experts(chunk)
        return recvs, sends


# ----------------------------------------------------------------------------- exchanges

class DistExchange:
    """Exchange over torch.distributed (NCCL between GPUs, gloo between CPU processes): an
    all-gather of the kept counts, grouped point-to-point row blocks, a sum of the router
    gradient."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather_kept(self, kept: torch.Tensor) -> np.ndarray:
        out = [torch.empty_like(kept) for _ in range(self.world)]
        self.dist.all_gather(out, kept, group=self.group)
        return torch.stack(out).cpu().numpy().astype(np.int64)

    def move(self, src_buf: torch.Tensor, dst_buf: torch.Tensor, sends, recvs):
        """Start the transfer of row blocks: sends (peer, _, row, n) read src_buf rows, recvs
        write dst_buf rows; blocks to this rank itself are copied directly.  Returns the works
        to wait on."""
        ops, local_src, local_dst = [], [], []
        for peer, _, row, n in sends:
            if peer == self.rank:
                local_src.append(src_buf[row:row + n])
            else:
                ops.append(self.dist.P2POp(self.dist.isend, src_buf[row:row + n], peer, self.group))
        for peer, _, row, n in recvs:
            if peer == self.rank:
                local_dst.append(dst_buf[row:row + n])
            else:
                ops.append(self.dist.P2POp(self.dist.irecv, dst_buf[row:row + n], peer, self.group))
        for a, b in zip(local_src, local_dst):   # own blocks: same expert order on both sides
            b.copy_(a)
        return self.dist.batch_isend_irecv(ops) if ops else []

    @staticmethod
    def wait(works):
        for w in works:
            w.wait()

    def all_reduce_sum(self, t: torch.Tensor):
        self.dist.all_reduce(t, group=self.group)


# ----------------------------------------------------------------------------- one rank

def _empty(rows, cols, dtype, device, zero=False):
    f = torch.zeros if zero else torch.empty
    return f(max(rows, 1), cols, dtype=dtype, device=device)


@dataclass
class _Chunk:
    cfg: moe.Config
    r0: int                 # first row of the chunk in the receive space
    rows: int               # rows the chunk's tensor maps may cover (its layout's R)
    e0: int
    e1: int
    offsets: torch.Tensor   # [e1 - e0 + 1] rows relative to r0, on the device
    scratch: torch.Tensor


class EPRank:
    """This rank's part of an expert-parallel layer: its tokens' route, dispatch and combine
    (full E routing, the token-side state in a MoELayer), and its E/N experts' forward and
    backward on the rows it receives.  Every arithmetic step is one of the library's entry
    points; the exchanges between the steps are done by the caller (see step())."""

    def __init__(self, shape: LayerShape, rank: int, world: int, device="cuda", chunks: int = 1):
        if shape.n_shared:
            raise ValueError("expert parallelism here takes layers without shared experts")
        if shape.fwd_only:
            raise ValueError("expert parallelism here runs forward and backward")
        self.shape, self.rank, self.world, self.chunks = shape, rank, world, chunks
        self.device = torch.device(device)
        self.tok = MoELayer(shape, device=self.device)     # token side: ctx, scratch, y, dx, dWg
        self.dt = act_dtype(shape)
        self.El = shape.E // world
        self.plan = None

    # --- forward -------------------------------------------------------------------------
    def route_dispatch(self, x, Wg, bias):
        """Steps 1-2 on this rank's tokens; returns the kept counts (device, int32 [E])."""
        L = self.tok
        moe.route(L.cfg, x, Wg, bias, L.view("logits"), L.view("topk_idx"), L.view("topk_w"))
        moe.dispatch(L.cfg, x, L.view("topk_idx"), L.view("counts"), L.view("kept"),
                     L.view("offsets"), L.view("slot"), L.view("row_token"), L.view("Xd"),
                     L.scratch)
        return L.view("kept")

    def set_plan(self, kept_all):
        """Plan the exchange and size the receive space from every rank's kept counts."""
        s = self.shape
        self.plan = p = EPPlan(kept_all, self.rank, self.world, int(self.tok.L.routed_row0),
                               self.chunks)
        self.parts = []
        end = 0
        for c in range(self.chunks):
            e0, e1 = p.bounds[c], p.bounds[c + 1]
            n = int(p.recv_n[e0:e1].sum())
            cfg = moe.make_config(replace(s, name="ep_experts", T=max(n, 1), E=e1 - e0, k=1,
                                          capacity_factor=None, bias="none", aux_loss_coef=0.0,
                                          choice_major=False), capacity=DROPLESS)
            lay = moe.get_layout(cfg)
            r0 = int(p.recv_off[e0])
            offs = torch.tensor(p.recv_off[e0:e1 + 1] - r0, dtype=torch.int32, device=self.device)
            scratch = torch.zeros(lay.scratch_bytes, dtype=torch.uint8, device=self.device)
            self.parts.append(_Chunk(cfg, r0, int(lay.rows), e0, e1, offs, scratch))
            end = max(end, r0 + int(lay.rows))
        # receive space: padding rows must read as zero, and every chunk's tensor maps must stay
        # inside the allocation
        d, F, dev, dt = s.d, s.d_ff, self.device, self.dt
        self.R_recv = end
        self.Xd_r = _empty(end, d, dt, dev, zero=True)
        self.O_r = _empty(end, d, dt, dev)
        self.Gu_r = _empty(end, F, dt, dev)
        self.Gv_r = _empty(end, F, dt, dev) if s.act == 1 else None
        self.H_r = _empty(end, F, dt, dev)
        self.dO_r = _empty(end, d, dt, dev, zero=True)
        self.dXd_r = _empty(end, d, dt, dev)
        return p

    def experts_fwd(self, W1l, W3l, W2l, chunk: int):
        """Step 3 on the received rows of one chunk of this rank's experts."""
        c = self.parts[chunk]
        sl = slice(c.r0, c.r0 + c.rows)
        w3 = None if W3l is None else W3l[c.e0:c.e1]
        gv = None if self.Gv_r is None else self.Gv_r[sl]
        moe.expert_ffn(c.cfg, self.Xd_r[sl], self.Xd_r[sl], c.offsets, W1l[c.e0:c.e1], w3,
                       W2l[c.e0:c.e1], self.Gu_r[sl], gv, self.H_r[sl], self.O_r[sl], c.scratch)

    def combine(self):
        L = self.tok
        moe.combine(L.cfg, L.view("O"), L.view("slot"), L.view("topk_w"), L.y)
        return L.y

    # --- backward ------------------------------------------------------------------------
    def combine_bwd(self, dy):
        """Step 4 backward: dg, dlogits into scratch and dO (the token side's row space)."""
        L = self.tok
        if not hasattr(self, "dO"):
            self.dO = torch.zeros(L.L.rows, self.shape.d, dtype=self.dt, device=self.device)
            self.dXd = torch.zeros(L.L.rows, self.shape.d, dtype=self.dt, device=self.device)
        moe.combine_bwd(L.cfg, L.ctx, dy, self.dO, L.scratch)

    def experts_bwd(self, W1l, W3l, W2l, dW1l, dW3l, dW2l, chunk: int):
        c = self.parts[chunk]
        sl = slice(c.r0, c.r0 + c.rows)
        w3 = None if W3l is None else W3l[c.e0:c.e1]
        dw3 = None if dW3l is None else dW3l[c.e0:c.e1]
        gv = None if self.Gv_r is None else self.Gv_r[sl]
        moe.expert_ffn_bwd(c.cfg, self.dO_r[sl], None, self.Xd_r[sl], None, c.offsets,
                           W1l[c.e0:c.e1], w3, W2l[c.e0:c.e1], self.Gu_r[sl], gv, self.H_r[sl],
                           self.dXd_r[sl], dW1l[c.e0:c.e1], dw3, dW2l[c.e0:c.e1], c.scratch)

    def router_bwd(self, x, Wg):
        """Steps 1-2 backward: this rank's dWg (before the sum over ranks) and dx."""
        L = self.tok
        moe.router_bwd(L.cfg, L.ctx, x, Wg, self.dXd, L.dx, L.dWg, L.scratch)
        return L.dx, L.dWg

    def status(self):
        st = self.tok.status()
        for c in self.parts:
            s2 = moe.read_status(c.scratch)
            st = st or s2
        return st


def step(r: EPRank, ex: DistExchange, x, Wg, bias, W1l, W3l, W2l, dy=None, grads=None):
    """One forward (+ backward) of the expert-parallel layer on this rank.

    x: this rank's tokens; W1l, W3l, W2l: this rank's experts [E/N, ...]; grads: (dW1l, dW3l,
    dW2l) float buffers of this rank's experts.  Chunk c's exchange is issued before chunk c - 1's
    compute, so on GPUs the transfer of one chunk overlaps the expert GEMMs of the previous one
    (the exchange runs on the communication library's stream).  Returns y, and with dy also
    (dx, dWg) where dWg is already summed over all ranks (the replicated router)."""
    kept = r.route_dispatch(x, Wg, bias)
    p = r.set_plan(ex.all_gather_kept(kept))
    L = r.tok
    Xd, O = L.view("Xd"), L.view("O")
    n = p.chunks
    works = [ex.move(Xd, r.Xd_r, *p.blocks_to_experts(c)) for c in range(n)]
    back = []
    for c in range(n):
        ex.wait(works[c])
        r.experts_fwd(W1l, W3l, W2l, c)
        back.append(ex.move(r.O_r, O, *p.blocks_back(c)))
    for w in back:
        ex.wait(w)
    y = r.combine()
    if dy is None:
        return y
    r.combine_bwd(dy)
    works = [ex.move(r.dO, r.dO_r, *p.blocks_to_experts(c)) for c in range(n)]
    back = []
    for c in range(n):
        ex.wait(works[c])
        r.experts_bwd(W1l, W3l, W2l, *grads, c)
        back.append(ex.move(r.dXd_r, r.dXd, *p.blocks_back(c)))
    for w in back:
        ex.wait(w)
    dx, dWg = r.router_bwd(x, Wg)
    ex.all_reduce_sum(dWg)
    return y, dx, dWg


# ----------------------------------------------------------------------------- one process

def step_local(ranks, xs, Wg, bias, Wl, dys=None, grads=None):
    """N ranks emulated in one process on one device, in lockstep: the same steps as step(),
    with every exchange a device-to-device copy between the ranks' buffers (nothing waits on
    another rank, so any number of ranks runs on one GPU).

    ranks: EPRank objects 0..N-1; xs: each rank's tokens; Wl[q] = (W1, W3, W2) of rank q's experts;
    grads[q] = (dW1, dW3, dW2) of rank q's experts.  Returns ys and, with dys, (dxs, dWg) with dWg
    the sum over ranks of the router gradient."""
    N = len(ranks)
    kept_all = np.stack([r.route_dispatch(x, Wg, bias).cpu().numpy() for r, x in zip(ranks, xs)])
    plans = [r.set_plan(kept_all) for r in ranks]

    def move(src_bufs, dst_bufs, to_experts: bool):
        # every block is named by (source rank, expert): its rows on the token side are
        # plans[src].send_off[e] + [0, n), on the expert side plans[q].recv_start[src, l] + [0, n)
        for q in range(N):
            _, recvs = plans[q].blocks_to_experts()
            for src, e, row, n in recvs:
                srow = int(plans[src].send_off[e])
                if to_experts:
                    dst_bufs[q][row:row + n].copy_(src_bufs[src][srow:srow + n])
                else:
                    dst_bufs[src][srow:srow + n].copy_(src_bufs[q][row:row + n])

    move([r.tok.view("Xd") for r in ranks], [r.Xd_r for r in ranks], True)
    for q, r in enumerate(ranks):
        for c in range(r.chunks):
            r.experts_fwd(*Wl[q], c)
    move([r.O_r for r in ranks], [r.tok.view("O") for r in ranks], False)
    ys = [r.combine() for r in ranks]
    if dys is None:
        return ys
    for r, dy in zip(ranks, dys):
        r.combine_bwd(dy)
    move([r.dO for r in ranks], [r.dO_r for r in ranks], True)
    for q, r in enumerate(ranks):
        for c in range(r.chunks):
            r.experts_bwd(*Wl[q], *grads[q], c)
    move([r.dXd_r for r in ranks], [r.dXd for r in ranks], False)
    outs = [r.router_bwd(x, Wg) for r, x in zip(ranks, xs)]
    dWg = outs[0][1].clone()
    for _, g in outs[1:]:
        dWg += g
    return ys, [dx for dx, _ in outs], dWg
