"""Expert parallelism for the MoE layer.  The E routed experts are split over the W ranks of
a process group, and every rank routes its own tokens.

dots.llm1 Technical Report, §3.2: training with expert parallelism, the all-to-all dispatch
and combine around the grouped GEMM.  Rank r owns E_l = E / W experts,
r·E_l .. (r+1)·E_l - 1.  The S shared experts run on every rank, on its own tokens.

Forward:
  1. Gate and top-k, then the padded permutation of this rank's tokens over all E experts
     (moe_gate_topk, moe_permute_align).  x_perm holds one P-padded segment per expert, in
     expert order, so the segments bound for one owner are adjacent.
  2. The per-expert counts go to the owners (an all-to-all of E int32 values).  Both
     tables come to the host: they give the size of every segment to move.
  3. Dispatch.  Each segment goes to its owner (grouped send/recv).  An owner lays out its
     received rows expert-major: for each of its experts, the segments of ranks 0..W-1,
     each still padded to P.  So every local expert is one group of rows
     sum_s pad(c[s, e]) of the grouped GEMM, and grouped_gemm_set_groups builds the table.
  4. The local grouped GEMM (grouped_gemm_fwd with E_l routed groups).  The shared experts'
     groups read this rank's x.
  5. Return.  The Y rows of each segment go back to their source rank, into its permuted
     layout.  moe_combine_split adds them to the shared experts' rows, which never left.

Backward:
  * The same exchange carries dY to the owners and the dX rows back.
  * A routed expert's dW stays on its owner, which holds all of that expert's rows.
  * The router backward and the bias step run on the source rank.  The bias step uses the
    loads of all ranks (layer.dp_bias_step).
  * The shared experts' dW are data-parallel: sum them with layer.dp_allreduce_grads.

Exchanges go through torch.distributed (NCCL between GPUs): all_to_all_single for the
counts and batch_isend_irecv for the segments.  A rank's segments to itself are copied
locally.  Every step runs in libmoe.so; this module only moves rows and sequences the calls.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L
from . import layer
from .layer import MoEBuffers


def _pad(c, P):
    return (np.asarray(c, np.int64) + P - 1) // P * P


class EPPlan:
    """Host tables of one step's exchange, for rank ``rank`` of ``world``.

    counts_own [E]: this rank's tokens per expert (moe_permute_align's counts).
    counts_in [W, E_l]: the tokens rank s sends to each of this rank's experts.

    ``to_owner``: (owner rank, local expert e, first row, rows), one per expert of the
    whole layer, in expert order.  These are this rank's padded segments in x_perm.
    ``from_source``: (source rank, local expert e, first row, rows), in the owner's
    expert-major order.  Each is a received segment in the local row space.
    ``local_counts`` [E_l]: the rows of each local group, all padded to P.
    Segments of zero rows are listed but move nothing.  Between two ranks, segments travel
    in increasing expert order on both sides, which is how the sends and receives pair up.
    """

    def __init__(self, counts_own, counts_in, rank: int, world: int, P: int):
        counts_own = np.asarray(counts_own, np.int64).reshape(-1)
        E = counts_own.size
        if E % world:
            raise ValueError(f"E = {E} experts do not split over {world} ranks")
        El = E // world
        counts_in = np.asarray(counts_in, np.int64).reshape(world, El)
        pad_own = _pad(counts_own, P)
        off_own = np.concatenate([[0], np.cumsum(pad_own)])
        self.rank, self.world, self.El, self.P = rank, world, El, P
        self.to_owner = [(g // El, g % El, int(off_own[g]), int(pad_own[g])) for g in range(E)]
        pad_in = _pad(counts_in, P)
        self.local_counts = pad_in.sum(axis=0).astype(np.int32)
        self.from_source = []
        row = 0
        for e in range(El):
            for s in range(world):
                n = int(pad_in[s, e])
                self.from_source.append((s, e, row, n))
                row += n
        self.recv_rows = row
        self.send_rows = int(off_own[-1])


def exchange(sends, recvs, rank: int, group=None):
    """Grouped point-to-point transfer of row blocks.  ``sends`` and ``recvs`` are lists
    of (peer rank in ``group``, tensor), in the same order per peer on both ends.
    Blocks a rank sends to itself are copied in place; the others go through
    batch_isend_irecv, which is waited on before returning."""
    import torch.distributed as dist
    mine_s = [t for p, t in sends if p == rank and t.numel()]
    mine_r = [t for p, t in recvs if p == rank and t.numel()]
    if len(mine_s) != len(mine_r):
        raise RuntimeError("self sends and receives do not pair up")
    for d, s in zip(mine_r, mine_s):
        d.copy_(s)
    glob = (lambda p: p) if group is None else (lambda p: dist.get_global_rank(group, p))
    ops = [dist.P2POp(dist.isend, t, glob(p), group) for p, t in sends if p != rank and t.numel()]
    ops += [dist.P2POp(dist.irecv, t, glob(p), group) for p, t in recvs if p != rank and t.numel()]
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()


def dispatch_lists(plan: EPPlan, src, dst):
    """(sends, recvs) that move this rank's padded segments of ``src`` (its permuted rows)
    to their owners' ``dst`` (expert-major local rows)."""
    sends = [(o, src[a:a + n]) for o, e, a, n in plan.to_owner]
    recvs = [(s, dst[a:a + n]) for s, e, a, n in plan.from_source]
    return sends, recvs


def return_lists(plan: EPPlan, src, dst):
    """(sends, recvs) that move each received segment's rows of ``src`` (local rows) back
    into the source rank's permuted rows ``dst``."""
    sends = [(s, src[a:a + n]) for s, e, a, n in plan.from_source]
    recvs = [(o, dst[a:a + n]) for o, e, a, n in plan.to_owner]
    return sends, recvs


class EPBuffers:
    """Buffers of one rank.  ``full`` holds routing, permutation and combine over all E
    experts for this rank's T tokens (no expert buffers).  ``loc`` holds the local
    grouped GEMM over the E_l owned experts plus the S shared ones.  Its x_perm / y / dy /
    dxp rows are the received rows (up to ``recv_rows_cap``); its shared rows follow at
    row ``loc.Rr``.

    recv_rows_cap defaults to the most a rank can receive:
    W · (T · min(k, E_l) + E_l · (P - 1)).
    Each source token picks at most min(k, E_l) of one owner's experts, and each
    segment adds fewer than P pad rows."""

    def __init__(self, dims: L.MoeDims, rank: int, world: int, train: bool = False,
                 device="cuda", recv_rows_cap: int | None = None):
        """``rank`` / ``world``: this process's rank in, and the size of, the process
        group that the distributed driver is given."""
        if dims.E % world:
            raise ValueError(f"E = {dims.E} experts do not split over {world} ranks")
        El = dims.E // world
        cap = recv_rows_cap or world * (dims.T * min(dims.k, El) + El * (dims.P - 1))
        self.rank, self.world, self.El, self.train = rank, world, El, train
        self.dims = dims
        self.dims_loc = L.MoeDims.of(dims.T, dims.d, El, min(dims.k, El), dims.S, dims.I,
                                     dims.P, cap)
        dev = torch.device(device)
        self.full = MoEBuffers(dims, device=dev, train=train, experts=False)
        self.loc = MoEBuffers(self.dims_loc, device=dev, train=train)
        self.counts_loc = torch.zeros(El, dtype=torch.int32, device=dev)
        self.plan: EPPlan | None = None


# ---------------------------------------------------------------- phases --
# The forward and backward are written as phases between the exchanges, so that the
# same calls serve the distributed driver below and drivers that move the rows some
# other way.

def route(eb: EPBuffers, x, wg, bias, stream=None, seq_balance=None):
    """Phase 1: gate, top-k and the padded permutation over all E experts (and the
    sequence-wise balance loss with ``seq_balance``)."""
    F = eb.full
    dm = F.dims
    L.moe_gate_topk(dm, x, wg, bias, F.topk_idx, F.topk_w, F.probs if eb.train else None, F.ws,
                    stream)
    L.moe_permute_align(dm, F.topk_idx, x, F.counts, F.offsets, F.sorted_ids, F.row_of, F.x_perm,
                        F.ws, stream)
    if eb.train:
        F.bal_seq_len = None
        if seq_balance is not None:
            alpha, seq_len = seq_balance
            L.moe_seq_balance_loss(dm, seq_len, alpha, F.topk_idx, F.probs, F.bal_loss,
                                   F.bal_grad, F.ws, stream)
            F.bal_seq_len = int(seq_len)


def make_plan(eb: EPBuffers, counts_own, counts_in) -> EPPlan:
    """This step's exchange tables from the host copies of the counts."""
    return EPPlan(counts_own, counts_in, eb.rank, eb.world, eb.dims.P)


def set_plan(eb: EPBuffers, counts_own, counts_in, plan: EPPlan | None = None):
    """Phase 2: this step's exchange tables (``plan``, or made from the counts) and the
    local groups' table.  Raises when this rank would receive more rows than its buffers
    hold (the distributed driver first agrees on that across the ranks)."""
    plan = plan or make_plan(eb, counts_own, counts_in)
    if plan.recv_rows > eb.loc.Rr:
        raise RuntimeError(f"rank {eb.rank} receives {plan.recv_rows} rows, more than its "
                           f"{eb.loc.Rr}-row buffers (recv_rows_cap)")
    eb.plan = plan
    eb.counts_loc.copy_(torch.from_numpy(plan.local_counts))
    L.grouped_gemm_set_groups(eb.dims_loc, eb.counts_loc, eb.loc.offsets, eb.loc.ws)
    return plan


def experts_forward(eb: EPBuffers, x, w1_loc, w2_loc, stream=None):
    """Phase 4: the local grouped GEMM over the received rows (eb.loc.x_perm) and the
    shared experts on this rank's x.  w1_loc [E_l + S, 2I, d], w2_loc [E_l + S, d, I]:
    the owned experts' weights followed by the shared experts'."""
    Lc = eb.loc
    L.grouped_gemm_fwd(eb.dims_loc, Lc.ws, Lc.x_perm, x, w1_loc, w2_loc, Lc.h, Lc.a1, Lc.y,
                       stream)


def combine(eb: EPBuffers, stream=None):
    """Phase 5: out = the routed rows returned into eb.full.y, weighted, plus the shared
    experts' rows of the local GEMM."""
    F, Lc = eb.full, eb.loc
    L.moe_combine_split(F.dims, F.y, Lc.y[Lc.Rr:], F.row_of, F.topk_w, F.out, stream)
    return F.out


def combine_backward(eb: EPBuffers, dout, stream=None):
    """Backward phase 1: dY of this rank's routed rows (eb.full.dy, pad rows zero) and the
    combine-weight gradient."""
    F = eb.full
    L.moe_combine_bwd(F.dims, F.ws, dout, F.y, F.row_of, F.topk_w, F.dy, F.dw_comb, stream)


def experts_backward(eb: EPBuffers, x, dout, w1_loc, w2_loc, stream=None):
    """Backward phase 2: dX and dW of the local experts over the received dY rows
    (eb.loc.dy), the shared experts' on this rank's upstream gradient."""
    Lc, dl = eb.loc, eb.dims_loc
    L.grouped_gemm_bwd_dx(dl, Lc.ws, L.MOE_GEMM2, Lc.dy, dout, w2_loc, Lc.a1, Lc.da, stream)
    L.grouped_gemm_bwd_dw(dl, Lc.ws, L.MOE_GEMM2, Lc.dy, dout, Lc.h, None, Lc.dw2, 0, stream)
    L.grouped_gemm_bwd_dx(dl, Lc.ws, L.MOE_GEMM1, Lc.da, None, w1_loc, None, Lc.dxp, stream)
    L.grouped_gemm_bwd_dw(dl, Lc.ws, L.MOE_GEMM1, Lc.da, None, Lc.x_perm, x, Lc.dw1, 0, stream)


def unpermute_and_router(eb: EPBuffers, x, wg=None, stream=None):
    """Backward phase 3: dX = the returned dX rows (eb.full.dxp) summed per token plus the
    shared experts' rows, then the router backward's term (with ``wg``)."""
    F, Lc = eb.full, eb.loc
    L.moe_combine_split(F.dims, F.dxp, Lc.dxp[Lc.Rr:], F.row_of, None, F.dx, stream)
    if wg is not None:
        if F.bal_seq_len is not None:
            L.moe_router_bwd_seqbal(F.dims, x, wg, F.probs, F.topk_idx, F.topk_w, F.dw_comb,
                                    F.bal_grad, F.bal_seq_len, None, F.dx, F.dwg, 0, F.ws, stream)
        else:
            L.moe_router_bwd(F.dims, x, wg, F.probs, F.topk_idx, F.topk_w, F.dw_comb, None, F.dx,
                             F.dwg, 0, F.ws, stream)
    return F.dx


# ------------------------------------------------------ distributed driver --

def check_capacity(recv_rows: int, cap: int, group=None, device=None):
    """Raise on every rank of ``group`` when any rank would receive more than ``cap``
    rows: the ranks agree (an all-reduce of the largest overflow) before any rows move,
    so that none is left waiting in the exchange for a rank that gave up."""
    import torch.distributed as dist
    over = torch.tensor([recv_rows - cap], dtype=torch.int64, device=device)
    dist.all_reduce(over, op=dist.ReduceOp.MAX, group=group)
    if int(over.item()) > 0:
        raise RuntimeError(f"a rank would receive {int(over.item())} rows more than its "
                           f"{cap}-row buffers (recv_rows_cap)")


def forward(eb: EPBuffers, x, wg, bias, w1_loc, w2_loc, group=None, stream=None,
            seq_balance=None):
    """The layer's forward under expert parallelism over ``group`` (every rank calls it).
    Returns this rank's out [T, d].  The counts come to the host once per step."""
    import torch.distributed as dist
    F = eb.full
    with layer.on_stream(stream):
        route(eb, x, wg, bias, stream, seq_balance)
        counts_in = torch.empty_like(F.counts)
        dist.all_to_all_single(counts_in, F.counts, group=group)
        plan = make_plan(eb, F.counts.cpu().numpy(), counts_in.cpu().numpy())
        check_capacity(plan.recv_rows, eb.loc.Rr, group, F.counts.device)
        set_plan(eb, None, None, plan)
        exchange(*dispatch_lists(eb.plan, F.x_perm, eb.loc.x_perm), eb.rank, group)
        experts_forward(eb, x, w1_loc, w2_loc, stream)
        exchange(*return_lists(eb.plan, eb.loc.y, F.y), eb.rank, group)
        return combine(eb, stream)


def backward(eb: EPBuffers, x, dout, w1_loc, w2_loc, group=None, stream=None, wg=None,
             gamma=None, bias=None):
    """The layer's backward under expert parallelism, after ``forward`` (every rank calls
    it).  Leaves this rank's dX in eb.full.dx, the owned and shared experts' dW in
    eb.loc.dw1 / eb.loc.dw2, dWg in eb.full.dwg (with ``wg``), and, with ``gamma``, the
    next bias, from the loads of all ranks, in eb.full.bias_next."""
    if not eb.train:
        raise ValueError("buffers were allocated without train=True")
    F = eb.full
    with layer.on_stream(stream):
        combine_backward(eb, dout, stream)
        exchange(*dispatch_lists(eb.plan, F.dy, eb.loc.dy), eb.rank, group)
        experts_backward(eb, x, dout, w1_loc, w2_loc, stream)
        exchange(*return_lists(eb.plan, eb.loc.dxp, F.dxp), eb.rank, group)
        unpermute_and_router(eb, x, wg, stream)
        if gamma is not None:
            layer.dp_bias_step(F, gamma, bias, group, stream)
    return F.dx
