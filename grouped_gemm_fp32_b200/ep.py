"""Expert parallelism for the MoE layer, with the exchange on the device.

dots.llm1 Technical Report, §3.1 "Interleaved-1F1B based communication/computation
overlap" (the all-to-all dispatch and combine of expert parallelism, overlapped with
computation) and §3.2 (expert-aligned segments).  The E routed experts are split over the
W ranks of a process group: rank r owns E_l = E / W experts, r·E_l .. (r+1)·E_l - 1.  The
S shared experts run on every rank, on its own tokens.

Rows never pass through the host and no size does either.  Each rank routes and permutes
its own T tokens over all E experts (routing tables only: no x_perm), and one all-gather
of E int32 counts per rank gives every rank the whole count table, from which
``moe_ep_plan`` computes every offset on the device.  The rows then move by kernels that
write straight into the other ranks' buffers through peer pointers:

  forward   moe_ep_dispatch writes x rows into the owners' receive buffers, segment by
            segment, raising the owner's arrival counter of each expert as its segment
            lands; the owners' grouped GEMM runs its shared-expert tiles first and, before
            each local expert's tiles, waits (bounded) for that expert's segments from
            every source, so it starts on the first experts while later ones still
            arrive; its second GEMM writes each routed
            row of Y straight back into the source's buffer (``grouped_gemm_fwd_ep``); the
            source waits for every owner (``moe_ep_wait``) and combines.
  backward  moe_ep_combine_bwd writes dY rows into the owners' buffers; the owners run
            dX2, both dW and, last, dX1, whose routed rows go straight back to their
            sources (``grouped_gemm_bwd_dx_ep``); the source waits, un-permutes and runs
            the router backward.  A routed expert's dW stays on its owner; the shared
            experts' dW are data-parallel (``layer.dp_allreduce_grads``); the bias step
            uses all ranks' loads (``layer.dp_bias_step``).

Every sending kernel ends with its last CTA raising a counter in each receiving rank's EP
workspace, and receivers wait on the device until it reaches W × their step count, so a
whole step (the NCCL all-gather and all-reduce included) can be captured in a CUDA graph.

The buffers other ranks write into (the EP workspace, the receive buffers of x and dY
rows, the return buffers of Y and dX rows) come from an allocator the caller chooses:
symmetric memory (``torch.distributed._symmetric_memory``) between GPUs, plain device
memory for one rank or for ranks emulated in one process.  All compute runs in
libmoe.so; this module allocates, builds the peer tables and sequences the calls.
"""
from __future__ import annotations

import os

import torch

from . import _lib as L
from . import layer
from .layer import MoEBuffers


class EPBuffers:
    """Buffers of one rank.  ``full`` holds routing, permutation and combine over all E
    experts for this rank's T tokens (routing tables only: the x rows go straight to
    their owners).  ``loc`` holds the local grouped GEMM over the E_l owned experts plus
    the S shared ones; its x_perm / dy rows are the received rows (up to
    ``recv_rows_cap``), its y / dxp rows beyond ``loc.Rr`` the shared experts' own.

    recv_rows_cap defaults to the most a rank can receive:
    W · (T · min(k, E_l) + E_l · (P - 1)).

    ``alloc(shape, dtype)`` allocates the buffers other ranks write into (default: plain
    device memory); they are ``ep_ws``, ``loc.x_perm``, ``full.y`` and, for training,
    ``loc.dy`` and ``full.dxp``.  ``connect`` (or ``connect_emulated``) then gives this
    rank every rank's addresses of them."""

    def __init__(self, dims: L.MoeDims, rank: int, world: int, train: bool = False,
                 device="cuda", recv_rows_cap: int | None = None, alloc=None):
        if dims.E % world:
            raise ValueError(f"E = {dims.E} experts do not split over {world} ranks")
        if not 1 <= world <= L.MOE_EP_MAX_WORLD:
            raise ValueError(f"world {world} outside 1 .. {L.MOE_EP_MAX_WORLD}")
        El = dims.E // world
        cap = recv_rows_cap or world * (dims.T * min(dims.k, El) + El * (dims.P - 1))
        self.rank, self.world, self.El, self.train, self.cap = rank, world, El, train, cap
        self.dims = dims
        self.dims_loc = L.MoeDims.of(dims.T, dims.d, El, min(dims.k, El), dims.S, dims.I,
                                     dims.P, cap)
        dev = torch.device(device)
        alloc = alloc or (lambda shape, dtype: torch.empty(shape, dtype=dtype, device=dev))
        self.full = MoEBuffers(dims, device=dev, train=train, experts=False, gather=True)
        self.loc = MoEBuffers(self.dims_loc, device=dev, train=train)
        bf = torch.bfloat16
        d = dims.d
        self.ep_ws = alloc((L.moe_ep_workspace_size(dims, world),), torch.uint8)
        self.ep_ws.zero_()
        self.loc.x_perm = alloc((cap, d), bf)
        self.full.y = alloc((self.full.Rr, d), bf)
        if train:
            self.loc.dy = alloc((cap, d), bf)
            self.full.dxp = alloc((self.full.Rr, d), bf)
        self.counts_all = torch.zeros(world, dims.E, dtype=torch.int32, device=dev)
        self.counts_loc = torch.zeros(El, dtype=torch.int32, device=dev)
        self.peers = None

    def peer_visible(self):
        """The tensors other ranks write into, in the order ``connect`` exchanges them."""
        t = [self.ep_ws, self.loc.x_perm, self.full.y]
        if self.train:
            t += [self.loc.dy, self.full.dxp]
        return t

    def set_peer_addresses(self, addrs):
        """``addrs[i][o]``: rank o's device address (as mapped in this process) of the
        i-th tensor of ``peer_visible``.  Builds the peer tables of every call."""
        W, r = self.world, self.rank
        ws = addrs[0]
        P = L.MoeEpPeers.of
        self.peers = {
            "ws": P(r, W, ws),
            "x_in": P(r, W, ws, addrs[1], self.cap),        # owners' receive buffers of x rows
            "y_back": P(r, W, ws, addrs[2], self.full.Rr),  # sources' buffers of routed Y rows
        }
        if self.train:
            self.peers["dy_in"] = P(r, W, ws, addrs[3], self.cap)
            self.peers["dx_back"] = P(r, W, ws, addrs[4], self.full.Rr)


def connect(eb: EPBuffers, group=None):
    """Every rank's addresses of the peer-visible buffers, for a process group whose
    buffers were allocated with ``symmetric_alloc`` (collective: every rank calls it).
    A one-rank group needs no mapping."""
    import torch.distributed as dist
    if eb.world == 1:
        eb.set_peer_addresses([[t.data_ptr()] for t in eb.peer_visible()])
        return
    import torch.distributed._symmetric_memory as symm_mem
    grp = group if group is not None else dist.group.WORLD
    addrs = []
    for t in eb.peer_visible():
        h = symm_mem.rendezvous(t, grp)
        addrs.append([int(p) for p in h.buffer_ptrs])
    eb.set_peer_addresses(addrs)


def symmetric_alloc(world: int, device):
    """The allocator for ``EPBuffers`` under torch.distributed: symmetric memory between
    GPUs (multicast objects are not created: the exchange uses plain peer stores), plain
    device memory for a one-rank group."""
    if world == 1:
        return lambda shape, dtype: torch.empty(shape, dtype=dtype, device=device)
    os.environ.setdefault("TORCH_SYMM_MEM_DISABLE_MULTICAST", "1")
    import torch.distributed._symmetric_memory as symm_mem
    return lambda shape, dtype: symm_mem.empty(shape, dtype=dtype, device=device)


def connect_emulated(ebs):
    """Ranks emulated in one process on one GPU: each rank's peer addresses are the
    other emulated ranks' buffers."""
    cols = list(zip(*[eb.peer_visible() for eb in ebs]))
    addrs = [[t.data_ptr() for t in col] for col in cols]
    for eb in ebs:
        eb.set_peer_addresses(addrs)


# ---------------------------------------------------------------- phases --
# The forward and backward as phases between the points where a rank needs the other
# ranks (the count all-gather) or where it hands rows to them.  The distributed driver
# below runs them in order on every rank; an emulation of several ranks on one GPU runs
# each phase for every rank in turn.

def route(eb: EPBuffers, x, wg, bias, stream=None, seq_balance=None):
    """Gate, top-k and the routing tables of the padded permutation over all E experts
    (and the sequence-wise balance loss with ``seq_balance``)."""
    F = eb.full
    dm = F.dims
    L.moe_gate_topk(dm, x, wg, bias, F.topk_idx, F.topk_w, F.probs if eb.train else None, F.ws,
                    stream)
    L.moe_permute_align(dm, F.topk_idx, None, F.counts, F.offsets, F.sorted_ids, F.row_of,
                        None, F.ws, stream)
    if eb.train:
        F.bal_seq_len = None
        if seq_balance is not None:
            alpha, seq_len = seq_balance
            L.moe_seq_balance_loss(dm, seq_len, alpha, F.topk_idx, F.probs, F.bal_loss,
                                   F.bal_grad, F.ws, stream)
            F.bal_seq_len = int(seq_len)


def plan(eb: EPBuffers, stream=None):
    """With ``eb.counts_all`` [W, E] holding every rank's counts: the step's plan, the
    local group table and the pad rows of the x receive buffer."""
    L.moe_ep_plan(eb.dims, eb.peers["ws"], eb.counts_all, eb.counts_loc, eb.cap, stream)
    L.grouped_gemm_set_groups(eb.dims_loc, eb.counts_loc, eb.loc.offsets, eb.loc.ws, stream)
    L.moe_ep_zero_pads(eb.dims, eb.peers["ws"], eb.loc.x_perm, stream)


def dispatch(eb: EPBuffers, x, stream=None):
    """This rank's x rows into their owners' receive buffers."""
    F = eb.full
    L.moe_ep_dispatch(eb.dims, eb.peers["x_in"], F.sorted_ids, F.offsets, x, stream)


def experts_forward(eb: EPBuffers, x, w1_loc, w2_loc, stream=None):
    """The owner's grouped GEMM over the received rows and the shared experts on this
    rank's x; the routed Y rows go back into their sources' ``full.y``.
    w1_loc [E_l + S, 2I, d], w2_loc [E_l + S, d, I]: the owned experts' weights followed
    by the shared experts'."""
    Lc = eb.loc
    L.grouped_gemm_fwd_ep(eb.dims_loc, Lc.ws, eb.peers["y_back"], Lc.x_perm, x, w1_loc, w2_loc,
                          Lc.h, Lc.a1, Lc.y, stream)


def combine(eb: EPBuffers, stream=None):
    """out = the routed rows returned into ``full.y``, weighted, plus the shared experts'
    rows of the local GEMM (after waiting for every owner)."""
    F, Lc = eb.full, eb.loc
    L.moe_ep_wait(eb.peers["ws"], L.MOE_EP_WAIT_Y, stream)
    L.moe_combine_split(F.dims, F.y, Lc.y[Lc.Rr:], F.row_of, F.topk_w, F.out, stream)
    return F.out


def backward_dispatch(eb: EPBuffers, dout, stream=None):
    """The combine-weight gradient, and this rank's dY rows into their owners' receive
    buffers (whose pad rows the owner zeroes here)."""
    F = eb.full
    L.moe_ep_zero_pads(eb.dims, eb.peers["ws"], eb.loc.dy, stream)
    L.moe_ep_combine_bwd(eb.dims, eb.peers["dy_in"], dout, F.y, F.row_of, F.topk_w, F.topk_idx,
                         F.offsets, F.dw_comb, stream)


def experts_backward(eb: EPBuffers, x, dout, w1_loc, w2_loc, stream=None):
    """The owner's dX and dW over the received dY rows (the shared experts' on this rank's
    upstream gradient).  dX1 runs last: its routed rows go back to their sources, and a
    source starts its next step's rows only after every owner has returned them, so by
    then this owner has read its receive buffers for the last time."""
    Lc, dl = eb.loc, eb.dims_loc
    L.grouped_gemm_bwd_dx_ep(dl, Lc.ws, eb.peers["ws"], L.MOE_GEMM2, Lc.dy, dout, w2_loc, Lc.a1,
                             Lc.da, stream)
    L.grouped_gemm_bwd_dw(dl, Lc.ws, L.MOE_GEMM2, Lc.dy, dout, Lc.h, None, Lc.dw2, 0, stream)
    L.grouped_gemm_bwd_dw(dl, Lc.ws, L.MOE_GEMM1, Lc.da, None, Lc.x_perm, x, Lc.dw1, 0, stream)
    L.grouped_gemm_bwd_dx_ep(dl, Lc.ws, eb.peers["dx_back"], L.MOE_GEMM1, Lc.da, None, w1_loc,
                             None, Lc.dxp, stream)


def unpermute_and_router(eb: EPBuffers, x, wg=None, stream=None):
    """dX = the returned dX rows summed per token plus the shared experts' rows (after
    waiting for every owner), then the router backward's term (with ``wg``)."""
    F, Lc = eb.full, eb.loc
    L.moe_ep_wait(eb.peers["ws"], L.MOE_EP_WAIT_DX, stream)
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

def gather_counts(eb: EPBuffers, group=None, stream=None):
    """Every rank's per-expert counts into ``eb.counts_all`` [W, E] (an all-gather of E
    int32 per rank; sizes are fixed, so it stays on the device)."""
    import torch.distributed as dist
    with layer.on_stream(stream):
        dist.all_gather_into_tensor(eb.counts_all.view(-1), eb.full.counts, group=group)


def forward(eb: EPBuffers, x, wg, bias, w1_loc, w2_loc, group=None, stream=None,
            seq_balance=None):
    """The layer's forward under expert parallelism over ``group`` (every rank calls it).
    Returns this rank's out [T, d].  Nothing comes to the host."""
    with layer.on_stream(stream):
        route(eb, x, wg, bias, stream, seq_balance)
        gather_counts(eb, group, stream)
        plan(eb, stream)
        dispatch(eb, x, stream)
        experts_forward(eb, x, w1_loc, w2_loc, stream)
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
        backward_dispatch(eb, dout, stream)
        experts_backward(eb, x, dout, w1_loc, w2_loc, stream)
        unpermute_and_router(eb, x, wg, stream)
        if gamma is not None:
            layer.dp_bias_step(F, gamma, bias, group, stream)
    return F.dx


def status(eb: EPBuffers, stream=None):
    """First device error of this rank's exchange and GEMMs (MOE_OK = 0), cleared."""
    for ws in (eb.ep_ws, eb.loc.ws, eb.full.ws):
        st = L.moe_get_device_status(ws, stream)
        if st != 0:
            return st
    return 0
