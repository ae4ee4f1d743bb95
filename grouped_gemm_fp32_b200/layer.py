"""One MoE FFN layer driven through the C ABI of libmoe.so.

``MoEBuffers`` owns the activations and workspace of one layer (torch device
tensors: torch is used for memory only); ``forward`` and ``backward`` issue the
C-ABI calls in the layer's order on one stream.  Every arithmetic step runs in
libmoe.so.

Layer (dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
and "Load balancing"; §3.2 "Efficient implementation of Grouped GEMM"):
    forward   moe_gate_topk -> moe_permute_align -> grouped_gemm_fwd[_gather] -> moe_combine
    backward  moe_combine_bwd -> grouped_gemm_bwd_dx(GEMM2) -> grouped_gemm_bwd_dw(GEMM2)
              -> grouped_gemm_bwd_dx(GEMM1) -> grouped_gemm_bwd_dw(GEMM1) [or _dw1_gather]
              -> moe_combine(weights = NULL)  (un-permute-sum of the dX rows)
              [-> moe_router_bwd (dlogits; gate term added into dX; dWg), or
                  moe_router_bwd_seqbal after forward's moe_seq_balance_loss]
              [-> moe_bias_update (next step's selection bias)]
The router backward runs when the gate weights are passed to ``backward``; the
bias step when an update speed ``gamma`` is.
Under token data parallelism, ``dp_bias_step`` (the bias step on the whole batch's
loads) and ``dp_allreduce_grads`` (the weight gradients' sum) exchange what the
ranks share, over torch.distributed.
"""
from __future__ import annotations

from contextlib import nullcontext

import torch

from . import _lib as L


class MoEBuffers:
    def __init__(self, dims: L.MoeDims, device="cuda", train: bool = False,
                 gather: bool = False, experts: bool = True):
        """``gather``: the first GEMM (and dW1) read the routed x rows straight from x
        through ``sorted_ids`` (grouped_gemm_fwd_gather / grouped_gemm_bwd_dw1_gather)
        and no x_perm [Rr, d] is allocated; otherwise (the default, faster on B200:
        the row copy costs less than the four-row gather copies) they read the
        permuted copy ``x_perm`` that moe_permute_align writes.
        ``experts=False``: the buffers of a rank whose routed rows are computed
        elsewhere (expert parallelism): routing, permutation, combine and router
        buffers, with y, dy and dxp holding the routed rows only [Rr, d]; no
        expert activations (h, a1, da) and no expert weight gradients."""
        self.dims = dims
        self.train = train
        self.gather = gather
        T, d, E, k, S, I = dims.T, dims.d, dims.E, dims.k, dims.S, dims.I
        G = E + S
        self.Rr = L.moe_rows_routed(dims)
        self.Rt = L.moe_rows_total(dims)
        if self.Rr < 0:
            raise ValueError(f"invalid dims {dims}")
        dev = torch.device(device)
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        e = lambda *s, dt=bf: torch.empty(*s, dtype=dt, device=dev)
        self.ws = torch.zeros(L.moe_workspace_size(dims), dtype=torch.uint8, device=dev)
        self.topk_idx = e(T, k, dt=i32)
        self.topk_w = e(T, k, dt=f32)
        self.counts = e(E, dt=i32)
        self.offsets = e(E + 1, dt=i32)
        self.sorted_ids = e(self.Rr, dt=i32)
        self.row_of = e(T, k, dt=i32)
        self.x_perm = None if gather else e(self.Rr, d)
        rows = self.Rt if experts else self.Rr
        self.h = e(self.Rt, I) if experts else None
        self.a1 = e(self.Rt, 2 * I) if train and experts else None
        self.y = e(rows, d)
        self.out = e(T, d)
        if train:
            self.dy = e(self.Rr, d)
            self.dw_comb = e(T, k, dt=f32)
            self.da = e(self.Rt, 2 * I) if experts else None
            self.dxp = e(rows, d)
            self.dx = e(T, d)
            self.dw1 = e(G, 2 * I, d, dt=f32) if experts else None
            self.dw2 = e(G, d, I, dt=f32) if experts else None
            self.probs = e(T, E, dt=f32)
            self.dwg = e(E, d, dt=f32)
            self.bias_next = e(E, dt=f32)
            # sequence-wise balance loss: its value and dL/dp per sequence (sequences
            # of >= 128 tokens, so at most ceil(T / 128) of them)
            self.bal_loss = torch.zeros(1, dtype=f32, device=dev)
            self.bal_grad = e(max(1, -(-T // 128)), E, dt=f32)
            self.bal_seq_len = None

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in vars(self).values()
                   if isinstance(t, torch.Tensor))


def forward(b: MoEBuffers, x, wg, bias, w1, w2, stream=None, routing=None, seq_balance=None):
    """out = MoE(x).  x [T, d] bf16, wg [E, d] f32, bias [E] f32, w1 [G, 2I, d], w2 [G, d, I].

    ``routing=(topk_idx, topk_w[, probs])`` (device int32 / f32 [T, k], f32 [T, E])
    replaces the gate's choice, e.g. to run the experts on a routing decided
    elsewhere.  With train buffers the gate also saves its affinities (probs) for
    the router backward.  ``seq_balance=(alpha, seq_len)`` (train buffers) also
    computes the sequence-wise balance loss into ``b.bal_loss``; ``backward``
    then adds its gradient to the router's."""
    dm = b.dims
    probs = b.probs if b.train else None
    if routing is None:
        L.moe_gate_topk(dm, x, wg, bias, b.topk_idx, b.topk_w, probs, b.ws, stream)
    else:
        b.topk_idx.copy_(routing[0])
        b.topk_w.copy_(routing[1])
        if probs is not None and len(routing) > 2:
            probs.copy_(routing[2])
    L.moe_permute_align(dm, b.topk_idx, x, b.counts, b.offsets, b.sorted_ids, b.row_of, b.x_perm,
                        b.ws, stream)
    if b.gather:
        L.grouped_gemm_fwd_gather(dm, b.ws, b.sorted_ids, x, w1, w2, b.h, b.a1, b.y, stream)
    else:
        L.grouped_gemm_fwd(dm, b.ws, b.x_perm, x, w1, w2, b.h, b.a1, b.y, stream)
    L.moe_combine(dm, b.y, b.row_of, b.topk_w, b.out, stream)
    if b.train:
        b.bal_seq_len = None
        if seq_balance is not None:
            alpha, seq_len = seq_balance
            L.moe_seq_balance_loss(dm, seq_len, alpha, b.topk_idx, b.probs, b.bal_loss,
                                   b.bal_grad, b.ws, stream)
            b.bal_seq_len = int(seq_len)
    return b.out


def backward(b: MoEBuffers, x, dout, w1, w2, stream=None, wg=None, gamma=None, bias=None):
    """Gradients after ``forward``: dx [T, d], dw1, dw2 (f32) and the combine-weight
    gradient dw_comb [T, k].  dx holds the gradient through the experts, plus the
    router's (dlogit Wg) when ``wg`` is given; then ``b.dwg`` [E, d] f32 holds dL/dWg.
    With ``gamma`` (and the step's ``bias``) ``b.bias_next`` receives the
    aux-loss-free bias step."""
    if not b.train:
        raise ValueError("buffers were allocated without train=True")
    dm = b.dims
    L.moe_combine_bwd(dm, b.ws, dout, b.y, b.row_of, b.topk_w, b.dy, b.dw_comb, stream)
    L.grouped_gemm_bwd_dx(dm, b.ws, L.MOE_GEMM2, b.dy, dout, w2, b.a1, b.da, stream)
    L.grouped_gemm_bwd_dw(dm, b.ws, L.MOE_GEMM2, b.dy, dout, b.h, None, b.dw2, 0, stream)
    L.grouped_gemm_bwd_dx(dm, b.ws, L.MOE_GEMM1, b.da, None, w1, None, b.dxp, stream)
    if b.gather:
        L.grouped_gemm_bwd_dw1_gather(dm, b.ws, b.sorted_ids, b.da, x, b.dw1, 0, stream)
    else:
        L.grouped_gemm_bwd_dw(dm, b.ws, L.MOE_GEMM1, b.da, None, b.x_perm, x, b.dw1, 0, stream)
    L.moe_combine(dm, b.dxp, b.row_of, None, b.dx, stream)
    if wg is not None:
        if b.bal_seq_len is not None:
            L.moe_router_bwd_seqbal(dm, x, wg, b.probs, b.topk_idx, b.topk_w, b.dw_comb,
                                    b.bal_grad, b.bal_seq_len, None, b.dx, b.dwg, 0, b.ws, stream)
        else:
            L.moe_router_bwd(dm, x, wg, b.probs, b.topk_idx, b.topk_w, b.dw_comb, None, b.dx,
                             b.dwg, 0, b.ws, stream)
    if gamma is not None:
        L.moe_bias_update(dm, b.counts, gamma, bias, b.bias_next, stream)
    return b.dx, b.dw1, b.dw2, b.dw_comb


# ------------------------------------------------------------- data parallel --
# Token data parallelism: every rank holds the same weights and its own tokens.
# The layer's forward and backward need nothing from the other ranks; two steps
# do.  The bias step balances the loads of the whole batch, i.e. of all ranks'
# tokens (dots.llm1 Technical Report, §"Load balancing": the bias follows the
# experts' loads).  The weight gradients of the batch are the sums of the ranks'
# own.  Both are all-reduces over torch.distributed (NCCL between GPUs), issued
# on the layer's stream.

def on_stream(stream):
    """``torch.cuda.stream(stream)`` for a torch stream, else no change of stream."""
    return torch.cuda.stream(stream) if isinstance(stream, torch.cuda.Stream) else nullcontext()


def dp_load_counts(counts, group=None, stream=None):
    """Per-expert loads of the whole data-parallel batch: ``counts`` (int32 [E], this
    rank's tokens per expert, as moe_permute_align writes them) summed over the ranks
    of ``group``.  Returns a new tensor; ``counts`` itself is left as it is (the
    backward GEMMs still read it)."""
    import torch.distributed as dist
    with on_stream(stream):
        total = counts.clone()
        dist.all_reduce(total, op=dist.ReduceOp.SUM, group=group)
    return total


def dp_dims(dims: L.MoeDims, world: int) -> L.MoeDims:
    """The dims of the whole data-parallel batch: ``world`` ranks of ``dims.T`` tokens
    each (every rank must hold the same number of tokens)."""
    return L.MoeDims.of(dims.T * world, dims.d, dims.E, dims.k, dims.S, dims.I, dims.P,
                        dims.rows_cap)


def dp_bias_step(b: MoEBuffers, gamma, bias, group=None, stream=None):
    """The aux-loss-free bias step on the loads of the whole batch:
    ``b.bias_next = bias + gamma * sign(mean - load)`` with load = the experts' token
    counts summed over the ranks of ``group`` and mean = world·T·k/E.  Every rank
    gets the same ``b.bias_next``.  Returns the summed counts."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    total = dp_load_counts(b.counts, group, stream)
    L.moe_bias_update(dp_dims(b.dims, world), total, gamma, bias, b.bias_next, stream)
    return total


def dp_allreduce_grads(grads, group=None, stream=None):
    """Sum each gradient tensor (e.g. ``b.dw1``, ``b.dw2``, ``b.dwg``) over the ranks
    of ``group``, in place: the gradients of the whole data-parallel batch."""
    import torch.distributed as dist
    with on_stream(stream):
        for g in grads:
            dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
    return grads


class HostPipeline:
    """Forward (+ backward) steps fed from and returned to pinned host memory,
    with the copies of neighbouring steps overlapped with compute.

    Two device buffer sets alternate: while step i computes on set i % 2, the
    inputs of step i + 1 are copied in on an upload stream and the results of
    step i - 1 are copied out on a download stream.  Every step still moves its
    inputs host -> device and its results device -> host; only the overlap is
    added.  All arithmetic runs in libmoe.so; torch provides memory and streams.
    """

    def __init__(self, dims: L.MoeDims, w1, w2, wg, bias, train: bool, device="cuda",
                 gamma=None, graphs: bool = True, gather: bool = False, seq_balance=None):
        self.dims, self.train, self.gamma = dims, train, gamma
        self.seq_balance = seq_balance if train else None
        self.w1, self.w2, self.wg, self.bias = w1, w2, wg, bias
        dev = torch.device(device)
        T, d = dims.T, dims.d
        self.bufs = [MoEBuffers(dims, device=dev, train=train, gather=gather) for _ in range(2)]
        # zero-filled: with graphs, one step runs on them before the capture
        e = lambda: torch.zeros(T, d, dtype=torch.bfloat16, device=dev)
        self.x = [e(), e()]
        self.dout = [e(), e()] if train else [None, None]
        self.compute = torch.cuda.Stream(device=dev)
        self.up = torch.cuda.Stream(device=dev)
        self.down = torch.cuda.Stream(device=dev)
        self.uploaded = [torch.cuda.Event(), torch.cuda.Event()]
        self.computed = [torch.cuda.Event(), torch.cuda.Event()]
        self.downloaded = [torch.cuda.Event(), torch.cuda.Event()]
        self.consumed = [torch.cuda.Event(), torch.cuda.Event()]
        for ev in self.downloaded + self.consumed:
            ev.record(self.compute)
        # one captured step per buffer set (the graphs keep the sets' addresses)
        self.graphs = None
        if graphs:
            self.graphs = [GraphStep(self.bufs[j], self.x[j], wg, bias, w1, w2,
                                     dout=self.dout[j] if train else None,
                                     gamma=gamma if train else None,
                                     seq_balance=self.seq_balance) for j in range(2)]

    def _upload(self, j, hx, hd):
        with torch.cuda.stream(self.up):
            self.up.wait_event(self.consumed[j])      # step j-2 no longer reads set j
            self.x[j].copy_(hx, non_blocking=True)
            if self.train:
                self.dout[j].copy_(hd, non_blocking=True)
            self.uploaded[j].record(self.up)

    def run(self, host_x, host_dout, host_out, host_dx, steps: int):
        """``steps`` steps; step i reads host_x[i % n] (and host_dout) and writes
        host_out[i % n] (and host_dx).  Returns after all copies are issued;
        synchronise the streams (or ``self.down``) to wait for the results."""
        n = len(host_x)
        self._upload(0, host_x[0], host_dout[0] if self.train else None)
        for i in range(steps):
            j = i & 1
            if i + 1 < steps:
                self._upload(1 - j, host_x[(i + 1) % n],
                             host_dout[(i + 1) % n] if self.train else None)
            b = self.bufs[j]
            s = self.compute
            with torch.cuda.stream(s):
                s.wait_event(self.uploaded[j])
                s.wait_event(self.downloaded[j])  # results of step i-2 have left set j
                if self.graphs is not None:
                    self.graphs[j].replay()
                else:
                    forward(b, self.x[j], self.wg, self.bias, self.w1, self.w2, stream=s,
                            seq_balance=self.seq_balance)
                    if self.train:
                        backward(b, self.x[j], self.dout[j], self.w1, self.w2, stream=s,
                                 wg=self.wg, gamma=self.gamma, bias=self.bias)
                self.computed[j].record(s)
                self.consumed[j].record(s)
            with torch.cuda.stream(self.down):
                self.down.wait_event(self.computed[j])
                host_out[i % n].copy_(b.out, non_blocking=True)
                if self.train:
                    host_dx[i % n].copy_(b.dx, non_blocking=True)
                self.downloaded[j].record(self.down)

    def synchronize(self):
        for st in (self.up, self.compute, self.down):
            st.synchronize()


class GraphStep:
    """One layer step -- forward, and with ``dout`` the backward (router backward
    and bias step included when ``gamma`` is given, the sequence-wise balance loss
    when ``seq_balance=(alpha, seq_len)`` is) -- captured once as a CUDA
    graph and replayed.  Every node is one of the same C-ABI calls as in eager
    mode, on the captured stream; the graph keeps the buffers' addresses, so new
    inputs are written into ``x`` / ``dout`` in place before ``replay``.

    The step runs once eagerly before the capture: the library's first calls set
    kernel attributes and look up driver entry points, which must not happen
    inside a capture."""

    def __init__(self, b: MoEBuffers, x, wg, bias, w1, w2, dout=None, gamma=None,
                 seq_balance=None):
        self.b = b
        self.stream = torch.cuda.Stream(device=x.device)
        args = (b, x, wg, bias, w1, w2, dout, gamma, seq_balance)
        with torch.cuda.stream(self.stream):
            self._step(self.stream, *args)
        self.stream.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            self._step(self.stream, *args)
        self.stream.synchronize()

    @staticmethod
    def _step(s, b, x, wg, bias, w1, w2, dout, gamma, seq_balance):
        forward(b, x, wg, bias, w1, w2, stream=s,
                seq_balance=seq_balance if dout is not None else None)
        if dout is not None:
            backward(b, x, dout, w1, w2, stream=s, wg=wg, gamma=gamma,
                     bias=bias if gamma is not None else None)

    def replay(self):
        self.graph.replay()
