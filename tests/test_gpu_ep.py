"""Expert parallelism (grouped_gemm_fp32_b200.ep) on one GPU.

W ranks are emulated in one process.  Every rank has its own buffers, tokens and
upstream gradient, and owns E / W routed experts; its peer tables point at the other
emulated ranks' buffers, so the exchange kernels write rows across "ranks" exactly as
they write into other GPUs' memory through peer pointers.  The phases of ep.forward /
ep.backward run for every rank in turn, so every arrival counter a kernel waits on has
been raised by kernels earlier on the same stream: no kernel waits on another one
running beside it.  The count all-gather (the only collective) is replaced by a copy of
the stacked counts.  The device plan is checked against its definition written out in
tests/common.py, and the distributed driver runs over NCCL in a one-rank group, eagerly
and captured in a CUDA graph.

Reference: the single-GPU layer (its own parity against the oracle is tested
elsewhere) on the concatenated batch, with the same weights.  A token's output and dX
rows come from the same GEMM rows whichever rank computes them.  Each expert's dW sums
the same rows in another order (the segments of the ranks, each padded to P).  The shared
experts' dW and dWg are summed over the ranks, as the data-parallel all-reduce would.

Passage: dots.llm1 Technical Report, §3.1 (all-to-all dispatch and combine of expert
parallelism, overlapped with computation) and §3.2 (expert-aligned segments).
"""
import numpy as np
import pytest
import torch
import torch.distributed as dist

import synth
from common import dims_of, ep_plan_reference
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import ep, layer

pytestmark = pytest.mark.gpu

ROW_TOL = 1e-2   # bf16 outputs, relative to max|ref| (the layer's own bar)
DW_TOL = 1e-4    # f32 sums of the same products in another order


def _rank_inputs(wl, W):
    """Tokens and upstream gradient of W ranks (rank-dependent seeds), shared weights."""
    base = synth.make_inputs(wl)
    xs, douts = [], []
    for r in range(W):
        seed = wl.seed + 7919 * (r + 1)
        xs.append(synth.normal_bf16(seed, synth.SID_X, (wl.dims.T, wl.dims.d), wl.x_std))
        douts.append(synth.normal_bf16(seed, synth.SID_DOUT, (wl.dims.T, wl.dims.d), 1.0))
    return base, xs, douts


def _device_plan(eb):
    """The plan arrays moe_ep_plan wrote into a rank's EP workspace."""
    W, E, El = eb.world, eb.dims.E, eb.El
    v = eb.ep_ws.view(torch.int32).cpu().numpy().astype(np.int64)
    o = 16
    out = {"send_dst": v[o:o + E]}
    o += E
    for key in ("recv_row", "recv_cnt", "recv_real", "src_off"):
        out[key] = v[o:o + W * El].reshape(W, El)
        o += W * El
    out["over"] = v[o:o + W]
    return out


def _rel(got, ref):
    got, ref = got.float(), ref.float()
    return float((got - ref).abs().max() / ref.abs().max().clamp_min(1e-30))


@pytest.mark.parametrize("W,E,k,T,P,off", [
    (2, 8, 2, 300, 64, None),      # two ranks, k <= E_l
    (4, 16, 6, 200, 64, None),     # four ranks, k = 6 > E_l = 4 (a token may pick all of an owner's)
    (2, 8, 3, 130, 128, None),     # pad block 128, ragged segments
    (4, 16, 2, 96, 64, (4, 8)),    # rank 1's experts switched off: it receives nothing from anyone
])
def test_expert_parallel_matches_single_gpu_layer(W, E, k, T, P, off):
    wl = synth.Workload("ep", synth.Dims(T=T, d=128, E=E, k=k, S=1, I=64, P=P), seed=21,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    base, xs, douts = _rank_inputs(wl, W)
    if off is not None:
        base["bias"][off[0]:off[1]] = -1.0
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).cuda()
    w1, w2 = bf(base["w1"]), bf(base["w2"])
    wg, bias = torch.from_numpy(base["wg"]).cuda(), torch.from_numpy(base["bias"]).cuda()
    x = [bf(a) for a in xs]
    dout = [bf(a) for a in douts]
    dims = dims_of(wl)
    El, S = E // W, wl.dims.S
    gamma = 1e-3

    # ---- reference: one GPU, the concatenated batch
    dref = moe.MoeDims.of(W * T, dims.d, E, k, S, dims.I, P)
    ref = layer.MoEBuffers(dref, train=True)
    layer.forward(ref, torch.cat(x), wg, bias, w1, w2)
    layer.backward(ref, torch.cat(x), torch.cat(dout), w1, w2, wg=wg, gamma=gamma, bias=bias)

    # ---- W emulated ranks
    ebs = [ep.EPBuffers(dims, r, W, train=True) for r in range(W)]
    ep.connect_emulated(ebs)
    wl1 = [torch.cat([w1[r * El:(r + 1) * El], w1[E:]]).contiguous() for r in range(W)]
    wl2 = [torch.cat([w2[r * El:(r + 1) * El], w2[E:]]).contiguous() for r in range(W)]
    for r, eb in enumerate(ebs):
        ep.route(eb, x[r], wg, bias)
    table = torch.stack([eb.full.counts for eb in ebs])     # what the all-gather gives
    for eb in ebs:
        eb.counts_all.copy_(table)
        ep.plan(eb)
    torch.cuda.synchronize()
    for r, eb in enumerate(ebs):                             # the device plan, exactly
        want = ep_plan_reference(table.cpu().numpy(), r, P, eb.cap)
        got = _device_plan(eb)
        for key in got:
            assert np.array_equal(got[key], want[key]), (r, key)
        assert np.array_equal(eb.counts_loc.cpu().numpy(), want["counts_loc"])
    if off is not None:
        assert int(ebs[1].counts_loc.sum()) == 0
    for r, eb in enumerate(ebs):
        ep.dispatch(eb, x[r])
    for r, eb in enumerate(ebs):
        ep.experts_forward(eb, x[r], wl1[r], wl2[r])
    out = [ep.combine(eb).clone() for eb in ebs]
    for r, eb in enumerate(ebs):
        ep.backward_dispatch(eb, dout[r])
    for r, eb in enumerate(ebs):
        ep.experts_backward(eb, x[r], dout[r], wl1[r], wl2[r])
    dx = [ep.unpermute_and_router(eb, x[r], wg).clone() for r, eb in enumerate(ebs)]
    # the bias step on the loads of all ranks (what layer.dp_bias_step all-reduces)
    total = torch.stack([eb.full.counts for eb in ebs]).sum(0).to(torch.int32)
    moe.moe_bias_update(layer.dp_dims(dims, W), total, gamma, bias, ebs[0].full.bias_next)
    torch.cuda.synchronize()
    for eb in ebs:
        assert ep.status(eb) == 0

    # ---- compare
    assert _rel(torch.cat(out), ref.out) <= ROW_TOL
    assert _rel(torch.cat(dx), ref.dx) <= ROW_TOL
    assert torch.equal(torch.cat([eb.full.topk_idx for eb in ebs]), ref.topk_idx)
    dw_comb = torch.cat([eb.full.dw_comb for eb in ebs])
    assert _rel(dw_comb, ref.dw_comb) <= DW_TOL
    for r, eb in enumerate(ebs):
        if off is not None and r == 1:   # no rows: its experts' dW are exactly zero
            assert not eb.loc.dw1[:El].any() and not eb.loc.dw2[:El].any()
            assert not ref.dw1[r * El:(r + 1) * El].any()
            continue
        assert _rel(eb.loc.dw1[:El], ref.dw1[r * El:(r + 1) * El]) <= DW_TOL
        assert _rel(eb.loc.dw2[:El], ref.dw2[r * El:(r + 1) * El]) <= DW_TOL
    assert _rel(sum(eb.loc.dw1[El:] for eb in ebs), ref.dw1[E:]) <= DW_TOL
    assert _rel(sum(eb.loc.dw2[El:] for eb in ebs), ref.dw2[E:]) <= DW_TOL
    assert _rel(sum(eb.full.dwg for eb in ebs), ref.dwg) <= DW_TOL
    assert torch.equal(ebs[0].full.bias_next, ref.bias_next)


@pytest.fixture
def nccl_one_rank():
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        yield
    finally:
        dist.destroy_process_group()


def test_distributed_driver_on_one_rank_matches_the_layer(nccl_one_rank):
    """ep.forward / ep.backward through NCCL (the all-gather of the counts) in a group of
    one, where every peer pointer is the rank's own buffer: the single-GPU layer's
    results.  Then the same step captured in a CUDA graph and replayed twice: the same
    bits each time, so the step count and arrival counters carry over correctly."""
    wl = synth.Workload("ep1", synth.Dims(T=257, d=128, E=8, k=2, S=2, I=64, P=64), seed=23,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    inp = synth.make_inputs(wl)
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).cuda()
    x, w1, w2, dout = bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]), bf(inp["dout"])
    wg, bias = torch.from_numpy(inp["wg"]).cuda(), torch.from_numpy(inp["bias"]).cuda()
    dims = dims_of(wl)
    s = torch.cuda.Stream()
    ref = layer.MoEBuffers(dims, train=True)
    eb = ep.EPBuffers(dims, 0, 1, train=True, alloc=ep.symmetric_alloc(1, "cuda"))
    ep.connect(eb)

    def step():
        ep.forward(eb, x, wg, bias, w1, w2, stream=s)
        ep.backward(eb, x, dout, w1, w2, stream=s, wg=wg, gamma=1e-3, bias=bias)

    with torch.cuda.stream(s):
        layer.forward(ref, x, wg, bias, w1, w2, stream=s)
        layer.backward(ref, x, dout, w1, w2, stream=s, wg=wg, gamma=1e-3, bias=bias)
        step()
    s.synchronize()
    assert ep.status(eb) == 0
    assert _rel(eb.full.out, ref.out) <= ROW_TOL
    assert _rel(eb.full.dx, ref.dx) <= ROW_TOL
    assert _rel(eb.loc.dw1, ref.dw1) <= DW_TOL and _rel(eb.loc.dw2, ref.dw2) <= DW_TOL
    assert _rel(eb.full.dwg, ref.dwg) <= DW_TOL
    assert torch.equal(eb.full.bias_next, ref.bias_next)
    eager = [t.clone() for t in (eb.full.out, eb.full.dx, eb.loc.dw1, eb.loc.dw2, eb.full.dwg)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for _ in range(2):
        with torch.cuda.stream(s):
            g.replay()
        s.synchronize()
        assert ep.status(eb) == 0
        for a, b in zip(eager, (eb.full.out, eb.full.dx, eb.loc.dw1, eb.loc.dw2, eb.full.dwg)):
            assert torch.equal(a, b)
    del g


def test_combine_split_is_the_combine_bit_for_bit():
    """moe_combine_split with the shared rows in their own buffer gives moe_combine's
    bits (same sums, same order, same rounding), weighted and as un-permute-sum."""
    dims = moe.MoeDims.of(333, 256, 8, 3, 2, 64, 16)
    Rr, Rt = moe.moe_rows_routed(dims), moe.moe_rows_total(dims)
    g = torch.Generator(device="cuda").manual_seed(5)
    y = torch.randn(Rt, 256, device="cuda", generator=g).to(torch.bfloat16)
    row_of = torch.randperm(Rr, device="cuda", generator=g)[:333 * 3].view(333, 3).to(torch.int32)
    row_of[7, 1] = -1  # a pick without a row adds nothing
    w = torch.rand(333, 3, device="cuda", generator=g)
    shared = y[Rr:].clone()  # a buffer of its own
    for wt in (w, None):
        a = torch.empty(333, 256, dtype=torch.bfloat16, device="cuda")
        b = torch.empty_like(a)
        moe.moe_combine(dims, y, row_of, wt, a)
        moe.moe_combine_split(dims, y[:Rr], shared, row_of, wt, b)
        torch.cuda.synchronize()
        assert torch.equal(a, b)


def test_owner_over_capacity_is_reported_without_writes_or_hangs():
    """Receive buffers smaller than what a step sends an owner: every rank's plan flags
    that owner (MOE_ERR_BAD_ROUTING in the EP workspace), no sender writes into it, its
    group table is refused, and the step still completes (every arrival counter moves, so
    no wait runs out).  Every buffer other ranks write into sits between guard bands that
    must stay intact."""
    from test_gpu_guard import Guarded
    W, E, k, T, P = 2, 8, 2, 256, 64
    wl = synth.Workload("epcap", synth.Dims(T=T, d=128, E=E, k=k, S=1, I=64, P=P), seed=31,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    base, xs, douts = _rank_inputs(wl, W)
    base["bias"][:E // W] = 1.0           # every token picks owner 0's experts
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).cuda()
    w1, w2 = bf(base["w1"]), bf(base["w2"])
    wg, bias = torch.from_numpy(base["wg"]).cuda(), torch.from_numpy(base["bias"]).cuda()
    x = [bf(a) for a in xs]
    dout = [bf(a) for a in douts]
    dims = dims_of(wl)
    El = E // W
    g = Guarded()
    alloc = lambda shape, dtype: g.wrap(torch.zeros(shape, dtype=dtype, device="cuda"))
    cap = 3 * P                           # far below the 2 * T * k rows owner 0 is sent
    ebs = [ep.EPBuffers(dims, r, W, train=True, recv_rows_cap=cap, alloc=alloc)
           for r in range(W)]
    ep.connect_emulated(ebs)
    wl1 = [torch.cat([w1[r * El:(r + 1) * El], w1[E:]]).contiguous() for r in range(W)]
    wl2 = [torch.cat([w2[r * El:(r + 1) * El], w2[E:]]).contiguous() for r in range(W)]
    for r, eb in enumerate(ebs):
        ep.route(eb, x[r], wg, bias)
    table = torch.stack([eb.full.counts for eb in ebs])
    for eb in ebs:
        eb.counts_all.copy_(table)
        ep.plan(eb)
    for r, eb in enumerate(ebs):
        ep.dispatch(eb, x[r])
    for r, eb in enumerate(ebs):
        ep.experts_forward(eb, x[r], wl1[r], wl2[r])
    for eb in ebs:
        ep.combine(eb)
    for r, eb in enumerate(ebs):
        ep.backward_dispatch(eb, dout[r])
    for r, eb in enumerate(ebs):
        ep.experts_backward(eb, x[r], dout[r], wl1[r], wl2[r])
    for r, eb in enumerate(ebs):
        ep.unpermute_and_router(eb, x[r], wg)
    torch.cuda.synchronize()
    for eb in ebs:
        assert _device_plan(eb)["over"].tolist() == [1, 0]
    statuses = [moe.moe_get_device_status(eb.ep_ws) for eb in ebs]
    assert statuses == [-5, -5], statuses          # the plan's report, on both ranks
    assert moe.moe_get_device_status(ebs[0].loc.ws) == -5   # owner 0's group table refused
    assert moe.moe_get_device_status(ebs[1].loc.ws) == 0
    assert g.intact(), "a write landed outside a receive or return buffer"
