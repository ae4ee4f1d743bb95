"""Expert parallelism (grouped_gemm_fp32_b200.ep) on one GPU.

W ranks are emulated in one process.  Every rank has its own buffers, tokens and
upstream gradient, and owns E / W routed experts.  The phases of ep.forward /
ep.backward run for every rank in turn.  Between phases, rows move by device copies
along the same EPPlan tables that the distributed driver hands to NCCL.  No kernel
waits on another rank.  The distributed exchange itself is covered on CPU
(tests/test_dist_cpu.py, gloo), and over NCCL in a one-rank group below.

Reference: the single-GPU layer (its own parity against the oracle is tested
elsewhere) on the concatenated batch, with the same weights.  A token's output and dX
rows come from the same GEMM rows whichever rank computes them.  Each expert's dW sums
the same rows in another order (the segments of the ranks, each padded to P).  The shared
experts' dW and dWg are summed over the ranks, as the data-parallel all-reduce would.

Passage: dots.llm1 Technical Report, §3.2 (expert parallelism, all-to-all dispatch and
combine around the grouped GEMM).
"""
import numpy as np
import pytest
import torch
import torch.distributed as dist

import synth
from common import dims_of
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


def _move(ebs, src_of, dst_of, back=False):
    """Emulated exchange: copy every segment along the ranks' plans (dispatch, or with
    ``back`` the return)."""
    for s, eb in enumerate(ebs):
        for o, e, a, n in eb.plan.to_owner:
            peer = ebs[o].plan
            b, m = next((b, m) for s2, e2, b, m in peer.from_source if (s2, e2) == (s, e))
            assert m == n
            if n == 0:
                continue
            if back:
                dst_of(eb)[a:a + n].copy_(src_of(ebs[o])[b:b + n])
            else:
                dst_of(ebs[o])[b:b + n].copy_(src_of(eb)[a:a + n])


def _rel(got, ref):
    got, ref = got.float(), ref.float()
    return float((got - ref).abs().max() / ref.abs().max().clamp_min(1e-30))


@pytest.mark.parametrize("W,E,k,T,P", [
    (2, 8, 2, 300, 64),     # two ranks, k <= E_l
    (4, 16, 6, 200, 64),    # four ranks, k = 6 > E_l = 4 (a token may pick all of an owner's)
    (2, 8, 3, 130, 128),    # pad block 128, ragged segments
])
def test_expert_parallel_matches_single_gpu_layer(W, E, k, T, P):
    wl = synth.Workload("ep", synth.Dims(T=T, d=128, E=E, k=k, S=1, I=64, P=P), seed=21,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    base, xs, douts = _rank_inputs(wl, W)
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
    wl1 = [torch.cat([w1[r * El:(r + 1) * El], w1[E:]]).contiguous() for r in range(W)]
    wl2 = [torch.cat([w2[r * El:(r + 1) * El], w2[E:]]).contiguous() for r in range(W)]
    for r, eb in enumerate(ebs):
        ep.route(eb, x[r], wg, bias)
    counts = [eb.full.counts.cpu().numpy() for eb in ebs]
    for r, eb in enumerate(ebs):
        cin = np.stack([counts[s][r * El:(r + 1) * El] for s in range(W)])
        ep.set_plan(eb, counts[r], cin)
    _move(ebs, lambda eb: eb.full.x_perm, lambda eb: eb.loc.x_perm)
    for r, eb in enumerate(ebs):
        ep.experts_forward(eb, x[r], wl1[r], wl2[r])
    _move(ebs, lambda eb: eb.loc.y, lambda eb: eb.full.y, back=True)
    out = [ep.combine(eb).clone() for eb in ebs]
    for r, eb in enumerate(ebs):
        ep.combine_backward(eb, dout[r])
    _move(ebs, lambda eb: eb.full.dy, lambda eb: eb.loc.dy)
    for r, eb in enumerate(ebs):
        ep.experts_backward(eb, x[r], dout[r], wl1[r], wl2[r])
    _move(ebs, lambda eb: eb.loc.dxp, lambda eb: eb.full.dxp, back=True)
    dx = [ep.unpermute_and_router(eb, x[r], wg).clone() for r, eb in enumerate(ebs)]
    # the bias step on the loads of all ranks (what layer.dp_bias_step all-reduces)
    total = torch.stack([eb.full.counts for eb in ebs]).sum(0).to(torch.int32)
    moe.moe_bias_update(layer.dp_dims(dims, W), total, gamma, bias, ebs[0].full.bias_next)
    torch.cuda.synchronize()
    for eb in ebs:
        assert moe.moe_get_device_status(eb.full.ws) == 0
        assert moe.moe_get_device_status(eb.loc.ws) == 0

    # ---- compare
    assert _rel(torch.cat(out), ref.out) <= ROW_TOL
    assert _rel(torch.cat(dx), ref.dx) <= ROW_TOL
    assert torch.equal(torch.cat([eb.full.topk_idx for eb in ebs]), ref.topk_idx)
    dw_comb = torch.cat([eb.full.dw_comb for eb in ebs])
    assert _rel(dw_comb, ref.dw_comb) <= DW_TOL
    for r, eb in enumerate(ebs):
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
    """ep.forward / ep.backward through NCCL (all_to_all_single of the counts; every
    segment a self copy) in a group of one: the single-GPU layer's results."""
    wl = synth.Workload("ep1", synth.Dims(T=257, d=128, E=8, k=2, S=2, I=64, P=64), seed=23,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    inp = synth.make_inputs(wl)
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).cuda()
    x, w1, w2, dout = bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]), bf(inp["dout"])
    wg, bias = torch.from_numpy(inp["wg"]).cuda(), torch.from_numpy(inp["bias"]).cuda()
    dims = dims_of(wl)
    s = torch.cuda.Stream()
    ref = layer.MoEBuffers(dims, train=True)
    eb = ep.EPBuffers(dims, 0, 1, train=True)
    with torch.cuda.stream(s):
        layer.forward(ref, x, wg, bias, w1, w2, stream=s)
        layer.backward(ref, x, dout, w1, w2, stream=s, wg=wg, gamma=1e-3, bias=bias)
        ep.forward(eb, x, wg, bias, w1, w2, stream=s)
        ep.backward(eb, x, dout, w1, w2, stream=s, wg=wg, gamma=1e-3, bias=bias)
    s.synchronize()
    assert _rel(eb.full.out, ref.out) <= ROW_TOL
    assert _rel(eb.full.dx, ref.dx) <= ROW_TOL
    assert _rel(eb.loc.dw1, ref.dw1) <= DW_TOL and _rel(eb.loc.dw2, ref.dw2) <= DW_TOL
    assert _rel(eb.full.dwg, ref.dwg) <= DW_TOL
    assert torch.equal(eb.full.bias_next, ref.bias_next)


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
