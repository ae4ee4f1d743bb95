"""Edge cases of the whole layer through the C ABI: an empty batch, and the
shape limits (k = E, S = 8 shared experts), against the oracle; the layer-level
cases run with x_perm and with x rows gathered through sorted_ids.

Passages: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
(routed top-k plus always-on shared experts) and "Load balancing" (no token
dropped); §3.2 (padded segments).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from common import assert_close, dev, dims_of, host
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gather", [False, True])
def test_empty_batch_runs_every_call(gather):
    dm = moe.MoeDims.of(0, 128, 8, 2, 1, 64, 64)
    b = layer.MoEBuffers(dm, train=True, gather=gather)
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    wg = torch.ones(8, 128, device="cuda")
    bias = torch.zeros(8, device="cuda")
    w1 = torch.ones(9, 128, 128, dtype=torch.bfloat16, device="cuda")
    w2 = torch.ones(9, 128, 64, dtype=torch.bfloat16, device="cuda")
    b.bal_loss.fill_(5.0)
    out = layer.forward(b, x, wg, bias, w1, w2, seq_balance=(1e-2, 128))
    layer.backward(b, x, x, w1, w2, wg=wg, gamma=1e-3, bias=bias)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    assert out.shape == (0, 128)
    assert float(b.bal_loss.item()) == 0.0  # no sequence: loss 0
    assert torch.all(b.counts == 0)
    assert torch.all(b.dw1 == 0) and torch.all(b.dw2 == 0) and torch.all(b.dwg == 0)
    assert torch.equal(b.bias_next, bias)  # load 0 == mean load 0: sign 0, no step


@pytest.mark.parametrize("gather", [False, True])
def test_all_experts_chosen_and_eight_shared(gather):
    # k = E: every token uses every routed expert (w = p); S = 8 shared experts (G = 16)
    wl = synth.Workload("edge_kE_S8", synth.Dims(T=200, d=128, E=8, k=8, S=8, I=64, P=64),
                        seed=21, w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    inp = synth.make_inputs(wl)
    dm = dims_of(wl)
    b = layer.MoEBuffers(dm, train=True, gather=gather)
    x, w1, w2 = dev(inp["x"], True), dev(inp["w1"], True), dev(inp["w2"], True)
    wg = dev(inp["wg"])
    out = layer.forward(b, x, wg, dev(inp["bias"]), w1, w2)
    layer.backward(b, x, dev(inp["dout"], True), w1, w2, wg=wg)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    p, idx, w, _ = oracle.route(oracle.gate_logits(inp["x"], inp["wg"]), inp["bias"], 8)
    # the set is every expert: compare per expert, whatever the order
    assert np.all(np.sort(host(b.topk_idx), axis=1) == np.arange(8))
    np.testing.assert_allclose(host(b.counts), 200)
    ref = oracle.layer_fwd(inp["x"], idx, w, inp["w1"], inp["w2"], 8)
    assert_close(host(out), ref, "out")
    rdx, rdw = oracle.layer_bwd(inp["x"], idx, w, inp["w1"], inp["w2"], inp["dout"], 8)
    _, gdx, gdwg = oracle.router_bwd(inp["x"], inp["wg"], idx, rdw)
    assert_close(host(b.dx), rdx + gdx, "dx")
    assert_close(host(b.dwg), gdwg, "dWg")


@pytest.mark.parametrize("gather", [False, True])
def test_nan_tokens_still_get_valid_distinct_experts(gather):
    # non-finite hidden states make NaN scores; the gate must still name k distinct,
    # valid experts for them (so nothing downstream indexes out of range), and the
    # finite tokens must route as the oracle does
    wl = synth.Workload("edge_nan", synth.Dims(T=256, d=128, E=16, k=4, S=1, I=64, P=64),
                        seed=23, w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    inp = synth.make_inputs(wl)
    bad = [3, 77, 200]
    inp["x"][bad, 5] = 0x7FC0  # bf16 NaN
    dm = dims_of(wl)
    b = layer.MoEBuffers(dm, train=True, gather=gather)
    x, w1, w2 = dev(inp["x"], True), dev(inp["w1"], True), dev(inp["w2"], True)
    wg = dev(inp["wg"])
    layer.forward(b, x, wg, dev(inp["bias"]), w1, w2)
    layer.backward(b, x, dev(inp["dout"], True), w1, w2, wg=wg)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    idx = host(b.topk_idx)
    assert idx.min() >= 0 and idx.max() < 16
    assert all(len(set(r)) == 4 for r in idx)
    good = np.setdiff1d(np.arange(256), bad)
    _, oidx, _, margin = oracle.route(oracle.gate_logits(inp["x"][good], inp["wg"]), inp["bias"], 4)
    same = np.all(np.sort(idx[good], axis=1) == np.sort(oidx, axis=1), axis=1)
    assert np.all(same | (margin < 1e-5))


def test_invalid_routing_leaves_no_stale_rows():
    # a caller's routing with an expert id out of range: the permutation is refused
    # (status MOE_ERR_BAD_ROUTING), every pick is marked row -1, and the combine and
    # its backward then add only the shared experts and give the picks no gradient
    T, d, E, k, S = 64, 128, 8, 2, 1
    dm = moe.MoeDims.of(T, d, E, k, S, 64, 16)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    idx[9, 0] = 40
    Rr, Rt = moe.moe_rows_routed(dm), moe.moe_rows_total(dm)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sorted_ids = torch.empty(Rr, dtype=torch.int32, device="cuda")
    row_of = torch.full((T, k), 123456, dtype=torch.int32, device="cuda")  # stale garbage
    x_perm = torch.zeros(Rr, d, dtype=torch.bfloat16, device="cuda")
    x = dev(synth.normal_bf16(3, 1, (T, d), 1.0), True)
    moe.moe_permute_align(dm, dev(idx), x, counts, offsets, sorted_ids, row_of, x_perm, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == -5
    assert torch.all(row_of == -1)
    y = dev(synth.normal_bf16(3, 2, (Rt, d), 1.0), True)
    w = torch.full((T, k), 0.5, dtype=torch.float32, device="cuda")
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(dm, y, row_of, w, out)
    dy = torch.zeros(Rr, d, dtype=torch.bfloat16, device="cuda")
    dwc = torch.full((T, k), 9.0, dtype=torch.float32, device="cuda")
    moe.moe_combine_bwd(dm, ws, x, y, row_of, w, dy, dwc)
    torch.cuda.synchronize()
    assert torch.equal(out, y[Rr:Rr + T])  # only the shared expert's rows
    assert torch.all(dwc == 0) and torch.all(dy == 0)


@pytest.mark.parametrize("gather", [False, True])
def test_256_experts_full_layer(gather):
    # E = 256 routed experts (the largest supported) + 2 shared: G = 258 groups, many of
    # them short or empty; forward, backward and the router backward against the oracle
    # with the oracle's routing injected
    wl = synth.Workload("edge_e256", synth.Dims(T=1024, d=256, E=256, k=8, S=2, I=128, P=64),
                        seed=25, w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    inp = synth.make_inputs(wl)
    dm = dims_of(wl)
    p, oidx, ow, _ = oracle.route(oracle.gate_logits(inp["x"], inp["wg"]), inp["bias"], 8)
    b = layer.MoEBuffers(dm, train=True, gather=gather)
    x, w1, w2 = dev(inp["x"], True), dev(inp["w1"], True), dev(inp["w2"], True)
    wg = dev(inp["wg"])
    out = layer.forward(b, x, wg, dev(inp["bias"]), w1, w2,
                        routing=(dev(oidx), dev(ow.astype(np.float32)), dev(p.astype(np.float32))))
    layer.backward(b, x, dev(inp["dout"], True), w1, w2, wg=wg)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    assert host(b.counts).sum() == 1024 * 8  # no token dropped
    toks = np.arange(0, 1024, 7)
    ref = oracle.layer_fwd(inp["x"], oidx, ow, inp["w1"], inp["w2"], 2, tokens=toks)
    assert_close(host(out)[toks], ref, "out")
    rdx, rdw = oracle.layer_bwd(inp["x"], oidx, ow, inp["w1"], inp["w2"], inp["dout"], 2)
    _, gdx, gdwg = oracle.router_bwd(inp["x"], inp["wg"], oidx, rdw)
    assert_close(host(b.dx), rdx + gdx, "dx")
    assert_close(host(b.dwg), gdwg, "dWg")
    DW1, DW2 = host(b.dw1), host(b.dw2)
    for g in (0, 97, 255, 256, 257):  # routed groups and both shared groups
        r1, r2 = oracle.group_dw(inp["x"], oidx, ow, inp["w1"], inp["w2"], inp["dout"], 2, g)
        if np.max(np.abs(r1)) == 0:
            assert np.all(DW1[g] == 0) and np.all(DW2[g] == 0)
            continue
        assert_close(DW1[g], r1, f"dW1[{g}]")
        assert_close(DW2[g], r2, f"dW2[{g}]")
