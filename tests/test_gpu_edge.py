"""Edge cases of the whole layer through the C ABI: an empty batch, and the
shape limits (k = E, S = 8 shared experts), against the oracle.

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


def test_empty_batch_runs_every_call():
    dm = moe.MoeDims.of(0, 128, 8, 2, 1, 64, 64)
    b = layer.MoEBuffers(dm, train=True)
    x = torch.empty(0, 128, dtype=torch.bfloat16, device="cuda")
    wg = torch.ones(8, 128, device="cuda")
    bias = torch.zeros(8, device="cuda")
    w1 = torch.ones(9, 128, 128, dtype=torch.bfloat16, device="cuda")
    w2 = torch.ones(9, 128, 64, dtype=torch.bfloat16, device="cuda")
    out = layer.forward(b, x, wg, bias, w1, w2)
    layer.backward(b, x, x, w1, w2, wg=wg, gamma=1e-3, bias=bias)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    assert out.shape == (0, 128)
    assert torch.all(b.counts == 0)
    assert torch.all(b.dw1 == 0) and torch.all(b.dw2 == 0) and torch.all(b.dwg == 0)
    assert torch.equal(b.bias_next, bias)  # load 0 == mean load 0: sign 0, no step


def test_all_experts_chosen_and_eight_shared():
    # k = E: every token uses every routed expert (w = p); S = 8 shared experts (G = 16)
    wl = synth.Workload("edge_kE_S8", synth.Dims(T=200, d=128, E=8, k=8, S=8, I=64, P=64),
                        seed=21, w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    inp = synth.make_inputs(wl)
    dm = dims_of(wl)
    b = layer.MoEBuffers(dm, train=True)
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
