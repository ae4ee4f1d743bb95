"""GPU parity of the router backward (moe_router_bwd) and the bias step
(moe_bias_update) against the oracle (its own pins: test_oracle_router_bwd.py).

Passages: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
(FP32 gate; the combine weights are the chosen experts' affinities) and "Load
balancing" (bias for selection only, adjusted during training).

Bars: dlogits and dWg are FP32 results: max|diff| <= 1e-4 * max|ref|.  The gate
term of dX lands in a bf16 tensor: the spec bar, 2e-2 * max|ref| (and
1e-2 when dX starts at zero, where only one bf16 rounding is involved).  The
bias step is one correctly rounded FP32 addition: bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from common import REL_TOL, assert_close, dev, dims_of, host, workload_inputs
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu

FP32_TOL = 1e-4


def _router_case(T, d, E, k, seed):
    """Inputs with the oracle's routing: x, wg, probs (f32), idx, w (f32), dw (f32)."""
    x = synth.normal_bf16(seed, 1, (T, d), 1.0)
    wg = synth.normal_f32(seed, 2, (E, d), 0.05)
    p, idx, w, _ = oracle.route(oracle.gate_logits(x, wg), np.zeros(E, np.float32), k)
    dw = synth.normal_f32(seed, 6, (T, k), 1.0)
    return x, wg, p.astype(np.float32), idx, w.astype(np.float32), dw


def _gpu_router(T, d, E, k, x, wg, probs, idx, w, dw, accumulate=0, dwg0=None):
    dm = moe.MoeDims.of(T, d, E, k, 0, 64, 64)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    dl = torch.full((T, E), 7.0, dtype=torch.float32, device="cuda")
    dx = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    dwg = (torch.full((E, d), 5.0, dtype=torch.float32, device="cuda") if dwg0 is None
           else dev(dwg0))
    moe.moe_router_bwd(dm, dev(x, True), dev(wg), dev(probs), dev(idx), dev(w), dev(dw), dl, dx,
                       dwg, accumulate, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    return host(dl), host(dx), host(dwg)


@pytest.mark.parametrize("T,d,E,k", [(300, 128, 8, 2),      # ragged T, E < 32
                                     (1000, 192, 96, 6),    # E_pad = 96: a half-empty K block;
                                                            # d = 192: a partial N tile
                                     (129, 256, 256, 8),    # E = 256: two M tiles of dWg
                                     (5000, 512, 128, 6)])
def test_router_bwd_matches_oracle(T, d, E, k):
    x, wg, probs, idx, w, dw = _router_case(T, d, E, k, seed=T + E)
    dl, dx, dwg = _gpu_router(T, d, E, k, x, wg, probs, idx, w, dw)
    rdl, rdx, rdwg = oracle.router_bwd(x, wg, idx, dw.astype(np.float64))
    assert_close(dl, rdl, "dlogits", FP32_TOL)
    assert_close(dx, rdx, "gate dX", 1e-2)
    assert_close(dwg, rdwg, "dWg", FP32_TOL)
    np.testing.assert_allclose(dl.sum(axis=1), 0.0, atol=1e-6 * np.abs(rdl).max())


def test_router_bwd_accumulates_dwg():
    T, d, E, k = 300, 128, 8, 2
    x, wg, probs, idx, w, dw = _router_case(T, d, E, k, seed=3)
    base = synth.normal_f32(4, 9, (E, d), 1.0)
    _, _, dwg = _gpu_router(T, d, E, k, x, wg, probs, idx, w, dw, accumulate=1, dwg0=base)
    _, _, rdwg = oracle.router_bwd(x, wg, idx, dw.astype(np.float64))
    assert_close(dwg - base, rdwg, "accumulated dWg", 1e-3)


def test_router_bwd_no_tokens():
    dm = moe.MoeDims.of(0, 128, 8, 2, 0, 64, 64)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    wg = torch.ones(8, 128, device="cuda")
    dwg = torch.full((8, 128), 3.0, device="cuda")
    moe.moe_router_bwd(dm, None, wg, None, None, None, None, None, None, dwg, 0, ws)
    torch.cuda.synchronize()
    assert torch.all(dwg == 0)


def test_layer_backward_with_router_matches_oracle():
    # forward + backward through the layer with the oracle's routing injected; dX is
    # the expert path plus the router's term
    wl = synth.Workload("small_train", synth.Dims(T=300, d=128, E=8, k=2, S=1, I=64, P=64),
                        seed=11, w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    inp = synth.make_inputs(wl)
    dm = dims_of(wl)
    p, oidx, ow, _ = oracle.route(oracle.gate_logits(inp["x"], inp["wg"]), inp["bias"], 2)
    b = layer.MoEBuffers(dm, train=True)
    x, w1, w2 = dev(inp["x"], True), dev(inp["w1"], True), dev(inp["w2"], True)
    wg = dev(inp["wg"])
    layer.forward(b, x, wg, dev(inp["bias"]), w1, w2,
                  routing=(dev(oidx), dev(ow.astype(np.float32)), dev(p.astype(np.float32))))
    layer.backward(b, x, dev(inp["dout"], True), w1, w2, wg=wg)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    rdx, rdw = oracle.layer_bwd(inp["x"], oidx, ow, inp["w1"], inp["w2"], inp["dout"], 1)
    _, gdx, gdwg = oracle.router_bwd(inp["x"], inp["wg"], oidx, rdw)
    assert_close(host(b.dx), rdx + gdx, "dx (experts + router)")
    assert_close(host(b.dwg), gdwg, "dWg", REL_TOL)


def test_router_bwd_train_workload_sampled():
    """Full train shapes (T=16384, d=4096, E=128, k=6), the launch configuration the
    benchmark times: the GPU's own gate, combine backward and router backward; the
    oracle's dlogits for every token, dX and dWg entries sampled against them."""
    name = "train"
    wl = synth.WORKLOADS[name]
    inp = workload_inputs(name)
    dm = dims_of(wl)
    b = layer.MoEBuffers(dm, train=True)
    x, w1, w2 = dev(inp["x"], True), dev(inp["w1"], True), dev(inp["w2"], True)
    wg, bias = dev(inp["wg"]), dev(inp["bias"])
    layer.forward(b, x, wg, bias, w1, w2)
    dout = dev(inp["dout"], True)
    layer.backward(b, x, dout, w1, w2)
    torch.cuda.synchronize()
    dx_experts = b.dx.clone()
    dl = torch.empty(dm.T, dm.E, dtype=torch.float32, device="cuda")
    moe.moe_router_bwd(dm, x, wg, b.probs, b.topk_idx, b.topk_w, b.dw_comb, dl, b.dx, b.dwg, 0,
                       b.ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    idx, dwc = host(b.topk_idx), host(b.dw_comb).astype(np.float64)
    rdl, _, _ = oracle.router_bwd(inp["x"], inp["wg"], idx, dwc, want_dx=False, want_dwg=False)
    rdl_max = np.abs(rdl).max()
    assert np.max(np.abs(host(dl) - rdl)) <= FP32_TOL * rdl_max
    rng = np.random.default_rng(0)
    xs = synth.bf16_to_f32(inp["x"]).astype(np.float64)
    # dX: 64 sampled tokens, all columns (gate term = dX after - dX before, each bf16)
    ts = rng.choice(dm.T, 64, replace=False)
    ref = rdl[ts] @ inp["wg"].astype(np.float64)
    got = host(b.dx)[ts] - host(dx_experts)[ts]
    scale = np.abs(host(dx_experts)[ts]).max() + np.abs(ref).max()
    assert np.max(np.abs(got - ref)) <= REL_TOL * scale
    # dWg: 8 experts x 64 columns, summed over all tokens
    es, cs = rng.choice(dm.E, 8, replace=False), rng.choice(dm.d, 64, replace=False)
    ref = rdl[:, es].T @ xs[:, cs]
    got = host(b.dwg)[np.ix_(es, cs)]
    assert np.max(np.abs(got - ref)) <= FP32_TOL * np.abs(ref).max()


def test_bias_update_is_exact():
    name = "train"
    inp = workload_inputs(name, with_weights=False)
    wl = synth.WORKLOADS[name]
    dm = dims_of(wl)
    _, idx, _, _ = oracle.route(oracle.gate_logits(inp["x"][:4096], inp["wg"]), inp["bias"], dm.k)
    counts = np.bincount(idx.ravel(), minlength=dm.E).astype(np.int32)
    dm4 = moe.MoeDims.of(4096, dm.d, dm.E, dm.k, dm.S, dm.I, dm.P)
    ref = oracle.bias_update(idx, dm.E, inp["bias"], 1e-3).astype(np.float32)
    bias = dev(inp["bias"])
    out = torch.empty_like(bias)
    moe.moe_bias_update(dm4, dev(counts), 1e-3, bias, out)
    inplace = bias.clone()
    moe.moe_bias_update(dm4, dev(counts), 1e-3, inplace, inplace)
    torch.cuda.synchronize()
    assert np.array_equal(host(out), ref)
    assert np.array_equal(host(inplace), ref)
    assert torch.equal(bias, dev(inp["bias"]))  # input untouched when out differs
