"""GPU parity of the sequence-wise balance loss (moe_seq_balance_loss) and of the
router backward that carries its gradient (moe_router_bwd_seqbal), against the
oracle (its own pins: test_oracle_seqbal.py).

Passage: dots.llm1 Technical Report, §Architecture "Load balancing" (a
sequence-wise balance loss besides the aux-loss-free bias; formula read from
the report the pages cite for their method).

Bars: FP32 results, max|diff| <= 1e-4 * max|ref| (loss: relative 1e-5); the
gate term of dX is bf16: 1e-2 * max|ref| when dX starts at zero.  The balance
gradient (alpha f / (n_seq L_s)) is far smaller than the combine-weight term,
so each case checks it alone (dL/dw = 0) and then the sum with alpha scaled to
make both terms of one size.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from common import assert_close, dev, dims_of, host, workload_inputs
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu

FP32_TOL = 1e-4


def _case(T, d, E, k, seed):
    x = synth.normal_bf16(seed, 1, (T, d), 1.0)
    wg = synth.normal_f32(seed, 2, (E, d), 0.05)
    logits = oracle.gate_logits(x, wg)
    p, idx, w, _ = oracle.route(logits, np.zeros(E, np.float32), k)
    return x, wg, logits, p.astype(np.float32), idx, w.astype(np.float32)


def _gpu(T, d, E, k, L, alpha, x, wg, probs, idx, w, dw):
    dm = moe.MoeDims.of(T, d, E, k, 0, 64, 64)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    loss = torch.full((1,), 7.0, dtype=torch.float32, device="cuda")
    g = torch.full((max(1, -(-T // L)), E), 7.0, dtype=torch.float32, device="cuda")
    pr, ix = dev(probs), dev(idx)
    moe.moe_seq_balance_loss(dm, L, alpha, ix, pr, loss, g, ws)
    dl = torch.empty(T, E, dtype=torch.float32, device="cuda")
    dx = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    dwg = torch.empty(E, d, dtype=torch.float32, device="cuda")
    moe.moe_router_bwd_seqbal(dm, dev(x, True), dev(wg), pr, ix, dev(w), dev(dw), g, L, dl, dx,
                              dwg, 0, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    return float(loss.item()), host(dl), host(dx), host(dwg)


@pytest.mark.parametrize("T,d,E,k,L", [
    (300, 128, 8, 2, 128),     # three sequences, the last of 44 tokens
    (1000, 192, 96, 6, 256),   # E = 96, last sequence of 232 tokens
    (129, 256, 256, 8, 128),   # E = 256, a last sequence of one token
    (700, 128, 16, 4, 4096),   # one sequence shorter than seq_len
])
def test_seq_balance_and_its_router_gradient(T, d, E, k, L):
    x, wg, logits, probs, idx, w = _case(T, d, E, k, seed=T + E)
    alpha = 0.05
    # the balance term alone (dL/dw = 0)
    loss, dl, dx, dwg = _gpu(T, d, E, k, L, alpha, x, wg, probs, idx, w, np.zeros((T, k),
                                                                                 np.float32))
    rloss, rdl_bal = oracle.seq_balance(logits, idx, L, alpha)
    assert loss == pytest.approx(rloss, rel=1e-5)
    rdl, rdx, rdwg = oracle.router_bwd(x, wg, idx, np.zeros((T, k)), dl_extra=rdl_bal)
    assert_close(dl, rdl, "balance dlogits", FP32_TOL)
    assert_close(dx, rdx, "balance gate dX", 1e-2)
    assert_close(dwg, rdwg, "balance dWg", FP32_TOL)
    # both terms, of one size: alpha scaled so the balance term matches the other
    dw = synth.normal_f32(T + 1, 6, (T, k), 1.0)
    rdl0, _, _ = oracle.router_bwd(x, wg, idx, dw.astype(np.float64), want_dx=False,
                                   want_dwg=False)
    alpha2 = alpha * np.abs(rdl0).max() / np.abs(rdl_bal).max()
    _, rdl_bal2 = oracle.seq_balance(logits, idx, L, alpha2)
    loss, dl, dx, dwg = _gpu(T, d, E, k, L, alpha2, x, wg, probs, idx, w, dw)
    rdl, rdx, rdwg = oracle.router_bwd(x, wg, idx, dw.astype(np.float64), dl_extra=rdl_bal2)
    assert_close(dl, rdl, "dlogits (combine + balance)", FP32_TOL)
    assert_close(dx, rdx, "gate dX (combine + balance)", 1e-2)
    assert_close(dwg, rdwg, "dWg (combine + balance)", FP32_TOL)


def test_seq_balance_is_deterministic():
    T, d, E, k, L = 1000, 128, 32, 4, 128
    x, wg, logits, probs, idx, w = _case(T, d, E, k, seed=5)
    dw = synth.normal_f32(5, 6, (T, k), 1.0)
    a = _gpu(T, d, E, k, L, 0.3, x, wg, probs, idx, w, dw)
    b = _gpu(T, d, E, k, L, 0.3, x, wg, probs, idx, w, dw)
    assert a[0] == b[0]
    for u, v in zip(a[1:], b[1:]):
        assert np.array_equal(u, v)


def test_layer_step_with_seq_balance():
    # forward computes the loss, backward adds its gradient: dX and dWg differ from
    # the step without it by exactly the balance term (oracle), the rest is unchanged
    wl = synth.Workload("seqbal", synth.Dims(T=600, d=128, E=16, k=4, S=1, I=64, P=64), seed=31,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
    inp = synth.make_inputs(wl)
    dm = dims_of(wl)
    x, w1, w2 = dev(inp["x"], True), dev(inp["w1"], True), dev(inp["w2"], True)
    wg, bias, dout = dev(inp["wg"]), dev(inp["bias"]), dev(inp["dout"], True)
    runs = {}
    for sb in (None, (20.0, 256)):  # alpha large: the term is visible in dWg
        b = layer.MoEBuffers(dm, train=True)
        layer.forward(b, x, wg, bias, w1, w2, seq_balance=sb)
        layer.backward(b, x, dout, w1, w2, wg=wg)
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(b.ws) == 0
        runs[sb is not None] = b
    on, off = runs[True], runs[False]
    assert torch.equal(on.dw1, off.dw1) and torch.equal(on.dw2, off.dw2)
    idx = host(on.topk_idx)
    logits = oracle.gate_logits(inp["x"], inp["wg"])
    rloss, rdl = oracle.seq_balance(logits, idx, 256, 20.0)
    assert float(on.bal_loss.item()) == pytest.approx(rloss, rel=1e-5)
    _, rdx, rdwg = oracle.router_bwd(inp["x"], inp["wg"], idx, np.zeros((600, 4)), dl_extra=rdl)
    # dX carries bf16 rounding of both runs: compare the difference against the term
    # with the bf16 bar on dX's own scale
    diff = host(on.dx) - host(off.dx)
    scale = np.abs(host(off.dx)).max()
    assert np.max(np.abs(diff - rdx)) <= 2e-2 * scale
    assert_close(host(on.dwg) - host(off.dwg), rdwg, "dWg balance term", 1e-3)


def test_seq_balance_train_workload():
    """Full train shapes (T=16384, E=128, k=6; sequences of 8192 tokens as in the
    pages' pre-training): the GPU gate's own routing, the loss and every dlogit
    of the balance term against the oracle; dX and dWg entries sampled."""
    name = "train"
    wl = synth.WORKLOADS[name]
    inp = workload_inputs(name, with_weights=False)
    dm = dims_of(wl)
    T, d, E, k, L = dm.T, dm.d, dm.E, dm.k, 8192
    x, wg = dev(inp["x"], True), dev(inp["wg"])
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    probs = torch.empty(T, E, dtype=torch.float32, device="cuda")
    moe.moe_gate_topk(dm, x, wg, dev(inp["bias"]), idx, w, probs, ws)
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    g = torch.empty(2, E, dtype=torch.float32, device="cuda")
    alpha = 1e-4
    moe.moe_seq_balance_loss(dm, L, alpha, idx, probs, loss, g, ws)
    dl = torch.empty(T, E, dtype=torch.float32, device="cuda")
    dx = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    dwg = torch.empty(E, d, dtype=torch.float32, device="cuda")
    moe.moe_router_bwd_seqbal(dm, x, wg, probs, idx, w, torch.zeros(T, k, device="cuda"), g, L,
                              dl, dx, dwg, 0, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    hidx = host(idx)
    logits = oracle.gate_logits(inp["x"], inp["wg"])
    rloss, rdl = oracle.seq_balance(logits, hidx, L, alpha)
    assert float(loss.item()) == pytest.approx(rloss, rel=1e-5)
    assert_close(host(dl), rdl, "balance dlogits", FP32_TOL)
    rng = np.random.default_rng(0)
    ts = rng.choice(T, 64, replace=False)
    assert_close(host(dx)[ts], rdl[ts] @ inp["wg"].astype(np.float64), "balance gate dX", 1e-2)
    es, cs = rng.choice(E, 8, replace=False), rng.choice(d, 64, replace=False)
    xs = synth.bf16_to_f32(inp["x"]).astype(np.float64)
    ref = rdl[:, es].T @ xs[:, cs]
    assert_close(host(dwg)[np.ix_(es, cs)], ref, "balance dWg", FP32_TOL)
