"""GPU parity of the layer backward (combine bwd, dX and dW grouped GEMMs,
SwiGLU backward, un-permute-sum) against the oracle's exact gradients.

The oracle's gradients are pinned by finite differences (test_oracle_bwd.py).
Bar: max|diff| <= 2e-2 * max|ref| per gradient tensor.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from common import (assert_close, dev, dims_of, host, oracle_routing, sample_tokens,
                    workload_inputs)
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu

SMALL = synth.Workload("small_train", synth.Dims(T=300, d=128, E=8, k=2, S=1, I=64, P=64),
                       seed=11, w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)


def _run(wl, inp, routing=None):
    """Forward + backward through the C ABI.  ``routing`` = the oracle's (idx, w):
    the experts then see exactly the oracle's token sets (the gate has its own
    parity test), so near-tie tokens cannot shift a group's dW."""
    dm = dims_of(wl)
    b = layer.MoEBuffers(dm, train=True)
    x = dev(inp["x"], True)
    w1, w2 = dev(inp["w1"], True), dev(inp["w2"], True)
    rt = None if routing is None else (dev(routing[0]), dev(routing[1].astype(np.float32)))
    layer.forward(b, x, dev(inp["wg"]), dev(inp["bias"]), w1, w2, routing=rt)
    dx, dw1, dw2, dwc = layer.backward(b, x, dev(inp["dout"], True), w1, w2)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    return b, dx, dw1, dw2, dwc


SMALL_2048 = synth.Workload("small_train_2048", synth.Dims(T=200, d=2048, E=8, k=2, S=1, I=64,
                                                         P=64),
                            seed=12, w1_std=0.02, w2_std=0.05, wg_std=0.02, backward=True)


@pytest.mark.parametrize("wl", [SMALL, SMALL_2048], ids=["d128", "d2048"])
def test_backward_small_full(wl):
    inp = synth.make_inputs(wl)
    S = wl.dims.S
    p, oidx, ow, margin = oracle.route(oracle.gate_logits(inp["x"], inp["wg"]), inp["bias"],
                                       wl.dims.k)
    b, dx, dw1, dw2, dwc = _run(wl, inp, routing=(oidx, ow))
    rdx, rdw = oracle.layer_bwd(inp["x"], oidx, ow, inp["w1"], inp["w2"], inp["dout"], S)
    assert_close(host(dx), rdx, "dx")
    assert_close(host(dwc), rdw, "d(combine weight)")
    DW1, DW2 = host(dw1), host(dw2)
    for g in range(wl.dims.G):
        r1, r2 = oracle.group_dw(inp["x"], oidx, ow, inp["w1"], inp["w2"], inp["dout"], S, g)
        if np.max(np.abs(r1)) == 0:
            assert np.all(DW1[g] == 0) and np.all(DW2[g] == 0)
            continue
        assert_close(DW1[g], r1, f"dW1[{g}]")
        assert_close(DW2[g], r2, f"dW2[{g}]")


def test_backward_empty_expert_gets_zero_dW():
    wl = SMALL
    inp = synth.make_inputs(wl)
    bias = np.zeros(wl.dims.E, np.float32)
    bias[3] = -1.0  # expert 3 never selected
    inp["bias"] = bias
    b, dx, dw1, dw2, dwc = _run(wl, inp)
    assert int(host(b.counts)[3]) == 0
    assert torch.all(dw1[3] == 0) and torch.all(dw2[3] == 0)


def test_dw_accumulate_adds():
    wl = SMALL
    inp = synth.make_inputs(wl)
    b, dx, dw1, dw2, dwc = _run(wl, inp)
    first = dw2.clone()
    moe.grouped_gemm_bwd_dw(b.dims, b.ws, moe.MOE_GEMM2, b.dy, dev(inp["dout"], True), b.h, None,
                            dw2, 1)
    torch.cuda.synchronize()
    assert torch.allclose(dw2, 2 * first, rtol=1e-6, atol=1e-6)


def test_backward_train_sampled():
    """Full-size training workload (T=16384, d=4096, 128 routed top-6 + 2 shared,
    I=1408), the configuration the benchmark times; sampled outputs."""
    name = "train"
    wl = synth.WORKLOADS[name]
    inp = workload_inputs(name)
    S, E, I = wl.dims.S, wl.dims.E, wl.dims.I
    p, oidx, ow, margin = oracle_routing(name)
    b, dx, dw1, dw2, dwc = _run(wl, inp, routing=(oidx, ow))
    # 512 tokens, among them the hottest and the least-loaded experts' tokens (each
    # token's out, dX and combine-weight gradient depend on that token alone)
    tokens = sample_tokens(oidx, np.arange(wl.dims.T), 512, 4)
    ref_out = oracle.layer_fwd(inp["x"], oidx, ow, inp["w1"], inp["w2"], S, tokens=tokens)
    assert_close(host(b.out)[tokens], ref_out, "out")
    rdx, rdw = oracle.layer_bwd(inp["x"], oidx, ow, inp["w1"], inp["w2"], inp["dout"], S,
                                tokens=tokens)
    assert_close(host(dx)[tokens], rdx, "dx")
    assert_close(host(dwc)[tokens], rdw, "d(combine weight)")
    # the whole dW1 and dW2 of four routed experts (most-loaded, least-loaded
    # non-empty, two random), each summing over every token of the expert
    rng = np.random.default_rng(4)
    counts = np.bincount(oidx.ravel(), minlength=E)
    nonempty = np.nonzero(counts)[0]
    groups = [int(counts.argmax()), int(nonempty[counts[nonempty].argmin()]),
              *map(int, rng.choice(E, 2, replace=False))]
    for g in groups:
        r1, r2 = oracle.group_dw(inp["x"], oidx, ow, inp["w1"], inp["w2"], inp["dout"], S, g)
        assert_close(dw1[g].cpu().numpy(), r1, f"dW1[{g}]")
        assert_close(dw2[g].cpu().numpy(), r2, f"dW2[{g}]")
    # shared expert 0 sums over all 16384 tokens (its whole dW is about 1 TFLOP of FP64
    # work in the oracle): every 8th row of dW1 and column of dW2, plus the edges of
    # the gate / up halves and of the 128-column tiles
    rows1 = np.unique(np.concatenate([np.arange(0, 2 * I, 8), [1, I - 1, I, 2 * I - 1]])
                      ).astype(np.int32)
    cols2 = np.unique(np.concatenate([np.arange(0, I, 8), [127, 128, I - 1]])).astype(np.int32)
    r1, r2 = oracle.group_dw(inp["x"], oidx, ow, inp["w1"], inp["w2"], inp["dout"], S, E,
                             w1_rows=rows1, w2_cols=cols2)
    assert_close(dw1[E][torch.from_numpy(rows1).long().cuda()].cpu().numpy(), r1, f"dW1[{E}]")
    assert_close(dw2[E][:, torch.from_numpy(cols2).long().cuda()].cpu().numpy(), r2,
                 f"dW2[{E}]")
