"""A layer step captured as a CUDA graph and replayed gives bit-identical results
to the same C-ABI calls run eagerly (forward, backward, router backward, bias
step), on the small training case and on the full train workload."""
import pytest
import torch

import synth
from common import dev, dims_of, workload_inputs
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu

SMALL = synth.Workload("small_train", synth.Dims(T=300, d=128, E=8, k=2, S=1, I=64, P=64),
                       seed=11, w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)

KEYS = ("out", "topk_idx", "topk_w", "dx", "dw1", "dw2", "dwg", "bias_next")


@pytest.mark.parametrize("case", ["small", "train"])
def test_graph_replay_matches_eager(case):
    if case == "small":
        wl, inp = SMALL, synth.make_inputs(SMALL)
    else:
        wl, inp = synth.WORKLOADS["train"], workload_inputs("train")
    dm = dims_of(wl)
    x, w1, w2 = dev(inp["x"], True), dev(inp["w1"], True), dev(inp["w2"], True)
    wg, bias, dout = dev(inp["wg"]), dev(inp["bias"]), dev(inp["dout"], True)
    eager = layer.MoEBuffers(dm, train=True)
    layer.forward(eager, x, wg, bias, w1, w2)
    layer.backward(eager, x, dout, w1, w2, wg=wg, gamma=1e-3, bias=bias)
    torch.cuda.synchronize()
    ref = {k: getattr(eager, k).clone() for k in KEYS}
    del eager
    b = layer.MoEBuffers(dm, train=True)
    g = layer.GraphStep(b, x, wg, bias, w1, w2, dout=dout, gamma=1e-3)
    for _ in range(2):  # replays after the capture step rewrite every output
        for k in KEYS:
            getattr(b, k).zero_()
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(b.ws) == 0
        for k in KEYS:
            assert torch.equal(getattr(b, k), ref[k]), k
