"""The grouped GEMM's run-time tile scheduler: the CTA pairs draw their tiles from a
counter in the workspace header (one word per GEMM mode, words 5..10), and the pair
that draws the launch's last ticket puts it back to 0.  So the same GEMM launched
again and again without a new routing call gives the same result bit for bit, every
mode leaves its counter at 0, and a launch whose waits ran out (tests/
test_gpu_timeout.py) leaves it at 0 as well.

Passage: dots.llm1 Technical Report, §3.2 "Efficient implementation of Grouped
GEMM" (tiles of aligned expert segments are scheduled like those of a plain GEMM;
the order in which CTAs take them does not change any tile's arithmetic).
"""
import pytest
import torch

import synth
from common import dev, dims_of
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu


def _counters(ws):
    return ws[20:44].view(torch.int32).tolist()


@pytest.mark.parametrize("wl_name", ["train_small"])
def test_repeated_launches_are_bit_identical_and_reset_the_counters(wl_name):
    wl = synth.WORKLOADS[wl_name]
    inp = synth.make_inputs(wl)
    dm = dims_of(wl)
    b = layer.MoEBuffers(dm, train=True)
    x, w1, w2 = dev(inp["x"], True), dev(inp["w1"], True), dev(inp["w2"], True)
    dout = dev(inp["dout"], True)
    layer.forward(b, x, dev(inp["wg"]), dev(inp["bias"]), w1, w2)
    layer.backward(b, x, dout, w1, w2)
    torch.cuda.synchronize()
    assert _counters(b.ws) == [0] * 6

    calls = {
        "fwd": (lambda: moe.grouped_gemm_fwd(dm, b.ws, b.x_perm, x, w1, w2, b.h, b.a1, b.y),
                (b.h, b.a1, b.y)),
        "dx2": (lambda: moe.grouped_gemm_bwd_dx(dm, b.ws, moe.MOE_GEMM2, b.dy, dout, w2, b.a1,
                                                b.da), (b.da,)),
        "dw2": (lambda: moe.grouped_gemm_bwd_dw(dm, b.ws, moe.MOE_GEMM2, b.dy, dout, b.h, None,
                                                b.dw2, 0), (b.dw2,)),
        "dx1": (lambda: moe.grouped_gemm_bwd_dx(dm, b.ws, moe.MOE_GEMM1, b.da, None, w1, None,
                                                b.dxp), (b.dxp,)),
        "dw1": (lambda: moe.grouped_gemm_bwd_dw(dm, b.ws, moe.MOE_GEMM1, b.da, None, b.x_perm,
                                                x, b.dw1, 0), (b.dw1,)),
    }
    for name, (call, outs) in calls.items():
        # outputs zeroed before every launch (rows past the last group's padded end are
        # never written), so a tile a launch skipped would show as zeros
        for o in outs:
            o.zero_()
        call()
        torch.cuda.synchronize()
        ref = [o.clone() for o in outs]
        for rep in range(3):
            for o in outs:
                o.zero_()
            call()
            torch.cuda.synchronize()
            assert moe.moe_get_device_status(b.ws) == 0, name
            for o, r in zip(outs, ref):
                assert torch.equal(o, r), (name, rep)
            assert _counters(b.ws) == [0] * 6, (name, _counters(b.ws))
