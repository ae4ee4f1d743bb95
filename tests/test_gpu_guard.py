"""Out-of-bounds writes, caught without a sanitizer: every buffer the layer writes
(activations, gradients, routing tables, the workspace) sits between two 4 KB
guard bands of a known byte pattern, and a whole step must leave every band
untouched.  Shapes are chosen to make edges likely: ragged T, small pad blocks,
partial N tiles, an empty expert."""
import numpy as np
import pytest
import torch

import synth
from common import dev, dims_of
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side
PATTERN = 0xA5


class Guarded:
    """Tensors carved out of larger byte buffers with guard bands around them."""

    def __init__(self):
        self.bases = []

    def wrap(self, t: torch.Tensor) -> torch.Tensor:
        nbytes = t.numel() * t.element_size()
        base = torch.full((GUARD + nbytes + 256 + GUARD,), PATTERN, dtype=torch.uint8,
                          device=t.device)
        body = base[GUARD:GUARD + nbytes].view(t.dtype).view(t.shape)
        body.copy_(t)
        self.bases.append((base, nbytes))
        return body

    def intact(self) -> bool:
        for base, nbytes in self.bases:
            head = base[:GUARD]
            tail = base[GUARD + nbytes:]
            if not (torch.all(head == PATTERN) and torch.all(tail == PATTERN)):
                return False
        return True


def _guard_buffers(b: layer.MoEBuffers, g: Guarded):
    for name, v in list(vars(b).items()):
        if isinstance(v, torch.Tensor):
            setattr(b, name, g.wrap(v))


@pytest.mark.parametrize("T,d,E,k,S,I,P,train", [
    (301, 192, 8, 2, 1, 64, 64, True),      # ragged T, d with a partial 256-wide N tile
    (77, 128, 16, 4, 2, 128, 16, False),    # pad block 16 < the 128-row MMA tile
    (1000, 256, 32, 6, 1, 192, 64, True),   # I = 192: a narrow last N tile in the dX/dW GEMMs
])
@pytest.mark.parametrize("gather", [False, True])
def test_no_write_outside_any_buffer(T, d, E, k, S, I, P, train, gather):
    wl = synth.Workload("guard", synth.Dims(T=T, d=d, E=E, k=k, S=S, I=I, P=P), seed=T + E,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=train)
    inp = synth.make_inputs(wl)
    bias = inp["bias"].copy()
    bias[1] = -1.0  # expert 1 empty
    dm = dims_of(wl)
    g = Guarded()
    b = layer.MoEBuffers(dm, train=train, gather=gather)
    _guard_buffers(b, g)
    x = g.wrap(dev(inp["x"], True))
    w1, w2 = g.wrap(dev(inp["w1"], True)), g.wrap(dev(inp["w2"], True))
    wg, bias_t = g.wrap(dev(inp["wg"])), g.wrap(dev(bias))
    # train steps include the sequence-wise balance loss (sequences of 128 tokens)
    layer.forward(b, x, wg, bias_t, w1, w2, seq_balance=(1e-2, 128) if train else None)
    if train:
        dout = g.wrap(dev(inp["dout"], True))
        layer.backward(b, x, dout, w1, w2, wg=wg, gamma=1e-3, bias=bias_t)
        assert b.bal_seq_len == 128
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    assert int(b.counts[1].item()) == 0
    assert g.intact(), "a guard band was overwritten"
    assert torch.all(torch.isfinite(b.out.float()))
