"""The data-parallel exchange steps (layer.dp_bias_step, layer.dp_allreduce_grads)
on one GPU over NCCL, in a process group of one rank: the all-reduces run through
NCCL on the layer's stream, and with one rank the results must equal the
single-GPU ones bit for bit.  The bias step is checked against the oracle's step
on the GPU's own routing as well.  The sums over several ranks are covered on CPU
(tests/test_dist_cpu.py, gloo); nothing here runs on more than one GPU.

Passage: dots.llm1 Technical Report, §Architecture "Load balancing" (the bias
follows the experts' loads, here the loads of the whole data-parallel batch).
"""
import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import synth
from common import dims_of, host
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu

SMALL = synth.Workload("dp_small", synth.Dims(T=300, d=128, E=8, k=2, S=1, I=64, P=64),
                       seed=13, w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)


@pytest.fixture
def nccl_one_rank():
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        yield
    finally:
        dist.destroy_process_group()


def test_dp_steps_on_one_rank_match_the_single_gpu_step(nccl_one_rank):
    inp = synth.make_inputs(SMALL)
    dm = dims_of(SMALL)
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).cuda()
    x, w1, w2, dout = bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]), bf(inp["dout"])
    wg, bias = torch.from_numpy(inp["wg"]).cuda(), torch.from_numpy(inp["bias"]).cuda()
    s = torch.cuda.Stream()
    b = layer.MoEBuffers(dm, train=True)
    gamma = 1e-3
    with torch.cuda.stream(s):
        layer.forward(b, x, wg, bias, w1, w2, stream=s)
        layer.backward(b, x, dout, w1, w2, stream=s, wg=wg, gamma=gamma, bias=bias)
    s.synchronize()
    plain = b.bias_next.clone()
    counts = b.counts.clone()
    grads = [b.dw1.clone(), b.dw2.clone(), b.dwg.clone()]
    b.bias_next.fill_(7.0)
    with torch.cuda.stream(s):
        total = layer.dp_bias_step(b, gamma, bias, stream=s)
        layer.dp_allreduce_grads([b.dw1, b.dw2, b.dwg], stream=s)
    s.synchronize()
    assert torch.equal(total, counts) and torch.equal(b.counts, counts)
    assert torch.equal(b.bias_next, plain)
    ref = oracle.bias_update(host(b.topk_idx), dm.E, inp["bias"], float(np.float32(gamma)))
    assert np.array_equal(host(b.bias_next).astype(np.float64),
                          ref.astype(np.float32).astype(np.float64))
    for got, want in zip((b.dw1, b.dw2, b.dwg), grads):
        assert torch.equal(got, want)
