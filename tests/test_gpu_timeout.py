"""Failure detection without a GPU fault: every wait inside the grouped GEMM and
the gate is bounded.  With a wait budget of 1 ns the kernel's roles give up, record
MOE_ERR_DEVICE_TIMEOUT in the workspace status word, drain the copies and MMAs
they already started and return (each pair still draws up to its ticket past the last
tile, so the launch's tile counter goes back to 0); the host reads the status and the
CUDA context stays usable.  Runs in a child process because the budget
(MOE_WAIT_BUDGET_NS) is read once per process."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys
sys.path.insert(0, ROOT)
import numpy as np
import torch
import grouped_gemm_fp32_b200 as moe
import synth
E, rows, d, I = 4, 512, 1024, 512
dm = moe.MoeDims.of(E * rows, d, E, 1, 0, I, 128, E * rows)
ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
counts = torch.full((E,), rows, dtype=torch.int32, device="cuda")
offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
moe.grouped_gemm_set_groups(dm, counts, offsets, ws)
bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).cuda()
x = bf(synth.normal_bf16(1, 1, (E * rows, d), 1.0))
w1 = bf(synth.normal_bf16(1, 4, (E, 2 * I, d), 0.03))
w2 = bf(synth.normal_bf16(1, 5, (E, d, I), 0.03))
h = torch.empty(E * rows, I, dtype=torch.bfloat16, device="cuda")
y = torch.empty(E * rows, d, dtype=torch.bfloat16, device="cuda")
moe.grouped_gemm_fwd(dm, ws, x, None, w1, w2, h, None, y)
torch.cuda.synchronize()
st = moe.moe_get_device_status(ws)
print("gemm status", st)
# the launch's tile counter is back at 0 although every role gave up early
print("tile counters", ws[20:44].view(torch.int32).tolist())
# the context still works: the status was cleared and a plain op runs
assert moe.moe_get_device_status(ws) == 0
# the gate's waits are bounded the same way
dg = moe.MoeDims.of(1024, 4096, 128, 6, 0, 64, 128)
wsg = torch.zeros(moe.moe_workspace_size(dg), dtype=torch.uint8, device="cuda")
xg = bf(synth.normal_bf16(2, 1, (1024, 4096), 1.0))
wg = torch.from_numpy(synth.normal_f32(2, 2, (128, 4096), 0.02)).cuda()
idx = torch.empty(1024, 6, dtype=torch.int32, device="cuda")
wt = torch.empty(1024, 6, dtype=torch.float32, device="cuda")
moe.moe_gate_topk(dg, xg, wg, None, idx, wt, None, wsg)
torch.cuda.synchronize()
print("gate status", moe.moe_get_device_status(wsg))
z = torch.arange(1000, device="cuda", dtype=torch.float32).sum().item()
print("context ok", z == 499500.0)
'''


@pytest.mark.gpu
def test_bounded_waits_report_timeout_and_keep_context():
    env = dict(os.environ, MOE_WAIT_BUDGET_NS="1")
    p = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD], env=env,
                       capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stdout + p.stderr
    assert "gemm status -4" in p.stdout, p.stdout
    assert "tile counters [0, 0, 0, 0, 0, 0]" in p.stdout, p.stdout
    assert "gate status -4" in p.stdout, p.stdout
    assert "context ok True" in p.stdout, p.stdout


CHILD_EP = r'''
import sys
sys.path.insert(0, ROOT)
import torch
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import ep
import synth
# one rank whose exchange partners never deliver: the owner's GEMM waits for rows that
# no dispatch sends, the source waits for Y rows that no owner returns
dims = moe.MoeDims.of(256, 128, 8, 2, 1, 64, 64)
eb = ep.EPBuffers(dims, 0, 1, train=False)
ep.connect(eb)
eb.counts_all.fill_(64)          # as if every expert had 64 tokens
ep.plan(eb)
bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).cuda()
x = bf(synth.normal_bf16(3, 1, (256, 128), 1.0))
w1 = bf(synth.normal_bf16(3, 4, (9, 128, 128), 0.05))
w2 = bf(synth.normal_bf16(3, 5, (9, 128, 64), 0.05))
ep.experts_forward(eb, x, w1, w2)          # no dispatch ran: its first routed tile waits
torch.cuda.synchronize()
print("gemm status", moe.moe_get_device_status(eb.loc.ws))
# the owner above returned (garbage) rows, so raise the step count once more and wait
# for an owner that never comes
ep.plan(eb)
moe.moe_ep_wait(eb.peers["ws"], moe.MOE_EP_WAIT_Y)
torch.cuda.synchronize()
print("wait status", moe.moe_get_device_status(eb.ep_ws))
z = torch.arange(1000, device="cuda", dtype=torch.float32).sum().item()
print("context ok", z == 499500.0)
'''


@pytest.mark.gpu
def test_expert_parallel_waits_report_timeout_and_keep_context():
    """Bounded waits of the expert-parallel exchange: rows that never arrive give
    MOE_ERR_DEVICE_TIMEOUT (in the GEMM's workspace, and in the EP workspace for the
    source's wait) within a 20 ms budget, and the context stays usable."""
    env = dict(os.environ, MOE_WAIT_BUDGET_NS="20000000")
    p = subprocess.run([sys.executable, "-c", f"ROOT = {ROOT!r}\n" + CHILD_EP], env=env,
                       capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stdout + p.stderr
    assert "gemm status -4" in p.stdout, p.stdout
    assert "wait status -4" in p.stdout, p.stdout
    assert "context ok True" in p.stdout, p.stdout
