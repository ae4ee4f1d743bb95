"""The debug build (libmoe_debug.so, MOE_DEBUG=1): device-side checks of the group
table and tile coordinates that record MOE_ERR_BAD_ROUTING and skip the work instead of
following a bad entry, with no trap and no access outside any buffer.

* On the guard-band shapes (tests/test_gpu_guard.py: ragged T, small pad blocks, partial
  N tiles, an empty expert) the debug build reports status 0, leaves every guard band
  intact and gives the release build's results bit for bit: the checks change no
  arithmetic.
* A group table that the host corrupts after grouped_gemm_set_groups (a group's first
  row far past the end of the grouped row space) makes the grouped GEMMs and the pad-row
  zeroing of the combine backward report MOE_ERR_BAD_ROUTING; every guard band stays
  intact and the context stays usable.  (The release build trusts the table its own
  kernels write; this corruption is only ever run against the debug build.)

Each debug run is a child process: MOE_LIB_DEBUG is read when the library loads.
Passage: dots.llm1 Technical Report, §Architecture "Load balancing" (no token is
dropped: every routed row must land in its expert's segment).
"""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

SHAPES = [  # (T, d, E, k, S, I, P, train), the guard-band test's shapes
    (301, 192, 8, 2, 1, 64, 64, True),
    (77, 128, 16, 4, 2, 128, 16, False),
    (1000, 256, 32, 6, 1, 192, 64, True),
]

STEP = r'''
import sys
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import numpy as np
import torch
import synth
from common import dev, dims_of
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer, _lib
from test_gpu_guard import Guarded, _guard_buffers
print("library", _lib.lib_path().rsplit("/", 1)[-1])
res = {}
for i, (T, d, E, k, S, I, P, train) in enumerate(SHAPES):
    wl = synth.Workload("guard", synth.Dims(T=T, d=d, E=E, k=k, S=S, I=I, P=P), seed=T + E,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=train)
    inp = synth.make_inputs(wl)
    bias = inp["bias"].copy()
    bias[1] = -1.0
    dm = dims_of(wl)
    g = Guarded()
    b = layer.MoEBuffers(dm, train=train)
    _guard_buffers(b, g)
    x = g.wrap(dev(inp["x"], True))
    w1, w2 = g.wrap(dev(inp["w1"], True)), g.wrap(dev(inp["w2"], True))
    wg, bias_t = g.wrap(dev(inp["wg"])), g.wrap(dev(bias))
    layer.forward(b, x, wg, bias_t, w1, w2, seq_balance=(1e-2, 128) if train else None)
    outs = [b.out]
    if train:
        dout = g.wrap(dev(inp["dout"], True))
        layer.backward(b, x, dout, w1, w2, wg=wg, gamma=1e-3, bias=bias_t)
        outs += [b.dx, b.dw1, b.dw2, b.dwg]
    torch.cuda.synchronize()
    print("shape", i, "status", moe.moe_get_device_status(b.ws), "intact", g.intact())
    for j, t in enumerate(outs):
        res[f"{i}_{j}"] = t.view(torch.int16).cpu().numpy() if t.dtype == torch.bfloat16 \
            else t.cpu().numpy()
np.savez(OUT, **res)
'''

CORRUPT = r'''
import sys
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import numpy as np
import torch
import synth
from common import dev, dims_of
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer, _lib
from test_gpu_guard import Guarded, _guard_buffers
assert _lib.lib_path().endswith("libmoe_debug.so")
wl = synth.Workload("bad", synth.Dims(T=300, d=128, E=8, k=2, S=1, I=64, P=64), seed=5,
                    w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=True)
inp = synth.make_inputs(wl)
dm = dims_of(wl)
g = Guarded()
b = layer.MoEBuffers(dm, train=True)
_guard_buffers(b, g)
x = g.wrap(dev(inp["x"], True))
w1, w2 = g.wrap(dev(inp["w1"], True)), g.wrap(dev(inp["w2"], True))
dout = g.wrap(dev(inp["dout"], True))
layer.forward(b, x, g.wrap(dev(inp["wg"])), g.wrap(dev(inp["bias"])), w1, w2)
torch.cuda.synchronize()
print("clean status", moe.moe_get_device_status(b.ws))
# the group record of routed expert 3 (16 bytes at byte 64 + 16 * 3: a_row, out_row,
# rows, rows_pad) now starts a billion rows in
rec = b.ws[64:64 + 16 * 9].view(torch.int32).view(9, 4)
rec[3, 1] = 1_000_000_000
moe.grouped_gemm_fwd(dm, b.ws, b.x_perm, x, w1, w2, b.h, b.a1, b.y)
torch.cuda.synchronize()
print("fwd status", moe.moe_get_device_status(b.ws))
moe.moe_combine_bwd(dm, b.ws, dout, b.y, b.row_of, b.topk_w, b.dy, b.dw_comb)
torch.cuda.synchronize()
print("combine_bwd status", moe.moe_get_device_status(b.ws))
for which, lhs, rhs, out in ((moe.MOE_GEMM2, b.dy, b.h, b.dw2), (moe.MOE_GEMM1, b.da, b.x_perm, b.dw1)):
    moe.grouped_gemm_bwd_dw(dm, b.ws, which, lhs, dout if which == moe.MOE_GEMM2 else None, rhs,
                            x if which == moe.MOE_GEMM1 else None, out, 0)
    torch.cuda.synchronize()
    print("dw", which, "status", moe.moe_get_device_status(b.ws))
print("intact", g.intact())
z = torch.arange(1000, device="cuda", dtype=torch.float32).sum().item()
print("context ok", z == 499500.0)
'''


def _child(script, tmp_path, debug):
    out = str(tmp_path / ("debug.npz" if debug else "release.npz"))
    env = dict(os.environ, MOE_LIB_DEBUG="1" if debug else "0")
    head = f"ROOT = {ROOT!r}\nOUT = {out!r}\nSHAPES = {SHAPES!r}\n"
    p = subprocess.run([sys.executable, "-c", head + script], env=env, capture_output=True,
                       text=True, timeout=600)
    assert p.returncode == 0, p.stdout + p.stderr
    return p.stdout, out


def test_debug_build_is_clean_and_bit_identical_on_guarded_shapes(tmp_path):
    from grouped_gemm_fp32_b200 import build
    build.build()
    dbg, dpath = _child(STEP, tmp_path, True)
    rel, rpath = _child(STEP, tmp_path, False)
    assert "library libmoe_debug.so" in dbg and "library libmoe.so" in rel
    for i in range(len(SHAPES)):
        assert f"shape {i} status 0 intact True" in dbg, dbg
        assert f"shape {i} status 0 intact True" in rel, rel
    a, b = np.load(dpath), np.load(rpath)
    assert sorted(a.files) == sorted(b.files)
    for key in a.files:
        assert np.array_equal(a[key], b[key]), key


def test_debug_build_reports_a_corrupted_group_table(tmp_path):
    from grouped_gemm_fp32_b200 import build
    build.build()
    out, _ = _child(CORRUPT, tmp_path, True)
    assert "clean status 0" in out, out
    assert "fwd status -5" in out, out
    assert "combine_bwd status -5" in out, out
    assert "dw 2 status -5" in out and "dw 1 status -5" in out, out
    assert "intact True" in out, out
    assert "context ok True" in out, out
