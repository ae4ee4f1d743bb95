"""GPU parity of the grouped GEMM forward, the combine and the whole layer
forward, against the oracle.

Passages: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
(fine-grained SwiGLU experts, 6 routed + 2 shared per token) and §3.2
"Efficient implementation of Grouped GEMM" (one tile = one expert's padded
segment).  Bar: max|diff| <= 2e-2 * max|ref| per output tensor.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from common import (assert_close, check_routing, dev, dims_of, host, oracle_routing,
                    sample_tokens, workload_inputs)
import grouped_gemm_fp32_b200 as moe
from grouped_gemm_fp32_b200 import layer

pytestmark = pytest.mark.gpu


def _gemm_only_case(dims: synth.Dims, group_rows, seed, w1_std, w2_std, check_rows):
    """Grouped GEMM alone: groups of given sizes over a permuted A."""
    E, d, I = dims.E, dims.d, dims.I
    pads = [-(-r // dims.P) * dims.P for r in group_rows]
    Rr = dims.rows_cap
    x_np = synth.normal_bf16(seed, 1, (Rr, d), 1.0)
    # rows beyond each group's real rows are pad rows: zero, as the permute leaves them
    off = np.concatenate([[0], np.cumsum(pads)])
    for e in range(E):
        x_np[off[e] + group_rows[e]:off[e + 1]] = 0
    w1 = synth.normal_bf16(seed, 4, (E, 2 * I, d), w1_std)
    w2 = synth.normal_bf16(seed, 5, (E, d, I), w2_std)
    dm = moe.MoeDims.of(dims.T, d, E, dims.k, 0, I, dims.P, Rr)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    counts = dev(np.array(group_rows, np.int32))
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    moe.grouped_gemm_set_groups(dm, counts, offsets, ws)
    Rt = moe.moe_rows_total(dm)
    h = torch.full((Rt, I), float("nan"), dtype=torch.bfloat16, device="cuda")
    a1 = torch.full((Rt, 2 * I), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = torch.full((Rt, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.grouped_gemm_fwd(dm, ws, dev(x_np, True), None, dev(w1, True), dev(w2, True), h, a1, y)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    assert np.array_equal(host(offsets), off)
    H, A1, Y = host(h), host(a1), host(y)
    for e in range(E):
        rows = sorted({r for r in check_rows(group_rows[e], pads[e]) if 0 <= r < pads[e]})
        if not rows:
            continue
        g, u, hh, yy = oracle.expert_fwd(x_np[off[e] + np.array(rows)], w1[e], w2[e])
        R = off[e] + np.array(rows)
        assert_close(H[R], hh, f"H group {e}")
        assert_close(A1[R], np.concatenate([g, u], axis=1), f"A1 group {e}")
        assert_close(Y[R], yy, f"Y group {e}")
    # every padded row of every group was written (no NaN left inside a segment)
    assert np.all(np.isfinite(H[:off[-1]])) and np.all(np.isfinite(Y[:off[-1]]))
    assert np.all(np.isfinite(A1[:off[-1]]))


def test_grouped_gemm_alone_16x512():
    wl = synth.WORKLOADS["gemm_only"]
    rows = lambda n, p: [0, 1, 63, 64, 127, 128, 200, 255, 256, 300, 383, 384, 450, 510, 511]
    _gemm_only_case(wl.dims, wl.group_rows, wl.seed, wl.w1_std, wl.w2_std, rows)


def test_grouped_gemm_ragged_groups():
    # empty group, groups shorter than a tile, a group spanning several tiles with a
    # ragged tail, I = 64 (64-wide gate/up halves), d = 192 (partial 256-wide N tile)
    dims = synth.Dims(T=1000, d=192, E=6, k=1, S=0, I=64, P=16, rows_cap=1000)
    group_rows = [0, 5, 130, 16, 300, 17]
    every = lambda n, p: range(p)
    _gemm_only_case(dims, group_rows, 21, 0.08, 0.1, every)


def _layer_forward(name, dims_override=None, inputs=None):
    wl = synth.WORKLOADS[name]
    inp = inputs if inputs is not None else workload_inputs(name)
    dm = dims_of(dims_override or wl)
    b = layer.MoEBuffers(dm, train=False)
    x = dev(inp["x"], True)
    w1, w2 = dev(inp["w1"], True), dev(inp["w2"], True)
    out = layer.forward(b, x, dev(inp["wg"]), dev(inp["bias"]), w1, w2)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    return inp, b, out


@pytest.mark.parametrize("name,nsample", [("tiny", None), ("layer", 512), ("skewed", 512)])
def test_layer_forward_matches_oracle(name, nsample):
    inp, b, out = _layer_forward(name)
    wl = synth.WORKLOADS[name]
    S = wl.dims.S
    p, oidx, ow, margin = oracle_routing(name)
    same, align = check_routing(host(b.topk_idx), host(b.topk_w), p, oidx, ow, margin,
                                inp["bias"])
    T = wl.dims.T
    if nsample is None:
        tokens = np.nonzero(same)[0]
    else:
        # 512 tokens: the hottest and the least-loaded experts' tokens among them
        tokens = sample_tokens(oidx, np.nonzero(same)[0], nsample, wl.seed)
    ref, yr, ys = oracle.layer_fwd(inp["x"], oidx, ow, inp["w1"], inp["w2"], S, tokens=tokens,
                                   want_y=True)
    assert_close(host(out)[tokens], ref, f"{name} out")
    # the expert output rows behind the combine
    Y = host(b.y)
    rof = np.take_along_axis(host(b.row_of), align, axis=1)  # in the oracle's pick order
    assert_close(Y[rof[tokens]], yr, f"{name} routed Y rows")
    for s in range(S):
        assert_close(Y[b.Rr + s * T + tokens], ys[:, s], f"{name} shared Y rows {s}")


def test_combine_unpermute_identity():
    # one-hot combine of the permuted rows gives x back exactly (k = 1, no shared expert)
    T, d, E, k = 256, 128, 8, 1
    dm = moe.MoeDims.of(T, d, E, k, 0, 64, 16)
    rng = np.random.default_rng(4)
    idx = rng.integers(0, E, size=(T, 1)).astype(np.int32)
    x_np = synth.normal_bf16(4, 1, (T, d), 1.0)
    Rr = moe.moe_rows_routed(dm)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    row_of = torch.empty(T, k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(Rr, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute_align(dm, dev(idx), dev(x_np, True),
                          torch.empty(E, dtype=torch.int32, device="cuda"),
                          torch.empty(E + 1, dtype=torch.int32, device="cuda"),
                          torch.empty(Rr, dtype=torch.int32, device="cuda"), row_of, x_perm, ws)
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(dm, x_perm, row_of, dev(np.ones((T, k), np.float32)), out)
    torch.cuda.synchronize()
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), x_np)


@pytest.mark.parametrize("weighted", [True, False], ids=["combine", "unpermute_sum"])
def test_combine_f32_is_the_unrounded_combine(weighted):
    # moe_combine_f32 keeps the FP32 sums moe_combine rounds: rounding them to bf16
    # gives moe_combine's bits, on the full layer workload (k + S = 8 rows a token)
    name = "layer"
    inp, b, out = _layer_forward(name)
    dm = dims_of(synth.WORKLOADS[name])
    w = b.topk_w if weighted else None
    ref16 = torch.empty_like(b.out)
    moe.moe_combine(dm, b.y, b.row_of, w, ref16)
    out32 = torch.full((dm.T, dm.d), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_combine_f32(dm, b.y, b.row_of, w, out32)
    torch.cuda.synchronize()
    assert torch.equal(out32.to(torch.bfloat16).view(torch.int16), ref16.view(torch.int16))
    if weighted:
        assert torch.equal(ref16.view(torch.int16), out.view(torch.int16))
        # against the oracle's combine of the GPU's own expert rows, FP64: FP32 sums
        Y = host(b.y)
        rof, tw = host(b.row_of), host(b.topk_w).astype(np.float64)
        ts = np.arange(0, dm.T, 97)
        ref = np.einsum("tj,tjd->td", tw[ts], Y[rof[ts]])
        for s in range(dm.S):
            ref += Y[b.Rr + s * dm.T + ts]
        assert np.max(np.abs(host(out32)[ts] - ref)) <= 1e-5 * np.abs(ref).max()
