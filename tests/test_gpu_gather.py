"""Gathered x rows: the first GEMM and dW1 read the routed rows of x through
sorted_ids (tile::gather4 tensor copies) instead of a permuted copy x_perm.

Passage: dots.llm1 Technical Report, §3.2 "Efficient implementation of Grouped
GEMM" (each expert's rows form one aligned segment; which rows they are is
given by the permutation).

Three checks:
  * the gathered GEMM alone against the oracle, with hostile ids in the pad
    rows (-1, past T, negative) that the kernel must replace by a real row;
  * the whole layer step with and without x_perm: every result that has a
    definition (real rows of h, a1, y; out; dX; dW1; dW2) is bit-identical,
    since the same products meet in the same order -- up to the full train
    shapes and the launch configuration the benchmark times;
  * moe_permute_align without x_perm writes the same routing tables.
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


def _bits(t):
    return t.contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32)


def test_gather_gemm_alone_matches_oracle():
    # groups shorter than a tile, an empty group, a group over several tiles with a
    # ragged tail; pad block 16 so pair tiles run past a group's end into the next
    T, d, E, I, P = 700, 192, 6, 64, 16
    group_rows = [0, 5, 130, 16, 300, 17]
    pads = [-(-r // P) * P for r in group_rows]
    off = np.concatenate([[0], np.cumsum(pads)]).astype(np.int64)
    Rr = T + E * (P - 1)
    dm = moe.MoeDims.of(T, d, E, 1, 0, I, P, Rr)
    rng = np.random.default_rng(5)
    x_np = synth.normal_bf16(5, 1, (T, d), 1.0)
    ids = np.full(Rr, -1, np.int32)
    hostile = [-1, T, T + 1000, -7]
    for e in range(E):
        ids[off[e]:off[e] + group_rows[e]] = rng.choice(T, group_rows[e], replace=False)
        npad = pads[e] - group_rows[e]
        ids[off[e] + group_rows[e]:off[e + 1]] = [hostile[i % 4] for i in range(npad)]
    w1 = synth.normal_bf16(5, 4, (E, 2 * I, d), 0.08)
    w2 = synth.normal_bf16(5, 5, (E, d, I), 0.1)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    moe.grouped_gemm_set_groups(dm, dev(np.array(group_rows, np.int32)), offsets, ws)
    Rt = moe.moe_rows_total(dm)
    h = torch.full((Rt, I), float("nan"), dtype=torch.bfloat16, device="cuda")
    a1 = torch.full((Rt, 2 * I), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = torch.full((Rt, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.grouped_gemm_fwd_gather(dm, ws, dev(ids), dev(x_np, True), dev(w1, True), dev(w2, True),
                                h, a1, y)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    H, A1, Y = host(h), host(a1), host(y)
    for e in range(E):
        if group_rows[e] == 0:
            continue
        R = off[e] + np.arange(group_rows[e])
        g, u, hh, yy = oracle.expert_fwd(x_np[ids[R]], w1[e], w2[e])
        assert_close(H[R], hh, f"H group {e}")
        assert_close(A1[R], np.concatenate([g, u], axis=1), f"A1 group {e}")
        assert_close(Y[R], yy, f"Y group {e}")
        # a pad row holds the group's first token's results (never a row outside x)
        if pads[e] > group_rows[e]:
            p0 = off[e] + group_rows[e]
            assert np.array_equal(H[p0], H[off[e]]) and np.array_equal(Y[p0], Y[off[e]])
    assert np.all(np.isfinite(H[:off[-1]])) and np.all(np.isfinite(Y[:off[-1]]))


def _step(wl, inp, gather, train):
    dm = dims_of(wl)
    b = layer.MoEBuffers(dm, train=train, gather=gather)
    x = dev(inp["x"], True)
    w1, w2 = dev(inp["w1"], True), dev(inp["w2"], True)
    wg, bias = dev(inp["wg"]), dev(inp["bias"])
    layer.forward(b, x, wg, bias, w1, w2)
    if train:
        layer.backward(b, x, dev(inp["dout"], True), w1, w2, wg=wg)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(b.ws) == 0
    return b


def _same_results(a, b, train):
    assert torch.equal(a.sorted_ids, b.sorted_ids) and torch.equal(a.row_of, b.row_of)
    real = torch.cat([a.sorted_ids >= 0,
                      torch.ones(a.Rt - a.Rr, dtype=torch.bool, device="cuda")])
    for name in ("h", "y") + (("a1",) if train else ()):
        ta, tb = getattr(a, name), getattr(b, name)
        assert torch.equal(_bits(ta[real]), _bits(tb[real])), name
    assert torch.equal(_bits(a.out), _bits(b.out)), "out"
    if train:
        for name in ("dx", "dw1", "dw2", "dwg", "dw_comb"):
            assert torch.equal(_bits(getattr(a, name)), _bits(getattr(b, name))), name


@pytest.mark.parametrize("T,d,E,k,S,I,P,train", [
    (301, 192, 8, 2, 1, 64, 64, True),      # ragged T, partial N tile
    (77, 128, 16, 4, 2, 128, 16, False),    # pad block 16: pair tiles cross group ends
    (1000, 256, 32, 6, 1, 192, 64, True),   # narrow last N tile in dW1 / dX
])
def test_layer_gather_equals_x_perm_path(T, d, E, k, S, I, P, train):
    wl = synth.Workload("gather", synth.Dims(T=T, d=d, E=E, k=k, S=S, I=I, P=P), seed=T + k,
                        w1_std=0.05, w2_std=0.05, wg_std=0.05, backward=train)
    inp = synth.make_inputs(wl)
    _same_results(_step(wl, inp, True, train), _step(wl, inp, False, train), train)


@pytest.mark.parametrize("name,train", [("layer", False), ("train", True)])
def test_full_size_gather_equals_x_perm_path(name, train):
    """The benchmark's shapes (T=8192 forward; T=16384 forward + backward with
    the router backward): the gathered path against the x_perm path, bit for bit."""
    wl = synth.WORKLOADS[name]
    inp = workload_inputs(name)
    a = _step(wl, inp, True, train)
    b = _step(wl, inp, False, train)
    _same_results(a, b, train)


def test_permute_without_x_perm_writes_the_same_tables():
    wl = synth.WORKLOADS["skewed"]
    inp = workload_inputs("skewed", with_weights=False)
    dm = dims_of(wl)
    _, idx, _, _ = oracle.route(oracle.gate_logits(inp["x"][:2048], inp["wg"]), inp["bias"],
                                dm.k)
    dm2 = moe.MoeDims.of(2048, dm.d, dm.E, dm.k, dm.S, dm.I, dm.P)
    Rr = moe.moe_rows_routed(dm2)
    x = dev(inp["x"][:2048], True)

    def run(with_copy):
        ws = torch.zeros(moe.moe_workspace_size(dm2), dtype=torch.uint8, device="cuda")
        o = dict(counts=torch.empty(dm.E, dtype=torch.int32, device="cuda"),
                 offsets=torch.empty(dm.E + 1, dtype=torch.int32, device="cuda"),
                 sorted_ids=torch.empty(Rr, dtype=torch.int32, device="cuda"),
                 row_of=torch.empty(2048, dm.k, dtype=torch.int32, device="cuda"))
        xp = torch.zeros(Rr, dm.d, dtype=torch.bfloat16, device="cuda") if with_copy else None
        moe.moe_permute_align(dm2, dev(idx), x if with_copy else None, o["counts"], o["offsets"],
                              o["sorted_ids"], o["row_of"], xp, ws)
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(ws) == 0
        return o, ws

    a, wsa = run(True)
    b, wsb = run(False)
    for key in a:
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(wsa, wsb)  # the group table (and every other workspace byte)


def test_gather_after_refused_permutation_reads_nothing_routed():
    # an expert id out of range: the permutation is refused, the group table holds no
    # routed rows and sorted_ids stays -1; the gathered GEMM then runs the shared
    # expert only, exactly as the x_perm GEMM does
    T, d, E, k, S, I = 64, 128, 8, 2, 1, 64
    dm = moe.MoeDims.of(T, d, E, k, S, I, 16)
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    idx[9, 0] = 40
    Rr, Rt = moe.moe_rows_routed(dm), moe.moe_rows_total(dm)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    i32 = lambda n: torch.empty(n, dtype=torch.int32, device="cuda")
    sorted_ids, row_of = i32(Rr), i32(T * k)
    x_np = synth.normal_bf16(3, 1, (T, d), 1.0)
    x = dev(x_np, True)
    x_perm = torch.zeros(Rr, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute_align(dm, dev(idx), x, i32(E), i32(E + 1), sorted_ids, row_of, x_perm, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == -5
    assert torch.all(sorted_ids == -1)
    w1 = dev(synth.normal_bf16(3, 4, (E + S, 2 * I, d), 0.05), True)
    w2 = dev(synth.normal_bf16(3, 5, (E + S, d, I), 0.05), True)
    outs = []
    for gather in (False, True):
        h = torch.full((Rt, I), 7.0, dtype=torch.bfloat16, device="cuda")
        y = torch.full((Rt, d), 7.0, dtype=torch.bfloat16, device="cuda")
        if gather:
            moe.grouped_gemm_fwd_gather(dm, ws, sorted_ids, x, w1, w2, h, None, y)
        else:
            moe.grouped_gemm_fwd(dm, ws, x_perm, x, w1, w2, h, None, y)
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(ws) == 0
        outs.append((h, y))
    (h0, y0), (h1, y1) = outs
    assert torch.all(y1[:Rr] == 7.0)                 # no routed row written
    assert torch.equal(_bits(h0), _bits(h1)) and torch.equal(_bits(y0), _bits(y1))
    _, _, _, ys = oracle.expert_fwd(x_np, synth.normal_bf16(3, 4, (E + S, 2 * I, d), 0.05)[E],
                                    synth.normal_bf16(3, 5, (E + S, d, I), 0.05)[E])
    assert_close(host(y1[Rr:]), ys, "shared expert Y")
