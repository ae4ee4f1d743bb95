"""GPU parity of the gate / top-k and of the permutation, against the oracle.

Passages: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
(FP32 gating), "Load balancing" (bias for selection only, no dropped token),
§3.2 (segments padded to a fixed block).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from common import (MARGIN_EXEMPT, W_TOL, check_routing, dev, dims_of, host, oracle_routing,
                    workload_inputs)
import grouped_gemm_fp32_b200 as moe

pytestmark = pytest.mark.gpu


def _gate(dm, x, wg, bias, with_probs=True):
    T, E, k = dm.T, dm.E, dm.k
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    probs = torch.empty(T, E, dtype=torch.float32, device="cuda") if with_probs else None
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    moe.moe_gate_topk(dm, x, wg, bias, idx, w, probs, ws)
    torch.cuda.synchronize()
    return idx, w, probs


@pytest.mark.parametrize("name", ["tiny", "layer", "skewed", "train"])
def test_gate_topk_matches_oracle(name):
    wl = synth.WORKLOADS[name]
    inp = workload_inputs(name, with_weights=False)
    dm = dims_of(wl)
    idx, w, probs = _gate(dm, dev(inp["x"], True), dev(inp["wg"]), dev(inp["bias"]))
    p, oidx, ow, margin = oracle_routing(name)
    same, align = check_routing(host(idx), host(w), p, oidx, ow, margin, inp["bias"])
    assert np.max(np.abs(host(probs) - p)) <= W_TOL
    np.testing.assert_allclose(host(w).sum(axis=1), 1.0, atol=1e-5)
    order_diff = int((np.any(align != np.arange(dm.k), axis=1) & same).sum())
    print(f"{name}: {int((~same).sum())} of {dm.T} tokens chose another near-tied set "
          f"(margin < {MARGIN_EXEMPT}); {order_diff} ordered two near-tied picks differently")


def test_gate_ties_go_to_lower_index():
    # x = 0 -> every logit is 0 -> p = 1/8 exactly; biases on a 2^-10 grid make exact ties
    T, d, E, k = 8, 64, 8, 3
    dm = moe.MoeDims.of(T, d, E, k, 0, 64, 16)
    x = np.zeros((T, d), np.uint16)
    wg = synth.normal_f32(9, 2, (E, d), 0.1)
    bias = (np.array([0, 3, 3, 1, 3, 0, 2, 2]) / 1024.0).astype(np.float32)
    idx, w, _ = _gate(dm, dev(x, True), dev(wg), dev(bias))
    _, oidx, ow, _ = oracle.route(np.zeros((T, E)), bias, k)
    assert np.array_equal(host(idx), oidx)
    assert list(oidx[0]) == [1, 2, 4]
    np.testing.assert_allclose(host(w), ow, atol=1e-7)


def test_gate_resolves_fp32_weight_bits():
    # Gate weights 1 + e * 2^-22 differ only below bf16's 8-bit significand; with x = +1, -1,
    # +1, ... the logits are exactly e * 2^-11 (d = 4096), so an FP32 gate ranks the experts
    # 7, 6, 5 (score gaps ~6e-5, above the margin exemption) where a gate that rounded Wg to
    # bf16 would see equal logits and pick 0, 1, 2.  (FP32 gate: §Architecture "Mixture of
    # Experts layer".)
    T, d, E, k = 256, 4096, 8, 3
    sign = np.where(np.arange(d) % 2 == 0, 1.0, -1.0).astype(np.float32)
    x = np.tile((sign.view(np.uint32) >> 16).astype(np.uint16), (T, 1))
    wg = np.ones((E, d), np.float32)
    wg[:, 0::2] += (np.arange(E, dtype=np.float32) * np.float32(2.0 ** -22))[:, None]
    dm = moe.MoeDims.of(T, d, E, k, 0, 64, 16)
    idx, w, probs = _gate(dm, dev(x, True), dev(wg), None)
    p, oidx, ow, margin = oracle.route(oracle.gate_logits(x, wg), np.zeros(E, np.float32), k)
    assert oidx[0].tolist() == [7, 6, 5] and margin.min() > MARGIN_EXEMPT
    assert np.array_equal(host(idx), oidx)
    np.testing.assert_allclose(host(w), ow, atol=1e-6)
    np.testing.assert_allclose(host(probs), p, atol=1e-7)


def test_gate_bias_none_equals_zero_bias():
    wl = synth.WORKLOADS["tiny"]
    inp = workload_inputs("tiny", with_weights=False)
    dm = dims_of(wl)
    a = _gate(dm, dev(inp["x"], True), dev(inp["wg"]), None)
    b = _gate(dm, dev(inp["x"], True), dev(inp["wg"]), dev(np.zeros(dm.E, np.float32)))
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def _permute(dm, idx_np, x_np):
    T, k, E, d = dm.T, dm.k, dm.E, dm.d
    Rr = moe.moe_rows_routed(dm)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    out = dict(
        counts=torch.empty(E, dtype=torch.int32, device="cuda"),
        offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
        sorted_ids=torch.empty(Rr, dtype=torch.int32, device="cuda"),
        row_of=torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
        x_perm=torch.full((Rr, d), 3.0, dtype=torch.bfloat16, device="cuda"),
    )
    moe.moe_permute_align(dm, dev(idx_np), dev(x_np, True), out["counts"], out["offsets"],
                          out["sorted_ids"], out["row_of"], out["x_perm"], ws)
    torch.cuda.synchronize()
    return out, ws


def _check_permute(dm, idx_np, x_np, out):
    Rr = moe.moe_rows_routed(dm)
    ref = oracle.permute(idx_np, dm.E, dm.P, Rr)
    for key in ("counts", "offsets", "sorted_ids", "row_of"):
        assert np.array_equal(host(out[key]), ref[key]), key
    total = ref["total"]
    xp = out["x_perm"].view(torch.int16).cpu().numpy().view(np.uint16)[:total]
    ids = ref["sorted_ids"][:total]
    real = ids >= 0
    assert np.array_equal(xp[real], x_np[ids[real]])       # x_perm[row_of[t, j]] = x[t]
    assert np.all(xp[~real] == 0)                            # pad rows are zero
    return ref


@pytest.mark.parametrize("name", ["tiny", "layer", "skewed", "train"])
def test_permute_matches_oracle(name):
    wl = synth.WORKLOADS[name]
    inp = workload_inputs(name, with_weights=False)
    _, oidx, _, _ = oracle_routing(name)
    dm = dims_of(wl)
    out, ws = _permute(dm, oidx, inp["x"])
    ref = _check_permute(dm, oidx, inp["x"], out)
    assert moe.moe_get_device_status(ws) == 0
    if name == "skewed":
        assert (ref["counts"] == 0).sum() >= 8


@pytest.mark.parametrize("T,E,k,P,d", [(1, 8, 2, 16, 64), (37, 8, 8, 8, 128), (500, 256, 1, 128, 64),
                                       (333, 16, 4, 64, 192)])
def test_permute_edge_shapes(T, E, k, P, d):
    rng = np.random.default_rng(T + E)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    idx[idx == 1] = 0 if k == 1 else idx[idx == 1]  # leave expert 1 empty when k == 1
    x = synth.normal_bf16(T, 1, (T, d), 1.0)
    dm = moe.MoeDims.of(T, d, E, k, 1, 64, P)
    out, ws = _permute(dm, idx, x)
    _check_permute(dm, idx, x, out)


def test_permute_is_deterministic():
    inp = workload_inputs("layer", with_weights=False)
    _, oidx, _, _ = oracle_routing("layer")
    dm = dims_of(synth.WORKLOADS["layer"])
    a, _ = _permute(dm, oidx, inp["x"])
    b, _ = _permute(dm, oidx, inp["x"])
    for key in a:
        assert torch.equal(a[key], b[key]), key


def test_permute_rejects_bad_expert_id():
    T, E, k, d = 16, 8, 2, 64
    idx = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    idx[5, 1] = 9  # out of range
    dm = moe.MoeDims.of(T, d, E, k, 0, 64, 16)
    out, ws = _permute(dm, idx, synth.normal_bf16(1, 1, (T, d), 1.0))
    assert moe.moe_get_device_status(ws) == -5  # MOE_ERR_BAD_ROUTING
    assert moe.moe_get_device_status(ws) == 0   # read clears it
    assert np.all(host(out["sorted_ids"]) == -1)
