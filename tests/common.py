"""Helpers shared by the tests: workload inputs, device upload, tolerances."""
from __future__ import annotations

import os

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# Floating-point bar for bf16-in / FP32-accumulate outputs and gradients:
# max|got - ref| <= REL_TOL * max|ref| per output tensor.
REL_TOL = 2e-2
# Routing indices must match except for tokens whose oracle margin between the
# k-th and (k+1)-th biased score is below this.
MARGIN_EXEMPT = 1e-5
# Combine weights: absolute tolerance (FP32 softmax against the FP64 oracle).
W_TOL = 1e-5


def fitted_bias(name: str) -> np.ndarray:
    vals = []
    with open(os.path.join(GOLDEN, f"{name}_bias.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(float(line))
    return np.array(vals, dtype=np.float32)


def workload_inputs(name: str, with_weights: bool = True) -> dict:
    wl = synth.WORKLOADS[name]
    bias = fitted_bias(name) if name in ("skewed", "train") else None
    return synth.make_inputs(wl, with_weights=with_weights, bias_override=bias)


def dims_of(wl_or_dims):
    from grouped_gemm_fp32_b200 import MoeDims
    dm = wl_or_dims.dims if hasattr(wl_or_dims, "dims") else wl_or_dims
    return MoeDims.of(dm.T, dm.d, dm.E, dm.k, dm.S, dm.I, dm.P, dm.rows_cap)


def dev(a, bf16: bool = False):
    """numpy -> CUDA tensor (uint16 bit patterns become torch.bfloat16)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if bf16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def host(t) -> np.ndarray:
    """CUDA tensor -> numpy (bf16 widened to float64)."""
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def rel_err(got, ref) -> float:
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    scale = np.max(np.abs(ref))
    return float(np.max(np.abs(got - ref)) / (scale if scale > 0 else 1.0))


def assert_close(got, ref, what: str, tol: float = REL_TOL):
    e = rel_err(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert e <= tol, f"{what}: max|diff|/max|ref| = {e:.3e} > {tol}"
    return e


_ROUTING_CACHE: dict = {}


def oracle_routing(name: str):
    """Oracle router on a workload's own inputs (cached per process):
    (probs, idx, w, margin) with idx/w in the oracle's order."""
    if name not in _ROUTING_CACHE:
        import oracle
        inp = workload_inputs(name, with_weights=False)
        k = synth.WORKLOADS[name].dims.k
        _ROUTING_CACHE[name] = oracle.route(oracle.gate_logits(inp["x"], inp["wg"]), inp["bias"], k)
    return _ROUTING_CACHE[name]


def check_routing(gidx, gw, probs, oidx, ow, margin, bias):
    """GPU routing vs the oracle.

    * The chosen SET is identical wherever the oracle margin (k-th minus
      (k+1)-th biased score) is >= 1e-5; elsewhere every GPU pick must score
      within 1e-5 of the oracle's k-th.
    * The ORDER (biased score descending) is identical except between chosen
      experts whose oracle scores differ by less than 1e-5: the GPU's order must
      be non-increasing in the oracle's scores up to 1e-5.
    * Weights match per expert within W_TOL.
    Returns (same_set mask [T], align [T, k]) with gidx[t, align[t, j]] == oidx[t, j]
    for tokens of the same set."""
    T, k = oidx.shape
    s = probs + bias[None, :].astype(np.float64)
    same = np.sort(gidx, axis=1) == np.sort(oidx, axis=1)
    same = np.all(same, axis=1)
    exempt = margin < MARGIN_EXEMPT
    bad = ~same & ~exempt
    assert not bad.any(), f"{bad.sum()} tokens chose a different expert set with margin >= {MARGIN_EXEMPT}"
    for t in np.nonzero(~same)[0]:
        kth = s[t, oidx[t, k - 1]]
        assert len(set(gidx[t])) == k
        assert np.all(s[t, gidx[t]] >= kth - MARGIN_EXEMPT), t
    gs = np.take_along_axis(s, gidx.astype(np.int64), axis=1)
    assert np.all(gs[:, :-1] >= gs[:, 1:] - MARGIN_EXEMPT), "GPU order is not by biased score"
    align = np.zeros((T, k), dtype=np.int64)
    for t in np.nonzero(same)[0]:
        pos = {int(e): j for j, e in enumerate(gidx[t])}
        align[t] = [pos[int(e)] for e in oidx[t]]
    if same.any():
        gw_al = np.take_along_axis(gw, align, axis=1)
        assert np.max(np.abs(gw_al[same] - ow[same])) <= W_TOL
    return same, align


def sample_tokens(oidx, cand, n, seed, per_expert=16):
    """A seeded sample of ``n`` tokens for full-size parity checks: tokens of the
    most-loaded and of the least-loaded non-empty routed experts (``per_expert``
    of each), the first and last candidates, and random ones, all from ``cand``
    (tokens eligible for an exact comparison), sorted and unique."""
    rng = np.random.default_rng(seed)
    cand = np.asarray(cand, dtype=np.int64)
    E = int(oidx.max()) + 1
    counts = np.bincount(oidx.ravel(), minlength=E)
    nonempty = np.nonzero(counts)[0]
    pick = []
    for e in (int(counts.argmax()), int(nonempty[counts[nonempty].argmin()])):
        mask = np.any(oidx[cand] == e, axis=1)
        pick.extend(cand[mask][:per_expert].tolist())
    pick.extend([int(cand[0]), int(cand[-1])])
    rest = np.setdiff1d(cand, np.array(pick, dtype=np.int64))
    need = max(0, n - len(set(pick)))
    pick.extend(rng.choice(rest, min(need, len(rest)), replace=False).tolist())
    return np.unique(np.array(pick, dtype=np.int64))


def ep_plan_reference(counts_all, rank, P, cap):
    """The exchange plan of expert parallelism written out from its definition, for
    checking the device plan (moe_ep_plan) and the cross-rank agreement of offsets.
    counts_all [W, E]: rank s's tokens per expert.  Rank o owns experts o E_l ..
    (o + 1) E_l - 1 and lays out what it receives expert-major: for each local expert,
    the P-padded segments of ranks 0 .. W - 1.  Returns a dict of numpy int arrays:
    send_dst [E] (this rank's segment of expert g starts at that row of its owner's
    buffer), recv_row / recv_cnt / recv_real / src_off [W, E_l] (this rank as owner: where
    source s's segment of local expert e lands, its padded and real rows, and where it
    starts in source s's permuted rows), counts_loc [E_l], over [W]."""
    c = np.asarray(counts_all, dtype=np.int64)
    W, E = c.shape
    El = E // W
    pad = (c + P - 1) // P * P
    out = {k: np.zeros((W, El), np.int64) for k in ("recv_row", "recv_cnt", "recv_real",
                                                       "src_off")}
    send_dst = np.zeros(E, np.int64)
    over = np.zeros(W, np.int64)
    for o in range(W):
        row = 0
        for e in range(El):
            g = o * El + e
            for s in range(W):
                if s == rank:
                    send_dst[g] = row
                if o == rank:
                    out["recv_row"][s, e] = row
                    out["recv_cnt"][s, e] = pad[s, g]
                    out["recv_real"][s, e] = c[s, g]
                    out["src_off"][s, e] = pad[s, :g].sum()
                row += pad[s, g]
        over[o] = row > cap
    out["send_dst"] = send_dst
    out["counts_loc"] = pad[:, rank * El:(rank + 1) * El].sum(axis=0)
    out["over"] = over
    return out
