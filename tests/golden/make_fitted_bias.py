"""Write the fitted selection biases of the ``skewed`` and ``train`` workloads.

Calls only ``oracle`` (router) and ``synth`` (inputs).  Run from the repo root:

    python tests/golden/make_fitted_bias.py

Passage: dots.llm1 Technical Report, §Architecture "Load balancing": the
per-expert bias is added to the affinity scores to decide the top-k routing
and is adjusted during training to steer expert loads.  The pages give no
update formula; the plainest reading, used here only to *construct inputs*,
is a sign step toward a target load:  b_e += gamma * sign(target_e - load_e).

* ``train`` (T=16384, uniform routing): target T*k/E for every expert.
* ``skewed`` (T=8192, Zipf s=1.2): 8 experts are switched off with bias -1
  (a score p - 1 <= 0 never beats an expert with bias >= 0, so they receive no
  token); the other 120, in a seeded random rank order, target n_r ~ r^-1.2,
  capped at T (an expert can take each token at most once) with the excess
  water-filled down the ranks so the targets sum to T*k.

Loads are computed with the oracle's FP64 router on the workload's own X and
Wg.  Output: one bias per line (f32 repr) plus a header with the achieved
load statistics.
"""
from __future__ import annotations

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def loads(probs, bias, k):
    s = probs + bias[None, :].astype(np.float64)
    # top-k by s, equal scores to the lower index (the oracle router's rule)
    order = np.lexsort((np.broadcast_to(np.arange(s.shape[1]), s.shape), -s), axis=1)
    sel = order[:, :k]
    return np.bincount(sel.ravel(), minlength=s.shape[1])


def fit(probs, k, target, bias0, active, rounds=400, gamma0=0.02, halve_every=50):
    b = bias0.astype(np.float64).copy()
    for r in range(rounds):
        gamma = gamma0 * 0.5 ** (r // halve_every)
        ld = loads(probs, b.astype(np.float32), k)
        step = np.sign(target - ld) * gamma
        b[active] += step[active]
    return b.astype(np.float32)


def zipf_targets(T, k, n_active, s=1.2):
    w = np.arange(1, n_active + 1, dtype=np.float64) ** -s
    tot = T * k
    tgt = np.zeros(n_active)
    free = np.ones(n_active, bool)
    remaining = float(tot)
    while True:  # water-fill: cap at T, spread the excess over the uncapped ranks
        share = remaining * w / w[free].sum()
        share[~free] = 0
        over = free & (share > T)
        if not over.any():
            tgt[free] = share[free]
            break
        tgt[over] = T
        free &= ~over
        remaining = tot - tgt[~free].sum()
    return tgt


def probs_of(wl):
    inp = synth.make_inputs(wl, with_weights=False)
    p, *_ = oracle.route(oracle.gate_logits(inp["x"], inp["wg"]),
                         np.zeros(wl.dims.E, np.float32), wl.dims.k)
    return p


def write(name, bias, ld, note):
    mean = ld.sum() / len(ld)
    path = os.path.join(HERE, f"{name}_bias.txt")
    with open(path, "w") as f:
        f.write(f"# fitted selection bias of the '{name}' workload; written by make_fitted_bias.py\n")
        f.write(f"# {note}\n")
        f.write(f"# achieved loads: max {ld.max()} min {ld.min()} mean {mean:.1f} "
                f"empty {(ld == 0).sum()} above_4x_mean {(ld > 4 * mean).sum()}\n")
        for v in bias:
            f.write(f"{float(v)!r}\n")
    print(path, "max/mean", ld.max() / mean, "empty", (ld == 0).sum(), ">4x", (ld > 4 * mean).sum())


def main():
    # uniform routing for the training workload
    wl = synth.WORKLOADS["train"]
    dm = wl.dims
    p = probs_of(wl)
    tgt = np.full(dm.E, dm.T * dm.k / dm.E)
    b = fit(p, dm.k, tgt, np.zeros(dm.E), np.ones(dm.E, bool), rounds=200, gamma0=1e-3)
    write("train", b, loads(p, b, dm.k), "target: equal loads T*k/E (sign-step fit)")

    # Zipf(1.2) loads for the skewed workload
    wl = synth.WORKLOADS["skewed"]
    dm = wl.dims
    p = probs_of(wl)
    rank = np.argsort(synth.uniform_f32(wl.seed, 7, (dm.E,), 0.0, 1.0), kind="stable")
    off, on = rank[dm.E - 8:], rank[:dm.E - 8]       # last 8 in the random order: no tokens
    tgt = np.zeros(dm.E)
    tgt[on] = zipf_targets(dm.T, dm.k, len(on))
    b0 = np.zeros(dm.E)
    b0[off] = -1.0
    active = np.zeros(dm.E, bool)
    active[on] = True
    b = fit(p, dm.k, tgt, b0, active)
    ld = loads(p, b, dm.k)
    write("skewed", b, ld, "target: Zipf(1.2) over 120 ranked experts, capped at T; 8 experts off")


if __name__ == "__main__":
    main()
