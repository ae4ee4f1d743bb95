"""Benchmark of the MoE FFN layer (dots.llm1 fine-grained MoE) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload train|layer]
                    [--impl ours|reference]

One step = one pass of the whole hot path over one batch:
  train (default): T=16384 tokens, d=4096, 128 routed experts top-6 + 2 shared,
                   I=1408, pad block 128; forward (gate, top-k, permute, grouped
                   SwiGLU GEMMs, combine) + backward (combine bwd, dX and dW
                   grouped GEMMs, SwiGLU bwd, un-permute-sum, router backward
                   into dX and dWg) + the aux-loss-free bias step.
  layer:           T=8192, same layer, forward only.
  skewed:          layer with Zipf-shaped expert loads (8 empty experts, the
                   hottest taking every token), forward only.
  gemm_only:       the grouped GEMM forward alone (16 groups x 512 rows, d=4096,
                   I=1408): a small case for profiles, not the headline.
  train_small:     train with E=16, T=2048 (same rows per expert): profiles.
  gate_only:       the gate + top-k alone on the layer shapes: profiles.
  tiny:            T=64, d=128, E=8: host-side checks of the launch plumbing.
Inputs are synthetic (seeded generator), resident in HBM for ``value``; the
weights alone (4.5 GB) exceed L2, so no flush is needed between steps.

``value`` is whole-job tokens/s (device time, CUDA events, max over ranks);
``e2e`` is the same metric through the C ABI with the step's inputs copied from
pinned host memory and its results copied back inside the timed region.
``--impl reference`` times the FP64 CPU oracle on host cores instead.
For N > 1 (torchrun) each rank runs an independent replica of the step on its
own GPU (weak scaling; the single-GPU path has no exchange step).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# Update speed of the aux-loss-free bias step in the train step (the pages give no
# value; 1e-3 per step is an illustrative choice, applied to a copy of the bias so
# every timed step routes the same synthetic batch the same way).
GAMMA = 1e-3
# Sequence-wise balance loss of the train step: (alpha, tokens per sequence).  The
# pages give no alpha (a small illustrative value here); 8192 tokens is the
# pre-training sequence length they state.
SEQ_BALANCE = (1e-4, 8192)

METRIC = "MoE layer tokens/s and grouped-GEMM TFLOP/s (% of B200 BF16 peak), 1 GPU"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="train",
                    choices=["train", "layer", "skewed", "gemm_only", "train_small", "gate_only",
                             "tiny"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-layer", action="store_true",
                    help="skip the T = 8192 layer-forward measurement that the train run adds "
                         "(key north_star_c3)")
    ap.add_argument("--eager", action="store_true",
                    help="time the step as eager C-ABI calls instead of a replayed CUDA graph")
    ap.add_argument("--gather", action="store_true",
                    help="the first GEMM and dW1 gather x rows through sorted_ids instead of "
                         "reading the permuted copy x_perm")
    ap.add_argument("--ep", action="store_true",
                    help="a line of its own: the train step under expert parallelism over the "
                         "ranks (one rank: every peer pointer the rank's own buffer)")
    ap.add_argument("--library-gemm", action="store_true",
                    help="context, not the contract line: cuBLAS (torch.bmm) on the same GEMM "
                         "shapes with uniform groups, timed interleaved with this library's "
                         "grouped-GEMM calls (1 GPU, train workload)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def fitted_bias(name):
    path = os.path.join(ROOT, "tests", "golden", f"{name}_bias.txt")
    if not os.path.exists(path):
        return None
    vals = [float(l) for l in open(path) if l.strip() and not l.startswith("#")]
    return np.array(vals, dtype=np.float32)


def workload(name):
    import synth
    if name == "gate_only":
        wl = synth.WORKLOADS["layer"]
        return wl, synth.make_inputs(wl, with_weights=False)
    wl = synth.WORKLOADS[name]
    return wl, synth.make_inputs(wl, bias_override=fitted_bias(name))


def rank_shard(wl, inp, rank):
    """This rank's batch: its own tokens (X and the upstream gradient drawn from a
    rank-dependent seed), the replicated weights, gate and bias unchanged.  Rank 0
    keeps the workload's own batch."""
    if rank == 0:
        return inp
    import synth
    dm, seed = wl.dims, wl.seed + 7919 * rank
    out = dict(inp)
    out["x"] = synth.normal_bf16(seed, synth.SID_X, (dm.T, dm.d), wl.x_std)
    if "dout" in inp:
        out["dout"] = synth.normal_bf16(seed, synth.SID_DOUT, (dm.T, dm.d), 1.0)
    return out


def gemm_flops(dm, backward):
    """Algorithmic FLOPs of the grouped GEMMs (real rows only: T*k routed + S*T shared)."""
    R = dm.T * dm.k + dm.S * dm.T
    fwd1, fwd2 = 2 * R * dm.d * 2 * dm.I, 2 * R * dm.I * dm.d
    f = {"fwd": fwd1 + fwd2}
    if backward:
        f.update(dx2=2 * R * dm.d * dm.I, dw2=2 * R * dm.d * dm.I, dx1=2 * R * 2 * dm.I * dm.d,
                 dw1=2 * R * 2 * dm.I * dm.d)
    return f


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ggemm_dram_traffic_train.txt")
TRAFFIC_SOURCES = ["ggemm.cu", "sm100.cuh", "moe_internal.cuh", "permute.cu"]


def gemm_traffic(name):
    """DRAM bytes of one step's grouped-GEMM launches, from the committed ncu capture
    of the train workload, while the kernel sources still hash to the captured ones
    (None otherwise: the counters no longer describe the kernel that runs)."""
    import hashlib
    if name != "train" or not os.path.exists(TRAFFIC_FILE):
        return None, "no capture for this workload"
    fields = {}
    for line in open(TRAFFIC_FILE):
        if ":" in line and not line.startswith("#"):
            key, val = line.split(":", 1)
            fields[key.strip()] = val.strip()
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "grouped_gemm_fp32_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != fields.get("sources_sha256"):
        return None, "kernel sources changed since the capture"
    return float(fields["dram_bytes_per_step"]), (
        f"ncu dram__bytes_read.sum + dram__bytes_write.sum over the step's six GEMM launches "
        f"({os.path.relpath(TRAFFIC_FILE, ROOT)}); algorithmic "
        f"{float(fields['algorithmic_bytes_per_step']):.4g} B")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        backend = "nccl" if args.impl == "ours" else "gloo"
        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=600))
    elif args.impl == "ours":
        torch.cuda.set_device(local)
    return world, rank, local


def dist_max(v, world, device=None):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------- CPU (oracle) --
def oracle_sample_step(wl, inp, ntok):
    """The oracle on the first ``ntok`` tokens of the workload: gate + route +
    permute + expert forward (+ backward incl. every group's dW, the router
    backward and the bias step when the workload trains).  Returns seconds."""
    import oracle
    dm = wl.dims
    x = inp["x"][:ntok]
    t0 = time.perf_counter()
    lg = oracle.gate_logits(x, inp["wg"])
    _, idx, w, _ = oracle.route(lg, inp["bias"], dm.k)
    oracle.permute(idx, dm.E, dm.P, ntok * dm.k + dm.E * (dm.P - 1))
    oracle.layer_fwd(x, idx, w, inp["w1"], inp["w2"], dm.S)
    if wl.backward:
        dout = inp["dout"][:ntok]
        _, dw = oracle.layer_bwd(x, idx, w, inp["w1"], inp["w2"], dout, dm.S)
        used = set(np.unique(idx).tolist()) | set(range(dm.E, dm.E + dm.S))
        for g in sorted(used):
            oracle.group_dw(x, idx, w, inp["w1"], inp["w2"], dout, dm.S, g)
        _, dl_bal = oracle.seq_balance(lg, idx, SEQ_BALANCE[1], SEQ_BALANCE[0])
        oracle.router_bwd(x, inp["wg"], idx, dw, dl_extra=dl_bal)
        oracle.bias_update(idx, dm.E, inp["bias"], GAMMA)
    return time.perf_counter() - t0


def cpu_baseline(wl, inp, target_s=20.0):
    """The oracle on a sample of the workload's tokens sized from a 16-token probe
    for ``target_s`` seconds of host work (the probe overstates the per-token
    cost, so the sample itself takes less: about 10-15 s)."""
    import oracle
    oracle.build()
    oracle_sample_step(wl, inp, 2)  # warm the library and the page cache
    probe = oracle_sample_step(wl, inp, 16)
    ntok = int(min(wl.dims.T, max(16, 16 * target_s / max(probe, 1e-6))))
    secs = oracle_sample_step(wl, inp, ntok)
    return {"value": ntok / secs, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"first {ntok} tokens of the workload, full "
                      f"{'forward+backward (all dW, router backward, bias step)' if wl.backward else 'forward'} in FP64, "
                      f"{secs:.1f} s; tokens/s scales linearly in tokens"}


def run_reference(args):
    # under torchrun only rank 0 runs the oracle; the other ranks have no work
    if int(os.environ.get("RANK", "0")) != 0:
        return
    wl, inp = workload(args.workload)
    ntok = 16
    for _ in range(args.warmup):
        oracle_sample_step(wl, inp, ntok)
    total = 0.0
    for _ in range(args.steps):
        total += oracle_sample_step(wl, inp, ntok)
    import oracle
    val = ntok * args.steps / total
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": describe(wl), "sample_tokens_per_step": ntok},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "kind": "oracle",
                             "cores": oracle.num_threads(),
                             "sample": f"{ntok} tokens per step, full layer step in FP64"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def describe(wl):
    dm = wl.dims
    return (f"{wl.name}: T={dm.T} d={dm.d} E={dm.E} k={dm.k} S={dm.S} I={dm.I} P={dm.P}, "
            f"{'forward+backward' if wl.backward else 'forward'}")


# ---------------------------------------------------------------- GPU (ours) --
class Case:
    """One workload on this GPU: its inputs in HBM, the layer's buffers and the
    step as C-ABI calls, with an optional event between consecutive calls."""

    def __init__(self, name, args, dev, rank=0):
        import torch
        import grouped_gemm_fp32_b200 as moe
        from grouped_gemm_fp32_b200 import layer

        wl, inp = workload(name)
        inp = rank_shard(wl, inp, rank)  # data parallel: each rank its own tokens
        dm = wl.dims
        self.name, self.wl, self.inp, self.dm = name, wl, inp, dm
        self.dims = dims = moe.MoeDims.of(dm.T, dm.d, dm.E, dm.k, dm.S, dm.I, dm.P, dm.rows_cap)
        self.train = wl.backward
        self.gemm_only = wl.group_rows is not None
        self.gate_only = name == "gate_only"
        self.gather = args.gather
        bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).to(dev)
        self.x = bf(inp["x"])
        self.w1 = bf(inp["w1"]) if not self.gate_only else None
        self.w2 = bf(inp["w2"]) if not self.gate_only else None
        self.wg = torch.from_numpy(inp["wg"]).to(dev) if not self.gemm_only else None
        self.bias = torch.from_numpy(inp["bias"]).to(dev) if not self.gemm_only else None
        self.dout = bf(inp["dout"]) if self.train else None
        if self.gate_only:
            class _GateBufs:  # the gate's outputs only
                topk_idx = torch.empty(dm.T, dm.k, dtype=torch.int32, device=dev)
                topk_w = torch.empty(dm.T, dm.k, dtype=torch.float32, device=dev)
                ws = torch.zeros(moe.moe_workspace_size(dims), dtype=torch.uint8, device=dev)
                out = torch.empty(dm.T, dm.d, dtype=torch.bfloat16, device=dev)
            self.b = _GateBufs()
        else:
            self.b = layer.MoEBuffers(dims, device=dev, train=self.train, gather=self.gather)
        if self.gemm_only:
            counts = torch.tensor(wl.group_rows, dtype=torch.int32, device=dev)
            moe.grouped_gemm_set_groups(dims, counts, self.b.offsets, self.b.ws)
        # the calls of one step, in order; an event before the first and after each
        self.names = (["t0", "gate"] if self.gate_only else
                      ["t0", "fwd"] if self.gemm_only else
                      ["t0", "gate", "permute", "fwd", "combine"]) + (
            ["seq_balance", "combine_bwd", "dx2", "dw2", "dx1", "dw1", "unpermute", "router_bwd",
             "bias_step"] if self.train else [])
        torch.cuda.synchronize()

    def step(self, s, xx=None, gg=None, ev=None):
        """One step on stream ``s``; with ``ev`` (name -> event) an event is recorded
        before the first call and after each call, under the names of ``self.names``."""
        import grouped_gemm_fp32_b200 as L
        from grouped_gemm_fp32_b200 import layer
        xx = self.x if xx is None else xx
        gg = self.dout if gg is None else gg
        b, dims, train = self.b, self.dims, self.train
        wg, bias, w1, w2 = self.wg, self.bias, self.w1, self.w2
        rec = (lambda k: ev[k].record(s)) if ev is not None else (lambda k: None)
        if self.gate_only:
            rec("t0")
            L.moe_gate_topk(dims, xx, wg, bias, b.topk_idx, b.topk_w, None, b.ws, s)
            rec("gate")
            return
        if self.gemm_only:
            rec("t0")
            L.grouped_gemm_fwd(dims, b.ws, xx, None, w1, w2, b.h, None, b.y, s)
            rec("fwd")
            return
        if ev is None:  # the layer's own driver: the calls below, without events
            layer.forward(b, xx, wg, bias, w1, w2, stream=s,
                          seq_balance=SEQ_BALANCE if train else None)
            if train:
                layer.backward(b, xx, gg, w1, w2, stream=s, wg=wg, gamma=GAMMA, bias=bias)
            return
        rec("t0")
        L.moe_gate_topk(dims, xx, wg, bias, b.topk_idx, b.topk_w, b.probs if train else None,
                        b.ws, s)
        rec("gate")
        L.moe_permute_align(dims, b.topk_idx, xx, b.counts, b.offsets, b.sorted_ids, b.row_of,
                            b.x_perm, b.ws, s)
        rec("permute")
        if b.gather:
            L.grouped_gemm_fwd_gather(dims, b.ws, b.sorted_ids, xx, w1, w2, b.h, b.a1, b.y, s)
        else:
            L.grouped_gemm_fwd(dims, b.ws, b.x_perm, xx, w1, w2, b.h, b.a1, b.y, s)
        rec("fwd")
        L.moe_combine(dims, b.y, b.row_of, b.topk_w, b.out, s)
        rec("combine")
        if not train:
            return
        L.moe_seq_balance_loss(dims, SEQ_BALANCE[1], SEQ_BALANCE[0], b.topk_idx, b.probs,
                               b.bal_loss, b.bal_grad, b.ws, s)
        rec("seq_balance")
        L.moe_combine_bwd(dims, b.ws, gg, b.y, b.row_of, b.topk_w, b.dy, b.dw_comb, s)
        rec("combine_bwd")
        L.grouped_gemm_bwd_dx(dims, b.ws, L.MOE_GEMM2, b.dy, gg, w2, b.a1, b.da, s)
        rec("dx2")
        L.grouped_gemm_bwd_dw(dims, b.ws, L.MOE_GEMM2, b.dy, gg, b.h, None, b.dw2, 0, s)
        rec("dw2")
        L.grouped_gemm_bwd_dx(dims, b.ws, L.MOE_GEMM1, b.da, None, w1, None, b.dxp, s)
        rec("dx1")
        if b.gather:
            L.grouped_gemm_bwd_dw1_gather(dims, b.ws, b.sorted_ids, b.da, xx, b.dw1, 0, s)
        else:
            L.grouped_gemm_bwd_dw(dims, b.ws, L.MOE_GEMM1, b.da, None, b.x_perm, xx, b.dw1, 0, s)
        rec("dw1")
        L.moe_combine(dims, b.dxp, b.row_of, None, b.dx, s)
        rec("unpermute")
        L.moe_router_bwd_seqbal(dims, xx, wg, b.probs, b.topk_idx, b.topk_w, b.dw_comb,
                                b.bal_grad, SEQ_BALANCE[1], None, b.dx, b.dwg, 0, b.ws, s)
        rec("router_bwd")
        L.moe_bias_update(dims, b.counts, GAMMA, bias, b.bias_next, s)
        rec("bias_step")

    def check_status(self, stream, when):
        import grouped_gemm_fp32_b200 as moe
        status = moe.moe_get_device_status(self.b.ws, stream)
        if status != 0:
            raise RuntimeError(f"device status {when}: {moe.moe_status_string(status)}")


def timed_region(case, stream, steps, use_graph, world, dev, local):
    """The headline timing: ``steps`` steps between a barrier + synchronize and a
    synchronize + barrier, CUDA events on the launching stream, max over ranks, SM
    clocks sampled meanwhile.  With ``use_graph`` every step is a replayed CUDA graph
    of the step's C-ABI calls (one graph per timed step, captured beforehand).  Each
    step also records an event before its first call and after each call (event
    nodes inside the graphs), so the per-call breakdown comes from the timed steps
    themselves.  Returns (ms per step, per-call ms, clocks, gap between steps in ms)."""
    import torch
    names = case.names
    evs = [{n: torch.cuda.Event(enable_timing=True, external=use_graph) for n in names}
           for _ in range(steps)]
    graphs = []
    if use_graph:
        for i in range(steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                case.step(stream, ev=evs[i])
            graphs.append(g)
        torch.cuda.synchronize(dev)
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.25)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(steps):
            if use_graph:
                graphs[i].replay()
            else:
                case.step(stream, ev=evs[i])
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = clk.stop()
    ms = dist_max(e0.elapsed_time(e1) / steps, world, dev)
    per = {}
    for i in range(1, len(names)):
        per[names[i]] = sum(ev[names[i - 1]].elapsed_time(ev[names[i]]) for ev in evs) / steps
    inside = sum(ev[names[0]].elapsed_time(ev[names[-1]]) for ev in evs) / steps
    del graphs
    return ms, per, clocks, ms - inside


def gemm_roofline(case, per, pk, pk_src):
    """The grouped GEMM's algorithmic TFLOP/s over its launches' event times."""
    flops = gemm_flops(case.dm, case.train)
    gemm_ms = sum(per[k] for k in flops)
    achieved = sum(flops.values()) / (gemm_ms / 1000.0) / 1e12
    burst = pk["bf16_tflops"]
    sustained = pk.get("bf16_tflops_sustained", burst)
    detail = {k: {"ms": round(per[k], 4), "tflops": round(flops[k] / per[k] / 1e9, 1)}
              for k in flops}
    return gemm_ms, achieved, burst, sustained, detail


def layer_forward_t8192(args, dev, local, pk, pk_src):
    """The layer forward at T = 8192 (d = 4096, 128 routed experts top-6 + 2 shared,
    I = 1408, pad block 128, near-uniform loads), whose grouped GEMM's share of the dense
    bf16 peak is reported under its own key: its own inputs, warm-up, timed graph
    replays, clocks and per-call event times."""
    import torch
    case = Case("layer", args, dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            case.step(stream)
    stream.synchronize()
    case.check_status(stream, "after the layer warm-up")
    steps = max(20, args.steps)
    ms, per, clocks, gap = timed_region(case, stream, steps, True, 1, dev, local)
    case.check_status(stream, "after the layer timing")
    gemm_ms, achieved, burst, sustained, _ = gemm_roofline(case, per, pk, pk_src)
    out = {"workload": describe(case.wl), "steps": steps, "ms_per_step": round(ms, 4),
           "tokens_per_s": case.dm.T / (ms / 1000.0),
           "grouped_gemm_ms": round(gemm_ms, 4), "grouped_gemm_tflops": round(achieved, 1),
           "frac_of_burst_peak": round(achieved / burst, 4),
           "frac_of_sustained_peak": round(achieved / sustained, 4),
           "peak_burst": burst, "peak_sustained": sustained, "peak_source": pk_src,
           "target_frac_of_burst": 0.60,
           "breakdown_ms": {k: round(v, 4) for k, v in per.items()},
           "breakdown_sum_over_step": round(sum(per.values()) / ms, 4),
           "clocks": clocks}
    del case
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch

    world, rank, local = dist_setup(args)
    import grouped_gemm_fp32_b200 as moe
    from grouped_gemm_fp32_b200 import layer

    dev = torch.device("cuda", local)
    case = Case(args.workload, args, dev, rank)
    wl, inp, dm, dims, b = case.wl, case.inp, case.dm, case.dims, case.b
    train, gemm_only, gate_only = case.train, case.gemm_only, case.gate_only
    x, w1, w2, wg, bias, dout = case.x, case.w1, case.w2, case.wg, case.bias, case.dout
    stream = torch.cuda.Stream(device=dev)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            case.step(stream)
    stream.synchronize()
    case.check_status(stream, "after warm-up")

    # ---- timed region: device-resident inputs; the step as replayed CUDA graphs of
    # the same C-ABI calls, per-call events inside them
    use_graph = not args.eager and not (gate_only or gemm_only)
    ms, per, clocks, gap = timed_region(case, stream, args.steps, use_graph, world, dev, local)
    ms_eager = None
    if use_graph:  # the same steps as eager calls of the layer driver, for comparison
        barrier(world)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.steps):
                case.step(stream)
            e1.record(stream)
        e1.synchronize()
        ms_eager = dist_max(e0.elapsed_time(e1) / args.steps, world, dev)
    tokens_per_s = world * dm.T / (ms / 1000.0)

    pk, pk_src = peaks()
    traffic, traffic_note = gemm_traffic(args.workload)
    if gate_only:  # the gate's FP32-equivalent FLOPs, run as bf16 MMAs of exact splits
        gemm_ms = per["gate"]
        achieved = 2 * dm.T * dm.d * dm.E / (gemm_ms / 1000.0) / 1e12
        burst = pk["bf16_tflops"]
        sustained = pk.get("bf16_tflops_sustained", burst)
        gemm_detail = {"gate": {"ms": round(gemm_ms, 4), "tflops": round(achieved, 1)}}
    else:
        gemm_ms, achieved, burst, sustained, gemm_detail = gemm_roofline(case, per, pk, pk_src)

    # ---- e2e: pinned host inputs in, results out, every step, through the same
    # C-ABI calls; neighbouring steps' copies overlap compute (layer.HostPipeline)
    pinned = lambda a: torch.from_numpy(a).view(torch.bfloat16).pin_memory()
    e2e_note = "inputs H2D and results D2H every step, overlapped with neighbouring steps"
    if gate_only or gemm_only:
        hx = pinned(inp["x"])
        ho = torch.empty(dm.T, dm.d, dtype=torch.bfloat16).pin_memory()
        dx_in = torch.empty_like(x)
        h2d, d2h = hx.numel() * 2, ho.numel() * 2
        out_dev = b.y[: dm.T] if gemm_only else b.out

        def e2e_run(nsteps):
            with torch.cuda.stream(stream):
                for _ in range(nsteps):
                    dx_in.copy_(hx, non_blocking=True)
                    case.step(stream, xx=dx_in)
                    ho.copy_(out_dev, non_blocking=True)
        e2e_streams = [stream]
        e2e_note = "inputs H2D and results D2H every step, serialised with compute"
    else:
        pipe = layer.HostPipeline(dims, w1, w2, wg, bias, train, device=dev,
                                  gamma=GAMMA if train else None, graphs=not args.eager,
                                  seq_balance=SEQ_BALANCE if train else None,
                                  gather=args.gather)
        hx = [pinned(inp["x"])]
        hd = [pinned(inp["dout"])] if train else [None]
        ho = [torch.empty(dm.T, dm.d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        hdx = [torch.empty(dm.T, dm.d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        h2d = hx[0].numel() * 2 + (hd[0].numel() * 2 if train else 0)
        d2h = ho[0].numel() * 2 + (hdx[0].numel() * 2 if train else 0)

        def e2e_run(nsteps):
            pipe.run(hx, hd, ho, hdx, nsteps)
        e2e_streams = [pipe.up, pipe.compute, pipe.down]

    e2e_run(2)
    for sst in e2e_streams:
        sst.synchronize()
    barrier(world)
    ne2e = max(3, args.steps)  # steady state: the pipeline's fill and drain spread over as many
    # steps as the device-timed loop
    torch.cuda.synchronize(dev)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(e2e_streams[0])
    for sst in e2e_streams[1:]:
        sst.wait_event(f0)
    e2e_run(ne2e)
    for sst in e2e_streams[:-1]:
        ev = torch.cuda.Event()
        ev.record(sst)
        e2e_streams[-1].wait_event(ev)
    f1.record(e2e_streams[-1])
    f1.synchronize()
    e2e_ms = dist_max(f0.elapsed_time(f1) / ne2e, world, dev)
    case.check_status(stream, "after timing")

    # kernels per step: gate 2 (weight split, gate), permute 3 (histogram, groups,
    # scatter; + the row copy, which also zeroes the pad rows, without gathering), forward
    # GEMMs 2, combine 1; train adds the balance loss 2 (chunk sums, finish), combine
    # backward 1 (dY pad rows zeroed by the same launch), backward GEMMs 4, un-permute 1,
    # router backward 5 (weight split, dlogits, dX GEMM, dWg GEMM, split-K sum), bias step 1
    permute_launches = 3 if args.gather else 4
    launches_per_step = (2 if gate_only else 2 if gemm_only else
                         2 + permute_launches + 2 + 1 + ((2 + 1 + 4 + 1 + 5 + 1) if train else 0))
    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": describe(wl), "tokens_per_gpu": dm.T,
                   "global_batch_tokens": world * dm.T,
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "step": ("CUDA graph replay (one captured graph per timed step, event "
                            "nodes between its C-ABI calls)" if use_graph
                            else "eager C-ABI calls"),
                   "x_rows": ("gathered from x by sorted_ids (tile::gather4)" if args.gather
                              else "permuted copy x_perm"),
                   "seq_balance": ({"alpha": SEQ_BALANCE[0], "seq_len": SEQ_BALANCE[1]}
                                   if train else None),
                   "ms_per_step_eager": ms_eager,
                   "l2": "no flush: weights (4.5 GB) and activations exceed the 126 MB L2"},
        "roofline": {"bound": "tensor", "kernel": "ggemm_kernel (all grouped-GEMM launches)",
                     "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                     "frac": achieved / burst if burst else None,
                     "peak_kind": f"{pk_src} bf16 burst (ms-scale launches; the clocks of the "
                                  f"timed steps are in 'clocks')",
                     "frac_of_sustained_peak": achieved / sustained if sustained else None,
                     "peak_sustained": sustained,
                     "timing": "event pairs around each grouped-GEMM call inside the timed steps",
                     "traffic": traffic, "traffic_unit": "bytes per step",
                     "traffic_note": traffic_note},
        "grouped_gemm": gemm_detail,
        "breakdown_ms": {k: round(v, 4) for k, v in per.items()},
        "breakdown_sum_over_step": round(sum(per.values()) / ms, 4),
        "gap_between_steps_ms": round(gap, 4),
        "e2e": {"value": world * dm.T / (e2e_ms / 1000.0), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "note": e2e_note},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if args.workload == "train" and world == 1 and not args.no_layer:
        del pipe
        torch.cuda.empty_cache()
        line["north_star_c3"] = layer_forward_t8192(args, dev, local, pk, pk_src)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not (gemm_only or gate_only):
        line["cpu_baseline"] = cpu_baseline(wl, inp)
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_library_gemm(args, rounds=8, timed=3):
    """cuBLAS on the grouped GEMMs' shapes, for context.  Every expert gets exactly
    T*k/E rows (cuBLAS has no ragged batches), the shared experts T rows; operands are
    bf16, outputs bf16 (this library writes the dW in f32 and fuses SwiGLU and its
    backward into its epilogues, which cuBLAS does not do here).  The weights are the
    workload's own tensors, passed as (transposed) views.  Each round times every
    mode once with cuBLAS and once with this library, back to back, so both see the
    same clocks; the line reports medians over the rounds and the median of the
    per-round ratios."""
    import torch
    import grouped_gemm_fp32_b200 as moe
    from grouped_gemm_fp32_b200 import layer

    wl, inp = workload("train")
    dm = wl.dims
    T, d, E, k, S, I = dm.T, dm.d, dm.E, dm.k, dm.S, dm.I
    assert (T * k) % E == 0
    Mr = T * k // E
    dims = moe.MoeDims.of(T, d, E, k, S, I, dm.P, dm.rows_cap)
    dev = torch.device("cuda", 0)
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).to(dev)
    x, w1, w2, dout = bf(inp["x"]), bf(inp["w1"]), bf(inp["w2"]), bf(inp["dout"])
    wg, bias = torch.from_numpy(inp["wg"]).to(dev), torch.from_numpy(inp["bias"]).to(dev)
    b = layer.MoEBuffers(dims, device=dev, train=True)
    layer.forward(b, x, wg, bias, w1, w2)
    layer.backward(b, x, dout, w1, w2)
    torch.cuda.synchronize()

    g = torch.Generator(device=dev).manual_seed(11)
    rnd = lambda *s: torch.randn(*s, device=dev, generator=g).to(torch.bfloat16)
    w1r, w1s, w2r, w2s = w1[:E], w1[E:], w2[:E], w2[E:]
    ops = {  # mode: ((A, B) routed, (A, B) shared)
        "fwd1": ((rnd(E, Mr, d), w1r.transpose(1, 2)), (rnd(S, T, d), w1s.transpose(1, 2))),
        "fwd2": ((rnd(E, Mr, I), w2r.transpose(1, 2)), (rnd(S, T, I), w2s.transpose(1, 2))),
        "dx2": ((rnd(E, Mr, d), w2r), (rnd(S, T, d), w2s)),
        "dx1": ((rnd(E, Mr, 2 * I), w1r), (rnd(S, T, 2 * I), w1s)),
        "dw2": ((rnd(E, Mr, d).transpose(1, 2), rnd(E, Mr, I)),
                (rnd(S, T, d).transpose(1, 2), rnd(S, T, I))),
        "dw1": ((rnd(E, Mr, 2 * I).transpose(1, 2), rnd(E, Mr, d)),
                (rnd(S, T, 2 * I).transpose(1, 2), rnd(S, T, d))),
    }
    L = moe
    ours = {
        "fwd1+fwd2": lambda: L.grouped_gemm_fwd(dims, b.ws, b.x_perm, x, w1, w2, b.h, b.a1, b.y),
        "dx2": lambda: L.grouped_gemm_bwd_dx(dims, b.ws, L.MOE_GEMM2, b.dy, dout, w2, b.a1, b.da),
        "dw2": lambda: L.grouped_gemm_bwd_dw(dims, b.ws, L.MOE_GEMM2, b.dy, dout, b.h, None,
                                             b.dw2, 0),
        "dx1": lambda: L.grouped_gemm_bwd_dx(dims, b.ws, L.MOE_GEMM1, b.da, None, w1, None, b.dxp),
        "dw1": lambda: L.grouped_gemm_bwd_dw(dims, b.ws, L.MOE_GEMM1, b.da, None, b.x_perm, x,
                                             b.dw1, 0),
    }
    lib = {
        "fwd1+fwd2": lambda: [torch.bmm(*ops[m][j]) for m in ("fwd1", "fwd2") for j in (0, 1)],
        **{m: (lambda m=m: [torch.bmm(*ops[m][j]) for j in (0, 1)])
           for m in ("dx2", "dw2", "dx1", "dw1")},
    }
    fl = gemm_flops(dm, True)
    flops = {"fwd1+fwd2": fl["fwd"], **{m: fl[m] for m in ("dx2", "dw2", "dx1", "dw1")}}

    def t_ms(f):
        f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(timed):
            f()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1) / timed

    res = {m: {"cublas": [], "ours": []} for m in ours}
    for r in range(rounds):
        for m in ours:
            pair = [("cublas", lib[m]), ("ours", ours[m])]
            for name, f in (pair if r % 2 == 0 else pair[::-1]):
                res[m][name].append(t_ms(f))
    med = lambda v: sorted(v)[len(v) // 2]
    modes = {}
    for m, v in res.items():
        c, o = med(v["cublas"]), med(v["ours"])
        modes[m] = {"cublas_ms": round(c, 4), "ours_ms": round(o, 4),
                    "cublas_tflops": round(flops[m] / c / 1e9, 1),
                    "ours_tflops": round(flops[m] / o / 1e9, 1),
                    "ours_over_cublas_time": round(med([a / b_ for a, b_ in
                                                        zip(v["ours"], v["cublas"])]), 3)}
    line = {"library_gemm": "cuBLAS torch.bmm, bf16 in/out, f32 accumulate, uniform groups",
            "workload": f"train GEMM shapes: {E} routed experts x {Mr} rows + {S} shared x {T} "
                        f"rows, d={d}, I={I}",
            "rounds": rounds, "timed_per_round": timed, "modes": modes,
            "total_ms": {"cublas": round(sum(v["cublas_ms"] for v in modes.values()), 3),
                         "ours": round(sum(v["ours_ms"] for v in modes.values()), 3)},
            "note": "ours: ragged groups padded to 128 rows (the routing of the workload's own "
                    "batch), SwiGLU / SwiGLU-backward epilogues, saved activations, f32 dW; "
                    "cuBLAS: plain products, bf16 outputs"}
    print(json.dumps(line), flush=True)


def run_ep(args):
    """The train step under expert parallelism (grouped_gemm_fp32_b200.ep) over the ranks:
    every rank routes its own T tokens over all E experts and owns E / W of them; rows move
    by kernels writing into the other ranks' buffers (symmetric memory), with an NCCL
    all-gather of the counts and all-reduce of the loads, and no host sync, so the step is
    captured in a CUDA graph and replayed.  With one process the group has one rank (every
    peer pointer the rank's own buffer): the EP code path with no link traffic, timed
    beside the single-GPU layer step in the same process (alternating rounds, same clocks).
    A line of its own, not the contract's."""
    import torch
    import torch.distributed as dist
    import grouped_gemm_fp32_b200 as moe
    from grouped_gemm_fp32_b200 import ep, layer

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    if world == 1:
        dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                                device_id=dev)
    wl, inp = workload("train")
    inp = rank_shard(wl, inp, rank)
    dm = wl.dims
    E, El = dm.E, dm.E // world
    dims = moe.MoeDims.of(dm.T, dm.d, dm.E, dm.k, dm.S, dm.I, dm.P, dm.rows_cap)
    bf = lambda a: torch.from_numpy(a).view(torch.bfloat16).to(dev)
    x, dout = bf(inp["x"]), bf(inp["dout"])
    w1, w2 = bf(inp["w1"]), bf(inp["w2"])
    w1l = torch.cat([w1[rank * El:(rank + 1) * El], w1[E:]]).contiguous()
    w2l = torch.cat([w2[rank * El:(rank + 1) * El], w2[E:]]).contiguous()
    if world > 1:
        del w1, w2
    wg, bias = torch.from_numpy(inp["wg"]).to(dev), torch.from_numpy(inp["bias"]).to(dev)
    eb = ep.EPBuffers(dims, rank, world, train=True, device=dev,
                      alloc=ep.symmetric_alloc(world, dev))
    ep.connect(eb)
    stream = torch.cuda.Stream(device=dev)

    def step():
        ep.forward(eb, x, wg, bias, w1l, w2l, stream=stream, seq_balance=SEQ_BALANCE)
        ep.backward(eb, x, dout, w1l, w2l, stream=stream, wg=wg, gamma=GAMMA, bias=bias)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    st = ep.status(eb, stream)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {moe.moe_status_string(st)}")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    single = None
    if world == 1:  # the single-GPU layer step on the same batch, for the same-clock ratio
        b1 = layer.MoEBuffers(dims, device=dev, train=True)
        single = layer.GraphStep(b1, x, wg, bias, w1, w2, dout=dout, gamma=GAMMA,
                                 seq_balance=SEQ_BALANCE)

    def timed(replay, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(n):
                replay()
            e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / n

    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.25)
    barrier(world)
    torch.cuda.synchronize(dev)
    rounds = 4 if single is not None else 1
    per = max(1, args.steps // rounds)
    ep_ms, one_ms = [], []
    for r in range(rounds):
        pair = [("ep", lambda: graph.replay()), ("one", lambda: single.replay())]
        if single is None:
            pair = pair[:1]
        for name, f in (pair if r % 2 == 0 else pair[::-1]):
            (ep_ms if name == "ep" else one_ms).append(timed(f, per))
    barrier(world)
    clocks = clk.stop()
    st = ep.status(eb, stream)
    if st != 0:
        raise RuntimeError(f"device status after timing: {moe.moe_status_string(st)}")
    ms = dist_max(sum(ep_ms) / len(ep_ms), world, dev)
    med = lambda v: sorted(v)[len(v) // 2]
    if rank == 0:
        line = {"metric": METRIC, "value": world * dm.T / (ms / 1000.0), "unit": "tokens/s",
                "n_gpus": world, "steps": per * rounds, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "ours-ep",
                "config": {"workload": describe(wl) + ", expert parallel",
                           "parallelism": f"ep{world}", "experts_per_rank": El,
                           "tokens_per_gpu": dm.T, "seq_balance": {"alpha": SEQ_BALANCE[0],
                                                                   "seq_len": SEQ_BALANCE[1]},
                           "recv_rows_cap": eb.cap,
                           "step": "CUDA graph replay: gate, routing tables, NCCL all-gather "
                                   "of the counts, device plan, rows written into the owners' "
                                   "buffers, owners' grouped GEMMs (shared tiles first, "
                                   "a bounded wait per expert for its segments), outputs written back into "
                                   "the sources' buffers, combine; backward likewise; no "
                                   "host sync"},
                "clocks": clocks}
        if one_ms:
            line["single_gpu_step_ms"] = sum(one_ms) / len(one_ms)
            line["ep_over_single_gpu"] = med([a / b for a, b in zip(ep_ms, one_ms)])
        print(json.dumps(line), flush=True)
    del graph
    barrier(world)
    dist.destroy_process_group()


def main():
    args = parse()
    if args.ep:
        run_ep(args)
        return
    if args.library_gemm:
        run_library_gemm(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
