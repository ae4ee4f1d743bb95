"""Oracle: plain FP64 CPU statement of the dots.llm1 MoE layer (test infrastructure).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library never loads it, and it shares no code with the CUDA path.

The arithmetic lives in ``moe_oracle.cpp`` (C++17, OpenMP, double
accumulation); this file only compiles it and marshals numpy arrays.  Each
function cites the passage of the dots.llm1 Technical Report it follows:

* ``gate_logits``  -- §Architecture "Mixture of Experts layer": the gating layer
  is computed in FP32 (here: in FP64, exact products of the widened inputs).
* ``route``        -- §Architecture "Load balancing": the per-expert bias is added
  to the affinity scores only to choose the top-k experts.
* ``permute``      -- §3.2 "Efficient implementation of Grouped GEMM": each
  expert's segment M_i is padded to a fixed block; §"Load balancing": no token
  is dropped.
* ``expert_fwd`` / ``layer_fwd`` -- §"Mixture of Experts layer": fine-grained
  two-layer SwiGLU experts, 6 routed + 2 shared per token.
* ``layer_bwd`` / ``group_dw``   -- the exact gradient of ``layer_fwd``
  (bf16 storage points treated as the identity).
* ``router_bwd``   -- the gradient of the combine weights (the chosen experts'
  affinities, §"Mixture of Experts layer") through the renormalisation and
  the softmax, into the gate's input and weights.
* ``bias_update``  -- §"Load balancing": the bias is adjusted during training
  to keep the loads balanced (sign step towards the mean load).
* ``seq_balance``  -- §"Load balancing": the sequence-wise balance loss the
  pages add without a formula, read as the one in the report they cite for
  their method (DeepSeek-V3), with softmax affinities; value and gradient.

Pins (what this oracle is checked against, other than itself) live in
``tests/test_oracle_*.py``.  Parity of every function here is pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (g++, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O3", "-std=c++17", "-fPIC", "-shared", "-fopenmp",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _p(a):
    return a.ctypes.data if a is not None else None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i32, i64, vp, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
        lib.oracle_num_threads.restype = i32
        lib.oracle_round_bf16.restype = dbl
        lib.oracle_round_bf16.argtypes = [dbl]
        lib.oracle_gate_logits.argtypes = [vp, vp, i64, i32, i32, vp]
        lib.oracle_route.argtypes = [vp, vp, i64, i32, i32, vp, vp, vp, vp]
        lib.oracle_router_bwd.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, vp, vp, vp, vp]
        lib.oracle_seq_balance.restype = dbl
        lib.oracle_seq_balance.argtypes = [vp, vp, i64, i32, i32, i64, dbl, vp]
        lib.oracle_bias_update.argtypes = [vp, i64, i32, i32, vp, ctypes.c_float, vp]
        lib.oracle_permute.restype = i64
        lib.oracle_permute.argtypes = [vp, i64, i32, i32, i32, i64, vp, vp, vp, vp]
        for sfx in ("_bf16", "_f64"):
            getattr(lib, "oracle_expert_fwd" + sfx).argtypes = [vp, i64, vp, vp, i32, i32, i32,
                                                                vp, vp, vp, vp]
            getattr(lib, "oracle_layer_fwd" + sfx).argtypes = [vp, vp, vp, vp, vp, i32, i32, i32,
                                                               i32, i32, vp, i64, i32, vp, vp, vp]
            getattr(lib, "oracle_layer_bwd" + sfx).argtypes = [vp, vp, vp, vp, vp, vp, i32, i32,
                                                               i32, i32, i32, vp, i64, i32, vp,
                                                               vp]
            getattr(lib, "oracle_group_dw" + sfx).argtypes = [vp, vp, vp, vp, vp, vp, i64, i32,
                                                              i32, i32, i32, i32, i32, vp, i32,
                                                              vp, i32, vp, vp]
        _lib = lib
    return _lib


def _kind(*arrays):
    """'_bf16' when the float inputs are bf16 bit patterns (uint16), '_f64' when double."""
    dts = {np.asarray(a).dtype for a in arrays}
    if dts == {np.dtype(np.uint16)}:
        return "_bf16", np.uint16
    if dts <= {np.dtype(np.float64)}:
        return "_f64", np.float64
    raise TypeError(f"inputs must all be bf16 bits (uint16) or all float64, got {dts}")


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def round_bf16(v: float) -> float:
    return float(_load().oracle_round_bf16(float(v)))


def gate_logits(x: np.ndarray, wg: np.ndarray) -> np.ndarray:
    """logit[t, e] = sum_j X[t, j] Wg[e, j] in FP64.  x: bf16 bits [T, d]; wg: f32 [E, d]."""
    x, wg = _c(x, np.uint16), _c(wg, np.float32)
    T, d = x.shape
    E = wg.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    _load().oracle_gate_logits(_p(x), _p(wg), T, d, E, _p(out))
    return out


def route(logits: np.ndarray, bias: np.ndarray, k: int):
    """Softmax affinities, biased top-k selection, renormalised weights.

    Returns (probs [T,E] f64, idx [T,k] i32, w [T,k] f64, margin [T] f64).
    """
    logits, bias = _c(logits, np.float64), _c(bias, np.float32)
    T, E = logits.shape
    probs = np.empty((T, E), dtype=np.float64)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    margin = np.empty((T,), dtype=np.float64)
    _load().oracle_route(_p(logits), _p(bias), T, E, k, _p(probs), _p(idx), _p(w), _p(margin))
    return probs, idx, w, margin


def router_bwd(x: np.ndarray, wg: np.ndarray, idx: np.ndarray, dw: np.ndarray,
               want_dx: bool = True, want_dwg: bool = True, dl_extra=None):
    """Gradient of the combine weights through the renormalisation and the softmax:
    (dlogits [T,E], dx [T,d], dwg [E,d]), all FP64 (dx / dwg None when not wanted).
    x: bf16 bits [T,d]; wg: f32 [E,d]; idx [T,k] the chosen experts; dw [T,k] = dL/dw.
    dl_extra [T,E] (optional): a further dL/dlogit term (``seq_balance``'s) added to
    dlogits before dx and dwg are formed."""
    x, wg, idx, dw = _c(x, np.uint16), _c(wg, np.float32), _c(idx, np.int32), _c(dw, np.float64)
    T, d = x.shape
    E = wg.shape[0]
    k = idx.shape[1]
    extra = None if dl_extra is None else _c(dl_extra, np.float64)
    dl = np.empty((T, E))
    dx = np.empty((T, d)) if want_dx else None
    dwg = np.empty((E, d)) if want_dwg else None
    _load().oracle_router_bwd(_p(x), _p(wg), _p(idx), _p(dw), T, d, E, k, _p(extra), _p(dl),
                              _p(dx), _p(dwg))
    return dl, dx, dwg


def seq_balance(logits: np.ndarray, idx: np.ndarray, seq_len: int, alpha: float,
                want_grad: bool = True):
    """Sequence-wise balance loss (mean over the batch's sequences of seq_len
    tokens) and its gradient dL/dlogit [T,E] (FP64; None when not wanted)."""
    logits, idx = _c(logits, np.float64), _c(idx, np.int32)
    T, E = logits.shape
    k = idx.shape[1]
    dl = np.empty((T, E)) if want_grad else None
    loss = _load().oracle_seq_balance(_p(logits), _p(idx), T, E, k, int(seq_len), float(alpha),
                                      _p(dl))
    return float(loss), dl


def bias_update(idx: np.ndarray, E: int, bias: np.ndarray, gamma: float) -> np.ndarray:
    """One aux-loss-free bias step: bias_e + gamma * sign(T k / E - load_e), FP64."""
    idx, bias = _c(idx, np.int32), _c(bias, np.float32)
    T, k = idx.shape
    out = np.empty(E)
    _load().oracle_bias_update(_p(idx), T, E, k, _p(bias), float(gamma), _p(out))
    return out


def permute(idx: np.ndarray, E: int, P: int, rows_cap: int):
    """Padded, stable per-expert segments.  Returns dict with counts [E],
    offsets [E+1], sorted_ids [rows_cap] (-1 on pad rows), row_of [T,k], total."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    sorted_ids = np.empty(rows_cap, dtype=np.int32)
    row_of = np.empty((T, k), dtype=np.int32)
    total = _load().oracle_permute(_p(idx), T, E, k, P, rows_cap, _p(counts), _p(offsets),
                                   _p(sorted_ids), _p(row_of))
    if total < 0:
        raise ValueError("padded total exceeds rows_cap")
    return {"counts": counts, "offsets": offsets, "sorted_ids": sorted_ids, "row_of": row_of,
            "total": int(total)}


def expert_fwd(a: np.ndarray, w1g: np.ndarray, w2g: np.ndarray, rnd: bool = True):
    """One expert on rows a [M, d].  Returns G, U, H [M, I] and Y [M, d] (f64)."""
    sfx, dt = _kind(a, w1g, w2g)
    a, w1g, w2g = _c(a, dt), _c(w1g, dt), _c(w2g, dt)
    M, d = a.shape
    I = w2g.shape[1]
    g = np.empty((M, I)); u = np.empty((M, I)); h = np.empty((M, I)); y = np.empty((M, d))
    getattr(_load(), "oracle_expert_fwd" + sfx)(_p(a), M, _p(w1g), _p(w2g), d, I, int(rnd),
                                                 _p(g), _p(u), _p(h), _p(y))
    return g, u, h, y


def layer_fwd(x, idx, w, w1, w2, S: int, tokens=None, rnd: bool = True, want_y: bool = False):
    """out[t] = sum_j w[t,j] Y_{idx[t,j]}(x_t) + sum_s Y_{E+s}(x_t) for the listed tokens.

    Returns out [n, d] (and y_routed [n,k,d], y_shared [n,S,d] when ``want_y``).
    """
    sfx, dt = _kind(x, w1, w2)
    x, w1, w2 = _c(x, dt), _c(w1, dt), _c(w2, dt)
    idx, w = _c(idx, np.int32), _c(w, np.float64)
    T, d = x.shape
    k = idx.shape[1]
    G, I2, _ = w1.shape
    E, I = G - S, I2 // 2
    tokens = np.arange(T, dtype=np.int64) if tokens is None else _c(tokens, np.int64)
    n = tokens.shape[0]
    out = np.empty((n, d))
    yr = np.empty((n, k, d)) if want_y else None
    ys = np.empty((n, max(S, 1), d)) if want_y else None
    getattr(_load(), "oracle_layer_fwd" + sfx)(_p(x), _p(idx), _p(w), _p(w1), _p(w2), d, E, k,
                                                S, I, _p(tokens), n, int(rnd), _p(out), _p(yr),
                                                _p(ys))
    return (out, yr, ys) if want_y else out


def layer_bwd(x, idx, w, w1, w2, dout, S: int, tokens=None, rnd: bool = True):
    """Gradients for the listed tokens: dx [n, d] (through the experts) and dw [n, k]."""
    sfx, dt = _kind(x, w1, w2, dout)
    x, w1, w2, dout = _c(x, dt), _c(w1, dt), _c(w2, dt), _c(dout, dt)
    idx, w = _c(idx, np.int32), _c(w, np.float64)
    T, d = x.shape
    k = idx.shape[1]
    G, I2, _ = w1.shape
    E, I = G - S, I2 // 2
    tokens = np.arange(T, dtype=np.int64) if tokens is None else _c(tokens, np.int64)
    n = tokens.shape[0]
    dx = np.empty((n, d))
    dw = np.empty((n, k))
    getattr(_load(), "oracle_layer_bwd" + sfx)(_p(x), _p(idx), _p(w), _p(w1), _p(w2), _p(dout),
                                                d, E, k, S, I, _p(tokens), n, int(rnd), _p(dx),
                                                _p(dw))
    return dx, dw


def group_dw(x, idx, w, w1, w2, dout, S: int, grp: int, w1_rows=None, w2_cols=None,
             rnd: bool = True):
    """Selected entries of dW1_grp (rows of [2I, d]) and dW2_grp (columns of [d, I]).

    Defaults select everything.  Returns (dw1 [n1, d], dw2 [d, n2]).
    """
    sfx, dt = _kind(x, w1, w2, dout)
    x, w1, w2, dout = _c(x, dt), _c(w1, dt), _c(w2, dt), _c(dout, dt)
    idx, w = _c(idx, np.int32), _c(w, np.float64)
    T, d = x.shape
    k = idx.shape[1]
    G, I2, _ = w1.shape
    E, I = G - S, I2 // 2
    r1 = _c(np.arange(2 * I) if w1_rows is None else w1_rows, np.int32)
    c2 = _c(np.arange(I) if w2_cols is None else w2_cols, np.int32)
    dw1 = np.empty((r1.shape[0], d))
    dw2 = np.empty((d, c2.shape[0]))
    getattr(_load(), "oracle_group_dw" + sfx)(_p(x), _p(idx), _p(w), _p(w1), _p(w2), _p(dout),
                                               T, d, E, k, I, grp, int(rnd), _p(r1),
                                               r1.shape[0], _p(c2), c2.shape[0], _p(dw1),
                                               _p(dw2))
    return dw1, dw2
