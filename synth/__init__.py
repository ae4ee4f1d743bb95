"""Seeded synthetic inputs for the MoE layer (shared by the oracle side and the CUDA side).

This module draws numbers; it computes nothing of the layer.  The generator is
counter-based SplitMix64 with Box-Muller normals (see ``synth.c``), so every
tensor is a pure function of ``(seed, stream id, element index)``.

Workloads follow the configurations the layer is measured on:

* ``tiny``      T=64, d=128, E=8 routed top-2, S=1 shared, I=64, pad 16, seed 0.
* ``gemm_only`` 16 groups x 512 rows, d=4096, I=1408 (grouped GEMM alone), seed 1.
* ``layer``     T=8192, d=4096, E=128 top-6, S=2, I=1408, pad 128, seed 2.
* ``skewed``    as ``layer`` with a Zipf(1.2)-shaped load bias, seed 3.
* ``train``     T=16384, rest as ``layer``, forward+backward, seed 4.
* ``train_small`` T=2048, E=16, rest as ``train`` (a small case for profiles), seed 5.

Stream ids: 1 hidden states X (or the permuted A of ``gemm_only``), 2 gate
weights Wg, 3 selection bias, 4 W1 (gate|up), 5 W2 (down), 6 upstream grad.
Biases that must be *fitted* to a load shape (``skewed``, ``train``) are not
drawn here: they are stored fixtures written by a script that uses the oracle
router; ``bias_override`` lets the caller pass them in.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

SID_X, SID_WG, SID_BIAS, SID_W1, SID_W2, SID_DOUT = 1, 2, 3, 4, 5, 6


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O3", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.synth_raw.restype = u64
        lib.synth_raw.argtypes = [u64, u64, u64]
        for name in ("synth_normal_bf16", "synth_normal_f32", "synth_uniform_f32"):
            getattr(lib, name).restype = None
            getattr(lib, name).argtypes = [u64, u64, i64, dbl, dbl, vp]
        lib.synth_uniform_int.restype = None
        lib.synth_uniform_int.argtypes = [u64, u64, i64, i64, vp]
        _lib = lib
    return _lib


def raw(seed: int, sid: int, i: int) -> int:
    return int(_load().synth_raw(seed, sid, i))


def normal_bf16(seed: int, sid: int, shape, std: float, mean: float = 0.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(mean, std^2) samples."""
    out = np.empty(shape, dtype=np.uint16)
    _load().synth_normal_bf16(seed, sid, out.size, mean, std, out.ctypes.data)
    return out


def normal_f32(seed: int, sid: int, shape, std: float, mean: float = 0.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _load().synth_normal_f32(seed, sid, out.size, mean, std, out.ctypes.data)
    return out


def uniform_f32(seed: int, sid: int, shape, lo: float, hi: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _load().synth_uniform_f32(seed, sid, out.size, lo, hi, out.ctypes.data)
    return out


def uniform_int(seed: int, sid: int, n: int, m: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    _load().synth_uniform_int(seed, sid, n, m, out.ctypes.data)
    return out


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (no arithmetic, a bit shift)."""
    return (h.astype(np.uint32) << 16).view(np.float32)


@dataclass
class Dims:
    """Shapes of one MoE layer.  ``rows_cap`` = rows of the permuted buffers
    (0 means the worst case T*k + E*(P-1))."""
    T: int
    d: int
    E: int
    k: int
    S: int
    I: int
    P: int
    rows_cap: int = 0

    @property
    def G(self) -> int:
        return self.E + self.S

    def routed_cap(self) -> int:
        return self.rows_cap if self.rows_cap else self.T * self.k + self.E * (self.P - 1)

    def total_cap(self) -> int:
        return self.routed_cap() + self.S * self.T


@dataclass
class Workload:
    name: str
    dims: Dims
    seed: int
    x_std: float = 1.0
    w1_std: float = 0.02
    w2_std: float = 0.02
    wg_std: float = 0.02
    bias_lo: float = -0.01
    bias_hi: float = 0.01
    backward: bool = False
    group_rows: list | None = None     # gemm_only: fixed rows per group
    notes: str = ""
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny": Workload("tiny", Dims(T=64, d=128, E=8, k=2, S=1, I=64, P=16), seed=0),
    "gemm_only": Workload("gemm_only", Dims(T=8192, d=4096, E=16, k=1, S=0, I=1408, P=128,
                                            rows_cap=8192),
                          seed=1, w1_std=1.0 / 64.0, w2_std=1.0 / float(np.sqrt(1408.0)),
                          group_rows=[512] * 16),
    "layer": Workload("layer", Dims(T=8192, d=4096, E=128, k=6, S=2, I=1408, P=128), seed=2),
    "skewed": Workload("skewed", Dims(T=8192, d=4096, E=128, k=6, S=2, I=1408, P=128), seed=3),
    "train": Workload("train", Dims(T=16384, d=4096, E=128, k=6, S=2, I=1408, P=128), seed=4,
                      backward=True),
    # profiling stand-in for ``train``: the same ~768 rows per routed expert and
    # the same d, I, k, P, with 16 experts so a capture holds ~2.5 GB
    "train_small": Workload("train_small", Dims(T=2048, d=4096, E=16, k=6, S=2, I=1408, P=128),
                            seed=5, backward=True),
}


def make_inputs(wl: Workload, *, with_weights: bool = True, bias_override=None) -> dict:
    """Host numpy arrays of one workload.  bf16 tensors are uint16 bit patterns.

    Keys: x [T,d] bf16, wg [E,d] f32, bias [E] f32, w1 [G,2I,d] bf16,
    w2 [G,d,I] bf16, dout [T,d] bf16 (backward workloads only).
    """
    dm, s = wl.dims, wl.seed
    out = {"x": normal_bf16(s, SID_X, (dm.T, dm.d), wl.x_std)}
    if wl.group_rows is None:
        out["wg"] = normal_f32(s, SID_WG, (dm.E, dm.d), wl.wg_std)
        out["bias"] = (np.asarray(bias_override, dtype=np.float32) if bias_override is not None
                       else uniform_f32(s, SID_BIAS, (dm.E,), wl.bias_lo, wl.bias_hi))
    if with_weights:
        out["w1"] = normal_bf16(s, SID_W1, (dm.G, 2 * dm.I, dm.d), wl.w1_std)
        out["w2"] = normal_bf16(s, SID_W2, (dm.G, dm.d, dm.I), wl.w2_std)
    if wl.backward:
        out["dout"] = normal_bf16(s, SID_DOUT, (dm.T, dm.d), 1.0)
    return out
