"""ctypes binding of libmoe.so: one Python function per C entry point, same name.

Arguments are torch CUDA tensors (their ``data_ptr()`` is passed), ``None``
(NULL) or plain integers.  ``stream`` defaults to torch's current stream.  A
negative status raises ``MoeError``.  Nothing here computes anything.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIB_DEBUG=1 loads the debug build (libmoe_debug.so: device-side checks of the
# group table and tile coordinates, MOE_ERR_BAD_ROUTING instead of a bad access)
_LIB_PATH = os.path.join(_HERE, "libmoe_debug.so" if os.environ.get("MOE_LIB_DEBUG") == "1"
                         else "libmoe.so")
_lib = None

MOE_GEMM1, MOE_GEMM2 = 1, 2
EXPORTS = (
    "moe_rows_routed", "moe_rows_total", "moe_workspace_size", "moe_gate_topk",
    "moe_permute_align", "moe_permute_align_static", "grouped_gemm_set_groups",
    "grouped_gemm_fwd", "grouped_gemm_fwd_gather", "grouped_gemm_bwd_dx", "grouped_gemm_bwd_dw",
    "grouped_gemm_bwd_dw1_gather", "moe_combine", "moe_combine_split", "moe_combine_f32",
    "moe_combine_bwd", "moe_router_bwd", "moe_router_bwd_seqbal", "moe_seq_balance_loss",
    "moe_bias_update", "moe_get_device_status",
    "moe_status_string", "moe_last_cuda_error",
    "moe_ep_workspace_size", "moe_ep_plan", "moe_ep_dispatch", "moe_ep_zero_pads", "moe_ep_wait",
    "moe_ep_combine_bwd", "grouped_gemm_fwd_ep", "grouped_gemm_bwd_dx_ep",
)
MOE_EP_MAX_WORLD = 8
MOE_EP_WAIT_Y, MOE_EP_WAIT_DX = 3, 5


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = f"{what} failed: {moe_status_string(status)} ({status})"
        if status == -3:
            msg += f": {moe_last_cuda_error()}"
        super().__init__(msg)
        self.status = status


class MoeDims(ctypes.Structure):
    """Mirror of ``struct moe_dims`` in include/moe.h."""
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("S", ctypes.c_int32), ("I", ctypes.c_int32),
                ("P", ctypes.c_int32), ("rows_cap", ctypes.c_int64)]

    @classmethod
    def of(cls, T, d, E, k, S, I, P, rows_cap=0):
        return cls(int(T), int(d), int(E), int(k), int(S), int(I), int(P), int(rows_cap))

    def __repr__(self):
        return ("MoeDims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")")


class MoeEpPeers(ctypes.Structure):
    """Mirror of ``struct moe_ep_peers`` in include/moe.h: this rank, the world, and
    every rank's EP workspace and destination rows as device addresses mapped in
    this process."""
    _fields_ = [("rank", ctypes.c_int32), ("world", ctypes.c_int32),
                ("rows_cap", ctypes.c_int64),
                ("ep_ws", ctypes.c_void_p * MOE_EP_MAX_WORLD),
                ("rows", ctypes.c_void_p * MOE_EP_MAX_WORLD)]

    @classmethod
    def of(cls, rank, world, ep_ws, rows=None, rows_cap=0):
        """``ep_ws`` / ``rows``: per-rank device addresses (ints) or tensors."""
        p = cls()
        p.rank, p.world, p.rows_cap = int(rank), int(world), int(rows_cap)
        for o in range(world):
            p.ep_ws[o] = _p(ep_ws[o])
            p.rows[o] = _p(rows[o]) if rows is not None else None
        return p


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load libmoe.so (built in-tree by ``grouped_gemm_fp32_b200.build``); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m grouped_gemm_fp32_b200.build` (there is no fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    D = ctypes.POINTER(MoeDims)
    sig = {
        "moe_rows_routed": (i64, [D]),
        "moe_rows_total": (i64, [D]),
        "moe_workspace_size": (sz, [D]),
        "moe_gate_topk": (i32, [D, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "moe_permute_align": (i32, [D, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "moe_permute_align_static": (i32, [D, vp, vp, vp, vp, vp, vp, vp, vp]),
        "grouped_gemm_set_groups": (i32, [D, vp, vp, vp, sz, vp]),
        "grouped_gemm_fwd": (i32, [D, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "grouped_gemm_fwd_gather": (i32, [D, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "grouped_gemm_bwd_dx": (i32, [D, vp, i32, vp, vp, vp, vp, vp, vp]),
        "grouped_gemm_bwd_dw1_gather": (i32, [D, vp, vp, vp, vp, vp, i32, vp]),
        "grouped_gemm_bwd_dw": (i32, [D, vp, i32, vp, vp, vp, vp, vp, i32, vp]),
        "moe_combine": (i32, [D, vp, vp, vp, vp, vp]),
        "moe_combine_f32": (i32, [D, vp, vp, vp, vp, vp]),
        "moe_combine_split": (i32, [D, vp, vp, vp, vp, vp, vp]),
        "moe_router_bwd": (i32, [D, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]),
        "moe_router_bwd_seqbal": (i32, [D, vp, vp, vp, vp, vp, vp, vp, i64, vp, vp, vp, i32, vp,
                                        sz, vp]),
        "moe_seq_balance_loss": (i32, [D, i64, ctypes.c_float, vp, vp, vp, vp, vp, sz, vp]),
        "moe_bias_update": (i32, [D, vp, ctypes.c_float, vp, vp, vp]),
        "moe_combine_bwd": (i32, [D, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_get_device_status": (i32, [vp, vp, vp]),
        "moe_ep_workspace_size": (sz, [D, i32]),
        "moe_ep_plan": (i32, [D, ctypes.POINTER(MoeEpPeers), vp, vp, i64, vp]),
        "moe_ep_dispatch": (i32, [D, ctypes.POINTER(MoeEpPeers), vp, vp, vp, vp]),
        "moe_ep_zero_pads": (i32, [D, ctypes.POINTER(MoeEpPeers), vp, vp]),
        "moe_ep_wait": (i32, [ctypes.POINTER(MoeEpPeers), i32, vp]),
        "moe_ep_combine_bwd": (i32, [D, ctypes.POINTER(MoeEpPeers), vp, vp, vp, vp, vp, vp, vp,
                                     vp]),
        "grouped_gemm_fwd_ep": (i32, [D, vp, ctypes.POINTER(MoeEpPeers), vp, vp, vp, vp, vp, vp,
                                      vp, vp]),
        "grouped_gemm_bwd_dx_ep": (i32, [D, vp, ctypes.POINTER(MoeEpPeers), i32, vp, vp, vp, vp,
                                         vp, vp]),
        "moe_status_string": (ctypes.c_char_p, [i32]),
        "moe_last_cuda_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _p(t):
    """Device pointer of a tensor (or an int address), NULL for None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ck(rc: int, what: str):
    if rc != 0:
        raise MoeError(rc, what)


def moe_status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


def moe_last_cuda_error() -> str:
    return load().moe_last_cuda_error().decode()


def moe_rows_routed(dims: MoeDims) -> int:
    return int(load().moe_rows_routed(ctypes.byref(dims)))


def moe_rows_total(dims: MoeDims) -> int:
    return int(load().moe_rows_total(ctypes.byref(dims)))


def moe_workspace_size(dims: MoeDims) -> int:
    return int(load().moe_workspace_size(ctypes.byref(dims)))


def moe_gate_topk(dims, x, wg, bias, topk_idx, topk_w, probs, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _ck(load().moe_gate_topk(ctypes.byref(dims), _p(x), _p(wg), _p(bias), _p(topk_idx),
                             _p(topk_w), _p(probs), _p(ws), nbytes, _s(stream)),
        "moe_gate_topk")


def moe_permute_align(dims, topk_idx, x, counts, offsets, sorted_ids, row_of, x_perm, ws,
                      stream=None):
    nbytes = ws.numel() * ws.element_size()
    _ck(load().moe_permute_align(ctypes.byref(dims), _p(topk_idx), _p(x), _p(counts),
                                 _p(offsets), _p(sorted_ids), _p(row_of), _p(x_perm), _p(ws),
                                 nbytes, _s(stream)), "moe_permute_align")


def moe_permute_align_static(dims, topk_idx, x, counts, offsets, sorted_ids, row_of, x_perm,
                             stream=None):
    """moe_permute_align for callers that cannot allocate: no workspace argument."""
    _ck(load().moe_permute_align_static(ctypes.byref(dims), _p(topk_idx), _p(x), _p(counts),
                                        _p(offsets), _p(sorted_ids), _p(row_of), _p(x_perm),
                                        _s(stream)), "moe_permute_align_static")


def grouped_gemm_set_groups(dims, counts, offsets, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _ck(load().grouped_gemm_set_groups(ctypes.byref(dims), _p(counts), _p(offsets), _p(ws),
                                       nbytes, _s(stream)), "grouped_gemm_set_groups")


def grouped_gemm_fwd(dims, ws, x_perm, x, w1, w2, h, a1, y, stream=None):
    _ck(load().grouped_gemm_fwd(ctypes.byref(dims), _p(ws), _p(x_perm), _p(x), _p(w1), _p(w2),
                                _p(h), _p(a1), _p(y), _s(stream)), "grouped_gemm_fwd")


def grouped_gemm_fwd_gather(dims, ws, sorted_ids, x, w1, w2, h, a1, y, stream=None):
    _ck(load().grouped_gemm_fwd_gather(ctypes.byref(dims), _p(ws), _p(sorted_ids), _p(x), _p(w1),
                                       _p(w2), _p(h), _p(a1), _p(y), _s(stream)),
        "grouped_gemm_fwd_gather")


def grouped_gemm_bwd_dx(dims, ws, which, dy_routed, dy_shared, w, a1, out, stream=None):
    _ck(load().grouped_gemm_bwd_dx(ctypes.byref(dims), _p(ws), int(which), _p(dy_routed),
                                   _p(dy_shared), _p(w), _p(a1), _p(out), _s(stream)),
        "grouped_gemm_bwd_dx")


def grouped_gemm_bwd_dw(dims, ws, which, lhs_routed, lhs_shared, rhs_routed, rhs_shared, dw,
                        accumulate=0, stream=None):
    _ck(load().grouped_gemm_bwd_dw(ctypes.byref(dims), _p(ws), int(which), _p(lhs_routed),
                                   _p(lhs_shared), _p(rhs_routed), _p(rhs_shared), _p(dw),
                                   int(accumulate), _s(stream)), "grouped_gemm_bwd_dw")


def grouped_gemm_bwd_dw1_gather(dims, ws, sorted_ids, da, x, dw1, accumulate=0, stream=None):
    _ck(load().grouped_gemm_bwd_dw1_gather(ctypes.byref(dims), _p(ws), _p(sorted_ids), _p(da),
                                           _p(x), _p(dw1), int(accumulate), _s(stream)),
        "grouped_gemm_bwd_dw1_gather")


def moe_combine(dims, y, row_of, topk_w, out, stream=None):
    _ck(load().moe_combine(ctypes.byref(dims), _p(y), _p(row_of), _p(topk_w), _p(out),
                           _s(stream)), "moe_combine")


def moe_combine_split(dims, y_routed, y_shared, row_of, topk_w, out, stream=None):
    _ck(load().moe_combine_split(ctypes.byref(dims), _p(y_routed), _p(y_shared), _p(row_of),
                                 _p(topk_w), _p(out), _s(stream)), "moe_combine_split")


def moe_combine_f32(dims, y, row_of, topk_w, out, stream=None):
    _ck(load().moe_combine_f32(ctypes.byref(dims), _p(y), _p(row_of), _p(topk_w), _p(out),
                               _s(stream)), "moe_combine_f32")


def moe_combine_bwd(dims, ws, dout, y, row_of, topk_w, dy_routed, dw, stream=None):
    _ck(load().moe_combine_bwd(ctypes.byref(dims), _p(ws), _p(dout), _p(y), _p(row_of),
                               _p(topk_w), _p(dy_routed), _p(dw), _s(stream)), "moe_combine_bwd")


def moe_router_bwd(dims, x, wg, probs, topk_idx, topk_w, dw, dlogits, dx, dwg, accumulate, ws,
                   stream=None):
    nbytes = ws.numel() * ws.element_size()
    _ck(load().moe_router_bwd(ctypes.byref(dims), _p(x), _p(wg), _p(probs), _p(topk_idx),
                              _p(topk_w), _p(dw), _p(dlogits), _p(dx), _p(dwg), int(accumulate),
                              _p(ws), nbytes, _s(stream)), "moe_router_bwd")


def moe_router_bwd_seqbal(dims, x, wg, probs, topk_idx, topk_w, dw, seq_grad, seq_len, dlogits,
                          dx, dwg, accumulate, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _ck(load().moe_router_bwd_seqbal(ctypes.byref(dims), _p(x), _p(wg), _p(probs), _p(topk_idx),
                                     _p(topk_w), _p(dw), _p(seq_grad), int(seq_len),
                                     _p(dlogits), _p(dx), _p(dwg), int(accumulate), _p(ws),
                                     nbytes, _s(stream)), "moe_router_bwd_seqbal")


def moe_seq_balance_loss(dims, seq_len, alpha, topk_idx, probs, loss, seq_grad, ws, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _ck(load().moe_seq_balance_loss(ctypes.byref(dims), int(seq_len), float(alpha),
                                    _p(topk_idx), _p(probs), _p(loss), _p(seq_grad), _p(ws),
                                    nbytes, _s(stream)), "moe_seq_balance_loss")


def moe_bias_update(dims, counts, gamma, bias_in, bias_out, stream=None):
    _ck(load().moe_bias_update(ctypes.byref(dims), _p(counts), float(gamma), _p(bias_in),
                               _p(bias_out), _s(stream)), "moe_bias_update")


def moe_get_device_status(ws, stream=None) -> int:
    out = ctypes.c_int32(0)
    _ck(load().moe_get_device_status(_p(ws), ctypes.addressof(out), _s(stream)),
        "moe_get_device_status")
    return int(out.value)


# ------------------------------------------------------ expert parallelism --
def moe_ep_workspace_size(dims, world) -> int:
    return int(load().moe_ep_workspace_size(ctypes.byref(dims), int(world)))


def moe_ep_plan(dims, peers, counts_all, counts_loc, recv_cap, stream=None):
    _ck(load().moe_ep_plan(ctypes.byref(dims), ctypes.byref(peers), _p(counts_all),
                           _p(counts_loc), int(recv_cap), _s(stream)), "moe_ep_plan")


def moe_ep_dispatch(dims, peers, sorted_ids, offsets, x, stream=None):
    _ck(load().moe_ep_dispatch(ctypes.byref(dims), ctypes.byref(peers), _p(sorted_ids),
                               _p(offsets), _p(x), _s(stream)), "moe_ep_dispatch")


def moe_ep_zero_pads(dims, peers, recv, stream=None):
    _ck(load().moe_ep_zero_pads(ctypes.byref(dims), ctypes.byref(peers), _p(recv), _s(stream)),
        "moe_ep_zero_pads")


def moe_ep_wait(peers, which, stream=None):
    _ck(load().moe_ep_wait(ctypes.byref(peers), int(which), _s(stream)), "moe_ep_wait")


def moe_ep_combine_bwd(dims, peers, dout, y, row_of, topk_w, topk_idx, offsets, dw, stream=None):
    _ck(load().moe_ep_combine_bwd(ctypes.byref(dims), ctypes.byref(peers), _p(dout), _p(y),
                                  _p(row_of), _p(topk_w), _p(topk_idx), _p(offsets), _p(dw),
                                  _s(stream)), "moe_ep_combine_bwd")


def grouped_gemm_fwd_ep(dims, ws, peers, x_recv, x, w1, w2, h, a1, y, stream=None):
    _ck(load().grouped_gemm_fwd_ep(ctypes.byref(dims), _p(ws), ctypes.byref(peers), _p(x_recv),
                                   _p(x), _p(w1), _p(w2), _p(h), _p(a1), _p(y), _s(stream)),
        "grouped_gemm_fwd_ep")


def grouped_gemm_bwd_dx_ep(dims, ws, peers, which, dy_recv, dy_shared, w, a1, out, stream=None):
    _ck(load().grouped_gemm_bwd_dx_ep(ctypes.byref(dims), _p(ws), ctypes.byref(peers), int(which),
                                      _p(dy_recv), _p(dy_shared), _p(w), _p(a1), _p(out),
                                      _s(stream)), "grouped_gemm_bwd_dx_ep")
