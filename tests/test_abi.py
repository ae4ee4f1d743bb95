"""The C-ABI library builds for sm_100a, loads, and exports every entry point
that include/moe.h declares (CPU only: no kernel is launched here).  The
host-side parts that need no GPU (row counts, workspace size, argument and
shape validation, status strings) are exercised too."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    from grouped_gemm_fp32_b200 import build
    build.build()
    import grouped_gemm_fp32_b200 as moe
    return moe


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\**([a-z_][a-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_layer_calls():
    names = declared_functions()
    for n in ("moe_gate_topk", "moe_permute_align", "grouped_gemm_fwd", "grouped_gemm_bwd_dx",
              "grouped_gemm_bwd_dw", "moe_combine", "moe_combine_bwd"):
        assert n in names


def declaration_comments():
    """Each declared function with the comment block that precedes it (a
    comment may cover several consecutive declarations)."""
    src = open(HEADER).read()
    out = {}
    last = ""
    pos = 0
    for m in re.finditer(r"/\*.*?\*/|;", src, flags=re.S):
        chunk = src[pos:m.start()]
        for n in re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\**"
                            r"([a-z_][a-z0-9_]*)\s*\(", chunk, flags=re.M):
            out[n] = last
        if m.group(0).startswith("/*"):
            last = m.group(0)
        pos = m.end()
    return out


def test_every_entry_point_cites_its_passage():
    """Every call of the layer names the passage of the pages that defines the
    operation; host-side helpers and additions say the pages have none."""
    comments = declaration_comments()
    assert set(comments) == set(declared_functions())
    for name in ("moe_gate_topk", "moe_permute_align", "grouped_gemm_fwd", "grouped_gemm_bwd_dx",
                 "grouped_gemm_bwd_dw", "moe_combine", "moe_combine_bwd", "moe_router_bwd",
                 "moe_seq_balance_loss", "moe_bias_update"):
        assert "Passage:" in comments[name], name
    for name, text in comments.items():
        flat = " ".join(re.sub(r"\n\s*\*(?!/)", " ", text).split()).lower()
        assert "passage:" in flat or "no counterpart" in flat, name


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    from grouped_gemm_fp32_b200._lib import EXPORTS
    assert set(EXPORTS) == set(declared_functions())


def test_library_is_sm100a_only(lib):
    # the fat binary holds sm_100a code (cuobjdump is not used: list the ELF sections' arch tags
    # through the build flags instead)
    from grouped_gemm_fp32_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.NVCC_FLAGS)


def test_row_counts_and_workspace(lib):
    d = lib.MoeDims.of(8192, 4096, 128, 6, 2, 1408, 128)
    assert lib.moe_rows_routed(d) == 8192 * 6 + 128 * 127
    assert lib.moe_rows_total(d) == 8192 * 6 + 128 * 127 + 2 * 8192
    assert lib.moe_workspace_size(d) >= 16 * 4 + 130 * 16
    d2 = lib.MoeDims.of(8192, 4096, 16, 1, 0, 1408, 128, 8192)
    assert lib.moe_rows_routed(d2) == 8192 and lib.moe_rows_total(d2) == 8192
    bad = lib.MoeDims.of(-1, 4096, 16, 1, 0, 1408, 128)
    assert lib.moe_rows_routed(bad) == -1 and lib.moe_workspace_size(bad) == 0


def _call(lib, name, *args):
    return getattr(lib.load(), name)(*args)


def test_validation_rejects_before_any_launch(lib):
    L = lib.load()
    ok = lib.MoeDims.of(64, 128, 8, 2, 1, 64, 16)
    nul = None
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    # unsupported shapes
    for bad in (lib.MoeDims.of(64, 100, 8, 2, 1, 64, 16),    # d % 64
                lib.MoeDims.of(64, 128, 8, 2, 1, 96, 16),    # I % 64
                lib.MoeDims.of(64, 128, 300, 2, 1, 64, 16),  # E > 256
                lib.MoeDims.of(64, 128, 8, 9, 1, 64, 16),    # k > E
                lib.MoeDims.of(64, 128, 8, 2, 1, 64, 12)):   # P % 8
        assert L.moe_combine(ctypes.byref(bad), p, p, p, p, nul) == -2
        assert L.moe_combine_f32(ctypes.byref(bad), p, p, p, p, nul) == -2
    assert L.moe_combine_f32(ctypes.byref(ok), p, p, p, nul, nul) == -1
    # split combine: the shared rows' buffer is required when S > 0
    assert L.moe_combine_split(ctypes.byref(ok), p, nul, p, p, p, nul) == -1
    assert L.moe_combine_split(ctypes.byref(ok), nul, p, p, p, p, nul) == -1
    # backward needs P % 64 == 0
    assert L.grouped_gemm_bwd_dx(ctypes.byref(ok), p, 1, p, p, p, p, p, nul) == -2
    # null pointers / bad enum / small workspace
    assert L.moe_gate_topk(ctypes.byref(ok), nul, p, p, p, p, nul, p, 1 << 30, nul) == -1
    assert L.moe_gate_topk(ctypes.byref(ok), p, p, p, p, p, nul, p, 8, nul) == -1  # small ws
    assert L.moe_gate_topk(ctypes.byref(ok), p, p, p, p, p, nul, nul, 1 << 30, nul) == -1
    assert L.moe_permute_align(ctypes.byref(ok), p, p, p, p, p, p, p, p, 8, nul) == -1
    ok64 = lib.MoeDims.of(64, 128, 8, 2, 1, 64, 64)
    assert L.grouped_gemm_bwd_dx(ctypes.byref(ok64), p, 7, p, p, p, p, p, nul) == -1
    assert L.grouped_gemm_bwd_dw(ctypes.byref(ok64), p, 2, p, p, p, p, p, 5, nul) == -1
    assert L.moe_gate_topk(None, p, p, p, p, p, nul, p, 1 << 30, nul) == -1
    # gathered-row GEMMs: sorted_ids and x are required (T > 0), dW1 needs P % 64
    assert L.grouped_gemm_fwd_gather(ctypes.byref(ok), p, nul, p, p, p, p, nul, p, nul) == -1
    assert L.grouped_gemm_fwd_gather(ctypes.byref(ok), p, p, nul, p, p, p, nul, p, nul) == -1
    assert L.grouped_gemm_fwd_gather(ctypes.byref(ok), nul, p, p, p, p, p, nul, p, nul) == -1
    assert L.grouped_gemm_bwd_dw1_gather(ctypes.byref(ok), p, p, p, p, p, 0, nul) == -2
    assert L.grouped_gemm_bwd_dw1_gather(ctypes.byref(ok64), p, nul, p, p, p, 0, nul) == -1
    assert L.grouped_gemm_bwd_dw1_gather(ctypes.byref(ok64), p, p, p, nul, p, 0, nul) == -1
    assert L.grouped_gemm_bwd_dw1_gather(ctypes.byref(ok64), p, p, p, p, p, 5, nul) == -1
    # permute without x_perm: x is optional then, but not when x_perm is given
    assert L.moe_permute_align(ctypes.byref(ok), p, nul, p, p, p, p, p, p, 8, nul) == -1  # small ws
    # router backward: workspace, pointers, shapes; bias step: pointers
    big = 1 << 40
    assert L.moe_router_bwd(ctypes.byref(ok), p, p, p, p, p, p, nul, p, p, 0, nul, big, nul) == -1
    assert L.moe_router_bwd(ctypes.byref(ok), p, p, p, p, p, p, nul, p, p, 0, p, 8, nul) == -1
    assert L.moe_router_bwd(ctypes.byref(ok), nul, p, p, p, p, p, nul, p, p, 0, p, big, nul) == -1
    assert L.moe_router_bwd(ctypes.byref(ok), p, p, p, p, p, p, nul, p, nul, 0, p, big, nul) == -1
    e12 = lib.MoeDims.of(64, 128, 12, 2, 1, 64, 16)  # E % 8
    assert L.moe_router_bwd(ctypes.byref(e12), p, p, p, p, p, p, nul, p, p, 0, p, big, nul) == -2
    # sequence-wise balance loss: seq_len >= 128, loss / seq_grad / workspace required
    f32 = ctypes.c_float(1e-4)
    assert L.moe_seq_balance_loss(ctypes.byref(ok), 64, f32, p, p, p, p, p, big, nul) == -2
    assert L.moe_seq_balance_loss(ctypes.byref(ok), 128, f32, p, p, nul, p, p, big, nul) == -1
    assert L.moe_seq_balance_loss(ctypes.byref(ok), 128, f32, p, p, p, nul, p, big, nul) == -1
    assert L.moe_seq_balance_loss(ctypes.byref(ok), 128, f32, p, p, p, p, p, 8, nul) == -1
    assert L.moe_router_bwd_seqbal(ctypes.byref(ok), p, p, p, p, p, p, nul, 128, nul, p, p, 0,
                                   p, big, nul) == -1
    assert L.moe_router_bwd_seqbal(ctypes.byref(ok), p, p, p, p, p, p, p, 100, nul, p, p, 0,
                                   p, big, nul) == -1
    assert L.moe_bias_update(None, p, 1e-3, p, p, nul) == -1
    assert L.moe_bias_update(ctypes.byref(ok), nul, 1e-3, p, p, nul) == -1
    assert L.moe_bias_update(ctypes.byref(ok), p, 1e-3, p, nul, nul) == -1


def test_status_strings(lib):
    assert lib.moe_status_string(0) == "MOE_OK"
    assert lib.moe_status_string(-4) == "MOE_ERR_DEVICE_TIMEOUT"
    assert lib.moe_status_string(-5) == "MOE_ERR_BAD_ROUTING"
    assert lib.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import grouped_gemm_fp32_b200._lib as L
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "_LIB_PATH", str(tmp_path / "libmoe.so"))
    with pytest.raises(ImportError):
        L.load()
