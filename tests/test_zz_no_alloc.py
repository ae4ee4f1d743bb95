"""moe_permute_align_static: the permutation for callers that cannot allocate.

Such callers (code inside a framework whose allocator owns all device memory,
foreign-function callers that pass only inputs and outputs, paths where
cudaMalloc is not allowed) get the permutation without a workspace argument;
the scratch sits in a fixed device array inside the library.  This checks,
through the C ABI, that its outputs equal moe_permute_align's (integer and
copied rows: bit for bit) on two calls in a row with different routings, so
nothing left in the shared array by one call leaks into the next.

The file name sorts last so that a run stopping at the first failure has run
every other test first.
"""
import numpy as np
import pytest
import torch

import grouped_gemm_fp32_b200 as moe
import synth

pytestmark = pytest.mark.gpu


def _outputs(dm):
    E, k, d, T = dm.E, dm.k, dm.d, dm.T
    Rr = moe.moe_rows_routed(dm)
    return dict(counts=torch.full((E,), -9, dtype=torch.int32, device="cuda"),
                offsets=torch.full((E + 1,), -9, dtype=torch.int32, device="cuda"),
                sorted_ids=torch.full((Rr,), -9, dtype=torch.int32, device="cuda"),
                row_of=torch.full((T, k), -9, dtype=torch.int32, device="cuda"),
                x_perm=torch.zeros(Rr, d, dtype=torch.bfloat16, device="cuda"))


def _case(seed, T, d, E, k, P, S=2):
    rng = np.random.default_rng(seed)
    # k distinct experts per token: the first k of a random order of all E
    idx = np.argsort(rng.random((T, E), dtype=np.float32), axis=1)[:, :k].astype(np.int32)
    x = synth.normal_bf16(seed, 1, (T, d), 1.0)
    return moe.MoeDims.of(T, d, E, k, S, 64, P), torch.from_numpy(idx).cuda(), \
        torch.from_numpy(x).view(torch.bfloat16).cuda()


def _routing_table_bytes(T, E, k, S):
    """The scratch the call needs, as include/moe.h states it: a 64-byte header,
    16 G bytes of group table, 4 (G + 1) of tile prefix, 4 G of group order and
    4 E max(1, ceil(T k / 1024)) of chunk histograms, each part on a 16-byte
    boundary, the sum rounded up to 256."""
    up = lambda v, a: (v + a - 1) // a * a
    G = E + S
    off = 64
    off = up(off, 16) + 16 * G
    off = up(off, 16) + 4 * (G + 1)
    off = up(off, 16) + 4 * G
    off = up(off, 16) + 4 * E * max(1, -(-T * k // 1024))
    return up(off, 256)


def _same(a, b, total):
    for key in ("counts", "offsets", "sorted_ids", "row_of"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["x_perm"][:total], b["x_perm"][:total])


def test_static_permute_matches_workspace_permute_twice():
    cases = [_case(1, 4096, 512, 128, 6, 128),   # many chunks, padded segments
             _case(2, 300, 192, 16, 3, 16)]      # a different, smaller routing next
    for dm, idx, x in cases:
        _run_both(dm, idx, x)


LIMIT = 1 << 20   # the fixed scratch array's size


def _run_both(dm, idx, x):
    ref = _outputs(dm)
    ws = torch.zeros(moe.moe_workspace_size(dm), dtype=torch.uint8, device="cuda")
    moe.moe_permute_align(dm, idx, x, ref["counts"], ref["offsets"], ref["sorted_ids"],
                          ref["row_of"], ref["x_perm"], ws)
    got = _outputs(dm)
    moe.moe_permute_align_static(dm, idx, x, got["counts"], got["offsets"], got["sorted_ids"],
                                 got["row_of"], got["x_perm"])
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    _same(got, ref, int(ref["offsets"][-1].item()))


def test_static_permute_limit_is_exactly_one_mib_of_routing_tables():
    # E = 256, k = 8: every 128 tokens add one 1024-assignment histogram chunk
    # (1 KiB).  The largest T whose routing tables fit 1 MiB is accepted and
    # matches the workspace form bit for bit; one token more is refused with
    # MOE_ERR_UNSUPPORTED_SHAPE before anything runs.
    E, k, S = 256, 8, 0
    T = 128
    while _routing_table_bytes(T + 128, E, k, S) <= LIMIT:
        T += 128
    assert _routing_table_bytes(T, E, k, S) <= LIMIT < _routing_table_bytes(T + 1, E, k, S)
    # the 1 MiB bound is the routing tables alone, well below the whole workspace
    dm_in, idx, x = _case(3, T, 64, E, k, 8, S)
    assert moe.moe_workspace_size(dm_in) > LIMIT
    _run_both(dm_in, idx, x)
    dm_out = moe.MoeDims.of(T + 1, 64, E, k, S, 64, 8)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_align_static(dm_out, 16, 16, 16, 16, 16, 16, 16)
    assert e.value.status == -2


def test_static_permute_rejects_what_every_entry_point_rejects():
    # the shared shape checks: P not a multiple of 8, k > E
    for dm in (moe.MoeDims.of(64, 128, 8, 2, 1, 64, 12), moe.MoeDims.of(64, 128, 8, 9, 1, 64, 16)):
        with pytest.raises(moe.MoeError) as e:
            moe.moe_permute_align_static(dm, 16, 16, 16, 16, 16, 16, 16)
        assert e.value.status == -2
