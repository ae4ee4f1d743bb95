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


def _case(seed, T, d, E, k, P):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    x = synth.normal_bf16(seed, 1, (T, d), 1.0)
    return moe.MoeDims.of(T, d, E, k, 2, 64, P), torch.from_numpy(idx).cuda(), \
        torch.from_numpy(x).view(torch.bfloat16).cuda()


def _same(a, b, total):
    for key in ("counts", "offsets", "sorted_ids", "row_of"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["x_perm"][:total], b["x_perm"][:total])


def test_static_permute_matches_workspace_permute_twice():
    cases = [_case(1, 4096, 512, 128, 6, 128),   # many chunks, padded segments
             _case(2, 300, 192, 16, 3, 16)]      # a different, smaller routing next
    for dm, idx, x in cases:
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


def test_static_permute_rejects_shapes_beyond_its_scratch():
    # E = 256 and 4M routed assignments need more than the fixed 1 MiB of scratch
    dm = moe.MoeDims.of(1 << 20, 64, 256, 4, 0, 64, 8)
    assert moe.moe_workspace_size(dm) > (1 << 20)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_align_static(dm, 16, 16, 16, 16, 16, 16, 16)
    assert e.value.status == -2
