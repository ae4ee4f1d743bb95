"""Checks of the seeded input generator (CPU only).  The generator holds none of
the layer's arithmetic; these tests only check it draws what it says."""
import numpy as np
import torch

import synth


def test_splitmix64_reference_value():
    # SplitMix64 from state 0 yields 0xE220A8397B1DCDAF first (Steele et al. 2014);
    # draw(key, 0) = mix(key + GAMMA), so stream_key == 0 would give that value.
    # The exported raw draw is deterministic and differs across streams and seeds.
    a, b, c = synth.raw(1, 2, 0), synth.raw(1, 3, 0), synth.raw(2, 2, 0)
    assert len({a, b, c}) == 3 and synth.raw(1, 2, 0) == a


def test_moments_and_ranges():
    z = synth.bf16_to_f32(synth.normal_bf16(0, 1, (1 << 20,), 1.0)).astype(np.float64)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3
    u = synth.uniform_f32(0, 3, (1 << 18,), -0.01, 0.01)
    assert u.min() >= -0.01 and u.max() <= 0.01 and abs(u.mean()) < 1e-4


def test_bf16_rounding_matches_torch():
    f = synth.normal_f32(5, 9, (1 << 16,), 3.0)
    ours = synth.normal_bf16(5, 9, (1 << 16,), 3.0)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_slices_regenerate_identically():
    a = synth.normal_bf16(4, 4, (1000,), 0.02)
    b = synth.normal_bf16(4, 4, (1001,), 0.02)
    assert np.array_equal(a, b[:1000])
