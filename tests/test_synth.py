"""The seeded input generator (no GPU): Philox known answers, slicing, distributions."""
import math

import numpy as np

import synth


def test_philox_known_answers():
    # known-answer vectors published with the Random123 library (Salmon et al., SC'11)
    assert list(synth.philox4x32_10([0, 0, 0, 0], [0, 0])) == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    assert list(synth.philox4x32_10([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2)) == [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]
    assert list(synth.philox4x32_10([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0])) == \
        [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]


def test_slices_are_consistent():
    full = synth.normal_bf16(0, 3, 0, 10001, 0.5)
    for off, n in [(0, 7), (1, 10), (333, 1000), (9990, 11)]:
        assert np.array_equal(synth.normal_bf16(0, 3, off, n, 0.5), full[off:off + n])
    inp = synth.Inputs(synth.WORKLOADS["tiny"])
    x = inp.x()
    assert np.array_equal(inp.x_rows(5, 9), x[5:14].ravel())
    w1 = inp.w1()
    assert np.array_equal(inp.expert_rows("w1", 3, 2), w1[3:5].ravel())


def test_normal_moments():
    v = synth.bf16_bits_to_f32(synth.normal_bf16(0, 1, 0, 1 << 20, 1.0)).astype(np.float64)
    assert abs(v.mean()) < 5e-3 and abs(v.std() - 1) < 5e-3
    w = synth.bf16_bits_to_f32(synth.normal_bf16(0, 2, 0, 1 << 18, 1 / 64)).astype(np.float64)
    assert abs(w.std() * 64 - 1) < 1e-2
    u = synth.uniform_f32(0, 9, 0, 1 << 16, -0.1, 0.1).astype(np.float64)
    assert u.min() >= -0.1 and u.max() < 0.1 and abs(u.mean()) < 2e-3


def test_skew_recipe_unit_vector_and_shift():
    inp = synth.Inputs(synth.WORKLOADS["skew"])
    u = inp.u()
    assert abs(np.dot(u, u) - 1) < 1e-12
    b = inp.zipf_shift()
    assert b.shape == (64,) and np.all(np.diff(b[:8]) < 0)        # most popular expert gets the largest shift
    x = synth.bf16_bits_to_f32(inp.x_rows(0, 64)).reshape(64, -1).astype(np.float64)
    proj = x @ u
    assert abs(proj.mean() - 4.0) < 0.5                           # hidden states shifted by mu*u


def test_workloads_match_shapes():
    W = synth.WORKLOADS
    assert (W["mixtral"].T, W["mixtral"].d, W["mixtral"].E, W["mixtral"].k, W["mixtral"].f) == (4096, 4096, 8, 2, 14336)
    assert (W["qwen3"].T, W["qwen3"].E, W["qwen3"].k, W["qwen3"].f) == (16384, 128, 8, 1536)
    assert (W["dsv3"].d, W["dsv3"].E, W["dsv3"].f_shared, W["dsv3"].bias_range) == (7168, 256, 2048, 0.1)
    s = W["skew"]
    assert int(s.T * s.k / s.E * s.capacity_factor) == 1280
    assert math.isclose(s.zipf_s, 1.2)
