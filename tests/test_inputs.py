"""Pins for the seeded input generator (SplitMix64 + Box-Muller + round-to-nearest-even)."""
import math

import numpy as np
import pytest
import torch

from sequence_ring_self_b200 import inputs


def test_splitmix64_published_vector():
    # first outputs of SplitMix64 for seed 1234567, as published with the generator's
    # reference C code (Vigna, splitmix64.c)
    got = [int(x) for x in inputs.splitmix64(1234567, 0, 5)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_splitmix64_matches_scalar_definition():
    def ref(seed, n):
        out, state = [], seed
        for _ in range(n):
            state = (state + 0x9E3779B97F4A7C15) & (2**64 - 1)
            z = state
            z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & (2**64 - 1)
            z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & (2**64 - 1)
            out.append(z ^ (z >> 31))
        return out

    for seed in (0, 1, 2**63 + 5):
        assert [int(x) for x in inputs.splitmix64(seed, 0, 9)] == ref(seed, 9)
        assert [int(x) for x in inputs.splitmix64(seed, 4, 5)] == ref(seed, 9)[4:]


def test_box_muller_pair_and_offsets():
    a, b = (int(x) for x in inputs.splitmix64(3, 0, 2))
    u1 = ((a >> 11) + 1) / 2.0**53
    u2 = (b >> 11) / 2.0**53
    r = math.sqrt(-2 * math.log(u1))
    z = inputs.normals(3, 0, 2)
    assert z[0] == pytest.approx(r * math.cos(2 * math.pi * u2), rel=1e-15)
    assert z[1] == pytest.approx(r * math.sin(2 * math.pi * u2), rel=1e-15)
    full = inputs.normals(3, 0, 101)
    np.testing.assert_array_equal(inputs.normals(3, 37, 40), full[37:77])


def test_normal_moments():
    z = inputs.normals(0, 0, 1_000_000)
    assert abs(z.mean()) < 5e-3
    assert abs(z.var() - 1) < 5e-3
    assert abs((z**4).mean() - 3) < 3e-2


def _bf16_nearest_even(x):
    # brute force over the two bf16 neighbours of x
    f = np.float32(x)
    u = int(f.view(np.uint32)) & 0xFFFF0000
    lo = np.uint32(u).view(np.float32)
    hi = np.uint32(u + 0x10000).view(np.float32)
    lo, hi = float(lo), float(hi)
    if abs(x) < abs(lo):
        lo, hi = float(np.uint32(u - 0x10000).view(np.float32)), lo
    cands = sorted({lo, hi}, key=lambda c: (abs(c - x), (int(np.float32(c).view(np.uint32)) >> 16) & 1))
    return cands[0]


def test_bf16_rounding_ties_and_brute_force():
    assert inputs.round_to_bf16(np.array([1 + 2**-8]))[0] == 1.0               # tie -> even
    assert inputs.round_to_bf16(np.array([1 + 3 * 2**-8]))[0] == 1 + 2**-6     # tie -> even
    assert inputs.round_to_bf16(np.array([1 + 2**-8 + 2**-40]))[0] == 1 + 2**-7  # above tie
    rng = np.random.default_rng(0)
    x = rng.standard_normal(2000) * 10.0 ** rng.integers(-6, 6, 2000)
    got = inputs.round_to_bf16(x)
    for a, g in zip(x, got):
        assert g == _bf16_nearest_even(a)
    # fp32 inputs: torch's fp32 -> bf16 conversion is also round-to-nearest-even
    f32 = x.astype(np.float32).astype(np.float64)
    t = torch.from_numpy(f32.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(inputs.round_to_bf16(f32), t)


def test_make_inputs_layout_and_storage():
    x = inputs.make_inputs(2, 3, 8, 4, seed=2, dtype="bf16")
    n = 2 * 3 * 8 * 4
    z = inputs.normals(2, 0, 4 * n)
    np.testing.assert_array_equal(x.k, inputs.round_to_bf16(z[n:2 * n].reshape(2, 3, 8, 4) / 2.0))
    np.testing.assert_array_equal(x.do, inputs.round_to_bf16(z[3 * n:].reshape(2, 3, 8, 4)))
    t = x.torch("q")
    assert t.dtype == torch.bfloat16 and tuple(t.shape) == (2, 3, 8, 4)
    np.testing.assert_array_equal(t.to(torch.float64).numpy(), x.q)
    y = inputs.make_inputs(1, 2, 8, 4, seed=0, dtype="f32")
    assert y.torch("v").dtype == torch.float32
    np.testing.assert_array_equal(y.torch("v").double().numpy(), y.v)
