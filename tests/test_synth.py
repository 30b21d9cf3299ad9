"""Pins of the seeded input generator (host twin) against its written definition."""
import numpy as np
import pytest

import synth
from synth import workloads as W


def test_key_matches_python_definition():
    for seed in (0, 1, 2, 3, 4, 12345):
        for t in (1, 2, 3, 4, 5):
            for layer in (0, 1, 22):
                assert synth.key(seed, t, layer) == synth.py_key(seed, t, layer)


@pytest.mark.parametrize("sigma", [1.0, 0.02])
def test_c_generator_equals_python_loop(sigma):
    k = synth.key(7, 3, 5)
    for off in (0, 1, 999_983):
        a = synth.normal_bf16(k, 1500, sigma, offset=off)
        b = synth.py_normal_bf16(k, 1500, sigma, offset=off)
        assert np.array_equal(a, b)


def test_counter_based_random_access():
    k = synth.key(2, 3, 0)
    full = synth.normal_bf16(k, 50_000, 0.02)
    part = synth.normal_bf16(k, 1000, 0.02, offset=31_000)
    assert np.array_equal(full[31_000:32_000], part)


def test_moments_and_support():
    k = synth.key(1, 1, 0)
    z = synth.normal_f32(k, 2_000_000, 1.0).astype(np.float64)
    assert abs(z.mean()) < 3e-3
    assert abs(z.std() - 1.0) < 3e-3
    assert np.abs(z).max() <= 6.0
    # Irwin-Hall(12) kurtosis is 3 - 1.2/12 = 2.9
    kurt = np.mean(z ** 4) / np.mean(z ** 2) ** 2
    assert abs(kurt - 2.9) < 0.03


def test_zipf_bias_is_zipf():
    b = W.zipf_bias(3, 128).astype(np.float64)
    p = np.exp(b - b.max())
    p /= p.sum()
    ranks = np.argsort(-p)
    expect = np.arange(1, 129, dtype=np.float64) ** -1.1
    expect /= expect.sum()
    assert np.allclose(np.sort(p)[::-1], expect, rtol=1e-5)
    assert len(set(ranks.tolist())) == 128


def test_expert_subset_matches_full_bank():
    w = W.WORKLOADS[0]
    full = W.host_w_up(w)
    sub = W.host_w_up(w, experts=[5, 2])
    assert np.array_equal(sub[0], full[5]) and np.array_equal(sub[1], full[2])
    fulld = W.host_w_down(w)
    subd = W.host_w_down(w, experts=[7])
    assert np.array_equal(subd[0], fulld[7])
