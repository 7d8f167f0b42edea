"""Pins of the oracle's sensitivity profile (layer groups and sketch dims).

Pinned against closed forms (variance of an arithmetic sequence), exhaustive
search over every boundary list and every sketch-dim vector on small cases, the
pages' own A-QJL boundaries for an evenly spread variance ramp, and the
Lagrange optimum m_g proportional to the square root of the group variance.
"""
import itertools

import numpy as np
import pytest

from oracle import sensitivity as sens


def test_key_variance_closed_form():
    # 0, 1, ..., N-1 in any shape: population variance (N^2 - 1) / 12
    N = 4 * 3 * 50 * 8
    K = np.arange(N, dtype=np.float64).reshape(4, 3, 50, 8)
    assert abs(sens.key_variance(K) - (N * N - 1) / 12.0) < 1e-9 * N * N
    # +-a in equal numbers (and a shift c): variance a^2
    K = np.where(np.arange(1000) % 2 == 0, 2.5, -2.5) + 7.0
    assert abs(sens.key_variance(K) - 6.25) < 1e-12


def _sse(v, bounds):
    e = [0] + list(bounds) + [len(v)]
    return sum(((v[e[i]:e[i + 1]] - v[e[i]:e[i + 1]].mean()) ** 2).sum() for i in range(len(e) - 1))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_segmentation_equals_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    v = rng.gamma(2.0, 1.0, size=9)
    for k in range(1, 5):
        got = sens.segment_layers(v, k)
        costs = {}
        for b in itertools.combinations(range(1, 9), k - 1):
            costs[b] = _sse(v, b)
        best = min(costs.values())
        assert abs(_sse(v, got) - best) < 1e-12
        # the tie rule: the lexicographically smallest optimal boundary list
        assert tuple(got) == min(b for b, c in costs.items() if c <= best + 1e-12)


def test_even_variance_ramp_gives_the_pages_boundaries():
    # 32 layers with variance 1 + 2 l / 31 (evenly spread): four equal groups,
    # the boundaries 8, 16, 24 of the A-QJL deployment config
    v = 1.0 + 2.0 * np.arange(32) / 31.0
    assert sens.segment_layers(v, 4) == [8, 16, 24]
    assert sens.segment_layers(v, 2) == [16]


def test_equal_variance_gets_equal_dims():
    v = np.full(32, 1.7)
    b = [8, 16, 24]
    assert sens.allocate_sketch_dims(v, b, 256) == [256, 256, 256, 256]


@pytest.mark.parametrize("seed", [3, 4, 5])
def test_allocation_equals_exhaustive_search_for_equal_groups(seed):
    rng = np.random.default_rng(seed)
    v = np.repeat(rng.gamma(2.0, 1.0, size=3), 2)          # 3 groups of 2 layers
    b = [2, 4]
    m_avg, m_min, m_max = 160, 32, 384
    got = sens.allocate_sketch_dims(v, b, m_avg, m_min, m_max)
    grid = range(m_min, m_max + 1, 32)
    best = min(sens.objective(v, b, m) for m in itertools.product(grid, repeat=3)
               if 2 * sum(m) <= 6 * m_avg)
    assert abs(sens.objective(v, b, got) - best) < 1e-12
    assert 2 * sum(got) <= 6 * m_avg


def test_allocation_follows_the_square_root_rule():
    # the continuous optimum of sum n s / m under sum n m = M is m proportional
    # to sqrt(s); on the 32-grid each dim is within one step of it
    s = np.array([1.0, 2.0, 4.0, 9.0])
    v = np.repeat(s, 8)
    b = [8, 16, 24]
    m_avg = 512
    got = np.array(sens.allocate_sketch_dims(v, b, m_avg, 32, 4096))
    cont = 4 * m_avg * np.sqrt(s) / np.sqrt(s).sum()
    assert np.all(np.abs(got - cont) <= 32 + 1e-9)
    assert np.all(np.diff(got) >= 0)                      # more variance, more sketch bits
    assert 8 * got.sum() <= 32 * m_avg


def test_budget_and_limits_hold():
    rng = np.random.default_rng(6)
    v = rng.gamma(1.5, 2.0, size=32)
    b, m = sens.profile(v, 4, 300, 64, 512)
    e = [0] + b + [32]
    assert sum((e[i + 1] - e[i]) * m[i] for i in range(4)) <= 32 * 300
    assert all(64 <= x <= 512 and x % 32 == 0 for x in m)
    with pytest.raises(ValueError):
        sens.allocate_sketch_dims(v, b, 16, 32)
