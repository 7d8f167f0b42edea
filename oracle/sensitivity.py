"""Sensitivity profile for the adaptive per-layer-group sketch dimension.

[AQJL] §敏感度分析器 (sensitivity analyser): each layer's sensitivity to
compression is judged from the variance of its key vectors, computed on
calibration data; the analyser outputs the layer-group boundaries and the
per-group sketch dimensions (the A-QJL config of §实际部署, boundaries such as
"8,16,24" and dims such as "512,384,256,192").  The pages give no formula.
Readings taken (test infrastructure; the same steps are restated, not shared,
by the library):

* statistic: the population variance of all key entries of a layer (every
  batch, head, token and channel), float64;
* groups: contiguous layers, the boundaries minimising the summed squared
  deviation of the per-layer variances from their group means (an exact
  segmentation by dynamic programming; among equal optima the
  lexicographically smallest boundary list);
* sketch dims: the QJL term's variance for a key of squared norm ||k||^2 is
  proportional to ||k||^2 / m ([TQ] §四 estimator; ||k||^2 = d * variance),
  so the profile minimises sum_g n_g s_g / m_g (n_g layers of mean variance
  s_g) under the sign-bit budget sum_g n_g m_g <= L * m_avg, each m_g a
  multiple of 32 in [m_min, m_max]: every group starts at m_min and 32 is added,
  one step at a time, to the group whose step lowers the objective most per
  sign bit spent, among the steps that still fit (ties: the lower group).
"""
from __future__ import annotations

import numpy as np

STEP = 32


def _mean(xs) -> float:
    """Sequential float64 mean (a fixed summation order: the group decisions below
    are integers decided by these sums)."""
    t = 0.0
    for x in xs:
        t += float(x)
    return t / len(xs)


def key_variance(K) -> float:
    """Population variance of every entry of one layer's keys, float64."""
    x = np.asarray(K, dtype=np.float64).ravel()
    if x.size == 0:
        raise ValueError("no keys")
    mu = x.sum() / x.size
    return float(((x - mu) ** 2).sum() / x.size)


def segment_layers(var, num_groups: int):
    """First layer of groups 1..num_groups-1 (contiguous groups)."""
    v = np.asarray(var, dtype=np.float64)
    L = v.size
    if not 1 <= num_groups <= L:
        raise ValueError("need 1 <= num_groups <= number of layers")

    def sse(a, b):          # layers a..b-1, sequential float64 sums
        mu = _mean(v[a:b])
        t = 0.0
        for x in v[a:b]:
            t += (float(x) - mu) * (float(x) - mu)
        return t

    INF = float("inf")
    # best[g][l]: minimal cost of the first l layers in g groups, with its boundaries
    best = [[(INF, None)] * (L + 1) for _ in range(num_groups + 1)]
    best[0][0] = (0.0, [])
    for g in range(1, num_groups + 1):
        for l in range(g, L + 1):
            cand = (INF, None)
            for a in range(g - 1, l):           # last group is layers a..l-1
                prev_cost, prev_b = best[g - 1][a]
                if prev_b is None:
                    continue
                cost = prev_cost + sse(a, l)
                bnd = prev_b + ([a] if g > 1 else [])
                if cost < cand[0] or (cost == cand[0] and bnd < cand[1]):
                    cand = (cost, bnd)
            best[g][l] = cand
    return best[num_groups][L][1]


def allocate_sketch_dims(var, bounds, m_avg: int, m_min: int = 32, m_max: int = 1024):
    """Sketch dim of each group for boundaries `bounds` under the budget L * m_avg."""
    v = np.asarray(var, dtype=np.float64)
    L = v.size
    edges = [0] + list(bounds) + [L]
    n = [edges[i + 1] - edges[i] for i in range(len(edges) - 1)]
    s = [_mean(v[edges[i]:edges[i + 1]]) for i in range(len(n))]
    m = [m_min] * len(n)
    left = L * m_avg - sum(ng * m_min for ng in n)
    if left < 0:
        raise ValueError("budget below m_min for every layer")
    while True:
        pick, gain = -1, 0.0
        for g in range(len(n)):
            if m[g] + STEP > m_max or n[g] * STEP > left:
                continue
            # objective decrease per sign bit of this step
            d = n[g] * s[g] * (1.0 / m[g] - 1.0 / (m[g] + STEP)) / (n[g] * STEP)
            if d > gain:
                pick, gain = g, d
        if pick < 0:
            return m
        m[pick] += STEP
        left -= n[pick] * STEP


def objective(var, bounds, m) -> float:
    v = np.asarray(var, dtype=np.float64)
    edges = [0] + list(bounds) + [v.size]
    return float(sum(v[edges[i]:edges[i + 1]].sum() / m[i] for i in range(len(m))))


def profile(var, num_groups: int, m_avg: int, m_min: int = 32, m_max: int = 1024):
    """(boundaries, sketch dims) of the layers with variances `var`."""
    b = segment_layers(var, num_groups)
    return b, allocate_sketch_dims(var, b, m_avg, m_min, m_max)
