"""Lloyd-Max scalar codebook for one coordinate of a rotated unit vector.

[TQ] §二: after x/||x|| is rotated by Pi every coordinate follows the same
scaled Beta law (close to N(0, 1/d) in high dimension); the codebook is the
continuous 1-D k-means (Lloyd-Max) optimum for that law with 2^(b-1) levels,
looked up per coordinate by decision boundaries.

Law of one coordinate t of a uniform point on S^(d-1):
    f(t) = (1 - t^2)^p / Z on [-1, 1],  p = (d - 3)/2,  Z = B(1/2, p + 1),
equivalently (1 + t)/2 ~ Beta((d-1)/2, (d-1)/2).

Lloyd-Max fixed point (the two optimality conditions, iterated in turn):
    boundary  beta_k = (c_k + c_{k+1}) / 2
    centroid  c_k = E[t | beta_{k-1} < t <= beta_k]
with the interval mass from the regularised incomplete beta function and the
partial first moment in closed form
    int_a^b t (1 - t^2)^p dt = [(1 - a^2)^(p+1) - (1 - b^2)^(p+1)] / (2 (p + 1)).

Readings taken: start from Gaussian quantiles c_k = Phi^-1((k + 1/2)/L)/sqrt(d);
stop when max |delta c| < 1e-13 max |c|; the density is symmetric and log-concave, so
the optimum is unique (Fleischer 1964) and antisymmetric, and the result is
symmetrised exactly (c_{L-1-k} = -c_k, middle boundary exactly 0) before the
fp32 storage rounding.  Stored: fp32 centroids and fp32 boundaries rounded from
the float64 midpoints.
"""
from __future__ import annotations

import numpy as np
from scipy import special


class NotConverged(RuntimeError):
    pass


def _law(d: int):
    p = (d - 3) / 2.0
    a = (d - 1) / 2.0
    Z = np.exp(special.betaln(0.5, p + 1.0))
    return p, a, Z


def cdf(t, d: int):
    """P(coordinate <= t) on the sphere S^(d-1)."""
    _, a, _ = _law(d)
    s = np.clip((1.0 + np.asarray(t, dtype=np.float64)) / 2.0, 0.0, 1.0)
    return special.betainc(a, a, s)


def partial_moment(lo, hi, d: int):
    """E[t ; lo < t <= hi] (unnormalised by the mass), closed form."""
    p, _, Z = _law(d)
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    # (1 - t^2)^(p+1) as exp((p+1) log1p(-t^2)): accurate for large p.
    with np.errstate(divide="ignore"):
        ga = np.exp((p + 1.0) * np.log1p(-lo * lo))
        gb = np.exp((p + 1.0) * np.log1p(-hi * hi))
    return (ga - gb) / (2.0 * (p + 1.0) * Z)


def lloyd_max(d: int, bits: int, tol: float = 1e-13, max_iter: int = 200000):
    """Float64 centroids (ascending, length 2^bits) and the iteration count.

    Stops when max |delta c| < tol * max |c| (relative to the codebook's scale)."""
    L = 1 << bits
    c = special.ndtri((np.arange(L) + 0.5) / L) / np.sqrt(d)
    for it in range(1, max_iter + 1):
        beta = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate(([-1.0], beta, [1.0]))
        mass = cdf(edges[1:], d) - cdf(edges[:-1], d)
        new = partial_moment(edges[:-1], edges[1:], d) / mass
        delta = np.max(np.abs(new - c))
        c = new
        if delta < tol * np.max(np.abs(c)):
            break
    else:
        raise NotConverged(f"Lloyd-Max d={d} bits={bits}: no convergence in {max_iter} steps")
    half = L // 2
    pos = 0.5 * (c[half:] - c[:half][::-1])
    c = np.concatenate((-pos[::-1], pos))
    return c, it


def build(d: int, bits: int):
    """Stored codebook: fp32 centroids [2^bits], fp32 boundaries [2^bits - 1]."""
    c, _ = lloyd_max(d, bits)
    beta = 0.5 * (c[:-1] + c[1:])
    beta[len(beta) // 2] = 0.0
    return c.astype(np.float32), beta.astype(np.float32)


def distortion(c, d: int) -> float:
    """E[(t - q(t))^2] of the nearest-centroid quantiser with centroids c (float64)."""
    c = np.asarray(c, dtype=np.float64)
    beta = 0.5 * (c[:-1] + c[1:])
    edges = np.concatenate(([-1.0], beta, [1.0]))
    mass = cdf(edges[1:], d) - cdf(edges[:-1], d)
    m1 = partial_moment(edges[:-1], edges[1:], d)
    # int (t - c)^2 f = E[t^2; I] - 2 c m1 + c^2 mass, and E[t^2] = 1/d overall.
    return float(1.0 / d - np.sum(2.0 * c * m1 - c * c * mass))
