"""Pins of the Lloyd-Max codebook oracle (CPU only)."""
import numpy as np
import pytest
from scipy import integrate, special

from conftest import read_golden
from oracle import codebook


def _density(t, d):
    p = (d - 3) / 2.0
    Z = np.exp(special.betaln(0.5, p + 1.0))
    return (1.0 - t * t) ** p / Z


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 1), (128, 2), (128, 3), (256, 3), (256, 4)])
def test_fixed_point_conditions_by_quadrature(d, bits):
    """Each centroid is the conditional mean of its cell, recomputed by adaptive
    quadrature (an independent route from the incomplete-beta closed form)."""
    c, _ = codebook.lloyd_max(d, bits)
    beta = 0.5 * (c[:-1] + c[1:])
    edges = np.concatenate(([-1.0], beta, [1.0]))
    for k in range(len(c)):
        lo, hi = edges[k], edges[k + 1]
        m0 = integrate.quad(lambda t: _density(t, d), lo, hi, epsabs=0, epsrel=1e-13, limit=200)[0]
        m1 = integrate.quad(lambda t: t * _density(t, d), lo, hi, epsabs=0, epsrel=1e-13, limit=200)[0]
        assert abs(m1 / m0 - c[k]) < 1e-11 * np.max(np.abs(c))


def test_density_normalised_and_cdf():
    for d in (8, 128):
        tot = integrate.quad(lambda t: _density(t, d), -1, 1, points=[-0.3, 0.0, 0.3],
                             epsabs=0, epsrel=1e-13, limit=200)[0]
        assert abs(tot - 1.0) < 1e-12
        a = integrate.quad(lambda t: _density(t, d), -1, 0.05, points=[-0.3, 0.0],
                           epsabs=0, epsrel=1e-13, limit=200)[0]
        assert abs(codebook.cdf(0.05, d) - a) < 1e-12


@pytest.mark.parametrize("d", [3, 8, 128, 256])
def test_one_bit_closed_form(d):
    # 1 bit: the two cells are the half lines, c = +-E|t| = Gamma(d/2)/(sqrt(pi) Gamma((d+1)/2)).
    c, _ = codebook.lloyd_max(d, 1)
    want = np.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / np.sqrt(np.pi)
    assert abs(c[1] - want) < 1e-13 and c[0] == -c[1]


def test_symmetry_and_storage():
    for bits in (1, 2, 3):
        c32, b32 = codebook.build(128, bits)
        L = 1 << bits
        assert c32.dtype == np.float32 and b32.dtype == np.float32
        assert np.array_equal(c32, -c32[::-1])
        assert b32[L // 2 - 1] == 0.0
        c64, _ = codebook.lloyd_max(128, bits)
        assert np.array_equal(b32, (0.5 * (c64[:-1] + c64[1:])).astype(np.float32) * (b32 != 0))
        assert np.all(np.diff(c32) > 0) and np.all(c32[:-1] < b32) and np.all(b32 < c32[1:])


def test_large_d_limit_is_max_1960_gaussian_table():
    d = 65536
    for row in read_golden("max1960_gaussian_lloyd_max.txt"):
        vals = [float(x) for x in row.split()]
        bits, mse, cents = int(vals[0]), vals[1], vals[2:]
        c, _ = codebook.lloyd_max(d, bits)
        # table printed to 4 significant figures
        assert abs(d * codebook.distortion(c, d) - mse) <= 6e-4 * mse + 1e-6
        pos = c[len(c) // 2:] * np.sqrt(d)
        for got, want in zip(pos, cents):
            assert abs(got - want) <= 6e-4 * want


def test_distortion_falls_roughly_as_quarter_per_bit():
    # [TQ] section 1, "Theorem 3": distortion scales as 1/4^b.
    d = 128
    D = [codebook.distortion(codebook.lloyd_max(d, b)[0], d) for b in (1, 2, 3, 4)]
    ratios = [D[i] / D[i + 1] for i in range(3)]
    assert all(2.8 < r < 4.0 for r in ratios)
    assert ratios[0] < ratios[1] < ratios[2]


def test_distortion_formula_by_monte_carlo():
    d, bits = 32, 2
    c, _ = codebook.lloyd_max(d, bits)
    beta = 0.5 * (c[:-1] + c[1:])
    rng = np.random.default_rng(0)
    x = rng.standard_normal((200_000, d))
    t = (x / np.linalg.norm(x, axis=1, keepdims=True)).ravel()
    q = c[np.searchsorted(beta, t, side="left")]
    mc = np.mean((t - q) ** 2)
    se = np.std((t - q) ** 2) / np.sqrt(t.size)
    assert abs(mc - codebook.distortion(c, d)) < 5 * se


def test_lloyd_max_is_a_local_minimum():
    d, bits = 128, 2
    c, _ = codebook.lloyd_max(d, bits)
    base = codebook.distortion(c, d)
    rng = np.random.default_rng(1)
    for _ in range(20):
        pert = c + 1e-3 * np.max(np.abs(c)) * rng.standard_normal(c.size)
        pert.sort()
        assert codebook.distortion(pert, d) > base
