"""Pins of the oracle's generator and projections (CPU only)."""
import numpy as np
import pytest

from conftest import read_golden
from oracle import philox, projections


def test_philox_known_answers():
    for row in read_golden("philox4x64_10_kat.txt"):
        w = [int(x, 16) for x in row.split()]
        ctr, key, want = w[0:4], w[4:6], w[6:10]
        got = philox.philox4x64_10([np.uint64(c) for c in ctr], key)
        assert [int(g) for g in got] == want


def test_philox_matches_numpy_bitgenerator():
    # numpy.random.Philox is Philox4x64-10; it advances the counter before each block.
    rng = np.random.default_rng(5)
    for _ in range(20):
        key = [int(x) for x in rng.integers(0, 2**63, 2, dtype=np.uint64)]
        ctr = [int(x) for x in rng.integers(1, 2**63, 4, dtype=np.uint64)]
        bg = np.random.Philox(key=np.array(key, np.uint64),
                              counter=np.array([ctr[0] - 1] + ctr[1:], np.uint64))
        want = [int(x) for x in bg.random_raw(4)]
        got = philox.philox4x64_10([np.uint64(c) for c in ctr], key)
        assert [int(g) for g in got] == want


def test_philox_vectorised_equals_scalar():
    k = np.arange(17, dtype=np.uint64)
    z = np.zeros_like(k)
    vec = philox.philox4x64_10((k, z, z, z), (42, 1))
    for i in range(17):
        sc = philox.philox4x64_10((np.uint64(i), np.uint64(0), np.uint64(0), np.uint64(0)), (42, 1))
        assert all(int(vec[j][i]) == int(sc[j]) for j in range(4))


def test_uniform_open_interval_and_gaussian_moments():
    w = np.array([0, 2**64 - 1], dtype=np.uint64)
    u = philox.uniform53(w)
    assert u[0] == 2.0 ** -54 and u[1] == 1.0      # (0, 1]: never 0
    z = philox.gaussian(1_000_000, seed=42, stream=0)
    n = z.size
    assert abs(z.mean()) < 5 / np.sqrt(n)
    assert abs(z.var() - 1.0) < 5 * np.sqrt(2.0 / n)
    # fourth moment of N(0,1) is 3 (se of the sample 4th moment ~ sqrt(96/n))
    assert abs(np.mean(z ** 4) - 3.0) < 5 * np.sqrt(96.0 / n)


def test_layer_seed_rule():
    assert projections.layer_seed(0) == 42
    assert projections.layer_seed(5) == 77


@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_rotation_is_orthogonal_with_positive_r(d):
    seed = projections.layer_seed(3)
    Pi = projections.rotation(d, seed)
    assert np.max(np.abs(Pi.T @ Pi - np.eye(d))) < 1e-13
    G = projections.gaussian_matrix(d, d, seed, projections.STREAM_PI)
    R = Pi.T @ G                      # = R of G = Pi R
    assert np.max(np.abs(np.tril(R, -1))) < 1e-10 * np.max(np.abs(R))
    assert np.all(np.diag(R) > 0)


def test_projection_storage_and_streams():
    p = projections.make_projections(128, 128, layer=1)
    assert p["Pi"].dtype == np.float32 and p["Pi"].nbytes == 65536   # 64 KB at d = 128
    S64 = projections.gaussian_matrix(128, 128, 49, projections.STREAM_S)
    assert np.array_equal(p["S"], S64.astype(np.float32))
    assert np.allclose(p["T"], p["S"].astype(np.float64) @ p["Pi"].astype(np.float64).T,
                       rtol=0, atol=1e-5)
    q = projections.make_projections(128, 128, layer=2)
    assert not np.array_equal(p["S"], q["S"])
    pure = projections.make_projections(128, 192, layer=0, with_rotation=False)
    assert pure["Pi"] is None and np.array_equal(pure["T"], pure["S"])


def test_rotation_is_haar_distributed():
    # For Haar Q, E[Q_ij] = 0 and E[Q_ij^2] = 1/d; average over many seeds.
    d = 16
    acc = np.zeros((d, d))
    acc2 = np.zeros((d, d))
    n = 400
    for s in range(n):
        Q = projections.rotation(d, 1000 + s)
        acc += Q
        acc2 += Q * Q
    assert np.max(np.abs(acc / n)) < 5 * np.sqrt(1.0 / d / n)
    assert abs(np.mean(acc2 / n) - 1.0 / d) < 0.01 / d


def _fwht(v):
    """Plain in-place butterfly Walsh-Hadamard transform (unnormalised), O(d log d)."""
    v = np.array(v, dtype=np.float64)
    h = 1
    while h < v.shape[-1]:
        for i in range(0, v.shape[-1], 2 * h):
            a = v[..., i:i + h].copy()
            b = v[..., i + h:i + 2 * h].copy()
            v[..., i:i + h] = a + b
            v[..., i + h:i + 2 * h] = a - b
        h *= 2
    return v


@pytest.mark.parametrize("d", [2, 8, 64, 256])
def test_sylvester_hadamard_closed_form(d):
    """H_d of the recursion has entry (r, c) = (-1)^popcount(r & c)."""
    H = projections.sylvester_hadamard(d)
    r = np.arange(d)[:, None]
    c = np.arange(d)[None, :]
    par = np.vectorize(lambda x: bin(x).count("1") & 1)(r & c)
    assert np.array_equal(H, np.where(par == 1, -1.0, 1.0))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_hadamard_rotation_orthogonal_flat_and_fast(d):
    """Pi = H diag(s) / sqrt(d): orthogonal, every entry of magnitude 1/sqrt(d) (so a
    single large coordinate is spread evenly over all d), and Pi u equals the fast
    Walsh-Hadamard transform of s * u divided by sqrt(d)."""
    seed = projections.layer_seed(3)
    Pi = projections.hadamard_rotation(d, seed)
    assert np.max(np.abs(Pi.T @ Pi - np.eye(d))) < 1e-12
    assert np.allclose(np.abs(Pi), 1.0 / np.sqrt(d), rtol=0, atol=1e-15)
    s = projections.hadamard_signs(d, seed)
    rng = np.random.default_rng(5)
    u = rng.standard_normal((3, d))
    assert np.max(np.abs(u @ Pi.T - _fwht(u * s) / np.sqrt(d))) < 1e-12
    e = np.zeros(d)
    e[d // 3] = 7.0                                    # an outlier coordinate
    assert np.allclose(np.abs(Pi @ e), 7.0 / np.sqrt(d), rtol=0, atol=1e-12)
    st = projections.make_projections(d, 32, 3, structured=True)
    assert np.all(np.abs(st["Pi"]) == np.float32(1.0 / np.sqrt(d)))


def test_hadamard_signs_from_philox_stream_2():
    """s_c = +1 iff the top bit of word 0 of Philox draw c under key (seed, 2) is 0;
    checked draw by draw against the scalar generator, and balanced."""
    seed = 42
    s = projections.hadamard_signs(4096, seed)
    for c in (0, 1, 777, 4095):
        w0 = philox.philox4x64_10((np.uint64(c), 0, 0, 0), (seed, 2))[0]
        assert s[c] == (1.0 if int(w0) >> 63 == 0 else -1.0)
    assert abs(s.mean()) < 5.0 / np.sqrt(4096)
    assert not np.array_equal(s, projections.hadamard_signs(4096, seed + 7))
