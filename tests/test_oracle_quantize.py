"""Pins of the key/value quantisers and the estimator (CPU only)."""
import numpy as np
import pytest

from conftest import page_figures
from oracle import attention, codebook, projections, quantize

ALPHA = np.sqrt(np.pi / 2)


def _setup(d, m, b1, layer=0):
    p = projections.make_projections(d, m, layer, with_rotation=b1 > 0)
    cb = codebook.build(d, b1) if b1 > 0 else (None, None)
    return p, cb


def test_codes_equal_exhaustive_nearest_centroid_small_d():
    d, m, b1 = 8, 8, 2
    p, (c32, b32) = _setup(d, m, b1)
    rng = np.random.default_rng(0)
    X = rng.standard_normal((300, d))
    out = quantize.quantize_keys(X, p["Pi"], p["S"], c32, b32, b1)
    Pi = p["Pi"].astype(np.float64)
    for t in range(X.shape[0]):
        u = X[t] / np.sqrt(sum(v * v for v in X[t]))
        for j in range(d):
            y = float(np.float32(sum(Pi[j, i] * u[i] for i in range(d))))
            dist = [abs(y - float(ck)) for ck in c32]
            best = min(range(len(dist)), key=lambda k: (dist[k], k))   # ties -> lower index
            assert out["idx"][t, j] == best


def test_residual_and_signs_by_explicit_sums_small_d():
    d, m, b1 = 8, 16, 2
    p, (c32, b32) = _setup(d, m, b1)
    rng = np.random.default_rng(1)
    X = rng.standard_normal((40, d))
    out = quantize.quantize_keys(X, p["Pi"], p["S"], c32, b32, b1)
    Pi, S = p["Pi"].astype(np.float64), p["S"].astype(np.float64)
    for t in range(X.shape[0]):
        rho = np.sqrt(sum(v * v for v in X[t]))
        xt = [rho * sum(Pi[j, i] * float(c32[out["idx"][t, j]]) for j in range(d)) for i in range(d)]
        r = [X[t, i] - xt[i] for i in range(d)]
        for k in range(m):
            zk = sum(S[k, i] * r[i] for i in range(d))
            assert out["bits"][t, k] == (1 if zk >= 0 else 0)
        assert abs(float(out["rnorm"][t]) - np.sqrt(sum(v * v for v in r))) < 1e-6 * rho
        assert out["rho"][t] == np.float32(rho)


def test_mse_term_equals_query_dot_reconstruction():
    # rho <Pi q, c[idx]> == <q, rho Pi^T c[idx]> = <q, x~> (Pi orthogonal in float64 of the
    # stored fp32 values up to the fp32 rounding of Pi).
    d, m, b1 = 128, 128, 2
    p, (c32, b32) = _setup(d, m, b1)
    rng = np.random.default_rng(2)
    X = rng.standard_normal((64, d))
    q = rng.standard_normal((3, d))
    keys = quantize.quantize_keys(X, p["Pi"], p["S"], c32, b32, b1)
    Pi = p["Pi"].astype(np.float64)
    xt = keys["rho"].astype(np.float64)[:, None] * (c32.astype(np.float64)[keys["idx"]] @ Pi)
    zero_r = dict(keys, rnorm=np.zeros_like(keys["rnorm"]))
    got = attention.logits_compressed(q, zero_r, p["Pi"], p["S"], c32, b1)
    assert np.max(np.abs(got - q @ xt.T)) < 1e-12 * np.max(np.abs(got))


def test_qjl_term_by_explicit_pm1_sums():
    d, m, b1 = 16, 32, 2
    p, (c32, b32) = _setup(d, m, b1)
    rng = np.random.default_rng(3)
    X = rng.standard_normal((10, d))
    q = rng.standard_normal((2, d))
    keys = quantize.quantize_keys(X, p["Pi"], p["S"], c32, b32, b1)
    S, Pi = p["S"].astype(np.float64), p["Pi"].astype(np.float64)
    got = attention.logits_compressed(q, keys, p["Pi"], p["S"], c32, b1)
    for h in range(2):
        qr = [sum(Pi[j, i] * q[h, i] for i in range(d)) for j in range(d)]
        sq = [sum(S[k, i] * q[h, i] for i in range(d)) for k in range(m)]
        for t in range(10):
            mse = float(keys["rho"][t]) * sum(qr[j] * float(c32[keys["idx"][t, j]]) for j in range(d))
            qjl = sum(sq[k] * (1.0 if keys["bits"][t, k] else -1.0) for k in range(m))
            want = mse + float(keys["rnorm"][t]) * ALPHA / m * qjl
            assert abs(got[h, t] - want) < 1e-10 * (1 + abs(want))


def test_zero_key():
    d, m, b1 = 128, 128, 2
    p, (c32, b32) = _setup(d, m, b1)
    out = quantize.quantize_keys(np.zeros((1, d)), p["Pi"], p["S"], c32, b32, b1)
    assert np.all(out["idx"] == 1) and np.all(out["bits"] == 1)
    assert out["rho"][0] == 0 and out["rnorm"][0] == 0
    pure = quantize.quantize_keys(np.zeros((1, d)), None, p["S"], None, None, 0)
    assert np.all(pure["bits"] == 1) and pure["rho"][0] == 0


@pytest.mark.parametrize("b1,d,m,structured", [(2, 16, 16, False), (1, 16, 16, False), (0, 16, 32, False),
                                                (2, 16, 16, True)])
def test_estimator_unbiased_over_sketch_draws(b1, d, m, structured):
    """E_S[estimate] = <q, x> ([TQ] section 4/5), with the QR rotation and with the
    structured Hadamard one.  Draw N independent S matrices; stacking them as one
    sketch of N*m rows makes the oracle's own estimator return the mean of the N
    per-draw estimates (its 1/m becomes 1/(N m))."""
    rng = np.random.default_rng(10 + b1)
    x = rng.standard_normal(d)
    q = x + 0.8 * rng.standard_normal(d)             # |<q,x>| well away from 0
    assert abs(q @ x) > 0.5 * np.linalg.norm(q) * np.linalg.norm(x)
    rot = projections.hadamard_rotation if structured else projections.rotation
    Pi = rot(d, 7).astype(np.float32) if b1 else None
    c32, b32 = codebook.build(d, b1) if b1 else (None, None)
    N = 100_000
    S = rng.standard_normal((N * m, d)).astype(np.float32)
    keys = quantize.quantize_keys(x[None, :], Pi, S, c32, b32, b1)
    mean_est = attention.logits_compressed(q[None, :], keys, Pi, S, c32, b1)[0, 0]
    # per-draw estimates for the standard error
    sq = S.astype(np.float64) @ q
    pm = 2.0 * keys["bits"][0].astype(np.float64) - 1.0
    per = (sq * pm).reshape(N, m).sum(axis=1) * ALPHA / m
    scale = float(keys["rnorm"][0]) if b1 else float(keys["rho"][0])
    per = per * scale
    if b1:
        per = per + (mean_est - scale * ALPHA / (N * m) * np.sum(sq * pm))
    assert abs(per.mean() - mean_est) < 1e-9 * abs(mean_est)
    se = per.std() / np.sqrt(N)
    truth = q @ x
    assert abs(mean_est - truth) < 5 * se
    assert abs(mean_est - truth) / abs(truth) < 0.005       # relative bias below 0.5%


def test_qjl_variance_matches_closed_form():
    # Var of the QJL estimate of <q, r>: ((pi/2) |q|^2 |r|^2 - <q, r>^2) / m.
    d, m = 16, 8
    rng = np.random.default_rng(20)
    r = rng.standard_normal(d)
    q = rng.standard_normal(d)
    N = 200_000
    S = rng.standard_normal((N * m, d))
    est = ((S @ q) * np.where(S @ r >= 0, 1.0, -1.0)).reshape(N, m).sum(1) * ALPHA / m * np.linalg.norm(r)
    want = ((np.pi / 2) * (q @ q) * (r @ r) - (q @ r) ** 2) / m
    assert abs(est.var() / want - 1.0) < 0.02


def test_distortion_of_key_reconstruction_falls_with_bits():
    d = 128
    rng = np.random.default_rng(4)
    X = rng.standard_normal((2000, d))
    err = []
    for b1 in (1, 2, 3, 4):
        p, (c32, b32) = _setup(d, 128, b1)
        k = quantize.quantize_keys(X, p["Pi"], p["S"], c32, b32, b1)
        err.append(np.mean(k["rnorm"].astype(np.float64) ** 2 / np.sum(X * X, 1)))
    ratios = [err[i] / err[i + 1] for i in range(3)]
    assert all(2.8 < r < 4.0 for r in ratios)          # [TQ] section 1: ~1/4^b


def test_recall_at_8_three_bit_keys():
    figs = page_figures()
    d, m, b1 = 128, 128, 2
    p, (c32, b32) = _setup(d, m, b1)
    rng = np.random.default_rng(5)
    X = rng.standard_normal((1024, d))
    Q = rng.standard_normal((64, d))
    keys = quantize.quantize_keys(X, p["Pi"], p["S"], c32, b32, b1)
    est = attention.logits_compressed(Q, keys, p["Pi"], p["S"], c32, b1)
    true = Q @ X.T
    rec = np.mean([len(set(np.argsort(-est[i])[:8]) & set(np.argsort(-true[i])[:8])) / 8
                   for i in range(Q.shape[0])])
    assert rec >= float(figs["recall_at_8_threshold"])


def test_value_quantisation_properties():
    rng = np.random.default_rng(6)
    V = rng.standard_normal((512, 128)).astype(np.float32)
    for vb, g in ((2, 32), (4, 32), (4, 64)):
        codes, s, mn = quantize.quantize_values(V, vb, g)
        vh = quantize.dequantize_values(codes, s, mn, g)
        assert codes.max() <= (1 << vb) - 1
        err = np.abs(vh - V.astype(np.float64)).reshape(512, -1, g)
        assert np.all(err <= 0.5 * s.astype(np.float64)[:, :, None] * (1 + 1e-6) + 1e-12)
        vg = V.reshape(512, -1, g)
        assert np.array_equal(mn, vg.min(2))
        assert np.all(codes.reshape(512, -1, g)[vg == vg.min(2, keepdims=True)] == 0)
        assert np.all(codes.reshape(512, -1, g)[vg == vg.max(2, keepdims=True)] == (1 << vb) - 1)


def test_value_cosine_similarity_matches_page():
    figs = page_figures()
    rng = np.random.default_rng(7)
    V = rng.standard_normal((4096, 128)).astype(np.float32)
    for vb, key in ((2, "value_cos_2bit"), (4, "value_cos_4bit")):
        codes, s, mn = quantize.quantize_values(V, vb, 32)
        vh = quantize.dequantize_values(codes, s, mn, 32)
        cos = np.mean(np.sum(vh * V, 1) / np.linalg.norm(vh, axis=1) / np.linalg.norm(V, axis=1))
        assert abs(cos - float(figs[key])) < 0.012


def test_value_constant_group_and_half_even_rounding():
    v = np.full((1, 32), 1.5, np.float32)
    codes, s, mn = quantize.quantize_values(v, 2, 32)
    assert s[0, 0] == 0 and np.all(codes == 0) and mn[0, 0] == np.float32(1.5)
    # group {0, 3, 1.5, 4.5, ...}: s = 1, (v - mn)/s = 1.5 and 4.5 -> rint half-even: 2, 4
    v = np.zeros((1, 32), np.float32)
    v[0, 1], v[0, 2] = 15.0, 7.5
    v[0, 3] = 2.5
    codes, s, _ = quantize.quantize_values(v, 4, 32)
    assert s[0, 0] == 1.0 and codes[0, 2] == 8 and codes[0, 3] == 2 and codes[0, 1] == 15


def test_exemption_masks():
    y = np.array([[0.1, -0.1, 1e-9, 0.5]], np.float32)
    beta = np.array([-0.1, 0.0, 0.1], np.float32)
    ex = quantize.code_exempt(y, beta)
    assert ex.tolist() == [[True, True, True, False]]
    z = np.array([[1.0, -1.0, 1e-7, 0.0]])
    assert quantize.sign_exempt(z).tolist() == [[False, False, True, True]]


def test_band_agreement_counts_planted_mismatches():
    """The comparison rule of the parity checks: a code flipped at an element
    inside the boundary band counts as in-band (and its token's signs are left
    out), a code flipped elsewhere and a sign flipped away from zero count as
    outside the band."""
    d, m, b1 = 16, 32, 2
    p, (c32, b32) = _setup(d, m, b1)
    rng = np.random.default_rng(5)
    X = rng.standard_normal((50, d))
    ref = quantize.quantize_keys(X, p["Pi"], p["S"], c32, b32, b1)
    same = quantize.band_agreement(ref["idx"].copy(), ref["bits"].copy(), ref, b32)
    assert same["outside_band"] == 0 and same["code_mismatch_in_band"] == 0
    # plant y exactly on a boundary for token 3, coordinate 2: that element is exempt
    ref2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in ref.items()}
    ref2["y32"][3, 2] = b32[1]
    idx = ref2["idx"].copy()
    idx[3, 2] ^= 1
    bits = ref2["bits"].copy()
    bits[3, 0] ^= 1                         # dropped: token 3 has a flipped code
    c = quantize.band_agreement(idx, bits, ref2, b32)
    assert c["code_mismatch_in_band"] == 1 and c["tokens_with_a_flipped_code"] == 1
    assert c["outside_band"] == 0
    idx[7, 5] = (idx[7, 5] + 2) % 4          # far from any boundary (checked below)
    assert not quantize.code_exempt(ref2["y32"], b32)[7, 5]
    bits[9, np.argmax(np.abs(ref2["z"][9]))] ^= 1     # the largest |z|: never exempt
    c = quantize.band_agreement(idx, bits, ref2, b32)
    assert c["outside_band"] == 2
