"""Pins of the oracle's multi-token (chunked prefill) attention.

The oracle scores a chunk of new tokens against the compressed history, the ring
and, causally, the chunk itself.  Pinned here against things other than the
oracle's own loop: causal softmax attention written out with scalar loops, the
decode of a cache whose ring is wide enough to hold the chunk's tokens, and the
causal mask (later tokens of the chunk must not move an earlier query).
"""
import math

import numpy as np

from oracle import cache, codebook, projections


def _bf16(x):
    u = np.asarray(x, np.float32).view(np.uint32)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def _mk(W, B=2, Hkv=2, d=64, b1=2, m=64, cap=400):
    p = projections.make_projections(d, m, 0)
    cb = codebook.build(d, b1) if b1 > 0 else None
    return cache.OracleCache(B, Hkv, d, b1, m, 2, 32, W, cap, "bf16", p, cb)


def _inputs(seed, B, Hkv, Hq, n_hist, n, d):
    rng = np.random.default_rng(seed)
    K = _bf16(rng.standard_normal((B, Hkv, n_hist + n, d)))
    V = _bf16(rng.standard_normal((B, Hkv, n_hist + n, d)))
    Q = rng.standard_normal((B, n, Hq, d))
    return K, V, Q


def test_prefill_without_history_is_causal_attention_by_scalar_loops():
    """No compressed tokens (history shorter than the ring): every key is exact, so
    query i of the chunk is softmax attention over the ring tokens and chunk tokens
    0..i, here summed term by term."""
    B, Hkv, Hq, d, W, n_hist, n = 1, 2, 4, 64, 16, 6, 5
    c = _mk(W, B=B, Hkv=Hkv, d=d)
    K, V, Q = _inputs(1, B, Hkv, Hq, n_hist, n, d)
    c.append(K[:, :, :n_hist], V[:, :, :n_hist])
    assert c.n_comp == 0
    out = c.prefill(Q, K[:, :, n_hist:], V[:, :, n_hist:])
    G = Hq // Hkv
    for b in range(B):
        for i in range(n):
            for hq in range(Hq):
                h = hq // G
                visible = list(range(n_hist + i + 1))     # history (all in the ring) + chunk 0..i
                s = []
                for t in visible:
                    acc = 0.0
                    for j in range(d):
                        acc += float(Q[b, i, hq, j]) * float(K[b, h, t, j])
                    s.append(acc / math.sqrt(d))
                mx = max(s)
                e = [math.exp(x - mx) for x in s]
                z = sum(e)
                for ch in range(0, d, 7):
                    want = sum(e[k] * float(V[b, h, t, ch]) for k, t in enumerate(visible)) / z
                    assert abs(out[b, i, hq, ch] - want) < 1e-12


def test_prefill_equals_decode_with_a_wider_ring():
    """Query i of a chunk scored before the append equals a decode of a cache whose
    ring is i + 1 slots wider and which has appended chunk tokens 0..i: that cache
    compresses the same history tokens and keeps the same ring tokens plus chunk
    tokens 0..i at full precision."""
    B, Hkv, Hq, d, W, n_hist, n = 2, 2, 8, 64, 16, 77, 4
    for b1 in (2, 0):
        c = _mk(W, B=B, Hkv=Hkv, d=d, b1=b1)
        K, V, Q = _inputs(2 + b1, B, Hkv, Hq, n_hist, n, d)
        c.append(K[:, :, :n_hist], V[:, :, :n_hist])
        assert c.n_comp == n_hist - W
        out = c.prefill(Q, K[:, :, n_hist:], V[:, :, n_hist:])
        for i in range(n):
            wide = _mk(W + i + 1, B=B, Hkv=Hkv, d=d, b1=b1)
            wide.append(K[:, :, :n_hist], V[:, :, :n_hist])
            wide.append(K[:, :, n_hist:n_hist + i + 1], V[:, :, n_hist:n_hist + i + 1])
            assert wide.n_comp == c.n_comp
            want, _ = wide.decode(Q[:, i])
            assert np.max(np.abs(out[:, i] - want)) < 1e-12


def test_prefill_is_causal():
    """Changing chunk token j moves queries i >= j and leaves queries i < j bit-identical."""
    B, Hkv, Hq, d, W, n_hist, n, j = 1, 2, 4, 64, 8, 50, 6, 3
    c = _mk(W, B=B, Hkv=Hkv, d=d)
    K, V, Q = _inputs(4, B, Hkv, Hq, n_hist, n, d)
    c.append(K[:, :, :n_hist], V[:, :, :n_hist])
    Kn, Vn = K[:, :, n_hist:].copy(), V[:, :, n_hist:].copy()
    base = c.prefill(Q, Kn, Vn)
    Kn[:, :, j] += 3.0
    Vn[:, :, j] -= 2.0
    moved = c.prefill(Q, Kn, Vn)
    assert np.array_equal(base[:, :j], moved[:, :j])
    assert np.all(np.max(np.abs(base[:, j:] - moved[:, j:]), axis=-1) > 1e-6)


def test_prefill_single_token_of_an_empty_cache_is_its_value():
    """The first token of an empty cache sees only itself: out = v."""
    c = _mk(4, B=1, Hkv=1, d=64)
    K, V, Q = _inputs(5, 1, 1, 2, 0, 1, 64)
    out = c.prefill(Q, K, V)
    assert np.max(np.abs(out[0, 0] - V[0, 0, 0][None, :])) < 1e-12
