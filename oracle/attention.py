"""Logits on the compressed keys and single-token decode attention.

Estimator ([TQ] §四, §五, §六): for a query q and a stored key
(idx, sign bits, ||r||, rho)
    <q, x> ~ rho <Pi q, c[idx]> + ||r|| sqrt(pi/2)/m <S q, 2 bits - 1>,
whose expectation over S is <q, x>: the first term is <q, x~> (Pi orthogonal),
the second is the QJL estimate of <q, r>.  The page writes sqrt(pi/2)/d because
its sketch has m = d rows; it is 1/m in general.  The query is rotated forward
(Pi q) and sketched once (S q) instead of rotating keys back ([TQ] §六).

Pure QJL keys ([AQJL] §QJL, asymmetric estimator): <q, x> ~ rho sqrt(pi/2)/m <S q, 2 bits - 1>.

Decode ([TQ] §六 fused decode attention, ring buffer): logits over the
compressed tokens plus exact <q, k> over the ring tokens, softmax with scale
1/sqrt(d) (reading taken: the standard scale), output sum_t p_t v^_t with
v^ = mn + code * s for compressed tokens and the exact v for ring tokens.  GQA:
query head hq reads KV head hq // (Hq / Hkv).  All float64, dense softmax.

Multi-token (chunked prefill) attention over the same store ([TQ] §六 for the
history and the ring; §七 notes that the page's own hybrid path dequantises the
history for this step): a chunk of n new tokens is scored before it is
appended.  Readings taken where the pages are silent: query i of the chunk sees
the compressed history (estimator logits, v^ values), the ring (exact), and the
chunk's own tokens 0..i (exact keys and values in their input precision, causal
order, the query's own token included); the softmax scale is the decode's.
"""
from __future__ import annotations

import numpy as np

ALPHA = np.sqrt(np.pi / 2.0)


def logits_compressed(q, keys: dict, Pi32, S32, c32, b1: int):
    """q: [G, d] queries of one GQA group; keys: record dict of n tokens.
    Returns unscaled logits [G, n] (float64)."""
    q = np.asarray(q, dtype=np.float64)
    S = np.asarray(S32, dtype=np.float64)
    m = S.shape[0]
    sq = q @ S.T                                        # [G, m]  (S q)
    pm = 2.0 * keys["bits"].astype(np.float64) - 1.0    # [n, m]  (+-1)
    qjl = (ALPHA / m) * (sq @ pm.T)                     # [G, n]
    if b1 == 0:
        return keys["rho"].astype(np.float64)[None, :] * qjl
    Pi = np.asarray(Pi32, dtype=np.float64)
    c = np.asarray(c32, dtype=np.float64)
    qr = q @ Pi.T                                       # [G, d]  (Pi q)
    mse = qr @ c[keys["idx"]].T                         # [G, n]  <Pi q, c[idx]>
    return (keys["rho"].astype(np.float64)[None, :] * mse
            + keys["rnorm"].astype(np.float64)[None, :] * qjl)


def softmax_attention(logits, values, scale: float):
    """o = softmax(scale * logits) @ values; logits [G, n], values [n, d]."""
    s = scale * np.asarray(logits, dtype=np.float64)
    s = s - np.max(s, axis=1, keepdims=True)
    p = np.exp(s)
    p /= np.sum(p, axis=1, keepdims=True)
    return p @ np.asarray(values, dtype=np.float64)


def decode_group(q, comp_keys, comp_vhat, ring_k, ring_v, Pi32, S32, c32, b1: int,
                 scale: float):
    """One (batch, KV head): q [G, d]; comp_keys record of n_c tokens (or None);
    comp_vhat [n_c, d]; ring_k / ring_v [n_r, d].  Returns (out [G, d], logits [G, n_c + n_r])."""
    q = np.asarray(q, dtype=np.float64)
    parts_l, parts_v = [], []
    if comp_keys is not None and comp_vhat.shape[0] > 0:
        parts_l.append(logits_compressed(q, comp_keys, Pi32, S32, c32, b1))
        parts_v.append(np.asarray(comp_vhat, dtype=np.float64))
    if ring_k is not None and ring_k.shape[0] > 0:
        parts_l.append(q @ np.asarray(ring_k, dtype=np.float64).T)
        parts_v.append(np.asarray(ring_v, dtype=np.float64))
    logits = np.concatenate(parts_l, axis=1)
    values = np.concatenate(parts_v, axis=0)
    return softmax_attention(logits, values, scale), logits


def prefill_group(Qg, comp_keys, comp_vhat, ring_k, ring_v, new_k, new_v, Pi32, S32, c32, b1: int,
                  scale: float):
    """One (batch, KV head) of a chunk: Qg [n, G, d] the queries of the chunk's n tokens;
    new_k / new_v [n, d] the chunk's keys and values.  Query i is a decode over the
    history plus an exact segment of the ring followed by chunk tokens 0..i.
    Returns out [n, G, d]."""
    Qg = np.asarray(Qg, dtype=np.float64)
    n, G, d = Qg.shape
    new_k = np.asarray(new_k, dtype=np.float64)
    new_v = np.asarray(new_v, dtype=np.float64)
    rk0 = np.zeros((0, d)) if ring_k is None else np.asarray(ring_k, dtype=np.float64)
    rv0 = np.zeros((0, d)) if ring_v is None else np.asarray(ring_v, dtype=np.float64)
    out = np.zeros((n, G, d))
    for i in range(n):
        ek = np.concatenate((rk0, new_k[:i + 1]), axis=0)
        ev = np.concatenate((rv0, new_v[:i + 1]), axis=0)
        out[i], _ = decode_group(Qg[i], comp_keys, comp_vhat, ek, ev, Pi32, S32, c32, b1, scale)
    return out
