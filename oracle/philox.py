"""Philox4x64-10 and the Box-Muller Gaussian used for the random projections.

The pages fix only that Pi and S are random (QR of a Gaussian matrix, a
Gaussian S) with the per-layer seed 42 + 7*layer ([TQ] §二, §六); they name no
generator.  Reading taken: the counter-based Philox4x64 with 10 rounds from
Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as easy as 1, 2, 3"
(SC'11), so that the CPU and GPU sides can each implement the same published
generator independently.

Draw k of stream s under seed q: counter (k, 0, 0, 0), key (q, s); words w0, w1
give u_i = ((w_i >> 11) + 0.5) * 2^-53 in (0, 1] (double rounding of the
largest values gives exactly 1; never 0, so the logarithm is finite); z = sqrt(-2 ln u0) cos(2 pi u1).
"""
from __future__ import annotations

import numpy as np

# Round multipliers and Weyl key increments of Philox4x64 (Salmon et al., SC'11).
PHILOX_M0 = np.uint64(0xD2E7470EE14C6C93)
PHILOX_M1 = np.uint64(0xCA5A826395121157)
PHILOX_W0 = np.uint64(0x9E3779B97F4A7C15)
PHILOX_W1 = np.uint64(0xBB67AE8584CAA73B)

_M32 = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)


def mulhilo64(a: np.ndarray, b: np.uint64):
    """Full 64x64 -> 128-bit product of uint64 arrays, as (hi, lo), via 32-bit limbs."""
    a = np.asarray(a, dtype=np.uint64)
    b = np.uint64(b)
    al, ah = a & _M32, a >> _S32
    bl, bh = b & _M32, b >> _S32
    ll = al * bl
    lh = al * bh
    hl = ah * bl
    hh = ah * bh
    mid = (ll >> _S32) + (lh & _M32) + (hl & _M32)
    lo = (ll & _M32) | ((mid & _M32) << _S32)
    hi = hh + (lh >> _S32) + (hl >> _S32) + (mid >> _S32)
    return hi, lo


def philox4x64_10(ctr, key):
    """Philox4x64 with 10 rounds.  ``ctr``: 4 uint64 arrays (broadcastable);
    ``key``: 2 uint64 scalars.  Returns the 4 output words."""
    with np.errstate(over="ignore"):
        c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) for c in ctr)
        k0, k1 = np.uint64(key[0]), np.uint64(key[1])
        for r in range(10):
            if r > 0:
                k0 = np.uint64((int(k0) + int(PHILOX_W0)) & 0xFFFFFFFFFFFFFFFF)
                k1 = np.uint64((int(k1) + int(PHILOX_W1)) & 0xFFFFFFFFFFFFFFFF)
            hi0, lo0 = mulhilo64(c0, PHILOX_M0)
            hi1, lo1 = mulhilo64(c2, PHILOX_M1)
            c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def uniform53(w: np.ndarray) -> np.ndarray:
    """Top 53 bits of a 64-bit word, offset by half a step: a double in (0, 1]."""
    return ((np.asarray(w, dtype=np.uint64) >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53


TWO_PI = 6.283185307179586  # the double nearest 2*pi


def gaussian(n: int, seed: int, stream: int) -> np.ndarray:
    """Draws 0..n-1 of a stream: standard normal doubles (Box-Muller, cosine branch)."""
    k = np.arange(n, dtype=np.uint64)
    zero = np.zeros_like(k)
    w0, w1, _, _ = philox4x64_10((k, zero, zero, zero), (seed, stream))
    u0 = uniform53(w0)
    u1 = uniform53(w1)
    return np.sqrt(-2.0 * np.log(u0)) * np.cos(TWO_PI * u1)
