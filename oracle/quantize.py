"""Key and value quantisation, step by step as the pages state it.

Keys ([TQ] §二 three-stage pipeline, §五 ``ProdQuantized`` 4-tuple):
  1. rho = ||x||;  u = x / rho;  y = Pi u                      (normalise + rotate)
  2. idx_j = #{k : beta_k < y_j}                              (Lloyd-Max, b-1 bits)
  3. x~ = rho Pi^T c[idx];  r = x - x~;  z = S r;  bit_i = [z_i >= 0]; ||r||
                                                               (QJL residual sketch)
Pure QJL keys ([AQJL] §QJL): JL-project the key and keep only the sign:
  z = S x, bit_i = [z_i >= 0], plus rho.

Readings taken: y is rounded to fp32 before the boundary comparison (the codes
are decided in the kernel's precision, fp32); a value equal to a boundary goes
to the lower index; sign(0) = +1; a zero key gets u = 0 (so every code is the
one just below the middle boundary, r = 0, all sign bits 1, ||r|| = 0); the
residual is taken in the original space, unnormalised.

Values ([TQ] §二 table: 2 bits per dimension, plain min-max group quantisation;
§七: 4-bit for quality):  per token, per contiguous group of g channels, in
IEEE fp32 with this operation order:
  mn = min, mx = max, s = (mx - mn) / (2^vb - 1),
  code = clamp(rint((v - mn) / s), 0, 2^vb - 1)  (round half to even; 0 if s = 0),
  v^ = mn + code * s.
Readings taken: groups run along channels within one token; round half to
even; fp32 (s, mn) metadata (what reproduces the page's 4.41x figure).
"""
from __future__ import annotations

import numpy as np


def quantize_keys(K, Pi32, S32, c32, beta32, b1: int):
    """K: [n, d] real values (any float dtype; used in float64).

    Returns dict with idx [n,d] uint8 (absent for b1 = 0), bits [n,m] uint8 in
    {0,1}, rho [n] fp32, rnorm [n] fp32 (absent for b1 = 0), and the
    pre-quantisation values y32 [n,d] (fp32) and z [n,m] (float64) used to
    decide which elements lie near a decision boundary.
    """
    x = np.asarray(K, dtype=np.float64)
    S = np.asarray(S32, dtype=np.float64)
    rho = np.sqrt(np.sum(x * x, axis=1))
    out = {"rho": rho.astype(np.float32)}
    if b1 == 0:
        z = x @ S.T
        out["bits"] = (z >= 0).astype(np.uint8)
        out["z"] = z
        return out
    Pi = np.asarray(Pi32, dtype=np.float64)
    c = np.asarray(c32, dtype=np.float64)
    beta = np.asarray(beta32, dtype=np.float64)
    safe = np.where(rho > 0, rho, 1.0)
    u = np.where(rho[:, None] > 0, x / safe[:, None], 0.0)
    y32 = (u @ Pi.T).astype(np.float32)
    idx = np.sum(beta[None, None, :] < y32.astype(np.float64)[:, :, None], axis=2)
    x_tilde = rho[:, None] * (c[idx] @ Pi)
    r = x - x_tilde
    z = r @ S.T
    out.update(idx=idx.astype(np.uint8), bits=(z >= 0).astype(np.uint8),
               rnorm=np.sqrt(np.sum(r * r, axis=1)).astype(np.float32),
               y32=y32, z=z)
    return out


def quantize_values(V, vbits: int, group: int):
    """V: [n, d] values exactly representable in fp32.  Returns codes [n,d]
    uint8, scale [n, d/group] fp32, vmin [n, d/group] fp32 (all bit-exact)."""
    v = np.asarray(V, dtype=np.float32)
    n, d = v.shape
    vg = v.reshape(n, d // group, group)
    mn = vg.min(axis=2)
    mx = vg.max(axis=2)
    levels = np.float32((1 << vbits) - 1)
    s = (mx - mn) / levels                       # fp32 subtract, fp32 divide
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint((vg - mn[:, :, None]) / s[:, :, None])
    q = np.where(s[:, :, None] == 0, np.float32(0), q)
    q = np.clip(q, 0, levels)
    return q.reshape(n, d).astype(np.uint8), s.astype(np.float32), mn.astype(np.float32)


def dequantize_values(codes, scale, vmin, group: int):
    """v^ = mn + code * s, in float64 from the stored fp32 metadata."""
    n, d = codes.shape
    c = codes.astype(np.float64).reshape(n, d // group, group)
    out = vmin.astype(np.float64)[:, :, None] + c * scale.astype(np.float64)[:, :, None]
    return out.reshape(n, d)


def code_exempt(y32, beta32, rel: float = 1e-5):
    """[n,d] bool: y lies within rel of a decision boundary.  The band around a
    boundary beta is rel * max(|beta|, ||y||/sqrt(d)): relative to the boundary,
    or to the rms coordinate for the boundary at zero."""
    y = np.asarray(y32, dtype=np.float64)
    d = y.shape[1]
    scale = np.sqrt(np.sum(y * y, axis=1, keepdims=True)) / np.sqrt(d)
    beta = np.asarray(beta32, dtype=np.float64)
    band = rel * np.maximum(np.abs(beta)[None, None, :], scale[:, :, None])
    return np.any(np.abs(y[:, :, None] - beta[None, None, :]) <= band, axis=2)


def sign_exempt(z, rel: float = 1e-5):
    """[n,m] bool: |z_i| <= rel * ||z|| / sqrt(m) (relative to the rms entry)."""
    z = np.asarray(z, dtype=np.float64)
    m = z.shape[1]
    return np.abs(z) <= rel * np.sqrt(np.sum(z * z, axis=1, keepdims=True)) / np.sqrt(m)


def band_agreement(idx_got, bits_got, ref: dict, beta32) -> dict:
    """Codes and sign bits decided elsewhere (idx_got [n, d] or None for pure QJL,
    bits_got [n, m]) against this oracle's (``ref``: the quantize_keys output,
    with its fp32 y and its z).  A code may differ only where ``code_exempt``
    holds and a sign bit only where ``sign_exempt`` holds; a token with a
    differing code has its sign bits left out (they depend on the code).
    Returns the counts; ``outside_band`` > 0 means a disagreement."""
    n = ref["bits"].shape[0]
    flipped = np.zeros(n, bool)
    code_mis = code_out = 0
    if idx_got is not None:
        mis = np.asarray(idx_got) != ref["idx"]
        ex = code_exempt(ref["y32"], beta32)
        code_mis = int(mis.sum())
        code_out = int((mis & ~ex).sum())
        flipped = np.any(mis, axis=1)
    smis = (np.asarray(bits_got) != ref["bits"]) & ~flipped[:, None]
    sign_out = int((smis & ~sign_exempt(ref["z"])).sum())
    return {"tokens": int(n), "code_mismatch_in_band": code_mis - code_out,
            "sign_mismatch_in_band": int(smis.sum()) - sign_out,
            "tokens_with_a_flipped_code": int(flipped.sum()),
            "outside_band": code_out + sign_out}
