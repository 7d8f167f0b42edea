"""Compressed KV store with a full-precision ring of recent tokens.

[TQ] §六: the store appends chunk by chunk into a flat cache (the page's store
concatenates lazily; here the flat cache is the preallocated byte layout of
``oracle.layout``); the most recent tokens stay at full precision in a ring
buffer and the compressed path covers the older history.

Semantics (reading taken): after every append the ring holds the last
min(W, total) tokens; every older token has been quantised, in token order,
exactly once; tokens leave the ring oldest first.  Token t sits in ring slot
t mod W.  All sequences of the batch advance together.
"""
from __future__ import annotations

import numpy as np

from . import attention, layout, quantize


class OracleCache:
    def __init__(self, B, Hkv, d, b1, m, vbits, group, W, capacity, dtype, proj, cb):
        self.lay = layout.Layout(B, Hkv, d, b1, m, vbits, group, W, capacity, dtype)
        self.B, self.Hkv, self.d, self.b1, self.m = B, Hkv, d, b1, m
        self.vbits, self.group, self.W, self.capacity, self.dtype = vbits, group, W, capacity, dtype
        self.proj, self.cb = proj, cb           # proj: dict Pi/S; cb: (centroids, boundaries)
        self.n_total = 0
        self.ring_k = np.zeros((B, Hkv, max(W, 1), d))
        self.ring_v = np.zeros((B, Hkv, max(W, 1), d))
        self.rec = [[None for _ in range(Hkv)] for _ in range(B)]   # dict of arrays per (b, h)

    @property
    def n_comp(self) -> int:
        return max(0, self.n_total - self.W)

    @property
    def n_ring(self) -> int:
        return min(self.W, self.n_total)

    def quantize_tokens(self, k, v):
        """Quantise n tokens of one (b, h): k, v [n, d] -> record dict."""
        c32, beta32 = self.cb if self.cb is not None else (None, None)
        keys = quantize.quantize_keys(k, self.proj["Pi"], self.proj["S"], c32, beta32, self.b1)
        codes, scale, vmin = quantize.quantize_values(v, self.vbits, self.group)
        keys.update(codes=codes, scale=scale, vmin=vmin)
        return keys

    def append(self, K, V):
        """K, V: [B, Hkv, n, d] values of the input dtype."""
        K = np.asarray(K, dtype=np.float64)
        V = np.asarray(V, dtype=np.float64)
        n = K.shape[2]
        n_old, n_tot = self.n_total, self.n_total + n
        c_old, c_new = max(0, n_old - self.W), max(0, n_tot - self.W)
        if c_new > self.capacity:
            raise ValueError("capacity exceeded")
        for b in range(self.B):
            for h in range(self.Hkv):
                from_ring = np.arange(c_old, min(c_new, n_old))
                from_new = np.arange(max(c_old, n_old), c_new) - n_old
                ks = np.concatenate((self.ring_k[b, h, from_ring % max(self.W, 1)],
                                     K[b, h, from_new]), axis=0)
                vs = np.concatenate((self.ring_v[b, h, from_ring % max(self.W, 1)],
                                     V[b, h, from_new]), axis=0)
                if ks.shape[0]:
                    r = self.quantize_tokens(ks, vs.astype(np.float32))
                    old = self.rec[b][h]
                    self.rec[b][h] = r if old is None else {
                        key: np.concatenate((old[key], r[key]), axis=0) for key in r}
                keep = np.arange(max(n_old, n_tot - self.W), n_tot)
                if keep.size:
                    self.ring_k[b, h, keep % self.W] = K[b, h, keep - n_old]
                    self.ring_v[b, h, keep % self.W] = V[b, h, keep - n_old]
        self.n_total = n_tot

    def ring_slots(self):
        """Ring slots holding tokens, oldest first."""
        return [t % self.W for t in range(self.n_total - self.n_ring, self.n_total)]

    def to_bytes(self) -> np.ndarray:
        """The whole cache buffer in the layout of ``oracle.layout`` (unused bytes 0)."""
        lay = self.lay
        buf = np.zeros(lay.total_bytes, dtype=np.uint8)
        for b in range(self.B):
            for h in range(self.Hkv):
                r = self.rec[b][h]
                if r is None:
                    continue
                f = layout.token_fields(r, r["codes"], r["scale"], r["vmin"], lay)
                layout.write_region(buf, lay, b, h, 0, f)
        if self.W > 0:
            for off, ring in ((lay.ring_k_off, self.ring_k), (lay.ring_v_off, self.ring_v)):
                raw = _to_dtype_bytes(ring[:, :, :self.W, :], self.dtype)
                buf[off:off + raw.size] = raw
        return buf

    def decode(self, Q, scale=None):
        """Q: [B, Hq, d].  Returns (out [B, Hq, d], logits list per (b, h) of [G, n])."""
        Q = np.asarray(Q, dtype=np.float64)
        Hq = Q.shape[1]
        G = Hq // self.Hkv
        scale = 1.0 / np.sqrt(self.d) if scale is None else scale
        out = np.zeros((self.B, Hq, self.d))
        logits = {}
        slots = self.ring_slots()
        for b in range(self.B):
            for h in range(self.Hkv):
                r = self.rec[b][h]
                vhat = (quantize.dequantize_values(r["codes"], r["scale"], r["vmin"], self.group)
                        if r is not None else np.zeros((0, self.d)))
                rk = self.ring_k[b, h, slots] if slots else None
                rv = self.ring_v[b, h, slots] if slots else None
                o, lg = attention.decode_group(
                    Q[b, h * G:(h + 1) * G], r, vhat, rk, rv, self.proj.get("Pi"),
                    self.proj["S"], self.cb[0] if self.cb is not None else None, self.b1, scale)
                out[b, h * G:(h + 1) * G] = o
                logits[(b, h)] = lg
        return out, logits


    def prefill(self, Q, Knew, Vnew, scale=None):
        """Attention of a chunk of n new tokens before they are appended (the cache is
        not changed).  Q: [B, n, Hq, d] (token-major); Knew, Vnew: [B, Hkv, n, d] as
        ``append`` takes them.  Returns out [B, n, Hq, d]."""
        Q = np.asarray(Q, dtype=np.float64)
        Knew = np.asarray(Knew, dtype=np.float64)
        Vnew = np.asarray(Vnew, dtype=np.float64)
        n, Hq = Q.shape[1], Q.shape[2]
        G = Hq // self.Hkv
        scale = 1.0 / np.sqrt(self.d) if scale is None else scale
        out = np.zeros((self.B, n, Hq, self.d))
        slots = self.ring_slots()
        for b in range(self.B):
            for h in range(self.Hkv):
                r = self.rec[b][h]
                vhat = (quantize.dequantize_values(r["codes"], r["scale"], r["vmin"], self.group)
                        if r is not None else np.zeros((0, self.d)))
                rk = self.ring_k[b, h, slots] if slots else None
                rv = self.ring_v[b, h, slots] if slots else None
                out[b, :, h * G:(h + 1) * G] = attention.prefill_group(
                    Q[b, :, h * G:(h + 1) * G], r, vhat, rk, rv, Knew[b, h], Vnew[b, h],
                    self.proj.get("Pi"), self.proj["S"], self.cb[0] if self.cb is not None else None,
                    self.b1, scale)
        return out


def _to_dtype_bytes(x, dtype: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return np.ascontiguousarray(x.astype("<f4")).view(np.uint8).ravel()
    if dtype == "f16":
        return np.ascontiguousarray(x.astype("<f2")).view(np.uint8).ravel()
    # bf16: the values are exactly representable, so the top half of the fp32 pattern.
    u = np.ascontiguousarray(x.astype("<f4")).view("<u4")
    return np.ascontiguousarray((u >> 16).astype("<u2")).view(np.uint8).ravel()
