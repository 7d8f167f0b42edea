"""Byte layout of the packed compressed KV cache.

[TQ] §二: the d sign bits are packed into d/8 bytes and stored with ||r||;
§五: ``quantize()`` yields the 4-tuple (MSE indices, QJL sign bytes, residual
norm, original norm), all bit-packed.  Everything beyond that is a format
choice of this project, written down here and in the library's header:

Token record (little-endian, LSB-first bit order):
  idx    b1 bit-planes of d bits each: plane p, byte j>>3, bit j&7 = bit p of idx_j
  signs  m bits: byte i>>3, bit i&7 = [z_i >= 0]
  rho    fp32 ||x||
  rnorm  fp32 ||r||           (absent when b1 = 0, pure QJL)
  vcodes d codes of vb bits: code j at byte (j*vb)>>3, bit (j*vb)&7
  vscale d/g fp32 scales
  vmin   d/g fp32 minima

Block: TB = 64 consecutive tokens, stored field by field (all 64 idx records,
then all 64 sign records, ...); every field is a multiple of 16 bytes long, so
a block is one contiguous, 16-byte aligned chunk.  The value codes of a block
are the one field not stored token by token: they form 32 token-pair records
(tokens 2i and 2i+1 of the block), each of d*vb/16 little-endian 32-bit words.
Cut a token's vcodes (above) into 16-bit halves, half x holding the 16/vb
channels starting at (16/vb)*x; with H = g*vb/16 halves per value group and
NG = d/g groups, half x = gi*H + s of token 2i goes to the low 16 bits and that
of token 2i+1 to the high 16 bits of word s*NG + gi of the pair record.

Cache buffer: for each (batch b, kv head h) a region of ceil(capacity/TB)
blocks, regions in (b, h) order; then, at the next 256-byte boundary, the ring
of keys [B, Hkv, W, d] in the input dtype, then (256-aligned) the ring of
values.  A token with absolute index t lives in ring slot t mod W.
"""
from __future__ import annotations

import numpy as np

TB = 64
_ESIZE = {"f32": 4, "f16": 2, "bf16": 2}


def _align(x: int, a: int) -> int:
    return (x + a - 1) // a * a


class Layout:
    def __init__(self, B, Hkv, d, b1, m, vbits, group, W, capacity, dtype):
        self.B, self.Hkv, self.d, self.b1, self.m = B, Hkv, d, b1, m
        self.vbits, self.group, self.W, self.capacity, self.dtype = vbits, group, W, capacity, dtype
        self.f_idx = b1 * d // 8
        self.f_sign = m // 8
        self.f_rho = 4
        self.f_rnorm = 4 if b1 > 0 else 0
        self.f_vcode = d * vbits // 8
        self.f_vmeta = 4 * (d // group)
        self.token_bytes = (self.f_idx + self.f_sign + self.f_rho + self.f_rnorm
                            + self.f_vcode + 2 * self.f_vmeta)
        sizes = [self.f_idx, self.f_sign, self.f_rho, self.f_rnorm, self.f_vcode,
                 self.f_vmeta, self.f_vmeta]
        offs, o = [], 0
        for s in sizes:
            offs.append(o)
            o += TB * s
        (self.o_idx, self.o_sign, self.o_rho, self.o_rnorm, self.o_vcode,
         self.o_vscale, self.o_vmin) = offs
        self.block_bytes = o
        self.nblk = (capacity + TB - 1) // TB
        self.region_bytes = self.nblk * self.block_bytes
        self.packed_bytes = B * Hkv * self.region_bytes
        es = _ESIZE[dtype]
        self.ring_bytes = B * Hkv * W * d * es
        self.ring_k_off = _align(self.packed_bytes, 256)
        self.ring_v_off = _align(self.ring_k_off + self.ring_bytes, 256)
        self.total_bytes = _align(self.ring_v_off + self.ring_bytes, 256)

    def region_off(self, b: int, h: int) -> int:
        return (b * self.Hkv + h) * self.region_bytes


def pack_bits(bits) -> np.ndarray:
    """[n, nbits] {0,1} -> [n, nbits/8] bytes, bit i at byte i>>3, bit i&7."""
    return np.packbits(np.asarray(bits, dtype=np.uint8), axis=1, bitorder="little")


def unpack_bits(packed, nbits: int) -> np.ndarray:
    return np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1, count=nbits,
                         bitorder="little")


def pack_codes(codes, vbits: int) -> np.ndarray:
    """[n, d] codes < 2^vbits -> [n, d*vbits/8] bytes, code j at bit (j*vb)&7 of
    byte (j*vb)>>3."""
    c = np.asarray(codes, dtype=np.uint8)
    n, d = c.shape
    per = 8 // vbits
    c = c.reshape(n, d // per, per).astype(np.uint16)
    out = np.zeros((n, d // per), dtype=np.uint16)
    for k in range(per):
        out |= c[:, :, k] << (k * vbits)
    return out.astype(np.uint8)


def unpack_codes(packed, vbits: int, d: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    per = 8 // vbits
    mask = (1 << vbits) - 1
    out = np.stack([(p >> (k * vbits)) & mask for k in range(per)], axis=2)
    return out.reshape(p.shape[0], d).astype(np.uint8)


def token_fields(keys: dict, codes, scale, vmin, lay: Layout) -> dict:
    """Per-token byte fields for n tokens (dict of [n, field_bytes] uint8)."""
    n = codes.shape[0]
    f = {}
    if lay.b1 > 0:
        planes = [pack_bits((keys["idx"] >> p) & 1) for p in range(lay.b1)]
        f["idx"] = np.concatenate(planes, axis=1)
    else:
        f["idx"] = np.zeros((n, 0), np.uint8)
    f["sign"] = pack_bits(keys["bits"])
    f["rho"] = np.ascontiguousarray(keys["rho"].astype("<f4")).view(np.uint8).reshape(n, 4)
    if lay.b1 > 0:
        f["rnorm"] = np.ascontiguousarray(keys["rnorm"].astype("<f4")).view(np.uint8).reshape(n, 4)
    else:
        f["rnorm"] = np.zeros((n, 0), np.uint8)
    f["vcode"] = pack_codes(codes, lay.vbits)
    f["vscale"] = np.ascontiguousarray(scale.astype("<f4")).view(np.uint8).reshape(n, -1)
    f["vmin"] = np.ascontiguousarray(vmin.astype("<f4")).view(np.uint8).reshape(n, -1)
    return f


_FIELDS = ("idx", "sign", "rho", "rnorm", "vcode", "vscale", "vmin")


def _field_geom(lay: Layout):
    return {"idx": (lay.o_idx, lay.f_idx), "sign": (lay.o_sign, lay.f_sign),
            "rho": (lay.o_rho, lay.f_rho), "rnorm": (lay.o_rnorm, lay.f_rnorm),
            "vcode": (lay.o_vcode, lay.f_vcode), "vscale": (lay.o_vscale, lay.f_vmeta),
            "vmin": (lay.o_vmin, lay.f_vmeta)}


def _dest(lay: Layout, b: int, h: int, t, name: str):
    """Byte addresses [n, size] of field ``name`` of tokens t (array) in region (b, h)."""
    off, size = _field_geom(lay)[name]
    t = np.asarray(t, dtype=np.int64)
    blk = lay.region_off(b, h) + (t // TB) * lay.block_bytes + off
    k = np.arange(size, dtype=np.int64)[None, :]
    if name != "vcode":
        return (blk + (t % TB) * size)[:, None] + k
    # byte k of the token's vcodes: half x = k // 2, byte k % 2 of that half
    H = lay.group * lay.vbits // 16
    NG = lay.d // lay.group
    x = k // 2
    word = (x % H) * NG + x // H
    tt = t % TB
    pair = blk + (tt // 2) * (2 * size) + 2 * (tt % 2)
    return pair[:, None] + 4 * word + k % 2


def write_region(buf: np.ndarray, lay: Layout, b: int, h: int, t0: int, fields: dict):
    """Write the fields of tokens t0 .. t0+n-1 of region (b, h) into ``buf``."""
    n = fields["sign"].shape[0]
    t = np.arange(t0, t0 + n)
    for name in _FIELDS:
        if _field_geom(lay)[name][1]:
            buf[_dest(lay, b, h, t, name)] = fields[name]


def read_region(buf: np.ndarray, lay: Layout, b: int, h: int, n: int) -> dict:
    """Fields of tokens 0 .. n-1 of region (b, h) (inverse of ``write_region``)."""
    t = np.arange(n)
    out = {}
    for name in _FIELDS:
        size = _field_geom(lay)[name][1]
        out[name] = buf[_dest(lay, b, h, t, name)] if size else np.zeros((n, 0), np.uint8)
    return out


def decode_fields(f: dict, lay: Layout) -> dict:
    """Unpack byte fields back to (idx, bits, rho, rnorm, codes, scale, vmin)."""
    n = f["sign"].shape[0]
    out = {"bits": unpack_bits(f["sign"], lay.m),
           "rho": np.ascontiguousarray(f["rho"]).view("<f4").reshape(n)}
    if lay.b1 > 0:
        nb = lay.d // 8
        idx = np.zeros((n, lay.d), np.uint8)
        for p in range(lay.b1):
            idx |= unpack_bits(f["idx"][:, p * nb:(p + 1) * nb], lay.d) << p
        out["idx"] = idx
        out["rnorm"] = np.ascontiguousarray(f["rnorm"]).view("<f4").reshape(n)
    out["codes"] = unpack_codes(f["vcode"], lay.vbits, lay.d)
    out["scale"] = np.ascontiguousarray(f["vscale"]).view("<f4").reshape(n, -1)
    out["vmin"] = np.ascontiguousarray(f["vmin"]).view("<f4").reshape(n, -1)
    return out
