"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module holds no arithmetic of the compression method: it only draws keys,
values and queries with the shapes and value distributions of the five
workloads below, and rounds them to the storage dtype.  Both sides of a parity
test receive the very same tensor from here.

Generation uses ``torch.Generator`` on the device the caller asks for, seeded
from ``(seed, layer, tensor_id)``; the draws on CPU and on CUDA differ, so a
test draws once and hands that one tensor to both the oracle and the library.

Tensor ids: K=1, V=2, Q=3, outlier-channel choice=4, per-token norm factor=5.

Workloads (statement of each: the workload's own description):

* ``tiny``     d=128, 512 cached tokens, 1 KV head, fp32.  Keys N(0,1) with 4
               outlier channels x10; values N(0,1); 4 queries N(0,1).
               3-bit keys (2-bit Lloyd-Max + 1-bit QJL, m=128), 2-bit values,
               group 32.  The four single-head decodes are run as one decode
               with 4 query heads over the one KV head (identical arithmetic).
* ``gqa32k``   batch 8, 32 query heads over 8 KV heads, d=128, context 32768,
               bf16, K/V N(0,1) with 2% of channels (3 of 128) x8, ring of 16.
* ``quant``    8 KV heads, d=128, 131072 tokens appended in chunks of 4096,
               bf16, K and V = N(0,I) * exp(0.5 * N(0,1)) per token.
* ``aqjl``     32 layers, m = 512/384/256/192 for layer groups 0-7/8-15/16-23/
               24-31, pure 1-bit QJL keys, fp16, key variance 1 + 2*l/31,
               batch 16, 32 query heads over 8 KV heads, context 65536.
* ``wide``     batch 4, 16 query heads over 4 KV heads, d=256, context 262144,
               bf16, K/V N(0,1) with 1% of channels (3 of 256) x10; 4-bit keys
               (3-bit Lloyd-Max + QJL m=256), 4-bit values group 64.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

TENSOR_K, TENSOR_V, TENSOR_Q, TENSOR_OUTLIER, TENSOR_NORM = 1, 2, 3, 4, 5

_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int                 # tokens in the cache at decode time (or appended)
    W: int                 # full-precision ring size
    b1: int                # Lloyd-Max bits per coordinate (0 = pure QJL)
    m: int                 # sketch dimension (layer 0's for multi-layer)
    vbits: int
    group: int
    dtype: str             # "f32" | "f16" | "bf16"
    seed: int = 0
    layers: int = 1
    k_outlier_frac: float = 0.0     # fraction of channels scaled (keys)
    v_outlier_frac: float = 0.0     # fraction of channels scaled (values)
    k_outlier_count: int = 0        # explicit count (overrides the fraction)
    outlier_scale: float = 1.0
    lognormal_sigma: float = 0.0    # per-token norm factor exp(sigma * N(0,1))
    var_ramp: bool = False          # key variance 1 + 2*l/(layers-1)
    chunk: int = 0                  # append chunk size (quantize workload)
    group_bounds: Sequence[int] = ()
    group_m: Sequence[int] = ()
    n_queries: int = 1

    @property
    def torch_dtype(self) -> torch.dtype:
        return _DTYPES[self.dtype]

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def m_for_layer(self, layer: int) -> int:
        if not self.group_m:
            return self.m
        g = 0
        for bnd in self.group_bounds:
            if layer >= bnd:
                g += 1
        return self.group_m[g]

    def key_sigma(self, layer: int) -> float:
        if not self.var_ramp or self.layers <= 1:
            return 1.0
        return math.sqrt(1.0 + 2.0 * layer / (self.layers - 1))

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=1, d=128, T=512, W=0, b1=2, m=128,
                     vbits=2, group=32, dtype="f32", seed=0,
                     k_outlier_count=4, outlier_scale=10.0, n_queries=4),
    "gqa32k": Workload("gqa32k", B=8, Hq=32, Hkv=8, d=128, T=32768, W=16, b1=2,
                       m=128, vbits=2, group=32, dtype="bf16", seed=0,
                       k_outlier_frac=0.02, v_outlier_frac=0.02, outlier_scale=8.0),
    "quant": Workload("quant", B=1, Hq=8, Hkv=8, d=128, T=131072, W=0, b1=2, m=128,
                      vbits=2, group=32, dtype="bf16", seed=0,
                      lognormal_sigma=0.5, chunk=4096),
    "aqjl": Workload("aqjl", B=16, Hq=32, Hkv=8, d=128, T=65536, W=16, b1=0, m=512,
                     vbits=2, group=32, dtype="f16", seed=0, layers=32, var_ramp=True,
                     group_bounds=(8, 16, 24), group_m=(512, 384, 256, 192)),
    "wide": Workload("wide", B=4, Hq=16, Hkv=4, d=256, T=262144, W=16, b1=3, m=256,
                     vbits=4, group=64, dtype="bf16", seed=0,
                     k_outlier_frac=0.01, v_outlier_frac=0.01, outlier_scale=10.0),
}


def _generator(seed: int, layer: int, tensor_id: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(((seed * 1_000_003 + layer) * 1009 + tensor_id) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def outlier_channels(w: Workload, layer: int, tensor_id: int) -> torch.Tensor:
    """Channel indices scaled by ``w.outlier_scale`` for K (tensor_id 1) or V (2)."""
    if tensor_id == TENSOR_K:
        n = w.k_outlier_count or int(round(w.k_outlier_frac * w.d))
    else:
        n = int(round(w.v_outlier_frac * w.d))
    if n == 0:
        return torch.zeros(0, dtype=torch.long)
    g = _generator(w.seed, layer, TENSOR_OUTLIER * 10 + tensor_id, "cpu")
    return torch.randperm(w.d, generator=g)[:n].sort().values


def _draw(w: Workload, layer: int, tensor_id: int, shape, device) -> torch.Tensor:
    g = _generator(w.seed, layer, tensor_id, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return x


def keys_values(w: Workload, layer: int = 0, device="cpu", T: Optional[int] = None):
    """K, V of shape [B, Hkv, T, d] in the workload's dtype."""
    T = w.T if T is None else T
    shape = (w.B, w.Hkv, T, w.d)
    out = []
    for tid in (TENSOR_K, TENSOR_V):
        x = _draw(w, layer, tid, shape, device)
        ch = outlier_channels(w, layer, tid).to(x.device)
        if ch.numel():
            x[..., ch] *= w.outlier_scale
        if tid == TENSOR_K:
            x *= w.key_sigma(layer)
        if w.lognormal_sigma:
            gn = _generator(w.seed, layer, TENSOR_NORM * 10 + tid, device)
            f = torch.exp(w.lognormal_sigma *
                          torch.randn(w.B, w.Hkv, T, 1, generator=gn, device=device))
            x *= f
        out.append(x.to(w.torch_dtype))
        del x
    return out[0], out[1]


def queries(w: Workload, layer: int = 0, device="cpu"):
    """Decode queries [B, Hq, d] in the workload's dtype."""
    x = _draw(w, layer, TENSOR_Q, (w.B, w.Hq, w.d), device)
    return x.to(w.torch_dtype)


def decode_stream(w: Workload, n_steps: int, layer: int = 0, device="cpu"):
    """Per-step decode inputs: Q [n, B, Hq, d] and one new token per sequence,
    K_new / V_new [n, B, Hkv, 1, d] (contiguous per step), same distributions as
    the workload's cache (drawn under layer id ``1000 + layer``)."""
    ws = w.scaled(T=n_steps)
    K, V = keys_values(ws, layer=1000 + layer, device=device)
    Kn = K.permute(2, 0, 1, 3).unsqueeze(3).contiguous()
    Vn = V.permute(2, 0, 1, 3).unsqueeze(3).contiguous()
    g = _generator(w.seed, 1000 + layer, TENSOR_Q, device)
    Q = torch.randn(n_steps, w.B, w.Hq, w.d, generator=g, device=device).to(w.torch_dtype)
    return Q, Kn, Vn


def prefill_chunk(w: Workload, n: int, layer: int = 0, device="cpu"):
    """Inputs of a chunk of n new tokens scored against the cache: Q [B, n, Hq, d]
    (token-major) and K, V [B, Hkv, n, d], with the workload's distributions (drawn
    under layer id ``2000 + layer``)."""
    K, V = keys_values(w.scaled(T=n), layer=2000 + layer, device=device)
    g = _generator(w.seed, 2000 + layer, TENSOR_Q, device)
    Q = torch.randn(w.B, n, w.Hq, w.d, generator=g, device=device).to(w.torch_dtype)
    return Q, K, V
