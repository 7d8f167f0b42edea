"""The allocation-free decode entry point against the workspace one.

Some callers cannot give the library device memory for scratch (an engine
plugin whose host framework owns all device allocations, or a process whose
memory is reserved up front): tq_decode_attention_noalloc serves them from a
static device array.  This file runs last so that a failure here leaves every
other test already run; it passes alone in a fresh process as well.
"""
import math

import numpy as np
import pytest
import torch

import synth
from gpu_common import TORCH_DT, check_out, host, nat

pytestmark = pytest.mark.gpu


def _setup(w, cap):
    from compressed_attention_turboquantprod_b200 import Codebook, CompressedKVCache, Projections
    pj, cb = Projections(w.d, w.m, 0, rotation=w.b1 > 0), (Codebook(w.d, w.b1) if w.b1 else None)
    cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, cap,
                              dtype=TORCH_DT[w.dtype])
    return pj, cb, cache


@pytest.mark.parametrize("kw,splits", [
    (dict(), 0),                               # tensor-core path, automatic splits
    (dict(b1=0, m=256, dtype="f16"), 0),       # pure QJL, tensor-core path
    (dict(), 7),                               # explicit split count
    (dict(d=64, Hq=6, Hkv=2, dtype="f32"), 0),     # CUDA-core path (d = 64, G = 3)
    (dict(d=64, Hq=6, Hkv=2, dtype="f32"), 5),
])
def test_noalloc_decode_equals_workspace_decode_twice(kw, splits):
    n = nat()
    base = dict(name="t", B=2, Hq=8, Hkv=2, d=128, T=900, W=16, b1=2, m=128, vbits=2, group=32,
                dtype="bf16", seed=21, k_outlier_frac=0.02, v_outlier_frac=0.02, outlier_scale=8.0)
    base.update(kw)
    w = synth.Workload(**base)
    pj, cb, cache = _setup(w, 1024)
    K, V = synth.keys_values(w, device="cuda")
    cache.append(K, V, pj, cb)
    cent = cb.centroids if cb else None
    scale = 1.0 / math.sqrt(w.d)
    for call in range(2):
        Q = synth.queries(w.scaled(seed=100 + call), device="cuda")
        ref = cache.decode(Q, pj, cb, num_splits=splits)
        out = torch.full_like(Q, float("nan"))
        n.tq_decode_attention_noalloc(cache.state, Q, scale, pj.Pi, pj.S, cent, out,
                                      num_splits=splits)
        # the wait-limit flag of the static scratch (NULL workspace): clear
        n.tq_decode_check(cache.state, w.Hq, splits, None)
        torch.cuda.synchronize()
        assert not torch.isnan(out).any()
        check_out(host(out), host(ref), w.dtype)


def test_noalloc_explicit_splits_on_a_short_context_fit():
    """An explicit split count larger than the context's blocks is clamped as the
    decode clamps it, so the scratch check does not reject it."""
    n = nat()
    w = synth.Workload("t", B=2, Hq=8, Hkv=2, d=128, T=100, W=16, b1=2, m=128, vbits=2,
                       group=32, dtype="bf16", seed=3)
    pj, cb, cache = _setup(w, 128)
    K, V = synth.keys_values(w, device="cuda")
    cache.append(K, V, pj, cb)
    Q = synth.queries(w, device="cuda")
    ref = cache.decode(Q, pj, cb, num_splits=60000)
    out = torch.full_like(Q, float("nan"))
    n.tq_decode_attention_noalloc(cache.state, Q, 1.0 / math.sqrt(w.d), pj.Pi, pj.S,
                                  cb.centroids, out, num_splits=60000)
    torch.cuda.synchronize()
    check_out(host(out), host(ref), w.dtype)


def test_noalloc_rejects_scratch_beyond_the_static_maximum():
    n = nat()
    w = synth.Workload("t", B=64, Hq=64, Hkv=8, d=128, T=64, W=16, b1=0, m=1024, vbits=2,
                       group=32, dtype="bf16")
    pj, cb, cache = _setup(w, 64)
    K, V = synth.keys_values(w, device="cuda")
    cache.append(K, V, pj, cb)
    Q = synth.queries(w, device="cuda")
    out = torch.zeros_like(Q)
    with pytest.raises(n.TQError) as ei:
        n.tq_decode_attention_noalloc(cache.state, Q, 0.1, None, pj.S, None, out)
    assert ei.value.status == n.TQ_ERR_UNSUPPORTED and "static maximum" in ei.value.message
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
