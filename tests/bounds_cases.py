"""Small ragged cases of every kernel path, run in a child process by
test_gpu_bounds_build.py with either library (TQ_LIBRARY unset: libtq.so;
TQ_LIBRARY=bounds: the bounds-checked libtq_bounds.so).  Writes the caches,
outputs and logits to an .npz file and, for the bounds-checked build, asserts
that no device check fired.

usage: python tests/bounds_cases.py OUT.npz
"""
import math
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from compressed_attention_turboquantprod_b200 import (Codebook, CompressedKVCache,  # noqa: E402
                                                       Projections, native)

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _w(**kw):
    base = dict(name="t", B=2, Hq=8, Hkv=2, d=128, T=333, W=16, b1=2, m=128, vbits=2, group=32,
                dtype="bf16", seed=9, k_outlier_frac=0.02, v_outlier_frac=0.02, outlier_scale=8.0)
    base.update(kw)
    return synth.Workload(**base)


CASES = [
    # name, workload, appends (chunk sizes), decode steps, prefill chunk, structured rotation
    ("tensor_core", _w(), (300, 5), (1, 2), 12, False),
    ("tensor_core_hadamard", _w(T=140), (120, 3), (1,), 7, True),
    ("wide", _w(d=256, b1=3, m=256, vbits=4, group=64, T=150), (130, 1), (1,), 3, False),
    ("cuda_core", _w(d=64, Hq=6, Hkv=2, dtype="f32", W=5, T=77, m=64), (70, 2), (1,), 3, False),
    ("pure_qjl", _w(b1=0, m=192, dtype="f16", T=100), (90,), (2,), 0, False),
]


def run(out_path):
    dev = torch.device("cuda", 0)
    res = {}
    for name, w, appends, steps, npre, structured in CASES:
        pj = Projections(w.d, w.m, 0, rotation=w.b1 > 0, device=dev, structured=structured)
        cb = Codebook(w.d, w.b1, device=dev) if w.b1 else None
        total = sum(appends) + sum(steps)
        K, V = synth.keys_values(w, device=dev, T=total)
        cache = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, total + 3,
                                  dtype=TORCH_DT[w.dtype], device=dev, structured=structured)
        t = 0
        for n in appends:
            cache.append(K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous(), pj, cb)
            t += n
        Q = synth.queries(w, device=dev)
        o, lg = cache.decode(Q, pj, cb, want_logits=True)
        res[f"{name}_decode"] = o.float().cpu().numpy()
        res[f"{name}_logits"] = lg.cpu().numpy()
        if npre:
            Qp, Kp, Vp = synth.prefill_chunk(w, npre, device=dev)
            res[f"{name}_prefill"] = cache.prefill(Qp, Kp, Vp, pj, cb).float().cpu().numpy()
        for i, n in enumerate(steps):
            Qs = synth.queries(w.scaled(seed=40 + i), device=dev)
            o = cache.decode_step(K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous(),
                                  Qs, pj, cb)
            res[f"{name}_step{i}"] = o.float().cpu().numpy()
            t += n
        torch.cuda.synchronize()
        res[f"{name}_cache"] = cache.buffer.cpu().numpy()
    # the standalone quantise calls (token-major arrays), a ragged count
    w = _w()
    pj, cb = Projections(w.d, w.m, 0, device=dev), Codebook(w.d, w.b1, device=dev)
    K, V = synth.keys_values(w.scaled(B=1, Hkv=1), device=dev, T=37)
    n = 37
    idx = torch.zeros(n, w.b1 * w.d // 8, dtype=torch.uint8, device=dev)
    sg = torch.zeros(n, w.m // 8, dtype=torch.uint8, device=dev)
    rho = torch.zeros(n, dtype=torch.float32, device=dev)
    rn = torch.zeros(n, dtype=torch.float32, device=dev)
    native.tq_quantize_keys(K[0, 0], w.b1, w.m, pj.Pi, pj.T, cb.centroids, cb.boundaries, idx, sg,
                            rho, rn)
    torch.cuda.synchronize()
    res["arrays_keys"] = np.concatenate([idx.cpu().numpy().ravel(), sg.cpu().numpy().ravel(),
                                         rho.cpu().numpy().view(np.uint8).ravel(),
                                         rn.cpu().numpy().view(np.uint8).ravel()])
    enabled = native.lib.tq_debug_bounds_enabled()
    native.tq_debug_bounds_check()          # raises TQError if any device check fired
    res["bounds_enabled"] = np.array([enabled])
    np.savez(out_path, **res)


if __name__ == "__main__":
    run(sys.argv[1])
