"""GPU parity of multi-token (chunked prefill) attention against the oracle.

The cache bytes are built by the oracle and copied to the device (the GPU append
is checked byte for byte elsewhere), so both sides score the same stored codes;
the chunk's queries, keys and values are the same seeded tensors on both sides.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_common import TORCH_DT, check_out, host, oracle_setup, to_dev
from oracle import cache as ocache

pytestmark = pytest.mark.gpu


def _workload(**kw):
    base = dict(name="t", B=2, Hq=8, Hkv=2, d=128, T=300, W=16, b1=2, m=128, vbits=2, group=32,
                dtype="bf16", seed=21, k_outlier_frac=0.02, v_outlier_frac=0.02, outlier_scale=8.0)
    base.update(kw)
    return synth.Workload(**base)


class _Proj:
    def __init__(self, po):
        self.Pi, self.S, self.T = to_dev(po["Pi"]), to_dev(po["S"]), to_dev(po["T"])


class _Cb:
    def __init__(self, cb):
        self.centroids, self.boundaries = to_dev(cb[0]), to_dev(cb[1])


def _prefill(w, n_hist, n, num_splits=0, capacity=None):
    from compressed_attention_turboquantprod_b200 import CompressedKVCache
    capacity = capacity or max(256, n_hist + 64)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    oc = ocache.OracleCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, capacity, w.dtype,
                            po, cb if w.b1 > 0 else None)
    if n_hist:
        K, V = synth.keys_values(w, device="cuda", T=n_hist)
        oc.append(host(K), host(V))
    gc = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, capacity,
                           dtype=TORCH_DT[w.dtype])
    gc.buffer.copy_(torch.from_numpy(oc.to_bytes()))
    gc.state.n_total = oc.n_total
    Q, Kn, Vn = synth.prefill_chunk(w, n, device="cuda")
    ws = torch.empty(_ws_bytes(gc, w.Hq, n, num_splits), dtype=torch.uint8, device="cuda")
    out = gc.prefill(Q, Kn, Vn, _Proj(po), _Cb(cb) if w.b1 else None, num_splits=num_splits,
                     workspace=ws)
    torch.cuda.synchronize()
    from compressed_attention_turboquantprod_b200 import native
    native.tq_prefill_check(gc.state, w.Hq, n, num_splits, ws)
    want = oc.prefill(host(Q), host(Kn), host(Vn))
    err = check_out(host(out), want, w.dtype)
    return gc, err


def _ws_bytes(gc, Hq, n, num_splits):
    from compressed_attention_turboquantprod_b200 import native
    return native.tq_prefill_workspace_bytes(gc.state, Hq, n, num_splits)


@pytest.mark.parametrize("n_hist,n,splits", [
    (300, 16, 0), (300, 16, 1), (300, 5, 3), (300, 1, 0), (300, 17, 0), (300, 33, 2),
    (1000, 8, 7), (4096 + 16 + 63, 16, 0), (2000, 40, 0), (17, 4, 0), (16, 3, 0), (5, 6, 0),
    (0, 9, 0), (80, 2, 40),
])
def test_prefill_lengths_chunks_and_splits(n_hist, n, splits):
    _prefill(_workload(), n_hist, n, splits)


@pytest.mark.parametrize("kw", [
    # tensor-core history path (d=128, G=4, 2-bit values g=32)
    dict(b1=1, m=64), dict(b1=0, m=128, dtype="f16"), dict(b1=0, m=512, dtype="f16"),
    dict(m=256), dict(b1=1, m=384, W=7), dict(b1=0, m=192, dtype="f16", W=0),
    dict(dtype="f32", W=20), dict(B=3, Hkv=5, Hq=20, W=1),
    # CUDA-core history path (other shapes)
    dict(d=64, m=64, group=16, Hq=16, Hkv=2),
    dict(d=256, b1=3, m=256, vbits=4, group=64, Hq=16, Hkv=4),
    dict(b1=1, m=96, vbits=4, dtype="f32"),
    dict(W=0, dtype="f32", B=1, Hq=1, Hkv=1),
])
def test_prefill_shapes(kw):
    _prefill(_workload(**kw), 333, 11)


def test_prefill_gqa32k_shape_reduced_context():
    """The 32K GQA workload's shape (B=8, 32 query heads over 8 KV heads, bf16,
    3-bit keys, 2-bit values) on a shorter history, a 16-token chunk."""
    w = _workload(B=8, Hq=32, Hkv=8, seed=0, k_outlier_frac=0.02, v_outlier_frac=0.0)
    _prefill(w, 2000, 16)


def test_prefill_then_append_matches_decode_of_last_token():
    """After prefill the caller appends the chunk; a chunk of one token equals the
    decode step of that token when nothing leaves the ring (history < W)."""
    from compressed_attention_turboquantprod_b200 import CompressedKVCache
    w = _workload(W=16)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    gc = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, 256,
                           dtype=TORCH_DT[w.dtype])
    K, V = synth.keys_values(w, device="cuda", T=10)
    gc.append(K, V, _Proj(po), _Cb(cb))
    Q, Kn, Vn = synth.prefill_chunk(w, 1, device="cuda")
    out_p = gc.prefill(Q, Kn, Vn, _Proj(po), _Cb(cb))
    gc.append(Kn, Vn, _Proj(po), _Cb(cb))
    out_d = gc.decode(Q[:, 0].contiguous(), _Proj(po), _Cb(cb))
    torch.cuda.synchronize()
    assert torch.allclose(out_p[:, 0].float(), out_d.float(), atol=2e-3, rtol=0)
