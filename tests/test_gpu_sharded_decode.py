"""Context-sharded decode on one GPU: the context is split by token range over two
caches (the earlier range with no ring, the later one with the ring), each cache
yields its split partials, and the merge of both equals the oracle's decode of
the whole context.  (On several GPUs the partials travel by an all-gather; here
the two shards share one device, and no kernel waits on another.)"""
import numpy as np
import pytest
import torch

import synth
from gpu_common import TORCH_DT, check_out, host, oracle_setup, to_dev
from oracle import cache as ocache

pytestmark = pytest.mark.gpu


def _workload(**kw):
    base = dict(name="t", B=2, Hq=8, Hkv=2, d=128, T=1500, W=16, b1=2, m=128, vbits=2, group=32,
                dtype="bf16", seed=31, k_outlier_frac=0.02, v_outlier_frac=0.02, outlier_scale=8.0)
    base.update(kw)
    return synth.Workload(**base)


class _Proj:
    def __init__(self, po):
        self.Pi, self.S, self.T = to_dev(po["Pi"]), to_dev(po["S"]), to_dev(po["T"])


class _Cb:
    def __init__(self, cb):
        self.centroids, self.boundaries = to_dev(cb[0]), to_dev(cb[1])


def _shard(w, W, K, V, po, cb):
    from compressed_attention_turboquantprod_b200 import CompressedKVCache
    n = K.shape[2]
    oc = ocache.OracleCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, W, n + 64, w.dtype, po,
                            cb if w.b1 > 0 else None)
    oc.append(host(K), host(V))
    gc = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, W, n + 64,
                           dtype=TORCH_DT[w.dtype])
    gc.buffer.copy_(torch.from_numpy(oc.to_bytes()))
    gc.state.n_total = oc.n_total
    return oc, gc


@pytest.mark.parametrize("kw,cut,splits", [
    (dict(), 700, (0, 0)), (dict(), 1000, (3, 5)), (dict(), 64, (1, 0)),
    (dict(d=64, m=64, group=16, Hq=16, Hkv=2), 777, (0, 2)),                       # CUDA-core path
    (dict(d=256, b1=3, m=256, vbits=4, group=64, Hq=16, Hkv=4, T=900), 450, (0, 0)),  # head dim 256
    (dict(b1=0, m=256, dtype="f16"), 1200, (2, 0)),
])
def test_two_shards_merge_to_the_whole_context(kw, cut, splits):
    from compressed_attention_turboquantprod_b200 import merge_partials, stack_partials
    w = _workload(**kw)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    K, V = synth.keys_values(w, device="cuda")
    whole, _ = _shard(w, w.W, K, V, po, cb)
    _, ga = _shard(w, 0, K[:, :, :cut].contiguous(), V[:, :, :cut].contiguous(), po, cb)
    _, gb = _shard(w, w.W, K[:, :, cut:].contiguous(), V[:, :, cut:].contiguous(), po, cb)
    Q = synth.queries(w, device="cuda")
    pj, cbd = _Proj(po), (_Cb(cb) if w.b1 else None)
    parts = [g.decode_partials(Q, pj, cbd, num_splits=s) for g, s in zip((ga, gb), splits)]
    slots = max(p[0].shape[1] for p in parts)
    ml, o = stack_partials(parts, slots)
    out = torch.empty(w.B * w.Hq, w.d, dtype=TORCH_DT[w.dtype], device="cuda")
    merge_partials(ml, o, out)
    torch.cuda.synchronize()
    want, _ = whole.decode(host(Q))
    check_out(host(out).reshape(w.B, w.Hq, w.d), want, w.dtype)
