"""tq_decode_step (append + decode as one call) against tq_append followed by
tq_decode_attention on a twin cache: the packed cache, the ring, the outputs and
the logits must be identical after every step, whichever path the call takes
(the fused two-launch path, or the two calls).  The fused step's cache and
output are also compared with the oracle's own append and decode of the same
tokens after every step."""
import math

import numpy as np
import pytest
import torch

import synth
from gpu_common import (TORCH_DT, check_logits, check_out, compare_keys, host, oracle_setup,
                        record, to_dev)
from oracle import cache as ocache
from oracle import layout as olayout

pytestmark = pytest.mark.gpu


class _Proj:
    def __init__(self, po):
        self.Pi, self.S, self.T = to_dev(po["Pi"]), to_dev(po["S"]), to_dev(po["T"])


class _Cb:
    def __init__(self, cb):
        self.centroids, self.boundaries = to_dev(cb[0]), to_dev(cb[1])


def _unit_flips(gpu_buf, oc, b, h, label):
    """Tokens of unit (b, h) whose key codes differ from the oracle's (each
    difference inside the boundary band); value fields and ring bit-exact."""
    lay = oc.lay
    ref = oc.to_bytes()
    r = oc.rec[b][h]
    if r is None:
        return 0
    n = r["rho"].shape[0]
    fg = olayout.read_region(gpu_buf, lay, b, h, n)
    fr = olayout.read_region(ref, lay, b, h, n)
    for name in ("vcode", "vscale", "vmin"):
        assert np.array_equal(fg[name], fr[name]), name
    got = {"idx": fg["idx"], "signs": fg["sign"],
           "rho": np.ascontiguousarray(fg["rho"]).view("<f4").ravel(),
           "rnorm": np.ascontiguousarray(fg["rnorm"]).view("<f4").ravel() if oc.b1 else None}
    return compare_keys(got, r, oc.d, oc.b1, oc.m, oc.cb[1] if oc.b1 else None,
                        label=label)["skipped_tokens"]


def _check_against_oracle(cache, oc, out, logits, Q, w, label):
    """The GPU cache after a step vs the oracle's, then the step's output and
    logits vs the oracle's decode for every unit whose codes are identical.
    Returns the number of units checked."""
    buf = cache.buffer.cpu().numpy()
    lay = oc.lay
    ref = oc.to_bytes()
    assert np.array_equal(buf[lay.ring_k_off:], ref[lay.ring_k_off:]), "ring differs"
    ro, rl = oc.decode(host(Q))
    G = w.Hq // w.Hkv
    o = host(out)
    lg = logits.cpu().numpy().astype(np.float64)
    checked = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            if _unit_flips(buf, oc, b, h, f"{label} unit ({b},{h})") == 0:
                hs = slice(h * G, (h + 1) * G)
                check_out(o[b:b + 1, hs], ro[b:b + 1, hs], w.dtype)
                check_logits(lg[b, hs], rl[(b, h)])
                checked += 1
    return checked


def _workload(**kw):
    base = dict(name="t", B=2, Hq=8, Hkv=2, d=128, T=400, W=16, b1=2, m=128, vbits=2, group=32,
                dtype="bf16", seed=5, k_outlier_frac=0.02, v_outlier_frac=0.02, outlier_scale=8.0)
    base.update(kw)
    return synth.Workload(**base)


@pytest.mark.parametrize("n0", [100, 150, 220])
def test_decode_step_single_split_early_stages(n0):
    """One split per unit: the partial kernel requests the packed blocks below the one
    that receives the token leaving the ring before it waits for the fused quantise,
    and the others after.  n0 = 100 / 150 / 220 puts that boundary after the first /
    second / third of its four stages."""
    from compressed_attention_turboquantprod_b200 import CompressedKVCache
    w = _workload()
    steps = [1, 1, 2]
    total = n0 + sum(steps)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    pj, cbd = _Proj(po), _Cb(cb)
    K, V = synth.keys_values(w, device="cuda", T=total)
    caches = [CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, total + 64,
                                dtype=TORCH_DT[w.dtype]) for _ in range(2)]
    oc = ocache.OracleCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, total + 64,
                            w.dtype, po, cb)
    for c in caches:
        c.append(K[:, :, :n0].contiguous(), V[:, :, :n0].contiguous(), pj, cbd)
    oc.append(host(K[:, :, :n0]), host(V[:, :, :n0]))
    t, checked = n0, 0
    for i, n in enumerate(steps):
        k, v = K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous()
        Q = synth.queries(w.scaled(seed=70 + i), device="cuda")
        o1, l1 = caches[0].decode_step(k, v, Q, pj, cbd, want_logits=True, num_splits=1)
        caches[1].append(k, v, pj, cbd)
        o2, l2 = caches[1].decode(Q, pj, cbd, want_logits=True, num_splits=1)
        oc.append(host(k), host(v))
        torch.cuda.synchronize()
        t += n
        assert torch.equal(caches[0].buffer, caches[1].buffer), f"cache bytes differ after step {i}"
        assert torch.equal(o1, o2), f"outputs differ after step {i}"
        assert torch.equal(l1, l2), f"logits differ after step {i}"
        checked += _check_against_oracle(caches[0], oc, o1, l1, Q, w, f"single-split step {i}")
    assert checked >= 1


@pytest.mark.parametrize("kw,n0,steps", [
    (dict(), 300, [1, 1, 1, 1, 1]),                                     # full ring, one token a step
    (dict(), 5, [3, 8, 8, 1]),                                          # ring filling up
    (dict(dtype="f32", W=20, b1=1, m=64), 40, [2, 5, 1]),
    (dict(b1=0, m=256, dtype="f16"), 100, [1, 4]),                      # pure QJL
    (dict(d=256, b1=3, m=256, vbits=4, group=64, Hq=16, Hkv=4), 200, [1, 2, 1]),   # head dim 256
    (dict(Hq=2, Hkv=2), 150, [1, 1]),                                   # G = 1: the two calls
    (dict(W=3), 50, [5, 1]),                                            # n_new > W: the two calls
])
def test_decode_step_matches_append_then_decode(kw, n0, steps):
    from compressed_attention_turboquantprod_b200 import CompressedKVCache
    w = _workload(**kw)
    total = n0 + sum(steps)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    pj, cbd = _Proj(po), (_Cb(cb) if w.b1 else None)
    K, V = synth.keys_values(w, device="cuda", T=total)
    caches = [CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, total + 64,
                                dtype=TORCH_DT[w.dtype]) for _ in range(2)]
    oc = ocache.OracleCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, total + 64,
                            w.dtype, po, cb if w.b1 else None)
    for c in caches:
        c.append(K[:, :, :n0].contiguous(), V[:, :, :n0].contiguous(), pj, cbd)
    oc.append(host(K[:, :, :n0]), host(V[:, :, :n0]))
    t = n0
    checked = 0
    for i, n in enumerate(steps):
        k, v = K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous()
        Q = synth.queries(w.scaled(seed=50 + i), device="cuda")
        o1, l1 = caches[0].decode_step(k, v, Q, pj, cbd, want_logits=True)
        caches[1].append(k, v, pj, cbd)
        o2, l2 = caches[1].decode(Q, pj, cbd, want_logits=True)
        oc.append(host(k), host(v))
        torch.cuda.synchronize()
        t += n
        assert caches[0].n_total == caches[1].n_total == t
        assert torch.equal(caches[0].buffer, caches[1].buffer), f"cache bytes differ after step {i}"
        assert torch.equal(o1, o2), f"outputs differ after step {i}"
        assert torch.equal(l1, l2), f"logits differ after step {i}"
        assert torch.isfinite(o1.float()).all()
        checked += _check_against_oracle(caches[0], oc, o1, l1, Q, w, f"decode step {i}")
    record(f"decode step {kw} vs oracle", unit_steps_checked=checked,
           unit_steps_skipped=len(steps) * w.B * w.Hkv - checked)
    assert checked >= 1


@pytest.mark.parametrize("kw,n0,steps", [
    (dict(), 300, [1, 1, 1]),                                           # fused path
    (dict(W=3), 50, [5]),                                               # the two calls
])
def test_decode_step_on_pinned_host_buffers(kw, n0, steps):
    """The new tokens, the queries and the output of tq_decode_step in pinned host
    memory (mapped into the device address space; the kernels read and write them
    across the host link): identical cache, output and logits to device buffers."""
    from compressed_attention_turboquantprod_b200 import CompressedKVCache, native
    w = _workload(**kw)
    total = n0 + sum(steps)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    pj, cbd = _Proj(po), _Cb(cb)
    K, V = synth.keys_values(w, device="cuda", T=total)
    caches = [CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, total + 64,
                                dtype=TORCH_DT[w.dtype]) for _ in range(2)]
    for c in caches:
        c.append(K[:, :, :n0].contiguous(), V[:, :, :n0].contiguous(), pj, cbd)
    scale = 1.0 / math.sqrt(w.d)
    t = n0
    for i, n in enumerate(steps):
        k, v = K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous()
        Q = synth.queries(w.scaled(seed=70 + i), device="cuda")
        kh, vh, qh = k.cpu().pin_memory(), v.cpu().pin_memory(), Q.cpu().pin_memory()
        outs, logs = [], []
        for c, (kk, vv, qq, host) in zip(caches, ((k, v, Q, False), (kh, vh, qh, True))):
            out = torch.empty(w.B, w.Hq, w.d, dtype=TORCH_DT[w.dtype],
                              device="cpu" if host else "cuda")
            if host:
                out = out.pin_memory()
            lg = torch.empty(w.B, w.Hq, c.n_total + n, dtype=torch.float32, device="cuda")
            ws = c.workspace(w.Hq)
            native.tq_decode_step(c.state, kk, vv, qq, scale, pj.Pi, pj.S, pj.T, cbd.centroids,
                                  cbd.boundaries, out, lg, 0, ws)
            outs.append(out)
            logs.append(lg)
        torch.cuda.synchronize()
        assert torch.equal(outs[0].cpu().view(torch.uint8), outs[1].view(torch.uint8))
        assert torch.equal(logs[0], logs[1])
        assert torch.equal(caches[0].buffer, caches[1].buffer)
        t += n
