"""GPU parity of append (packed bytes) and decode attention against the oracle."""
import math

import numpy as np
import pytest
import torch

import synth
from gpu_common import (TORCH_DT, check_logits, check_out, compare_keys, host, nat, oracle_setup,
                        record, to_dev)
from oracle import cache as ocache
from oracle import layout as olayout

pytestmark = pytest.mark.gpu


def _workload(**kw):
    base = dict(name="t", B=2, Hq=8, Hkv=2, d=128, T=300, W=16, b1=2, m=128, vbits=2, group=32,
                dtype="bf16", seed=11, k_outlier_frac=0.02, v_outlier_frac=0.02, outlier_scale=8.0)
    base.update(kw)
    return synth.Workload(**base)


def _gpu_cache(w, capacity):
    from compressed_attention_turboquantprod_b200 import CompressedKVCache
    return CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, capacity,
                             dtype=TORCH_DT[w.dtype])


class _Proj:
    def __init__(self, po):
        self.Pi, self.S, self.T = to_dev(po["Pi"]), to_dev(po["S"]), to_dev(po["T"])


class _Cb:
    def __init__(self, cb):
        self.centroids, self.boundaries = to_dev(cb[0]), to_dev(cb[1])


def _oracle_cache(w, capacity, po, cb):
    return ocache.OracleCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, capacity,
                              w.dtype, po, cb if w.b1 > 0 else None)


def _compare_cache_bytes(gpu_buf: np.ndarray, oc: ocache.OracleCache, per_unit=False,
                         label=None):
    """Packed cache vs the oracle's: total tokens with a flipped code, or with
    per_unit, {(b, h): tokens with a flipped code}."""
    ref = oc.to_bytes()
    assert gpu_buf.shape == ref.shape
    units = {(b, h): 0 for b in range(oc.B) for h in range(oc.Hkv)}
    if np.array_equal(gpu_buf, ref):
        if label is not None:
            record(label, code_mismatch=0, sign_mismatch=0, skipped_tokens=0)
        return units if per_unit else 0
    lay = oc.lay
    # rings and value fields must match exactly; key fields may differ only on exempt elements
    assert np.array_equal(gpu_buf[lay.ring_k_off:], ref[lay.ring_k_off:])
    skipped = 0
    for b in range(oc.B):
        for h in range(oc.Hkv):
            r = oc.rec[b][h]
            if r is None:
                continue
            n = r["rho"].shape[0]
            fg = olayout.read_region(gpu_buf, lay, b, h, n)
            fr = olayout.read_region(ref, lay, b, h, n)
            for name in ("vcode", "vscale", "vmin"):
                assert np.array_equal(fg[name], fr[name]), name
            got = {"idx": fg["idx"], "signs": fg["sign"],
                   "rho": np.ascontiguousarray(fg["rho"]).view("<f4").ravel(),
                   "rnorm": np.ascontiguousarray(fg["rnorm"]).view("<f4").ravel() if oc.b1 else None}
            st = compare_keys(got, r, oc.d, oc.b1, oc.m, oc.cb[1] if oc.b1 else None,
                              label=None if label is None else f"{label} unit ({b},{h})")
            skipped += st["skipped_tokens"]
            units[(b, h)] = st["skipped_tokens"]
    return units if per_unit else skipped


def test_append_packed_bytes_match_oracle_across_chunks():
    w = _workload(B=2, Hkv=2, d=128, T=540)
    cap = 600
    po, cb = oracle_setup(w.d, w.b1, w.m)
    K, V = synth.keys_values(w, device="cuda")
    gc = _gpu_cache(w, cap)
    oc = _oracle_cache(w, cap, po, cb)
    t = 0
    for n in (5, 11, 1, 100, 64, 300, 1, 58):
        k = K[:, :, t:t + n].contiguous()
        v = V[:, :, t:t + n].contiguous()
        gc.append(k, v, _Proj(po), _Cb(cb))
        oc.append(host(k), host(v))
        t += n
        torch.cuda.synchronize()
        assert gc.n_total == oc.n_total and gc.n_comp == oc.n_comp and gc.n_ring == oc.n_ring
        _compare_cache_bytes(gc.buffer.cpu().numpy(), oc)


def test_append_chunks_that_write_the_ring_in_the_tile_kernel():
    """Chunks of at least W tokens are quantised by a tile kernel that also writes
    the new ring and may start before the previous append's kernel has finished:
    a first chunk into an empty cache, chunks that replace the ring after
    tile-kernel and ring-kernel appends, a chunk of exactly W, and appends that
    take the separate ring kernel in between, issued back to back (no
    synchronisation between appends, so the kernels do overlap); packed bytes
    (ring included) equal the oracle's at the end."""
    w = _workload(B=2, Hkv=3, d=128, T=700, W=16, seed=5)
    cap = 700
    po, cb = oracle_setup(w.d, w.b1, w.m)
    K, V = synth.keys_values(w, device="cuda")
    gc = _gpu_cache(w, cap)
    oc = _oracle_cache(w, cap, po, cb)
    pj, cbd = _Proj(po), _Cb(cb)
    chunks, t = [], 0
    for n in (40, 20, 16, 9, 30, 3, 200, 17, 300, 12):
        chunks.append((K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous()))
        t += n
    torch.cuda.synchronize()
    for k, v in chunks:
        gc.append(k, v, pj, cbd)
    torch.cuda.synchronize()
    for k, v in chunks:
        oc.append(host(k), host(v))
    assert gc.n_total == oc.n_total == t
    skipped = _compare_cache_bytes(gc.buffer.cpu().numpy(), oc)
    nat().tq_quantize_check()
    record("appends writing the ring in the tile kernel", tokens=t, skipped_tokens=skipped)
    assert skipped <= 3


def test_append_degenerate_tokens_every_quantise_path():
    """Zero keys, constant value rows (s = 0), exact half-step value ties and zero
    value rows through the tensor-core tile kernel (a 300-token chunk), the
    single-token kernel (chunks of 1 and 5) and the fused decode step: packed
    bytes equal the oracle's (codes outside the boundary band)."""
    w = _workload(B=1, Hkv=2, Hq=8, T=420)
    cap = 512
    po, cb = oracle_setup(w.d, w.b1, w.m)
    K, V = synth.keys_values(w, device="cuda")
    # A token is quantised when it leaves the 16-token ring: positions < 284 in the
    # 300-token chunk (tile kernel), 284..290 in the appends of 1, 5, 1 (single-token
    # kernel), 291..403 in the decode steps (fused pre-grid), 404.. stay in the ring.
    ties = (torch.arange(32, device="cuda") % 7).to(V.dtype) * 0.5   # range 3 -> s = 1
    for t in (3, 150, 284, 286, 301, 307, 411):
        K[0, 1, t].zero_()                                   # zero-norm keys
        V[0, 0, t] = 0.75                                    # constant rows: s = 0
        V[0, 1, t, :32] = ties                               # exact half-step ties
    for t in (151, 287, 304):
        V[0, 0, t].zero_()
    gc = _gpu_cache(w, cap)
    oc = _oracle_cache(w, cap, po, cb)
    pj, cbd = _Proj(po), _Cb(cb)
    t = 0
    for n in (300, 1, 5, 1):                                 # tile kernel, then single-token
        k, v = K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous()
        gc.append(k, v, pj, cbd)
        oc.append(host(k), host(v))
        t += n
    while t < w.T:                                           # fused decode steps
        n = min(2, w.T - t)
        k, v = K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous()
        Q = synth.queries(w.scaled(seed=t), device="cuda")
        gc.decode_step(k, v, Q, pj, cbd)
        oc.append(host(k), host(v))
        t += n
    torch.cuda.synchronize()
    nat().tq_quantize_check()
    assert gc.n_total == oc.n_total == w.T
    buf = gc.buffer.cpu().numpy()
    _compare_cache_bytes(buf, oc)
    fg = olayout.read_region(buf, oc.lay, 0, 1, oc.rec[0][1]["rho"].shape[0])
    zero = [3, 150, 284, 286, 301, 307]                      # compressed zero keys
    rho = np.ascontiguousarray(fg["rho"]).view("<f4").ravel()
    rn = np.ascontiguousarray(fg["rnorm"]).view("<f4").ravel()
    assert np.all(rho[zero] == 0) and np.all(rn[zero] == 0)
    bits = olayout.unpack_bits(fg["sign"], w.m)
    assert np.array_equal(bits[zero], oc.rec[0][1]["bits"][zero])   # sign(0) convention


@pytest.mark.parametrize("b1,m,vb,g,dt", [(2, 128, 2, 32, "f32"), (0, 256, 2, 32, "f16"),
                                          (3, 256, 4, 64, "bf16"), (1, 64, 4, 16, "bf16")])
def test_append_quantize_variants(b1, m, vb, g, dt):
    w = _workload(B=1, Hkv=3, d=256 if b1 == 3 else 128, b1=b1, m=m, vbits=vb, group=g, dtype=dt,
                  W=5, T=200)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    K, V = synth.keys_values(w, device="cuda")
    gc = _gpu_cache(w, 256)
    oc = _oracle_cache(w, 256, po, cb)
    for a, b in ((0, 3), (3, 130), (130, 200)):
        k, v = K[:, :, a:b].contiguous(), V[:, :, a:b].contiguous()
        gc.append(k, v, _Proj(po), _Cb(cb) if b1 else None)
        oc.append(host(k), host(v))
    torch.cuda.synchronize()
    _compare_cache_bytes(gc.buffer.cpu().numpy(), oc)


@pytest.mark.parametrize("d,b1,m,vb,g,dt,chunks", [
    (256, 3, 256, 4, 64, "bf16", (9, 300)),          # the wide shape: Pi and T streamed
    (256, 0, 128, 2, 128, "f16", (130, 140)),        # pure QJL at d = 256, a group over two parts
    (256, 1, 96, 2, 16, "f32", (128, 129)),          # an N tail of 96 rows, 16-channel groups
    (256, 2, 512, 4, 32, "bf16", (200,)),            # 512 accumulator columns
    (128, 0, 512, 2, 32, "f16", (9, 257, 300)),      # the A-QJL shapes: m = 512 / 384 / 192
    (128, 0, 384, 2, 32, "f16", (129,)),
    (128, 0, 192, 4, 64, "bf16", (64, 300)),
    (128, 3, 64, 4, 128, "bf16", (150,)),            # one N-chunk of 64 rows, a group of 128
    (128, 2, 32, 2, 32, "f32", (12,)),
])
def test_append_tensor_core_general_shapes(d, b1, m, vb, g, dt, chunks):
    """Chunks of more than 8 tokens at shapes outside d = m = 128 run on the tensor
    cores with the operands streamed from a per-call image: packed bytes equal the
    oracle's (codes and signs outside the boundary band), values bit-exact, and the
    kernel's wait flag clear."""
    T = sum(chunks) + 7
    w = _workload(B=1, Hkv=2, d=d, b1=b1, m=m, vbits=vb, group=g, dtype=dt, W=7, T=T,
                  seed=31 + d + m + b1)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    K, V = synth.keys_values(w, device="cuda")
    gc = _gpu_cache(w, T)
    oc = _oracle_cache(w, T, po, cb)
    t = 0
    for n in chunks + (7,):
        k, v = K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous()
        gc.append(k, v, _Proj(po), _Cb(cb) if b1 else None)
        oc.append(host(k), host(v))
        t += n
    torch.cuda.synchronize()
    nat().tq_quantize_check()
    skipped = _compare_cache_bytes(gc.buffer.cpu().numpy(), oc,
                                   label=f"tensor-core append d={d} b1={b1} m={m}")
    assert skipped <= max(2, T // 100)


def test_append_tensor_core_many_tiles_per_cta():
    """More 128-token tiles than SMs, so persistent CTAs stream the operand pieces of
    several tiles in a row (the stages wrap across tiles): d = 256, b1 = 3, m = 256
    and pure QJL m = 512 against the oracle."""
    for (d, b1, m, vb, g, dt) in ((256, 3, 256, 4, 64, "bf16"), (128, 0, 512, 2, 32, "f16")):
        T = 128 * 40 + 19
        w = _workload(B=1, Hkv=4, d=d, b1=b1, m=m, vbits=vb, group=g, dtype=dt, W=16, T=T,
                      seed=77 + b1)
        po, cb = oracle_setup(w.d, w.b1, w.m)
        K, V = synth.keys_values(w, device="cuda")
        gc = _gpu_cache(w, T)
        oc = _oracle_cache(w, T, po, cb)
        gc.append(K, V, _Proj(po), _Cb(cb) if b1 else None)
        oc.append(host(K), host(V))
        torch.cuda.synchronize()
        nat().tq_quantize_check()
        skipped = _compare_cache_bytes(gc.buffer.cpu().numpy(), oc,
                                       label=f"tensor-core append, many tiles, d={d} m={m}")
        assert skipped <= max(2, w.Hkv * T // 200)


def _decode_identical_codes(w, n_tokens, capacity, num_splits=0, Hq=None):
    """Oracle-built cache bytes decoded by the GPU with the oracle's projections."""
    Hq = Hq or w.Hq
    po, cb = oracle_setup(w.d, w.b1, w.m)
    K, V = synth.keys_values(w, device="cuda", T=max(n_tokens, 1))
    oc = _oracle_cache(w, capacity, po, cb)
    if n_tokens:
        oc.append(host(K[:, :, :n_tokens]), host(V[:, :, :n_tokens]))
    gc = _gpu_cache(w, capacity)
    gc.buffer.copy_(torch.from_numpy(oc.to_bytes()))
    gc.state.n_total = oc.n_total
    Q = synth.queries(w.scaled(Hq=Hq), device="cuda")
    out, logits = gc.decode(Q, _Proj(po), _Cb(cb) if w.b1 else None, want_logits=True,
                            num_splits=num_splits)
    torch.cuda.synchronize()
    ro, rl = oc.decode(host(Q))
    G = Hq // w.Hkv
    lg = logits.cpu().numpy().astype(np.float64)
    for (b, h), want in rl.items():
        check_logits(lg[b, h * G:(h + 1) * G], want)
    err = check_out(host(out), ro, w.dtype)
    return err


@pytest.mark.parametrize("n_tokens,splits", [(300, 0), (300, 1), (300, 3), (17, 0), (64 + 16, 2),
                                             (1000, 7), (16, 0), (5, 0), (1, 0), (2000, 0),
                                             (4096 + 16 + 63, 5), (3000, 40)])
def test_decode_identical_codes_lengths_and_splits(n_tokens, splits):
    _decode_identical_codes(_workload(), n_tokens, max(1024, n_tokens + 64), splits)


@pytest.mark.parametrize("kw", [
    dict(d=64, m=64, group=16, Hq=16, Hkv=2),                       # G = 8
    dict(d=256, b1=3, m=256, vbits=4, group=64, Hq=4, Hkv=4),        # G = 1
    dict(b1=0, m=512, dtype="f16", Hq=8, Hkv=2),                    # pure QJL
    dict(b1=0, m=192, dtype="f16", W=0),
    dict(b1=1, m=96, vbits=4, dtype="f32"),
    dict(W=0, dtype="f32", B=1, Hq=4, Hkv=1, k_outlier_count=4, outlier_scale=10.0,
         k_outlier_frac=0.0, v_outlier_frac=0.0),                  # the tiny workload's shape
    # shapes of the tensor-core path (d=128, G=4, 2-bit values g=32)
    dict(m=256), dict(b1=1, m=64), dict(b1=0, m=128, dtype="f16"), dict(b1=0, m=256, W=3),
    dict(B=3, Hkv=5, Hq=20, W=1),
    dict(W=40), dict(dtype="f32", W=20), dict(dtype="f16", W=33, b1=1),   # several ring chunks
    dict(m=384), dict(b1=1, m=512, W=7), dict(b1=0, m=192, dtype="f16"),  # larger sketches
    # shapes of the head-dim-256 tensor-core path (G=4, 4-bit values g=64)
    dict(d=256, b1=3, m=256, vbits=4, group=64, Hq=16, Hkv=4),
    dict(d=256, b1=3, m=128, vbits=4, group=64, dtype="f32", W=5),
    dict(d=256, b1=2, m=256, vbits=4, group=64, W=20),
    dict(d=256, b1=0, m=128, vbits=4, group=64, Hq=4, Hkv=1, dtype="f16", W=0),
    dict(d=256, b1=1, m=256, vbits=4, group=64, dtype="f16", W=9),
])
def test_decode_identical_codes_shapes(kw):
    w = _workload(**kw)
    _decode_identical_codes(w, 333, 512)


@pytest.mark.parametrize("n_tokens,splits", [(3000, 0), (3000, 40), (333, 3)])
def test_staged_decode_fused_and_separate_merge(n_tokens, splits):
    """tq_decode_prep + tq_decode_partial(out) (splits merged by the last split of
    each unit) and tq_decode_prep + tq_decode_partial + tq_decode_combine agree with
    each other and with the oracle over consecutive calls on one workspace (the
    per-unit split counter is reset between calls)."""
    from compressed_attention_turboquantprod_b200 import native
    w = _workload()
    cap = max(1024, n_tokens + 64)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    K, V = synth.keys_values(w, device="cuda", T=n_tokens)
    oc = _oracle_cache(w, cap, po, cb)
    oc.append(host(K), host(V))
    gc = _gpu_cache(w, cap)
    gc.buffer.copy_(torch.from_numpy(oc.to_bytes()))
    gc.state.n_total = oc.n_total
    pj, cbd = _Proj(po), _Cb(cb)
    ws = gc.workspace(w.Hq, splits)
    scale = 1.0 / math.sqrt(w.d)
    for call in range(3):
        Q = synth.queries(w.scaled(seed=100 + call), device="cuda")
        fused = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=TORCH_DT[w.dtype], device="cuda")
        sep = torch.full_like(fused, float("nan"))
        native.tq_decode_prep(gc.state, Q, scale, pj.Pi, pj.S, cbd.centroids, splits, ws)
        native.tq_decode_partial(gc.state, w.Hq, scale, cbd.centroids, None, splits, ws, out=fused)
        native.tq_decode_prep(gc.state, Q, scale, pj.Pi, pj.S, cbd.centroids, splits, ws)
        native.tq_decode_partial(gc.state, w.Hq, scale, cbd.centroids, None, splits, ws)
        native.tq_decode_combine(gc.state, w.Hq, sep, splits, ws)
        torch.cuda.synchronize()
        native.tq_decode_check(gc.state, w.Hq, splits, ws)
        ro, _ = oc.decode(host(Q))
        check_out(host(fused), ro, w.dtype)
        check_out(host(sep), ro, w.dtype)
        diff = (fused.float() - sep.float()).abs().max().item()
        assert diff <= 2 * float(torch.finfo(TORCH_DT[w.dtype]).eps)


@pytest.mark.parametrize("n_tokens,splits", [(1, 0), (80, 2), (333, 3), (2000, 0), (3000, 40)])
def test_decode_identical_codes_wide_lengths_and_splits(n_tokens, splits):
    w = _workload(d=256, b1=3, m=256, vbits=4, group=64, Hq=8, Hkv=2)
    _decode_identical_codes(w, n_tokens, max(1024, n_tokens + 64), splits)


def test_decode_empty_cache_is_zero():
    w = _workload()
    from compressed_attention_turboquantprod_b200 import CompressedKVCache
    gc = _gpu_cache(w, 64)
    po, cb = oracle_setup(w.d, w.b1, w.m)
    Q = synth.queries(w, device="cuda")
    out = gc.decode(Q, _Proj(po), _Cb(cb))
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


def _flips(gc, oc, b, h, W_unit=None, label=None):
    """Number of tokens of GPU unit (b, h) whose key codes differ from the oracle's
    (each difference is asserted to lie in the boundary band)."""
    lay = oc.lay
    st = gc.state
    off = (b * gc.desc.Hkv + h) * st.region_bytes
    buf = np.zeros(lay.total_bytes, np.uint8)
    buf[:lay.region_bytes] = gc.buffer[off:off + st.region_bytes].cpu().numpy()
    r = oc.rec[0][0]
    n = r["rho"].shape[0]
    fg = olayout.read_region(buf, lay, 0, 0, n)
    got = {"idx": fg["idx"], "signs": fg["sign"],
           "rho": np.ascontiguousarray(fg["rho"]).view("<f4").ravel(),
           "rnorm": np.ascontiguousarray(fg["rnorm"]).view("<f4").ravel() if oc.b1 else None}
    return compare_keys(got, r, oc.d, oc.b1, oc.m, oc.cb[1] if oc.b1 else None,
                        label=label)["skipped_tokens"]


# End-to-end output checks (library quantisation + library decode against the
# oracle's quantisation + decode) are made for units whose codes came out
# identical: a single near-boundary code flip, which the bit-exactness rule
# allows, legitimately moves an output of a short, peaked context by more than
# the output tolerance.  The decode itself is checked given identical codes in
# test_decode_identical_codes_*.
def test_tiny_workload_end_to_end_with_library_projections():
    """The tiny workload (d=128, 512 fp32 tokens, 4 outlier channels x10, 4 queries):
    library-made projections + codebook, GPU append + decode, vs the oracle run on
    its own projections from the same seed."""
    from compressed_attention_turboquantprod_b200 import Codebook, Projections
    w = synth.WORKLOADS["tiny"]
    checked = 0
    for W in (0, 16):
        wl = w.scaled(W=W)
        K, V = synth.keys_values(wl, device="cuda")
        Q = synth.queries(wl, device="cuda")
        pg, cbg = Projections(wl.d, wl.m, 0), Codebook(wl.d, wl.b1)
        gc = _gpu_cache(wl, 512)
        gc.append(K, V, pg, cbg)
        out, logits = gc.decode(Q, pg, cbg, want_logits=True)
        torch.cuda.synchronize()
        po, cb = oracle_setup(wl.d, wl.b1, wl.m)
        oc = _oracle_cache(wl, 512, po, cb)
        oc.append(host(K), host(V))
        ro, rl = oc.decode(host(Q))
        if _flips(gc, oc, 0, 0, label=f"tiny W={W}") == 0:
            check_out(host(out), ro, wl.dtype)
            check_logits(logits.cpu().numpy()[0].astype(np.float64), rl[(0, 0)])
            checked += 1
    record("tiny end-to-end output checks", cases_checked=checked, cases_skipped=2 - checked)
    assert checked >= 1


def test_hadamard_rotation_end_to_end():
    """The structured rotation through the whole path: library-made Hadamard
    projections, GPU append (tensor-core quantise) + decode, vs the oracle with
    its own Hadamard projections from the same seed."""
    from compressed_attention_turboquantprod_b200 import Codebook, Projections
    w = _workload(B=2, Hkv=2, Hq=8, T=700, W=16)
    K, V = synth.keys_values(w, device="cuda")
    Q = synth.queries(w, device="cuda")
    pg, cbg = Projections(w.d, w.m, 2, structured=True), Codebook(w.d, w.b1)
    gc = _gpu_cache(w, 768)
    gc.append(K, V, pg, cbg)
    out, logits = gc.decode(Q, pg, cbg, want_logits=True)
    torch.cuda.synchronize()
    po, cb = oracle_setup(w.d, w.b1, w.m, layer=2, structured=True)
    oc = _oracle_cache(w, 768, po, cb)
    oc.append(host(K), host(V))
    ro, rl = oc.decode(host(Q))
    flips = _compare_cache_bytes(gc.buffer.cpu().numpy(), oc, per_unit=True,
                                 label="hadamard rotation")
    assert sum(flips.values()) <= 4
    # outputs and logits of every unit whose codes came out identical
    G = w.Hq // w.Hkv
    lg = logits.cpu().numpy().astype(np.float64)
    o, r = host(out), ro
    checked = 0
    for (b, h), f in flips.items():
        if f == 0:
            hs = slice(h * G, (h + 1) * G)
            check_out(o[b:b + 1, hs], r[b:b + 1, hs], w.dtype)
            check_logits(lg[b, hs], rl[(b, h)])
            checked += 1
    record("hadamard end-to-end output checks", units_checked=checked,
           units_skipped=len(flips) - checked)
    assert checked >= 1


def test_gqa32k_shape_reduced_context_end_to_end():
    from compressed_attention_turboquantprod_b200 import Codebook, Projections
    w = synth.WORKLOADS["gqa32k"].scaled(T=2000)
    K, V = synth.keys_values(w, device="cuda")
    Q = synth.queries(w, device="cuda")
    pg, cbg = Projections(w.d, w.m, 0), Codebook(w.d, w.b1)
    gc = _gpu_cache(w, 2048)
    gc.append(K[:, :, :1500].contiguous(), V[:, :, :1500].contiguous(), pg, cbg)
    for t in range(1500, 2000, 100):
        gc.append(K[:, :, t:t + 100].contiguous(), V[:, :, t:t + 100].contiguous(), pg, cbg)
    out = gc.decode(Q, pg, cbg)
    torch.cuda.synchronize()
    po, cb = oracle_setup(w.d, w.b1, w.m)
    checked = 0
    for b, h in ((0, 0), (7, 5), (3, 1), (5, 6)):
        oc2 = _oracle_cache(w.scaled(B=1, Hkv=1, Hq=4), 2048, po, cb)
        oc2.append(host(K[b:b + 1, h:h + 1]), host(V[b:b + 1, h:h + 1]))
        if _flips(gc, oc2, b, h) == 0:
            ro, _ = oc2.decode(host(Q[b:b + 1, 4 * h:4 * h + 4]))
            check_out(host(out[b:b + 1, 4 * h:4 * h + 4]), ro, w.dtype)
            checked += 1
    assert checked >= 2


@pytest.mark.parametrize("kw", [
    dict(),                                                          # d=128: tensor-core paths
    dict(d=256, b1=3, m=256, vbits=4, group=64, Hq=8, Hkv=2),        # d=256: tile quantiser + wide
    dict(d=64, b1=2, m=64, Hq=4, Hkv=2, dtype="f32"),                # CUDA-core decode (G = 2)
])
def test_hadamard_fast_transform_every_rotation_site(kw):
    """A cache flagged with the structured rotation applies Pi = H diag(s)/sqrt(d)
    as a fast Walsh-Hadamard transform wherever the rotation runs on CUDA cores:
    the append of up to 8 tokens, the tile quantiser of shapes without the
    tensor-core path, the fused decode step and the query preparation.  Given the
    oracle's (dense) Hadamard projections, the packed cache agrees with the
    oracle's outside the boundary band and the outputs with the oracle's decode."""
    from compressed_attention_turboquantprod_b200 import CompressedKVCache
    w = _workload(T=400, **kw)
    po, cb = oracle_setup(w.d, w.b1, w.m, layer=3, structured=True)
    pj, cbd = _Proj(po), _Cb(cb)
    K, V = synth.keys_values(w, device="cuda")
    cap = 448
    gc = CompressedKVCache(w.B, w.Hkv, w.d, w.b1, w.m, w.vbits, w.group, w.W, cap,
                           dtype=TORCH_DT[w.dtype], structured=True)
    oc = _oracle_cache(w, cap, po, cb)
    G = w.Hq // w.Hkv
    t, checked, units = 0, 0, 0
    for i, (n, how) in enumerate(((300, "append"), (5, "append"), (1, "step"), (3, "step"),
                                  (1, "append"), (2, "step"))):
        k, v = K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous()
        Q = synth.queries(w.scaled(seed=200 + i), device="cuda")
        if how == "append":
            gc.append(k, v, pj, cbd)
            oc.append(host(k), host(v))
            out, lg = gc.decode(Q, pj, cbd, want_logits=True)
        else:
            out, lg = gc.decode_step(k, v, Q, pj, cbd, want_logits=True)
            oc.append(host(k), host(v))
        torch.cuda.synchronize()
        t += n
        flips = _compare_cache_bytes(gc.buffer.cpu().numpy(), oc, per_unit=True,
                                     label=f"hadamard transform {w.d} step {i}")
        ro, rl = oc.decode(host(Q))
        o, lgs = host(out), lg.cpu().numpy().astype(np.float64)
        for (b, h), f in flips.items():
            units += 1
            if f == 0:
                hs = slice(h * G, (h + 1) * G)
                check_logits(lgs[b, hs], rl[(b, h)])
                check_out(o[b:b + 1, hs], ro[b:b + 1, hs], w.dtype)
                checked += 1
    record(f"hadamard transform d={w.d} end-to-end checks", unit_steps_checked=checked,
           unit_steps_skipped=units - checked)
    assert checked >= 1
