"""The C-ABI library loads, exports every call of include/tq.h, and its host-side
logic (layout, argument checks, capacity, fault injection, layer groups) works
without a GPU.  No call here reaches a CUDA API."""
import ctypes
import os
import re

import pytest
import torch

from conftest import ROOT, page_figures
from oracle import layout as olayout

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="host-only checks use fake device pointers")


@pytest.fixture(scope="module")
def nat():
    from compressed_attention_turboquantprod_b200 import build
    build.build()
    from compressed_attention_turboquantprod_b200 import native
    return native


def _declared():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(nat):
    names = _declared()
    assert len(names) >= 20
    lib = ctypes.CDLL(nat.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert nat.lib.tq_version() == 1


def test_every_declared_call_has_a_binding(nat):
    """The Python binding marshals every call the header declares (same names)."""
    src = open(os.path.join(ROOT, "compressed_attention_turboquantprod_b200", "native.py")).read()
    bound = set(re.findall(r'"(tq_[a-z0-9_]+)": \(', src))
    assert [n for n in _declared() if n not in bound] == []


@pytest.mark.parametrize("cfg", [
    (8, 8, 128, 2, 128, 2, 32, 16, 32768, "bf16"),
    (4, 4, 256, 3, 256, 4, 64, 16, 262144, "bf16"),
    (16, 8, 128, 0, 512, 2, 32, 16, 65536, "f16"),
    (1, 1, 128, 2, 128, 2, 32, 0, 512, "f32"),
    (2, 3, 64, 1, 96, 4, 16, 5, 100, "f32"),
])
def test_layout_matches_oracle_format(nat, cfg):
    B, Hkv, d, b1, m, vb, g, W, cap, dt = cfg
    code = {"f32": 0, "f16": 1, "bf16": 2}[dt]
    c = nat.tq_cache_layout(nat.make_desc(B, Hkv, d, b1, m, vb, g, W, cap, code))
    o = olayout.Layout(B, Hkv, d, b1, m, vb, g, W, cap, dt)
    assert c.block_bytes == o.block_bytes and c.token_bytes == o.token_bytes
    assert c.region_bytes == o.region_bytes
    assert (c.o_idx, c.o_sign, c.o_rho, c.o_rnorm, c.o_vcode, c.o_vscale, c.o_vmin) == \
        (o.o_idx, o.o_sign, o.o_rho, o.o_rnorm, o.o_vcode, o.o_vscale, o.o_vmin)
    assert (c.ring_k_off, c.ring_v_off, c.bytes) == (o.ring_k_off, o.ring_v_off, o.total_bytes)
    assert nat.tq_cache_bytes(nat.make_desc(B, Hkv, d, b1, m, vb, g, W, cap, code)) == o.total_bytes


def _status(nat, fn, *args):
    return fn(*args)


FAKE = ctypes.c_void_p(1 << 20)    # 16/256-byte aligned, never dereferenced


def test_argument_checks_return_before_any_launch(nat):
    L = nat.lib
    S = None
    # unsupported head dim / bit widths / sketch dims
    assert L.tq_quantize_keys(FAKE, 2, 10, 100, 2, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_UNSUPPORTED
    assert "head dim" in L.tq_last_error().decode()
    assert L.tq_quantize_keys(FAKE, 2, 10, 128, 4, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_quantize_keys(FAKE, 2, 10, 128, 2, 48, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_quantize_keys(FAKE, 7, 10, 128, 2, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_quantize_keys(None, 2, 10, 128, 2, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_quantize_keys(FAKE, 2, 10, 128, 2, 128, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_quantize_keys(ctypes.c_void_p((1 << 20) + 4), 2, 10, 128, 2, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_quantize_keys(FAKE, 2, -1, 128, 2, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_INVALID_ARG
    # n == 0 is a no-op success without touching CUDA
    assert L.tq_quantize_keys(FAKE, 2, 0, 128, 2, 128, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S) == nat.TQ_OK
    assert L.tq_quantize_values(FAKE, 2, 10, 128, 3, 32, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_quantize_values(FAKE, 2, 10, 128, 2, 24, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_quantize_values(FAKE, 2, 10, 64, 2, 128, FAKE, FAKE, FAKE, S) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_codebook_build(128, 5, FAKE, FAKE, S) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_codebook_build(8, 2, FAKE, FAKE, S) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_codebook_build(128, 2, None, FAKE, S) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_make_projections(96, 128, 0, 42, 7, FAKE, FAKE, FAKE, FAKE, 1 << 30, S) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_make_projections(128, 100, 0, 42, 7, FAKE, FAKE, FAKE, FAKE, 1 << 30, S) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_make_projections(128, 128, 0, 42, 7, FAKE, FAKE, FAKE, FAKE, 16, S) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_make_projections(128, 128, -1, 42, 7, FAKE, FAKE, FAKE, FAKE, 1 << 30, S) == nat.TQ_ERR_INVALID_ARG


def _fake_cache(nat, **kw):
    p = dict(B=2, Hkv=2, d=128, b1=2, m=128, vbits=2, group=32, W=16, capacity=100, dtype=2)
    p.update(kw)
    desc = nat.make_desc(p["B"], p["Hkv"], p["d"], p["b1"], p["m"], p["vbits"], p["group"],
                         p["W"], p["capacity"], p["dtype"])
    c = nat.tq_cache_layout(desc)
    c.base = 1 << 20
    return c


def test_append_capacity_checked_before_launch(nat):
    c = _fake_cache(nat)
    st = nat.lib.tq_append(ctypes.byref(c), FAKE, FAKE, 117, FAKE, FAKE, FAKE, FAKE, None)
    assert st == nat.TQ_ERR_CAPACITY and c.n_total == 0
    assert "capacity" in nat.lib.tq_last_error().decode()
    c.n_total = 100      # 84 compressed + 16 ring; 17 more would need 101 slots
    st = nat.lib.tq_append(ctypes.byref(c), FAKE, FAKE, 17, FAKE, FAKE, FAKE, FAKE, None)
    assert st == nat.TQ_ERR_CAPACITY and c.n_total == 100
    assert nat.lib.tq_append(ctypes.byref(c), FAKE, FAKE, 0, None, None, None, None, None) == nat.TQ_OK
    assert nat.lib.tq_append(ctypes.byref(c), None, FAKE, 3, FAKE, FAKE, FAKE, FAKE, None) == nat.TQ_ERR_INVALID_ARG
    assert nat.lib.tq_append(None, FAKE, FAKE, 3, FAKE, FAKE, FAKE, FAKE, None) == nat.TQ_ERR_INVALID_ARG
    bad = _fake_cache(nat)
    bad.block_bytes += 16        # struct not produced by init/layout
    assert nat.lib.tq_append(ctypes.byref(bad), FAKE, FAKE, 3, FAKE, FAKE, FAKE, FAKE, None) == nat.TQ_ERR_INVALID_ARG


def test_decode_checks(nat):
    c = _fake_cache(nat)
    c.n_total = 90
    L = nat.lib
    need = L.tq_decode_workspace_bytes(ctypes.byref(c), 8, 0)
    assert need > 0
    assert L.tq_decode_workspace_bytes(ctypes.byref(c), 7, 0) == 0
    assert L.tq_decode_attention(ctypes.byref(c), FAKE, 7, 0.1, FAKE, FAKE, FAKE, FAKE, None, 0, FAKE, need, None) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_decode_attention(ctypes.byref(c), FAKE, 18, 0.1, FAKE, FAKE, FAKE, FAKE, None, 0, FAKE, need, None) == nat.TQ_ERR_UNSUPPORTED
    assert L.tq_decode_attention(ctypes.byref(c), FAKE, 8, 0.1, FAKE, FAKE, FAKE, FAKE, None, 0, FAKE, 64, None) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_decode_attention(ctypes.byref(c), None, 8, 0.1, FAKE, FAKE, FAKE, FAKE, None, 0, FAKE, need, None) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_decode_attention(ctypes.byref(c), FAKE, 8, float("nan"), FAKE, FAKE, FAKE, FAKE, None, 0, FAKE, need, None) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_decode_attention(ctypes.byref(c), FAKE, 8, 0.1, FAKE, FAKE, FAKE, FAKE, None, -2, FAKE, need, None) == nat.TQ_ERR_INVALID_ARG
    # the automatic split count stays within the workspace sized for the capacity
    for n in (0, 1, 16, 17, 80, 116):
        c.n_total = n
        s = L.tq_decode_auto_splits(ctypes.byref(c), 8)
        assert 1 <= s
        assert L.tq_decode_workspace_bytes(ctypes.byref(c), 8, 0) == need


def test_auto_splits_balance_the_sms(nat):
    """The tensor-core decode takes one wave of CTAs (148 SMs x 4 at head dim 128,
    x 2 at 256) when that loads the SMs evenly, and twice the splits when the wave
    leaves some SMs a whole CTA ahead: the most loaded SM carries about
    ceil(units s / 148) CTAs of ceil(blocks / s) blocks."""
    L = nat.lib
    cases = [
        # 64 units x 9 = 576 CTAs: 4 x 57 blocks; 18 splits give 8 x 29, no better
        (dict(B=8, Hkv=8, capacity=32768), 32, 9),
        # 128 units x 4 = 512 CTAs in 592 slots: 4 x 256 blocks; 8 splits: 7 x 128
        (dict(B=16, Hkv=8, b1=0, m=512, dtype=1, capacity=65536), 32, 8),
        # 16 units x 18 = 288 CTAs: 2 x 228 blocks; 36 splits give 4 x 114, no better
        (dict(B=4, Hkv=4, d=256, b1=3, m=256, vbits=4, group=64, capacity=262144), 16, 18),
    ]
    for geo, Hq, want in cases:
        c = _fake_cache(nat, **geo)
        need = L.tq_decode_workspace_bytes(ctypes.byref(c), Hq, 0)
        c.n_total = geo["capacity"]
        assert L.tq_decode_auto_splits(ctypes.byref(c), Hq) == want
        # the workspace sized for the capacity covers every length's automatic count
        for n in (0, 17, 4096, geo["capacity"] // 2, geo["capacity"]):
            c.n_total = n
            s = L.tq_decode_auto_splits(ctypes.byref(c), Hq)
            assert 1 <= s <= 2 * want
            assert L.tq_decode_workspace_bytes(ctypes.byref(c), Hq, s) <= need


def test_fault_injection_is_host_side_and_one_shot(nat):
    c = _fake_cache(nat)
    nat.tq_debug_fail_next("tq_append")
    st = nat.lib.tq_append(ctypes.byref(c), FAKE, FAKE, 1000, FAKE, FAKE, FAKE, FAKE, None)
    assert st == nat.TQ_ERR_CUDA and nat.lib.tq_last_error().decode() == "injected fault"
    st = nat.lib.tq_append(ctypes.byref(c), FAKE, FAKE, 1000, FAKE, FAKE, FAKE, FAKE, None)
    assert st == nat.TQ_ERR_CAPACITY          # armed once only
    nat.tq_debug_fail_next("tq_decode_attention")
    nat.tq_debug_fail_next(None)              # cleared
    assert nat.lib.tq_decode_attention(ctypes.byref(c), FAKE, 7, 0.1, FAKE, FAKE, FAKE, FAKE, None, 0, FAKE, 1, None) == nat.TQ_ERR_UNSUPPORTED


def test_layer_groups_from_page_config(nat):
    figs = page_figures()
    g = nat.tq_layer_groups_parse(figs["aqjl_layer_group_boundaries"], figs["aqjl_key_bits_per_group"])
    want = [512] * 8 + [384] * 8 + [256] * 8 + [192] * 8
    assert [nat.tq_m_for_layer(g, l) for l in range(32)] == want
    assert nat.tq_m_for_layer(g, 1000) == 192
    for bad in (("8,16", "512,384,256,192"), ("16,8,24", "512,384,256,192"),
                ("8,16,24", "512,384,256,100"), ("8,x,24", "512,384,256,192"), ("", "")):
        with pytest.raises(nat.TQError):
            nat.tq_layer_groups_parse(*bad)
    one = nat.tq_layer_groups_parse("", "256")
    assert nat.tq_m_for_layer(one, 7) == 256


def test_prefill_checks(nat):
    c = _fake_cache(nat)
    c.n_total = 90
    L = nat.lib
    n = 5
    need = L.tq_prefill_workspace_bytes(ctypes.byref(c), 8, n, 0)
    assert need > 0
    assert L.tq_prefill_workspace_bytes(ctypes.byref(c), 7, n, 0) == 0      # Hq % Hkv
    assert L.tq_prefill_workspace_bytes(ctypes.byref(c), 8, 0, 0) == 0      # empty chunk
    # more query tokens need more workspace (a virtual batch of B * n queries)
    assert L.tq_prefill_workspace_bytes(ctypes.byref(c), 8, 2 * n, 0) > need

    def call(Q=FAKE, Hq=8, nn=n, K=FAKE, V=FAKE, scale=0.1, Pi=FAKE, S=FAKE, cent=FAKE, out=FAKE,
             splits=0, ws=FAKE, wsb=need):
        return L.tq_prefill_attention(ctypes.byref(c), Q, Hq, nn, K, V, scale, Pi, S, cent, out,
                                      splits, ws, wsb, None)

    assert call(Hq=7) == nat.TQ_ERR_UNSUPPORTED
    assert call(nn=0) == nat.TQ_ERR_INVALID_ARG
    assert call(nn=70000) == nat.TQ_ERR_INVALID_ARG
    assert call(wsb=64) == nat.TQ_ERR_INVALID_ARG
    assert call(Q=None) == nat.TQ_ERR_INVALID_ARG
    assert call(K=None) == nat.TQ_ERR_INVALID_ARG
    assert call(V=None) == nat.TQ_ERR_INVALID_ARG
    assert call(out=None) == nat.TQ_ERR_INVALID_ARG
    assert call(scale=float("nan")) == nat.TQ_ERR_INVALID_ARG
    assert call(splits=-1) == nat.TQ_ERR_INVALID_ARG
    # the workspace sized at the current length covers every later length
    for t in (0, 1, 16, 17, 80, 116):
        c.n_total = t
        assert L.tq_prefill_workspace_bytes(ctypes.byref(c), 8, n, 0) == need


def test_sensitivity_profile_equals_oracle(nat):
    """Host-only call: the groups and sketch dims equal the oracle's exactly (both
    take the integer decisions in sequential IEEE double sums)."""
    import numpy as np
    from oracle import sensitivity as sens
    rng = np.random.default_rng(7)
    for trial in range(120):
        L = int(rng.integers(1, 33))
        k = int(rng.integers(1, min(8, L) + 1))
        kind = trial % 3
        v = (rng.gamma(2.0, 1.0, size=L) if kind == 0 else
             np.full(L, 1.5) if kind == 1 else 1 + 2 * np.arange(L) / max(L - 1, 1))
        m_min = int(rng.choice([32, 64]))
        m_max = int(rng.choice([256, 512, 1024]))
        m_avg = int(rng.integers(m_min, m_max + 1))
        b, m = sens.profile(v, k, m_avg, m_min, m_max)
        g = nat.tq_sensitivity_profile(v, k, m_avg, m_min, m_max)
        assert g.n == k
        assert [g.bound[i] for i in range(k - 1)] == list(b)
        assert [g.m[i] for i in range(k)] == list(m)
        for layer in range(L):
            gi = sum(1 for x in b if layer >= x)
            assert nat.tq_m_for_layer(g, layer) == m[gi]


def test_sensitivity_profile_checks(nat):
    import numpy as np
    v = np.linspace(1.0, 3.0, 32)
    for args in ((v, 0, 256), (v, 9, 256), (v[:3], 4, 256), (v, 4, 16)):
        with pytest.raises(nat.TQError):
            nat.tq_sensitivity_profile(*args)
    with pytest.raises(nat.TQError):
        nat.tq_sensitivity_profile(v, 4, 256, 48, 512)           # m_min not a multiple of 32
    with pytest.raises(nat.TQError):
        nat.tq_sensitivity_profile(np.r_[v[:-1], -1.0], 4, 256)  # negative variance
    L = nat.lib
    assert L.tq_key_moments(None, 2, 10, FAKE, FAKE, 1 << 20, None) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_key_moments(FAKE, 2, 0, FAKE, FAKE, 1 << 20, None) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_key_moments(FAKE, 7, 10, FAKE, FAKE, 1 << 20, None) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_key_moments(FAKE, 2, 10, FAKE, FAKE, 8, None) == nat.TQ_ERR_INVALID_ARG


def test_sharded_decode_calls_checked_on_the_host(nat):
    c = _fake_cache(nat)
    c.n_total = 90
    L = nat.lib
    need = L.tq_decode_workspace_bytes(ctypes.byref(c), 8, 0)
    ml, o, s = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_int()
    ws = ctypes.c_void_p(1 << 24)
    assert L.tq_decode_partials_view(ctypes.byref(c), 8, 0, ws, need, ctypes.byref(ml),
                                     ctypes.byref(o), ctypes.byref(s)) == nat.TQ_OK
    assert s.value == L.tq_decode_auto_splits(ctypes.byref(c), 8)
    assert (1 << 24) < ml.value < o.value < (1 << 24) + need
    assert L.tq_decode_partials_view(ctypes.byref(c), 8, 0, ws, 64, ctypes.byref(ml),
                                     ctypes.byref(o), ctypes.byref(s)) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_decode_partials_view(ctypes.byref(c), 7, 0, ws, need, ctypes.byref(ml),
                                     ctypes.byref(o), ctypes.byref(s)) == nat.TQ_ERR_UNSUPPORTED
    for args in ((None, FAKE, 4, 3, 128, 2), (FAKE, FAKE, 0, 3, 128, 2), (FAKE, FAKE, 4, 0, 128, 2),
                 (FAKE, FAKE, 4, 3, 2048, 2), (FAKE, FAKE, 4, 3, 128, 9)):
        assert L.tq_merge_partials(*args, FAKE, None) == nat.TQ_ERR_INVALID_ARG
    assert L.tq_merge_partials(FAKE, FAKE, 4, 3, 128, 2, None, None) == nat.TQ_ERR_INVALID_ARG


def test_rotation_field_of_the_descriptor(nat):
    """rotation 0 (dense) and 1 (Hadamard) give the same layout; anything else is
    rejected before any device work."""
    base = (2, 2, 128, 2, 128, 2, 32, 16, 1000, 2)
    dense = nat.tq_cache_bytes(nat.make_desc(*base, rotation=nat.TQ_ROTATION_DENSE))
    had = nat.tq_cache_bytes(nat.make_desc(*base, rotation=nat.TQ_ROTATION_HADAMARD))
    assert dense == had > 0
    assert nat.tq_cache_bytes(nat.make_desc(*base, rotation=2)) == 0
    with pytest.raises(nat.TQError) as ei:
        nat.tq_cache_layout(nat.make_desc(*base, rotation=-1))
    assert ei.value.status == nat.TQ_ERR_INVALID_ARG and "rotation" in ei.value.message
