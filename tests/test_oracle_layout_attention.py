"""Pins of the packed layout, decode attention and the append/ring oracle (CPU only)."""
import numpy as np
import pytest
from scipy import special

from conftest import page_figures
from oracle import attention, cache, codebook, layout, projections, quantize


def test_token_bytes_and_page_compression_ratio():
    figs = page_figures()
    # head_dim 256, 3-bit keys (2-bit Lloyd-Max + m = 256 signs), 2-bit values g = 32
    lay = layout.Layout(1, 1, 256, 2, 256, 2, 32, 0, 64, "bf16")
    ratio = (2 * 256 * 2) / lay.token_bytes
    assert lay.token_bytes == 232
    assert round(ratio, 2) == float(figs["compression_ratio_d256_3bK_2bV"])
    # three bits per coordinate for the key codes proper (b1 d + m bits, m = d)
    assert (lay.f_idx + lay.f_sign) * 8 == 3 * 256


@pytest.mark.parametrize("d,b1,m,vb,g,want", [
    (128, 2, 128, 2, 32, 120), (256, 3, 256, 4, 64, 296),
    (128, 0, 512, 2, 32, 132), (128, 0, 384, 2, 32, 116),
    (128, 0, 256, 2, 32, 100), (128, 0, 192, 2, 32, 92)])
def test_bytes_per_token_head(d, b1, m, vb, g, want):
    lay = layout.Layout(2, 3, d, b1, m, vb, g, 16, 1000, "bf16")
    assert lay.token_bytes == want
    assert lay.block_bytes == layout.TB * want
    for off in (lay.o_idx, lay.o_sign, lay.o_rho, lay.o_rnorm, lay.o_vcode, lay.o_vscale, lay.o_vmin):
        assert off % 16 == 0
    assert lay.ring_k_off % 256 == 0 and lay.ring_v_off % 256 == 0
    assert lay.nblk == 16 and lay.packed_bytes == 6 * 16 * lay.block_bytes


def test_pack_round_trip():
    rng = np.random.default_rng(0)
    for vb in (2, 4):
        codes = rng.integers(0, 1 << vb, (37, 128)).astype(np.uint8)
        assert np.array_equal(layout.unpack_codes(layout.pack_codes(codes, vb), vb, 128), codes)
    bits = rng.integers(0, 2, (37, 192)).astype(np.uint8)
    packed = layout.pack_bits(bits)
    assert packed.shape == (37, 24)
    assert np.array_equal(layout.unpack_bits(packed, 192), bits)
    # explicit bit order: bit i at byte i >> 3, position i & 7
    for i in (0, 5, 8, 191):
        assert (packed[0, i >> 3] >> (i & 7)) & 1 == bits[0, i]
    c = np.zeros((1, 8), np.uint8)
    c[0, 1] = 3
    assert layout.pack_codes(c, 2)[0, 0] == 0b1100


def test_region_write_read_round_trip():
    d, b1, m = 128, 2, 128
    p = projections.make_projections(d, m, 0)
    cb = codebook.build(d, b1)
    lay = layout.Layout(2, 2, d, b1, m, 2, 32, 0, 150, "f32")
    rng = np.random.default_rng(1)
    X = rng.standard_normal((150, d))
    V = rng.standard_normal((150, d)).astype(np.float32)
    k = quantize.quantize_keys(X, p["Pi"], p["S"], *cb, b1)
    codes, s, mn = quantize.quantize_values(V, 2, 32)
    f = layout.token_fields(k, codes, s, mn, lay)
    buf = np.zeros(lay.total_bytes, np.uint8)
    layout.write_region(buf, lay, 1, 0, 0, f)
    back = layout.decode_fields(layout.read_region(buf, lay, 1, 0, 150), lay)
    assert np.array_equal(back["idx"], k["idx"]) and np.array_equal(back["bits"], k["bits"])
    assert np.array_equal(back["rho"], k["rho"]) and np.array_equal(back["rnorm"], k["rnorm"])
    assert np.array_equal(back["codes"], codes) and np.array_equal(back["scale"], s)
    assert np.array_equal(back["vmin"], mn)
    assert not buf[:lay.region_off(1, 0)].any()            # other regions untouched


@pytest.mark.parametrize("d,vb,g,tok,ch,byte,bit", [
    # d 128, 2-bit, g 32: token 5 = high half of pair 2 (64-byte records); channel
    # 37 = group 1, half s 0 (8 channels a half), 6th code -> word 0*4 + 1, bits 10-11
    (128, 2, 32, 5, 37, 2 * 64 + 4 * 1 + 2 + 1, 2),
    # d 256, 4-bit, g 64: token 10 = low half of pair 5 (256-byte records); channel
    # 200 = group 3, half s 2 (4 channels a half), 1st code -> word 2*4 + 3, bits 0-3
    (256, 4, 64, 10, 200, 5 * 256 + 4 * 11, 0),
    # second block, g 16: token 64 + 3 = high half of pair 1; channel 127 = group 7,
    # half s 1 (2 halves a group), 8th code -> word 1*8 + 7, bits 14-15
    (128, 2, 16, 67, 127, 1 * 64 + 4 * 15 + 2 + 1, 6)])
def test_value_code_pair_records_by_hand(d, vb, g, tok, ch, byte, bit):
    lay = layout.Layout(1, 1, d, 0, 64, vb, g, 0, 128, "f32")
    n = tok + 1
    codes = np.zeros((n, d), np.uint8)
    codes[tok, ch] = (1 << vb) - 1
    f = {"idx": np.zeros((n, 0), np.uint8), "sign": np.zeros((n, 8), np.uint8),
         "rho": np.zeros((n, 4), np.uint8), "rnorm": np.zeros((n, 0), np.uint8),
         "vcode": layout.pack_codes(codes, vb),
         "vscale": np.zeros((n, 4 * d // g), np.uint8), "vmin": np.zeros((n, 4 * d // g), np.uint8)}
    buf = np.zeros(lay.total_bytes, np.uint8)
    layout.write_region(buf, lay, 0, 0, 0, f)
    at = (tok // layout.TB) * lay.block_bytes + lay.o_vcode + byte
    assert buf[at] == ((1 << vb) - 1) << bit
    assert np.count_nonzero(buf) == 1
    back = layout.decode_fields(layout.read_region(buf, lay, 0, 0, n), lay)
    assert np.array_equal(back["codes"], codes)


def test_all_exact_decode_equals_dense_attention():
    rng = np.random.default_rng(2)
    G, d, n = 4, 64, 40
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    out, logits = attention.decode_group(q, None, np.zeros((0, d)), K, V, None, None, None, 2,
                                         1 / np.sqrt(d))
    want = special.softmax(q @ K.T / np.sqrt(d), axis=1) @ V
    assert np.max(np.abs(out - want)) < 1e-12
    assert np.max(np.abs(logits - q @ K.T)) < 1e-12


def test_decode_special_cases():
    d, m, b1 = 128, 128, 2
    p = projections.make_projections(d, m, 0)
    cb = codebook.build(d, b1)
    rng = np.random.default_rng(3)
    X = rng.standard_normal((5, d))
    V = rng.standard_normal((5, d)).astype(np.float32)
    k = quantize.quantize_keys(X, p["Pi"], p["S"], *cb, b1)
    codes, s, mn = quantize.quantize_values(V, 2, 32)
    vh = quantize.dequantize_values(codes, s, mn, 32)
    one = {key: val[:1] for key, val in k.items()}
    o, _ = attention.decode_group(rng.standard_normal((2, d)), one, vh[:1], None, None,
                                  p["Pi"], p["S"], cb[0], b1, 0.1)
    assert np.max(np.abs(o - vh[0][None, :])) < 1e-12      # one token: o = v^
    o, _ = attention.decode_group(np.zeros((1, d)), k, vh, None, None, p["Pi"], p["S"], cb[0],
                                  b1, 0.1)
    assert np.max(np.abs(o[0] - vh.mean(0))) < 1e-12       # equal logits: mean of v^


def test_gqa_head_mapping():
    d, m, b1 = 64, 64, 2
    p = projections.make_projections(d, m, 0)
    cb = codebook.build(d, b1)
    c = cache.OracleCache(1, 2, d, b1, m, 2, 32, 0, 64, "f32", p, cb)
    rng = np.random.default_rng(4)
    K = rng.standard_normal((1, 2, 20, d)).astype(np.float32)
    V = rng.standard_normal((1, 2, 20, d)).astype(np.float32)
    V[0, 1] += 5.0                                          # head 1 values shifted
    c.append(K, V)
    Q = rng.standard_normal((1, 6, d))
    out, _ = c.decode(Q)
    assert np.all(out[0, :3].mean(1) < 2.0) and np.all(out[0, 3:].mean(1) > 3.0)


def _mk_cache(W, cap=400, dtype="bf16"):
    d, m, b1 = 64, 64, 2
    p = projections.make_projections(d, m, 0)
    cb = codebook.build(d, b1)
    return cache.OracleCache(2, 2, d, b1, m, 2, 32, W, cap, dtype, p, cb)


def _bf16(x):
    u = np.asarray(x, np.float32).view(np.uint32)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def test_chunked_append_equals_one_shot_byte_for_byte():
    rng = np.random.default_rng(5)
    K = _bf16(rng.standard_normal((2, 2, 300, 64)))
    V = _bf16(rng.standard_normal((2, 2, 300, 64)))
    one = _mk_cache(16)
    one.append(K, V)
    many = _mk_cache(16)
    for a, b in ((0, 7), (7, 8), (8, 100), (100, 101), (101, 300)):
        many.append(K[:, :, a:b], V[:, :, a:b])
    assert np.array_equal(one.to_bytes(), many.to_bytes())
    # and the compressed part equals quantising tokens 0 .. n-W-1 directly
    assert one.n_comp == 284 and one.n_ring == 16
    r = one.quantize_tokens(K[1, 1, :284], V[1, 1, :284])
    assert np.array_equal(one.rec[1][1]["idx"], r["idx"])
    assert np.array_equal(one.rec[1][1]["codes"], r["codes"])


def test_ring_fifo_semantics():
    rng = np.random.default_rng(6)
    K = _bf16(rng.standard_normal((2, 2, 40, 64)))
    V = _bf16(rng.standard_normal((2, 2, 40, 64)))
    c = _mk_cache(16)
    c.append(K[:, :, :10], V[:, :, :10])
    assert c.n_comp == 0 and c.n_ring == 10 and c.rec[0][0] is None
    for t in range(10, 40):
        c.append(K[:, :, t:t + 1], V[:, :, t:t + 1])
        assert c.n_comp == max(0, t + 1 - 16)
    slots = c.ring_slots()
    assert np.array_equal(c.ring_k[0, 0, slots], K[0, 0, 24:40])
    buf = c.to_bytes()
    ring = buf[c.lay.ring_k_off:c.lay.ring_k_off + c.lay.ring_bytes].view("<u2")
    ring = (ring.astype(np.uint32) << 16).view(np.float32).reshape(2, 2, 16, 64)
    assert np.array_equal(ring[1, 0, 40 % 16 - 1], K[1, 0, 39])


def test_capacity_exceeded_raises():
    c = _mk_cache(0, cap=10)
    with pytest.raises(ValueError):
        c.append(np.zeros((2, 2, 11, 64)), np.zeros((2, 2, 11, 64)))
