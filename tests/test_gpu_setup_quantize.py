"""GPU parity of the setup calls and the quantisers against the oracle."""
import numpy as np
import pytest
import torch

import synth
from gpu_common import (compare_keys, host, nat, oracle_setup, to_dev)
from oracle import codebook as ocb
from oracle import projections as oproj
from oracle import quantize as oq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3])
def test_codebook_matches_oracle(d, bits):
    n = nat()
    L = 1 << bits
    c = torch.empty(L, dtype=torch.float32, device="cuda")
    b = torch.empty(L - 1, dtype=torch.float32, device="cuda")
    n.tq_codebook_build(d, bits, c, b)
    c32, b32 = ocb.build(d, bits)
    cg, bg = c.cpu().numpy(), b.cpu().numpy()
    assert np.all(np.abs(cg - c32) <= np.spacing(np.abs(c32)))     # at most 1 ulp
    assert np.all(np.abs(bg - b32) <= np.spacing(np.abs(b32)) + 0.0)
    assert np.array_equal(cg, -cg[::-1]) and bg[L // 2 - 1] == 0.0


def test_codebook_large_d_and_four_bits():
    n = nat()
    for d, bits in ((16, 2), (1024, 2), (128, 4)):
        L = 1 << bits
        c = torch.empty(L, dtype=torch.float32, device="cuda")
        b = torch.empty(L - 1, dtype=torch.float32, device="cuda")
        n.tq_codebook_build(d, bits, c, b)
        c32, _ = ocb.build(d, bits)
        assert np.all(np.abs(c.cpu().numpy() - c32) <= 2 * np.spacing(np.abs(c32)))


@pytest.mark.parametrize("d,m,layer,rot", [(128, 128, 0, True), (128, 128, 5, True),
                                           (256, 256, 0, True), (64, 96, 1, True),
                                           (128, 512, 3, False), (128, 192, 31, False)])
def test_projections_match_oracle(d, m, layer, rot):
    from compressed_attention_turboquantprod_b200 import Projections
    pg = Projections(d, m, layer, rotation=rot)
    po = oproj.make_projections(d, m, layer, with_rotation=rot)
    S = pg.S.cpu().numpy()
    assert np.mean(S == po["S"]) > 0.999
    assert np.all(np.abs(S - po["S"]) <= np.spacing(np.abs(po["S"])))
    T = pg.T.cpu().numpy()
    assert np.max(np.abs(T - po["T"])) <= 2e-6 * max(1.0, np.max(np.abs(po["T"])))
    if rot:
        Pi = pg.Pi.cpu().numpy()
        assert np.max(np.abs(Pi - po["Pi"])) < 1e-6
        P64 = Pi.astype(np.float64)
        assert np.max(np.abs(P64.T @ P64 - np.eye(d))) < 1e-5


@pytest.mark.parametrize("d,m,layer", [(128, 128, 0), (256, 256, 3), (64, 96, 1)])
def test_hadamard_projections_match_oracle(d, m, layer):
    """The structured rotation: Pi bit-exact (every entry +-fl32(1/sqrt(d)), signs
    from Philox stream 2), S the same as the QR call's, T = S Pi^T as there."""
    from compressed_attention_turboquantprod_b200 import Projections
    pg = Projections(d, m, layer, structured=True)
    po = oproj.make_projections(d, m, layer, structured=True)
    assert np.array_equal(pg.Pi.cpu().numpy(), po["Pi"])
    S = pg.S.cpu().numpy()
    assert np.all(np.abs(S - po["S"]) <= np.spacing(np.abs(po["S"])))
    T = pg.T.cpu().numpy()
    assert np.max(np.abs(T - po["T"])) <= 2e-6 * max(1.0, np.max(np.abs(po["T"])))
    assert np.array_equal(S, Projections(d, m, layer).S.cpu().numpy())


@pytest.mark.parametrize("b1,n", [(2, 1000), (3, 300), (1, 129)])
def test_quantize_keys_with_hadamard_rotation(b1, n):
    """Keys quantised with the structured rotation on the tensor-core path: codes,
    signs and norms against the oracle with the same rotation."""
    d, m = 128, 128
    w = synth.Workload("t", B=1, Hq=1, Hkv=1, d=d, T=n, W=0, b1=b1, m=m, vbits=2, group=32,
                       dtype="bf16", seed=21 + b1, k_outlier_count=3, outlier_scale=8.0)
    K, _ = synth.keys_values(w, device="cuda")
    K = K[0, 0].contiguous()
    po, (c32, b32) = oracle_setup(d, b1, m, structured=True)
    got = _keys_gpu(K, b1, m, to_dev(po["Pi"]), to_dev(po["T"]), to_dev(c32), to_dev(b32))
    ref = oq.quantize_keys(host(K), po["Pi"], po["S"], c32, b32, b1)
    stats = compare_keys(got, ref, d, b1, m, b32)
    assert stats["skipped_tokens"] <= max(2, n // 200)


def _keys_gpu(K, b1, m, Pi, T, c, b):
    n_ = nat()
    n, d = K.shape
    dev = dict(device="cuda")
    idx = torch.empty(n, max(b1, 1) * d // 8, dtype=torch.uint8, **dev)
    signs = torch.empty(n, m // 8, dtype=torch.uint8, **dev)
    rho = torch.empty(n, dtype=torch.float32, **dev)
    rn = torch.empty(n, dtype=torch.float32, **dev)
    n_.tq_quantize_keys(K, b1, m, Pi, T, c, b, idx if b1 else None, signs, rho, rn if b1 else None)
    torch.cuda.synchronize()
    return {"idx": idx.cpu().numpy(), "signs": signs.cpu().numpy(), "rho": rho.cpu().numpy(),
            "rnorm": rn.cpu().numpy()}


@pytest.mark.parametrize("d,b1,m,dt,n", [
    (128, 2, 128, "bf16", 1000), (128, 2, 128, "f32", 512), (128, 1, 128, "f16", 300),
    (256, 3, 256, "bf16", 777), (64, 2, 64, "bf16", 129), (128, 0, 512, "f16", 700),
    (128, 0, 192, "f16", 65), (128, 2, 96, "bf16", 200), (256, 2, 256, "f32", 64)])
def test_quantize_keys_given_oracle_projections(d, b1, m, dt, n):
    """Codes and signs bit-exact (outside the boundary band), with the oracle's own
    Pi, T and codebook handed to the kernel."""
    w = synth.Workload("t", B=1, Hq=1, Hkv=1, d=d, T=n, W=0, b1=b1, m=m, vbits=2, group=32,
                       dtype=dt, seed=3, k_outlier_count=3, outlier_scale=8.0)
    K, _ = synth.keys_values(w, device="cuda")
    K = K[0, 0].contiguous()
    po, (c32, b32) = oracle_setup(d, b1, m)
    got = _keys_gpu(K, b1, m, to_dev(po["Pi"]), to_dev(po["T"]), to_dev(c32), to_dev(b32))
    ref = oq.quantize_keys(host(K), po["Pi"], po["S"], c32, b32, b1)
    stats = compare_keys(got, ref, d, b1, m, b32)
    assert stats["skipped_tokens"] <= max(2, n // 200)


@pytest.mark.parametrize("b1", [1, 2, 3])
@pytest.mark.parametrize("n,dt", [(9, "bf16"), (127, "f32"), (128, "bf16"), (129, "f16"),
                                  (1000, "bf16")])
def test_quantize_keys_tensor_core_tiles(b1, n, dt):
    """The batched tensor-core path (d = m = 128, more than 8 keys) at tile edges:
    one partial 128-row tile, exactly one tile, one row into a second tile, many
    tiles over the persistent grid; codes, signs and norms against the oracle, and
    the kernel's wait flag clear."""
    d, m = 128, 128
    w = synth.Workload("t", B=1, Hq=1, Hkv=1, d=d, T=n, W=0, b1=b1, m=m, vbits=2, group=32,
                       dtype=dt, seed=11 + b1, k_outlier_count=3, outlier_scale=8.0,
                       lognormal_sigma=0.5)
    K, _ = synth.keys_values(w, device="cuda")
    K = K[0, 0].contiguous()
    po, (c32, b32) = oracle_setup(d, b1, m)
    got = _keys_gpu(K, b1, m, to_dev(po["Pi"]), to_dev(po["T"]), to_dev(c32), to_dev(b32))
    nat().tq_quantize_check()
    ref = oq.quantize_keys(host(K), po["Pi"], po["S"], c32, b32, b1)
    stats = compare_keys(got, ref, d, b1, m, b32)
    assert stats["skipped_tokens"] <= max(2, n // 200)


def test_quantize_keys_end_to_end_projections_and_zero_key():
    """Library-made Pi/T/codebook; a zero key and a key equal to its codebook point."""
    from compressed_attention_turboquantprod_b200 import Codebook, Projections
    d, b1, m = 128, 2, 128
    pg, cbg = Projections(d, m, 0), Codebook(d, b1)
    w = synth.Workload("t", B=1, Hq=1, Hkv=1, d=d, T=500, W=0, b1=b1, m=m, vbits=2, group=32,
                       dtype="bf16", seed=4)
    K, _ = synth.keys_values(w, device="cuda")
    K = K[0, 0].contiguous()
    K[7].zero_()
    got = _keys_gpu(K, b1, m, pg.Pi, pg.T, cbg.centroids, cbg.boundaries)
    po, (c32, b32) = oracle_setup(d, b1, m)
    ref = oq.quantize_keys(host(K), po["Pi"], po["S"], c32, b32, b1)
    compare_keys(got, ref, d, b1, m, b32)
    assert got["rho"][7] == 0 and got["rnorm"][7] == 0 and np.all(got["signs"][7] == 255)


@pytest.mark.parametrize("d,vb,g,dt,n", [(128, 2, 32, "bf16", 1000), (128, 4, 32, "f32", 333),
                                         (256, 4, 64, "bf16", 200), (64, 2, 16, "f16", 77),
                                         (256, 2, 128, "f32", 65)])
def test_quantize_values_bit_exact(d, vb, g, dt, n):
    n_ = nat()
    w = synth.Workload("t", B=1, Hq=1, Hkv=1, d=d, T=n, W=0, b1=2, m=128, vbits=vb, group=g,
                       dtype=dt, seed=5, lognormal_sigma=0.5)
    _, V = synth.keys_values(w, device="cuda")
    V = V[0, 0].contiguous()
    V[3] = 1.25                                     # constant token: s = 0
    V[4, :g] = torch.arange(g, device="cuda", dtype=V.dtype) * 0.5   # exact half steps
    codes = torch.empty(n, d * vb // 8, dtype=torch.uint8, device="cuda")
    sc = torch.empty(n, d // g, dtype=torch.float32, device="cuda")
    mn = torch.empty(n, d // g, dtype=torch.float32, device="cuda")
    n_.tq_quantize_values(V, vb, g, codes, sc, mn)
    from oracle import layout as olayout
    rc, rs, rm = oq.quantize_values(V.float().cpu().numpy(), vb, g)
    assert np.array_equal(codes.cpu().numpy(), olayout.pack_codes(rc, vb))
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(mn.cpu().numpy().view(np.uint32), rm.view(np.uint32))
