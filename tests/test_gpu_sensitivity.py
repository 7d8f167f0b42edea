"""GPU parity of the sensitivity profile's key moments against the oracle, and the
profile of synthetic calibration layers (the A-QJL variance ramp)."""
import numpy as np
import pytest
import torch

import synth
from gpu_common import host
from oracle import sensitivity as sens

pytestmark = pytest.mark.gpu

# entries shifted in fp32, sums and squares in fp64: far below fp32 rounding
VAR_REL = 1e-9


@pytest.mark.parametrize("shape,dtype", [
    ((2, 2, 257, 128), torch.bfloat16), ((3, 1, 1001, 64), torch.float16),
    ((1, 4, 333, 128), torch.float32), ((1, 1, 1, 7), torch.bfloat16),
    ((16, 8, 512, 128), torch.float16), ((1, 1, 5, 3), torch.float32),
])
def test_key_moments_match_oracle(shape, dtype):
    from compressed_attention_turboquantprod_b200 import key_variance
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    K = (torch.randn(*shape, generator=g, device="cuda") * 1.7 + 0.3).to(dtype)
    got = key_variance(K)
    want = sens.key_variance(host(K))
    assert abs(got - want) <= VAR_REL * want, (got, want)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_key_variance_large_mean_small_spread(dtype):
    """Mean 1e3 and standard deviation 1: the one-pass sum of squares would lose
    about six digits here; the library's shifted sums match the oracle's
    two-pass variance to 1e-9 relative."""
    from compressed_attention_turboquantprod_b200 import key_variance, native
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    K = (torch.randn(4, 8, 1024, 128, generator=g, device="cuda") + 1000.0).to(dtype)
    got = key_variance(K)
    want = sens.key_variance(host(K))
    assert abs(got - want) <= 1e-9 * want, (got, want)
    out = torch.empty(2, dtype=torch.float64, device="cuda")
    ws = torch.empty(native.tq_key_moments_workspace_bytes(), dtype=torch.uint8, device="cuda")
    native.tq_key_moments(K, out, ws)
    mean = float(out[0].item())
    assert abs(mean - float(host(K).mean())) <= 1e-12 * 1000.0


def test_profile_of_synthetic_calibration_layers():
    """32 layers of synthetic calibration keys with variance 1 + 2 l / 31: the
    device variances give the oracle's profile (boundaries 8, 16, 24), and the
    library's host step equals the oracle's on the same variances."""
    from compressed_attention_turboquantprod_b200 import LayerGroups, key_variance
    w = synth.WORKLOADS["aqjl"].scaled(B=2, T=512)
    gpu_v, ref_v = [], []
    for layer in range(32):
        K, _ = synth.keys_values(w, layer=layer, device="cuda")
        gpu_v.append(key_variance(K))
        ref_v.append(sens.key_variance(host(K)))
    gpu_v, ref_v = np.array(gpu_v), np.array(ref_v)
    assert np.all(np.abs(gpu_v - ref_v) <= VAR_REL * ref_v)
    b_ref, m_ref = sens.profile(ref_v, 4, 336)
    lg = LayerGroups.from_variances(gpu_v, 4, 336)
    assert b_ref == [8, 16, 24]
    assert lg.boundaries == b_ref and lg.sketch_dims == m_ref
    b2, m2 = sens.profile(gpu_v, 4, 336)
    assert lg.boundaries == b2 and lg.sketch_dims == m2
