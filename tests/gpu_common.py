"""Shared pieces of the GPU parity tests: the library under test, and helpers
that run the oracle on the very tensors given to the library and compare."""
import math

import numpy as np
import torch

from oracle import codebook as ocb
from oracle import layout as olayout
from oracle import projections as oproj
from oracle import quantize as oq

# Tolerances (stated once, used by every parity test):
#  - codes, sign bits, value codes/scales/minima: bit-exact (key codes and signs
#    except elements within 1e-5 relative of a decision boundary or zero);
#  - rho: 4 ulp; ||r||: 2e-6 relative (fp32 rounding of y = Pi x / rho feeds
#    e = y - c[idx]; ~1e-8 absolute on entries of size ~3e-2 over d terms);
#  - logits given identical codes: 1e-3 relative or 1e-4 absolute;
#  - attention outputs: max(2e-3, half an ulp of the output dtype at |o| + 1e-3).
#    2e-3 is the budget, half of it allowed to the kernel's arithmetic (whose
#    error scales with the values averaged, not with |o|: logits within their
#    own 1e-4 tolerance move an output over ~20-sized outlier values by several
#    1e-4), so the bound is 2e-3 itself wherever the dtype's rounding leaves
#    room (bf16 below |o| = 0.5, every f32 output) and the correctly rounded
#    value plus that allowance elsewhere (2.95e-3 at bf16 |o| in [0.5, 1)).
RHO_ULP = 4
RNORM_ULP = 4
LOGIT_REL, LOGIT_ABS = 1e-3, 1e-4
OUT_ABS = 2e-3
OUT_ARITH = 1e-3

# Near-boundary exemptions seen by compare_keys calls given a label: (label, counts).
# The session summary (conftest.py) prints them, so every GPU test log carries them.
PARITY_COUNTS = []

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def nat():
    from compressed_attention_turboquantprod_b200 import build
    build.build()
    from compressed_attention_turboquantprod_b200 import native
    return native


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def oracle_setup(d, b1, m, layer=0, structured=False):
    """The oracle's own stored projections and codebook (numpy fp32); structured:
    the Hadamard rotation."""
    p = oproj.make_projections(d, m, layer, with_rotation=b1 > 0, structured=structured)
    cb = ocb.build(d, b1) if b1 > 0 else (None, None)
    return p, cb


def to_dev(a, device="cuda"):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device)


def unpack_bits_dev(packed: torch.Tensor, nbits: int) -> np.ndarray:
    return olayout.unpack_bits(packed.cpu().numpy(), nbits)


def compare_keys(gpu: dict, ref: dict, d: int, b1: int, m: int, beta32, label=None):
    """gpu: dict of host numpy arrays (idx planes bytes, signs bytes, rho, rnorm);
    ref: oracle quantize_keys output.  Asserts parity; returns counts (recorded
    in PARITY_COUNTS under `label` when one is given)."""
    n = ref["rho"].shape[0]
    bits_g = olayout.unpack_bits(gpu["signs"], m)
    skip_tok = np.zeros(n, bool)
    n_code_mis = n_code_ex = 0
    if b1 > 0:
        idx_g = np.zeros((n, d), np.uint8)
        nb = d // 8
        for p in range(b1):
            idx_g |= olayout.unpack_bits(gpu["idx"][:, p * nb:(p + 1) * nb], d) << p
        ex = oq.code_exempt(ref["y32"], beta32)
        mis = idx_g != ref["idx"]
        n_code_ex = int(ex.sum())
        n_code_mis = int(mis.sum())
        assert not np.any(mis & ~ex), f"{int((mis & ~ex).sum())} non-exempt code mismatches"
        skip_tok = np.any(mis, axis=1)
    sex = oq.sign_exempt(ref["z"])
    smis = (bits_g != ref["bits"]) & ~skip_tok[:, None]
    assert not np.any(smis & ~sex), f"{int((smis & ~sex).sum())} non-exempt sign mismatches"
    rho_g = gpu["rho"].astype(np.float32)
    ulp = np.spacing(np.abs(ref["rho"]).astype(np.float32))
    assert np.all(np.abs(rho_g - ref["rho"]) <= RHO_ULP * ulp + 0.0)
    if b1 > 0:
        rn_g = gpu["rnorm"].astype(np.float64)
        rn_r = ref["rnorm"].astype(np.float64)
        # ||r|| = rho ||y - c[idx]|| with y from the fp32 rotation: |dy_j| <= 2^-21 |u| = 2^-21,
        # so |d||r||| <= rho sqrt(d) 2^-21, plus the fp32 rounding of the stored value
        tol = RNORM_ULP * np.spacing(np.abs(rn_r).astype(np.float32)) + \
            ref["rho"].astype(np.float64) * np.sqrt(d) * 2.0 ** -21
        ok = np.abs(rn_g - rn_r) <= tol
        assert np.all(ok | skip_tok), f"rnorm max err / tol {np.max((np.abs(rn_g - rn_r) / tol)[~skip_tok])}"
    # tokens whose stored codes or sign bits differ (inside the band): their logits
    # legitimately differ from the oracle's, so end-to-end checks skip their units
    flip_tok = skip_tok | np.any(smis, axis=1)
    counts = {"tokens": int(n), "code_mismatch": n_code_mis, "code_exempt": n_code_ex,
              "sign_mismatch": int(smis.sum()), "sign_exempt": int(sex.sum()),
              "skipped_tokens": int(flip_tok.sum())}
    if label is not None:
        PARITY_COUNTS.append((label, counts))
    return counts


def record(label, **counts):
    """Record a count that is not a key comparison (e.g. units whose end-to-end
    output check was skipped because a code flipped inside the boundary band)."""
    PARITY_COUNTS.append((label, counts))


def check_logits(got: np.ndarray, want: np.ndarray):
    err = np.abs(got - want)
    ok = (err <= LOGIT_REL * np.abs(want)) | (err <= LOGIT_ABS)
    assert np.all(ok), f"logit mismatch: worst {np.max(err)} at |want| {np.abs(want).flat[np.argmax(err)]}"


HALF_ULP_BITS = {"f32": 24, "f16": 11, "bf16": 8}    # significand bits of each storage type


def storage_half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Half an ulp of |x| in the output dtype (rounding-to-nearest error bound)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return 0.5 * np.exp2(e - (HALF_ULP_BITS[dtype] - 1))


def out_tolerance(want: np.ndarray, dtype: str) -> np.ndarray:
    """max(2e-3, half an ulp of the output dtype at |o| + 1e-3)."""
    return np.maximum(OUT_ABS, storage_half_ulp(want, dtype) + OUT_ARITH)


# worst error / bound seen by check_out in this session (printed with the counts)
OUT_WORST = {"ratio": 0.0, "err": 0.0, "abs_o": 0.0}


def check_out(got: np.ndarray, want: np.ndarray, dtype: str = "bf16"):
    if not got.size:
        return 0.0
    err = np.abs(got - want)
    tol = out_tolerance(want, dtype)
    i = int(np.argmax(err / tol))
    if err.flat[i] / tol.flat[i] > OUT_WORST["ratio"]:
        OUT_WORST.update(ratio=float(err.flat[i] / tol.flat[i]), err=float(err.flat[i]),
                         abs_o=float(abs(want.flat[i])))
    assert np.all(err <= tol), (f"output error {err.flat[i]:.3g} over its bound {tol.flat[i]:.3g} "
                                f"at |o| = {abs(want.flat[i]):.3g} (max |o| {np.max(np.abs(want)):.3g})")
    return float(np.max(err))
