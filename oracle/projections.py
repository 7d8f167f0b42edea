"""Per-layer random rotation Pi and Gaussian sketch S.

[TQ] §二: the rotation is an orthogonal matrix from a QR factorisation (d x d,
64 KB at d = 128, i.e. stored as fp32), one per layer with a fixed seed; the
residual is projected by a random Gaussian matrix S.  [TQ] §六: each layer uses
seed 42 + 7 * layer so that the noise of different layers is uncorrelated.

Readings taken where the pages are silent:

* generator: Philox4x64-10 + Box-Muller (``oracle.philox``); stream 0 is the
  Gaussian source of Pi, stream 1 is S; element (i, j) of a row-major matrix
  with ``cols`` columns is draw ``i * cols + j``.
* Pi = Q diag(sign(diag R)) from the QR factorisation G = Q R of the d x d
  Gaussian G: the sign fix makes the factorisation unique (R_ii > 0), which is
  what makes Q Haar-distributed (Mezzadri 2007).  Rotation convention y = Pi u.
* S is the m x d Gaussian, no normalisation (the 1/m lives in the estimator).
* T = S Pi^T (m x d) is the sketch written in rotated coordinates; the oracle
  itself never uses it (it sketches r in the original space) but it is a stored
  output of the library's projection call, so its expected value is defined here.

Structured variant ([NQ] "无需训练即可将大模型的 KV 缓存压缩 33 倍", six-stage
pipeline, step 4: a Hadamard rotation spreads the energy of a vector evenly over
the coordinates and removes outliers before quantisation): Pi = H diag(s) / sqrt(d)
with H the Sylvester Hadamard matrix (H_1 = [1], H_2n = [[H, H], [H, -H]]), d a
power of two, and random signs s_c = +1 when the top bit of word w0 of Philox
draw c on stream 2 is 0, else -1 (reading: the page names neither the sign
source nor the normalisation; 1/sqrt(d) makes Pi orthogonal).  Pi u is then a
fast Walsh-Hadamard transform of s * u, O(d log d).
"""
from __future__ import annotations

import numpy as np

from . import philox

STREAM_PI, STREAM_S, STREAM_HD = 0, 1, 2


def layer_seed(layer: int, base_seed: int = 42, stride: int = 7) -> int:
    """[TQ] §六: per-layer seed 42 + 7 * layer."""
    return base_seed + stride * layer


def gaussian_matrix(rows: int, cols: int, seed: int, stream: int) -> np.ndarray:
    return philox.gaussian(rows * cols, seed, stream).reshape(rows, cols)


def rotation(d: int, seed: int) -> np.ndarray:
    """Pi (float64, before storage rounding): Q of G = QR with positive diag(R)."""
    G = gaussian_matrix(d, d, seed, STREAM_PI)
    Q, R = np.linalg.qr(G)
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s[None, :]


def sylvester_hadamard(d: int) -> np.ndarray:
    """H_d by the Sylvester recursion (d a power of two), float64 entries +-1."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def hadamard_signs(d: int, seed: int) -> np.ndarray:
    """s_c in {+1, -1}: +1 when the top bit of word w0 of Philox draw c (stream 2) is 0."""
    w0 = philox.philox4x64_10((np.arange(d, dtype=np.uint64), 0, 0, 0), (seed, STREAM_HD))[0]
    return np.where((w0 >> np.uint64(63)) == 0, 1.0, -1.0)


def hadamard_rotation(d: int, seed: int) -> np.ndarray:
    """Pi = H diag(s) / sqrt(d) (float64, before storage rounding)."""
    return sylvester_hadamard(d) * hadamard_signs(d, seed)[None, :] / np.sqrt(d)


def make_projections(d: int, m: int, layer: int, base_seed: int = 42, stride: int = 7,
                     with_rotation: bool = True, structured: bool = False):
    """Stored (fp32) projections of one layer: dict with Pi [d,d] (None for pure
    QJL), S [m,d] and T = S Pi^T [m,d] (T = S for pure QJL).  structured: the
    Hadamard rotation instead of the QR one."""
    seed = layer_seed(layer, base_seed, stride)
    S32 = gaussian_matrix(m, d, seed, STREAM_S).astype(np.float32)
    if with_rotation:
        Pi32 = (hadamard_rotation(d, seed) if structured else rotation(d, seed)).astype(np.float32)
        T32 = (S32.astype(np.float64) @ Pi32.astype(np.float64).T).astype(np.float32)
    else:
        Pi32 = None
        T32 = S32.copy()
    return {"Pi": Pi32, "S": S32, "T": T32, "seed": seed}
