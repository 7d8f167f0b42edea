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
"""
from __future__ import annotations

import numpy as np

from . import philox

STREAM_PI, STREAM_S = 0, 1


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


def make_projections(d: int, m: int, layer: int, base_seed: int = 42, stride: int = 7,
                     with_rotation: bool = True):
    """Stored (fp32) projections of one layer: dict with Pi [d,d] (None for pure
    QJL), S [m,d] and T = S Pi^T [m,d] (T = S for pure QJL)."""
    seed = layer_seed(layer, base_seed, stride)
    S32 = gaussian_matrix(m, d, seed, STREAM_S).astype(np.float32)
    if with_rotation:
        Pi32 = rotation(d, seed).astype(np.float32)
        T32 = (S32.astype(np.float64) @ Pi32.astype(np.float64).T).astype(np.float32)
    else:
        Pi32 = None
        T32 = S32.copy()
    return {"Pi": Pi32, "S": S32, "T": T32, "seed": seed}
