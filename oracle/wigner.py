"""Real Wigner-D matrices, fp64 (oracle; test infrastructure).

The pages (gist.science, Technical Summary 2.1) rotate features into the
frame of the inter-atomic axis but fix no convention. Reading taken: D^l(R)
is the matrix with

    Y_l(R v) = D^l(R) Y_l(v)    for every direction v,

Y_l the real harmonics of ``oracle.sh``. This module evaluates that
definition directly: it samples directions v_k, evaluates both sides and
solves the (over-determined, exactly consistent) linear system for D^l.
"""
from __future__ import annotations

import numpy as np

from .sh import real_sh

_rng = np.random.default_rng(12345)
_DIRS = _rng.normal(size=(96, 3))
_DIRS /= np.linalg.norm(_DIRS, axis=1, keepdims=True)


def wigner_D(l: int, R: np.ndarray) -> np.ndarray:
    """D^l(R), shape [2l+1, 2l+1], for one 3x3 rotation R."""
    R = np.asarray(R, dtype=np.float64)
    s = slice(l * l, (l + 1) ** 2)
    Y = real_sh(l, _DIRS)[:, s]                 # [n, 2l+1]
    Yr = real_sh(l, _DIRS @ R.T)[:, s]          # Y(R v_k)
    # rows: Yr[k] = D @ Y[k]  ->  Y @ D^T = Yr
    Dt, *_ = np.linalg.lstsq(Y, Yr, rcond=None)
    return Dt.T


def wigner_D_all(L: int, R: np.ndarray) -> list[np.ndarray]:
    return [wigner_D(l, R) for l in range(L + 1)]


def rotate_irreps(x: np.ndarray, L: int, R: np.ndarray) -> np.ndarray:
    """Apply D^l(R) to every degree of x[..., (L+1)^2, C]."""
    out = np.empty_like(x, dtype=np.float64)
    for l in range(L + 1):
        s = slice(l * l, (l + 1) ** 2)
        out[..., s, :] = np.einsum("ab,...bc->...ac", wigner_D(l, R), x[..., s, :])
    return out


def random_rotation(rng) -> np.ndarray:
    a = rng.normal(size=(3, 3))
    q, r = np.linalg.qr(a)
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] *= -1
    return q


def rot_z(a: float) -> np.ndarray:
    c, s = np.cos(a), np.sin(a)
    return np.array([[c, -s, 0.0], [s, c, 0.0], [0.0, 0.0, 1.0]])


def rot_y(a: float) -> np.ndarray:
    c, s = np.cos(a), np.sin(a)
    return np.array([[c, 0.0, s], [0.0, 1.0, 0.0], [-s, 0.0, c]])
