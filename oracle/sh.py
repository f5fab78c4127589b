"""Real spherical harmonics of a direction, fp64 (oracle; test infrastructure).

The pages (gist.science, Technical Summary 2.1, "SO(3) -> SO(2) Change of
Basis") speak of spherical harmonics of the inter-atomic axis without fixing
a basis. Reading taken: orthonormal real harmonics on the unit sphere,
ordered m = -l..l at flat index l*l + l + m, built from the associated
Legendre functions WITHOUT the Condon-Shortley phase:

    Y_l0  = N_l0 P_l(z)
    Y_lm  = sqrt(2) N_lm P_l^m(cos t) cos(m p)      (m > 0)
    Y_l-m = sqrt(2) N_lm P_l^m(cos t) sin(m p)      (m > 0)
    N_lm  = sqrt((2l+1)/(4 pi) (l-m)!/(l+m)!)

so Y_1(-1,0,1) is proportional to (y, z, x). Written in Cartesian form: with
rho^m cos(m p) = Re (x+iy)^m and rho^m sin(m p) = Im (x+iy)^m, and
P_l^m(z) = rho^m d^m P_l/dz^m, every harmonic is a polynomial in (x, y, z).
Solid harmonics would only rescale each degree by |r|^l; the layer applies
them to unit vectors.
"""
from __future__ import annotations

from functools import lru_cache
from math import factorial, pi, sqrt

import numpy as np
from numpy.polynomial import legendre as _leg
from numpy.polynomial import polynomial as _poly


def sh_index(l: int, m: int) -> int:
    return l * l + l + m


@lru_cache(maxsize=None)
def _dm_legendre(l: int, m: int) -> np.ndarray:
    """Power-series coefficients of d^m/dz^m P_l(z)."""
    c = np.zeros(l + 1)
    c[l] = 1.0
    p = _leg.leg2poly(c)
    return _poly.polyder(p, m) if m > 0 else p


def real_sh(lmax: int, vec) -> np.ndarray:
    """Y_lm(vec/|vec|) for l <= lmax; shape [..., (lmax+1)^2]."""
    v = np.asarray(vec, dtype=np.float64)
    shape = v.shape[:-1]
    v = v.reshape(-1, 3)
    u = v / np.linalg.norm(v, axis=1, keepdims=True)
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    out = np.empty((u.shape[0], (lmax + 1) ** 2))
    xy = x + 1j * y
    for l in range(lmax + 1):
        for m in range(l + 1):
            n = sqrt((2 * l + 1) / (4 * pi) * factorial(l - m) / factorial(l + m))
            q = _poly.polyval(z, _dm_legendre(l, m))
            if m == 0:
                out[:, sh_index(l, 0)] = n * q
            else:
                w = xy ** m
                out[:, sh_index(l, m)] = sqrt(2.0) * n * q * w.real
                out[:, sh_index(l, -m)] = sqrt(2.0) * n * q * w.imag
    return out.reshape(*shape, (lmax + 1) ** 2)


def real_from_complex(l: int) -> np.ndarray:
    """Unitary U_l with Y_real = U_l Y_complex (complex SH with the
    Condon-Shortley phase). Rows: real m = -l..l; columns: complex mu."""
    U = np.zeros((2 * l + 1, 2 * l + 1), dtype=complex)
    s = 1.0 / sqrt(2.0)
    for m in range(-l, l + 1):
        r = m + l
        if m > 0:
            U[r, m + l] = (-1) ** m * s
            U[r, -m + l] = s
        elif m < 0:
            U[r, m + l] = 1j * s
            U[r, -m + l] = -1j * (-1) ** (-m) * s
        else:
            U[r, l] = 1.0
    return U
