"""Clebsch-Gordan coefficients and real coupling tensors, fp64 (oracle; test
infrastructure).

The pages (gist.science, Technical Summary 2.1) describe the standard layer
as a dense sum over Clebsch-Gordan coefficients, O(L^6), which EAAS replaces.
This module writes that dense coupling out:

* ``cg_complex`` is Racah's closed form for <l1 m1 l2 m2 | l3 m3>, evaluated in
  exact rational arithmetic and rounded once to fp64.
* ``real_cg`` is the coupling tensor Q[m1, m2, m3] between real harmonics of
  degrees l1 (x), l2 (the edge harmonic Y) and l3 (the output): if x and y
  transform like the real harmonics, z[m3] = sum Q[m1,m2,m3] x[m1] y[m2]
  transforms like them too. With Y_real = U Y_complex,

      Q = sum_mu U3[m3,mu3] conj(U1[m1,mu1]) conj(U2[m2,mu2]) <l1 mu1 l2 mu2|l3 mu3>,

  which is real when l1+l2+l3 is even and purely imaginary when it is odd;
  the non-zero part is returned. Any per-path scalar factor would be absorbed
  by the path weight w_{l1 l2 l3}, so the layer's output does not depend on it.
"""
from __future__ import annotations

from fractions import Fraction
from functools import lru_cache
from math import factorial, sqrt

import numpy as np

from .sh import real_from_complex


def cg_complex(l1: int, m1: int, l2: int, m2: int, l3: int, m3: int) -> float:
    """<l1 m1 l2 m2 | l3 m3> by Racah's formula (Condon-Shortley phase)."""
    if m1 + m2 != m3 or abs(m1) > l1 or abs(m2) > l2 or abs(m3) > l3:
        return 0.0
    if l3 < abs(l1 - l2) or l3 > l1 + l2:
        return 0.0
    f = factorial
    pre = Fraction((2 * l3 + 1) * f(l3 + l1 - l2) * f(l3 - l1 + l2) * f(l1 + l2 - l3),
                   f(l1 + l2 + l3 + 1))
    pre *= f(l3 + m3) * f(l3 - m3) * f(l1 - m1) * f(l1 + m1) * f(l2 - m2) * f(l2 + m2)
    s = Fraction(0)
    for k in range(0, l1 + l2 - l3 + 1):
        args = (k, l1 + l2 - l3 - k, l1 - m1 - k, l2 + m2 - k, l3 - l2 + m1 + k, l3 - l1 - m2 + k)
        if min(args) < 0:
            continue
        den = 1
        for a in args:
            den *= f(a)
        s += Fraction((-1) ** k, den)
    if s == 0:
        return 0.0
    sign = 1.0 if s > 0 else -1.0
    return sign * sqrt(float(s * s * pre))


@lru_cache(maxsize=None)
def cg_complex_tensor(l1: int, l2: int, l3: int) -> np.ndarray:
    C = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for a in range(-l1, l1 + 1):
        for b in range(-l2, l2 + 1):
            c = a + b
            if abs(c) <= l3:
                C[a + l1, b + l2, c + l3] = cg_complex(l1, a, l2, b, l3, c)
    return C


@lru_cache(maxsize=None)
def real_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    """Real coupling tensor Q[m1, m2, m3] (indices offset by l)."""
    U1, U2, U3 = real_from_complex(l1), real_from_complex(l2), real_from_complex(l3)
    Q = np.einsum("ci,aj,bk,jki->abc", U3, U1.conj(), U2.conj(), cg_complex_tensor(l1, l2, l3))
    if (l1 + l2 + l3) % 2 == 0:
        assert np.abs(Q.imag).max() < 1e-12
        out = Q.real
    else:
        assert np.abs(Q.real).max() < 1e-12
        out = Q.imag
    out = np.ascontiguousarray(out)
    out.setflags(write=False)
    return out


def paths(L: int):
    """All (l1, l2, l3) with l1, l3 <= L and |l1-l3| <= l2 <= l1+l3."""
    return [(l1, l2, l3) for l1 in range(L + 1) for l3 in range(L + 1)
            for l2 in range(abs(l1 - l3), l1 + l3 + 1)]
