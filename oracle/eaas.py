"""SO(2) (EAAS) weights <-> dense Clebsch-Gordan path weights, fp64 (oracle;
test infrastructure).

Source: gist.science, Technical Summary 2.1 (EAAS): in the frame whose z axis
is the inter-atomic axis, the edge harmonics are zero except at m = 0
(Lemma 4.1), and commuting the rotation through the tensor product collapses
the dense contraction into a re-indexing rule (Eq. 13) with sparse blockwise
linear maps; the fugumt abstract calls it "sparse parity re-indexing". The
pages do not print Eq. 13. Reading taken (and pinned by tests against the
dense contraction): with c_l2 = Y_l2,0(z) = sqrt((2 l2 + 1)/(4 pi)) and the
real coupling tensor Q of ``oracle.cg``, for every l1, l3 and 0 <= m <= min(l1, l3)

    A(m)[l3, l1] = sum over l2 with l1+l2+l3 even of c_l2 Q^{l1 l2 l3}[ m, 0, m] w_{l1 l2 l3}
    B(m)[l3, l1] = sum over l2 with l1+l2+l3 odd  of c_l2 Q^{l1 l2 l3}[ m, 0,-m] w_{l1 l2 l3}

and the aligned-frame message is, per |m| block,

    o[l3, +m] = sum_l1 A(m)[l3,l1] h[l1,+m] - B(m)[l3,l1] h[l1,-m]
    o[l3, -m] = sum_l1 B(m)[l3,l1] h[l1,+m] + A(m)[l3,l1] h[l1,-m]

(m = 0: only A(0)). Each (l1, l3) pair has 2 min(l1,l3) + 1 paths and as many
(A, B) coefficients, and the map between them is square and invertible, so
the SO(2) weights that the library takes are a one-to-one re-parametrisation
of the dense path weights. ``paths_from_so2`` inverts it, so the oracle can
evaluate the layer the dense way from the library's own inputs.

Packed storage of the SO(2) weights: A(0), then A(m), B(m) for m = 1..L;
block m is a row-major square matrix indexed [(l3, c_out), (l1, c_in)] with
l3, l1 running over m..L.
"""
from __future__ import annotations

from math import pi, sqrt

import numpy as np

from .cg import real_cg


def _c(l2: int) -> float:
    return sqrt((2 * l2 + 1) / (4 * pi))


def unpack_so2(flat: np.ndarray, L: int, C: int):
    """Packed vector -> (A, B): dicts m -> square fp64 matrix (B has m >= 1)."""
    flat = np.asarray(flat, dtype=np.float64)
    A, B, o = {}, {}, 0
    n = (L + 1) * C
    A[0] = flat[o:o + n * n].reshape(n, n)
    o += n * n
    for m in range(1, L + 1):
        n = (L + 1 - m) * C
        A[m] = flat[o:o + n * n].reshape(n, n)
        o += n * n
        B[m] = flat[o:o + n * n].reshape(n, n)
        o += n * n
    assert o == flat.size, "packed SO(2) weight vector has the wrong length"
    return A, B


def pack_so2(A, B, L: int) -> np.ndarray:
    parts = [A[0].ravel()]
    for m in range(1, L + 1):
        parts += [A[m].ravel(), B[m].ravel()]
    return np.concatenate(parts)


def _blk(M: np.ndarray, m: int, l3: int, l1: int, C: int) -> np.ndarray:
    return M[(l3 - m) * C:(l3 - m + 1) * C, (l1 - m) * C:(l1 - m + 1) * C]


def _systems(l1: int, l3: int):
    """Coefficient matrices of the even-parity (A) and odd-parity (B) maps."""
    mn = min(l1, l3)
    lo, hi = abs(l1 - l3), l1 + l3
    even = [l2 for l2 in range(lo, hi + 1) if (l1 + l2 + l3) % 2 == 0]
    odd = [l2 for l2 in range(lo, hi + 1) if (l1 + l2 + l3) % 2 == 1]
    Me = np.array([[_c(l2) * real_cg(l1, l2, l3)[m + l1, l2, m + l3] for l2 in even]
                   for m in range(0, mn + 1)])
    Mo = np.array([[_c(l2) * real_cg(l1, l2, l3)[m + l1, l2, -m + l3] for l2 in odd]
                   for m in range(1, mn + 1)]).reshape(mn, len(odd))
    return even, odd, Me, Mo


def so2_from_paths(w: dict, L: int, C: int):
    """Dense path weights {(l1,l2,l3): [C_out, C_in]} -> (A, B) SO(2) blocks."""
    A = {0: np.zeros(((L + 1) * C,) * 2)}
    B = {}
    for m in range(1, L + 1):
        n = (L + 1 - m) * C
        A[m] = np.zeros((n, n))
        B[m] = np.zeros((n, n))
    for l1 in range(L + 1):
        for l3 in range(L + 1):
            even, odd, Me, Mo = _systems(l1, l3)
            for m in range(0, min(l1, l3) + 1):
                _blk(A[m], m, l3, l1, C)[...] = sum(Me[m, e] * w[(l1, l2, l3)] for e, l2 in enumerate(even))
                if m >= 1:
                    _blk(B[m], m, l3, l1, C)[...] = sum(Mo[m - 1, o] * w[(l1, l2, l3)] for o, l2 in enumerate(odd))
    return A, B


def paths_from_so2(A, B, L: int, C: int) -> dict:
    """Inverse of ``so2_from_paths``: solve each (l1, l3) system."""
    w = {}
    for l1 in range(L + 1):
        for l3 in range(L + 1):
            even, odd, Me, Mo = _systems(l1, l3)
            mn = min(l1, l3)
            Ae = np.stack([_blk(A[m], m, l3, l1, C) for m in range(0, mn + 1)])   # [mn+1, C, C]
            we = np.einsum("em,mab->eab", np.linalg.inv(Me), Ae)
            for e, l2 in enumerate(even):
                w[(l1, l2, l3)] = we[e]
            if mn >= 1:
                Bo = np.stack([_blk(B[m], m, l3, l1, C) for m in range(1, mn + 1)])
                wo = np.einsum("om,mab->oab", np.linalg.inv(Mo), Bo)
                for o, l2 in enumerate(odd):
                    w[(l1, l2, l3)] = wo[o]
    return w
