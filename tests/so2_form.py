"""SO(2)-form evaluator of one value message, fp64 (test helper).

Evaluates v = D(R)^T SO2_W(D(R) h) with R a rotation taking the edge
direction to +z (E2Former-V2, gist.science Technical Summary 2.1: rotate into
the frame of the inter-atomic axis, apply the sparse blockwise maps of the
re-indexing rule, Eq. 13). It is used only to prove that the dense oracle's
CG form equals the SO(2) form; it is never the GPU parity reference.
"""
from __future__ import annotations

import numpy as np

from oracle.wigner import wigner_D


def edge_frame(r: np.ndarray) -> np.ndarray:
    """A rotation R with R r^ = +z (built from r^'s polar and azimuthal angles)."""
    rh = r / np.linalg.norm(r)
    x, y, z = rh
    rho = np.hypot(x, y)
    cp, sp = (x / rho, y / rho) if rho > 0 else (1.0, 0.0)
    return np.array([[z * cp, z * sp, -rho], [-sp, cp, 0.0], [x, y, z]])


def so2_apply(ht: np.ndarray, A: dict, B: dict, L: int, C: int) -> np.ndarray:
    """Aligned-frame map: ht[(L+1)^2, C] -> o[(L+1)^2, C]."""
    o = np.zeros_like(ht)

    def k(l, m):
        return l * l + l + m

    for m in range(0, L + 1):
        ls = range(m, L + 1)
        hp = np.concatenate([ht[k(l, m)] for l in ls])
        if m == 0:
            op = A[0] @ hp
            for a, l in enumerate(ls):
                o[k(l, 0)] = op[a * C:(a + 1) * C]
            continue
        hm = np.concatenate([ht[k(l, -m)] for l in ls])
        op = A[m] @ hp - B[m] @ hm
        om = B[m] @ hp + A[m] @ hm
        for a, l in enumerate(ls):
            o[k(l, m)] = op[a * C:(a + 1) * C]
            o[k(l, -m)] = om[a * C:(a + 1) * C]
    return o


def so2_message(r, h, A, B, L, C, R=None):
    R = edge_frame(r) if R is None else R
    Ds = [wigner_D(l, R) for l in range(L + 1)]
    ht = np.concatenate([Ds[l] @ h[l * l:(l + 1) ** 2] for l in range(L + 1)])
    o = so2_apply(ht, A, B, L, C)
    return np.concatenate([Ds[l].T @ o[l * l:(l + 1) ** 2] for l in range(L + 1)])
