"""The Wigner-6j node-level convolution, computed edge by edge in fp64
(oracle; test infrastructure).

Source: the fugumt abstract page (the E2Former-V2 abstract, where EAAS
starts from the Wigner-6j convolution; the E2Former conclusion on the same
page, where that convolution moves the work from edges to nodes, O(|E|) to
O(|V|)), and gist.science, Technical Summary 3 (EAAS joins Wigner-6j
recoupling with the SO(2) axis alignment). The pages name the operation and
its complexity but print no formula. The reading taken here is the plainest
layer whose edge tensor product can be moved onto the nodes:

  geometry   open boundaries; r_ij = x_j - x_i
  harmonics  S^l_m(r) = sqrt(4 pi/(2l+1)) |r|^l Y_lm(r/|r|)  (regular solid
             harmonics in the real basis of ``oracle.sh``; S^0 = 1, and
             S^l(0) = 0 for l > 0)
  value      v_ij[l3,m3,c] = sum over paths (l1,l2,l3) of w_{l1l2l3}[c]
             sum_{m1,m2} Q^{l1l2l3}[m1,m2,m3] x_j[l1,m1,c] S^l2_m2(r_ij),
             paths: l1, l3 <= L, |l1-l3| <= l2 <= min(l1+l3, Lf); one weight
             per path and channel (no radial gate on the value, so the
             product of x_j with the harmonic can be split over the nodes)
  logit      as the main layer: a_ij^h = g_a^h <q_i^h, k_j^h> / sqrt(C/H),
             g_a = rho(|r_ij|) W_rad with W_rad [n_rbf, H]
  output     out_i[l,m,c] = sum_j softmax_j(a_ij^{h(c)}) v_ij[l,m,c];
             0 when N(i) is empty

Why the node split exists (the reason the CUDA path may take it, and what
the pins in the tests check): S^l2(a + b) = sum_lam sqrt(binom(2 l2, 2 lam))
[S^lam(a) (x) S^(l2-lam)(b)]^l2 (the addition theorem of solid harmonics),
and the re-coupling of x_j (x) [S^lam (x) S^mu]^l2 into
[[x_j (x) S^lam]^k (x) S^mu]^l3 has the 6j symbols
{l1 lam k; mu l3 l2} as coefficients. This module evaluates only the edge
form above; ``wigner_6j`` is Racah's closed form, for the pins.
"""
from __future__ import annotations

from fractions import Fraction
from math import factorial, pi, sqrt

import numpy as np

from .cg import real_cg
from .layer import edge_vectors, radial_basis, softmax_two_pass
from .sh import real_sh


def solid_harmonics(lmax: int, r) -> np.ndarray:
    """S^l_m(r) for l <= lmax, flat index l*l + l + m; shape [..., (lmax+1)^2]."""
    r = np.asarray(r, np.float64)
    shape = r.shape[:-1]
    r = r.reshape(-1, 3)
    n = np.linalg.norm(r, axis=1)
    out = np.zeros((r.shape[0], (lmax + 1) ** 2))
    out[:, 0] = 1.0
    nz = n > 0
    if lmax > 0 and nz.any():
        Y = real_sh(lmax, r[nz])
        for l in range(1, lmax + 1):
            sl = slice(l * l, (l + 1) ** 2)
            out[nz, sl] = sqrt(4 * pi / (2 * l + 1)) * n[nz, None] ** l * Y[:, sl]
    return out.reshape(*shape, (lmax + 1) ** 2)


def sixj_paths(L: int, Lf: int):
    """The layer's paths in their packed order: l1, then l3, then l2 ascending."""
    return [(l1, l2, l3) for l1 in range(L + 1) for l3 in range(L + 1)
            for l2 in range(abs(l1 - l3), min(l1 + l3, Lf) + 1)]


def _delta(a: int, b: int, c: int) -> Fraction:
    f = factorial
    return Fraction(f(a + b - c) * f(a - b + c) * f(-a + b + c), f(a + b + c + 1))


def wigner_6j(j1: int, j2: int, j3: int, j4: int, j5: int, j6: int) -> float:
    """{j1 j2 j3; j4 j5 j6} for integer arguments, Racah's formula in exact
    rationals (one square root at the end)."""
    tri = [(j1, j2, j3), (j1, j5, j6), (j4, j2, j6), (j4, j5, j3)]
    for a, b, c in tri:
        if c < abs(a - b) or c > a + b:
            return 0.0
    pre = Fraction(1)
    for a, b, c in tri:
        pre *= _delta(a, b, c)
    f = factorial
    lo = max(j1 + j2 + j3, j1 + j5 + j6, j4 + j2 + j6, j4 + j5 + j3)
    hi = min(j1 + j2 + j4 + j5, j2 + j3 + j5 + j6, j3 + j1 + j6 + j4)
    s = Fraction(0)
    for t in range(lo, hi + 1):
        den = (f(t - j1 - j2 - j3) * f(t - j1 - j5 - j6) * f(t - j4 - j2 - j6) * f(t - j4 - j5 - j3)
               * f(j1 + j2 + j4 + j5 - t) * f(j2 + j3 + j5 + j6 - t) * f(j3 + j1 + j6 + j4 - t))
        s += Fraction((-1) ** t * f(t + 1), den)
    if s == 0:
        return 0.0
    return (1.0 if s > 0 else -1.0) * sqrt(float(s * s * pre))


class SixjLayer:
    """The edge form of the layer, one destination node at a time."""

    def __init__(self, L, Lf, C, H, n_rbf, cutoff, Wq, Wk, Wrad, w_path):
        self.L, self.Lf, self.C, self.H, self.n_rbf, self.cutoff = L, Lf, C, H, n_rbf, float(cutoff)
        self.Wq = np.asarray(Wq, np.float64)
        self.Wk = np.asarray(Wk, np.float64)
        self.Wrad = np.asarray(Wrad, np.float64).reshape(n_rbf, H)
        P = sixj_paths(L, Lf)
        w = np.asarray(w_path, np.float64).reshape(len(P), C)
        self.w = {p: w[n] for n, p in enumerate(P)}

    def messages(self, x, r, j):
        """v[e, k, c] for edges with vectors r[e] from neighbours j[e]."""
        S = solid_harmonics(self.Lf, r)
        v = np.zeros((r.shape[0], (self.L + 1) ** 2, self.C))
        for (l1, l2, l3), wc in self.w.items():
            Q = real_cg(l1, l2, l3)
            t = np.einsum("abc,eai,eb->eci", Q, x[j, l1 * l1:(l1 + 1) ** 2, :],
                          S[:, l2 * l2:(l2 + 1) ** 2], optimize=True)
            v[:, l3 * l3:(l3 + 1) ** 2, :] += t * wc
        return v

    def __call__(self, pos, row_ptr, col, x, nodes=None):
        L, C, H = self.L, self.C, self.H
        x = np.asarray(x, np.float64)
        N = x.shape[0]
        nodes = np.arange(N) if nodes is None else np.asarray(nodes)
        dh = C // H
        q = x[:, 0, :] @ self.Wq.T
        k = x[:, 0, :] @ self.Wk.T
        row_ptr = np.asarray(row_ptr, np.int64)
        col = np.asarray(col, np.int64)
        out = np.zeros((nodes.size, (L + 1) ** 2, C))
        for n, i in enumerate(nodes):
            j = col[row_ptr[i]:row_ptr[i + 1]]
            if j.size == 0:
                continue
            r = edge_vectors(pos, None, np.full(j.size, i), j)
            d = np.linalg.norm(r, axis=1)
            g_a = radial_basis(d, self.cutoff, self.n_rbf) @ self.Wrad
            dots = (q[i].reshape(H, dh)[None] * k[j].reshape(-1, H, dh)).sum(-1)
            alpha = softmax_two_pass(g_a * dots / np.sqrt(dh))
            v = self.messages(x, r, j)
            out[n] = np.einsum("ec,ekc->kc", np.repeat(alpha, dh, axis=1), v)
        return out
