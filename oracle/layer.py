"""The on-the-fly equivariant attention layer, computed the dense way in fp64
(oracle; test infrastructure).

Source: gist.science, Technical Summary 2.1 and 2.2; fugumt abstract. What
the pages fix: queries and keys are SO(3)-invariant scalar projections of
the node features (Eq. 6), the geometry enters only through the value path,
the value path is the equivariant tensor product of a neighbour's features
with the harmonics of the inter-atomic axis, and each node's output is the
softmax-weighted sum of its neighbours' messages. The pages print none of
the formulas; the readings taken are:

  geometry   r = mic(x_j - x_i), d = |r|, r^ = r/d (direction j - i)
  radial     rho_k(d) = u(d) exp(-((d - mu_k)/delta)^2), k = 0..n_rbf-1,
             mu_k = k rc/(n_rbf-1), delta = rc/(n_rbf-1),
             u(d) = (cos(pi d/rc) + 1)/2;  [g_v | g_a] = rho W_rad
  value      h_j[l,m,c] = g_v[l,c] x_j[l,m,c];
             v_ij[l3,m3,o] = sum over paths (l1,l2,l3) of
                             sum_c w_{l1l2l3}[o,c] sum_{m1,m2} Q[m1,m2,m3] h_j[l1,m1,c] Y_l2m2(r^)
             with l2 up to 2L and w converted from the SO(2) weights
  logit      q = W_q x[l=0], k = W_k x[l=0], split in H heads of d = C/H;
             a_ij^h = g_a^h <q_i^h, k_j^h> / sqrt(d)
  softmax    over j in N(i), per head, two passes (max, then sum)
  output     out_i[l,m,c] = sum_j alpha_ij^{head(c)} v_ij[l,m,c]; 0 if N(i) is empty

Inputs are the library's own (packed bf16/fp32 values given here as exact
fp64 numbers), so input rounding is not counted as error.
"""
from __future__ import annotations

import numpy as np

from .cg import real_cg
from .eaas import paths_from_so2, unpack_so2
from .sh import real_sh


def radial_basis(d: np.ndarray, cutoff: float, n_rbf: int) -> np.ndarray:
    mu = np.arange(n_rbf) * (cutoff / (n_rbf - 1))
    delta = cutoff / (n_rbf - 1)
    u = 0.5 * (np.cos(np.pi * d / cutoff) + 1.0)
    return u[:, None] * np.exp(-(((d[:, None] - mu[None, :]) / delta) ** 2))


def edge_vectors(pos, box, i, j):
    p = np.asarray(pos, np.float64)
    r = p[j] - p[i]
    if box is not None:
        b = np.asarray(box, np.float64)
        r = r - b * np.rint(r / b)
    return r


def dense_messages(h: np.ndarray, Y: np.ndarray, w: dict) -> np.ndarray:
    """v[e, k, c_out] from gated features h[e, k, c_in] and edge harmonics Y[e, :]."""
    v = np.zeros_like(h)
    for (l1, l2, l3), W in w.items():
        Q = real_cg(l1, l2, l3)
        t = np.einsum("abc,eai,eb->eci", Q, h[:, l1 * l1:(l1 + 1) ** 2, :],
                      Y[:, l2 * l2:(l2 + 1) ** 2], optimize=True)
        v[:, l3 * l3:(l3 + 1) ** 2, :] += t @ W.T
    return v


def softmax_two_pass(a: np.ndarray) -> np.ndarray:
    """Softmax over axis 0 of a[E, H]: max pass, then sum pass."""
    m = a.max(axis=0, keepdims=True)
    e = np.exp(a - m)
    return e / e.sum(axis=0, keepdims=True)


class DenseLayer:
    """Holds the converted weights; evaluates destination nodes in chunks."""

    def __init__(self, L, C, H, n_rbf, cutoff, Wq, Wk, Wrad, Wso2_f64):
        self.L, self.C, self.H, self.n_rbf, self.cutoff = L, C, H, n_rbf, float(cutoff)
        self.Wq = np.asarray(Wq, np.float64)
        self.Wk = np.asarray(Wk, np.float64)
        self.Wrad = np.asarray(Wrad, np.float64)
        A, B = unpack_so2(Wso2_f64, L, C)
        self.w = paths_from_so2(A, B, L, C)

    def edge_terms(self, pos, box, x, i, j):
        """Per-edge gates and dense messages for edges (i <- j)."""
        L, C, H = self.L, self.C, self.H
        r = edge_vectors(pos, box, i, j)
        d = np.linalg.norm(r, axis=1)
        g = radial_basis(d, self.cutoff, self.n_rbf) @ self.Wrad
        g_v = g[:, :(L + 1) * C].reshape(-1, L + 1, C)
        g_a = g[:, (L + 1) * C:]
        lk = np.concatenate([np.full(2 * l + 1, l) for l in range(L + 1)])
        h = g_v[:, lk, :] * x[j]
        Y = real_sh(2 * L, r)
        v = dense_messages(h, Y, self.w)
        return g_a, v

    def __call__(self, pos, box, row_ptr, col, x, nodes=None, chunk_edges=4096):
        L, C, H = self.L, self.C, self.H
        x = np.asarray(x, np.float64)
        N = x.shape[0]
        nodes = np.arange(N) if nodes is None else np.asarray(nodes)
        dh = C // H
        q = x[:, 0, :] @ self.Wq.T
        k = x[:, 0, :] @ self.Wk.T
        out = np.zeros((nodes.size, (L + 1) ** 2, C))
        row_ptr = np.asarray(row_ptr, np.int64)
        col = np.asarray(col, np.int64)
        s = 0
        while s < nodes.size:
            e_tot, t = 0, s
            while t < nodes.size and (t == s or e_tot + row_ptr[nodes[t] + 1] - row_ptr[nodes[t]] <= chunk_edges):
                e_tot += row_ptr[nodes[t] + 1] - row_ptr[nodes[t]]
                t += 1
            sel = nodes[s:t]
            seg = [np.arange(row_ptr[n], row_ptr[n + 1]) for n in sel]
            eidx = np.concatenate(seg) if seg else np.zeros(0, np.int64)
            if eidx.size:
                ii = np.repeat(sel, [g.size for g in seg])
                jj = col[eidx]
                g_a, v = self.edge_terms(pos, box, x, ii, jj)
                dots = (q[ii].reshape(-1, H, dh) * k[jj].reshape(-1, H, dh)).sum(-1)
                a = g_a * dots / np.sqrt(dh)
                o = 0
                for r_, g in enumerate(seg):
                    if g.size == 0:
                        continue
                    alpha = softmax_two_pass(a[o:o + g.size])           # [deg, H]
                    wgt = np.repeat(alpha, dh, axis=1)                  # [deg, C]
                    out[s + r_] = np.einsum("ec,ekc->kc", wgt, v[o:o + g.size])
                    o += g.size
            s = t
        return out
