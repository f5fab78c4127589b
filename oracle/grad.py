"""Gradients of the on-the-fly equivariant attention layer, fp64, by reverse-mode
differentiation of the dense definition (oracle; test infrastructure).

Source: gist.science, Technical Summary 2.1 and 2.2 (the layer), and the
pages' conservative variant, whose forces are the negative gradient of the
energy with respect to the positions: the backward pass of the layer is the
step that follows the forward. The pages print no backward formulas. This
module restates the layer of ``oracle.layer`` (same readings: geometry,
radial basis, gates, dense Clebsch-Gordan messages with l2 up to 2L, the
path weights obtained from the SO(2) weights, the Q/K logits, a softmax over
each node's neighbours, the weighted sum) in plain PyTorch fp64 CPU
operations, and differentiates the scalar loss sum(G * out) for a given
upstream gradient G with torch.autograd. The neighbour list is fixed (an
input), and the periodic image shift is piecewise constant, so it carries no
gradient.

Outputs: d loss / d (pos, x, W_q, W_k, W_rad, W_so2), each in its input's
shape (W_so2 in the packed order of the library).
"""
from __future__ import annotations

from math import factorial, pi, sqrt

import numpy as np
import torch

from .cg import real_cg
from .eaas import _systems
from .sh import _dm_legendre, sh_index


def _horner(coeffs: np.ndarray, z: torch.Tensor) -> torch.Tensor:
    acc = torch.zeros_like(z)
    for c in coeffs[::-1]:
        acc = acc * z + float(c)
    return acc


def real_sh_t(lmax: int, r: torch.Tensor) -> torch.Tensor:
    """Real harmonics of r/|r| (the convention of ``oracle.sh.real_sh``), differentiable."""
    u = r / torch.linalg.norm(r, dim=1, keepdim=True)
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    cs = [torch.ones_like(x)]
    sn = [torch.zeros_like(x)]
    for _ in range(1, lmax + 1):  # Re and Im of (x + i y)^m
        cs.append(x * cs[-1] - y * sn[-1])
        sn.append(x * sn[-1] + y * cs[-2])
    cols = [None] * (lmax + 1) ** 2
    for l in range(lmax + 1):
        for m in range(l + 1):
            n = sqrt((2 * l + 1) / (4 * pi) * factorial(l - m) / factorial(l + m))
            q = _horner(_dm_legendre(l, m), z)
            if m == 0:
                cols[sh_index(l, 0)] = n * q
            else:
                cols[sh_index(l, m)] = sqrt(2.0) * n * q * cs[m]
                cols[sh_index(l, -m)] = sqrt(2.0) * n * q * sn[m]
    return torch.stack(cols, dim=1)


def paths_from_so2_t(flat: torch.Tensor, L: int, C: int, M: int | None = None) -> dict:
    """Dense path weights from the packed SO(2) weights (``oracle.eaas.paths_from_so2``
    as a differentiable linear map). Blocks with m > M are absent (zero)."""
    M = L if M is None or M < 0 or M > L else M
    A, B, o = {}, {}, 0
    for m in range(0, M + 1):
        n = (L + 1 - m) * C
        A[m] = flat[o:o + n * n].reshape(n, n)
        o += n * n
        if m >= 1:
            B[m] = flat[o:o + n * n].reshape(n, n)
            o += n * n
    assert o == flat.numel(), "packed SO(2) weight vector has the wrong length"

    def blk(Mx, m, l3, l1):
        if m not in Mx:
            return torch.zeros((C, C), dtype=flat.dtype)
        return Mx[m][(l3 - m) * C:(l3 - m + 1) * C, (l1 - m) * C:(l1 - m + 1) * C]

    w = {}
    for l1 in range(L + 1):
        for l3 in range(L + 1):
            even, odd, Me, Mo = _systems(l1, l3)
            mn = min(l1, l3)
            Ae = torch.stack([blk(A, m, l3, l1) for m in range(0, mn + 1)])
            we = torch.einsum("em,mab->eab", torch.from_numpy(np.linalg.inv(Me)), Ae)
            for e, l2 in enumerate(even):
                w[(l1, l2, l3)] = we[e]
            if mn >= 1:
                Bo = torch.stack([blk(B, m, l3, l1) for m in range(1, mn + 1)])
                wo = torch.einsum("om,mab->oab", torch.from_numpy(np.linalg.inv(Mo)), Bo)
                for o_, l2 in enumerate(odd):
                    w[(l1, l2, l3)] = wo[o_]
    return w


def layer_t(L, C, H, n_rbf, cutoff, pos, box, row_ptr, col, x, Wq, Wk, Wrad, Wso2, M=None):
    """out[N, (L+1)^2, C] of the layer, as a differentiable function of the tensors."""
    N = x.shape[0]
    row_ptr = np.asarray(row_ptr, np.int64)
    col = np.asarray(col, np.int64)
    deg = np.diff(row_ptr)
    ii = torch.from_numpy(np.repeat(np.arange(N), deg))
    jj = torch.from_numpy(col)
    E = jj.numel()
    K = (L + 1) ** 2
    dh = C // H
    # geometry
    r = pos[jj] - pos[ii]
    if box is not None:
        b = torch.tensor([float(v) for v in box], dtype=torch.float64)
        r = r - b * torch.round((r / b).detach())
    d = torch.linalg.norm(r, dim=1)
    # radial basis and gates
    mu = torch.arange(n_rbf, dtype=torch.float64) * (cutoff / (n_rbf - 1))
    delta = cutoff / (n_rbf - 1)
    u = 0.5 * (torch.cos(pi * d / cutoff) + 1.0)
    rho = u[:, None] * torch.exp(-(((d[:, None] - mu[None, :]) / delta) ** 2))
    g = rho @ Wrad
    g_v = g[:, :(L + 1) * C].reshape(E, L + 1, C)
    g_a = g[:, (L + 1) * C:]
    lk = torch.from_numpy(np.concatenate([np.full(2 * l + 1, l) for l in range(L + 1)]))
    h = g_v[:, lk, :] * x[jj]
    # dense messages
    Y = real_sh_t(2 * L, r)
    w = paths_from_so2_t(Wso2, L, C, M)
    blocks = [torch.zeros((E, 2 * l + 1, C), dtype=torch.float64) for l in range(L + 1)]
    for (l1, l2, l3), W in w.items():
        Q = torch.from_numpy(np.array(real_cg(l1, l2, l3)))
        t = torch.einsum("abc,eai,eb->eci", Q, h[:, l1 * l1:(l1 + 1) ** 2, :], Y[:, l2 * l2:(l2 + 1) ** 2])
        blocks[l3] = blocks[l3] + t @ W.T
    v = torch.cat(blocks, dim=1)
    # logits and the softmax over each node's neighbours (max pass, then sum pass)
    q = x[:, 0, :] @ Wq.T
    k = x[:, 0, :] @ Wk.T
    dots = (q[ii].reshape(E, H, dh) * k[jj].reshape(E, H, dh)).sum(-1)
    a = g_a * dots / sqrt(dh)
    amax = torch.full((N, H), -torch.inf, dtype=torch.float64)
    amax = amax.scatter_reduce(0, ii[:, None].expand(E, H), a.detach(), reduce="amax")
    ex = torch.exp(a - amax[ii])
    s = torch.zeros((N, H), dtype=torch.float64).index_add(0, ii, ex)
    alpha = ex / s[ii]
    wgt = alpha.repeat_interleave(dh, dim=1)  # [E, C]
    return torch.zeros((N, K, C), dtype=torch.float64).index_add(0, ii, wgt[:, None, :] * v)


def layer_grads(L, C, H, n_rbf, cutoff, pos, box, row_ptr, col, x, Wq, Wk, Wrad, Wso2, G, M=None):
    """(out, grads) with grads = d sum(G * out) / d (pos, x, Wq, Wk, Wrad, Wso2), all fp64 numpy."""
    leaves = [torch.tensor(np.asarray(a, np.float64), requires_grad=True) for a in (pos, x, Wq, Wk, Wrad, Wso2)]
    out = layer_t(L, C, H, n_rbf, cutoff, *leaves[:1], box, row_ptr, col, *leaves[1:], M=M)
    loss = (out * torch.from_numpy(np.asarray(G, np.float64))).sum()
    grads = torch.autograd.grad(loss, leaves, allow_unused=True)
    names = ("pos", "x", "Wq", "Wk", "Wrad", "Wso2")
    res = {}
    for nm, lf, gr in zip(names, leaves, grads):
        res[nm] = np.zeros(lf.shape) if gr is None else gr.numpy()
    return out.detach().numpy(), res
