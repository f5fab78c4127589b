"""Edge-materialising GPU baseline of the on-the-fly equivariant attention
forward (E2Former-V2, gist.science Technical Summary 2.1-2.2), in plain
PyTorch on the GPU.

It computes the same layer as e2f_onfly_attention, the way an
edge-centric implementation does: every per-edge tensor is materialised in
HBM (the gathered neighbour features x_j, the rotated and gated features,
the SO(2) outputs and the rotated-back messages, each E x (L+1)^2 x C in
fp32), the softmax goes through scatter reductions over E x H logits, and
the messages are summed with index_add. The pages contrast the node-centric
kernel with exactly this kind of implementation (TFLOPS and activation
memory); bench.py --impl naive measures it on the same B200 for context.

Only the per-edge Wigner blocks come from the library
(e2f_edge_wigner_blocks); everything else is torch ops. It is a measurement
baseline, not a product path: nothing in the package imports it.
"""
from __future__ import annotations

import math

import torch

import atomistic_cell_list_b200 as e2f


def so2_blocks(Wso2: torch.Tensor, L: int, C: int):
    """Views of the packed SO(2) weights: A0, then (A_m, B_m) for m = 1..L."""
    w = Wso2.float().reshape(-1)
    o = 0
    n0 = (L + 1) * C
    A0 = w[o:o + n0 * n0].view(n0, n0)
    o += n0 * n0
    blocks = []
    for m in range(1, L + 1):
        nm = (L + 1 - m) * C
        A = w[o:o + nm * nm].view(nm, nm)
        o += nm * nm
        B = w[o:o + nm * nm].view(nm, nm)
        o += nm * nm
        blocks.append((A, B))
    return A0, blocks


def naive_attention(cfg, pos, box, row_ptr, col, x, Wq, Wk, Wrad, Wso2):
    """out[N, (L+1)^2, C] fp32, computed with edge-sized tensors."""
    L, C, H, n_rbf, rc = cfg.L, cfg.C, cfg.H, cfg.n_rbf, float(cfg.cutoff)
    N, K, dh = pos.shape[0], (L + 1) ** 2, C // H
    dev = pos.device
    deg = (row_ptr[1:] - row_ptr[:-1]).long()
    i = torch.repeat_interleave(torch.arange(N, device=dev), deg)
    j = col.long()
    E = j.numel()
    # geometry (fp32, minimum image)
    r = pos[j] - pos[i]
    if box is not None:
        b = torch.tensor(box, dtype=torch.float32, device=dev)
        r = r - b * torch.round(r * (1.0 / b))
    d = torch.sqrt((r * r).sum(1))
    D = e2f.e2f_edge_wigner_blocks(r.contiguous(), L)  # [E, sum (2l+1)^2]
    Dl = []
    off = 0
    for l in range(L + 1):
        w_ = 2 * l + 1
        Dl.append(D[:, off:off + w_ * w_].view(E, w_, w_))
        off += w_ * w_
    # radial basis and gates
    mu = torch.arange(n_rbf, device=dev, dtype=torch.float32) * (rc / (n_rbf - 1))
    delta = rc / (n_rbf - 1)
    u = 0.5 * (torch.cos(math.pi * d / rc) + 1.0)
    rho = u[:, None] * torch.exp(-(((d[:, None] - mu[None, :]) / delta) ** 2))
    g = rho @ Wrad
    gv = g[:, :(L + 1) * C].view(E, L + 1, C)
    ga = g[:, (L + 1) * C:]
    # gathered, gated, rotated neighbour features (E x K x C)
    xj = x[j].float()
    xt = torch.empty_like(xj)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) * (l + 1))
        xt[:, sl, :] = torch.bmm(Dl[l], xj[:, sl, :] * gv[:, l:l + 1, :])
    del xj
    # SO(2) maps per |m| (Eq. 13 form): o+ = A h+ - B h-, o- = B h+ + A h-
    A0, blocks = so2_blocks(Wso2, L, C)
    o = torch.zeros_like(xt)
    rows0 = [l * l + l for l in range(L + 1)]
    h0 = xt[:, rows0, :].reshape(E, -1)
    o[:, rows0, :] = (h0 @ A0.T).view(E, L + 1, C)
    for m in range(1, L + 1):
        A, B = blocks[m - 1]
        rp = [l * l + l + m for l in range(m, L + 1)]
        rm = [l * l + l - m for l in range(m, L + 1)]
        hp = xt[:, rp, :].reshape(E, -1)
        hm = xt[:, rm, :].reshape(E, -1)
        o[:, rp, :] = (hp @ A.T - hm @ B.T).view(E, L + 1 - m, C)
        o[:, rm, :] = (hp @ B.T + hm @ A.T).view(E, L + 1 - m, C)
    del xt
    # rotate back: v = D^T o
    v = torch.empty_like(o)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) * (l + 1))
        v[:, sl, :] = torch.bmm(Dl[l].transpose(1, 2), o[:, sl, :])
    del o
    # logits and softmax over each node's edges, per head
    x0 = x[:, 0, :].float()
    q = x0 @ Wq.T
    k = x0 @ Wk.T
    a = ga * (q[i].view(E, H, dh) * k[j].view(E, H, dh)).sum(-1) / math.sqrt(dh)
    amax = torch.full((N, H), -float("inf"), device=dev).scatter_reduce(0, i[:, None].expand(E, H), a, "amax")
    p = torch.exp(a - amax[i])
    s = torch.zeros((N, H), device=dev).index_add_(0, i, p)
    alpha = p / s[i]
    # weighted sum of messages
    out = torch.zeros((N, K, C), device=dev)
    out.index_add_(0, i, v * alpha.repeat_interleave(dh, dim=1)[:, None, :])
    return out
