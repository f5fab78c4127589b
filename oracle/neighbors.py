"""Neighbour lists from the exact fp32 cutoff predicate (oracle; test
infrastructure).

The pages never describe how neighbours are found (they iterate over
"j in N(i)", gist.science Technical Summary 2.2). Reading taken: N(i) is every
j != i in the same graph whose minimum-image distance is inside the cutoff,
decided in fp32 by this exact sequence of IEEE round-to-nearest operations
(no fused multiply-add):

    dx  = x_j - x_i                          (per axis)
    if periodic:  dx = dx - box * rint(dx * inv_box),  inv_box = 1/box in fp32,
                  rint rounding half to even
    d2  = (dx*dx + dy*dy) + dz*dz
    keep  d2 < rc*rc                          (rc*rc rounded to fp32)

numpy float32 arithmetic rounds every operation separately, so writing the
sequence out in numpy gives the reference bits. Rows are in the caller's atom
order and columns ascend. Periodic boxes need rc <= box/2, so each pair has
one image.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32


def predicate_f32(pi: np.ndarray, pj: np.ndarray, box, cutoff: float) -> np.ndarray:
    """Boolean mask for pairs (broadcast over leading axes); pi, pj float32 [...,3]."""
    dx = (pj - pi).astype(F32)
    if box is not None:
        b = np.asarray(box, dtype=F32)
        inv = (F32(1.0) / b).astype(F32)
        dx = (dx - b * np.rint(dx * inv)).astype(F32)
    d2 = (dx[..., 0] * dx[..., 0] + dx[..., 1] * dx[..., 1]) + dx[..., 2] * dx[..., 2]
    rc2 = F32(cutoff) * F32(cutoff)
    return d2 < rc2


def _graph_of(n, graph_ptr):
    if graph_ptr is None:
        return np.zeros(n, np.int64), np.array([0, n])
    gp = np.asarray(graph_ptr, np.int64)
    return np.repeat(np.arange(gp.size - 1), np.diff(gp)), gp


def to_csr(n, rows, cols):
    order = np.lexsort((cols, rows))
    rows, cols = rows[order], cols[order]
    row_ptr = np.zeros(n + 1, np.int64)
    np.add.at(row_ptr, rows + 1, 1)
    return np.cumsum(row_ptr).astype(np.int32), cols.astype(np.int32)


def neighbors_bruteforce(pos, box, cutoff, graph_ptr=None, chunk=512):
    """O(N^2) within each graph: (row_ptr int32 [N+1], col int32 [E])."""
    pos = np.asarray(pos, dtype=F32)
    n = pos.shape[0]
    _, gp = _graph_of(n, graph_ptr)
    rows, cols = [], []
    for g in range(gp.size - 1):
        a, b = int(gp[g]), int(gp[g + 1])
        for s in range(a, b, chunk):
            e = min(b, s + chunk)
            m = predicate_f32(pos[s:e, None, :], pos[None, a:b, :], box, cutoff)
            ii = np.arange(s, e)[:, None]
            jj = np.arange(a, b)[None, :]
            m &= ii != jj
            r, c = np.nonzero(m)
            rows.append(r + s)
            cols.append(c + a)
    rows = np.concatenate(rows) if rows else np.zeros(0, np.int64)
    cols = np.concatenate(cols) if cols else np.zeros(0, np.int64)
    return to_csr(n, rows, cols)


def neighbors_kdtree(pos, box, cutoff, graph_ptr=None, margin=1e-3):
    """KD-tree superset at cutoff + margin, then the exact fp32 predicate."""
    from scipy.spatial import cKDTree

    pos = np.asarray(pos, dtype=F32)
    n = pos.shape[0]
    gid, _ = _graph_of(n, graph_ptr)
    p64 = pos.astype(np.float64)
    if box is not None:
        b = np.asarray(box, np.float64)
        tree = cKDTree(np.mod(p64, b) % b, boxsize=b)
    else:
        tree = cKDTree(p64)
    pr = tree.query_pairs(cutoff + margin, output_type="ndarray")
    i = np.concatenate([pr[:, 0], pr[:, 1]])
    j = np.concatenate([pr[:, 1], pr[:, 0]])
    keep = (gid[i] == gid[j]) & predicate_f32(pos[i], pos[j], box, cutoff)
    return to_csr(n, i[keep], j[keep])
