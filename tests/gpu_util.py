"""Helpers for the GPU parity tests: move seeded workloads to the device,
compute oracle references, and the error metric the tolerances use."""
from __future__ import annotations

import functools

import numpy as np
import torch

import workloads as W
from oracle.layer import DenseLayer
from oracle.neighbors import neighbors_bruteforce, neighbors_kdtree

# max relative error, normwise per output degree: fp32 features 1e-4, bf16
# features with fp32 accumulation 2e-2
TOL = {"f32": 1e-4, "bf16": 2e-2}


def dev():
    return torch.device("cuda:0")


def rel_err_per_degree(gpu: np.ndarray, ref: np.ndarray, L: int) -> float:
    """max over l of ||gpu - ref||_inf / ||ref||_inf on the degree-l block."""
    worst = 0.0
    for l in range(L + 1):
        s = slice(l * l, (l + 1) ** 2)
        den = np.abs(ref[:, s, :]).max()
        if den == 0:
            worst = max(worst, float(np.abs(gpu[:, s, :]).max()))
            continue
        worst = max(worst, float(np.abs(gpu[:, s, :] - ref[:, s, :]).max() / den))
    return worst


@functools.lru_cache(maxsize=None)
def oracle_csr(cfg_id: int):
    w = W.load_workload(cfg_id)
    if w.n_atoms <= 12000:
        return neighbors_bruteforce(w.pos, w.box, w.cutoff, w.graph_ptr)
    return neighbors_kdtree(w.pos, w.box, w.cutoff, w.graph_ptr)


class DeviceInputs:
    def __init__(self, cfg_id: int, seed_offset: int = 0):
        w = W.load_workload(cfg_id)
        self.w = w
        d = dev()
        self.pos = torch.from_numpy(w.pos).to(d)
        self.box = None if w.box is None else [float(v) for v in w.box]
        self.graph_ptr = None if w.graph_ptr is None else torch.from_numpy(w.graph_ptr).to(d)
        xs, self.x_f64 = W.make_features(cfg_id, w.n_atoms, w.L, w.C, w.dtype, seed_offset)
        wt = W.make_weights(cfg_id, w.L, w.C, w.H, w.n_rbf, w.dtype, seed_offset)
        self.weights = wt
        self.x = to_dev_storage(xs, w.dtype).reshape(w.n_atoms, w.K, w.C)
        self.Wq = torch.from_numpy(wt.Wq).to(d)
        self.Wk = torch.from_numpy(wt.Wk).to(d)
        self.Wrad = torch.from_numpy(wt.Wrad).to(d)
        self.Wso2 = to_dev_storage(wt.Wso2, w.dtype)

    def oracle(self):
        w, wt = self.w, self.weights
        return DenseLayer(w.L, w.C, w.H, w.n_rbf, w.cutoff, wt.Wq, wt.Wk, wt.Wrad, wt.Wso2_f64)


def to_dev_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        t = torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
    return t.to(dev())
