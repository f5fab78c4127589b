"""The edge-materialising PyTorch baseline computes the same layer: checked
against the fp64 oracle directly, and against this library, before it is used
as a measurement baseline."""
import os
import sys

import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
from gpu_util import TOL, DeviceInputs, oracle_csr, rel_err_per_degree

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from naive_baseline import naive_attention  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg_id", [1, 3])
def test_naive_baseline_matches_library(cfg_id):
    d = DeviceInputs(cfg_id)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    ours = e2f.e2f_onfly_attention(cfg, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    naive = naive_attention(cfg, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    err = rel_err_per_degree(naive.cpu().numpy(), ours.cpu().numpy(), w.L)
    assert err <= TOL[w.dtype], err


@pytest.mark.parametrize("cfg_id,n_sample", [(1, None), (3, 48)])
def test_naive_baseline_matches_the_oracle(cfg_id, n_sample):
    d = DeviceInputs(cfg_id)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    naive = naive_attention(cfg, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2).cpu().numpy()
    rp0, col0 = oracle_csr(cfg_id)
    nodes = (np.arange(w.n_atoms) if n_sample is None
             else np.sort(np.random.default_rng(30 + cfg_id).choice(w.n_atoms, n_sample, replace=False)))
    ref = d.oracle()(w.pos, w.box, rp0, col0, d.x_f64, nodes=nodes)
    err = rel_err_per_degree(naive[nodes].astype(np.float64), ref, w.L)
    assert err <= TOL[w.dtype], err
