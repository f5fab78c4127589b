"""The edge-materialising PyTorch baseline computes the same layer: checked
against this library (whose output is checked against the oracle) before it
is used as a measurement baseline."""
import os
import sys

import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
from gpu_util import TOL, DeviceInputs, rel_err_per_degree

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
