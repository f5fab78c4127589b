"""Attention with the cell-list traversal fused in (no neighbour list in
memory): the same layer as the CSR call on the same neighbour sets, checked
against the CSR call, the oracle, and itself (repeatability)."""
import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
import workloads as W
from gpu_util import TOL, DeviceInputs, oracle_csr, rel_err_per_degree

pytestmark = pytest.mark.gpu


def _both(cfg_id):
    d = DeviceInputs(cfg_id)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    csr = e2f.e2f_onfly_attention(cfg, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    fused = e2f.e2f_onfly_attention_cells(cfg, d.pos, d.box, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    return d, cfg, csr, fused


@pytest.mark.parametrize("cfg_id", [3, 4])
def test_fused_traversal_matches_the_csr_call(cfg_id):
    d, cfg, csr, fused = _both(cfg_id)
    # same edges and per-edge arithmetic; the edges of a node come in another order, so
    # the per-node sums (about 90 terms of both signs) round differently in fp32
    assert rel_err_per_degree(fused.cpu().numpy(), csr.cpu().numpy(), d.w.L) <= 1e-3


def test_fused_traversal_matches_the_oracle_and_repeats():
    d, cfg, csr, fused = _both(3)
    w = d.w
    nodes = np.random.default_rng(11).choice(w.n_atoms, 24, replace=False)
    rp0, col0 = oracle_csr(3)
    ref = d.oracle()(w.pos, w.box, rp0, col0, d.x_f64, nodes=nodes)
    assert rel_err_per_degree(fused.cpu().numpy()[nodes].astype(np.float64), ref, w.L) <= TOL[w.dtype]
    again = e2f.e2f_onfly_attention_cells(cfg, d.pos, d.box, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    assert torch.equal(again, fused)


def test_fused_traversal_scope():
    d = DeviceInputs(3)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    f32 = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, "f32")
    with pytest.raises(e2f.E2FError) as ei:
        e2f.e2f_onfly_attention_cells(f32, d.pos, d.box, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    assert ei.value.code == 2


def test_fused_traversal_dense_nodes():
    # about 570 neighbours per atom: more than a tile (128 edges) and more than the
    # statistics pass buffers per window (256), on a 3 x 3 x 3 cell grid
    d = DeviceInputs(3)
    w = d.w
    n, side, rc = 4000, 17.0, 5.5
    pos = torch.from_numpy(np.random.default_rng(5).uniform(0.0, side, (n, 3)).astype(np.float32)).to(d.pos.device)
    box = [side] * 3
    x = d.x.repeat(2, 1, 1)[:n].contiguous()
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, rc, w.dtype)
    rp, col = e2f.e2f_build_neighbors(pos, box, rc)
    deg = (rp[1:] - rp[:-1]).cpu().numpy()
    assert deg.min() > 256 and deg.max() > 512
    csr = e2f.e2f_onfly_attention(cfg, pos, box, rp, col, x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    fused = e2f.e2f_onfly_attention_cells(cfg, pos, box, x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    assert rel_err_per_degree(fused.cpu().numpy(), csr.cpu().numpy(), w.L) <= 1e-3


def test_fused_traversal_with_truncated_maps():
    # m_max < L: the fused call and the CSR call apply the same truncated layer
    d = DeviceInputs(3)
    w = d.w
    M = 2
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype, m_max=M)
    n_so2 = sum(W.so2_block_sizes(w.L, w.C)[:2 * M + 1])
    wso2 = d.Wso2[:n_so2].contiguous()
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff)
    csr = e2f.e2f_onfly_attention(cfg, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, wso2)
    fused = e2f.e2f_onfly_attention_cells(cfg, d.pos, d.box, d.x, d.Wq, d.Wk, d.Wrad, wso2)
    assert rel_err_per_degree(fused.cpu().numpy(), csr.cpu().numpy(), w.L) <= 1e-3


def test_fused_traversal_open_boundaries():
    # the same atoms without the periodic box: hashed cells, open-boundary predicate
    d = DeviceInputs(3)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(d.pos, None, w.cutoff)
    csr = e2f.e2f_onfly_attention(cfg, d.pos, None, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    fused = e2f.e2f_onfly_attention_cells(cfg, d.pos, None, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    assert rel_err_per_degree(fused.cpu().numpy(), csr.cpu().numpy(), w.L) <= 1e-3
    # atoms near the faces have fewer neighbours than in the periodic box
    assert col.numel() < e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff)[1].numel()
