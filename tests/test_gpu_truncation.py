"""SO(2) truncation (m_max < L): the maps act on |m| <= m_max only. It is
the full layer with the blocks A(m), B(m), m > m_max, set to zero, so the
oracle checks it with zero-padded weights; the truncated call must also
equal, bit for bit, the full call on those zero-padded weights."""
import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
from gpu_util import TOL, DeviceInputs, oracle_csr, rel_err_per_degree, to_dev_storage
from oracle.layer import DenseLayer
from workloads import so2_block_sizes

pytestmark = pytest.mark.gpu


def truncated(flat, L, C, M):
    n = sum(so2_block_sizes(L, C)[:2 * M + 1])  # A0, then (A_m, B_m) for m <= M
    return flat[:n]


def zero_padded(flat_f64, L, C, M):
    n = sum(so2_block_sizes(L, C)[:2 * M + 1])
    out = np.zeros(sum(so2_block_sizes(L, C)))
    out[:n] = flat_f64[:n]
    return out


@pytest.mark.parametrize("cfg_id,M,n_sample", [(3, 0, 24), (3, 2, 24), (1, 0, None), (1, 1, None)])
def test_truncated_layer(cfg_id, M, n_sample):
    d = DeviceInputs(cfg_id)
    w, wt = d.w, d.weights
    assert M < w.L
    cfg_t = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype, m_max=M)
    cfg_f = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    W_t = to_dev_storage(truncated(wt.Wso2, w.L, w.C, M), w.dtype)
    # zero-padded full weights in storage form: the same stored values, zeros after the truncation point
    pad = np.zeros_like(wt.Wso2)
    pad[:W_t.numel()] = wt.Wso2[:W_t.numel()]
    W_p = to_dev_storage(pad, w.dtype)
    out_t = e2f.e2f_onfly_attention(cfg_t, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, W_t)
    out_f = e2f.e2f_onfly_attention(cfg_f, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, W_p)
    assert torch.equal(out_t, out_f)
    rp0, col0 = oracle_csr(cfg_id)
    layer = DenseLayer(w.L, w.C, w.H, w.n_rbf, w.cutoff, wt.Wq, wt.Wk, wt.Wrad,
                       zero_padded(wt.Wso2_f64, w.L, w.C, M))
    nodes = None
    if n_sample is not None:
        nodes = np.random.default_rng(7).choice(w.n_atoms, n_sample, replace=False)
    ref = layer(w.pos, w.box, rp0, col0, d.x_f64, nodes=nodes)
    got = out_t.cpu().numpy().astype(np.float64)
    if nodes is not None:
        got = got[nodes]
    assert rel_err_per_degree(got, ref, w.L) <= TOL[w.dtype]


def test_truncation_at_or_above_L_is_the_full_layer():
    d = DeviceInputs(1)
    w = d.w
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    outs = [e2f.e2f_onfly_attention(e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype, m_max=m),
                                    d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2) for m in (-1, w.L, 9)]
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
