"""Parity of the Wigner-6j node-level convolution (e2f_sixj_attention)
against the fp64 edge-form oracle (oracle/sixj.py), on the tiny open cube,
on batches of molecule graphs (up to the full 256-graph batch, sampled),
and on the degenerate cases: isolated atoms, one-atom graphs, no atoms."""
import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
import workloads as W
from gpu_util import dev, rel_err_per_degree
from oracle.sixj import SixjLayer, sixj_paths

pytestmark = pytest.mark.gpu

# fp32 inputs, logits and output; fp64 node sums (the expansion's
# cancellation stays within fp64): the error is fp32 rounding of the
# softmax and of the output, about 1e-7 normwise per degree
TOL = 1e-5


def _run(pos, graph_ptr, cutoff, L, Lf, C, H, n_rbf=16, nodes=None, seed=0):
    d = dev()
    n = pos.shape[0]
    P = len(sixj_paths(L, Lf))
    assert e2f.e2f_sixj_n_paths(L, Lf) == P
    x, x64 = W.make_features(100 + seed, n, L, C, "f32")
    Wq, Wk, Wrad, wp = W.make_sixj_weights(seed, C, H, n_rbf, P)
    pos_t = torch.from_numpy(np.ascontiguousarray(pos, np.float32)).to(d)
    gp = None if graph_ptr is None else torch.from_numpy(np.asarray(graph_ptr, np.int32)).to(d)
    rp, col = e2f.e2f_build_neighbors(pos_t, None, cutoff, gp)
    cfg = e2f.make_sixj_cfg(L, Lf, C, H, n_rbf, cutoff)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(d)
    out = e2f.e2f_sixj_attention(cfg, pos_t, rp, col, t(x).reshape(n, (L + 1) ** 2, C), t(Wq), t(Wk), t(Wrad),
                                 t(wp), graph_ptr=gp)
    torch.cuda.synchronize()
    lay = SixjLayer(L, Lf, C, H, n_rbf, cutoff, Wq, Wk, Wrad, wp)
    nodes = np.arange(n) if nodes is None else nodes
    ref = lay(pos, rp.cpu().numpy(), col.cpu().numpy(), x64.reshape(n, (L + 1) ** 2, C), nodes=nodes)
    return out.cpu().numpy()[nodes].astype(np.float64), ref, rp.cpu().numpy()


@pytest.mark.parametrize("L,Lf,H", [(2, 4, 1), (2, 2, 4), (1, 2, 2), (0, 0, 1)])
def test_sixj_tiny_cube_all_nodes(L, Lf, H):
    w = W.load_workload(1)
    got, ref, _ = _run(w.pos, None, w.cutoff, L, Lf, 16, H)
    assert rel_err_per_degree(got, ref, L) <= TOL


@pytest.mark.parametrize("L,Lf,C,H", [(4, 4, 32, 8), (4, 8, 16, 4), (3, 6, 48, 6)])
def test_sixj_molecule_graphs_all_nodes(L, Lf, C, H):
    w = W.load_workload(2)
    g = 8
    pos, gp = w.pos[:w.graph_ptr[g]], w.graph_ptr[:g + 1]
    got, ref, _ = _run(pos, gp, w.cutoff, L, Lf, C, H, seed=1)
    assert rel_err_per_degree(got, ref, L) <= TOL


def test_sixj_full_molecule_batch_sampled():
    # all 256 graphs (about 10,200 atoms), C = 64, H = 8 as the batch's main
    # layer; 96 nodes spread over the atom range are checked one by one
    w = W.load_workload(2)
    nodes = np.linspace(0, w.n_atoms - 1, 96).astype(np.int64)
    got, ref, _ = _run(w.pos, w.graph_ptr, w.cutoff, 4, 4, 64, 8, nodes=nodes, seed=2)
    assert rel_err_per_degree(got, ref, 4) <= TOL


def test_sixj_isolated_atoms_and_one_atom_graphs():
    rng = np.random.default_rng(7)
    # graph 0: a cluster with one far atom; graph 1: one atom; graph 2: a pair
    a = rng.normal(0, 1.5, size=(12, 3))
    a[5] = [40.0, 0.0, 0.0]
    pos = np.concatenate([a, [[0.1, 0.2, 0.3]], [[0.0, 0.0, 0.0], [0.0, 0.0, 1.3]]])
    gp = np.array([0, 12, 13, 15])
    got, ref, rp = _run(pos, gp, 5.0, 3, 5, 16, 2, seed=3)
    for i in (5, 12):
        assert rp[i + 1] == rp[i] and np.abs(got[i]).max() == 0.0
    assert rel_err_per_degree(got, ref, 3) <= TOL


def test_sixj_empty_and_unsupported():
    d = dev()
    cfg = e2f.make_sixj_cfg(2, 4, 16, 1, 16, 5.0)
    z = torch.zeros(0, dtype=torch.float32, device=d)
    rp = torch.zeros(1, dtype=torch.int32, device=d)
    col = torch.zeros(0, dtype=torch.int32, device=d)
    out = e2f.e2f_sixj_attention(cfg, z.reshape(0, 3), rp, col, z.reshape(0, 9, 16), z, z, z, z)
    assert out.shape == (0, 9, 16)
    with pytest.raises(e2f.E2FError):
        e2f.e2f_sixj_attention(e2f.make_sixj_cfg(2, 5, 16, 1, 16, 5.0), z.reshape(0, 3), rp, col,
                               z.reshape(0, 9, 16), z, z, z, z)
