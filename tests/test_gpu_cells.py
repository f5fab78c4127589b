"""Attention with the cell-list traversal fused in (no neighbour list in
memory): the same layer as the CSR call on the same neighbour sets, checked
against the CSR call, the oracle, and itself (repeatability)."""
import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
import workloads as W
from gpu_util import TOL, DeviceInputs, oracle_csr, rel_err_per_degree
from oracle.layer import DenseLayer

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


def test_fused_traversal_open_boundaries_matches_the_oracle():
    # the open mode has its own enumeration (hashed buckets): compare it with the oracle
    # directly, on random nodes and on the nodes nearest the faces of the cloud
    from oracle.neighbors import neighbors_bruteforce
    d = DeviceInputs(3)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    fused = e2f.e2f_onfly_attention_cells(cfg, d.pos, None, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)
    rp0, col0 = neighbors_bruteforce(w.pos, None, w.cutoff)
    p = w.pos.astype(np.float64)
    face = np.minimum(p - p.min(axis=0), p.max(axis=0) - p).min(axis=1)
    nodes = np.unique(np.concatenate([np.random.default_rng(12).choice(w.n_atoms, 24, replace=False),
                                      np.argsort(face)[:12]]))
    ref = d.oracle()(w.pos, None, rp0, col0, d.x_f64, nodes=nodes)
    assert rel_err_per_degree(fused.cpu().numpy()[nodes].astype(np.float64), ref, w.L) <= TOL[w.dtype]


def test_fused_traversal_dense_open_matches_the_oracle():
    # about 300-570 neighbours per atom without a box: several tiles and statistics windows
    # per node in the open mode, checked against the oracle on sampled nodes
    from oracle.neighbors import neighbors_bruteforce
    d = DeviceInputs(3)
    w = d.w
    n, side, rc = 4000, 17.0, 5.5
    pos = np.random.default_rng(6).uniform(0.0, side, (n, 3)).astype(np.float32)
    reps = -(-n // w.n_atoms)
    x = d.x.repeat(reps, 1, 1)[:n].contiguous()
    x_f64 = np.concatenate([d.x_f64] * reps)[:n]
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, rc, w.dtype)
    fused = e2f.e2f_onfly_attention_cells(cfg, torch.from_numpy(pos).to(d.pos.device), None, x, d.Wq, d.Wk,
                                          d.Wrad, d.Wso2)
    rp0, col0 = neighbors_bruteforce(pos, None, rc)
    deg = np.diff(rp0)
    assert deg.max() > 512
    nodes = np.unique(np.concatenate([np.random.default_rng(13).choice(n, 6, replace=False),
                                      np.argsort(-deg, kind="stable")[:3], np.argsort(deg, kind="stable")[:3]]))
    wt = d.weights  # the oracle layer with this case's cutoff (radial basis and envelope)
    ref = DenseLayer(w.L, w.C, w.H, w.n_rbf, rc, wt.Wq, wt.Wk, wt.Wrad, wt.Wso2_f64)(pos, None, rp0, col0, x_f64,
                                                                                    nodes=nodes)
    assert rel_err_per_degree(fused.cpu().numpy()[nodes].astype(np.float64), ref, w.L) <= TOL[w.dtype]


# ---- Verlet-skin reuse of the cell lists across MD steps ---------------------

SKIN = 1.0


def _skin_setup(periodic=True):
    d = DeviceInputs(3)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    box = d.box if periodic else None
    ws = torch.empty(e2f.e2f_attention_cells_skin_workspace_size(w.n_atoms, box, cfg, SKIN), dtype=torch.uint8,
                     device=d.pos.device)
    return d, cfg, box, ws


def _skin_call(d, cfg, box, ws, pos, rebuild):
    return e2f.e2f_onfly_attention_cells_skin(cfg, pos, box, SKIN, rebuild, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2, ws)


def _csr_call(d, cfg, box, pos):
    rp, col = e2f.e2f_build_neighbors(pos, box, d.w.cutoff)
    return e2f.e2f_onfly_attention(cfg, pos, box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2)


def _moved(pos, box, rng, radius):
    # every atom moved by at most `radius` (uniform direction and length),
    # wrapped back into the periodic box so that reuse must use the minimum image
    n = pos.shape[0]
    u = rng.normal(size=(n, 3))
    u *= (radius * rng.uniform(0.0, 1.0, (n, 1))) / np.linalg.norm(u, axis=1, keepdims=True)
    p = pos.cpu().numpy().astype(np.float64) + u
    if box is not None:
        p = np.mod(p, np.asarray(box, np.float64))
    return torch.from_numpy(p.astype(np.float32)).to(pos.device)


@pytest.mark.parametrize("periodic", [True, False])
def test_skin_rebuild_and_reuse_match_the_csr_call(periodic):
    d, cfg, box, ws = _skin_setup(periodic)
    out0 = _skin_call(d, cfg, box, ws, d.pos, True)
    assert rel_err_per_degree(out0.cpu().numpy(), _csr_call(d, cfg, box, d.pos).cpu().numpy(), d.w.L) <= 1e-3
    rng = np.random.default_rng(21)
    pos1 = _moved(d.pos, box, rng, 0.49 * SKIN)
    out1 = _skin_call(d, cfg, box, ws, pos1, False)
    ref1 = _csr_call(d, cfg, box, pos1)
    assert rel_err_per_degree(out1.cpu().numpy(), ref1.cpu().numpy(), d.w.L) <= 1e-3
    # the neighbour sets changed: the layer's output moved by far more than the tolerance
    assert rel_err_per_degree(out0.cpu().numpy(), ref1.cpu().numpy(), d.w.L) > 1e-2


def test_skin_reuse_matches_the_oracle_at_moved_positions():
    # the oracle's own neighbour list and dense layer at the moved positions
    from oracle.neighbors import neighbors_bruteforce
    d, cfg, box, ws = _skin_setup()
    w = d.w
    _skin_call(d, cfg, box, ws, d.pos, True)
    pos1 = _moved(d.pos, box, np.random.default_rng(33), 0.45 * SKIN)
    out = _skin_call(d, cfg, box, ws, pos1, False)
    p1 = pos1.cpu().numpy()
    rp0, col0 = neighbors_bruteforce(p1, w.box, w.cutoff)
    nodes = np.random.default_rng(12).choice(w.n_atoms, 24, replace=False)
    ref = d.oracle()(p1, w.box, rp0, col0, d.x_f64, nodes=nodes)
    assert rel_err_per_degree(out.cpu().numpy()[nodes].astype(np.float64), ref, w.L) <= TOL[w.dtype]


def test_skin_reuse_is_repeatable_and_equals_a_second_reuse():
    d, cfg, box, ws = _skin_setup()
    _skin_call(d, cfg, box, ws, d.pos, True)
    pos1 = _moved(d.pos, box, np.random.default_rng(3), 0.3 * SKIN)
    a = _skin_call(d, cfg, box, ws, pos1, False)
    b = _skin_call(d, cfg, box, ws, pos1, False)
    assert torch.equal(a, b)


def test_skin_reuse_flags_a_stale_list_and_recovers():
    d, cfg, box, ws = _skin_setup()
    _skin_call(d, cfg, box, ws, d.pos, True)
    pos1 = d.pos.clone()
    pos1[17, 0] += 0.51 * SKIN
    with pytest.raises(e2f.E2FError) as ei:
        _skin_call(d, cfg, box, ws, pos1, False)
    assert ei.value.code == 8
    out = _skin_call(d, cfg, box, ws, pos1, True)
    assert rel_err_per_degree(out.cpu().numpy(), _csr_call(d, cfg, box, pos1).cpu().numpy(), d.w.L) <= 1e-3


def test_skin_md_loop_rebuilds_only_when_needed():
    # a short trajectory: reuse while every atom stays within skin/2 of its
    # position at the last rebuild (checked on the host), else rebuild
    d, cfg, box, ws = _skin_setup()
    rng = np.random.default_rng(8)
    vel = rng.normal(size=(d.w.n_atoms, 3)) * 0.06
    p = d.pos.cpu().numpy().astype(np.float64)
    ref_pos = p.copy()
    L_box = np.asarray(box, np.float64)
    rebuilds = 0
    for step in range(6):
        if step:
            p = np.mod(p + vel, L_box)
        disp = p - ref_pos
        disp -= L_box * np.round(disp / L_box)
        rebuild = step == 0 or np.linalg.norm(disp, axis=1).max() > 0.5 * SKIN
        if rebuild:
            ref_pos = p.copy()
            rebuilds += 1
        pos = torch.from_numpy(p.astype(np.float32)).to(d.pos.device)
        out = _skin_call(d, cfg, box, ws, pos, rebuild)
        assert rel_err_per_degree(out.cpu().numpy(), _csr_call(d, cfg, box, pos).cpu().numpy(), d.w.L) <= 1e-3
    assert 1 < rebuilds < 6


def test_skin_reuse_rejects_a_changed_system():
    # the library records (n, box, cfg, skin) per workspace at each rebuild;
    # a reuse call with other values is refused before any launch
    d, cfg, box, ws = _skin_setup()
    _skin_call(d, cfg, box, ws, d.pos, True)
    bigger = [1.01 * float(v) for v in box]
    for args in [(d.pos, bigger), (d.pos[:-10].contiguous(), box)]:
        with pytest.raises(e2f.E2FError) as ei:
            e2f.e2f_onfly_attention_cells_skin(cfg, args[0], args[1], SKIN, False, d.x, d.Wq, d.Wk, d.Wrad,
                                               d.Wso2, ws)
        assert ei.value.code == 1
    # a workspace no rebuild was recorded for: 256 bytes into a new block (the
    # caching allocator's blocks start 512-byte aligned, so a recycled block
    # address recorded by an earlier rebuild cannot coincide with it)
    fresh = torch.empty(ws.numel() + 512, dtype=torch.uint8, device=ws.device)[256:256 + ws.numel()]
    assert fresh.data_ptr() % 512 == 256
    with pytest.raises(e2f.E2FError) as ei:
        _skin_call(d, cfg, box, fresh, d.pos, False)
    assert ei.value.code == 1
    _skin_call(d, cfg, box, ws, d.pos, False)          # the recorded system still reuses
