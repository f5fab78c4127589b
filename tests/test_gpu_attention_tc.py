"""Tensor-core (tcgen05) attention against the fp64 oracle on every node of
small systems: several 128-edge tiles per CTA (grid capped through
e2f_attention_set_debug), nodes straddling tiles, ragged tails, isolated atoms, and
the supported shapes (L = 1..4, C = 64, 128 or 256, H = 4..16)."""
import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
import workloads as W
from gpu_util import dev, rel_err_per_degree, to_dev_storage
from oracle.layer import DenseLayer
from oracle.neighbors import neighbors_bruteforce

pytestmark = pytest.mark.gpu


def random_system(seed, n, side, dmin, n_far=0):
    rng = np.random.default_rng(seed)
    pts = []
    while len(pts) < n:
        p = rng.uniform(0, side, 3)
        if pts:
            d = np.array(pts) - p
            d -= side * np.round(d / side)
            if (np.einsum("ij,ij->i", d, d) < dmin * dmin).any():
                continue
        pts.append(p)
    return np.array(pts, np.float32)


def run_case(seed, n, side, cutoff, L, C, H, max_ctas, rel_tol=2e-2, isolate=0):
    pos = random_system(seed, n, side, 0.9)
    box = np.full(3, side, np.float32)
    if isolate:  # open boundaries with a few far-away atoms
        box = None
        far = np.array([[1000.0 + 50 * k, -500.0, 0.0] for k in range(isolate)], np.float32)
        pos = np.concatenate([pos, far])
    n = pos.shape[0]
    x_st, x_f = W.round_to_dtype(np.random.default_rng(seed + 1).normal(size=(n, (L + 1) ** 2, C)), "bf16")
    wt = W.make_weights(9, L, C, H, 16, "bf16", seed_offset=seed)
    cfg = e2f.make_cfg(L, C, H, 16, cutoff, "bf16")
    assert e2f.e2f_attention_uses_tensor_cores(cfg)
    d = dev()
    pos_d = torch.from_numpy(pos).to(d)
    blist = None if box is None else box.tolist()
    rp, col = e2f.e2f_build_neighbors(pos_d, blist, cutoff)
    e2f.e2f_attention_set_debug(max_ctas=max_ctas)
    try:
        out = e2f.e2f_onfly_attention(cfg, pos_d, blist, rp, col, to_dev_storage(x_st, "bf16").reshape(n, -1, C),
                                      torch.from_numpy(wt.Wq).to(d), torch.from_numpy(wt.Wk).to(d),
                                      torch.from_numpy(wt.Wrad).to(d), to_dev_storage(wt.Wso2, "bf16"))
    finally:
        e2f.e2f_attention_set_debug()
    out = out.cpu().numpy().astype(np.float64)
    rp0, col0 = neighbors_bruteforce(pos, box, cutoff)
    np.testing.assert_array_equal(rp.cpu().numpy(), rp0)
    ref = DenseLayer(L, C, H, 16, cutoff, wt.Wq, wt.Wk, wt.Wrad, wt.Wso2_f64)(pos, box, rp0, col0, x_f)
    err = rel_err_per_degree(out, ref, L)
    assert np.isfinite(out).all()
    assert err <= rel_tol, err
    if isolate:
        assert np.all(out[-isolate:] == 0)
    return err, int(col0.size)


@pytest.mark.parametrize("L,C,H,max_ctas", [(4, 128, 8, 2), (4, 128, 8, 148), (3, 128, 4, 3), (2, 256, 16, 2),
                                            (1, 128, 8, 1), (4, 64, 8, 2), (3, 64, 4, 3), (2, 64, 8, 1),
                                            (1, 64, 8, 148)])
def test_tc_matches_oracle_every_node(L, C, H, max_ctas):
    err, E = run_case(10 + L, 90, 9.6, 4.6, L, C, H, max_ctas)
    assert E > 3 * 128


def test_tc_open_boundaries_with_isolated_atoms():
    run_case(21, 70, 8.0, 4.0, 2, 128, 8, 2, isolate=3)


def test_tc_repeat_runs_are_bitwise_identical():
    d = dev()
    from gpu_util import DeviceInputs
    di = DeviceInputs(3)
    w = di.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    assert e2f.e2f_attention_uses_tensor_cores(cfg)
    rp, col = e2f.e2f_build_neighbors(di.pos, di.box, w.cutoff)
    outs = [e2f.e2f_onfly_attention(cfg, di.pos, di.box, rp, col, di.x, di.Wq, di.Wk, di.Wrad, di.Wso2).cpu()
            for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
