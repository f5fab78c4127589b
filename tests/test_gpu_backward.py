"""Backward of the attention (e2f_onfly_attention_backward) against the
gradient oracle (PyTorch fp64 autograd of the dense layer, itself pinned by
finite differences), on small open and periodic systems, fp32 and bf16
storage, full and truncated SO(2) maps; and, at full size, properties that
hold at any size: forces sum to zero, and the position gradient agrees with a
central difference of the fp32 forward."""
import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
import workloads as W
from gpu_util import DeviceInputs, dev, to_dev_storage
from oracle.grad import layer_grads
from oracle.neighbors import neighbors_bruteforce

pytestmark = pytest.mark.gpu


def _positions(rng, n, side, min_sep, periodic):
    pos = np.zeros((0, 3))
    while pos.shape[0] < n:
        p = rng.uniform(0.0, side, 3)
        dv = pos - p
        if periodic:
            dv -= side * np.rint(dv / side)
        if pos.shape[0] == 0 or np.linalg.norm(dv, axis=1).min() >= min_sep:
            pos = np.vstack([pos, p])
    return pos.astype(np.float32)


def _system(seed, n, L, C, H, n_rbf, dtype, periodic, M=None):
    rng = np.random.default_rng(seed)
    side = 12.5 if periodic else 9.0
    cutoff = 6.0 if periodic else 5.0
    pos = _positions(rng, n, side, 1.0, periodic)
    box = [side] * 3 if periodic else None
    K = (L + 1) ** 2
    Mx = L if M is None else M
    n_so2 = sum(W.so2_block_sizes(L, C)[:2 * Mx + 1])
    xs, x64 = W.round_to_dtype(rng.normal(size=(n, K, C)), dtype)
    ws, w64 = W.round_to_dtype(rng.normal(size=n_so2) / np.sqrt(C), dtype)
    Wq = (rng.normal(size=(C, C)) / np.sqrt(C)).astype(np.float32)
    Wk = (rng.normal(size=(C, C)) / np.sqrt(C)).astype(np.float32)
    Wrad = (rng.normal(size=(n_rbf, (L + 1) * C + H)) / np.sqrt(C)).astype(np.float32)
    G = rng.normal(size=(n, K, C)).astype(np.float32)
    rp, col = neighbors_bruteforce(pos, box, cutoff)
    host = dict(pos=pos, box=box, rp=rp, col=col, x64=x64, w64=w64, Wq=Wq, Wk=Wk, Wrad=Wrad, G=G, cutoff=cutoff)
    d = dev()
    devt = dict(pos=torch.from_numpy(pos).to(d), rp=torch.from_numpy(rp.astype(np.int32)).to(d),
                col=torch.from_numpy(col.astype(np.int32)).to(d),
                x=to_dev_storage(xs, dtype).reshape(n, K, C), Wso2=to_dev_storage(ws, dtype),
                Wq=torch.from_numpy(Wq).to(d), Wk=torch.from_numpy(Wk).to(d), Wrad=torch.from_numpy(Wrad).to(d),
                G=torch.from_numpy(G).to(d))
    return host, devt


def _rel(gpu, ref):
    den = np.abs(ref).max()
    return float(np.abs(gpu - ref).max() / den) if den > 0 else float(np.abs(gpu).max())


CASES = [  # L, C, H, n_rbf, dtype, periodic, n, M
    (0, 16, 2, 8, "f32", False, 40, None),
    (1, 32, 2, 8, "f32", True, 40, None),
    (1, 128, 4, 16, "bf16", True, 40, None),
    (2, 16, 1, 16, "f32", False, 40, None),
    (2, 16, 4, 8, "f32", True, 48, None),
    (4, 128, 8, 16, "bf16", True, 40, None),
    (4, 128, 8, 16, "bf16", False, 32, 2),
    (3, 32, 2, 16, "bf16", True, 40, 0),
]


@pytest.mark.parametrize("L,C,H,n_rbf,dtype,periodic,n,M", CASES)
def test_backward_matches_the_oracle(L, C, H, n_rbf, dtype, periodic, n, M):
    h, t = _system(17 + L + C, n, L, C, H, n_rbf, dtype, periodic, M)
    assert h["col"].size > 4 * n
    cfg = e2f.make_cfg(L, C, H, n_rbf, h["cutoff"], dtype, m_max=-1 if M is None else M)
    g = e2f.e2f_onfly_attention_backward(cfg, t["pos"], h["box"], t["rp"], t["col"], t["x"], t["Wq"], t["Wk"],
                                         t["Wrad"], t["Wso2"], t["G"])
    torch.cuda.synchronize()
    _, ref = layer_grads(L, C, H, n_rbf, h["cutoff"], h["pos"].astype(np.float64), h["box"], h["rp"], h["col"],
                         h["x64"], h["Wq"], h["Wk"], h["Wrad"], h["w64"], h["G"], M=M)
    names = {"pos": "pos", "x": "x", "W_q": "Wq", "W_k": "Wk", "W_rad": "Wrad", "W_so2": "Wso2"}
    # fp32 storage: fp32 arithmetic (measured 0.3-1.4e-6 normwise): 1e-5. bf16 storage: the
    # SO(2) maps, their transposes and the weight-gradient contraction run on tensor cores
    # with fp16 operands (relative rounding 2^-11 per operand, fp32 accumulation; measured
    # 1.3-4.2e-4 normwise): 2e-3.
    tol = 2e-3 if dtype == "bf16" else 1e-5
    for k, rk in names.items():
        err = _rel(g[k].cpu().numpy().reshape(ref[rk].shape), ref[rk])
        assert err <= tol, (k, err)


def test_backward_isolated_node_and_position_gradient_only():
    h, t = _system(3, 24, 2, 16, 2, 8, "f32", False)
    # move atom 0 far away: no neighbours, so its gradients vanish
    t["pos"][0] = torch.tensor([100.0, 100.0, 100.0], device=t["pos"].device)
    pos = t["pos"].cpu().numpy()
    rp, col = neighbors_bruteforce(pos, None, 5.0)
    rp_d = torch.from_numpy(rp.astype(np.int32)).to(t["pos"].device)
    col_d = torch.from_numpy(col.astype(np.int32)).to(t["pos"].device)
    assert rp[1] == 0
    cfg = e2f.make_cfg(2, 16, 2, 8, 5.0, "f32")
    g = e2f.e2f_onfly_attention_backward(cfg, t["pos"], None, rp_d, col_d, t["x"], t["Wq"], t["Wk"], t["Wrad"],
                                         t["Wso2"], t["G"], want_weights=False)
    assert set(g) == {"pos", "x", "W_rad"}
    assert torch.all(g["pos"][0] == 0) and torch.all(g["x"][0] == 0)
    full = e2f.e2f_onfly_attention_backward(cfg, t["pos"], None, rp_d, col_d, t["x"], t["Wq"], t["Wk"], t["Wrad"],
                                            t["Wso2"], t["G"])
    assert torch.allclose(full["pos"], g["pos"], rtol=1e-5, atol=1e-6)


def test_backward_full_size_properties():
    # the 3000-atom water box with fp32 storage (the same bf16 values widened),
    # so the fp32 CUDA-core forward can serve a central difference
    d = DeviceInputs(3)
    w = d.w
    x32 = d.x.float().contiguous()
    so2 = d.Wso2.float().contiguous()
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, "f32")
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff)
    G = torch.randn((w.n_atoms, w.K, w.C), generator=torch.Generator().manual_seed(5)).to(d.pos.device)
    g = e2f.e2f_onfly_attention_backward(cfg, d.pos, d.box, rp, col, x32, d.Wq, d.Wk, d.Wrad, so2, G,
                                         want_weights=False)
    gp = g["pos"].double()
    assert torch.isfinite(gp).all() and torch.isfinite(g["x"]).all()
    # translation invariance: the forces sum to zero
    assert gp.sum(0).abs().max().item() <= 1e-4 * gp.abs().sum(0).max().item()
    # directional derivative against the forward
    dirn = torch.randn(d.pos.shape, generator=torch.Generator().manual_seed(9)).to(d.pos.device)
    eps = 2e-3

    def loss(p):
        out = e2f.e2f_onfly_attention(cfg, p, d.box, rp, col, x32, d.Wq, d.Wk, d.Wrad, so2)
        return (out.double() * G.double()).sum().item()

    fd = (loss(d.pos + eps * dirn) - loss(d.pos - eps * dirn)) / (2 * eps)
    an = (gp * dirn.double()).sum().item()
    assert abs(fd - an) <= 2e-2 * abs(an), (fd, an)


def test_backward_batched_graphs_sampled():
    # the 256-graph batch at full size; graphs do not interact, so the position and
    # feature gradients of the first four graphs equal the oracle's on those graphs alone
    d = DeviceInputs(2)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    G = np.random.default_rng(21).normal(size=(w.n_atoms, w.K, w.C)).astype(np.float32)
    g = e2f.e2f_onfly_attention_backward(cfg, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2,
                                         torch.from_numpy(G).to(d.pos.device), want_weights=False)
    gptr = np.asarray(w.graph_ptr)
    n_sub = int(gptr[4])
    rp0, col0 = neighbors_bruteforce(w.pos[:n_sub], None, w.cutoff, gptr[:5])
    wt = d.weights
    x64 = np.asarray(d.x_f64).reshape(w.n_atoms, w.K, w.C)[:n_sub]
    _, ref = layer_grads(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.pos[:n_sub].astype(np.float64), None, rp0, col0,
                         x64, wt.Wq, wt.Wk, wt.Wrad, wt.Wso2_f64, G[:n_sub])
    # bf16 storage: tensor-core maps with fp16 operands (see test_backward_matches_the_oracle)
    assert _rel(g["pos"].cpu().numpy()[:n_sub], ref["pos"]) <= 2e-3
    assert _rel(g["x"].cpu().numpy()[:n_sub], ref["x"]) <= 2e-3


def test_backward_without_edges_is_zero():
    h, t = _system(9, 8, 2, 16, 2, 8, "f32", False)
    t["pos"] *= 50.0  # spread the atoms far beyond the cutoff
    rp = torch.zeros(9, dtype=torch.int32, device=t["pos"].device)
    col = torch.zeros(0, dtype=torch.int32, device=t["pos"].device)
    cfg = e2f.make_cfg(2, 16, 2, 8, 5.0, "f32")
    g = e2f.e2f_onfly_attention_backward(cfg, t["pos"], None, rp, col, t["x"], t["Wq"], t["Wk"], t["Wrad"],
                                         t["Wso2"], t["G"])
    for k, v in g.items():
        assert torch.count_nonzero(v).item() == 0, k
