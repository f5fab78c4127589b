"""Pins for the gradient oracle (oracle.grad): its forward equals the numpy
dense layer, and every gradient matches central finite differences of the
numpy layer (an independent route: no autograd), on open and periodic
systems, full and truncated SO(2) maps; the position gradient of a
translation-invariant layer sums to zero."""
import numpy as np
import pytest

from oracle.grad import layer_grads
from oracle.layer import DenseLayer
from oracle.neighbors import neighbors_bruteforce
from workloads import so2_block_sizes


def _system(seed, n, side, periodic, L, C, H, n_rbf, M=None):
    rng = np.random.default_rng(seed)
    while True:  # positions with no pair distance within 0.05 of the cutoff
        pos = rng.uniform(0.0, side, (n, 3))
        dv = pos[:, None, :] - pos[None, :, :]
        if periodic:
            dv -= side * np.rint(dv / side)
        dist = np.linalg.norm(dv, axis=-1)[~np.eye(n, dtype=bool)]
        if dist.min() > 0.8 and np.abs(dist - 3.0).min() > 0.05:
            break
    box = [side] * 3 if periodic else None
    K = (L + 1) ** 2
    Mx = L if M is None else M
    n_so2 = sum(so2_block_sizes(L, C)[:2 * Mx + 1])
    d = dict(pos=pos, x=rng.normal(size=(n, K, C)), Wq=rng.normal(size=(C, C)) / np.sqrt(C),
             Wk=rng.normal(size=(C, C)) / np.sqrt(C), Wrad=rng.normal(size=(n_rbf, (L + 1) * C + H)),
             Wso2=rng.normal(size=n_so2) / np.sqrt(C), G=rng.normal(size=(n, K, C)))
    rp, col = neighbors_bruteforce(pos.astype(np.float32), box, 3.0)
    return d, box, rp, col


def _numpy_loss(L, C, H, n_rbf, box, rp, col, d, M=None):
    so2 = d["Wso2"]
    if M is not None and M < L:  # the numpy layer takes the full layer: zero blocks above M
        so2 = np.concatenate([so2, np.zeros(sum(so2_block_sizes(L, C)) - so2.size)])
    lay = DenseLayer(L, C, H, n_rbf, 3.0, d["Wq"], d["Wk"], d["Wrad"], so2)
    return float((lay(d["pos"], box, rp, col, d["x"]) * d["G"]).sum())


CASES = [(2, 4, 2, 6, False, None), (2, 4, 2, 6, True, None), (3, 4, 2, 5, True, None), (4, 2, 1, 4, False, None),
         (3, 4, 2, 5, False, 1)]


@pytest.mark.parametrize("L,C,H,n_rbf,periodic,M", CASES)
def test_gradients_match_finite_differences(L, C, H, n_rbf, periodic, M):
    d, box, rp, col = _system(100 + L * 7 + C, 10, 5.5 if periodic else 4.0, periodic, L, C, H, n_rbf, M)
    assert col.size > 20
    out, g = layer_grads(L, C, H, n_rbf, 3.0, d["pos"], box, rp, col, d["x"], d["Wq"], d["Wk"], d["Wrad"],
                         d["Wso2"], d["G"], M=M)
    rng = np.random.default_rng(7)
    eps = 1e-5
    for name in ("pos", "x", "Wq", "Wk", "Wrad", "Wso2"):
        dirn = rng.normal(size=d[name].shape)
        plus = dict(d)
        minus = dict(d)
        plus[name] = d[name] + eps * dirn
        minus[name] = d[name] - eps * dirn
        fd = (_numpy_loss(L, C, H, n_rbf, box, rp, col, plus, M) -
              _numpy_loss(L, C, H, n_rbf, box, rp, col, minus, M)) / (2 * eps)
        an = float((g[name] * dirn).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, fd, an)


@pytest.mark.parametrize("periodic", [False, True])
def test_forward_equals_numpy_layer_and_forces_sum_to_zero(periodic):
    L, C, H, n_rbf = 2, 4, 2, 6
    d, box, rp, col = _system(5, 12, 5.5 if periodic else 4.0, periodic, L, C, H, n_rbf)
    out, g = layer_grads(L, C, H, n_rbf, 3.0, d["pos"], box, rp, col, d["x"], d["Wq"], d["Wk"], d["Wrad"],
                         d["Wso2"], d["G"])
    lay = DenseLayer(L, C, H, n_rbf, 3.0, d["Wq"], d["Wk"], d["Wrad"], d["Wso2"])
    np.testing.assert_allclose(out, lay(d["pos"], box, rp, col, d["x"]), atol=1e-12, rtol=0)
    # a rigid translation changes nothing: the position gradient sums to zero
    assert np.abs(g["pos"].sum(axis=0)).max() <= 1e-10 * max(1.0, np.abs(g["pos"]).max())
    assert np.abs(g["pos"]).max() > 1e-3


def test_isolated_nodes_have_zero_gradient():
    L, C, H, n_rbf = 1, 2, 1, 4
    rng = np.random.default_rng(3)
    pos = np.array([[0.0, 0.0, 0.0], [10.0, 0.0, 0.0], [1.5, 0.0, 0.0]])
    rp, col = neighbors_bruteforce(pos.astype(np.float32), None, 3.0)
    x = rng.normal(size=(3, 4, C))
    W = dict(Wq=rng.normal(size=(C, C)), Wk=rng.normal(size=(C, C)), Wrad=rng.normal(size=(n_rbf, 2 * C + H)),
             Wso2=rng.normal(size=sum(so2_block_sizes(L, C))))
    G = rng.normal(size=(3, 4, C))
    out, g = layer_grads(L, C, H, n_rbf, 3.0, pos, None, rp, col, x, W["Wq"], W["Wk"], W["Wrad"], W["Wso2"], G)
    assert np.all(out[1] == 0) and np.all(g["pos"][1] == 0) and np.all(g["x"][1] == 0)
