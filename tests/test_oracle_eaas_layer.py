"""Pins for the oracle's EAAS conversion and the dense layer: brute force
against the SO(2) form, symmetries, closed-form special cases and the
streaming softmax."""
import numpy as np
import pytest

from oracle.cg import paths, real_cg
from oracle.eaas import pack_so2, paths_from_so2, so2_from_paths, unpack_so2
from oracle.layer import DenseLayer, dense_messages, radial_basis, softmax_two_pass
from oracle.neighbors import neighbors_bruteforce
from oracle.sh import real_sh
from oracle.wigner import random_rotation, rotate_irreps, rot_z
from so2_form import edge_frame, so2_apply, so2_message
from workloads import so2_block_sizes


def _rand_so2(rng, L, C):
    return rng.normal(size=sum(so2_block_sizes(L, C))) / np.sqrt(C)


@pytest.mark.parametrize("L,C", [(1, 2), (2, 3), (3, 2), (4, 2)])
def test_so2_path_round_trip(L, C):
    rng = np.random.default_rng(L * 10 + C)
    w = {p: rng.normal(size=(C, C)) for p in paths(L)}
    A, B = so2_from_paths(w, L, C)
    w2 = paths_from_so2(A, B, L, C)
    for p in w:
        np.testing.assert_allclose(w2[p], w[p], atol=1e-12)
    flat = _rand_so2(rng, L, C)
    A, B = unpack_so2(flat, L, C)
    np.testing.assert_array_equal(pack_so2(A, B, L), flat)
    A2, B2 = so2_from_paths(paths_from_so2(A, B, L, C), L, C)
    np.testing.assert_allclose(pack_so2(A2, B2, L), flat, atol=1e-12)


def test_number_of_paths_matches_so2_parameters():
    # each (l1,l3) has 2 min(l1,l3)+1 paths and as many (A,B) coefficients
    for L in range(5):
        n_paths = len(paths(L))
        n_so2 = sum(so2_block_sizes(L, 1))
        assert n_paths == n_so2


@pytest.mark.parametrize("L,C", [(1, 3), (2, 4), (4, 2)])
def test_eq13_so2_form_equals_dense_cg_contraction(L, C):
    # Brute force: the dense CG message (O(L^6) contraction over m1, m2 with
    # explicit edge harmonics) equals the rotated SO(2) form (Eq. 13).
    rng = np.random.default_rng(100 + L)
    A, B = unpack_so2(_rand_so2(rng, L, C), L, C)
    w = paths_from_so2(A, B, L, C)
    for _ in range(6):
        r = rng.normal(size=3)
        h = rng.normal(size=((L + 1) ** 2, C))
        vd = dense_messages(h[None], real_sh(2 * L, r)[None], w)[0]
        vs = so2_message(r, h, A, B, L, C)
        np.testing.assert_allclose(vs, vd, atol=1e-12 * np.abs(vd).max())
        # roll about the edge axis changes nothing
        vr = so2_message(r, h, A, B, L, C, R=rot_z(1.234) @ edge_frame(r))
        np.testing.assert_allclose(vr, vd, atol=1e-12 * np.abs(vd).max())


def test_aligned_edge_message_is_so2_map_directly():
    # Edge along +z: D = I, so the dense message is the SO(2) map of h itself.
    rng = np.random.default_rng(9)
    L, C = 4, 3
    A, B = unpack_so2(_rand_so2(rng, L, C), L, C)
    w = paths_from_so2(A, B, L, C)
    h = rng.normal(size=((L + 1) ** 2, C))
    vd = dense_messages(h[None], real_sh(2 * L, np.array([0.0, 0.0, 2.5]))[None], w)[0]
    np.testing.assert_allclose(vd, so2_apply(h, A, B, L, C), atol=1e-12)


def _small_system(rng, n, L, C, H, periodic=False):
    side = 7.0
    pos = rng.uniform(0, side, size=(n, 3)).astype(np.float32)
    box = np.full(3, side, np.float32) if periodic else None
    x = rng.normal(size=(n, (L + 1) ** 2, C))
    Wq, Wk = rng.normal(size=(C, C)) / np.sqrt(C), rng.normal(size=(C, C)) / np.sqrt(C)
    Wrad = rng.normal(size=(16, (L + 1) * C + H)) / np.sqrt(C)
    Wso2 = _rand_so2(rng, L, C)
    layer = DenseLayer(L, C, H, 16, 3.4, Wq, Wk, Wrad, Wso2)
    layer.flat_so2 = Wso2
    layer.ref_W = (Wq, Wk, Wrad)
    row_ptr, col = neighbors_bruteforce(pos, box, 3.4)
    return pos, box, x, layer, row_ptr, col


def test_layer_equivariant_under_global_rotation():
    rng = np.random.default_rng(10)
    L, C, H = 2, 4, 2
    pos, box, x, layer, rp, col = _small_system(rng, 9, L, C, H)
    assert col.size > 10
    out = layer(pos, box, rp, col, x)
    R = random_rotation(rng)
    pos_r = pos.astype(np.float64) @ R.T
    out_r = layer(pos_r, None, rp, col, rotate_irreps(x, L, R))
    np.testing.assert_allclose(out_r, rotate_irreps(out, L, R), atol=1e-12 * np.abs(out).max())


def test_layer_permutation_translation_and_image_shift():
    rng = np.random.default_rng(11)
    L, C, H = 2, 4, 2
    pos, box, x, layer, rp, col = _small_system(rng, 10, L, C, H, periodic=True)
    out = layer(pos, box, rp, col, x)
    # permutation: relabel atoms, rebuild the CSR from the permuted pairs
    perm = rng.permutation(pos.shape[0])
    inv = np.argsort(perm)
    rows = np.repeat(np.arange(pos.shape[0]), np.diff(rp))
    pr, pc = inv[rows], inv[col]
    order = np.lexsort((pc, pr))
    rp2 = np.concatenate([[0], np.cumsum(np.bincount(pr, minlength=pos.shape[0]))])
    out_p = layer(pos[perm], box, rp2, pc[order], x[perm])
    np.testing.assert_allclose(out_p, out[perm], atol=1e-12 * np.abs(out).max())
    # periodic image shift of single atoms: same output
    shift = rng.integers(-2, 3, size=pos.shape) * box
    out_s = layer(pos.astype(np.float64) + shift, box, rp, col, x)
    np.testing.assert_allclose(out_s, out, atol=1e-10 * np.abs(out).max())
    # global translation: same output
    out_t = layer(pos.astype(np.float64) + np.array([0.3, -1.1, 2.0]), box, rp, col, x)
    np.testing.assert_allclose(out_t, out, atol=1e-10 * np.abs(out).max())


def test_layer_L0_reduces_to_scalar_graph_attention():
    rng = np.random.default_rng(12)
    L, C, H = 0, 4, 2
    pos, box, x, layer, rp, col = _small_system(rng, 8, L, C, H)
    out = layer(pos, box, rp, col, x)
    # closed form: out_i = sum_j softmax_j(g_a <q_i,k_j>/sqrt(d)) * (A0 (g_v * x_j))
    A0 = layer.flat_so2.reshape(C, C)
    dh = C // H
    p = pos.astype(np.float64)
    Wq, Wk, Wrad = layer.ref_W
    q = x[:, 0, :] @ Wq.T
    k = x[:, 0, :] @ Wk.T
    for i in range(pos.shape[0]):
        js = col[rp[i]:rp[i + 1]]
        if js.size == 0:
            assert np.all(out[i] == 0)
            continue
        d = np.linalg.norm(p[js] - p[i], axis=1)
        g = radial_basis(d, 3.4, 16) @ Wrad
        a = g[:, C:] * (q[i].reshape(H, dh) * k[js].reshape(-1, H, dh)).sum(-1) / np.sqrt(dh)
        e = np.exp(a - a.max(0))
        al = np.repeat(e / e.sum(0), dh, axis=1)
        v = (g[:, :C] * x[js, 0, :]) @ A0.T
        np.testing.assert_allclose(out[i, 0], (al * v).sum(0), atol=1e-12)


def test_radial_basis_special_points():
    # 16 Gaussians at mu_k = k rc/15 of width rc/15 under the cosine envelope:
    # at d = 0 the envelope is 1 and basis k is exp(-k^2); at d = rc/2 (7.5
    # widths) the envelope is 1/2; at d = rc it is 0
    rc = 5.0
    k = np.arange(16)
    got = radial_basis(np.array([0.0, rc / 2, rc]), rc, 16)
    np.testing.assert_allclose(got[0], np.exp(-(k ** 2.0)), rtol=1e-12, atol=0)
    np.testing.assert_allclose(got[1], 0.5 * np.exp(-((7.5 - k) ** 2.0)), rtol=1e-12, atol=0)
    np.testing.assert_allclose(got[2], 0.0, atol=1e-16)


def test_single_neighbour_gets_full_weight_and_isolated_node_is_zero():
    rng = np.random.default_rng(13)
    L, C, H = 2, 2, 1
    pos = np.array([[0, 0, 0], [0.3, 0.4, 1.2], [20, 20, 20]], np.float32)
    x = rng.normal(size=(3, 9, C))
    Wso2 = _rand_so2(rng, L, C)
    layer = DenseLayer(L, C, H, 16, 3.0, np.eye(C), np.eye(C), rng.normal(size=(16, 3 * C + H)), Wso2)
    rp, col = neighbors_bruteforce(pos, None, 3.0)
    out = layer(pos, None, rp, col, x)
    assert np.all(out[2] == 0)
    g_a, v = layer.edge_terms(pos, None, x, np.array([0]), np.array([1]))
    np.testing.assert_allclose(out[0], v[0], atol=1e-13)


def test_online_softmax_equals_two_pass():
    # gist.science Technical Summary 2.2: the kernel keeps a running max,
    # normaliser and value accumulator; the result is the plain softmax.
    rng = np.random.default_rng(14)
    a = rng.normal(size=(57, 3)) * 6
    v = rng.normal(size=(57, 3, 5))
    ref = np.einsum("eh,ehc->hc", softmax_two_pass(a), v)
    m = np.full(3, -np.inf)
    s = np.zeros(3)
    acc = np.zeros((3, 5))
    for blk in range(0, 57, 8):
        ab, vb = a[blk:blk + 8], v[blk:blk + 8]
        m2 = np.maximum(m, ab.max(0))
        sc = np.exp(m - m2)
        p = np.exp(ab - m2)
        s = s * sc + p.sum(0)
        acc = acc * sc[:, None] + np.einsum("eh,ehc->hc", p, vb)
        m = m2
    np.testing.assert_allclose(acc / s[:, None], ref, atol=1e-14)
