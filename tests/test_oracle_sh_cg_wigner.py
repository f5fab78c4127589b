"""Pins for the oracle's spherical harmonics, Clebsch-Gordan coefficients and
Wigner-D matrices, against closed forms, library routines and invariants."""
import numpy as np
import pytest
from numpy.polynomial.legendre import leggauss
from scipy.special import eval_legendre, sph_harm_y
from sympy import S
from sympy.physics.wigner import clebsch_gordan

from oracle.cg import cg_complex, paths, real_cg
from oracle.sh import real_from_complex, real_sh
from oracle.wigner import random_rotation, rot_y, rot_z, wigner_D

PI = np.pi


def _dirs(n, seed=0):
    v = np.random.default_rng(seed).normal(size=(n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def test_sh_textbook_closed_forms_l_le_2():
    u = _dirs(40)
    x, y, z = u.T
    Y = real_sh(2, u)
    ref = np.stack([
        np.full_like(x, 0.5 / np.sqrt(PI)),
        np.sqrt(3 / (4 * PI)) * y, np.sqrt(3 / (4 * PI)) * z, np.sqrt(3 / (4 * PI)) * x,
        0.5 * np.sqrt(15 / PI) * x * y, 0.5 * np.sqrt(15 / PI) * y * z,
        0.25 * np.sqrt(5 / PI) * (3 * z * z - 1),
        0.5 * np.sqrt(15 / PI) * x * z, 0.25 * np.sqrt(15 / PI) * (x * x - y * y),
    ], axis=1)
    np.testing.assert_allclose(Y, ref, atol=1e-14)


def test_sh_matches_scipy_complex_harmonics_through_U():
    u = _dirs(64, 1)
    th = np.arccos(u[:, 2])
    ph = np.arctan2(u[:, 1], u[:, 0])
    Y = real_sh(8, u)
    for l in range(9):
        Yc = np.stack([sph_harm_y(l, m, th, ph) for m in range(-l, l + 1)], axis=1)
        Yr = Yc @ real_from_complex(l).T
        np.testing.assert_allclose(Yr.imag, 0, atol=1e-13)
        np.testing.assert_allclose(Yr.real, Y[:, l * l:(l + 1) ** 2], atol=1e-13)


def test_lemma_4_1_aligned_frame_harmonics_only_m0():
    # gist.science Technical Summary 2.1: along the axis only m = 0 survives.
    Y = real_sh(8, np.array([[0.0, 0.0, 1.0]]))[0]
    for l in range(9):
        for m in range(-l, l + 1):
            want = np.sqrt((2 * l + 1) / (4 * PI)) if m == 0 else 0.0
            assert abs(Y[l * l + l + m] - want) < 1e-13


def test_sh_addition_theorem():
    u, v = _dirs(30, 2), _dirs(30, 3)
    Yu, Yv = real_sh(8, u), real_sh(8, v)
    cosg = np.sum(u * v, axis=1)
    for l in range(9):
        s = slice(l * l, (l + 1) ** 2)
        lhs = np.sum(Yu[:, s] * Yv[:, s], axis=1)
        np.testing.assert_allclose(lhs, (2 * l + 1) / (4 * PI) * eval_legendre(l, cosg), atol=1e-13)


def test_sh_orthonormal_by_quadrature():
    # Gauss-Legendre in cos(theta) x uniform phi is exact for degree <= 16 here
    t, wt = leggauss(20)
    ph = np.arange(40) * (2 * PI / 40)
    ct, pp = np.meshgrid(t, ph, indexing="ij")
    st = np.sqrt(1 - ct ** 2)
    pts = np.stack([st * np.cos(pp), st * np.sin(pp), ct], -1).reshape(-1, 3)
    w = (wt[:, None] * np.full(ph.size, 2 * PI / ph.size)[None]).ravel()
    Y = real_sh(8, pts)
    G = (Y * w[:, None]).T @ Y
    np.testing.assert_allclose(G, np.eye(81), atol=1e-12)


@pytest.mark.parametrize("l1,m1,l2,m2,l3", [
    (1, 0, 1, 0, 2), (1, 1, 1, -1, 0), (2, 1, 3, -2, 4), (4, 2, 4, -1, 3), (3, 3, 2, -2, 1),
    (4, -4, 4, 4, 0), (4, 3, 4, -4, 8), (2, -2, 4, 1, 5), (3, 0, 2, 0, 1), (4, 0, 3, 1, 7)])
def test_cg_matches_sympy_exactly(l1, m1, l2, m2, l3):
    ref = float(clebsch_gordan(S(l1), S(l2), S(l3), S(m1), S(m2), S(m1 + m2)))
    assert abs(cg_complex(l1, m1, l2, m2, l3, m1 + m2) - ref) < 1e-15


def test_cg_selection_rules_and_orthogonality():
    for l1 in range(4):
        for l2 in range(4):
            # sum_{m1,m2} C(l3 m3) C(l3' m3') = delta: columns orthonormal
            rows = []
            for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                for m3 in range(-l3, l3 + 1):
                    rows.append([cg_complex(l1, a, l2, b, l3, m3)
                                 for a in range(-l1, l1 + 1) for b in range(-l2, l2 + 1)])
            M = np.array(rows)
            np.testing.assert_allclose(M @ M.T, np.eye(M.shape[0]), atol=1e-13)
            np.testing.assert_allclose(M.T @ M, np.eye(M.shape[1]), atol=1e-13)
    assert cg_complex(2, 1, 2, 1, 3, 1) == 0.0  # m3 != m1 + m2


def test_wigner_D_orthogonal_and_homomorphism():
    rng = np.random.default_rng(4)
    R1, R2 = random_rotation(rng), random_rotation(rng)
    for l in range(9):
        D1, D2 = wigner_D(l, R1), wigner_D(l, R2)
        np.testing.assert_allclose(D1 @ D1.T, np.eye(2 * l + 1), atol=1e-12)
        np.testing.assert_allclose(wigner_D(l, R1 @ R2), D1 @ D2, atol=1e-12)
        assert abs(np.linalg.det(D1) - 1.0) < 1e-11


def test_wigner_D_defining_relation_at_fresh_points():
    rng = np.random.default_rng(5)
    R = random_rotation(rng)
    v = _dirs(25, 6)
    Y, Yr = real_sh(6, v), real_sh(6, v @ R.T)
    for l in range(7):
        s = slice(l * l, (l + 1) ** 2)
        np.testing.assert_allclose(Yr[:, s], Y[:, s] @ wigner_D(l, R).T, atol=1e-12)


def test_wigner_D_z_rotation_closed_form():
    a = 0.83
    for l in range(5):
        D = wigner_D(l, rot_z(a))
        ref = np.zeros((2 * l + 1, 2 * l + 1))
        ref[l, l] = 1.0
        for m in range(1, l + 1):
            c, s = np.cos(m * a), np.sin(m * a)
            ref[l + m, l + m], ref[l + m, l - m] = c, -s
            ref[l - m, l - m], ref[l - m, l + m] = c, s
        np.testing.assert_allclose(D, ref, atol=1e-12)


def test_wigner_D_l1_is_permuted_rotation_matrix():
    R = random_rotation(np.random.default_rng(7)) @ rot_y(0.3)
    P = np.array([[0, 1, 0], [0, 0, 1], [1, 0, 0]])  # (x,y,z) -> (y,z,x)
    np.testing.assert_allclose(wigner_D(1, R), P @ R @ P.T, atol=1e-12)


def test_real_cg_is_equivariant():
    rng = np.random.default_rng(8)
    R = random_rotation(rng)
    D = [wigner_D(l, R) for l in range(9)]
    for (l1, l2, l3) in paths(4):
        Q = real_cg(l1, l2, l3)
        x, y = rng.normal(size=2 * l1 + 1), rng.normal(size=2 * l2 + 1)
        z = np.einsum("abc,a,b->c", Q, x, y)
        z2 = np.einsum("abc,a,b->c", Q, D[l1] @ x, D[l2] @ y)
        np.testing.assert_allclose(D[l3] @ z, z2, atol=1e-12)
        assert np.abs(Q).max() > 1e-3


def test_real_cg_aligned_frame_parity_reindexing():
    # fugumt abstract: "sparse parity re-indexing". With m2 = 0 the coupling
    # keeps |m|: m3 = m1 on even paths, m3 = -m1 on odd ones.
    for (l1, l2, l3) in paths(4):
        Q = real_cg(l1, l2, l3)
        par = (l1 + l2 + l3) % 2
        for m1 in range(-l1, l1 + 1):
            for m3 in range(-l3, l3 + 1):
                allowed = (m3 == m1) if par == 0 else (m3 == -m1 and m1 != 0)
                if not allowed:
                    assert abs(Q[m1 + l1, l2, m3 + l3]) < 1e-13
        for m in range(1, min(l1, l3) + 1):
            if par == 0:
                assert abs(Q[m + l1, l2, m + l3] - Q[-m + l1, l2, -m + l3]) < 1e-13
            else:
                assert abs(Q[-m + l1, l2, m + l3] + Q[m + l1, l2, -m + l3]) < 1e-13
