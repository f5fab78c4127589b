"""Pins for the oracle of the Wigner-6j node-level convolution (oracle/sixj.py):
the solid harmonics against textbook closed forms and their addition
theorem, Racah's 6j formula against sympy and its orthogonality, the claim
that the re-coupling coefficients are 6j symbols, and the edge-form layer
against its symmetries, a closed-form special case and an independent
node-split evaluation."""
import itertools
from math import comb, sqrt

import numpy as np
import pytest
from sympy.physics.wigner import wigner_6j as sympy_6j

from oracle.cg import real_cg
from oracle.layer import radial_basis, softmax_two_pass
from oracle.sixj import SixjLayer, sixj_paths, solid_harmonics, wigner_6j
from oracle.wigner import random_rotation, rotate_irreps


def test_solid_harmonics_closed_forms_l_le_2():
    r = np.random.default_rng(0).normal(size=(30, 3)) * 2.5
    x, y, z = r.T
    S = solid_harmonics(2, r)
    s3 = sqrt(3.0)
    ref = np.stack([np.ones_like(x), y, z, x,
                    s3 * x * y, s3 * y * z, z * z - 0.5 * (x * x + y * y),
                    s3 * x * z, 0.5 * s3 * (x * x - y * y)], axis=1)
    np.testing.assert_allclose(S, ref, atol=1e-12)
    np.testing.assert_array_equal(solid_harmonics(3, np.zeros((1, 3)))[0], np.eye(16)[0])


@pytest.mark.parametrize("l", range(9))
def test_solid_harmonics_addition_theorem(l):
    # S^l(a + b) = sum_lam sqrt(binom(2l, 2 lam)) [S^lam(a) (x) S^(l-lam)(b)]^l
    rng = np.random.default_rng(10 + l)
    a, b = rng.normal(size=(6, 3)), rng.normal(size=(6, 3))
    Sa, Sb = solid_harmonics(l, a), solid_harmonics(l, b)
    rhs = np.zeros((6, 2 * l + 1))
    for lam in range(l + 1):
        mu = l - lam
        rhs += sqrt(comb(2 * l, 2 * lam)) * np.einsum(
            "abc,ea,eb->ec", real_cg(lam, mu, l), Sa[:, lam * lam:(lam + 1) ** 2], Sb[:, mu * mu:(mu + 1) ** 2])
    lhs = solid_harmonics(l, a + b)[:, l * l:]
    np.testing.assert_allclose(rhs, lhs, atol=1e-10 * max(1.0, np.abs(lhs).max()))


def test_6j_matches_sympy():
    for args in itertools.product(range(4), repeat=6):
        if sum(args) % 3:
            continue  # a sparse, spread sample of the 4^6 arguments
        want = float(sympy_6j(*args))
        assert abs(wigner_6j(*args) - want) < 1e-13, args


def test_6j_special_values_and_orthogonality():
    for a, b, c in itertools.product(range(5), repeat=3):
        if abs(a - b) <= c <= a + b:
            want = (-1) ** (a + b + c) / sqrt((2 * b + 1) * (2 * c + 1))
            assert abs(wigner_6j(a, b, c, 0, c, b) - want) < 1e-14
    assert abs(wigner_6j(1, 1, 1, 1, 1, 1) - 1 / 6) < 1e-15
    # sum_x (2x+1)(2f+1) {a b x; c d f} {a b x; c d f'} = delta_ff'
    a, b, c, d = 2, 3, 2, 3
    fs = range(abs(b - c), b + c + 1)
    for f, g in itertools.product(fs, fs):
        s = sum((2 * x + 1) * (2 * f + 1) * wigner_6j(a, b, x, c, d, f) * wigner_6j(a, b, x, c, d, g)
                for x in range(0, 10))
        assert abs(s - (f == g)) < 1e-12, (f, g, s)


@pytest.mark.parametrize("l1,lam,mu,l3", [(1, 1, 1, 1), (2, 1, 2, 3), (2, 2, 2, 2), (3, 2, 1, 4), (4, 3, 2, 4)])
def test_recoupling_coefficients_are_6j_symbols(l1, lam, mu, l3):
    # x (x) [S^lam (x) S^mu]^l2 -> sum_k c_k [[x (x) S^lam]^k (x) S^mu]^l3 with
    # |c_k| = sqrt((2k+1)(2 l2+1)) |{l1 lam k; mu l3 l2}|, l2 = lam + mu
    l2 = lam + mu
    if not abs(l1 - l3) <= l2 <= l1 + l3:
        pytest.skip("not a path")
    TA = np.einsum("adc,bed->abec", real_cg(l1, l2, l3), real_cg(lam, mu, l2))
    rebuilt = np.zeros_like(TA)
    for k in range(abs(l1 - lam), l1 + lam + 1):
        if not abs(k - mu) <= l3 <= k + mu:
            continue
        TB = np.einsum("abk,kec->abec", real_cg(l1, lam, k), real_cg(k, mu, l3))
        ck = np.sum(TA * TB) / (2 * l3 + 1)
        want = sqrt((2 * k + 1) * (2 * l2 + 1)) * abs(wigner_6j(l1, lam, k, mu, l3, l2))
        assert abs(abs(ck) - want) < 1e-12, (k, ck, want)
        rebuilt += ck * TB
    np.testing.assert_allclose(rebuilt, TA, atol=1e-12)


def _layer(rng, L, Lf, C, H, n_rbf=8, cutoff=5.0, zero_except=None):
    P = sixj_paths(L, Lf)
    w = rng.normal(size=(len(P), C))
    if zero_except is not None:
        for n, p in enumerate(P):
            if not zero_except(p):
                w[n] = 0.0
    lay = SixjLayer(L, Lf, C, H, n_rbf, cutoff, rng.normal(size=(C, C)) / sqrt(C),
                    rng.normal(size=(C, C)) / sqrt(C), rng.normal(size=(n_rbf, H)), w)
    return lay


def _graph(rng, n=14, side=4.0, cutoff=5.0):
    pos = rng.uniform(0, side, size=(n, 3))
    d = np.linalg.norm(pos[:, None] - pos[None], axis=-1)
    adj = (d < cutoff) & ~np.eye(n, dtype=bool)
    adj[0, :] = False  # node 0 has no neighbours
    rp = np.concatenate([[0], np.cumsum(adj.sum(1))]).astype(np.int32)
    col = np.concatenate([np.nonzero(a)[0] for a in adj]).astype(np.int32)
    return pos, rp, col


def test_sixj_layer_rotation_equivariance_and_translation_invariance():
    rng = np.random.default_rng(3)
    L, Lf, C, H = 3, 5, 4, 2
    lay = _layer(rng, L, Lf, C, H)
    pos, rp, col = _graph(rng)
    x = rng.normal(size=(pos.shape[0], (L + 1) ** 2, C))
    out = lay(pos, rp, col, x)
    assert np.abs(out[0]).max() == 0.0
    R = random_rotation(rng)
    out_r = lay(pos @ R.T + np.array([3.0, -1.0, 7.5]), rp, col, rotate_irreps(x, L, R))
    np.testing.assert_allclose(out_r, rotate_irreps(out, L, R), atol=1e-9 * np.abs(out).max())


def test_sixj_layer_scalar_case_is_plain_attention():
    rng = np.random.default_rng(4)
    lay = _layer(rng, 0, 0, 3, 1)
    pos, rp, col = _graph(rng)
    x = rng.normal(size=(pos.shape[0], 1, 3))
    out = lay(pos, rp, col, x)
    q, k = x[:, 0] @ lay.Wq.T, x[:, 0] @ lay.Wk.T
    w = lay.w[(0, 0, 0)]
    for i in range(1, pos.shape[0]):
        j = col[rp[i]:rp[i + 1]]
        d = np.linalg.norm(pos[j] - pos[i], axis=1)
        a = (radial_basis(d, 5.0, 8) @ lay.Wrad)[:, 0] * (k[j] @ q[i]) / sqrt(3)
        al = np.exp(a - a.max())
        al /= al.sum()
        np.testing.assert_allclose(out[i, 0], w * (al @ x[j, 0]), atol=1e-12)


def test_sixj_layer_scalar_input_paths_are_the_harmonics():
    # with only the paths (0, l, l): v_ij^l = w x_j^0 S^l(r_ij), Q^{0ll} being the identity
    rng = np.random.default_rng(5)
    L, C = 3, 2
    lay = _layer(rng, L, 2 * L, C, 1, zero_except=lambda p: p[0] == 0)
    pos, rp, col = _graph(rng, n=8)
    x = rng.normal(size=(8, (L + 1) ** 2, C))
    out = lay(pos, rp, col, x)
    q, k = x[:, 0] @ lay.Wq.T, x[:, 0] @ lay.Wk.T
    for i in range(1, 8):
        j = col[rp[i]:rp[i + 1]]
        r = pos[j] - pos[i]
        a = (radial_basis(np.linalg.norm(r, axis=1), 5.0, 8) @ lay.Wrad)[:, 0] * (k[j] @ q[i]) / sqrt(C)
        al = softmax_two_pass(a[:, None])[:, 0]
        S = solid_harmonics(L, r)
        for l in range(L + 1):
            want = np.einsum("e,em,ec->mc", al, S[:, l * l:(l + 1) ** 2], x[j, 0, :]) * lay.w[(0, l, l)]
            np.testing.assert_allclose(out[i, l * l:(l + 1) ** 2], want, atol=1e-12)


def test_sixj_layer_equals_a_node_split_evaluation():
    # The same layer evaluated the node-level way, written out here in numpy:
    # a_j = x_j - o, b_i = o - x_i for any origin o; per node j the coupled
    # products [x_j^l1 (x) S^lam(a_j)]^k; per node i their softmax-weighted sum
    # Z_i, then out_i^l3 = sum w sqrt(binom(2 l2, 2 lam)) c_k [Z_i (x) S^mu(b_i)]^l3.
    rng = np.random.default_rng(6)
    L, Lf, C, H = 2, 4, 4, 2
    lay = _layer(rng, L, Lf, C, H)
    pos, rp, col = _graph(rng, n=10)
    N = pos.shape[0]
    x = rng.normal(size=(N, (L + 1) ** 2, C))
    want = lay(pos, rp, col, x)
    o = pos.mean(0) + np.array([0.3, -0.2, 0.1])
    Sa, Sb = solid_harmonics(Lf, pos - o), solid_harmonics(Lf, o - pos)
    dh = C // H
    q, k = x[:, 0] @ lay.Wq.T, x[:, 0] @ lay.Wk.T
    got = np.zeros_like(want)
    for i in range(N):
        j = col[rp[i]:rp[i + 1]]
        if j.size == 0:
            continue
        d = np.linalg.norm(pos[j] - pos[i], axis=1)
        a = (radial_basis(d, 5.0, 8) @ lay.Wrad) * (q[i].reshape(H, dh)[None] * k[j].reshape(-1, H, dh)).sum(-1)
        al = np.repeat(softmax_two_pass(a / sqrt(dh)), dh, axis=1)      # [deg, C]
        for (l1, l2, l3), wc in lay.w.items():
            for lam in range(l2 + 1):
                mu = l2 - lam
                TA = np.einsum("adc,bed->abec", real_cg(l1, l2, l3), real_cg(lam, mu, l2))
                for kk in range(abs(l1 - lam), l1 + lam + 1):
                    if not abs(kk - mu) <= l3 <= kk + mu:
                        continue
                    TB = np.einsum("abk,kec->abec", real_cg(l1, lam, kk), real_cg(kk, mu, l3))
                    ck = np.sum(TA * TB) / (2 * l3 + 1)
                    z = np.einsum("abk,eac,eb->ekc", real_cg(l1, lam, kk), x[j, l1 * l1:(l1 + 1) ** 2],
                                  Sa[j, lam * lam:(lam + 1) ** 2])
                    Z = np.einsum("ec,ekc->kc", al, z)
                    got[i, l3 * l3:(l3 + 1) ** 2] += sqrt(comb(2 * l2, 2 * lam)) * ck * wc * np.einsum(
                        "kem,kc,e->mc", real_cg(kk, mu, l3), Z, Sb[i, mu * mu:(mu + 1) ** 2])
    np.testing.assert_allclose(got, want, atol=1e-9 * np.abs(want).max())
