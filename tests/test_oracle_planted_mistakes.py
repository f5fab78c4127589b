"""Each test plants one plausible mistake in the oracle (on the CPU, through
monkeypatch) and checks that one of the pins catches it. This guards the
pins themselves: a pin that passes on a broken oracle would pin nothing."""
import numpy as np
import pytest

import oracle.eaas as eaas
import oracle.layer as layer_mod
import oracle.sh as sh_mod
import test_oracle_eaas_layer as T
import test_oracle_sh_cg_wigner as S


def _fails(fn, *a):
    with pytest.raises(AssertionError):
        fn(*a)


def test_z_axis_layer_message_is_so2_map_of_gated_neighbour():
    # Two atoms on the z axis: node 0's only neighbour sits at +z, so the
    # edge frame is the identity and out_0 = SO2_W(g_v * x_1) exactly.
    rng = np.random.default_rng(21)
    L, C, H = 3, 2, 2
    pos = np.array([[0, 0, 0], [0, 0, 1.7]], np.float32)
    x = rng.normal(size=(2, (L + 1) ** 2, C))
    flat = T._rand_so2(rng, L, C)
    Wrad = rng.normal(size=(16, (L + 1) * C + H))
    lay = layer_mod.DenseLayer(L, C, H, 16, 3.0, np.eye(C), np.eye(C), Wrad, flat)
    rp = np.array([0, 1, 2], np.int32)
    col = np.array([1, 0], np.int32)
    out = lay(pos, None, rp, col, x)
    g = layer_mod.radial_basis(np.array([float(np.float32(1.7))]), 3.0, 16) @ Wrad
    lk = np.concatenate([np.full(2 * l + 1, l) for l in range(L + 1)])
    h = g[0, :(L + 1) * C].reshape(L + 1, C)[lk] * x[1]
    A, B = eaas.unpack_so2(flat, L, C)
    from so2_form import so2_apply
    np.testing.assert_allclose(out[0], so2_apply(h, A, B, L, C), atol=1e-12)


def test_catches_transposed_channel_weight(monkeypatch):
    orig = layer_mod.dense_messages

    def bad(h, Y, w):
        return orig(h, Y, {p: W.T for p, W in w.items()})
    monkeypatch.setattr(layer_mod, "dense_messages", bad)
    monkeypatch.setattr(T, "dense_messages", bad)
    _fails(T.test_eq13_so2_form_equals_dense_cg_contraction, 2, 4)


def test_catches_sign_error_in_odd_parity_block(monkeypatch):
    orig = eaas._systems

    def bad(l1, l3):
        e, o, Me, Mo = orig(l1, l3)
        return e, o, Me, -Mo
    monkeypatch.setattr(eaas, "_systems", bad)
    _fails(T.test_eq13_so2_form_equals_dense_cg_contraction, 2, 4)


def test_catches_dropped_path(monkeypatch):
    orig = layer_mod.dense_messages

    def bad(h, Y, w):
        return orig(h, Y, {p: W for p, W in w.items() if p != (2, 1, 1)})
    monkeypatch.setattr(T, "dense_messages", bad)
    _fails(T.test_eq13_so2_form_equals_dense_cg_contraction, 2, 4)


def test_catches_wrong_sign_convention_of_sine_harmonics(monkeypatch):
    orig = sh_mod.real_sh

    def bad(lmax, vec):
        Y = orig(lmax, vec).copy()
        for l in range(1, lmax + 1):
            Y[..., l * l:l * l + l] *= -1
        return Y
    monkeypatch.setattr(S, "real_sh", bad)
    _fails(S.test_sh_textbook_closed_forms_l_le_2)


def test_catches_reversed_edge_direction(monkeypatch):
    orig = layer_mod.edge_vectors
    monkeypatch.setattr(layer_mod, "edge_vectors", lambda pos, box, i, j: -orig(pos, box, i, j))
    _fails(test_z_axis_layer_message_is_so2_map_of_gated_neighbour)


def test_catches_scrambled_output_index(monkeypatch):
    orig = layer_mod.DenseLayer.edge_terms

    def bad(self, pos, box, x, i, j):
        g_a, v = orig(self, pos, box, x, i, j)
        return g_a, v[:, ::-1, :].copy()
    monkeypatch.setattr(layer_mod.DenseLayer, "edge_terms", bad)
    _fails(test_z_axis_layer_message_is_so2_map_of_gated_neighbour)


def test_catches_swapped_query_and_key(monkeypatch):
    orig_init = layer_mod.DenseLayer.__init__

    def bad(self, *a, **k):
        orig_init(self, *a, **k)
        self.Wq, self.Wk = self.Wk.copy(), self.Wq.copy()
    monkeypatch.setattr(layer_mod.DenseLayer, "__init__", bad)
    monkeypatch.setattr(T, "DenseLayer", layer_mod.DenseLayer)
    _fails(T.test_layer_L0_reduces_to_scalar_graph_attention)


# ---- the neighbour and gradient oracles ---------------------------------------

def test_catches_non_strict_cutoff_test(monkeypatch):
    import oracle.neighbors as nb
    import test_oracle_neighbors as N
    orig = nb.predicate_f32

    def bad(pi, pj, box, cutoff):
        # d2 <= rc^2: keeps a pair exactly at the cutoff
        return orig(pi, pj, box, float(np.nextafter(np.float32(cutoff), np.float32(np.inf))))
    monkeypatch.setattr(nb, "predicate_f32", bad)
    monkeypatch.setattr(N, "predicate_f32", bad)
    _fails(N.test_exactly_at_cutoff_is_excluded_and_just_inside_is_kept)


def test_catches_missing_minimum_image(monkeypatch):
    import oracle.neighbors as nb
    import test_oracle_neighbors as N
    orig = nb.predicate_f32
    monkeypatch.setattr(nb, "predicate_f32", lambda pi, pj, box, cutoff: orig(pi, pj, None, cutoff))
    periodic = [c for c in N.parse_cases() if c["box"] is not None]
    assert periodic
    _fails(N.test_handmade_fixture, periodic[0])


def test_catches_position_gradient_without_the_direction_term(monkeypatch):
    import oracle.grad as gr
    import test_oracle_grad as G
    orig = gr.real_sh_t
    # the harmonics of the edge direction held constant: forward unchanged,
    # the position gradient loses the rotation's contribution
    monkeypatch.setattr(gr, "real_sh_t", lambda lmax, r: orig(lmax, r.detach()))
    _fails(G.test_gradients_match_finite_differences, 2, 4, 2, 6, False, None)


def test_catches_radial_basis_without_envelope_or_with_wrong_width(monkeypatch):
    def no_envelope(d, cutoff, n_rbf):
        mu = np.arange(n_rbf) * (cutoff / (n_rbf - 1))
        return np.exp(-(((d[:, None] - mu[None, :]) / (cutoff / (n_rbf - 1))) ** 2))

    def wrong_width(d, cutoff, n_rbf):
        mu = np.arange(n_rbf) * (cutoff / (n_rbf - 1))
        u = 0.5 * (np.cos(np.pi * d / cutoff) + 1.0)
        return u[:, None] * np.exp(-(((d[:, None] - mu[None, :]) / (cutoff / n_rbf)) ** 2))
    for bad in (no_envelope, wrong_width):
        monkeypatch.setattr(layer_mod, "radial_basis", bad)
        monkeypatch.setattr(T, "radial_basis", bad)
        _fails(T.test_radial_basis_special_points)


# --- the Wigner-6j node-level convolution oracle (oracle/sixj.py) ---

def test_catches_sign_flipped_odd_couplings_in_the_6j_layer(monkeypatch):
    import oracle.sixj as sixj_mod
    import test_oracle_sixj as X
    good = sixj_mod.real_cg
    monkeypatch.setattr(sixj_mod, "real_cg", lambda a, b, c: -good(a, b, c) if (a + b + c) % 2 else good(a, b, c))
    X.test_sixj_layer_rotation_equivariance_and_translation_invariance()  # still equivariant ...
    _fails(X.test_sixj_layer_equals_a_node_split_evaluation)             # ... but not the same layer


def test_catches_condon_shortley_phase_in_solid_harmonics(monkeypatch):
    import oracle.sixj as sixj_mod
    import test_oracle_sixj as X
    good = sixj_mod.real_sh

    def with_phase(lmax, v):
        Y = good(lmax, v).copy()
        for l in range(lmax + 1):
            for m in range(1, l + 1, 2):
                Y[..., l * l + l + m] *= -1
                Y[..., l * l + l - m] *= -1
        return Y
    monkeypatch.setattr(sixj_mod, "real_sh", with_phase)
    _fails(X.test_solid_harmonics_closed_forms_l_le_2)


def test_catches_a_wrong_triangle_coefficient_in_the_6j_symbol(monkeypatch):
    from fractions import Fraction
    from math import factorial as f

    import oracle.sixj as sixj_mod
    import test_oracle_sixj as X
    monkeypatch.setattr(sixj_mod, "_delta", lambda a, b, c: Fraction(f(a + b - c) * f(a - b + c) * f(-a + b + c)))
    _fails(X.test_6j_matches_sympy)


def test_catches_interleaved_heads_in_the_6j_layer(monkeypatch):
    # channel c must take the softmax of head c // (C/H); a plausible slip
    # assigns head c % H instead
    import oracle.sixj as sixj_mod
    import test_oracle_sixj as X

    real_repeat = np.repeat

    class _NP:
        def __getattr__(self, name):
            return getattr(np, name)

        @staticmethod
        def repeat(a, r, axis=None):
            if axis == 1:
                return np.tile(a, (1, r))
            return real_repeat(a, r, axis=axis)
    monkeypatch.setattr(sixj_mod, "np", _NP())
    _fails(X.test_sixj_layer_equals_a_node_split_evaluation)
