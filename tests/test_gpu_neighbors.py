"""GPU cell list against the oracle's exact fp32 predicate: bit-exact CSR."""
import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
from gpu_util import DeviceInputs, dev, oracle_csr
from test_oracle_neighbors import csr_from_expect, parse_cases

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_csr_bit_exact_on_workloads(cfg):
    d = DeviceInputs(cfg)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, d.w.cutoff, d.graph_ptr)
    rp0, col0 = oracle_csr(cfg)
    np.testing.assert_array_equal(rp.cpu().numpy(), rp0)
    np.testing.assert_array_equal(col.cpu().numpy(), col0)


@pytest.mark.parametrize("case", parse_cases(), ids=lambda c: c["name"])
def test_handmade_fixture(case):
    pos = torch.from_numpy(case["atoms"]).to(dev())
    gp = None if case["graph_ptr"] is None else torch.from_numpy(case["graph_ptr"]).to(dev())
    box = None if case["box"] is None else [float(v) for v in case["box"]]
    rp, col = e2f.e2f_build_neighbors(pos, box, case["cutoff"], gp)
    rp0, col0 = csr_from_expect(case["atoms"].shape[0], case["expect"])
    np.testing.assert_array_equal(rp.cpu().numpy(), rp0)
    np.testing.assert_array_equal(col.cpu().numpy(), col0)


def test_periodic_images_outside_the_box_give_the_same_list():
    d = DeviceInputs(3)
    rng = np.random.default_rng(0)
    shift = rng.integers(-3, 4, size=d.w.pos.shape).astype(np.float32) * d.w.box
    moved = torch.from_numpy(d.w.pos + shift).to(dev())
    rp, col = e2f.e2f_build_neighbors(moved, d.box, d.w.cutoff)
    rp0, col0 = oracle_csr(3)
    # the predicate's rint image choice is shift-invariant for pairs well inside rc
    from oracle.neighbors import neighbors_bruteforce
    rp1, col1 = neighbors_bruteforce(d.w.pos + shift, d.w.box, d.w.cutoff)
    np.testing.assert_array_equal(rp.cpu().numpy(), rp1)
    np.testing.assert_array_equal(col.cpu().numpy(), col1)
    assert abs(col1.size - col0.size) <= 8


def test_capacity_protocol_and_empty_inputs():
    d = DeviceInputs(1)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, d.w.cutoff, col_capacity=7)  # grows and retries
    rp0, col0 = oracle_csr(1)
    np.testing.assert_array_equal(col.cpu().numpy(), col0)
    empty = torch.zeros((0, 3), dtype=torch.float32, device=dev())
    rp, col = e2f.e2f_build_neighbors(empty, None, 5.0)
    assert rp.cpu().tolist() == [0] and col.numel() == 0
    one = torch.zeros((1, 3), dtype=torch.float32, device=dev())
    rp, col = e2f.e2f_build_neighbors(one, [10.0, 10.0, 10.0], 5.0)
    assert rp.cpu().tolist() == [0, 0] and col.numel() == 0


def test_nonfinite_positions_are_reported():
    pos = torch.zeros((5, 3), dtype=torch.float32, device=dev())
    pos[3, 1] = float("nan")
    with pytest.raises(e2f.E2FError) as ei:
        e2f.e2f_build_neighbors(pos, None, 2.0)
    assert ei.value.code == 7


def test_bad_graph_ptr_is_reported():
    pos = torch.zeros((5, 3), dtype=torch.float32, device=dev())
    gp = torch.tensor([0, 3, 2, 5], dtype=torch.int32, device=dev())
    with pytest.raises(e2f.E2FError) as ei:
        e2f.e2f_build_neighbors(pos, None, 2.0, gp)
    assert ei.value.code == 1


def test_small_boxes_with_few_cells_per_axis():
    # 3 to 11 half-width cells per axis: axes of fewer than five cells are
    # searched whole, larger ones with a stencil that wraps around the box
    rng = np.random.default_rng(3)
    from oracle.neighbors import neighbors_bruteforce
    for side, rc in [(10.0, 5.0), (10.5, 4.0), (7.0, 3.4), (13.0, 4.2)]:
        pos_np = rng.uniform(-side, 2 * side, size=(150, 3)).astype(np.float32)
        box = np.array([side, side * 1.3, side * 2.1], np.float32)
        rp, col = e2f.e2f_build_neighbors(torch.from_numpy(pos_np).to(dev()), box.tolist(), rc)
        rp0, col0 = neighbors_bruteforce(pos_np, box, rc)
        np.testing.assert_array_equal(rp.cpu().numpy(), rp0)
        np.testing.assert_array_equal(col.cpu().numpy(), col0)


def test_dense_rows_beyond_the_shared_memory_sort():
    # 1500 atoms inside a radius-2 ball with cutoff 5: every row has 1499
    # entries, more than the in-shared-memory sort holds
    rng = np.random.default_rng(4)
    v = rng.normal(size=(1500, 3))
    v = v / np.linalg.norm(v, axis=1, keepdims=True) * rng.uniform(0, 2, size=(1500, 1))
    pos_np = v.astype(np.float32)
    rp, col = e2f.e2f_build_neighbors(torch.from_numpy(pos_np).to(dev()), None, 5.0)
    from oracle.neighbors import neighbors_bruteforce
    rp0, col0 = neighbors_bruteforce(pos_np, None, 5.0)
    np.testing.assert_array_equal(rp.cpu().numpy(), rp0)
    np.testing.assert_array_equal(col.cpu().numpy(), col0)


@pytest.mark.parametrize("cfg", [2, 3])
def test_query_rows_equal_the_full_list_restricted(cfg):
    # rows of atoms 0 .. n_rows-1 only: those rows as in the full list (bit-exact, as the
    # oracle's), every later row empty; all atoms stay candidates
    d = DeviceInputs(cfg)
    rp0, col0 = oracle_csr(cfg)
    n = d.w.n_atoms
    for n_rows in (0, 1, n // 3, n):
        rp, col = e2f.e2f_build_neighbors(d.pos, d.box, d.w.cutoff, d.graph_ptr, rows=n_rows)
        rp, col = rp.cpu().numpy(), col.cpu().numpy()
        end = rp0[n_rows]
        np.testing.assert_array_equal(rp[:n_rows + 1], rp0[:n_rows + 1])
        assert (rp[n_rows:] == end).all()
        np.testing.assert_array_equal(col, col0[:end])
