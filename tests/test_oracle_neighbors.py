"""Pins for the oracle's neighbour search: hand-worked fixtures, brute force
against a KD-tree search, and the predicate's symmetry."""
import os

import numpy as np
import pytest

from oracle.neighbors import neighbors_bruteforce, neighbors_kdtree, predicate_f32
from workloads import load_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "neighbors_handmade.txt")


def parse_cases(path=GOLDEN):
    cases, cur, mode = [], None, None
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "case":
            cur = {"name": tok[1], "box": None, "graph_ptr": None, "atoms": [], "expect": {}}
            mode = None
        elif tok[0] == "box":
            cur["box"] = np.array([float(t) for t in tok[1:]], np.float32)
        elif tok[0] == "cutoff":
            cur["cutoff"] = float(tok[1])
        elif tok[0] == "graph_ptr":
            cur["graph_ptr"] = np.array([int(t) for t in tok[1:]], np.int32)
        elif tok[0] in ("atoms", "expect"):
            mode = tok[0]
        elif tok[0] == "end":
            cur["atoms"] = np.array(cur["atoms"], np.float32)
            cases.append(cur)
        elif mode == "atoms":
            cur["atoms"].append([float(t) for t in tok])
        elif mode == "expect":
            i = int(tok[0].rstrip(":"))
            cur["expect"][i] = [int(t) for t in tok[1:]]
    return cases


def csr_from_expect(n, expect):
    rp = np.zeros(n + 1, np.int32)
    cols = []
    for i in range(n):
        js = expect.get(i, [])
        rp[i + 1] = rp[i] + len(js)
        cols += js
    return rp, np.array(cols, np.int32)


@pytest.mark.parametrize("case", parse_cases(), ids=lambda c: c["name"])
def test_handmade_fixture(case):
    n = case["atoms"].shape[0]
    rp0, col0 = csr_from_expect(n, case["expect"])
    for fn in (neighbors_bruteforce, neighbors_kdtree):
        rp, col = fn(case["atoms"], case["box"], case["cutoff"], case["graph_ptr"])
        np.testing.assert_array_equal(rp, rp0)
        np.testing.assert_array_equal(col, col0)


def test_exactly_at_cutoff_is_excluded_and_just_inside_is_kept():
    p = np.array([[0, 0, 0], [2.0, 0, 0]], np.float32)
    assert not predicate_f32(p[0], p[1], None, 2.0)
    p[1, 0] = np.nextafter(np.float32(2.0), np.float32(0))
    assert predicate_f32(p[0], p[1], None, 2.0)


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_bruteforce_equals_kdtree_on_workloads(cfg):
    w = load_workload(cfg)
    a = neighbors_bruteforce(w.pos, w.box, w.cutoff, w.graph_ptr)
    b = neighbors_kdtree(w.pos, w.box, w.cutoff, w.graph_ptr)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    rp, col = a
    n = w.n_atoms
    rows = np.repeat(np.arange(n), np.diff(rp))
    assert np.all(rows != col)
    # symmetric: (i, j) present iff (j, i) present
    fwd = set(zip(rows.tolist(), col.tolist()))
    assert all((j, i) in fwd for (i, j) in fwd)
    # columns ascend within each row
    for i in range(0, n, max(1, n // 50)):
        seg = col[rp[i]:rp[i + 1]]
        assert np.all(np.diff(seg) > 0)
    if w.graph_ptr is not None:
        gid = np.repeat(np.arange(w.graph_ptr.size - 1), np.diff(w.graph_ptr))
        assert np.all(gid[rows] == gid[col])


def test_predicate_is_symmetric_under_swap():
    rng = np.random.default_rng(0)
    a = rng.uniform(0, 31.07, size=(2000, 3)).astype(np.float32)
    b = rng.uniform(0, 31.07, size=(2000, 3)).astype(np.float32)
    box = np.full(3, 31.07, np.float32)
    np.testing.assert_array_equal(predicate_f32(a, b, box, 6.0), predicate_f32(b, a, box, 6.0))
