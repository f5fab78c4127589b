"""GPU edge frames and Wigner-D blocks against the oracle's definition."""
import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f
from gpu_util import dev
from oracle.wigner import wigner_D

pytestmark = pytest.mark.gpu


def test_edge_frames_and_wigner_blocks():
    rng = np.random.default_rng(0)
    r = rng.normal(size=(64, 3))
    r[:4] = [[0, 0, 1], [0, 0, -2], [1e-7, 0, 1], [0, 3, 0]]
    L = 4
    out, fr = e2f.e2f_edge_wigner_blocks(torch.from_numpy(r.astype(np.float32)).to(dev()), L, with_frames=True)
    out, fr = out.cpu().numpy().astype(np.float64), fr.cpu().numpy().astype(np.float64)
    for e in range(r.shape[0]):
        R = fr[e]
        np.testing.assert_allclose(R @ R.T, np.eye(3), atol=2e-6)
        np.testing.assert_allclose(R @ (r[e] / np.linalg.norm(r[e])), [0, 0, 1], atol=2e-6)
        o = 0
        for l in range(L + 1):
            n = 2 * l + 1
            np.testing.assert_allclose(out[e, o:o + n * n].reshape(n, n), wigner_D(l, R), atol=1e-5)
            o += n * n
