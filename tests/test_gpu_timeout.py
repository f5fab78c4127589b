"""The bounded device-side waits of the tensor-core kernel: a withheld
producer arrival (a flag that nothing sets, through the test hook of
e2f_attention_set_debug) makes CTA 0's waits run out. The call must report
E2F_ERR_TIMEOUT through the workspace status word without hanging, and the
next normal call on the same workspace must succeed with the usual result.
No fault and no endless wait is involved: every wait ends by its own limit."""
import time

import pytest
import torch

import atomistic_cell_list_b200 as e2f
from gpu_util import DeviceInputs

pytestmark = pytest.mark.gpu

E2F_ERR_TIMEOUT = 5


def _call(d, cfg, rp, col, ws, check=True):
    return e2f.e2f_onfly_attention(cfg, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2, workspace=ws,
                                   check=check)


@pytest.mark.parametrize("max_ctas", [0, 8])
def test_withheld_arrival_times_out_and_the_next_call_is_normal(max_ctas):
    d = DeviceInputs(3)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    assert e2f.e2f_attention_uses_tensor_cores(cfg)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    ws = torch.empty(e2f.e2f_attention_workspace_size(w.n_atoms, col.numel(), cfg), dtype=torch.uint8,
                     device=d.pos.device)
    ref = _call(d, cfg, rp, col, ws)
    assert e2f.e2f_attention_status(ws) == 0
    # 0: one CTA per SM (CTA 0 has one or two tiles); 8: CTA 0 walks many tiles, so its
    # producer runs ahead and then waits for a buffer that is never released
    e2f.e2f_attention_set_debug(max_ctas=max_ctas, drop_arrive=True)
    try:
        t0 = time.time()
        _call(d, cfg, rp, col, ws, check=False)
        torch.cuda.synchronize()
        elapsed = time.time() - t0
    finally:
        e2f.e2f_attention_set_debug()
    assert e2f.e2f_attention_status(ws) == E2F_ERR_TIMEOUT
    assert elapsed < 30.0  # the waits ended by their limit (2 s each, the first expiry aborts the rest)
    again = _call(d, cfg, rp, col, ws)  # raises if the status word is not cleared or the call fails
    assert torch.equal(again, ref)
