"""The two profiling aids of the C-ABI: caller events around the main
tensor-core kernel, and the per-CTA role cycle counters."""
import os

import pytest
import torch

import atomistic_cell_list_b200 as e2f
from gpu_util import DeviceInputs

pytestmark = pytest.mark.gpu


def _call(d, cfg, rp, col, ws):
    return e2f.e2f_onfly_attention(cfg, d.pos, d.box, rp, col, d.x, d.Wq, d.Wk, d.Wrad, d.Wso2, workspace=ws)


def test_kernel_events_bracket_the_main_kernel():
    d = DeviceInputs(3)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    assert e2f.e2f_attention_uses_tensor_cores(cfg)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    ws = torch.empty(e2f.e2f_attention_workspace_size(w.n_atoms, col.numel(), cfg), dtype=torch.uint8,
                     device=d.pos.device)
    ref = _call(d, cfg, rp, col, ws)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    whole0, whole1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(); stop.record()  # materialise the events
    e2f.e2f_attention_set_kernel_events(start, stop)
    try:
        whole0.record()
        out = _call(d, cfg, rp, col, ws)
        whole1.record()
    finally:
        e2f.e2f_attention_set_kernel_events(None, None)
    torch.cuda.synchronize()
    ker, whole = start.elapsed_time(stop), whole0.elapsed_time(whole1)
    assert 0.0 < ker <= whole  # the main kernel alone, inside the whole call
    assert torch.equal(out, ref)  # recording events changes nothing


def test_debug_timers_count_every_tile():
    d = DeviceInputs(3)
    w = d.w
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(d.pos, d.box, w.cutoff, d.graph_ptr)
    ws = torch.empty(e2f.e2f_attention_workspace_size(w.n_atoms, col.numel(), cfg), dtype=torch.uint8,
                     device=d.pos.device)
    ref = _call(d, cfg, rp, col, ws)
    e2f.e2f_attention_set_debug(timers=True)
    try:
        out = _call(d, cfg, rp, col, ws)
    finally:
        e2f.e2f_attention_set_debug()
    t = e2f.e2f_attention_debug_timers(ws, w.n_atoms, cfg)
    tiles = int(t[:, 13].sum())
    # every 128-edge tile of every CTA is counted once: at least ceil(E / 128) tiles
    assert tiles >= (col.numel() + 127) // 128
    assert tiles <= (col.numel() + 127) // 128 + t.shape[0]  # at most one partial tile per CTA
    assert (t[:, 7] >= 0).all() and t[:, 7].max() > 0  # the MMA role ran and timed itself
    assert torch.equal(out, ref)  # the counters change nothing in the result
