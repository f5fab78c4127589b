"""Neighbour build in the library's static scratch (e2f_build_neighbors_noalloc).

Kept in a file collected last so that it also runs after every other test
has used the device. Each call is compared bit for bit with the workspace
entry point, e2f_build_neighbors, on the same inputs.
"""
import ctypes

import numpy as np
import pytest
import torch

import atomistic_cell_list_b200 as e2f


def _same(a, b):
    np.testing.assert_array_equal(a[0].cpu().numpy(), b[0].cpu().numpy())
    np.testing.assert_array_equal(a[1].cpu().numpy(), b[1].cpu().numpy())


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_two_calls_in_a_row_match_the_workspace_build(cfg):
    from gpu_util import DeviceInputs
    d = DeviceInputs(cfg)
    ref = e2f.e2f_build_neighbors(d.pos, d.box, d.w.cutoff, d.graph_ptr)
    n = d.pos.shape[0]
    for _ in range(2):  # the second call finds the first one's leftovers in the scratch
        rp = torch.full((n + 1,), -1, dtype=torch.int32, device=d.pos.device)
        col = torch.full((ref[1].numel() + 5,), -1, dtype=torch.int32, device=d.pos.device)
        got = e2f.e2f_build_neighbors_noalloc(d.pos, d.box, d.w.cutoff, d.graph_ptr, row_ptr=rp, col=col)
        _same(got, ref)


@pytest.mark.gpu
def test_alternating_problem_sizes_and_empty_input():
    from gpu_util import DeviceInputs
    small, large = DeviceInputs(1), DeviceInputs(3)
    ref_s = e2f.e2f_build_neighbors(small.pos, small.box, small.w.cutoff, small.graph_ptr)
    ref_l = e2f.e2f_build_neighbors(large.pos, large.box, large.w.cutoff, large.graph_ptr)
    for d, ref in [(large, ref_l), (small, ref_s), (large, ref_l)]:
        _same(e2f.e2f_build_neighbors_noalloc(d.pos, d.box, d.w.cutoff, d.graph_ptr), ref)
    empty = torch.zeros((0, 3), dtype=torch.float32, device=small.pos.device)
    rp, col = e2f.e2f_build_neighbors_noalloc(empty, None, 5.0)
    assert rp.cpu().tolist() == [0] and col.numel() == 0


@pytest.mark.gpu
def test_capacity_protocol():
    from gpu_util import DeviceInputs
    d = DeviceInputs(1)
    ref = e2f.e2f_build_neighbors(d.pos, d.box, d.w.cutoff, d.graph_ptr)
    small = torch.empty(3, dtype=torch.int32, device=d.pos.device)
    with pytest.raises(e2f.E2FError) as ei:
        e2f.e2f_build_neighbors_noalloc(d.pos, d.box, d.w.cutoff, d.graph_ptr, col=small)
    assert ei.value.code == 3
    _same(e2f.e2f_build_neighbors_noalloc(d.pos, d.box, d.w.cutoff, d.graph_ptr), ref)


def test_problems_beyond_the_scratch_are_refused_before_any_work():
    lib = e2f.lib()
    n = 10 ** 6  # needs about 40 MB of scratch with open boundaries
    assert e2f.e2f_neighbors_workspace_size(n, None, 6.0) > e2f.NOALLOC_SCRATCH_BYTES
    npairs = ctypes.c_int64(-7)
    code = lib.e2f_build_neighbors_noalloc(None, n, None, 6.0, None, 1, None, None, 0, ctypes.byref(npairs), None)
    assert code == 2 and npairs.value == -7  # E2F_ERR_UNSUPPORTED, nothing written
    code = lib.e2f_build_neighbors_noalloc(None, -1, None, 6.0, None, 1, None, None, 0, ctypes.byref(npairs), None)
    assert code == 1


@pytest.mark.gpu
def test_calls_allocate_no_device_memory():
    """With its outputs passed in, the call takes no device memory: neither
    torch's caching allocator nor the device's free memory changes across
    several calls and a synchronisation. The first calls run before the
    measurement, because loading the module places its static scratch."""
    from gpu_util import DeviceInputs
    d = DeviceInputs(3)
    ref = e2f.e2f_build_neighbors(d.pos, d.box, d.w.cutoff, d.graph_ptr)
    n = d.pos.shape[0]
    rp = torch.empty(n + 1, dtype=torch.int32, device=d.pos.device)
    col = torch.empty(ref[1].numel() + 16, dtype=torch.int32, device=d.pos.device)
    for _ in range(2):
        e2f.e2f_build_neighbors_noalloc(d.pos, d.box, d.w.cutoff, d.graph_ptr, row_ptr=rp, col=col)
    torch.cuda.synchronize()
    stats0 = torch.cuda.memory_stats()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        got = e2f.e2f_build_neighbors_noalloc(d.pos, d.box, d.w.cutoff, d.graph_ptr, row_ptr=rp, col=col)
    torch.cuda.synchronize()
    stats1 = torch.cuda.memory_stats()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    for key in ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current",
                "allocated_bytes.all.current"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key
    _same(got, ref)
