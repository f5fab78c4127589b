"""Python binding of libe2f.so: a GPU cell-list neighbour build and the
on-the-fly equivariant attention forward of E2Former-V2, written for B200
(sm_100a).

This module only marshals arguments: every step of the computation runs in
the library's CUDA kernels. PyTorch supplies device memory and the current
stream. Functions carry the C entry points' names (see include/e2f.h); the
library must be built (``python -m atomistic_cell_list_b200.build``) and a
CUDA device must be present, otherwise the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libe2f.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "e2f.h")

E2F_OK = 0
STATUS_NAMES = {0: "E2F_OK", 1: "E2F_ERR_INVALID_ARG", 2: "E2F_ERR_UNSUPPORTED", 3: "E2F_ERR_CAPACITY",
                4: "E2F_ERR_ALIGNMENT", 5: "E2F_ERR_TIMEOUT", 6: "E2F_ERR_CUDA", 7: "E2F_ERR_NONFINITE",
                8: "E2F_ERR_STALE"}
E2F_F32, E2F_BF16 = 0, 1


class E2FError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


class e2f_attn_cfg(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int), ("C", ctypes.c_int), ("H", ctypes.c_int), ("n_rbf", ctypes.c_int),
                ("cutoff", ctypes.c_float), ("feat_dtype", ctypes.c_int), ("m_max", ctypes.c_int)]


class e2f_sixj_cfg(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int), ("Lf", ctypes.c_int), ("C", ctypes.c_int), ("H", ctypes.c_int),
                ("n_rbf", ctypes.c_int), ("cutoff", ctypes.c_float)]


_lib = None
_vp, _i64, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t

_SIGS = {
    "e2f_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "e2f_neighbors_workspace_size": (_sz, [_i64, _vp, ctypes.c_float, ctypes.c_int32]),
    "e2f_build_neighbors": (ctypes.c_int, [_vp, _i64, _vp, ctypes.c_float, _vp, ctypes.c_int32, _vp, _vp, _i64,
                                           ctypes.POINTER(_i64), _vp, _sz, _vp]),
    "e2f_build_neighbors_rows": (ctypes.c_int, [_vp, _i64, _i64, _vp, ctypes.c_float, _vp, ctypes.c_int32, _vp, _vp,
                                                _i64, ctypes.POINTER(_i64), _vp, _sz, _vp]),
    "e2f_build_neighbors_noalloc": (ctypes.c_int, [_vp, _i64, _vp, ctypes.c_float, _vp, ctypes.c_int32, _vp, _vp,
                                                   _i64, ctypes.POINTER(_i64), _vp]),
    "e2f_attention_workspace_size": (_sz, [_i64, _i64, ctypes.POINTER(e2f_attn_cfg)]),
    "e2f_onfly_attention": (ctypes.c_int, [ctypes.POINTER(e2f_attn_cfg), _vp, _i64, _vp, _vp, _vp, _i64, _vp, _vp,
                                           _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "e2f_attention_status": (ctypes.c_int, [_vp, _sz, _vp]),
    "e2f_attention_cells_workspace_size": (_sz, [_i64, _vp, ctypes.POINTER(e2f_attn_cfg)]),
    "e2f_onfly_attention_cells": (ctypes.c_int, [ctypes.POINTER(e2f_attn_cfg), _vp, _i64, _vp, _vp, _vp, _vp, _vp,
                                                 _vp, _vp, _vp, _sz, _vp]),
    "e2f_attention_cells_skin_workspace_size": (_sz, [_i64, _vp, ctypes.POINTER(e2f_attn_cfg), ctypes.c_float]),
    "e2f_onfly_attention_cells_skin": (ctypes.c_int, [ctypes.POINTER(e2f_attn_cfg), _vp, _i64, _vp, ctypes.c_float,
                                                      ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "e2f_attention_backward_workspace_size": (_sz, [_i64, _i64, ctypes.POINTER(e2f_attn_cfg)]),
    "e2f_onfly_attention_backward": (ctypes.c_int, [ctypes.POINTER(e2f_attn_cfg), _vp, _i64, _vp, _vp, _vp, _i64,
                                                    _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                    _vp, _sz, _vp]),
    "e2f_edge_wigner_blocks": (ctypes.c_int, [_vp, _i64, ctypes.c_int, _vp, _vp, _vp]),
    "e2f_launch_count": (_i64, []),
    "e2f_attention_uses_tensor_cores": (ctypes.c_int, [ctypes.POINTER(e2f_attn_cfg)]),
    "e2f_attention_set_kernel_events": (None, [_vp, _vp]),
    "e2f_attention_set_debug": (None, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "e2f_attention_debug_timers": (ctypes.c_int, [_vp, _sz, _i64, ctypes.POINTER(e2f_attn_cfg),
                                                  ctypes.POINTER(_i64), ctypes.c_int, _vp]),
    "e2f_sixj_n_paths": (ctypes.c_int, [ctypes.c_int, ctypes.c_int]),
    "e2f_sixj_workspace_size": (_sz, [_i64, ctypes.POINTER(e2f_sixj_cfg)]),
    "e2f_sixj_attention": (ctypes.c_int, [ctypes.POINTER(e2f_sixj_cfg), _vp, _i64, _vp, ctypes.c_int32, _vp, _vp,
                                          _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
}


def lib() -> ctypes.CDLL:
    """Load libe2f.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m atomistic_cell_list_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype, f.argtypes = res, args
        _lib = h
    return _lib


def header_symbols(path: str = HEADER) -> list[str]:
    """Names of the functions include/e2f.h declares."""
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(e2f_[a-z0-9_]+)\s*\(", src)))


def status_string(code: int) -> str:
    return lib().e2f_status_string(int(code)).decode()


def e2f_status_string(code: int) -> str:
    return status_string(code)


def _check(code: int, where: str):
    if code != E2F_OK:
        raise E2FError(code, where)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _box_arg(box):
    if box is None:
        return None, None
    arr = (ctypes.c_float * 3)(*[float(v) for v in box])
    return ctypes.cast(arr, ctypes.c_void_p), arr


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def e2f_neighbors_workspace_size(n_atoms: int, box, cutoff: float, n_graphs: int = 1) -> int:
    b, keep = _box_arg(box)
    return int(lib().e2f_neighbors_workspace_size(int(n_atoms), b, float(cutoff), int(n_graphs)))


def e2f_build_neighbors(pos: torch.Tensor, box, cutoff: float, graph_ptr: torch.Tensor | None = None,
                        col_capacity: int | None = None, stream=None, rows: int | None = None):
    """CSR neighbour list (row_ptr int32 [N+1], col int32 [E]) by the GPU cell list; with
    rows = n, only the rows of atoms 0 .. n-1 (e2f_build_neighbors_rows)."""
    _need_cuda(pos, graph_ptr)
    assert pos.dtype == torch.float32 and pos.dim() == 2 and pos.shape[1] == 3
    n = pos.shape[0]
    n_graphs = 1 if graph_ptr is None else graph_ptr.numel() - 1
    dev = pos.device
    ws_bytes = e2f_neighbors_workspace_size(n, box, cutoff, n_graphs)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    row_ptr = torch.empty(n + 1, dtype=torch.int32, device=dev)
    cap = int(col_capacity) if col_capacity is not None else max(1024, 128 * n)
    b, keep = _box_arg(box)
    for _ in range(2):
        col = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
        npairs = ctypes.c_int64(0)
        if rows is None:
            code = lib().e2f_build_neighbors(_ptr(pos), n, b, float(cutoff), _ptr(graph_ptr), n_graphs,
                                             _ptr(row_ptr), _ptr(col), cap, ctypes.byref(npairs), _ptr(ws),
                                             ws_bytes, _stream(stream))
        else:
            code = lib().e2f_build_neighbors_rows(_ptr(pos), n, int(rows), b, float(cutoff), _ptr(graph_ptr),
                                                  n_graphs, _ptr(row_ptr), _ptr(col), cap, ctypes.byref(npairs),
                                                  _ptr(ws), ws_bytes, _stream(stream))
        if code == 3:  # capacity: grow to the exact size and retry
            cap = int(npairs.value)
            continue
        _check(code, "e2f_build_neighbors")
        return row_ptr, col[: npairs.value]
    raise E2FError(3, "e2f_build_neighbors")


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def e2f_build_neighbors_noalloc(pos: torch.Tensor, box, cutoff: float, graph_ptr: torch.Tensor | None = None,
                                row_ptr: torch.Tensor | None = None, col: torch.Tensor | None = None,
                                stream=None):
    """CSR neighbour list built in the library's static scratch (no workspace).

    row_ptr / col may be passed in (int32, [N+1] and [capacity]); the call
    then writes them and returns (row_ptr, col[:E]). With col=None a buffer
    of 128 N entries is made here, grown once on E2F_ERR_CAPACITY.
    """
    _need_cuda(pos, graph_ptr, row_ptr, col)
    assert pos.dtype == torch.float32 and pos.dim() == 2 and pos.shape[1] == 3
    n = pos.shape[0]
    n_graphs = 1 if graph_ptr is None else graph_ptr.numel() - 1
    if row_ptr is None:
        row_ptr = torch.empty(n + 1, dtype=torch.int32, device=pos.device)
    given = col is not None
    if col is None:
        col = torch.empty(max(1024, 128 * n), dtype=torch.int32, device=pos.device)
    b, keep = _box_arg(box)
    for _ in range(2):
        npairs = ctypes.c_int64(0)
        code = lib().e2f_build_neighbors_noalloc(_ptr(pos), n, b, float(cutoff), _ptr(graph_ptr), n_graphs,
                                                 _ptr(row_ptr), _ptr(col), col.numel(), ctypes.byref(npairs),
                                                 _stream(stream))
        if code == 3 and not given:
            col = torch.empty(int(npairs.value), dtype=torch.int32, device=pos.device)
            continue
        _check(code, "e2f_build_neighbors_noalloc")
        return row_ptr, col[: npairs.value]
    raise E2FError(3, "e2f_build_neighbors_noalloc")


def make_cfg(L: int, C: int, H: int, n_rbf: int, cutoff: float, dtype: str, m_max: int = -1) -> e2f_attn_cfg:
    """m_max: SO(2) truncation order (-1 = full layer; W_so2 then holds blocks m <= m_max only)."""
    return e2f_attn_cfg(L, C, H, n_rbf, float(cutoff), E2F_BF16 if dtype == "bf16" else E2F_F32, int(m_max))


def e2f_attention_workspace_size(n_atoms: int, n_pairs: int, cfg: e2f_attn_cfg) -> int:
    return int(lib().e2f_attention_workspace_size(int(n_atoms), int(n_pairs), ctypes.byref(cfg)))


def e2f_onfly_attention(cfg: e2f_attn_cfg, pos, box, row_ptr, col, x, W_q, W_k, W_rad, W_so2,
                        out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                        stream=None, check: bool = True) -> torch.Tensor:
    """out[N, (L+1)^2, C] fp32 = on-the-fly equivariant attention (see include/e2f.h)."""
    _need_cuda(pos, row_ptr, col, x, W_q, W_k, W_rad, W_so2, out, workspace)
    n = pos.shape[0]
    K = (cfg.L + 1) ** 2
    if out is None:
        out = torch.empty((n, K, cfg.C), dtype=torch.float32, device=pos.device)
    ws_bytes = e2f_attention_workspace_size(n, col.numel(), cfg)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=pos.device)
    b, keep = _box_arg(box)
    s = _stream(stream)
    code = lib().e2f_onfly_attention(ctypes.byref(cfg), _ptr(pos), n, b, _ptr(row_ptr), _ptr(col), col.numel(),
                                     _ptr(x), _ptr(W_q), _ptr(W_k), _ptr(W_rad), _ptr(W_so2), _ptr(out),
                                     _ptr(workspace), workspace.numel(), s)
    _check(code, "e2f_onfly_attention")
    if check:
        _check(lib().e2f_attention_status(_ptr(workspace), workspace.numel(), s), "e2f_onfly_attention (device)")
    return out


def e2f_attention_cells_workspace_size(n_atoms: int, box, cfg: e2f_attn_cfg) -> int:
    b, keep = _box_arg(box)
    return int(lib().e2f_attention_cells_workspace_size(int(n_atoms), b, ctypes.byref(cfg)))


def e2f_onfly_attention_cells(cfg: e2f_attn_cfg, pos, box, x, W_q, W_k, W_rad, W_so2,
                              out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                              stream=None, check: bool = True) -> torch.Tensor:
    """The attention with the cell-list traversal fused in: no neighbour list (see include/e2f.h)."""
    _need_cuda(pos, x, W_q, W_k, W_rad, W_so2, out, workspace)
    n = pos.shape[0]
    if out is None:
        out = torch.empty((n, (cfg.L + 1) ** 2, cfg.C), dtype=torch.float32, device=pos.device)
    ws_bytes = e2f_attention_cells_workspace_size(n, box, cfg)
    if ws_bytes == 0:
        raise E2FError(2, "e2f_onfly_attention_cells")
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=pos.device)
    b, keep = _box_arg(box)
    s = _stream(stream)
    code = lib().e2f_onfly_attention_cells(ctypes.byref(cfg), _ptr(pos), n, b, _ptr(x), _ptr(W_q), _ptr(W_k),
                                           _ptr(W_rad), _ptr(W_so2), _ptr(out), _ptr(workspace),
                                           workspace.numel(), s)
    _check(code, "e2f_onfly_attention_cells")
    if check:
        _check(lib().e2f_attention_status(_ptr(workspace), workspace.numel(), s),
               "e2f_onfly_attention_cells (device)")
    return out


def e2f_attention_cells_skin_workspace_size(n_atoms: int, box, cfg: e2f_attn_cfg, skin: float) -> int:
    b, keep = _box_arg(box)
    return int(lib().e2f_attention_cells_skin_workspace_size(int(n_atoms), b, ctypes.byref(cfg), float(skin)))


def e2f_onfly_attention_cells_skin(cfg: e2f_attn_cfg, pos, box, skin: float, rebuild: bool, x, W_q, W_k, W_rad,
                                   W_so2, workspace: torch.Tensor, out: torch.Tensor | None = None, stream=None,
                                   check: bool = True) -> torch.Tensor:
    """The fused attention with Verlet-skin reuse of the cell lists held in
    `workspace` (see include/e2f.h). With check, a stale reuse raises
    E2FError(E2F_ERR_STALE); the caller then calls again with rebuild=True."""
    _need_cuda(pos, x, W_q, W_k, W_rad, W_so2, out, workspace)
    n = pos.shape[0]
    if out is None:
        out = torch.empty((n, (cfg.L + 1) ** 2, cfg.C), dtype=torch.float32, device=pos.device)
    ws_bytes = e2f_attention_cells_skin_workspace_size(n, box, cfg, skin)
    if ws_bytes == 0:
        raise E2FError(2, "e2f_onfly_attention_cells_skin")
    if workspace.numel() < ws_bytes:
        raise E2FError(1, "e2f_onfly_attention_cells_skin: workspace too small")
    b, keep = _box_arg(box)
    s = _stream(stream)
    code = lib().e2f_onfly_attention_cells_skin(ctypes.byref(cfg), _ptr(pos), n, b, float(skin), int(bool(rebuild)),
                                                _ptr(x), _ptr(W_q), _ptr(W_k), _ptr(W_rad), _ptr(W_so2), _ptr(out),
                                                _ptr(workspace), workspace.numel(), s)
    _check(code, "e2f_onfly_attention_cells_skin")
    if check:
        _check(lib().e2f_attention_status(_ptr(workspace), workspace.numel(), s),
               "e2f_onfly_attention_cells_skin (device)")
    return out


def e2f_attention_backward_workspace_size(n_atoms: int, n_pairs: int, cfg: e2f_attn_cfg) -> int:
    return int(lib().e2f_attention_backward_workspace_size(int(n_atoms), int(n_pairs), ctypes.byref(cfg)))


def e2f_onfly_attention_backward(cfg: e2f_attn_cfg, pos, box, row_ptr, col, x, W_q, W_k, W_rad, W_so2, grad_out,
                                 want_weights: bool = True, workspace: torch.Tensor | None = None,
                                 out: dict | None = None, stream=None, check: bool = True) -> dict:
    """Gradients of sum(grad_out * layer(...)) (see include/e2f.h): a dict with
    pos, x, W_rad and, when want_weights, W_q, W_k, W_so2 (all fp32)."""
    _need_cuda(pos, row_ptr, col, x, W_q, W_k, W_rad, W_so2, grad_out, workspace)
    n = pos.shape[0]
    dev = pos.device
    f32 = torch.float32
    g = dict(out) if out is not None else {}
    g.setdefault("pos", torch.empty((n, 3), dtype=f32, device=dev))
    g.setdefault("x", torch.empty(x.shape, dtype=f32, device=dev))
    g.setdefault("W_rad", torch.empty(W_rad.shape, dtype=f32, device=dev))
    if want_weights:
        g.setdefault("W_q", torch.empty(W_q.shape, dtype=f32, device=dev))
        g.setdefault("W_k", torch.empty(W_k.shape, dtype=f32, device=dev))
        g.setdefault("W_so2", torch.empty(W_so2.shape, dtype=f32, device=dev))
    ws_bytes = e2f_attention_backward_workspace_size(n, col.numel(), cfg)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    b, keep = _box_arg(box)
    code = lib().e2f_onfly_attention_backward(
        ctypes.byref(cfg), _ptr(pos), n, b, _ptr(row_ptr), _ptr(col), col.numel(), _ptr(x), _ptr(W_q), _ptr(W_k),
        _ptr(W_rad), _ptr(W_so2), _ptr(grad_out), _ptr(g["pos"]), _ptr(g["x"]), _ptr(g.get("W_q")),
        _ptr(g.get("W_k")), _ptr(g["W_rad"]), _ptr(g.get("W_so2")), _ptr(workspace), workspace.numel(),
        _stream(stream))
    _check(code, "e2f_onfly_attention_backward")
    if check:
        _check(lib().e2f_attention_status(_ptr(workspace), workspace.numel(), _stream(stream)),
               "e2f_onfly_attention_backward (device)")
    return g


def e2f_attention_status(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().e2f_attention_status(_ptr(workspace), workspace.numel(), _stream(stream)))


def e2f_edge_wigner_blocks(r: torch.Tensor, L: int, with_frames: bool = False, stream=None):
    _need_cuda(r)
    n = r.shape[0]
    S = sum((2 * l + 1) ** 2 for l in range(L + 1))
    out = torch.empty((n, S), dtype=torch.float32, device=r.device)
    fr = torch.empty((n, 3, 3), dtype=torch.float32, device=r.device) if with_frames else None
    _check(lib().e2f_edge_wigner_blocks(_ptr(r), n, int(L), _ptr(out), _ptr(fr), _stream(stream)),
           "e2f_edge_wigner_blocks")
    return (out, fr) if with_frames else out


def e2f_attention_uses_tensor_cores(cfg: e2f_attn_cfg) -> bool:
    return bool(lib().e2f_attention_uses_tensor_cores(ctypes.byref(cfg)))


DEBUG_SLOTS = 32


def e2f_attention_debug_timers(workspace: torch.Tensor, n_atoms: int, cfg: e2f_attn_cfg, n_ctas: int = 160,
                               stream=None):
    """Per-CTA role cycle counters of the last tensor-core call (timers on: e2f_attention_set_debug)."""
    import numpy as np
    n = DEBUG_SLOTS * n_ctas
    buf = (_i64 * n)()
    _check(lib().e2f_attention_debug_timers(_ptr(workspace), workspace.numel(), int(n_atoms), ctypes.byref(cfg), buf,
                                            n, _stream(stream)), "e2f_attention_debug_timers")
    return np.frombuffer(buf, dtype=np.int64).reshape(n_ctas, DEBUG_SLOTS).copy()


def e2f_attention_set_kernel_events(start=None, stop=None):
    """Record torch.cuda.Event pair around the next calls' main kernel (None, None: off)."""
    a = None if start is None else ctypes.c_void_p(start.cuda_event)
    b = None if stop is None else ctypes.c_void_p(stop.cuda_event)
    lib().e2f_attention_set_kernel_events(a, b)


def e2f_attention_set_debug(max_ctas: int = 0, timers: bool = False, drop_arrive: bool = False):
    """Debug and test controls of the tensor-core kernel (process-wide; all off restores the default)."""
    lib().e2f_attention_set_debug(int(max_ctas), int(bool(timers)), int(bool(drop_arrive)))


def e2f_launch_count() -> int:
    return int(lib().e2f_launch_count())


def make_sixj_cfg(L: int, Lf: int, C: int, H: int, n_rbf: int, cutoff: float) -> e2f_sixj_cfg:
    return e2f_sixj_cfg(int(L), int(Lf), int(C), int(H), int(n_rbf), float(cutoff))


def e2f_sixj_n_paths(L: int, Lf: int) -> int:
    return int(lib().e2f_sixj_n_paths(int(L), int(Lf)))


def e2f_sixj_workspace_size(n_atoms: int, cfg: e2f_sixj_cfg) -> int:
    return int(lib().e2f_sixj_workspace_size(int(n_atoms), ctypes.byref(cfg)))


def e2f_sixj_attention(cfg: e2f_sixj_cfg, pos, row_ptr, col, x, W_q, W_k, W_rad, w_path,
                       graph_ptr: torch.Tensor | None = None, out: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[N, (L+1)^2, C] fp32 = the Wigner-6j node-level convolution layer (see include/e2f.h)."""
    _need_cuda(pos, row_ptr, col, x, W_q, W_k, W_rad, w_path, graph_ptr, out, workspace)
    n = pos.shape[0]
    if out is None:
        out = torch.empty((n, (cfg.L + 1) ** 2, cfg.C), dtype=torch.float32, device=pos.device)
    ws_bytes = e2f_sixj_workspace_size(n, cfg)
    if ws_bytes == 0:
        raise E2FError(2, "e2f_sixj_workspace_size")
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=pos.device)
    n_graphs = 0 if graph_ptr is None else graph_ptr.numel() - 1
    code = lib().e2f_sixj_attention(ctypes.byref(cfg), _ptr(pos), n, _ptr(graph_ptr), n_graphs, _ptr(row_ptr),
                                    _ptr(col), col.numel(), _ptr(x), _ptr(W_q), _ptr(W_k), _ptr(W_rad),
                                    _ptr(w_path), _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "e2f_sixj_attention")
    return out


# short aliases
build_neighbors = e2f_build_neighbors
onfly_attention = e2f_onfly_attention
edge_wigner_blocks = e2f_edge_wigner_blocks
