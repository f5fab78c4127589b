"""CPU checks of the C-ABI boundary: the library loads, exports every symbol
include/e2f.h declares, and rejects bad arguments before touching a GPU."""
import ctypes

import pytest

import atomistic_cell_list_b200 as e2f


def test_library_exports_every_declared_symbol():
    h = e2f.lib()
    syms = e2f.header_symbols()
    assert {"e2f_build_neighbors", "e2f_onfly_attention", "e2f_neighbors_workspace_size",
            "e2f_attention_workspace_size", "e2f_status_string"} <= set(syms)
    for s in syms:
        assert hasattr(h, s), s


def test_status_strings():
    for code in range(8):
        assert e2f.status_string(code) and e2f.status_string(code) != "unknown status"
    assert e2f.status_string(99) == "unknown status"


def test_workspace_queries_are_host_only():
    cfg = e2f.make_cfg(4, 128, 8, 16, 6.0, "bf16")
    assert e2f.e2f_attention_workspace_size(30000, 2_700_000, cfg) > 0
    assert e2f.e2f_neighbors_workspace_size(30000, [66.9, 66.9, 66.9], 6.0) > 0
    assert e2f.e2f_neighbors_workspace_size(10000, None, 5.0, 256) > 0
    bad = e2f.make_cfg(5, 128, 8, 16, 6.0, "bf16")
    assert e2f.e2f_attention_workspace_size(10, 10, bad) == 0
    assert e2f.e2f_attention_workspace_size(10, 10, e2f.make_cfg(2, 16, 1, 16, 5.0, "f32", m_max=-2)) == 0
    # the fp32 path keeps a repacked copy of the SO(2) weights: a truncated layer needs less
    full = e2f.e2f_attention_workspace_size(64, 1000, e2f.make_cfg(2, 16, 1, 16, 5.0, "f32"))
    trunc = e2f.e2f_attention_workspace_size(64, 1000, e2f.make_cfg(2, 16, 1, 16, 5.0, "f32", m_max=0))
    assert 0 < trunc < full


def _attn(cfg, **kw):
    a = dict(pos=1, n=4, box=None, rp=1, col=1, npairs=4, x=16, wq=1, wk=1, wr=16, ws=16, out=16, wsp=256,
             wsb=1 << 20)
    a.update(kw)
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    return e2f.lib().e2f_onfly_attention(ctypes.byref(cfg), v(a["pos"]), a["n"], a["box"], v(a["rp"]), v(a["col"]),
                                         a["npairs"], v(a["x"]), v(a["wq"]), v(a["wk"]), v(a["wr"]), v(a["ws"]),
                                         v(a["out"]), v(a["wsp"]), a["wsb"], None)


@pytest.mark.parametrize("L,C,H,nr,code", [(5, 128, 8, 16, 2), (4, 120, 8, 16, 2), (4, 128, 3, 16, 2),
                                           (4, 512, 8, 16, 2), (4, 128, 8, 1, 2), (4, 128, 8, 64, 2),
                                           (-1, 128, 8, 16, 1), (4, 0, 8, 16, 1)])
def test_attention_rejects_unsupported_shapes(L, C, H, nr, code):
    cfg = e2f.e2f_attn_cfg(L, C, H, nr, 6.0, e2f.E2F_BF16)
    assert _attn(cfg) == code


def test_attention_argument_checks():
    cfg = e2f.make_cfg(2, 16, 1, 16, 5.0, "f32")
    assert _attn(cfg, pos=None) == 1
    assert _attn(cfg, npairs=-1) == 1
    assert _attn(cfg, x=8) == 4            # x not 16-byte aligned
    assert _attn(cfg, wsp=128) == 4        # workspace not 256-byte aligned
    assert _attn(cfg, wsb=16) == 1         # workspace too small
    box = (ctypes.c_float * 3)(8.0, 8.0, 8.0)
    assert _attn(cfg, box=ctypes.cast(box, ctypes.c_void_p)) == 1   # cutoff > box/2
    bad_dtype = e2f.e2f_attn_cfg(2, 16, 1, 16, 5.0, 7)
    assert _attn(bad_dtype) == 2
    assert _attn(cfg, n=0) == 0            # nothing to do


def test_neighbor_argument_checks():
    f = e2f.lib().e2f_build_neighbors
    n = ctypes.c_int64(0)
    vp = ctypes.c_void_p
    assert f(vp(16), 4, None, 5.0, None, 1, vp(16), vp(16), 10, None, vp(256), 1 << 20, None) == 1
    assert f(vp(16), 4, None, -1.0, None, 1, vp(16), vp(16), 10, ctypes.byref(n), vp(256), 1 << 20, None) == 1
    assert f(vp(16), -4, None, 5.0, None, 1, vp(16), vp(16), 10, ctypes.byref(n), vp(256), 1 << 20, None) == 1
    box = (ctypes.c_float * 3)(9.0, 20.0, 20.0)
    assert f(vp(16), 4, ctypes.cast(box, vp), 5.0, None, 1, vp(16), vp(16), 10, ctypes.byref(n), vp(256), 1 << 20,
             None) == 1
    assert f(vp(16), 4, None, 5.0, None, 1, vp(16), vp(16), 10, ctypes.byref(n), vp(128), 1 << 20, None) == 4
    assert f(vp(16), 4, None, 5.0, vp(16), 0, vp(16), vp(16), 10, ctypes.byref(n), vp(256), 1 << 20, None) == 1
    assert f(vp(16), 4, None, 5.0, None, 1, vp(16), vp(16), 10, ctypes.byref(n), vp(256), 16, None) == 1
    g = e2f.lib().e2f_build_neighbors_rows  # query rows outside 0 .. n_atoms
    assert g(vp(16), 4, 5, None, 5.0, None, 1, vp(16), vp(16), 10, ctypes.byref(n), vp(256), 1 << 20, None) == 1
    assert g(vp(16), 4, -1, None, 5.0, None, 1, vp(16), vp(16), 10, ctypes.byref(n), vp(256), 1 << 20, None) == 1


def test_wigner_entry_checks():
    f = e2f.lib().e2f_edge_wigner_blocks
    assert f(ctypes.c_void_p(16), 4, 5, ctypes.c_void_p(16), None, None) == 2
    assert f(None, 4, 2, ctypes.c_void_p(16), None, None) == 1
    assert f(None, 0, 2, None, None, None) == 0


def test_tensor_core_dispatch_rule():
    uses = lambda *a: e2f.e2f_attention_uses_tensor_cores(e2f.make_cfg(*a))
    assert uses(4, 128, 8, 16, 6.0, "bf16")
    assert uses(2, 256, 16, 16, 6.0, "bf16")
    assert not uses(4, 128, 8, 16, 6.0, "f32")      # fp32 features: CUDA-core kernel
    assert uses(4, 64, 8, 16, 5.0, "bf16")          # C = 64: two degrees per 128-row block
    assert not uses(4, 96, 8, 16, 5.0, "bf16")      # C neither 64 nor a multiple of 128
    assert not uses(2, 16, 1, 16, 5.0, "bf16")
    assert not uses(0, 128, 8, 16, 5.0, "bf16")
    assert not uses(4, 128, 2, 16, 5.0, "bf16")     # H not a multiple of 4


def _bwd(cfg, **kw):
    a = dict(pos=16, n=4, box=None, rp=16, col=16, npairs=4, x=16, wq=16, wk=16, wr=16, ws=16, gout=16, gpos=16,
             gx=16, gwq=16, gwk=16, gwr=16, gws=16, wsp=256, wsb=1 << 24)
    a.update(kw)
    v = lambda p: None if p is None else ctypes.c_void_p(p)
    return e2f.lib().e2f_onfly_attention_backward(
        ctypes.byref(cfg), v(a["pos"]), a["n"], a["box"], v(a["rp"]), v(a["col"]), a["npairs"], v(a["x"]), v(a["wq"]),
        v(a["wk"]), v(a["wr"]), v(a["ws"]), v(a["gout"]), v(a["gpos"]), v(a["gx"]), v(a["gwq"]), v(a["gwk"]),
        v(a["gwr"]), v(a["gws"]), v(a["wsp"]), a["wsb"], None)


def test_backward_workspace_and_argument_checks():
    bf = e2f.make_cfg(4, 128, 8, 16, 6.0, "bf16")
    f32 = e2f.make_cfg(4, 128, 8, 16, 6.0, "f32")
    # an edge adds one float per head; with bf16 storage it also adds its two fp16 operand rows of the
    # weight gradient ((L+1)^2 C halves each), up to a chunk of 131072 edges, beyond which only the floats grow
    ws = e2f.e2f_attention_backward_workspace_size
    assert ws(100, 1000, bf) > 0 and ws(100, 1000, f32) > 0
    assert ws(100, 2000, f32) - ws(100, 1000, f32) >= 4 * 8 * 1000
    assert ws(100, 2000, bf) - ws(100, 1000, bf) >= 4 * 8 * 1000 + 2 * 2 * 25 * 128 * 1000
    assert ws(100, 400000, bf) - ws(100, 200000, bf) < 4 * 8 * 200000 + 4096
    assert e2f.e2f_attention_backward_workspace_size(100, 1000, e2f.make_cfg(5, 128, 8, 16, 6.0, "bf16")) == 0
    cfg = e2f.make_cfg(2, 16, 1, 16, 5.0, "f32")
    assert _bwd(cfg, gout=None) == 1
    assert _bwd(cfg, gpos=None) == 1
    assert _bwd(cfg, gx=8) == 4            # grad_x not 16-byte aligned
    assert _bwd(cfg, wsp=128) == 4
    assert _bwd(cfg, wsb=16) == 1
    assert _bwd(cfg, npairs=-1) == 1
    assert _bwd(cfg, n=0) == 0
    assert _bwd(e2f.make_cfg(2, 48, 3, 16, 5.0, "f32")) == 2        # 3 heads: not a divisor of the CTA size
    assert _bwd(e2f.make_cfg(4, 256, 8, 16, 6.0, "bf16")) == 2      # shared memory beyond 227 KB


def test_fused_traversal_argument_checks():
    cfg = e2f.make_cfg(4, 128, 8, 16, 6.0, "bf16")
    box = (ctypes.c_float * 3)(30.0, 30.0, 30.0)
    small = (ctypes.c_float * 3)(10.0, 30.0, 30.0)
    assert e2f.e2f_attention_cells_workspace_size(3000, box, cfg) > e2f.e2f_attention_workspace_size(3000, 0, cfg)
    assert e2f.e2f_attention_cells_workspace_size(3000, None, cfg) > 0       # open boundaries: hashed cells
    assert e2f.e2f_attention_cells_workspace_size(3000, small, cfg) == 0     # cutoff above half the box
    f = e2f.lib().e2f_onfly_attention_cells
    v = ctypes.c_void_p
    bx = ctypes.cast(box, v)
    args = lambda c, b, x=16: (ctypes.byref(c), v(16), 4, b, v(x), v(16), v(16), v(16), v(16), v(16), v(256), 1 << 26,
                               None)
    assert f(*args(e2f.make_cfg(4, 128, 8, 16, 6.0, "f32"), bx)) == 2  # the tensor-core shapes only
    assert f(*args(cfg, bx, x=0)) == 1                                # null features
    assert f(*args(cfg, bx, x=8)) == 4                                # misaligned features
    # Verlet-skin variant: 16 bytes per atom more for the reference positions
    assert e2f.e2f_attention_cells_skin_workspace_size(3000, box, cfg, 0.0) == \
        e2f.e2f_attention_cells_workspace_size(3000, box, cfg)
    assert e2f.e2f_attention_cells_skin_workspace_size(3000, None, cfg, 1.0) >= \
        e2f.e2f_attention_cells_workspace_size(3000, None, cfg) + 16 * 3000
    assert e2f.e2f_attention_cells_skin_workspace_size(3000, box, cfg, -1.0) == 0
    assert e2f.e2f_attention_cells_skin_workspace_size(3000, box, cfg, float("nan")) == 0
    fs = e2f.lib().e2f_onfly_attention_cells_skin
    sargs = lambda skin, rebuild: (ctypes.byref(cfg), v(16), 4, bx, skin, rebuild, v(16), v(16), v(16), v(16),
                                   v(16), v(16), v(256), 1 << 26, None)
    assert fs(*sargs(0.0, 0)) == 1              # reuse needs a skin
    assert fs(*sargs(1.0, 0)) == 1              # reuse of a workspace no rebuild was recorded for
    assert fs(*sargs(-0.5, 1)) == 1             # negative skin
    assert fs(*sargs(float("nan"), 1)) == 1


def test_sixj_host_queries_and_argument_checks():
    from oracle.sixj import sixj_paths
    for L in range(5):
        for Lf in range(2 * L + 1):
            assert e2f.e2f_sixj_n_paths(L, Lf) == len(sixj_paths(L, Lf))
    assert e2f.e2f_sixj_n_paths(2, 5) == -1 and e2f.e2f_sixj_n_paths(5, 2) == -1
    ok = e2f.make_sixj_cfg(4, 8, 64, 8, 16, 5.0)
    assert e2f.e2f_sixj_workspace_size(10000, ok) > 16 * 895 * 64 * 10000
    for bad in [e2f.make_sixj_cfg(2, 5, 16, 1, 16, 5.0), e2f.make_sixj_cfg(5, 2, 16, 1, 16, 5.0),
                e2f.make_sixj_cfg(2, 2, 16, 3, 16, 5.0), e2f.make_sixj_cfg(2, 2, 512, 1, 16, 5.0),
                e2f.make_sixj_cfg(2, 2, 16, 1, 1, 5.0), e2f.make_sixj_cfg(2, 2, 16, 1, 16, 0.0)]:
        assert e2f.e2f_sixj_workspace_size(10, bad) == 0
    cfg = e2f.make_sixj_cfg(2, 4, 16, 1, 16, 5.0)
    need = e2f.e2f_sixj_workspace_size(4, cfg)
    v = lambda p: None if p is None else ctypes.c_void_p(p)

    def call(pos=16, n=4, gp=None, ng=0, rp=16, col=16, npairs=4, ws=256, wsb=need):
        return e2f.lib().e2f_sixj_attention(ctypes.byref(cfg), v(pos), n, v(gp), ng, v(rp), v(col), npairs, v(16),
                                            v(16), v(16), v(16), v(16), v(16), v(ws), wsb, None)
    assert call(pos=None) == 1
    assert call(npairs=-1) == 1
    assert call(gp=16, ng=0) == 1
    assert call(ws=128) == 4
    assert call(wsb=need - 1) == 1
    assert call(n=0) == 0
