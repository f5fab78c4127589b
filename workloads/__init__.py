"""Seeded synthetic atom clouds, features and weights for the five workloads.

This module only makes inputs. It holds none of the layer's arithmetic: no
spherical harmonics, rotations, gates, softmax or neighbour predicate. Both
the CUDA path (through ``bench.py`` and the GPU tests) and the CPU oracle
read the arrays it returns, so they consume identical bytes.

Workloads (E2Former-V2, "Experimental Results": water box MD, a ~30k-atom
solvated protein, OMol25-scale systems up to 100k atoms on one GPU; the
pages publish no geometry, so these stand-ins are synthetic):

  1 tiny    64 atoms, random sequential addition (RSA) in an open 10 A cube,
            min separation 0.9 A, cutoff 5, L=2, C=16, H=1, fp32 features.
  2 batch   256 graphs of U{20..60} atoms, each an N(0, 3^2 I) cluster at the
            origin (graphs overlap in space), min separation 0.9 A inside a
            graph, open, cutoff 5, L=4, C=64, H=8, bf16.
  3 water   periodic cube at 0.1 atoms/A^3 (side 31.07 A): 1000 O by RSA with
            O-O >= 2.5 A, two H each at 0.96 A and 104.5 deg, Haar-random
            orientation, cutoff 6, L=4, C=128, H=8, bf16.
  4 chain   periodic cube of side 66.94 A: an 8000-bead growth walk (3.8 A
            steps, self-avoiding at 2.0 A, confined to a 33 A sphere at the
            box centre) plus 7333 water triplets and one lone O (O-O >= 2.5,
            O-chain >= 2.0), 30000 atoms, cutoff 6, L=4, C=128, H=8, bf16.
  5 water   periodic cube of side 100 A: 33333 triplets plus one lone O,
            100000 atoms, cutoff 6, L=4, C=128, H=8, bf16.

Seeds: positions 1000+k, features 2000+k, weights 3000+k (numpy PCG64).
Features ~ N(0, 1); every weight ~ N(0, 1/C). Values are drawn in fp64 and
rounded once to the workload's dtype; ``*_f64`` arrays hold the rounded
values exactly.
"""
from __future__ import annotations

import dataclasses
import math
import os

import numpy as np

N_RBF = 16


@dataclasses.dataclass
class Workload:
    cfg_id: int
    name: str
    pos: np.ndarray            # [N, 3] float32
    box: np.ndarray | None     # [3] float32, or None for open boundaries
    graph_ptr: np.ndarray | None  # [B+1] int32, or None for one graph
    cutoff: float
    L: int
    C: int
    H: int
    n_rbf: int
    dtype: str                 # "f32" or "bf16"

    @property
    def n_atoms(self) -> int:
        return int(self.pos.shape[0])

    @property
    def K(self) -> int:
        return (self.L + 1) ** 2


# --------------------------------------------------------------------------
# bf16 storage helpers (round-to-nearest-even of the fp32 value)
# --------------------------------------------------------------------------

def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (via fp32, ties to even); return uint16 bits."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    u = b.astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_to_dtype(a: np.ndarray, dtype: str):
    """Return (storage array, exact fp64 values of the stored numbers)."""
    if dtype == "f32":
        s = np.ascontiguousarray(a, dtype=np.float32)
        return s, s.astype(np.float64)
    if dtype == "bf16":
        s = f64_to_bf16_bits(a)
        return s, bf16_bits_to_f64(s)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# hard-sphere placement on a cell grid (at most one point per cell)
# --------------------------------------------------------------------------

class _Grid:
    """Occupancy grid for exclusion tests. Cell side h <= dmin/sqrt(3), so two
    points closer than dmin never share a cell and a stencil of radius
    ceil(dmin/h) cells finds every conflicting point."""

    def __init__(self, side: float, dmin: float, periodic: bool):
        self.side = float(side)
        self.periodic = periodic
        self.dmin = float(dmin)
        hmax = dmin / math.sqrt(3.0)
        if periodic:
            self.ng = max(1, int(math.ceil(self.side / hmax)))
            self.h = self.side / self.ng
        else:
            self.h = hmax
            self.ng = int(math.ceil(self.side / hmax)) + 1
        self.occ = -np.ones((self.ng,) * 3, dtype=np.int64)
        self.pts = np.zeros((1024, 3))
        self.n = 0
        r = int(math.ceil(dmin / self.h))
        o = np.arange(-r, r + 1)
        self.stencil = np.stack(np.meshgrid(o, o, o, indexing="ij"), -1).reshape(-1, 3)

    def _cell(self, p):
        c = np.floor(p / self.h).astype(np.int64)
        if self.periodic:
            c %= self.ng
        return c

    def conflicts(self, cand: np.ndarray, dmin: float | None = None) -> np.ndarray:
        """Boolean [B]: True where a candidate lies closer than dmin to a point."""
        dmin = self.dmin if dmin is None else dmin
        if self.n == 0:
            return np.zeros(cand.shape[0], bool)
        c = self._cell(cand)[:, None, :] + self.stencil[None]
        if self.periodic:
            c %= self.ng
            inside = np.ones(c.shape[:2], bool)
        else:
            inside = np.all((c >= 0) & (c < self.ng), axis=-1)
            c = np.clip(c, 0, self.ng - 1)
        idx = self.occ[c[..., 0], c[..., 1], c[..., 2]]
        idx = np.where(inside, idx, -1)
        q = self.pts[np.maximum(idx, 0)]
        d = q - cand[:, None, :]
        if self.periodic:
            d -= self.side * np.round(d / self.side)
        d2 = np.einsum("bsk,bsk->bs", d, d)
        return np.any((idx >= 0) & (d2 < dmin * dmin), axis=1)

    def add(self, p: np.ndarray) -> int:
        c = self._cell(p[None])[0]
        if self.occ[c[0], c[1], c[2]] >= 0:
            raise RuntimeError("grid cell already occupied")
        if self.n == self.pts.shape[0]:
            self.pts = np.concatenate([self.pts, np.zeros_like(self.pts)])
        k = self.n
        self.pts[k] = p
        self.n += 1
        self.occ[c[0], c[1], c[2]] = k
        return k

    def remove_last(self, n: int):
        for p in self.pts[self.n - n:self.n]:
            c = self._cell(p[None])[0]
            self.occ[c[0], c[1], c[2]] = -1
        self.n -= n


def _rsa(rng, n, side, dmin, periodic, extra=None, batch=256, lo=0.0, hi=None,
         max_tries=400):
    """Random sequential addition of n points with pairwise distance >= dmin.
    ``extra`` is an optional (grid, distance) pair of points to keep away from."""
    hi = side if hi is None else hi
    g = _Grid(side, dmin, periodic)
    out = []
    tries = 0
    while len(out) < n:
        tries += 1
        if tries > max_tries * max(1, n // batch + 1):
            raise RuntimeError(f"RSA jammed at {len(out)}/{n}")
        cand = rng.uniform(lo, hi, size=(batch, 3))
        bad = g.conflicts(cand)
        if extra is not None:
            bad |= extra[0].conflicts(cand, extra[1])
        for p in cand[~bad]:
            if len(out) >= n:
                break
            if g.conflicts(p[None])[0]:
                continue
            g.add(p)
            out.append(p)
    return np.array(out)


def _haar_rotations(rng, n):
    """n rotation matrices uniform on SO(3) (QR of a Gaussian, sign-fixed)."""
    a = rng.normal(size=(n, 3, 3))
    q, r = np.linalg.qr(a)
    s = np.sign(np.diagonal(r, axis1=1, axis2=2))
    q = q * s[:, None, :]
    det = np.linalg.det(q)
    q[det < 0, :, 0] *= -1
    return q


def _add_hydrogens(rng, O):
    ang = math.radians(104.5)
    h1 = np.array([0.96, 0.0, 0.0])
    h2 = np.array([0.96 * math.cos(ang), 0.96 * math.sin(ang), 0.0])
    R = _haar_rotations(rng, O.shape[0])
    H1 = O + R @ h1
    H2 = O + R @ h2
    # atom order: O, H, H per molecule
    return np.stack([O, H1, H2], axis=1).reshape(-1, 3)


def _chain(rng, n, step, dmin, radius, side, tries=256, back=50):
    centre = np.full(3, side / 2.0)
    g = _Grid(side, dmin, periodic=True)
    pts = [centre.copy()]
    g.add(centre)
    fails = 0
    while len(pts) < n:
        v = rng.normal(size=(tries, 3))
        v /= np.linalg.norm(v, axis=1, keepdims=True)
        cand = pts[-1] + step * v
        inside = np.linalg.norm(cand - centre, axis=1) <= radius
        ok = inside & ~g.conflicts(cand)
        if ok.any():
            p = cand[np.argmax(ok)]
            g.add(p)
            pts.append(p)
            continue
        fails += 1
        if fails > 20000:
            raise RuntimeError("chain growth stalled")
        k = min(back, len(pts) - 1)
        g.remove_last(k)
        del pts[-k:]
    return np.array(pts), g


def _wrap(p, side):
    return np.mod(p, side)


def make_workload(cfg_id: int) -> Workload:
    rng = np.random.default_rng(1000 + cfg_id)
    if cfg_id == 1:
        pos = _rsa(rng, 64, 10.0, 0.9, periodic=False)
        return Workload(1, "tiny open cube, 64 atoms", pos.astype(np.float32), None, None,
                        5.0, 2, 16, 1, N_RBF, "f32")
    if cfg_id == 2:
        blocks, ptr = [], [0]
        for _ in range(256):
            n = int(rng.integers(20, 61))
            pts = []
            while len(pts) < n:
                q = rng.normal(0.0, 3.0, size=3)
                if pts and (np.linalg.norm(np.array(pts) - q, axis=1) < 0.9).any():
                    continue
                pts.append(q)
            blocks.append(np.array(pts))
            ptr.append(ptr[-1] + n)
        pos = np.concatenate(blocks)
        return Workload(2, "256 molecule graphs, 20-60 atoms", pos.astype(np.float32), None,
                        np.array(ptr, np.int32), 5.0, 4, 64, 8, N_RBF, "bf16")
    if cfg_id == 3:
        side = (3000 / 0.1) ** (1.0 / 3.0)
        O = _rsa(rng, 1000, side, 2.5, periodic=True)
        pos = _wrap(_add_hydrogens(rng, O), side)
        box = np.full(3, side, np.float32)
        return Workload(3, "periodic water box, 3000 atoms", pos.astype(np.float32), box, None,
                        6.0, 4, 128, 8, N_RBF, "bf16")
    if cfg_id == 4:
        side = (30000 / 0.1) ** (1.0 / 3.0)
        chain, cg = _chain(rng, 8000, 3.8, 2.0, 33.0, side)
        O = _rsa(rng, 7334, side, 2.5, periodic=True, extra=(cg, 2.0))
        wat = _add_hydrogens(rng, O[:7333])
        pos = _wrap(np.concatenate([chain, wat, O[7333:]]), side)
        box = np.full(3, side, np.float32)
        return Workload(4, "chain + water, 30000 atoms", pos.astype(np.float32), box, None,
                        6.0, 4, 128, 8, N_RBF, "bf16")
    if cfg_id == 5:
        side = (100000 / 0.1) ** (1.0 / 3.0)
        O = _rsa(rng, 33334, side, 2.5, periodic=True)
        wat = _add_hydrogens(rng, O[:33333])
        pos = _wrap(np.concatenate([wat, O[33333:]]), side)
        box = np.full(3, side, np.float32)
        return Workload(5, "water, 100000 atoms", pos.astype(np.float32), box, None,
                        6.0, 4, 128, 8, N_RBF, "bf16")
    raise ValueError(cfg_id)


_CACHE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "build", "workloads")


def load_workload(cfg_id: int) -> Workload:
    """make_workload with an on-disk cache (build/, not versioned)."""
    path = os.path.join(_CACHE_DIR, f"cfg{cfg_id}.npz")
    if os.path.exists(path):
        try:
            z = np.load(path, allow_pickle=False)
            w = make_workload_meta(cfg_id)
            w.pos = z["pos"]
            w.box = z["box"] if z["box"].size else None
            w.graph_ptr = z["graph_ptr"] if z["graph_ptr"].size else None
            return w
        except Exception:
            pass
    w = make_workload(cfg_id)
    try:
        os.makedirs(_CACHE_DIR, exist_ok=True)
        tmp = path + f".{os.getpid()}.tmp.npz"
        np.savez(tmp, pos=w.pos,
                 box=w.box if w.box is not None else np.zeros(0, np.float32),
                 graph_ptr=w.graph_ptr if w.graph_ptr is not None else np.zeros(0, np.int32))
        os.replace(tmp, path)
    except OSError:
        pass
    return w


_META = {
    1: ("tiny open cube, 64 atoms", 5.0, 2, 16, 1, "f32"),
    2: ("256 molecule graphs, 20-60 atoms", 5.0, 4, 64, 8, "bf16"),
    3: ("periodic water box, 3000 atoms", 6.0, 4, 128, 8, "bf16"),
    4: ("chain + water, 30000 atoms", 6.0, 4, 128, 8, "bf16"),
    5: ("water, 100000 atoms", 6.0, 4, 128, 8, "bf16"),
}


def make_workload_meta(cfg_id: int) -> Workload:
    name, rc, L, C, H, dt = _META[cfg_id]
    return Workload(cfg_id, name, np.zeros((0, 3), np.float32), None, None, rc, L, C, H, N_RBF, dt)


# --------------------------------------------------------------------------
# features and weights
# --------------------------------------------------------------------------

def so2_block_sizes(L: int, C: int):
    """Sizes of the packed SO(2) weight blocks, in storage order:
    A(0); then A(m), B(m) for m = 1..L. Block m is square of side (L+1-m)*C."""
    out = [((L + 1) * C) ** 2]
    for m in range(1, L + 1):
        n = (L + 1 - m) * C
        out += [n * n, n * n]
    return out


def make_features(cfg_id: int, n_atoms: int, L: int, C: int, dtype: str, seed_offset: int = 0):
    """x ~ N(0,1), shape [N, (L+1)^2, C]. Returns (storage, exact fp64 values)."""
    rng = np.random.default_rng(2000 + cfg_id + seed_offset)
    x = rng.normal(size=(n_atoms, (L + 1) ** 2, C))
    return round_to_dtype(x, dtype)


@dataclasses.dataclass
class Weights:
    Wq: np.ndarray      # [C, C] float32
    Wk: np.ndarray      # [C, C] float32
    Wrad: np.ndarray    # [n_rbf, (L+1)C + H] float32
    Wso2: np.ndarray    # packed, float32 or uint16 (bf16 bits)
    Wso2_f64: np.ndarray  # exact values of the stored SO(2) weights


def make_weights(cfg_id: int, L: int, C: int, H: int, n_rbf: int, dtype: str,
                 seed_offset: int = 0) -> Weights:
    rng = np.random.default_rng(3000 + cfg_id + seed_offset)
    s = 1.0 / math.sqrt(C)
    Wq = (rng.normal(size=(C, C)) * s).astype(np.float32)
    Wk = (rng.normal(size=(C, C)) * s).astype(np.float32)
    Wrad = (rng.normal(size=(n_rbf, (L + 1) * C + H)) * s).astype(np.float32)
    n = sum(so2_block_sizes(L, C))
    W, Wf = round_to_dtype(rng.normal(size=n) * s, dtype)
    return Weights(Wq, Wk, Wrad, W, Wf)


def make_sixj_weights(seed: int, C: int, H: int, n_rbf: int, n_paths: int):
    """Weights of the Wigner-6j node-level convolution layer, float32:
    W_q, W_k [C, C], W_rad [n_rbf, H] (logit gates), w_path [n_paths, C]."""
    rng = np.random.default_rng(4000 + seed)
    s = 1.0 / math.sqrt(C)
    Wq = (rng.normal(size=(C, C)) * s).astype(np.float32)
    Wk = (rng.normal(size=(C, C)) * s).astype(np.float32)
    Wrad = rng.normal(size=(n_rbf, H)).astype(np.float32)
    w_path = (rng.normal(size=(n_paths, C)) * 0.3).astype(np.float32)
    return Wq, Wk, Wrad, w_path
