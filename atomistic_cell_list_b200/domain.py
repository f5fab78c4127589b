"""Spatial slab decomposition of one system over ranks, with one halo
exchange per attention layer.

The node-centric layer (gist.science Technical Summary 2.2, Eq. 6) needs,
for each destination node, only the positions and features of the atoms
within the cutoff. So a rank that owns the atoms of a slab of the periodic
box needs, besides its own atoms, the "halo": the atoms of other slabs
within the cutoff of its slab. After one exchange of those rows the layer
runs locally and each output row is written once, on its owner; there is
no reduction.

Positions are replicated on every rank (12 bytes per atom); features are
not (C * (L+1)^2 values per atom): each rank holds the rows of its own atoms
and receives its halo rows from their owners by point-to-point send/recv
(NCCL on GPUs, gloo in the CPU tests). Slabs cut the box along one axis;
every slab must be at least as wide as the cutoff, so a rank's halo comes
from its two neighbouring slabs only.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist


class SlabDecomposition:
    def __init__(self, box, cutoff: float, world: int, rank: int, axis: int = 0):
        if box is None:
            raise ValueError("the slab decomposition needs a periodic box")
        self.box = np.asarray(box, np.float64)
        self.cutoff = float(cutoff)
        self.world, self.rank, self.axis = int(world), int(rank), int(axis)
        self.width = self.box[self.axis] / self.world
        if self.world > 1 and self.width < self.cutoff:
            raise ValueError(f"slab width {self.width:.3f} is below the cutoff {self.cutoff}")

    # -- ownership -------------------------------------------------------
    def owner(self, pos: np.ndarray) -> np.ndarray:
        """Rank owning each atom: the slab of its wrapped coordinate."""
        u = np.mod(np.asarray(pos, np.float64)[:, self.axis], self.box[self.axis])
        return np.minimum((u / self.width).astype(np.int64), self.world - 1)

    def halo_of(self, pos: np.ndarray, r: int) -> np.ndarray:
        """Global indices of the atoms not owned by rank r within the cutoff of its slab."""
        L = self.box[self.axis]
        u = np.mod(np.asarray(pos, np.float64)[:, self.axis], L)
        lo, hi = r * self.width, (r + 1) * self.width
        # periodic distance of u to the slab [lo, hi)
        d_lo = np.mod(lo - u, L)   # how far below lo (wrapped)
        d_hi = np.mod(u - hi, L)   # how far above hi (wrapped)
        near = np.minimum(d_lo, d_hi) <= self.cutoff
        return np.nonzero(near & (self.owner(pos) != r))[0]

    def plan(self, pos: np.ndarray):
        """Index lists from the replicated positions: owned atoms, the local
        atom order (owned then halo), and per peer the rows to send and to
        receive. Every rank computes the same plan."""
        own = self.owner(pos)
        owned = np.nonzero(own == self.rank)[0]
        halo = self.halo_of(pos, self.rank)
        send, recv = {}, {}
        for p in range(self.world):
            if p == self.rank:
                continue
            hp = self.halo_of(pos, p)
            s = hp[own[hp] == self.rank]            # my atoms that p needs
            r = halo[own[halo] == p]                # p's atoms that I need
            if s.size:
                send[p] = s
            if r.size:
                recv[p] = r
        local = np.concatenate([owned, np.concatenate([recv[p] for p in sorted(recv)]) if recv else
                                np.zeros(0, np.int64)])
        return {"owned": owned, "local": local, "send": send, "recv": recv}

    # -- exchange --------------------------------------------------------
    def exchange(self, plan, x_owned: torch.Tensor) -> torch.Tensor:
        """Rows of the local atoms (owned then halo, in plan["local"] order)
        from this rank's owned rows (in plan["owned"] order)."""
        owned = plan["owned"]
        pos_in_owned = {int(g): k for k, g in enumerate(owned)}
        ops, bufs = [], {}
        for p in sorted(plan["send"]):
            rows = torch.as_tensor([pos_in_owned[int(g)] for g in plan["send"][p]], device=x_owned.device)
            ops.append(dist.P2POp(dist.isend, x_owned.index_select(0, rows).contiguous(), p))
        for p in sorted(plan["recv"]):
            bufs[p] = torch.empty((plan["recv"][p].size,) + tuple(x_owned.shape[1:]), dtype=x_owned.dtype,
                                  device=x_owned.device)
            ops.append(dist.P2POp(dist.irecv, bufs[p], p))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
        return torch.cat([x_owned] + [bufs[p] for p in sorted(bufs)], dim=0)

    # -- one step --------------------------------------------------------
    def step(self, plan, x_owned: torch.Tensor, layer, marks=None):
        """One layer step of this rank: the halo exchange, then layer(x_local) on the
        local atoms (owned then halo rows); returns what the layer returns (the owned
        rows). marks, if given, is called with "start", "exchanged" and "done", so
        that a caller can time the exchange and the local layer apart."""
        if marks:
            marks("start")
        x_local = self.exchange(plan, x_owned)
        if marks:
            marks("exchanged")
        out = layer(x_local)
        if marks:
            marks("done")
        return out

    # -- the layer on this rank's atoms -----------------------------------
    def attention(self, cfg, pos: np.ndarray, x_owned: torch.Tensor, Wq, Wk, Wrad, Wso2, plan=None):
        """out rows of this rank's owned atoms (plan["owned"] order), computed
        by the library on the local atoms after one halo exchange."""
        plan = self.plan(pos) if plan is None else plan
        x_local = self.exchange(plan, x_owned)
        return self.local_attention(cfg, pos, plan, x_local, Wq, Wk, Wrad, Wso2)

    def local_positions(self, pos: np.ndarray, plan, device) -> torch.Tensor:
        """Positions of the local atoms (owned then halo), on the device."""
        return torch.as_tensor(np.asarray(pos, np.float32)[plan["local"]], device=device)

    def local_attention(self, cfg, pos, plan, x_local: torch.Tensor, Wq, Wk, Wrad, Wso2):
        """The layer on the local atoms (owned then halo rows of x_local): the
        neighbour rows of the owned atoms only (halo atoms are candidates, their
        own rows are not searched), then the attention; returns the owned rows.
        pos: all positions (numpy), or the local positions already on the device."""
        import atomistic_cell_list_b200 as e2f
        p_local = pos if isinstance(pos, torch.Tensor) else self.local_positions(pos, plan, x_local.device)
        box = [float(b) for b in self.box]
        n_owned = plan["owned"].size
        rp, col = e2f.e2f_build_neighbors(p_local, box, float(cfg.cutoff), rows=n_owned)
        out = e2f.e2f_onfly_attention(cfg, p_local, box, rp, col, x_local, Wq, Wk, Wrad, Wso2)
        return out[:n_owned]


def owned_rows(row_ptr: torch.Tensor, col: torch.Tensor, n_owned: int):
    """CSR restricted to the first n_owned rows (the owned atoms); the halo
    rows become empty (their outputs are not needed on this rank)."""
    end = int(row_ptr[n_owned].item())
    rp = row_ptr.clone()
    rp[n_owned + 1:] = end
    return rp, col[:end]
