"""Slab decomposition with a halo exchange, two gloo ranks on the CPU. The
oracle stands in for the GPU layer on each rank's local atoms (owned then
halo); the owned rows gathered from both ranks must equal the oracle on the
whole system."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from atomistic_cell_list_b200.domain import SlabDecomposition, owned_rows
from oracle.layer import DenseLayer
from oracle.neighbors import neighbors_bruteforce
from workloads import so2_block_sizes

L, C, H, NRBF, RC = 2, 8, 2, 8, 3.2
BOX = np.array([13.0, 11.0, 12.0])


def system():
    rng = np.random.default_rng(42)
    n = 180
    pos = (rng.random((n, 3)) * BOX).astype(np.float32)
    x = rng.normal(size=(n, (L + 1) ** 2, C))
    Wq = rng.normal(size=(C, C)) / np.sqrt(C)
    Wk = rng.normal(size=(C, C)) / np.sqrt(C)
    Wrad = rng.normal(size=(NRBF, (L + 1) * C + H)) / np.sqrt(C)
    Wso2 = rng.normal(size=sum(so2_block_sizes(L, C))) / np.sqrt(C)
    return pos, x, DenseLayer(L, C, H, NRBF, RC, Wq, Wk, Wrad, Wso2)


def local_oracle(dec, plan, pos, x_local, layer):
    pl = pos[plan["local"]]
    rp, col = neighbors_bruteforce(pl, BOX.astype(np.float32), RC)
    rp_t, col_t = owned_rows(torch.as_tensor(rp), torch.as_tensor(col), plan["owned"].size)
    return layer(pl, BOX, rp_t.numpy(), col_t.numpy(), x_local, nodes=np.arange(plan["owned"].size))


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        pos, x, layer = system()
        dec = SlabDecomposition(BOX, RC, world, rank, axis=0)
        plan = dec.plan(pos)
        seen_marks = []

        def local_layer(x_local):  # the oracle stands in for the GPU layer (as in the bench's slab mode)
            assert np.array_equal(x_local.numpy(), x[plan["local"]])  # the halo rows arrived
            return local_oracle(dec, plan, pos, x_local.numpy(), layer)

        out = dec.step(plan, torch.as_tensor(x[plan["owned"]]), local_layer, marks=seen_marks.append)
        assert seen_marks == ["start", "exchanged", "done"]
        q.put((rank, plan["owned"], out, {p: v.size for p, v in plan["send"].items()}))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_equal_the_whole_system():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    pos, x, layer = system()
    rp, col = neighbors_bruteforce(pos, BOX.astype(np.float32), RC)
    ref = layer(pos, BOX, rp, col, x)
    seen = np.zeros(pos.shape[0], bool)
    for rank, owned, out, sends in res:
        assert sends, "each rank sends halo rows to its neighbour"
        np.testing.assert_allclose(out, ref[owned], rtol=1e-10, atol=1e-12)
        seen[owned] = True
    assert seen.all()  # every atom owned by exactly one rank (sizes add up below)
    assert sum(r[1].size for r in res) == pos.shape[0]


def test_plan_is_consistent_between_ranks():
    pos, _, _ = system()
    plans = [SlabDecomposition(BOX, RC, 3, r).plan(pos) for r in range(3)]
    for a in range(3):
        for b in range(3):
            if a != b:
                sa = plans[a]["send"].get(b, np.zeros(0, np.int64))
                rb = plans[b]["recv"].get(a, np.zeros(0, np.int64))
                assert np.array_equal(sa, rb)
