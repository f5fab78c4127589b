"""Benchmark of the hot path: GPU cell-list neighbour build + on-the-fly
equivariant attention forward (E2Former-V2), one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--impl ours|reference]

A step is one pass of the whole path over one system: e2f_build_neighbors
(CSR of the 30,000-atom chain + water box) then e2f_onfly_attention
(L=4, C=128, 8 heads, bf16 features). Inputs are resident in HBM when the
timed region starts; L2 is flushed between steps (outside the timed events).
`value` is neighbour pairs per second over the whole step; the attention's
achieved SO(2) TFLOP/s is reported beside it and in `roofline`.
With --gpus N > 1 (torchrun) every rank runs its own replica (weak scaling;
the path needs no collective for independent systems).
`--impl reference` times the fp64 CPU oracle (the dense CG formulation) on
the host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "neighbor pairs/s + achieved TFLOPS, fused equivariant attn fwd, 1×B200"


def so2_flops_per_edge(L: int, C: int, M: int | None = None) -> int:
    """Algorithmic SO(2) FLOPs per edge: 2((L+1)C)^2 + sum_{m=1..M} 8((L+1-m)C)^2 (M = L: full layer)."""
    M = L if M is None or M < 0 or M > L else M
    return 2 * ((L + 1) * C) ** 2 + sum(8 * ((L + 1 - m) * C) ** 2 for m in range(1, M + 1))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, \
        "fallback"


# DRAM traffic of one k_attn_tc launch on the 30000-atom workload, from an ncu
# capture of that kernel on that workload (dram__bytes_read/write). Valid only for
# the kernel source it was taken on (sha256 of the files below); otherwise the
# bench reports traffic null.
KERNEL_TRAFFIC = {
    "sources": ["atomistic_cell_list_b200/csrc/attention_tc.cu", "atomistic_cell_list_b200/csrc/attention_tc.cuh",
                "atomistic_cell_list_b200/csrc/common.cuh", "atomistic_cell_list_b200/csrc/cell_grid.cuh",
                "atomistic_cell_list_b200/csrc/tcgen05.cuh"],
    "sha256": "6ef021a39c664cae9d45c252abcc1e273a25ee4b60bf01328fcf28018c8a9583",
    "dram_read_bytes": 44.39e9,
    "dram_write_bytes": 24.08e9,
}


def kernel_traffic():
    import hashlib
    if KERNEL_TRAFFIC["sha256"] is None:
        return None
    h = hashlib.sha256()
    for f in KERNEL_TRAFFIC["sources"]:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if h.hexdigest() != KERNEL_TRAFFIC["sha256"]:
        return None
    return KERNEL_TRAFFIC["dram_read_bytes"] + KERNEL_TRAFFIC["dram_write_bytes"]


def workload_desc(w):
    return {"workload": f"cfg{w.cfg_id}: {w.name}, cutoff {w.cutoff} A, L={w.L} C={w.C} H={w.H}, "
                        f"{w.dtype} features",
            "n_atoms": w.n_atoms, "periodic": w.box is not None}


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# --------------------------------------------------------------------------
def oracle_rate(cfg_id: int, budget_s: float, seed: int = 0):
    """Oracle pairs/s on the full neighbour search + a node sample of the
    dense attention sized to about budget_s seconds."""
    import workloads as W
    from oracle.layer import DenseLayer
    from oracle.neighbors import neighbors_kdtree

    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    w = W.load_workload(cfg_id)
    t0 = time.perf_counter()
    rp, col = neighbors_kdtree(w.pos, w.box, w.cutoff, w.graph_ptr)
    t_nbr = time.perf_counter() - t0
    xs, xf = W.make_features(cfg_id, w.n_atoms, w.L, w.C, w.dtype)
    wt = W.make_weights(cfg_id, w.L, w.C, w.H, w.n_rbf, w.dtype)
    layer = DenseLayer(w.L, w.C, w.H, w.n_rbf, w.cutoff, wt.Wq, wt.Wk, wt.Wrad, wt.Wso2_f64)
    rng = np.random.default_rng(seed)
    order = rng.permutation(w.n_atoms)
    done_e, t_attn, k = 0, 0.0, 0
    while t_attn < budget_s and k < w.n_atoms:
        nodes = np.sort(order[k:k + 4])
        k += 4
        t0 = time.perf_counter()
        layer(w.pos, w.box, rp, col, xf, nodes=nodes)
        t_attn += time.perf_counter() - t0
        done_e += int(sum(rp[n + 1] - rp[n] for n in nodes))
    E = int(col.size)
    per_edge = t_attn / max(done_e, 1)
    rate = E / (t_nbr + per_edge * E)
    cores = len(os.sched_getaffinity(0))
    sample = (f"full KD-tree + exact fp32 neighbour search ({t_nbr:.2f} s for {E} pairs) + dense CG attention "
              f"on {k} sampled destination nodes ({done_e} edges, {t_attn:.1f} s), extrapolated per edge to all "
              f"{E} pairs")
    return {"value": rate, "unit": "pairs/s", "cores": min(cores, max(threads, 1)), "kind": "oracle",
            "sample": sample, "host_cores": cores, "blas_threads": threads,
            "oracle_attn_edges_per_s": done_e / max(t_attn, 1e-9), "oracle_nbr_s": t_nbr}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    budget = float(os.environ.get("E2F_REF_STEP_S", "4"))
    vals, t_steps = [], []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        r = oracle_rate(args.config, budget, seed=s)
        if s >= args.warmup:
            vals.append(r["value"])
            t_steps.append(time.perf_counter() - t0)
    import workloads as W
    w = W.make_workload_meta(args.config)
    wl = W.load_workload(args.config)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "pairs/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(t_steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_desc(wl),
            "cpu_baseline": {**r, "value": v},
            "e2e": {"value": v, "unit": "pairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def use_tc_path(e2f, cfg) -> bool:
    return bool(e2f.e2f_attention_uses_tensor_cores(cfg))


def run_ours(args):
    import torch
    import torch.distributed as dist

    import atomistic_cell_list_b200 as e2f
    import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    w = W.load_workload(args.config)
    xs, _ = W.make_features(args.config, w.n_atoms, w.L, w.C, w.dtype)
    wt = W.make_weights(args.config, w.L, w.C, w.H, w.n_rbf, w.dtype)

    def host(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a))

    M = w.L if args.m_max < 0 or args.m_max > w.L else args.m_max
    n_so2 = sum(W.so2_block_sizes(w.L, w.C)[:2 * M + 1])  # truncated layer: blocks m <= M
    h_inputs = {"pos": host(w.pos), "x": host(xs).reshape(w.n_atoms, w.K, w.C), "Wq": host(wt.Wq),
                "Wk": host(wt.Wk), "Wrad": host(wt.Wrad), "Wso2": host(np.ascontiguousarray(wt.Wso2[:n_so2]))}
    d = {k: v.to(dev) for k, v in h_inputs.items()}
    box = None if w.box is None else [float(b) for b in w.box]
    gptr = None if w.graph_ptr is None else torch.from_numpy(w.graph_ptr).to(dev)
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype, m_max=M)
    stream = torch.cuda.current_stream(dev)

    # buffers reused by every step
    rp, col = e2f.e2f_build_neighbors(d["pos"], box, w.cutoff, gptr)
    E = int(col.numel())
    col_buf = torch.empty(E + E // 8 + 1024, dtype=torch.int32, device=dev)
    out = torch.empty((w.n_atoms, w.K, w.C), dtype=torch.float32, device=dev)
    ws = torch.empty(e2f.e2f_attention_workspace_size(w.n_atoms, E, cfg), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2

    def step():
        rp_, col_ = e2f.e2f_build_neighbors(d["pos"], box, w.cutoff, gptr, col_capacity=col_buf.numel())
        return rp_, col_

    def attn(rp_, col_):
        e2f.e2f_onfly_attention(cfg, d["pos"], box, rp_, col_, d["x"], d["Wq"], d["Wk"], d["Wrad"], d["Wso2"],
                                out=out, workspace=ws, check=False)

    for _ in range(args.warmup):
        rp_, col_ = step()
        attn(rp_, col_)
    torch.cuda.synchronize(dev)
    assert e2f.e2f_attention_status(ws) == 0

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    # events around the main attention kernel alone (recorded by the library on this stream)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for pair in kev:
        for e_ in pair:
            e_.record(stream)  # materialise the CUDA events before handing them over
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    n0 = e2f.e2f_launch_count()
    with ClockSampler(local) as clk:
        for s in range(args.steps):
            flush.zero_()
            ev[s][0].record(stream)
            rp_, col_ = step()
            ev[s][1].record(stream)
            e2f.e2f_attention_set_kernel_events(kev[s][0], kev[s][1])
            attn(rp_, col_)
            ev[s][2].record(stream)
        torch.cuda.synchronize(dev)
    e2f.e2f_attention_set_kernel_events(None, None)
    launches = e2f.e2f_launch_count() - n0 - 0
    if world > 1:
        dist.barrier()
    status = e2f.e2f_attention_status(ws)
    assert status == 0, e2f.status_string(status)
    t_step = [ev[s][0].elapsed_time(ev[s][2]) for s in range(args.steps)]
    t_nbr = [ev[s][0].elapsed_time(ev[s][1]) for s in range(args.steps)]
    t_att = [ev[s][1].elapsed_time(ev[s][2]) for s in range(args.steps)]
    use_tc = e2f.e2f_attention_uses_tensor_cores(cfg)
    t_ker = [kev[s][0].elapsed_time(kev[s][1]) for s in range(args.steps)] if use_tc else t_att
    tot = torch.tensor([sum(t_step), sum(t_att), sum(t_nbr), sum(t_ker)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tot, op=dist.ReduceOp.MAX)
    ms_step = float(tot[0]) / args.steps
    ms_att = float(tot[1]) / args.steps
    ms_nbr = float(tot[2]) / args.steps
    ms_ker = float(tot[3]) / args.steps

    # the same step with the cell-list traversal fused into the attention (periodic boxes):
    # no neighbour list is written; the call sorts atoms into cells and enumerates each
    # node's neighbours inside the kernel
    fused = None
    if use_tc_path(e2f, cfg) and box is not None and gptr is None:
        ws_c = torch.empty(e2f.e2f_attention_cells_workspace_size(w.n_atoms, box, cfg), dtype=torch.uint8,
                           device=dev)
        out_c = torch.empty_like(out)

        def fused_step():
            e2f.e2f_onfly_attention_cells(cfg, d["pos"], box, d["x"], d["Wq"], d["Wk"], d["Wrad"], d["Wso2"],
                                          out=out_c, workspace=ws_c, check=False)
        for _ in range(args.warmup):
            fused_step()
        torch.cuda.synchronize(dev)
        assert e2f.e2f_attention_status(ws_c) == 0
        f_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for s in range(args.steps):
            flush.zero_()
            f_ev[s][0].record(stream)
            fused_step()
            f_ev[s][1].record(stream)
        torch.cuda.synchronize(dev)
        status = e2f.e2f_attention_status(ws_c)
        assert status == 0, e2f.status_string(status)
        t_f = torch.tensor([sum(e[0].elapsed_time(e[1]) for e in f_ev)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(t_f, op=dist.ReduceOp.MAX)
        ms_f = float(t_f[0]) / args.steps
        fused = {"ms_per_step": ms_f, "value": world * E / (ms_f * 1e-3), "unit": "pairs/s",
                 "workspace_bytes": int(ws_c.numel()), "neighbor_list_bytes": 0,
                 "note": "e2f_onfly_attention_cells: cell sort + attention with in-kernel neighbour "
                         "enumeration, same layer and neighbour sets as the CSR step"}
        del ws_c

        # Verlet-skin reuse: the lists are sorted once (cells >= cutoff + skin); each timed
        # step refreshes the positions, recounts the degrees and runs the attention
        skin = 1.0
        ws_s = torch.empty(e2f.e2f_attention_cells_skin_workspace_size(w.n_atoms, box, cfg, skin),
                           dtype=torch.uint8, device=dev)

        def skin_step(rebuild):
            e2f.e2f_onfly_attention_cells_skin(cfg, d["pos"], box, skin, rebuild, d["x"], d["Wq"], d["Wk"],
                                               d["Wrad"], d["Wso2"], ws_s, out=out_c, check=False)
        skin_step(True)
        for _ in range(args.warmup):
            skin_step(False)
        torch.cuda.synchronize(dev)
        assert e2f.e2f_attention_status(ws_s) == 0
        for s in range(args.steps):
            flush.zero_()
            f_ev[s][0].record(stream)
            skin_step(False)
            f_ev[s][1].record(stream)
        torch.cuda.synchronize(dev)
        status = e2f.e2f_attention_status(ws_s)
        assert status == 0, e2f.status_string(status)
        t_s = torch.tensor([sum(e[0].elapsed_time(e[1]) for e in f_ev)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(t_s, op=dist.ReduceOp.MAX)
        ms_s = float(t_s[0]) / args.steps
        fused["skin_reuse"] = {"ms_per_step": ms_s, "skin": skin, "value": world * E / (ms_s * 1e-3),
                               "note": "e2f_onfly_attention_cells_skin, rebuild=0: refresh + recount + "
                                       "attention over cells of cutoff + skin"}
        del ws_s, out_c

    # end to end through the public API with pinned host buffers: every step copies its inputs
    # in (195 MB > L2) and its output out. Steps are pipelined over three streams with two
    # buffer sets, so step s+1's copy-in and step s-1's copy-out overlap step s's attention.
    # Step s-1's copy-out is enqueued after step s's neighbour build has returned: the build
    # reads its pair count back with a small device-to-host copy, which would otherwise queue
    # behind the 384 MB output copy on the same copy engine.
    pinned = {k: v.pin_memory() for k, v in h_inputs.items()}
    h_outs = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = h_outs[0].numel() * 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dbuf = [{k: torch.empty_like(v) for k, v in d.items()} for _ in range(2)]
    obuf = [torch.empty_like(out) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def copy_out(b):
        s_out.wait_event(ev_cmp[b])
        with torch.cuda.stream(s_out):
            h_outs[b].copy_(obuf[b], non_blocking=True)
            ev_out[b].record(s_out)

    def e2e_run(n_steps, timed):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        t0.record(s_in)
        for s in range(n_steps):
            b = s % 2
            if s >= 2:
                s_in.wait_event(ev_cmp[b])     # buffer set b is free once step s-2's compute is done
            with torch.cuda.stream(s_in):
                for k, v in pinned.items():
                    dbuf[b][k].copy_(v, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if s >= 2:
                stream.wait_event(ev_out[b])   # output buffer b has been read back
            dd = dbuf[b]
            rp_, col_ = e2f.e2f_build_neighbors(dd["pos"], box, w.cutoff, gptr, col_capacity=col_buf.numel())
            if s >= 1:
                copy_out(1 - b)
            e2f.e2f_onfly_attention(cfg, dd["pos"], box, rp_, col_, dd["x"], dd["Wq"], dd["Wk"], dd["Wrad"],
                                    dd["Wso2"], out=obuf[b], workspace=ws, check=False)
            ev_cmp[b].record(stream)
        copy_out((n_steps - 1) % 2)
        s_out.wait_stream(stream)
        s_out.wait_stream(s_in)
        t1.record(s_out)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1)

    e2e_run(args.warmup, False)
    if world > 1:
        dist.barrier()
    t_e2e = torch.tensor([e2e_run(args.steps, True)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t_e2e, op=dist.ReduceOp.MAX)
    ms_e2e = float(t_e2e[0]) / args.steps

    peaks, peak_src = measured_peaks()
    F = so2_flops_per_edge(w.L, w.C, M)
    tflops = E * F / (ms_att * 1e-3) / 1e12          # whole attention call (with its O(N) pre-passes)
    tflops_ker = E * F / (ms_ker * 1e-3) / 1e12      # the main kernel alone
    path = "tensor" if use_tc else "simt"
    if path == "simt":
        clk_max = float(peaks.get("sm_max_mhz", 1965.0))
        peak = 148 * 128 * 2 * clk_max * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": tflops_ker, "peak": peak, "unit": "TFLOP/s", "frac": tflops_ker / peak,
                "traffic": None,
                "peak_note": f"fp32 FMA pipe: 148 SMs x 128 lanes x 2 FLOP x {clk_max:.0f} MHz (derived, "
                             f"{peak_src} clock)"}
    else:
        peak = float(peaks["bf16_tflops"])
        sus = float(peaks.get("bf16_tflops_sustained", peak))
        roof = {"bound": "tensor", "achieved": tflops_ker, "peak": peak, "unit": "TFLOP/s", "frac": tflops_ker / peak,
                "traffic": kernel_traffic(), "peak_note": f"bf16 dense burst, {peak_src}",
                "peak_sustained": sus, "frac_sustained": tflops_ker / sus}
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    if roof.get("traffic"):
        # DRAM bytes per launch (ncu) over the live launch time: the gather phase runs inside this kernel
        roof["dram_gbs"] = roof["traffic"] / (ms_ker * 1e-3) / 1e9
        roof["dram_frac_of_hbm"] = roof["dram_gbs"] / hbm
    roof["kernel"] = "k_attn_tc (tcgen05)" if path == "tensor" else "k_attn_simt (fp32 CUDA cores)"
    roof["ms_per_launch"] = ms_ker
    roof["units_per_launch"] = f"{E} edges x {F} SO(2) FLOP"
    roof["traffic_note"] = ("dram read+write bytes per launch from an ncu capture of k_attn_tc on this workload; "
                            "null when the kernel source differs from the profiled one")

    nbr_bytes = 16 * w.n_atoms + 4 * (w.n_atoms + 1) + 4 * E + 8 * w.n_atoms
    line = {"metric": METRIC, "value": world * E / (ms_step * 1e-3), "unit": "pairs/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32" if path == "simt" else "bf16",
            "data": "synthetic",
            "config": {**workload_desc(w), "n_pairs": E, "m_max": M, "parallelism": f"replicas x{world}",
                       "l2": "flushed (256 MB write) between timed steps"},
            "tflops": tflops, "tflops_kernel": tflops_ker, "ms_attention": ms_att, "ms_attention_kernel": ms_ker,
            "ms_neighbors": ms_nbr,
            "neighbor_build_hbm": {
                "algorithmic_bytes": nbr_bytes, "gb_per_s": nbr_bytes / (ms_nbr * 1e-3) / 1e9,
                "frac_of_hbm": nbr_bytes / (ms_nbr * 1e-3) / 1e9 / hbm,
                "note": "16N (positions and keys read) + 4(N+1) + 4E (CSR written) + 8N (one pass of the "
                        "sort); latency-bound at these sizes"},
            "neighbor_pairs_per_s": E / (ms_nbr * 1e-3), "attention_pairs_per_s": E / (ms_att * 1e-3),
            "roofline": roof,
            "e2e": {"value": world * E / (ms_e2e * 1e-3), "unit": "pairs/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                    "note": "public API with pinned host buffers; inputs copied in and the output read back "
                            "every step, steps pipelined over copy-in, compute and copy-out streams"},
            "gpu_launches": int(launches),
            "fused_traversal": fused,
            "activation_memory": {"workspace_bytes": int(ws.numel()), "edge_tensor_bytes": 0,
                                  "csr_bytes": 4 * (w.n_atoms + 1) + 4 * E,
                                  "note": "the library's only scratch is the caller's workspace: O(N) + O(SMs), "
                                          "no per-edge float tensor"},
            "clocks": clk.summary()}
    if world == 1 and not args.no_extra:
        # the other workloads (parity-test cases, not bench lines) and the backward, after the timed region
        del dbuf, obuf, pinned, h_outs
        line["per_config"] = {}
        for c in (2, 3, 4, 5):
            line["per_config"][f"cfg{c}"] = measure_config(c, dev, 3, 2, flush, peaks)
        line["backward"] = backward_record(args.config, dev, 2, peaks)
        try:
            line["sixj"] = sixj_record(dev, 3)
        except Exception as err:  # a record of a variant, never a reason to lose the bench line
            line["sixj"] = {"error": f"{type(err).__name__}: {err}"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_rate(args.config, float(os.environ.get("E2F_CPU_BUDGET_S", "15")))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def measure_config(cfg_id, dev, steps, warmup, flush, peaks):
    """One workload of the five: step time (neighbour build + attention, L2 flushed
    between steps), pairs/s, SO(2) TFLOP/s and its fraction of the measured peak of
    the path it runs on, and the peak activation memory of the attention call
    measured with the allocator (max_memory_allocated during a call that allocates
    its own workspace and output, minus the fp32 output), per atom."""
    import torch

    import atomistic_cell_list_b200 as e2f
    import workloads as W

    w = W.load_workload(cfg_id)
    xs, _ = W.make_features(cfg_id, w.n_atoms, w.L, w.C, w.dtype)
    wt = W.make_weights(cfg_id, w.L, w.C, w.H, w.n_rbf, w.dtype)

    def dt(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    pos, x = dt(w.pos), dt(xs).reshape(w.n_atoms, w.K, w.C)
    Wq, Wk, Wrad, Wso2 = dt(wt.Wq), dt(wt.Wk), dt(wt.Wrad), dt(wt.Wso2)
    box = None if w.box is None else [float(b) for b in w.box]
    gptr = None if w.graph_ptr is None else torch.from_numpy(w.graph_ptr).to(dev)
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    tc = bool(e2f.e2f_attention_uses_tensor_cores(cfg))
    rp, col = e2f.e2f_build_neighbors(pos, box, w.cutoff, gptr)
    E = int(col.numel())
    col_buf = torch.empty(E + E // 8 + 1024, dtype=torch.int32, device=dev)
    out = torch.empty((w.n_atoms, w.K, w.C), dtype=torch.float32, device=dev)
    ws = torch.empty(e2f.e2f_attention_workspace_size(w.n_atoms, E, cfg), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(mid=None):
        rp_, col_ = e2f.e2f_build_neighbors(pos, box, w.cutoff, gptr, col_capacity=col_buf.numel())
        if mid is not None:
            mid.record(stream)
        e2f.e2f_onfly_attention(cfg, pos, box, rp_, col_, x, Wq, Wk, Wrad, Wso2, out=out, workspace=ws, check=False)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    assert e2f.e2f_attention_status(ws) == 0
    ts, tn = [], []
    for _ in range(steps):
        flush.zero_()
        a, m, b = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(stream)
        step(m)
        b.record(stream)
        torch.cuda.synchronize(dev)
        ts.append(a.elapsed_time(b))
        tn.append(a.elapsed_time(m))
    assert e2f.e2f_attention_status(ws) == 0
    ms, ms_n = statistics.mean(ts), statistics.mean(tn)
    F = so2_flops_per_edge(w.L, w.C)
    tflops = E * F / (ms * 1e-3) / 1e12
    if tc:
        peak, bound = float(peaks["bf16_tflops"]), "bf16 tensor (burst, whole step)"
    else:
        peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
        bound = "fp32 FMA pipe (derived, whole step)"
    # peak activation memory of one call that allocates its own workspace and output
    del ws
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    o2 = e2f.e2f_onfly_attention(cfg, pos, box, rp, col, x, Wq, Wk, Wrad, Wso2)
    torch.cuda.synchronize(dev)
    act = torch.cuda.max_memory_allocated(dev) - base - o2.numel() * 4
    del o2
    fixed = int(e2f.e2f_attention_workspace_size(1, 0, cfg))  # per-SM scratch and other size-independent parts
    return {"workload": workload_desc(w)["workload"], "n_atoms": w.n_atoms, "n_pairs": E,
            "path": "tcgen05" if tc else "fp32 CUDA cores", "ms_per_step": ms, "pairs_per_s": E / (ms * 1e-3),
            "ms_neighbors": ms_n, "neighbor_pairs_per_s": E / (ms_n * 1e-3),
            "attention_pairs_per_s": E / ((ms - ms_n) * 1e-3),
            "tflops": tflops, "frac": tflops / peak, "peak": peak, "peak_note": bound,
            "peak_activation_bytes": int(act), "activation_mb_per_atom": act / w.n_atoms / 1e6,
            "fixed_scratch_bytes": fixed, "activation_bytes_per_atom_beyond_fixed": (act - fixed) / w.n_atoms,
            "csr_bytes": 4 * (w.n_atoms + 1) + 4 * E}


def backward_record(cfg_id, dev, steps, peaks):
    """The attention's backward (all gradients) on one workload: ms, pairs/s, and the
    SO(2) work 3 E F_so2 (recomputed forward maps, transposed maps, weight gradient)
    over the time, against the measured bf16 burst peak."""
    import torch

    import atomistic_cell_list_b200 as e2f
    import workloads as W

    w = W.load_workload(cfg_id)
    xs, _ = W.make_features(cfg_id, w.n_atoms, w.L, w.C, w.dtype)
    wt = W.make_weights(cfg_id, w.L, w.C, w.H, w.n_rbf, w.dtype)

    def dt(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    pos, x = dt(w.pos), dt(xs).reshape(w.n_atoms, w.K, w.C)
    Wq, Wk, Wrad, Wso2 = dt(wt.Wq), dt(wt.Wk), dt(wt.Wrad), dt(wt.Wso2)
    box = None if w.box is None else [float(b) for b in w.box]
    gptr = None if w.graph_ptr is None else torch.from_numpy(w.graph_ptr).to(dev)
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(pos, box, w.cutoff, gptr)
    E = int(col.numel())
    G = torch.randn((w.n_atoms, w.K, w.C), generator=torch.Generator().manual_seed(1)).to(dev)
    ws = torch.empty(e2f.e2f_attention_backward_workspace_size(w.n_atoms, E, cfg), dtype=torch.uint8, device=dev)
    outs = e2f.e2f_onfly_attention_backward(cfg, pos, box, rp, col, x, Wq, Wk, Wrad, Wso2, G, want_weights=True,
                                            workspace=ws)
    torch.cuda.synchronize(dev)
    ts = []
    for _ in range(steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        e2f.e2f_onfly_attention_backward(cfg, pos, box, rp, col, x, Wq, Wk, Wrad, Wso2, G, want_weights=True,
                                         workspace=ws, out=outs)
        b.record()
        torch.cuda.synchronize(dev)
        ts.append(a.elapsed_time(b))
    ms = statistics.mean(ts)
    F = so2_flops_per_edge(w.L, w.C)
    tflops = 3 * E * F / (ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    return {"workload": workload_desc(w)["workload"], "n_pairs": E, "ms": ms, "pairs_per_s": E / (ms * 1e-3),
            "tflops": tflops, "frac": tflops / peak, "peak": peak,
            "units": f"{E} edges x 3 x {F} SO(2) FLOP (all gradients)", "steps": steps}


def sixj_record(dev, steps):
    """The Wigner-6j node-level convolution variant (e2f_sixj_attention) on the
    batch of 256 molecule graphs, L = 4, Lf = 4, C = 64, H = 8, fp32 features:
    ms per call with inputs resident, pairs/s, and the workspace it needs."""
    import torch

    import atomistic_cell_list_b200 as e2f
    import workloads as W

    w = W.load_workload(2)
    L, Lf, C, H, n_rbf = 4, 4, 64, 8, 16
    n = w.n_atoms
    xs, _ = W.make_features(100, n, L, C, "f32")
    Wq, Wk, Wrad, wp = W.make_sixj_weights(0, C, H, n_rbf, e2f.e2f_sixj_n_paths(L, Lf))

    def dt(a):
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)

    pos, gp = dt(w.pos), torch.from_numpy(w.graph_ptr).to(dev)
    rp, col = e2f.e2f_build_neighbors(pos, None, w.cutoff, gp)
    cfg = e2f.make_sixj_cfg(L, Lf, C, H, n_rbf, w.cutoff)
    ws = torch.empty(e2f.e2f_sixj_workspace_size(n, cfg), dtype=torch.uint8, device=dev)
    args = (cfg, pos, rp, col, dt(xs).reshape(n, (L + 1) ** 2, C), dt(Wq), dt(Wk), dt(Wrad), dt(wp))
    out = e2f.e2f_sixj_attention(*args, graph_ptr=gp, workspace=ws)
    torch.cuda.synchronize(dev)
    ts = []
    for _ in range(steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        e2f.e2f_sixj_attention(*args, graph_ptr=gp, workspace=ws, out=out)
        b.record()
        torch.cuda.synchronize(dev)
        ts.append(a.elapsed_time(b))
    ms = statistics.mean(ts)
    E = int(col.numel())
    rec = {"workload": "256 molecule graphs, 20-60 atoms", "n_atoms": n, "n_pairs": E, "L": L, "Lf": Lf, "C": C,
           "H": H, "ms": ms, "pairs_per_s": E / (ms * 1e-3), "workspace_bytes": int(ws.numel()), "steps": steps}
    del ws, out
    torch.cuda.empty_cache()
    return rec


def run_slab(args):
    """One system over the ranks (--decompose slab): each rank owns a slab of the
    periodic box, receives its halo rows from the two neighbouring slabs by NCCL
    point-to-point (batch_isend_irecv), searches the neighbours of its owned atoms
    and runs the layer on them. The halo exchange and the local layer (neighbour
    rows + attention) are timed apart with CUDA events; every figure is the maximum
    over ranks. The total work is one system whatever the rank count (strong
    scaling); value = all ranks' pairs / the slowest rank's step time."""
    import torch
    import torch.distributed as dist

    import atomistic_cell_list_b200 as e2f
    import workloads as W
    from atomistic_cell_list_b200.domain import SlabDecomposition

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    w = W.load_workload(args.config)
    if w.box is None or w.graph_ptr is not None:
        raise SystemExit("--decompose slab needs one periodic system")
    xs, _ = W.make_features(args.config, w.n_atoms, w.L, w.C, w.dtype)
    wt = W.make_weights(args.config, w.L, w.C, w.H, w.n_rbf, w.dtype)

    def dt(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    x_all = torch.from_numpy(xs.view(np.int16).copy()).view(torch.bfloat16) if xs.dtype == np.uint16 \
        else torch.from_numpy(np.ascontiguousarray(xs))
    x_all = x_all.reshape(w.n_atoms, w.K, w.C)
    Wq, Wk, Wrad, Wso2 = dt(wt.Wq), dt(wt.Wk), dt(wt.Wrad), dt(wt.Wso2)
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    dec = SlabDecomposition(w.box, w.cutoff, world, rank)
    plan = dec.plan(w.pos)
    x_owned = x_all[torch.as_tensor(plan["owned"])].to(dev)
    p_local = dec.local_positions(w.pos, plan, dev)
    stream = torch.cuda.current_stream(dev)
    n_edges = [0]

    def layer(x_local):
        box = [float(b) for b in dec.box]
        rp, col = e2f.e2f_build_neighbors(p_local, box, float(cfg.cutoff), rows=plan["owned"].size)
        n_edges[0] = int(col.numel())
        return e2f.e2f_onfly_attention(cfg, p_local, box, rp, col, x_local, Wq, Wk, Wrad, Wso2, check=False)

    for _ in range(args.warmup):
        dec.step(plan, x_owned, layer)
    torch.cuda.synchronize(dev)
    evs = []

    def marks(name):
        e_ = torch.cuda.Event(enable_timing=True)
        e_.record(stream)
        evs[-1][name] = e_

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for _ in range(args.steps):
        evs.append({})
        dec.step(plan, x_owned, layer, marks=marks)
    torch.cuda.synchronize(dev)
    t_x = sum(e["start"].elapsed_time(e["exchanged"]) for e in evs)
    t_l = sum(e["exchanged"].elapsed_time(e["done"]) for e in evs)
    t_s = sum(e["start"].elapsed_time(e["done"]) for e in evs)
    tot = torch.tensor([t_s, t_x, t_l], dtype=torch.float64, device=dev)
    edges = torch.tensor([n_edges[0], plan["owned"].size, plan["local"].size - plan["owned"].size],
                         dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tot, op=dist.ReduceOp.MAX)
        dist.all_reduce(edges, op=dist.ReduceOp.SUM)
    ms_step, ms_x, ms_l = (float(v) / args.steps for v in tot)
    E = int(edges[0])
    line = {"metric": METRIC, "value": E / (ms_step * 1e-3), "unit": "pairs/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {**workload_desc(w), "n_pairs": E, "parallelism": f"slab x{world}"},
            "decompose": "slab", "ms_halo_exchange": ms_x, "ms_local_layer": ms_l,
            "halo_atoms": int(edges[2]), "owned_atoms": int(edges[1]),
            "note": "one system over the ranks: NCCL point-to-point halo exchange, then the neighbour rows of "
                    "the owned atoms and the attention on owned + halo atoms; times are the maximum over ranks"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_naive(args):
    """Edge-materialising PyTorch baseline (naive_baseline.py) beside this
    library on the same workload: time, SO(2) TFLOP/s and peak activation
    memory of both (context for the pages' node-centric vs edge-centric
    comparison; not the product path)."""
    import torch

    import atomistic_cell_list_b200 as e2f
    import workloads as W
    from naive_baseline import naive_attention

    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    cfg_id = args.config
    w = W.load_workload(cfg_id)
    xs, _ = W.make_features(cfg_id, w.n_atoms, w.L, w.C, w.dtype)
    wt = W.make_weights(cfg_id, w.L, w.C, w.H, w.n_rbf, w.dtype)

    def dt(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    pos, x = dt(w.pos), dt(xs).reshape(w.n_atoms, w.K, w.C)
    Wq, Wk, Wrad, Wso2 = dt(wt.Wq), dt(wt.Wk), dt(wt.Wrad), dt(wt.Wso2)
    box = None if w.box is None else [float(b) for b in w.box]
    gptr = None if w.graph_ptr is None else torch.from_numpy(w.graph_ptr).to(dev)
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(pos, box, w.cutoff, gptr)
    E = int(col.numel())
    out_bytes = w.n_atoms * w.K * w.C * 4

    def measure(fn):
        res = None
        for _ in range(max(1, args.warmup)):
            res = fn()
        torch.cuda.synchronize(dev)
        del res
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for _ in range(args.steps):
            a.record()
            res = fn()
            b.record()
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b))
            del res
        peak = torch.cuda.max_memory_allocated(dev) - base
        return statistics.median(ts), peak

    F = so2_flops_per_edge(w.L, w.C)
    ours_ms, ours_peak = measure(lambda: e2f.e2f_onfly_attention(cfg, pos, box, rp, col, x, Wq, Wk, Wrad, Wso2))
    line = {"impl": "naive", "metric": "edge-materialising PyTorch baseline vs this library, same workload",
            "config": {**workload_desc(w), "n_pairs": E}, "unit": "ms", "data": "synthetic",
            "ours": {"ms": ours_ms, "tflops": E * F / (ours_ms * 1e-3) / 1e12,
                     "peak_activation_bytes": int(ours_peak - out_bytes)}}
    try:
        naive_ms, naive_peak = measure(lambda: naive_attention(cfg, pos, box, rp, col, x, Wq, Wk, Wrad, Wso2))
        line["naive"] = {"ms": naive_ms, "tflops": E * F / (naive_ms * 1e-3) / 1e12,
                         "peak_activation_bytes": int(naive_peak - out_bytes)}
        line["speedup"] = naive_ms / ours_ms
        line["memory_ratio"] = (naive_peak - out_bytes) / max(1, ours_peak - out_bytes)
    except torch.cuda.OutOfMemoryError as exc:  # E x K x C tensors do not fit
        line["naive"] = {"oom": str(exc).splitlines()[0][:160]}
    line["note"] = ("peak_activation_bytes = max_memory_allocated during the call minus inputs, weights, CSR and "
                    "the fp32 output; this library's is its workspace")
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args):
    """The attention's backward (e2f_onfly_attention_backward) on the bench workload: all
    gradients (positions, features, every weight), and positions + features + W_rad only
    (what forces need). With bf16 storage the maps run on tensor cores (mma.sync) and the
    SO(2) weight gradient as GEMMs over edge chunks (cuBLAS); the node kernel's per-edge
    CUDA-core work (rotations, gates, reductions) bounds the call, so the roofline reported
    is the FP32 FMA pipe's."""
    import torch

    import atomistic_cell_list_b200 as e2f
    import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = W.load_workload(args.config)
    xs, _ = W.make_features(args.config, w.n_atoms, w.L, w.C, w.dtype)
    wt = W.make_weights(args.config, w.L, w.C, w.H, w.n_rbf, w.dtype)

    def host(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a))

    pos = host(w.pos).to(dev)
    x = host(xs).reshape(w.n_atoms, w.K, w.C).to(dev)
    Wq, Wk, Wrad, Wso2 = (host(a).to(dev) for a in (wt.Wq, wt.Wk, wt.Wrad, wt.Wso2))
    box = None if w.box is None else [float(b) for b in w.box]
    gptr = None if w.graph_ptr is None else torch.from_numpy(w.graph_ptr).to(dev)
    cfg = e2f.make_cfg(w.L, w.C, w.H, w.n_rbf, w.cutoff, w.dtype)
    rp, col = e2f.e2f_build_neighbors(pos, box, w.cutoff, gptr)
    E = int(col.numel())
    G = torch.randn((w.n_atoms, w.K, w.C), generator=torch.Generator().manual_seed(1)).to(dev)
    ws = torch.empty(e2f.e2f_attention_backward_workspace_size(w.n_atoms, E, cfg), dtype=torch.uint8, device=dev)
    F = so2_flops_per_edge(w.L, w.C)
    peaks, peak_src = measured_peaks()
    clk_max = float(peaks.get("sm_max_mhz", 1965.0))
    fma_peak = 148 * 128 * 2 * clk_max * 1e6 / 1e12
    res = {}
    for want in (True, False):
        outs = e2f.e2f_onfly_attention_backward(cfg, pos, box, rp, col, x, Wq, Wk, Wrad, Wso2, G,
                                                want_weights=want, workspace=ws)
        for _ in range(max(0, args.warmup - 1)):
            e2f.e2f_onfly_attention_backward(cfg, pos, box, rp, col, x, Wq, Wk, Wrad, Wso2, G,
                                             want_weights=want, workspace=ws, out=outs)
        torch.cuda.synchronize(dev)
        ts = []
        with ClockSampler(0) as clk:
            for _ in range(args.steps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                e2f.e2f_onfly_attention_backward(cfg, pos, box, rp, col, x, Wq, Wk, Wrad, Wso2, G,
                                                 want_weights=want, workspace=ws, out=outs)
                b.record()
                torch.cuda.synchronize(dev)
                ts.append(a.elapsed_time(b))
        ms = statistics.mean(ts)
        # algorithmic work: the SO(2) maps applied twice per edge (recomputed Y, then the
        # transposed maps) and, with weights, the weight-gradient contraction (one more F)
        flops = E * F * (3 if want else 2)
        res["all" if want else "forces"] = {"ms": ms, "pairs_per_s": E / (ms * 1e-3),
                                            "tflops": flops / (ms * 1e-3) / 1e12, "clocks": clk.summary()}
    line = {"metric": "attention backward pairs/s (all gradients), 1xB200", "impl": "ours", "value":
            res["all"]["pairs_per_s"], "unit": "pairs/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": res["all"]["ms"], "higher_is_better": True, "dtype": "f32", "data": "synthetic",
            "config": {**workload_desc(w), "n_pairs": E}, "forces_only": res["forces"],
            "roofline": {"bound": "alu", "achieved": res["all"]["tflops"], "peak": fma_peak, "unit": "TFLOP/s",
                         "frac": res["all"]["tflops"] / fma_peak, "traffic": None,
                         "peak_note": f"fp32 FMA pipe: 148 SMs x 128 lanes x 2 FLOP x {clk_max:.0f} MHz "
                                      f"(derived, {peak_src} clock); the contractions themselves run on "
                                      f"tensor cores for bf16 storage",
                         "units_per_launch": f"{E} edges x 3 x {F} SO(2) FLOP"},
            "clocks": res["all"]["clocks"]}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--impl", choices=["ours", "reference", "naive"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the per-config block and the backward record")
    ap.add_argument("--m-max", type=int, default=-1, help="SO(2) truncation order (-1: full layer)")
    ap.add_argument("--backward", action="store_true", help="time the attention's backward instead")
    ap.add_argument("--decompose", choices=["replicas", "slab"], default="replicas",
                    help="slab: one system over the ranks with a halo exchange (default: independent replicas)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.backward:
        return run_backward(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.impl == "naive":
        return run_naive(args)
    if args.decompose == "slab":
        return run_slab(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
