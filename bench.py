"""Benchmark of the tile-sparse attention layer (TripPool -> projection/score ->
Top-k -> tile-skipping attention) on the 245,760-token long-video workload
(B=1, H=32, d=128, grid 60x64x64, head-aware 128-token tiles, 1,920 tiles,
k=96 = 95% sparsity).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {veda,reference}]

A step is one pass of the whole layer over one batch of synthetic input.  The
timed region covers K steps on the device (CUDA events, barrier + synchronize
on both sides, max over ranks).  Inputs (Q/K/V 6 GB) are larger than L2.  The
metric is ms/layer and effective TFLOP/s: the FLOPs of the selected tile pairs
only (4 * B*H*nT*k*Bt^2*d = 4.948e13), mask preparation included in the time.

Multi-GPU: every rank runs its own layer (independent batch entries, no
data-path collective): weak scaling; value = FLOPs of all ranks / max time.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (the reference arm; rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "ms/layer and effective TFLOP/s of tile-sparse attention (+mask prep) at 95% sparsity"


# DRAM bytes (read + write) of one attention launch on the estimator's mask,
# with the kernel version and the capture they come from.  A kernel change
# empties the entry until the counters are taken again.  The long-video figure
# scales a single-launch capture at the 720P-like layer (1.112 GB read +
# 0.763 GB written for 24,000 query tiles) by query tiles (61,440), the size
# rule for counter captures keeping them off the 6 GB workload.
ATTN_DRAM_BYTES = {"long_video_245k": {"bytes": (1.112e9 + 0.763e9) * 61440 / 24000,
                                       "kernel": "sparse_attn_dual_kernel, commit d3c5c7b",
                                       "capture": "ncu --metrics dram__bytes_read.sum,"
                                                  "dram__bytes_write.sum, one launch at the "
                                                  "720P-like layer, scaled by query tiles"},
                   "720p": {"bytes": 1.112e9 + 0.763e9,
                            "kernel": "sparse_attn_dual_kernel, commit d3c5c7b",
                            "capture": "ncu --metrics dram__bytes_read.sum,"
                                       "dram__bytes_write.sum, one launch"}}


def _config(w, world):
    """The `config` object of both arms' JSON lines."""
    return dict(w.describe(),
                parallelism="replicas (one layer per GPU)" if world > 1 else "single GPU",
                l2=f"inputs larger than L2 (Q/K/V {3 * w.B * w.H * w.N * w.d * 2 / 1e9:.2f} GB)")


def key_tile_coverage(idx, nT):
    """Per (b, h): distinct key tiles the index lists select, and the share of
    all selections that fall on the k most-selected key tiles (how strongly the
    rows concentrate on a few key tiles, i.e. how much of K/V stays in L2)."""
    BH = idx.shape[0] * idx.shape[1]
    flat = idx.reshape(BH, -1).long()
    counts = torch.zeros((BH, nT), dtype=torch.int64, device=idx.device)
    counts.scatter_add_(1, flat, torch.ones_like(flat))
    distinct = (counts > 0).sum(1).double()
    k = idx.shape[-1]
    top = counts.sort(1, descending=True).values[:, :k].sum(1).double() / flat.shape[1]
    return {"distinct_key_tiles_per_head": {"mean": distinct.mean().item(),
                                            "min": distinct.min().item(),
                                            "max": distinct.max().item(), "of": nT},
            "share_of_selections_on_top_k_tiles": top.mean().item()}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


# ---------------------------------------------------------------- distributed
def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _job_tflops(flops_per_replica: float, ms_per_step_max: float, world: int) -> float:
    """Whole-job throughput: every rank runs one replica of the layer per step,
    so the job does world x the work in the slowest rank's time."""
    return world * flops_per_replica / (ms_per_step_max * 1e-3) / 1e12


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[3][1:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(w, t_host, heads=1, units_per_head=24, threads=None):
    """Times the fp64 oracle on a bounded sample of the layer and extrapolates.

    Sample: full mask preparation for ``heads`` heads (TripPool, projection,
    score, Top-k) and attention for ``units_per_head`` query tiles of each.
    Heads and query tiles are independent units of equal cost, so the full
    layer time is linear in them.
    """
    from oracle import Oracle
    o = Oracle()
    if threads:
        o.set_num_threads(threads)
    hs = list(range(heads))
    Qb = np.ascontiguousarray(t_host["Q"][:, hs])
    Kb = np.ascontiguousarray(t_host["K"][:, hs])
    Vb = np.ascontiguousarray(t_host["V"][:, hs])
    shapes = [w.tile_shapes[h] for h in hs]
    t0 = time.perf_counter()
    r = o.mask_prep(Qb, Kb, t_host["Wq"][hs], t_host["Wk"][hs], w.grid, shapes, w.k)
    t1 = time.perf_counter()
    rng = np.random.default_rng(0)
    units = np.array([(0, h, int(i)) for h in range(heads)
                      for i in rng.choice(w.nT, min(units_per_head, w.nT), replace=False)],
                     dtype=np.int64)
    o.sparse_attention(Qb, Kb, Vb, r["idx"], w.grid, shapes, w.scale, units=units)
    t2 = time.perf_counter()
    prep_per_head = (t1 - t0) / heads
    attn_per_unit = (t2 - t1) / len(units)
    full_s = prep_per_head * w.B * w.H + attn_per_unit * w.B * w.H * w.nT
    return dict(seconds_sampled=t2 - t0, full_layer_s=full_s, cores=o.num_threads(),
                sample=f"mask prep of {heads} head(s) + attention of {len(units)} query tiles "
                       f"of {w.name}; full layer extrapolated linearly over heads and query tiles")


def host_inputs(w, t):
    return {"Q": workloads.bf16_bits(t["Q"]), "K": workloads.bf16_bits(t["K"]),
            "V": workloads.bf16_bits(t["V"]), "Wq": t["Wq"].cpu().numpy(),
            "Wk": t["Wk"].cpu().numpy()}


# ---------------------------------------------------------------- reference arm
def run_reference(args, w, world, rank):
    if rank != 0:
        return 0
    # inputs drawn on the CPU: only the sampled heads are needed
    wh = workloads.Workload(w.name, w.B, 1, w.d, w.T, w.Hs, w.Ws, w.tile_shapes[:1], w.k,
                            w.sparsity, w.seed)
    t = workloads.generate(wh, device="cpu")
    th = host_inputs(wh, t)
    times = []
    res = None
    for s in range(args.warmup + args.steps):
        res = oracle_sample(w, th, heads=1, units_per_head=8)
        if s >= args.warmup:
            times.append(res["full_layer_s"])
    ms = 1e3 * statistics.mean(times)
    value = w.sparse_flops() / (ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(w, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": res["cores"],
                             "kind": "oracle", "sample": res["sample"]},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- main arm
def run_veda(args, w, world, rank, local):
    import tile_sparse_attention_b200 as vb
    vb.load_library()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = _peaks()
    t = workloads.generate(w, device=dev)
    prob = vb.Problem.from_workload(w)
    B, H, N, d, nT, k = w.B, w.H, w.N, w.d, w.nT, w.k
    statsQ = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device=dev)
    statsK = torch.empty_like(statsQ)
    S = torch.empty((B, H, nT, nT), dtype=torch.float32, device=dev)
    idx = torch.empty((B, H, nT, k), dtype=torch.int32, device=dev)
    O = torch.empty_like(t["Q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ws = vb.alloc_workspace(prob, dev)
    stream = torch.cuda.current_stream(dev)
    nk = 5  # CUDA events per step below (around tripool, tile score, topk, attention)
    # kernels of ours per step: tripool, both projections (one launch), score, topk, attention
    kernels_per_step = 5

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        vb.veda_tripool(prob, t["Q"], t["K"], statsQ, statsK)
        if ev is not None:
            ev[1].record(stream)
        vb.veda_tile_score(prob, statsQ, statsK, t["Wq"], t["Wk"], S, ws)
        if ev is not None:
            ev[2].record(stream)
        vb.veda_topk_mask(prob, S, None, idx)
        if ev is not None:
            ev[3].record(stream)
        vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], idx, O, lse, ws)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert vb.veda_get_status(ws) == 0, "device status after warm-up"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        _barrier(world)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for s in range(args.steps):
            step(evs[s])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        _barrier(world)
    clocks = clk.summary()
    status = vb.veda_get_status(ws)
    total_ms = start.elapsed_time(stop)
    total_ms = _max_over_ranks(total_ms, world)
    ms = total_ms / args.steps
    per = {n: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
           for i, n in enumerate(["tripool", "tile_score", "topk", "sparse_attn"])}
    flops = w.sparse_flops()
    value = _job_tflops(flops, ms, world)

    # mask-prep kernels as a fraction of HBM bandwidth (algorithmic bytes)
    tri_bytes = 2 * B * H * N * d * 2 + 2 * B * H * nT * 3 * d * 4
    stats_b = B * H * nT * 3 * d * 4
    score_bytes = 2 * stats_b + 2 * H * d * d * 4 + 2 * stats_b + 2 * stats_b + B * H * nT * nT * 4
    topk_bytes = B * H * nT * nT * 4 + B * H * nT * k * 4
    attn_tf = flops / (per["sparse_attn"] * 1e-3) / 1e12
    mask_prep = {
        "tripool": {"ms": per["tripool"], "GB_s": tri_bytes / per["tripool"] / 1e6,
                    "frac_hbm": tri_bytes / per["tripool"] / 1e6 / peaks["hbm"]},
        "tile_score": {"ms": per["tile_score"], "GB_s": score_bytes / per["tile_score"] / 1e6,
                       "frac_hbm": score_bytes / per["tile_score"] / 1e6 / peaks["hbm"],
                       "fp32_TFLOP_s": 2 * B * H * (2 * 3 * nT * d * d + nT * nT * 3 * d)
                       / (per["tile_score"] * 1e-3) / 1e12},
        "topk": {"ms": per["topk"], "GB_s": topk_bytes / per["topk"] / 1e6,
                 "frac_hbm": topk_bytes / per["topk"] / 1e6 / peaks["hbm"]},
    }

    # the build's own dense path (k = nT, no index list), outside the timed region
    dense_ms = None
    if not args.no_dense:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], None, O, lse, ws)
        e0.record(stream)
        vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], None, O, lse, ws)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        dense_ms = e0.elapsed_time(e1)

    # end to end through the public call with host buffers (pinned), every step:
    # veda_forward_host copies Q, K, V, Wq, Wk in, runs the layer and copies O
    # out, pipelined over chunks of heads (copies overlap the kernels).
    e2e = None
    if not args.no_e2e:
        hostQ = t["Q"].cpu().pin_memory()
        hostK = t["K"].cpu().pin_memory()
        hostV = t["V"].cpu().pin_memory()
        hostWq = t["Wq"].cpu().pin_memory()
        hostWk = t["Wk"].cpu().pin_memory()
        hostO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        dQ, dK, dV = torch.empty_like(t["Q"]), torch.empty_like(t["K"]), torch.empty_like(t["V"])
        dWq, dWk = torch.empty_like(t["Wq"]), torch.empty_like(t["Wk"])
        fws = vb.alloc_workspace(prob, dev)

        def e2e_step():
            vb.veda_forward_host(prob, hostQ, hostK, hostV, hostWq, hostWk, hostO, None, dQ, dK,
                                 dV, dWq, dWk, O, None, fws, 0)

        for _ in range(min(2, args.warmup)):
            e2e_step()
        torch.cuda.synchronize(dev)
        n_e2e = max(2, min(args.steps, 5))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        _barrier(world)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        _barrier(world)
        e_ms = _max_over_ranks(a.elapsed_time(b) / n_e2e, world)
        h2d = sum(x.numel() * x.element_size() for x in (hostQ, hostK, hostV, hostWq, hostWk))
        d2h = hostO.numel() * hostO.element_size()

        # the host link alone: plain pinned copies of the same bytes, one
        # direction at a time, on the same stream; the layer end to end can be
        # no faster than the slower direction
        def copy_ms(fn, reps=2):
            fn()
            torch.cuda.synchronize(dev)
            a2, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a2.record(stream)
            for _ in range(reps):
                fn()
            b2.record(stream)
            torch.cuda.synchronize(dev)
            return a2.elapsed_time(b2) / reps

        def h2d_copy():
            for d_, h_ in ((dQ, hostQ), (dK, hostK), (dV, hostV), (dWq, hostWq), (dWk, hostWk)):
                d_.copy_(h_, non_blocking=True)

        h2d_ms = copy_ms(h2d_copy)
        d2h_ms = copy_ms(lambda: hostO.copy_(O, non_blocking=True))
        floor_ms = max(h2d_ms, d2h_ms)
        e2e = {"value": _job_tflops(flops, e_ms, world), "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "link": {"h2d_GB_s": h2d / h2d_ms / 1e6, "d2h_GB_s": d2h / d2h_ms / 1e6,
                        "floor_ms": floor_ms, "frac": floor_ms / e_ms}}
        del hostQ, hostK, hostV, hostO, dQ, dK, dV

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        th = {n: workloads.bf16_bits(t[n].index_select(1, torch.tensor([0], device=dev)))
              for n in ("Q", "K", "V")}
        th["Wq"], th["Wk"] = t["Wq"].cpu().numpy(), t["Wk"].cpu().numpy()
        # about 10-15 s of fp64 work on the host cores at the long-video size
        res = oracle_sample(w, th, heads=1, units_per_head=512)
        cpu = {"value": flops / res["full_layer_s"] / 1e12, "unit": "TFLOP/s",
               "cores": res["cores"], "kind": "oracle", "sample": res["sample"],
               "seconds_sampled": res["seconds_sampled"],
               "full_layer_s_extrapolated": res["full_layer_s"]}

    if rank == 0:
        # the attention kernel is timed per launch (~50 ms): the burst peak applies
        peak = peaks["bf16"]
        traffic = ATTN_DRAM_BYTES.get(w.name)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": _config(w, world),
            "ms_per_layer": ms,
            "frac_of_peak": {"measured_bf16_burst": value / world / peaks["bf16"],
                             "measured_bf16_sustained": value / world / peaks["bf16_sus"],
                             "datasheet_dense_bf16_2250": value / world / 2250.0,
                             "peaks": peaks["source"]},
            "roofline": {"bound": "tensor", "kernel": "sparse_attn", "achieved": attn_tf,
                         "peak": peak, "unit": "TFLOP/s", "frac": attn_tf / peak,
                         "peak_kind": "bf16 burst (" + peaks["source"] + "), the kernel is "
                                      "timed per launch",
                         "frac_of_sustained": attn_tf / peaks["bf16_sus"],
                         "traffic": traffic["bytes"] if traffic else None,
                         "traffic_source": ({"kernel": traffic["kernel"],
                                             "capture": traffic["capture"]} if traffic else None),
                         "algorithmic_flops_per_launch": flops},
            "estimator_mask": key_tile_coverage(idx, nT),
            "kernels_ms": per,
            "mask_prep": mask_prep,
            "dense_path": {"attn_ms": dense_ms,
                           "speedup_attention": (dense_ms / per["sparse_attn"]) if dense_ms else None,
                           "speedup_layer": (dense_ms / ms) if dense_ms else None},
            "device_status": status,
            "gpu_launches": kernels_per_step * args.steps,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- mask kinds
def random_index_lists(w, device, seed=1):
    """Seeded index lists: per row, k distinct key tiles drawn uniformly, ascending."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    rows = w.B * w.H * w.nT
    out = torch.empty((rows, w.k), dtype=torch.int32, device=device)
    for r0 in range(0, rows, 8192):
        r1 = min(rows, r0 + 8192)
        u = torch.rand((r1 - r0, w.nT), generator=g, device=device)
        out[r0:r1] = u.topk(w.k, dim=1).indices.sort(dim=1).values.int()
    return out.view(w.B, w.H, w.nT, w.k)


def local_index_lists(w, device):
    """Per query tile, the k key tiles whose centres are nearest in (t, y, x)
    token coordinates (squared Euclidean distance, ties to the lower index):
    the spatio-temporal locality of video attention, ascending."""
    out = torch.empty((w.B, w.H, w.nT, w.k), dtype=torch.int32, device=device)
    for shape in sorted(set(w.tile_shapes)):
        pt, ph, pw = shape
        nh, nw = w.Hs // ph, w.Ws // pw
        j = torch.arange(w.nT, device=device, dtype=torch.int64)
        c = torch.stack([2 * (j // (nh * nw)) * pt + pt, 2 * ((j // nw) % nh) * ph + ph,
                         2 * (j % nw) * pw + pw], 1)  # doubled centres: integers
        lists = torch.empty((w.nT, w.k), dtype=torch.int32, device=device)
        for i0 in range(0, w.nT, 256):
            i1 = min(w.nT, i0 + 256)
            d2 = ((c[i0:i1, None, :] - c[None, :, :]) ** 2).sum(-1)
            key = d2 * w.nT + j[None, :]
            lists[i0:i1] = key.topk(w.k, dim=1, largest=False).indices.sort(dim=1).values.int()
        for h, sh in enumerate(w.tile_shapes):
            if sh == shape:
                out[:, h] = lists
    return out


def run_masks(args, w):
    """Attention alone on three kinds of index list at the same k: the
    estimator's mask (as in the layer), seeded uniformly random rows (every key
    tile in use, little reuse in L2) and the k nearest tiles in (t, y, x).  One
    JSON line per kind: time, effective TFLOP/s, fraction of the burst peak,
    key-tile coverage, clocks."""
    import tile_sparse_attention_b200 as vb
    vb.load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks = _peaks()
    t = workloads.generate(w, device=dev)
    prob = vb.Problem.from_workload(w)
    B, H, N, d, nT, k = w.B, w.H, w.N, w.d, w.nT, w.k
    ws = vb.alloc_workspace(prob, dev)
    est = torch.empty((B, H, nT, k), dtype=torch.int32, device=dev)
    vb.veda_forward(prob, t["Q"], t["K"], t["V"], t["Wq"], t["Wk"], torch.empty_like(t["Q"]),
                    None, est, None, ws)
    kinds = {"estimator": est, "random": random_index_lists(w, dev), "local": local_index_lists(w, dev)}
    O = torch.empty_like(t["Q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    flops = w.sparse_flops()
    reps = max(3, args.steps)
    for name, idx in kinds.items():
        fn = lambda: vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], idx, O, lse, ws)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        with ClockSampler(0) as clk:
            for r in range(reps):
                evs[r].record(stream)
                fn()
            evs[reps].record(stream)
            torch.cuda.synchronize(dev)
        ms = statistics.median(evs[r].elapsed_time(evs[r + 1]) for r in range(reps))
        tf = flops / (ms * 1e-3) / 1e12
        print(json.dumps({"row": "attention by mask kind", "mask": name, "workload": w.name,
                          "k": k, "launches": reps, "ms_median": ms, "TFLOP_s": tf,
                          "frac_bf16_burst": tf / peaks["bf16"],
                          "frac_bf16_sustained": tf / peaks["bf16_sus"],
                          "coverage": key_tile_coverage(idx, nT), "clocks": clk.summary(),
                          "status": vb.veda_get_status(ws)}), flush=True)
    return 0


# ---------------------------------------------------------------- next rows
def run_sweep(args):
    """The sweep: H=24, d=128, 48x80 latent plane, T frames, sparsity levels
    (one JSON line per point: layer time, effective TFLOP/s, and the speedup of
    the attention and of the layer over the dense schedule at the same T)."""
    import tile_sparse_attention_b200 as vb
    vb.load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks = _peaks()

    def timed(fn, reps, warm=2):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    for T in workloads.SWEEP_T:
        w0 = workloads.sweep(T, workloads.SWEEP_SPARSITY[0])
        t = workloads.generate(w0, device=dev)
        B, H, N, d, nT = w0.B, w0.H, w0.N, w0.d, w0.nT
        statsQ = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device=dev)
        statsK = torch.empty_like(statsQ)
        S = torch.empty((B, H, nT, nT), dtype=torch.float32, device=dev)
        O = torch.empty_like(t["Q"])
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        dense_ms = None
        for sp in workloads.SWEEP_SPARSITY:
            w = workloads.sweep(T, sp)
            prob = vb.Problem.from_workload(w)
            ws = vb.alloc_workspace(prob, dev)
            idx = torch.empty((B, H, nT, w.k), dtype=torch.int32, device=dev)
            if dense_ms is None:
                dense_ms = timed(lambda: vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], None, O,
                                                             lse, ws), reps=2, warm=1)

            def layer():
                vb.veda_tripool(prob, t["Q"], t["K"], statsQ, statsK)
                vb.veda_tile_score(prob, statsQ, statsK, t["Wq"], t["Wk"], S, ws)
                vb.veda_topk_mask(prob, S, None, idx)
                vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], idx, O, lse, ws)
            reps = 3 if w.k * nT <= 400_000 else 2
            with ClockSampler(0) as clk:
                ms = timed(layer, reps)
                attn_ms = timed(lambda: vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], idx, O,
                                                            lse, ws), reps)
            print(json.dumps({"row": "sweep", "workload": w.name, "T": T, "tokens": N, "tiles": nT,
                              "sparsity_pct": sp, "k": w.k, "ms_per_layer": ms, "attn_ms": attn_ms,
                              "TFLOP_s": w.sparse_flops() / (ms * 1e-3) / 1e12,
                              "attn_TFLOP_s": w.sparse_flops() / (attn_ms * 1e-3) / 1e12,
                              "attn_frac_bf16_burst": w.sparse_flops() / (attn_ms * 1e-3) / 1e12
                              / peaks["bf16"],
                              "dense_attn_ms": dense_ms, "speedup_attention": dense_ms / attn_ms,
                              "speedup_layer": dense_ms / ms, "clocks": clk.summary(),
                              "status": vb.veda_get_status(ws)}),
                  flush=True)
            del ws, idx
        del t, statsQ, statsK, S, O, lse
        torch.cuda.empty_cache()
    return 0


def run_rows(args, w, rows):
    """Times the training-side rows on `w` (one JSON line per row)."""
    import tile_sparse_attention_b200 as vb
    vb.load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    t = workloads.generate(w, device=dev)
    prob = vb.Problem.from_workload(w)
    B, H, N, d, nT, k = w.B, w.H, w.N, w.d, w.nT, w.k
    ws = vb.alloc_workspace(prob, dev)
    stream = torch.cuda.current_stream(dev)
    peaks = _peaks()

    def timed(fn, reps=3):
        fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    O = torch.empty_like(t["Q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    T = torch.empty((B, H, nT, nT), dtype=torch.float32, device=dev)
    dense_flops = w.dense_flops()
    qk_flops = dense_flops / 2
    if "f1" in rows:
        ms_teacher = timed(lambda: vb.veda_teacher(prob, t["Q"], t["K"], t["V"], O, lse, T, ws))
        ms_dense = timed(lambda: vb.veda_sparse_attn(prob, t["Q"], t["K"], t["V"], None, O, lse, ws))
        idx_o = torch.empty((B, H, nT, k), dtype=torch.int32, device=dev)
        idx_p = torch.empty_like(idx_o)
        ms_mask = timed(lambda: vb.veda_topk_mask(prob, T, None, idx_o))
        vb.veda_forward(prob, t["Q"], t["K"], t["V"], t["Wq"], t["Wk"], O, None, idx_p, None, ws)
        mean = torch.empty((1,), dtype=torch.float64, device=dev)
        ms_rec = timed(lambda: vb.veda_tile_recall(prob, idx_p, idx_o, None, mean, ws))
        ms_qk = ms_teacher - ms_dense
        print(json.dumps({"row": "f1 teacher + oracle mask + tile recall", "workload": w.name,
                          "teacher_ms": ms_teacher, "dense_attention_ms": ms_dense,
                          "teacher_qk_pass_ms": ms_qk,
                          "teacher_qk_TFLOP_s": qk_flops / (ms_qk * 1e-3) / 1e12,
                          "frac_bf16_burst": qk_flops / (ms_qk * 1e-3) / 1e12 / peaks["bf16"],
                          "oracle_mask_ms": ms_mask, "recall_ms": ms_rec,
                          "tile_recall_random_weights": mean.item(),
                          "status": vb.veda_get_status(ws)}), flush=True)
    if "f3" in rows:
        statsQ = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device=dev)
        statsK = torch.empty_like(statsQ)
        S = torch.empty((B, H, nT, nT), dtype=torch.float32, device=dev)
        vb.veda_tripool(prob, t["Q"], t["K"], statsQ, statsK)
        vb.veda_tile_score(prob, statsQ, statsK, t["Wq"], t["Wk"], S, ws)
        vb.veda_teacher(prob, t["Q"], t["K"], t["V"], O, lse, T, ws)
        loss = torch.empty((1,), dtype=torch.float64, device=dev)
        dWq, dWk = torch.empty_like(t["Wq"]), torch.empty_like(t["Wk"])
        dws = torch.empty(vb.veda_distill_workspace_size(prob), dtype=torch.uint8, device=dev)
        ms = timed(lambda: vb.veda_distill_kl(prob, statsQ, statsK, t["Wq"], t["Wk"], S, T, 1.0,
                                              loss, dWq, dWk, dws))
        gflop = 2 * B * H * (2 * 3 * nT * d * d + 2 * nT * nT * 3 * d + 2 * 3 * nT * d * d) / 1e9
        print(json.dumps({"row": "f3 KL distillation loss + dWq/dWk", "workload": w.name,
                          "ms": ms, "fp32_GFLOP": gflop,
                          "fp32_TFLOP_s": gflop / ms, "loss": loss.item(),
                          "status": vb.veda_get_status(dws)}), flush=True)
    if "f2" in rows:
        cands = [c for c in workloads.HEAD_SHAPES
                 if w.T % c[0] == 0 and w.Hs % c[1] == 0 and w.Ws % c[2] == 0]
        Oc = torch.empty_like(t["Q"])
        err = torch.empty((len(cands), B, H), dtype=torch.float64, device=dev)
        best = torch.empty((H,), dtype=torch.int32, device=dev)
        p0 = vb.Problem(B, H, d, w.grid, [cands[0]], k)
        ms = timed(lambda: vb.veda_tile_search(p0, cands, t["Q"], t["K"], t["V"], t["Wq"],
                                               t["Wk"], O, Oc, err, best, ws), reps=2)
        picks = np.bincount(best.cpu().numpy(), minlength=len(cands)).tolist()
        print(json.dumps({"row": "f2 head-aware tile search", "workload": w.name,
                          "candidates": cands, "ms": ms, "heads_per_candidate": picks,
                          "status": vb.veda_get_status(ws)}), flush=True)
    if "f4" in rows:
        statsQ = torch.empty((B, H, nT, 3, d), dtype=torch.float32, device=dev)
        statsK = torch.empty_like(statsQ)
        vb.veda_tripool(prob, t["Q"], t["K"], statsQ, statsK)
        S = torch.empty((B, H, nT, nT), dtype=torch.float32, device=dev)
        idx2 = torch.empty((B, H, nT, k), dtype=torch.int32, device=dev)
        idxf = torch.empty_like(idx2)
        ms_two = timed(lambda: (vb.veda_tile_score(prob, statsQ, statsK, t["Wq"], t["Wk"], S, ws),
                                vb.veda_topk_mask(prob, S, None, idx2)), reps=10)
        ms_fused = timed(lambda: vb.veda_mask_fused(prob, statsQ, statsK, t["Wq"], t["Wk"], None,
                                                    idxf, ws), reps=10)
        same = bool(torch.equal(idx2, idxf))
        # fp8 (E4M3) estimator weights: quantise, dequantise, mask, recall vs fp32
        W8 = torch.empty((H, d, d), dtype=torch.uint8, device=dev)
        sc = torch.empty((H,), dtype=torch.float32, device=dev)
        deq = {}
        for name in ("Wq", "Wk"):
            vb.veda_quantize_fp8(t[name], W8, sc)
            deq[name] = torch.empty_like(t[name])
            vb.veda_dequantize_fp8(W8, sc, deq[name])
        ms_q = timed(lambda: vb.veda_quantize_fp8(t["Wq"], W8, sc), reps=10)
        ms_dq = timed(lambda: vb.veda_dequantize_fp8(W8, sc, deq["Wq"]), reps=10)
        idx8 = torch.empty_like(idx2)
        vb.veda_mask_fused(prob, statsQ, statsK, deq["Wq"], deq["Wk"], None, idx8, ws)
        mean = torch.empty((1,), dtype=torch.float64, device=dev)
        vb.veda_tile_recall(prob, idx8, idxf, None, mean, ws)
        torch.cuda.synchronize(dev)
        print(json.dumps({"row": "f4 fused mask prep + fp8 estimator weights", "workload": w.name,
                          "score_plus_topk_ms": ms_two, "fused_mask_ms": ms_fused,
                          "fused_equals_two_call": same, "S_bytes_not_written": S.numel() * 4,
                          "fp8_quantize_ms": ms_q, "fp8_dequantize_ms": ms_dq,
                          "weight_bytes_fp32": 2 * H * d * d * 4, "weight_bytes_fp8": 2 * H * (d * d + 4),
                          "tile_recall_fp8_vs_fp32_mask": mean.item(),
                          "status": vb.veda_get_status(ws)}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["veda", "reference"], default="veda")
    ap.add_argument("--workload", default="long_video",
                    help="long_video | 720p | 480p | tiny | sweep:T:sparsity")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time the sweep points (T x sparsity) instead")
    ap.add_argument("--masks", action="store_true",
                    help="time the attention alone on estimator, random and local index lists")
    ap.add_argument("--rows", default="",
                    help="comma list of f1,f2,f3,f4: time the next rows instead")
    ap.add_argument("--heads", type=int, default=0,
                    help="long_video with its first N heads only (a smaller case for counter captures)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "veda":
        args.warmup = 3
    if args.workload.startswith("sweep:"):
        _, T, s = args.workload.split(":")
        w = workloads.sweep(int(T), int(s))
    elif args.heads and args.workload == "long_video":
        w = workloads.long_video(H=args.heads)
    else:
        w = workloads.CONFIGS[args.workload]()
    if args.sweep:
        return run_sweep(args)
    if args.rows:
        return run_rows(args, w, set(args.rows.split(",")))
    if args.masks:
        return run_masks(args, w)
    world, rank, local = _dist_init()
    try:
        if args.impl == "reference":
            return run_reference(args, w, world, rank)
        return run_veda(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
