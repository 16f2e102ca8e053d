"""Benchmark of the tile-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config small] [--impl ours|reference]

One step = the whole hot path over one batch of the workload: scatter Q, K, V into 4x4x4 tile
order, coarse selection (pool Q and K, score tile pairs, keep the top-k key tiles per query tile;
or the workload's own selection mode), block-sparse attention over the kept tile pairs, gather the
output back to raster order. Inputs are resident in HBM when the timed region starts; the raster
Q, K, V (264 MB at the small layer) exceed the 126 MB L2, so no flush is inserted.

The metric is effective TFLOPS over kept blocks (4 * 64 * 64 * D FLOPs per kept query-tile /
key-tile pair) per step, with ms per call, and the fraction of the roofline of the dominant kernel
(the attention) measured live with CUDA events. ``e2e`` repeats the measurement through the public
API with host buffers: every step copies Q, K, V from pinned host memory and the output back.

With N > 1 (torchrun), every rank runs its own replica of the workload (independent batches, no
data exchange; weak scaling), or with ``--shard heads`` the ranks share one layer by head, each
taking a contiguous head range of the same full-width rows (strong scaling, still no exchange);
``value`` is the kept-block FLOPs of all ranks over the max-over-ranks time.

``--impl reference`` times the CPU oracle (fp64 numpy) on a bounded sample of the same workload
on the host cores; it is the reported CPU baseline, not a target.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/call and effective TFLOPS (kept blocks) at 28,672 tok×12 heads; % of roofline"
FLOPS_PER_PAIR = lambda D: 4 * 64 * 64 * D  # noqa: E731


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def _describe(w) -> str:
    sel = {"topk": f"top-{w.k} of {w.nT} tiles",
           "bsa": f"BSA: prune cos>{w.cos_thresh}, mass {w.mass}",
           "mask": f"fixed {w.mask} block mask"}[w.mode]
    return (f"{w.name}: B={w.B}, heads={w.heads}, D={w.D}, grid {w.T}x{w.H}x{w.W} "
            f"({w.L:,} tokens, {w.nT} tiles of 4x4x4), {sel}")


# --------------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the measured window."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 100):
        self.index = index
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(period_ms)],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        with open(self.file.name) as f:
            rows = [[c.strip() for c in ln.split(",")] for ln in f if ln.strip()]
        os.unlink(self.file.name)
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------------- oracle arm

def oracle_sample(w, q, k, v, heads, q_tiles_per_head=None):
    """Run the CPU oracle's whole path for the given heads (tiling, pooling, scores, selection,
    attention for the first ``q_tiles_per_head`` query tiles, or all). Returns (seconds, flops,
    pairs) for the sample."""
    import numpy as np
    import torch

    from oracle import attention, bsa, pool, select, tiling

    D = w.D
    t0 = time.perf_counter()
    pairs = 0
    vc = tiling.variable_block_sizes(w.T, w.H, w.W)
    mask = None
    if w.mode == "mask":
        from block_sparse_video_tile3d_b200 import workloads
        mask = workloads.block_mask(w).numpy()
    for b in range(w.B):
        for h in heads:
            sl = lambda x: x[b:b + 1, :, h:h + 1].to(torch.float64).numpy()  # noqa: E731
            qt, kt, vt = (tiling.tile_scatter(sl(x), w.T, w.H, w.W) for x in (q, k, v))
            keep = src = None
            if w.mode == "mask":
                sets = select.map_to_sets(mask[b:b + 1, h:h + 1])
            else:
                pk = pool.tile_mean_pool(kt, vc)
                if w.mode == "bsa":
                    keep, src, _ = bsa.prune_queries(qt, w.cos_thresh)
                    pq = bsa.pooled_kept_queries(qt, keep)
                else:
                    pq = pool.tile_mean_pool(qt, vc)
                S = select.tile_scores(pq, pk)
                sets = select.select_topk(S, w.k) if w.mode == "topk" else \
                    select.select_mass(S, w.scale, w.mass, w.min_kv)
            n = w.nT if q_tiles_per_head is None else min(q_tiles_per_head, w.nT)
            tiles = [(0, 0, i) for i in range(n)]
            attention.block_sparse_attention(qt, kt, vt, vc, sets, w.scale, keep=keep, src=src,
                                             q_tiles=tiles)
            pairs += sum(len(sets[0][0][i]) for i in range(n))
    sec = time.perf_counter() - t0
    return sec, pairs * FLOPS_PER_PAIR(D), pairs


def _cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, q, k, v, budget_s: float = 20.0) -> dict:
    """Oracle throughput on a bounded sample (about ``budget_s`` of CPU work), in TFLOPS over the
    kept blocks it computed, with the full-call time extrapolated from it."""
    # calibrate on a quarter of one head, then size the sample in whole heads
    sec, fl, pairs = oracle_sample(w, q, k, v, [0], max(1, w.nT // 4))
    per_head = sec * 4
    nh = int(max(1, min(w.heads, budget_s // max(per_head, 1e-3))))
    sec, fl, pairs = oracle_sample(w, q, k, v, list(range(nh)))
    tflops = fl / sec / 1e12
    scale_up = (w.B * w.heads) / (w.B * nh)
    return {"value": tflops, "unit": "TFLOPS", "cores": _cores(), "kind": "oracle",
            "ms_per_call_est": sec * scale_up * 1e3,
            "sample": (f"fp64 numpy oracle, whole path (tile, pool, score, select, attend all "
                       f"{w.nT} query tiles) for heads 0..{nh - 1} of {w.heads} x batch {w.B}: "
                       f"{pairs:,} kept pairs in {sec:.1f} s; ms_per_call_est scales by "
                       f"{scale_up:.1f}")}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from block_sparse_video_tile3d_b200 import workloads
    q, k, v = workloads.make_qkv(w)
    n = max(1, w.nT // 8)  # bounded sample per step: one head, an eighth of its query tiles

    def step(h):
        return oracle_sample(w, q, k, v, [h % w.heads], n)

    for s in range(args.warmup):
        step(s)
    tot_s = tot_f = 0.0
    tot_pairs = 0
    for s in range(args.steps):
        sec, fl, pairs = step(s)
        tot_s += sec
        tot_f += fl
        tot_pairs += pairs
    tflops = tot_f / tot_s / 1e12
    sample = (f"fp64 numpy oracle, per step: one head's tiling, pooling, scores and selection plus "
              f"attention for {n} of its {w.nT} query tiles ({tot_pairs // max(args.steps, 1):,} "
              f"kept pairs)")
    line = {"metric": METRIC, "value": tflops, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_s / max(args.steps, 1) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": _describe(w), "l2": "n/a (host CPU)"},
            "cpu_baseline": {"value": tflops, "unit": "TFLOPS", "cores": _cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": tflops, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------ ranks (N > 1 replicas)
# The path has no exchange step: every rank runs the whole hot path on a problem of its own (a
# different seed of the same workload shape), so the only collectives are the host-side ones
# below: a barrier around the timed region, the max of the ranks' times and the sum of their FLOPs.

def rank_env() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_workload(w, rank: int):
    """The workload of one rank: the same shape, its own seed (rank 0 keeps the base seed)."""
    return w if rank == 0 else w.with_(seed=w.seed + 1_000_003 * rank)


def reduce_over_ranks(x: float, op: str, world: int, device=None) -> float:
    """Max or sum of a host scalar over all ranks (identity with one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def whole_job_tflops(flops_all_ranks: float, ms_per_step_max: float) -> float:
    """Throughput of the whole job: the FLOPs of every rank's step over the slowest rank's step."""
    return flops_all_ranks / (ms_per_step_max * 1e-3) / 1e12


# --------------------------------------------------------------------------------- our arm

def _stage_bytes(w, name, pairs, kmax):
    """Algorithmic HBM bytes of one stage launch (each input read once, each output written once)."""
    B, heads, D, L, Lp, nT = w.B, w.heads, w.D, w.L, 64 * w.nT, w.nT
    row = heads * D * 2
    if name.startswith("scatter_pool"):
        return B * L * row + B * Lp * row + B * heads * nT * D * 4
    if name.startswith("scatter"):
        return B * L * row + B * Lp * row
    if name == "gather":
        return 2 * B * L * row
    if name.startswith("pool"):
        return B * L * row + B * heads * nT * D * 4
    if name == "prune_q":
        return B * L * row + B * heads * nT * (D * 4 + 128)
    if name.startswith("select"):
        return 2 * B * heads * nT * D * 4 + B * heads * nT * (kmax + 1) * 4
    if name == "mask_to_index":
        return B * heads * nT * nT + B * heads * nT * (kmax + 1) * 4
    if name == "attention":
        return 4 * B * Lp * row + B * heads * nT * (kmax + 1) * 4
    return 0


ATTN_SOURCES = ("attn_sm100.cu", "common.cuh", "kernels.h", "sm100.cuh")  # the forward kernel's


def _source_sha() -> str:
    """Hash of the sources the forward attention kernel is compiled from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_video_tile3d_b200", "csrc")
    for n in sorted(ATTN_SOURCES):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode() + f.read())
    return h.hexdigest()[:16]


# Kernels of this library one call of each stage launches, read off the launch code (csrc/*.cu);
# used only when the profiler count below is unavailable. The attention calls also issue a 4-byte
# memset of the work-queue counter, which is not a kernel of this library.
STATIC_KERNELS = {
    "scatter_q": 1, "scatter_k": 1, "scatter_v": 1, "scatter_pool_q": 1, "scatter_pool_k": 1,
    "mask_to_index": 1, "prune_q": 1,
    "select_topk": 3,   # split, tensor-core scores, top-k rows
    "select_mass": 4,   # split, scores, mass rows, floor / cap fix-up
    "select": 3,        # packed: split, scores, per-span rows
    "attention": 1,
    "attention_packed": 2,  # packed: list rewrite into 64-row halves, attention
    "gather": 1,
    "backward": 5,      # dOe / delta, kept-pair map, key-to-query lists, dQ, dK / dV
}


def count_launches(stages, packed: bool = False) -> tuple[dict, str]:
    """Kernels each stage launches, counted on the device: every stage runs once more (untimed)
    under torch.profiler's CUDA activity trace and its kernel records are counted (memsets and
    copies excluded). Falls back to STATIC_KERNELS if the profiler cannot trace."""
    import torch
    key = {"attention": "attention_packed"} if packed else {}
    static = {n: STATIC_KERNELS[key.get(n, n)] for n, _ in stages}
    if os.environ.get("CUDA_INJECTION64_PATH"):  # under ncu: leave CUPTI to it
        return static, "static (launch code); another profiler is attached"
    try:
        from torch.autograd import DeviceType
        from torch.profiler import ProfilerActivity, profile
        counts = {}
        for name, launch in stages:
            torch.cuda.synchronize()
            with profile(activities=[ProfilerActivity.CUDA]) as prof:
                launch()
                torch.cuda.synchronize()
            counts[name] = sum(1 for e in prof.events()
                               if e.device_type == DeviceType.CUDA
                               and not e.name.startswith(("Memset", "Memcpy", "[")))
        if min(counts.values()) < 1:  # every stage launches at least one kernel
            return static, "static (launch code); the profiler recorded no kernels"
        return counts, "torch.profiler CUDA kernel records, one untimed call per stage"
    except Exception as exc:  # noqa: BLE001 - the count is a report, not a result
        return static, f"static (launch code); profiler unavailable: {type(exc).__name__}"


def _ncu_traffic(workload: str):
    """Per-launch DRAM bytes of the attention kernel from ``profiles/attn_traffic.json`` (written
    from an ncu capture), if that capture was taken on the current kernel source; else None. The
    file maps a workload name to ``{"source_sha": ..., "dram_bytes_per_launch": ...}``."""
    p = os.path.join(ROOT, "profiles", "attn_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f).get(workload)
        if rec and rec.get("source_sha") == _source_sha():
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    from block_sparse_video_tile3d_b200 import TileSparseAttention, workloads

    from block_sparse_video_tile3d_b200.sharding import head_partition

    world, rank, local = rank_env()
    shard_heads = args.shard == "heads" and world > 1
    if shard_heads and world > w.heads:
        raise SystemExit(f"--shard heads needs at most {w.heads} ranks for {w.name}")
    if not shard_heads:
        w = rank_workload(w, rank)
    h0, nh = head_partition(w.heads, world, rank) if shard_heads else (0, w.heads)
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    q, k, v = workloads.make_qkv(w)  # in head mode every rank holds the same full-width layer
    mask = workloads.block_mask(w)[:, h0:h0 + nh].contiguous() if w.mode == "mask" else None
    if w.mode == "bsa":
        pass  # the benchmark runs the workload's own data; query pruning drops what it finds
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    od = torch.empty_like(qd)
    model = TileSparseAttention(w.B, w.T, w.H, w.W, nh, w.D, mode=w.mode, topk=w.k or None,
                                mass=w.mass, min_k=w.min_kv, cos_thresh=w.cos_thresh, mask=mask,
                                device=dev, head0=h0, heads_total=w.heads)
    stages = model.stages(qd, kd, vd, od)
    names = [n for n, _ in stages]

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_over_ranks(x, "max", world, dev)

    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    for _ in range(max(args.warmup, 3)):
        for _, launch in stages:
            launch()
    torch.cuda.synchronize()
    pairs = int(model.kv_cnt.sum().item())
    flops = pairs * FLOPS_PER_PAIR(w.D)  # what the attention kernel computes: every row of a pair
    if model.keep is not None:
        # BSA: a pair's work counts the query rows that attend, 4 * kept_rows * 64 * D
        kept_rows = model.keep.to(torch.int64).sum(-1)
        flops_metric = int((model.kv_cnt.to(torch.int64) * kept_rows).sum().item()) * 4 * 64 * w.D
    else:
        flops_metric = flops
    flops_all = reduce_over_ranks(float(flops_metric), "sum", world, dev)

    # ---- device-resident timed region, events between stages on the launching stream
    nst = len(stages)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for s in range(args.steps):
        ev[s][0].record()
        for j, (_, launch) in enumerate(stages):
            launch()
            ev[s][j + 1].record()
    torch.cuda.synchronize()
    barrier()
    total_ms = ev[0][0].elapsed_time(ev[-1][-1])
    stage_ms = {n: sum(ev[s][j].elapsed_time(ev[s][j + 1]) for s in range(args.steps)) / args.steps
                for j, n in enumerate(names)}
    clocks = sampler.stop()
    launches, launch_src = count_launches(stages)
    total_ms = max_over_ranks(total_ms)
    ms_step = total_ms / args.steps
    status = model.device_status()

    # ---- end to end through the public API with pinned host buffers. Steps are pipelined the way a
    # serving loop would run them: each step's inputs go host -> device on one copy stream and its
    # output device -> host on another, into double-buffered device tensors, so step i + 1's upload
    # overlaps step i's compute and download. Every step's copies lie inside the timed region.
    # Two different host inputs alternate (set i & 1 for step i, with buffer i & 1), each with its
    # own reference output from the device-resident path, and every step's download is compared
    # with its reference, so a race between an upload and the compute that reads it would show.
    ref_out = [od.cpu()]
    q2, k2, v2 = workloads.make_qkv(w, seed=w.seed + 7)
    hosts = [tuple(x.pin_memory() for x in (q, k, v)), tuple(x.pin_memory() for x in (q2, k2, v2))]
    ins = [(qd, kd, vd), tuple(torch.empty_like(x) for x in (qd, kd, vd))]
    outs = [od, torch.empty_like(od)]
    for dst, src in zip(ins[1], hosts[1]):
        dst.copy_(src)
    model.forward(*ins[1], outs[1])
    torch.cuda.synchronize()
    ref_out.append(outs[1].cpu())
    out_bytes = od.numel() * od.element_size()
    e2e_steps = max(4, min(args.steps, 20, int(2e9 // out_bytes)))
    e2e_steps += e2e_steps & 1
    ohs = [torch.empty(od.shape, dtype=od.dtype).pin_memory() for _ in range(e2e_steps)]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_loop(n_steps):
        in_free = [None, None]   # compute of the step that last read input buffer b has finished
        out_free = [None, None]  # download of the step that last wrote output buffer b has finished
        done = None
        for i in range(n_steps):
            b = i & 1
            with torch.cuda.stream(up):
                if in_free[b] is not None:
                    up.wait_event(in_free[b])
                for dst, src in zip(ins[b], hosts[b]):
                    dst.copy_(src, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(up)
            comp.wait_event(ready)
            if out_free[b] is not None:
                comp.wait_event(out_free[b])
            model.forward(*ins[b], outs[b])
            computed = torch.cuda.Event()
            computed.record(comp)
            in_free[b] = computed
            with torch.cuda.stream(down):
                down.wait_event(computed)
                ohs[i].copy_(outs[b], non_blocking=True)
                done = torch.cuda.Event()
                done.record(down)
            out_free[b] = done
        comp.wait_event(done)
        for st in (up, down):  # the next region starts after every copy of this one
            st.wait_stream(comp)

    e2e_loop(2)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    up.wait_event(e0)
    down.wait_event(e0)
    e2e_loop(e2e_steps)
    e1.record(comp)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / e2e_steps
    e2e_same = all(torch.equal(ohs[i][:, :, h0:h0 + nh], ref_out[i & 1][:, :, h0:h0 + nh])
                   for i in range(e2e_steps))  # this rank's heads

    peaks = _peaks()
    wb = w.with_(heads=nh)  # this rank's share of the bytes
    attn_ms = stage_ms["attention"]
    achieved = flops / (attn_ms * 1e-3) / 1e12
    kmax = model.kmax
    stage_report = {}
    for n in names:
        byt = _stage_bytes(wb, n, pairs, kmax)
        stage_report[n] = {"ms": round(stage_ms[n], 4),
                           "gbs": round(byt / (stage_ms[n] * 1e-3) / 1e9, 1) if byt else None,
                           "bytes": byt}
    coarse_ms = sum(stage_ms[n] for n in names if n != "attention")
    coarse_bytes = sum(_stage_bytes(wb, n, pairs, kmax) for n in names if n != "attention")
    line = {
        "metric": METRIC,
        "value": whole_job_tflops(flops_all, ms_step),
        "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "ms_per_call": ms_step,
        "higher_is_better": True, "scaling": "strong" if shard_heads else "weak",
        "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": _describe(w), "kept_pairs": pairs,
                   "kept_block_gflop": flops / 1e9,
                   "metric_gflop": flops_metric / 1e9,
                   "metric_flops": ("4 * kept query rows * 64 * D per kept pair (pruned rows are "
                                    "computed but not counted)") if model.keep is not None else
                                   "4 * 64 * 64 * D per kept pair",
                   "density": pairs / (w.B * w.heads * w.nT * w.nT),
                   "l2": "no flush: raster Q/K/V inputs of "
                         f"{3 * w.B * w.L * w.heads * w.D * 2 / 1e6:.0f} MB exceed the 126 MB L2",
                   "parallelism": (f"one layer shared out by head over {world} GPUs (this rank: "
                                   f"heads {h0}..{h0 + nh - 1}), no data exchange")
                                  if shard_heads else
                                  f"{world} independent replica(s), one per GPU, each with its "
                                  "own seed of the workload"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "traffic": _ncu_traffic(w.name), "kernel": "block_sparse_attn_fwd",
                     "peak_source": f"{peaks['source']} bf16 dense (burst)",
                     "ms_per_launch": attn_ms},
        "coarse_and_tiling": {"ms": coarse_ms, "bytes": coarse_bytes,
                              "gbs": coarse_bytes / (coarse_ms * 1e-3) / 1e9,
                              "frac_hbm": coarse_bytes / (coarse_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                              "hbm_peak_gbs": peaks["hbm_gbs"]},
        "stages": stage_report,
        "e2e": {"value": whole_job_tflops(flops_all, e2e_ms), "unit": "TFLOPS",
                "ms_per_step": e2e_ms, "steps": e2e_steps, "output_matches_device_run": e2e_same,
                "pipelining": "host-to-device and device-to-host copies on their own streams, "
                              "double-buffered device tensors: step i + 1's upload overlaps step "
                              "i's compute and download",
                "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                "d2h_bytes_per_step": od.numel() * od.element_size()},
        "gpu_launches": args.steps * sum(launches.values()),
        "gpu_launches_per_step": {"by_stage": launches, "source": launch_src},
        "device_status": status,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, q, k, v, budget_s=args.cpu_budget)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_backward(args, w):
    """The backward pass on one GPU: selection and forward (with log-sum-exp) once, then K timed
    calls of block_sparse_attn_bwd for a seeded output gradient. FLOPs count the five products of
    the backward per kept pair (S = QK^T, dP = dO V^T, dV = P^T dO, dQ = dS K, dK = dS^T Q), each
    2 * 64 * 64 * D, whatever the kernels recompute."""
    import torch

    from block_sparse_video_tile3d_b200 import (TileSparseAttention, block_sparse_attn_bwd,
                                                block_sparse_attn_fwd_lse, tile3d_scatter,
                                                workloads)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    q, k, v = workloads.make_qkv(w)
    do = workloads.make_qkv(w, seed=w.seed + 11)[0]
    mask = workloads.block_mask(w) if w.mode == "mask" else None
    model = TileSparseAttention(w.B, w.T, w.H, w.W, w.heads, w.D, mode=w.mode, topk=w.k or None,
                                mass=w.mass, min_k=w.min_kv, cos_thresh=w.cos_thresh, mask=mask,
                                device=dev)
    model(q.to(dev), k.to(dev), v.to(dev))
    dot = tile3d_scatter(do.to(dev), w.T, w.H, w.W)
    o, lse = block_sparse_attn_fwd_lse(model.qt, model.kt, model.vt, model.kv_idx, model.kv_cnt,
                                       w.T, w.H, w.W, keep=model.keep, src_row=model.src_row)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    grads = [torch.empty_like(o) for _ in range(3)]

    def call():
        block_sparse_attn_bwd(model.qt, model.kt, model.vt, o, dot, lse, model.kv_idx,
                              model.kv_cnt, w.T, w.H, w.W, keep=model.keep, src_row=model.src_row,
                              dq=grads[0], dk=grads[1], dv=grads[2], dev_status=status)

    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    sampler = ClockSampler(0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    launches, launch_src = count_launches([("backward", call)])
    ms = e0.elapsed_time(e1) / args.steps
    pairs = int(model.kv_cnt.sum().item())
    flops = pairs * 10 * 64 * 64 * w.D
    peaks = _peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    line = {"metric": "backward: TFLOPS over kept blocks (5 products of 2*64*64*D per kept pair)",
            "value": tflops, "unit": "TFLOPS", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "pass": "backward",
            "config": {"workload": _describe(w), "kept_pairs": pairs, "gflop": flops / 1e9,
                       "l2": "no flush: Q, K, V, O, dO in tile order exceed the 126 MB L2"},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"],
                         "traffic": None, "kernel": "block_sparse_attn_bwd (all launches)",
                         "peak_source": f"{peaks['source']} bf16 dense (burst)"},
            "gpu_launches": args.steps * launches["backward"],
            "gpu_launches_per_step": {"by_stage": launches, "source": launch_src},
            "device_status": int(status.item()), "clocks": clocks}
    print(json.dumps(line), flush=True)
    return 0


def packed_oracle_sample(w, geo_ref, q, k, v, heads, q_tiles=None):
    """The CPU oracle's packed path for the given heads (scatter, pooling, scores, per-region
    selection, attention for the first ``q_tiles`` query tiles or all). Returns (seconds, flops,
    pairs)."""
    import torch

    from oracle import attention, packed, pool, select

    E = geo_ref["E"]
    t0 = time.perf_counter()
    pairs = 0
    rates = packed.span_keep_rates(len(geo_ref["spans"]), w.sparsity, w.ref_keep_rate, True)
    nT = len(geo_ref["vc"])
    for b in range(w.B):
        for h in heads:
            sl = lambda x: x[b:b + 1, :, h:h + 1].to(torch.float64).numpy()  # noqa: E731
            qt, kt, vt = (packed.scatter(sl(x), geo_ref) for x in (q, k, v))
            pq, pk = (pool.tile_mean_pool(x, geo_ref["vc"], E) for x in (qt, kt))
            sets = packed.select(select.tile_scores(pq, pk), geo_ref, rates)
            n = nT if q_tiles is None else min(q_tiles, nT)
            attention.block_sparse_attention(qt, kt, vt, geo_ref["vc"], sets, w.D ** -0.5,
                                             q_tiles=[(0, 0, i) for i in range(n)], tile_elems=E)
            pairs += sum(len(sets[0][0][i]) for i in range(n))
    sec = time.perf_counter() - t0
    return sec, pairs * 4 * E * E * w.D, pairs


def run_packed(args, w):
    """A packed multi-region sequence (dense prefix, reference and generated video regions) on one
    GPU: scatter, pooling, per-region selection, attention and gather, timed per stage."""
    import torch

    from block_sparse_video_tile3d_b200 import packed as P
    from block_sparse_video_tile3d_b200 import workloads

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("the packed workload runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    q, k, v = workloads.make_packed_qkv(w)
    mod = P.PackedTileSparseAttention(list(w.segments), w.heads, w.D, tile_size=w.tile_size,
                                      sparsity=w.sparsity, ref_keep_rate=w.ref_keep_rate, device=dev)
    g = mod.geo
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    od = torch.empty_like(qd)
    stages = mod.stages(qd, kd, vd, od)
    names = [n for n, _ in stages]
    sampler = ClockSampler(0)
    for _ in range(max(args.warmup, 3)):
        for _, launch in stages:
            launch()
    torch.cuda.synchronize()
    pairs = int(mod.kv_cnt.sum().item())
    E = g.E
    flops = pairs * 4 * E * E * w.D
    nst = len(stages)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    for st in range(args.steps):
        ev[st][0].record()
        for j, (_, launch) in enumerate(stages):
            launch()
            ev[st][j + 1].record()
    torch.cuda.synchronize()
    total_ms = ev[0][0].elapsed_time(ev[-1][-1])
    stage_ms = {n: sum(ev[st][j].elapsed_time(ev[st][j + 1]) for st in range(args.steps)) / args.steps
                for j, n in enumerate(names)}
    clocks = sampler.stop()
    launches, launch_src = count_launches(stages, packed=True)
    ms_step = total_ms / args.steps
    status = int(mod.status.item())
    # end to end: pinned host inputs in, output back, every step inside the timed region
    hosts = tuple(x.pin_memory() for x in (q, k, v))
    oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()
    ref = od.cpu()
    e2e_steps = max(4, min(args.steps, 20))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        for dst, src in zip((qd, kd, vd), hosts):
            dst.copy_(src, non_blocking=True)
        mod(qd, kd, vd, od)
        oh.copy_(od, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    peaks = _peaks()
    attn_ms = stage_ms["attention"]
    achieved = flops / (attn_ms * 1e-3) / 1e12
    row_bytes = w.heads * w.D * 2
    rows, buf = g.rows * w.B, g.buffer_rows * w.B
    pooled_bytes = w.B * w.heads * g.n_tiles * w.D * 4
    byt = {"scatter_pool_q": (rows + buf) * row_bytes + pooled_bytes,
           "scatter_pool_k": (rows + buf) * row_bytes + pooled_bytes,
           "scatter_v": (rows + buf) * row_bytes, "gather": (rows + buf) * row_bytes}
    kmax = mod.kv_idx.shape[-1]
    byt["select"] = 2 * pooled_bytes + w.B * w.heads * g.n_tiles * (kmax + 1) * 4
    stage_report = {n: {"ms": round(stage_ms[n], 4),
                        "gbs": round(byt[n] / (stage_ms[n] * 1e-3) / 1e9, 1) if n in byt else None,
                        "bytes": byt.get(n)} for n in names}
    coarse_ms = sum(stage_ms[n] for n in names if n != "attention")
    coarse_bytes = sum(byt[n] for n in names if n != "attention")
    line = {
        "metric": METRIC.replace("28,672 tok×12 heads", f"packed {g.rows:,} tok×{w.heads} heads"),
        "value": flops / (ms_step * 1e-3) / 1e12, "unit": "TFLOPS",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "ms_per_call": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": (f"{w.name}: B={w.B}, heads={w.heads}, D={w.D}, segments "
                                f"{list(w.segments)} (dense rows / region token grids), tile "
                                f"{E} ({'x'.join(map(str, g.tile_shape))}), {g.n_tiles} tiles "
                                f"({g.n_prefix} dense), generated keep {1 - w.sparsity:g}, "
                                f"reference keep {w.ref_keep_rate:g}"),
                   "kept_pairs": pairs, "metric_flops": f"4 * {E} * {E} * D per kept tile pair",
                   "kept_block_gflop": flops / 1e9,
                   "l2": f"no flush: packed Q/K/V of {3 * rows * row_bytes / 1e6:.0f} MB exceed "
                         "the 126 MB L2"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                     "kernel": "block_sparse_attn_fwd_packed",
                     "peak_source": f"{peaks['source']} bf16 dense (burst)", "ms_per_launch": attn_ms},
        "coarse_and_tiling": {"ms": coarse_ms, "bytes": coarse_bytes,
                              "gbs": coarse_bytes / (coarse_ms * 1e-3) / 1e9,
                              "frac_hbm": coarse_bytes / (coarse_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                              "hbm_peak_gbs": peaks["hbm_gbs"]},
        "stages": stage_report,
        "e2e": {"value": flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": e2e_ms,
                "steps": e2e_steps, "output_matches_device_run": bool(torch.equal(oh, ref)),
                "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                "d2h_bytes_per_step": od.numel() * od.element_size()},
        "gpu_launches": args.steps * sum(launches.values()),
        "gpu_launches_per_step": {"by_stage": launches, "source": launch_src},
        "device_status": status,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        from oracle import packed as opk
        ref_geo = opk.packed_geometry(list(w.segments), P.TILE_SHAPES[E])
        # calibrate on a small slice, then size the sample (whole heads, all query tiles) to the
        # CPU budget
        sec, fl, np_ = packed_oracle_sample(w, ref_geo, q, k, v, [0], max(1, g.n_tiles // 8))
        per_head = sec * 8
        nh = int(max(1, min(w.heads, args.cpu_budget // max(per_head, 1e-3))))
        sec, fl, np_ = packed_oracle_sample(w, ref_geo, q, k, v, list(range(nh)))
        line["cpu_baseline"] = {"value": fl / sec / 1e12, "unit": "TFLOPS", "cores": _cores(),
                                "kind": "oracle",
                                "sample": (f"fp64 numpy oracle, whole packed path (scatter, pool, "
                                           f"score, per-region select, attend all {g.n_tiles} "
                                           f"query tiles) for heads 0..{nh - 1} of {w.heads}: "
                                           f"{np_:,} kept pairs in {sec:.1f} s")}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="small",
                    help="workload: tiny, small, large, bsa, ragged_sliding, ragged_random, "
                         "packed, packed_tiny")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--pass", dest="which", default="forward", choices=["forward", "backward"],
                    help="forward: the whole hot path (the benchmark line); backward: the "
                         "gradients of the fine stage on one GPU")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: independent replicas (weak scaling) or one layer shared out by "
                         "head (strong scaling)")
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from block_sparse_video_tile3d_b200.workloads import PACKED_WORKLOADS, WORKLOADS
    if args.config in PACKED_WORKLOADS:
        if args.impl == "reference" or args.which == "backward":
            print(json.dumps({"impl": args.impl, "unavailable": "the packed workload has the forward "
                              "benchmark of this library only"}))
            return 0
        return run_packed(args, PACKED_WORKLOADS[args.config])
    w = WORKLOADS[args.config]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.which == "backward":
        return run_backward(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
