"""Host-side logic of the N > 1 paths, run as world-size-2 gloo process groups on CPU.

With several GPUs either every rank runs its own replica of the hot path, or the ranks share one
layer by head (each its own head range of the same rows); neither has a data-path collective. The
only cross-rank steps are the host reductions in bench.py: the max of the ranks' step times and the
sum of their kept-block FLOPs. These tests run those steps on CPU ranks, with per-rank problems whose
FLOPs come from the oracle's selection on the tiny workload; check that a layer shared by head and
reassembled equals the one-rank result bit for bit; and check that a rank that leaves before a
collective makes the other rank's collective fail with an error instead of waiting forever.
"""
from __future__ import annotations

import datetime
import io
import json
import os
import socket
import sys
import tempfile
import time
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank: int, port: int, timeout_s: float) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _replica_worker(rank: int, port: int, out_dir: str) -> None:
    import bench
    from block_sparse_video_tile3d_b200 import workloads
    from oracle import pipeline

    _init(rank, port, 60.0)
    try:
        world, r, local = bench.rank_env()
        assert (world, r, local) == (WORLD, rank, rank)
        base = workloads.WORKLOADS["tiny"]
        w = bench.rank_workload(base, rank)
        assert (w.B, w.heads, w.D, w.T, w.H, w.W, w.k) == (base.B, base.heads, base.D, base.T,
                                                          base.H, base.W, base.k)
        q, k, v = workloads.make_qkv(w)
        ref = pipeline.forward(q, k, v, w.T, w.H, w.W, "topk", scale=w.scale, topk=w.k)
        pairs = sum(len(s) for per_b in ref["sets"] for per_h in per_b for s in per_h)
        flops = float(pairs * bench.FLOPS_PER_PAIR(w.D))
        ms = 1.0 + 0.5 * rank  # this rank's step time; rank 1 is the slower one
        checksum = float(q.float().sum() + k.float().sum() + v.float().sum())

        ms_max = bench.reduce_over_ranks(ms, "max", world)
        flops_all = bench.reduce_over_ranks(flops, "sum", world)
        got = [torch.zeros(3, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, torch.tensor([flops, ms, checksum], dtype=torch.float64))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms_max": ms_max, "flops_all": flops_all,
                       "value": bench.whole_job_tflops(flops_all, ms_max),
                       "gathered": [t.tolist() for t in got], "seed": w.seed}, f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_replicas_reduce_to_whole_job_value():
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_replica_worker, args=(port, d), nprocs=WORLD, join=True,
                           start_method="spawn")
        res = [json.load(open(os.path.join(d, f"rank{r}.json"))) for r in range(WORLD)]
    gathered = res[0]["gathered"]
    flops = [g[0] for g in gathered]
    times = [g[1] for g in gathered]
    sums = [g[2] for g in gathered]
    assert res[0]["seed"] != res[1]["seed"]
    assert sums[0] != sums[1], "each rank must run a problem of its own"
    for r in res:
        assert r["gathered"] == gathered  # every rank saw the same values
        assert r["ms_max"] == max(times) == 1.5
        assert r["flops_all"] == sum(flops)
        assert r["value"] == pytest.approx(sum(flops) / (max(times) * 1e-3) / 1e12, rel=1e-12)
    # top-k keeps k tiles per query tile on every rank: equal FLOPs, different data
    assert flops[0] == flops[1] > 0


def _head_shard_worker(rank: int, port: int, out_dir: str, name: str) -> None:
    import numpy as np

    from block_sparse_video_tile3d_b200 import workloads
    from block_sparse_video_tile3d_b200.sharding import head_partition
    from oracle import pipeline

    _init(rank, port, 120.0)
    try:
        w = _shard_workload(name)
        q, k, v = workloads.make_qkv(w)  # every rank holds the same full-width layer
        mask = workloads.block_mask(w).numpy() if w.mode == "mask" else None
        h0, n = head_partition(w.heads, WORLD, rank)
        hs = slice(h0, h0 + n)
        kw = dict(scale=w.scale, topk=w.k) if w.mode == "topk" else dict(scale=w.scale,
                                                                          mask=mask[:, hs])
        mine = pipeline.forward(q[:, :, hs], k[:, :, hs], v[:, :, hs], w.T, w.H, w.W, w.mode,
                                **kw)["o"]
        parts = [None] * WORLD
        dist.all_gather_object(parts, (h0, n, mine))
        if rank == 0:
            full = np.zeros((w.B, w.L, w.heads, w.D))
            for ph0, pn, po in parts:
                full[:, :, ph0:ph0 + pn] = po
            kw1 = dict(scale=w.scale, topk=w.k) if w.mode == "topk" else dict(scale=w.scale,
                                                                               mask=mask)
            one = pipeline.forward(q, k, v, w.T, w.H, w.W, w.mode, **kw1)["o"]
            np.save(os.path.join(out_dir, "sharded.npy"), full)
            np.save(os.path.join(out_dir, "one.npy"), one)
            with open(os.path.join(out_dir, "ranges.json"), "w") as f:
                json.dump([[p[0], p[1]] for p in parts], f)
    finally:
        dist.destroy_process_group()


def _shard_workload(name):
    from block_sparse_video_tile3d_b200 import workloads
    if name == "tiny":
        return workloads.WORKLOADS["tiny"]
    # the ragged workload's recipe and mask on a smaller ragged grid, with an odd head count
    return workloads.WORKLOADS["ragged_sliding"].with_(B=2, T=9, H=10, W=13, heads=3)


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_two_ranks_share_a_layer_by_head(name):
    """Each rank runs the whole path (oracle) on its own head range of the same full-width layer;
    reassembled by head, the result equals the one-rank run bit for bit (no head depends on
    another, so no data exchange is needed)."""
    import numpy as np

    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_head_shard_worker, args=(port, d, name), nprocs=WORLD, join=True,
                           start_method="spawn")
        full = np.load(os.path.join(d, "sharded.npy"))
        one = np.load(os.path.join(d, "one.npy"))
        ranges = json.load(open(os.path.join(d, "ranges.json")))
    w = _shard_workload(name)
    assert sorted(h for h0, n in ranges for h in range(h0, h0 + n)) == list(range(w.heads))
    assert all(n >= 1 for _, n in ranges)
    np.testing.assert_array_equal(full, one)


def _leaver_worker(rank: int, port: int, out_dir: str) -> None:
    import bench

    _init(rank, port, 5.0)
    outcome = "left"
    if rank == 0:
        try:
            bench.reduce_over_ranks(1.0, "max", WORLD)
            outcome = "completed"
        except Exception as e:  # the collective must end with an error
            outcome = f"error: {type(e).__name__}"
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(outcome)
    if rank == 1:
        os._exit(0)  # leaves without joining the collective or tearing the group down


def test_rank_that_leaves_makes_the_collective_fail():
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        ctx = mp.start_processes(_leaver_worker, args=(port, d), nprocs=WORLD, join=False,
                                 start_method="spawn")
        deadline = time.monotonic() + 120.0
        done = False
        while not done and time.monotonic() < deadline:  # join() returns as each rank ends
            done = ctx.join(timeout=max(0.1, deadline - time.monotonic()))
        if not done:
            for p in ctx.processes:  # our own children, by handle
                if p.is_alive():
                    p.kill()
            pytest.fail("a rank did not finish within 120 s")
        outcome = open(os.path.join(d, "rank0.txt")).read()
    assert outcome.startswith("error"), outcome


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    from block_sparse_video_tile3d_b200 import workloads

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.argparse.Namespace(gpus=2, steps=1, warmup=0)
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.run_reference(args, workloads.WORKLOADS["tiny"])
    assert rc == 0 and buf.getvalue() == ""


def test_single_rank_reductions_are_identity():
    import bench

    from block_sparse_video_tile3d_b200 import workloads

    assert bench.reduce_over_ranks(3.25, "max", 1) == 3.25
    assert bench.reduce_over_ranks(7.0, "sum", 1) == 7.0
    w = workloads.WORKLOADS["small"]
    assert bench.rank_workload(w, 0) is w
    w1, w2 = bench.rank_workload(w, 1), bench.rank_workload(w, 2)
    assert len({w.seed, w1.seed, w2.seed}) == 3
    assert w1.with_(seed=w.seed) == w
