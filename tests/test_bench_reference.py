"""The benchmark's reference arm (the CPU oracle timed on the host cores) prints one JSON line that
carries every key of the benchmark contract, on rank 0, without a GPU."""
import io
import json
from contextlib import redirect_stdout

import bench
from block_sparse_video_tile3d_b200 import workloads

CONTRACT_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                 "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                 "cpu_baseline", "e2e"}


def test_reference_line_carries_the_contract(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    args = bench.argparse.Namespace(gpus=1, steps=2, warmup=1)
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(args, workloads.WORKLOADS["tiny"]) == 0
    lines = buf.getvalue().strip().splitlines()
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert CONTRACT_KEYS <= set(line)
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["steps"] == 2
    assert line["higher_is_better"] is True and line["vs_baseline"] is None
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith("tiny")


def test_launch_count_falls_back_to_the_launch_code_table(monkeypatch):
    """Without a device trace (no GPU here, or ncu attached) the per-stage kernel counts come from
    the table read off the launch code, labelled as such; every stage name the modules use has an
    entry (selection runs three kernels, mass selection four, the packed attention two)."""
    stages = [(n, lambda: None) for n in ("scatter_pool_q", "scatter_pool_k", "scatter_v",
                                          "select_topk", "attention", "gather")]
    counts, source = bench.count_launches(stages)
    assert counts == {"scatter_pool_q": 1, "scatter_pool_k": 1, "scatter_v": 1, "select_topk": 3,
                      "attention": 1, "gather": 1}
    assert source.startswith("static")
    monkeypatch.setenv("CUDA_INJECTION64_PATH", "/nonexistent")
    counts, source = bench.count_launches([("select", lambda: None), ("attention", lambda: None)],
                                          packed=True)
    assert counts == {"select": 3, "attention": 2} and "another profiler" in source
    for name in ("scatter_q", "scatter_k", "mask_to_index", "prune_q", "select_mass"):
        assert bench.STATIC_KERNELS[name] >= 1
