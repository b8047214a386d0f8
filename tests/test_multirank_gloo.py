"""The N>1 host path of bench.py on the CPU: two `gloo` ranks, world size 2.

The linear shards as independent replicas (no data-path collective), so the
multi-rank logic is the timing protocol: a barrier on both sides of the timed
region, the max over ranks of the per-step time, the whole-job aggregate, and
rank-0-only output (the reference arm runs on rank 0 alone)."""
import contextlib
import io
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ws, r, local = bench._dist()
        bench._barrier(ws)
        # a per-step time that differs by rank: the job's time is the slowest rank's
        ms_local = 1.0 + 0.5 * rank
        ms = bench._max_over_ranks(ms_local, ws, torch.device("cpu"))
        bench._barrier(ws)
        ops = 2.0 * bench.M0 * bench.N0 * bench.K0
        value = ws * ops / (ms * 1e-3) / 1e12  # the same aggregate run_cider prints
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"dist": [ws, r, local], "ms": ms, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_max_over_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["dist"] == [world, r, r]
        assert d["ms"] == pytest.approx(1.5)  # the slower rank's time, on both ranks
    ops = 2.0 * bench.M0 * bench.N0 * bench.K0
    assert res[0]["value"] == pytest.approx(world * ops / 1.5e-3 / 1e12)  # whole-job total
    assert res[0]["value"] == res[1]["value"]


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    """Under torchrun the reference arm's other ranks exit 0 without work."""
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = type("A", (), {"steps": 1, "warmup": 0})()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(args) == 0
    assert buf.getvalue() == ""


def test_single_rank_helpers_are_no_ops():
    assert bench._max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
    bench._barrier(1)  # no process group needed
