"""bench.py's host side without a GPU: the multi-rank aggregation on two gloo ranks (the job's time
is its slowest rank's, and the throughput counts every rank's tokens), and the reference arm's
JSON line (rank 0 alone runs it; other ranks exit without work)."""
import argparse
import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import torch.distributed as dist

    world, r, _ = bench.dist_setup(2, backend="gloo")
    try:
        slowest = bench.max_over_ranks(10.0 + 5.0 * r, world)  # rank 1 is the slow one
        again = bench.max_over_ranks(3.0 - r, world)
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"world": world, "rank": r, "slowest": slowest, "again": again}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp

    mp.spawn(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        got = json.load(open(tmp_path / f"rank{r}.json"))
        assert got == {"world": 2, "rank": r, "slowest": 15.0, "again": 3.0}


def test_single_rank_and_throughput(monkeypatch):
    for var in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(var, raising=False)
    assert bench.dist_setup(1) == (1, 0, 0)  # no process group with one rank
    assert bench.max_over_ranks(7.5, 1) == 7.5
    # 8192 tokens per rank, 2 ranks, 0.5 ms per step at the slowest rank
    assert bench.job_throughput(8192, 2, 0.5) == pytest.approx(2 * 8192 / 0.5e-3)


def _ref_args(steps=1, warmup=0):
    return argparse.Namespace(ref_step_rows=1, steps=steps, warmup=warmup, gpus=1)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    bench.run_reference(_ref_args(), world=2, rank=1)
    assert capsys.readouterr().out == ""


def test_reference_arm_line(capsys):
    bench.run_reference(_ref_args(), world=1, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
