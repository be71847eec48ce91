"""The bench's multi-rank host logic with two gloo ranks on the CPU.

Under torchrun every rank runs an independent replica of the layer (no
data-path collective); the only cross-rank steps are the barrier around the
timed region, the max over ranks of each time, and rank 0 alone printing. The
GPU work itself is not needed to check those, so the ranks here are CPU
processes on the gloo backend.
"""

from __future__ import annotations

import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, outdir: str) -> None:
    import argparse
    import contextlib
    import io

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["RANK"] = str(rank)
    os.environ["WORLD_SIZE"] = str(world)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # each rank measured a different time: everyone must report the slowest
        t = bench.reduce_max(10.0 + 5.0 * rank, "cpu")
        value = bench.job_tops(2.0e9, 100, world, t)
        dist.barrier()
        # the reference arm under torchrun: rank 0 runs and prints, the others exit 0 without work
        args = argparse.Namespace(config="tiny", steps=1, warmup=0, gpus=world)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            rc = bench.run_reference(args)
        dist.barrier()
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"t": t, "value": value, "rc": rc, "stdout": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_rank0_output(tmp_path):
    import torch.multiprocessing as mp

    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    assert [r["t"] for r in res] == [15.0, 15.0]
    # 2e9 ops x 100 steps x 2 ranks over 15 ms
    assert res[0]["value"] == pytest.approx(2.0e9 * 100 * 2 / 15e-3 / 1e12)
    assert res[0]["value"] == res[1]["value"]
    assert [r["rc"] for r in res] == [0, 0]
    assert res[1]["stdout"] == ""
    lines = [ln for ln in res[0]["stdout"].splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == world and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_single_rank_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max(3.5, "cpu") == 3.5
    assert bench.job_tops(1e12, 1, 1, 1000.0) == pytest.approx(1.0)
