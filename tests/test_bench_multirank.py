"""bench.py's multi-rank host logic on CPU: two gloo ranks over 127.0.0.1.

The timing of an N-GPU run is the maximum over ranks, the value counts the units of all
ranks, and only rank 0 prints; the reference arm runs on rank 0 alone.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # Rank r reports times (r + 1, 10 - r): the job's times are the per-element maxima.
        got = bench._max_over_ranks([rank + 1.0, 10.0 - rank], world)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump(got, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert json.load(open(tmp_path / f"r{r}.json")) == [2.0, 10.0]


def test_job_value_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    # 131072 tokens per rank-step, 5 steps, 4 ranks, slowest rank 25 ms.
    assert bench._job_value(131072, 5, 4, 25.0) == pytest.approx(131072 * 5 * 4 / 0.025)
    assert bench._max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]


def test_reference_arm_is_silent_on_other_ranks(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        workload, steps, warmup, gpus = "prefill_8k", 1, 0, 2
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(A())
    assert buf.getvalue() == ""
