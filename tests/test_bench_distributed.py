"""The replica (N > 1) plumbing of bench.py on CPU with the gloo backend, world size 2: the
max-over-ranks reduction of the timing and of the error flag, the per-world config, and the
reference arm's rank-0-only output."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        # rank r took 1 + r ms; only rank 1 saw an error
        got = bench.reduce_max_over_ranks(torch, dist, [1.0 + rank, 1.0 if rank == 1 else 0.0], "cpu")
        again = bench.reduce_max_over_ranks(torch, dist, [5.0 - rank], "cpu")
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"got": got, "again": again}, f)
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_ranks_gloo_world_2(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    for r in range(2):
        res = json.load(open(tmp_path / f"rank{r}.json"))
        assert res["got"] == [2.0, 1.0], res        # the slowest rank's time, any rank's error
        assert res["again"] == [5.0], res


def test_reduce_without_process_group_is_identity():
    assert bench.reduce_max_over_ranks(None, None, [3.5, 0], "cpu") == [3.5, 0.0]


def test_config_for_world_sizes():
    one, four = bench.config_for(1), bench.config_for(4)
    assert one["global_batch"] == 1 and one["parallelism"] == "single GPU"
    assert four["global_batch"] == 4 and four["parallelism"] == "replicas x4"
    assert set(one) == set(four)


def test_reference_arm_other_ranks_exit_without_output(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup, cpu_seconds = 1, 3, 0.1

    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.bench_reference(Args())
    assert buf.getvalue() == ""
