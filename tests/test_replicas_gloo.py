"""The multi-rank path of bench.py (replicas, no data-path collective) on two gloo ranks.

bench.py runs one independent replica per rank; the only collectives are the barrier and the
max-over-ranks reduction of the timings, and the reported value is the whole-job rate.  These
tests run that host logic with world size 2 on the CPU.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    import bench
    assert bench.dist_env() == (rank, world, rank)
    # rank-dependent timings: the max over ranks must come back on every rank
    mine = [1.0 + rank, 10.0 - rank, 3.5]
    got = bench.reduce_max(mine, world, device="cpu")
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": got}, f)


def test_reduce_max_over_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.spawn(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        with open(tmp_path / f"rank{r}.json") as f:
            assert json.load(f)["max"] == [2.0, 10.0, 3.5]


def test_reduce_max_is_identity_for_one_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max([3.0, 1.0], 1) == [3.0, 1.0]


def test_whole_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 10 steps x 1 GB each in 4 s (the slowest rank's time) -> 5 GB/s
    assert bench.aggregate_value(1e9, 10, 2, 4.0) == pytest.approx(5.0)
    assert bench.aggregate_value(1e9, 10, 1, 4.0) == pytest.approx(2.5)


def _reference_rank(rank, world, port, out_dir):
    import contextlib
    import io
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        if rank != 0:  # the other ranks of the reference arm exit without work or output
            bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "3"])
    with open(os.path.join(out_dir, f"ref{rank}.txt"), "w") as f:
        f.write(buf.getvalue())


def test_reference_arm_prints_only_on_rank_zero(tmp_path):
    mp.spawn(_reference_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    assert (tmp_path / "ref1.txt").read_text() == ""
