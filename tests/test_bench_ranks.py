"""bench.py's multi-rank timing on CPU: every rank reports the largest of the ranks' times
(world size 2 over gloo, the reduction the bench runs over NCCL with one rank per GPU)."""
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


def _worker(rank, world, port, outdir):
    from datetime import timedelta

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    # rank r took 1.5 + r seconds; the bench divides all ranks' work by the slowest rank's time
    t = bench.max_over_ranks(1.5 + rank, world, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(outdir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(t))


def test_max_over_ranks_world2(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [float((tmp_path / f"rank{r}.txt").read_text()) for r in range(world)]
    assert got == [2.5, 2.5]


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.125, 1, "cpu") == 0.125
