"""The benchmark's multi-rank timing plumbing (barrier and max over ranks) on
CPU with gloo, world size 2: every rank reports the slowest rank's time."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        barrier, maxr = bench.rank_helpers(world, device="cpu")
        barrier()
        out[rank] = maxr(1.5 + rank)
        barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    os.environ["PYTHONPATH"] = root + os.pathsep + os.environ.get("PYTHONPATH", "")
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_helpers_are_identity():
    import bench
    barrier, maxr = bench.rank_helpers(1)
    barrier()
    assert maxr(3.25) == 3.25
