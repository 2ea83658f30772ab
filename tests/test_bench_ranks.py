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


def test_reference_arm_prints_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON
    line with the contract's keys, on the workload it is asked for."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", "tiny_fp32",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, cwd=root, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["config"]["workload"] == "tiny_fp32"
    assert d["value"] > 0 and d["unit"] == "chunks/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_oracle_sample_is_bounded():
    """The CPU-baseline sample repeats one request's oracle run until enough
    work is timed, and never more than the cap."""
    import bench
    import workloads as wl
    cfg = wl.TINY_FP32
    W = wl.make_weights(cfg)
    ks, vs = wl.make_prefix(cfg, lengths=wl.prefix_lengths(cfg)[:1])
    noise = wl.make_noise(cfg, batch=1)
    one = bench.oracle_sample_times(cfg, W, ks, vs, noise, cfg.steps)
    assert len(one) == 1 and one[0] > 0
    capped = bench.oracle_sample_times(cfg, W, ks, vs, noise, cfg.steps, min_seconds=1e9, max_reps=3)
    assert len(capped) == 3 and all(t > 0 for t in capped)
    enough = bench.oracle_sample_times(cfg, W, ks, vs, noise, cfg.steps, min_seconds=1e-9, max_reps=5)
    assert len(enough) == 1
