"""The N > 1 path of bench.py on CPU: two gloo ranks.

Weak scaling with no data-path collective: each rank draws its own inputs (distinct seeds), and
only the timing is combined, as the max over ranks, into a whole-job rate. The reference arm
runs on rank 0 alone.
"""

import argparse
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads
        cfg = workloads.PYTHIA160M
        # per-rank inputs: distinct seeds, different tensors
        seed = bench.rank_seed(cfg.seed, rank)
        g = torch.Generator().manual_seed(seed)
        x = torch.randn(8, generator=g)
        xs = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(xs, x)
        # timing: each rank's own step time, combined as the max
        ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(ms, torch.device("cpu"), world)
        rate = bench.job_throughput(3.0e9, world, 7, mx)
        # reference arm: rank 0 alone does the work
        args = argparse.Namespace(steps=1, warmup=0)
        ref = bench.reference(args, rank, world) if rank != 0 else "skipped"
        out[rank] = {"seed": seed, "distinct": not torch.equal(xs[0], xs[1]), "max_ms": mx,
                     "rate": rate, "ref": ref}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["distinct"] and res[1]["distinct"]
    # every rank sees the slowest rank's time, and the job rate counts both ranks' work
    assert res[0]["max_ms"] == res[1]["max_ms"] == 15.0
    assert res[0]["rate"] == pytest.approx(3.0e9 * 2 * 7 / 15.0e-3)
    assert res[1]["ref"] is None  # non-zero ranks of the reference arm do no work
