"""The N > 1 path of bench.py on CPU: two gloo ranks run independent
replicas (no data-path collective); the only cross-rank step is the max of
the timings, and the whole-job rate counts every rank's work."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        mx = bench.max_over_ranks(ms, world, device="cpu")
        seed = bench.replica_seed(1, rank)
        rate = bench.whole_job_rate(1e12, world, mx)
        t = torch.tensor([mx, float(seed), rate], dtype=torch.float64)
        gathered = [torch.zeros(3, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, t)
        if rank == 0:
            out.put([g.tolist() for g in gathered])
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    (mx0, s0, r0), (mx1, s1, r1) = res
    assert mx0 == mx1 == 15.0          # both ranks report the slowest rank's time
    assert s0 != s1                    # independent inputs per replica
    assert r0 == r1 == pytest.approx(2 * 1e12 / 15e-3)
