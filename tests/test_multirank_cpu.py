"""Host logic of the N > 1 bench path on CPU: two gloo ranks (world size 2).

bench.py runs one weak-scaling replica per GPU; the job's time is the max over
ranks and the value counts every rank's work. Those pieces (barrier, max over
ranks, aggregate, the reference arm's rank-0-only rule) are checked here with
fake per-rank timings."""
import os
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms_local = 100.0 + 50.0 * rank          # rank 1 is the slow one
        value, ms = bench.aggregate(2.0e12, 4, ms_local, world)
        mx = bench.max_over_ranks(float(rank), world)

        class A:
            pass
        a = A()
        a.steps, a.warmup, a.gpus = 1, 3, world
        ref_rc = bench.run_reference(a, world, rank) if rank != 0 else 0
        q.put((rank, value, ms, mx, ref_rc))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_max_over_ranks_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms, mx, ref_rc in out:
        assert ms == 150.0                       # the slowest rank's time
        assert abs(value - 2 * 2.0e12 * 4 / 0.150 / 1e12) < 1e-9
        assert mx == 1.0
        assert ref_rc == 0                       # non-zero ranks skip the reference arm
