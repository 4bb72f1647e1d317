"""Host-side multi-rank logic of the benchmark, on CPU with the gloo backend
(world size 2): each rank runs an independent batch (its own seed), the window
time is the max over ranks, the value counts every rank's decode steps, and the
reference arm runs on rank 0 only."""
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


def _worker(rank, world, port, out):
    import sys

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slower one
    ms_max = bench.max_over_ranks(ms, dist)
    value = bench.whole_job_steps_per_s(world, 64, 8, ms_max)
    seed = bench.rank_seed("ctx500k", rank)
    args = argparse.Namespace(config="ctx500k", warmup=0, steps=1, gpus=world)
    ref_rc = bench.run_reference(args) if rank != 0 else None   # non-zero ranks return at once
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, ms_max, value, seed, ref_rc))


@pytest.mark.timeout(120)
def test_two_gloo_ranks_max_time_weak_value_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    (r0, m0, v0, s0, _), (r1, m1, v1, s1, rc1) = res
    assert m0 == m1 == 15.0                       # both ranks see the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 64 * 8 / 0.015)
    assert s0 != s1                               # independent batches
    assert rc1 == 0                               # reference arm: rank 1 exits without work
