"""The multi-process plumbing of bench.py on CPU: world_size 2 over gloo.

The path shards into independent replicas (no data-path collective); the
only cross-rank steps are the barrier and the max over ranks of the timed
region.  These run here without a GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "took" 1.0 + r seconds for the same 10 units of work
        t = bench.max_over_ranks(1.0 + rank, world, device="cpu")
        rate = bench.weak_scaling_rate(10.0, world, t)
        bench.barrier(world)
        ref = bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0",
                                                    "--cpu-seconds", "0.01"])) if rank == 1 else None
        q.put((rank, t, rate, ref))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_weak_scaling_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, rate0, _), (r1, t1, rate1, ref1) = res
    assert t0 == t1 == 2.0                     # every rank sees the slowest rank's time
    assert rate0 == rate1 == 10.0 * 2 / 2.0    # units of all ranks over that time
    assert ref1 is None                        # the reference arm runs on rank 0 only
