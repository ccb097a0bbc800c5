"""The benchmark's multi-rank host logic on CPU: world size 2 over gloo.

Replicas only (the path has no exchange step): each rank times its own
stream, the job time is the maximum over ranks, and the job's GB/s counts
every replica's bytes.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        vals = bench.max_over_ranks([1.0 + rank, 10.0 - rank])
        dist.barrier()
        out.put((rank, vals, bench.job_gbps(world, 1_000_000_000, vals[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_world2():
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
    for rank, vals, gbps in res:
        assert vals == [2.0, 10.0]  # max over ranks, element-wise
        assert gbps == pytest.approx(2 * 1e9 / 2e-3 / 1e9)  # both replicas' bytes over the slowest time


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks([3.5, 1.25]) == [3.5, 1.25]
    assert bench.job_gbps(1, 4_192_337_920, 1.0) == pytest.approx(4192.33792)
