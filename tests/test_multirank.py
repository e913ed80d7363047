"""The multi-rank logic of bench.py on CPU with gloo, world size 2: every
rank reports its own step time, the line uses the slowest rank's time and
the sum of all ranks' work (weak scaling, no collective on the data path)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = 10.0 + 5.0 * rank
        ms = bench.max_over_ranks(ms_local, world)
        value = bench.whole_job_tflops(1e12, world, ms)
        q.put((rank, bench.dist_env()[:2], ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    for rank, env, ms, value in out:
        assert env == (rank, 2)
        assert ms == 15.0                       # the slowest rank
        assert value == pytest.approx(2 * 1e12 / 15e-3 / 1e12)


def test_single_rank_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_tflops(2e12, 1, 1000.0) == pytest.approx(2.0)
