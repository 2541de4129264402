"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): rows are
independent, so ranks share no data; the only collectives are the barrier and
the max of the timed region over ranks."""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        elapsed = 10.0 + 5.0 * rank            # rank 1 is the slow one
        q.put((rank, bench.max_over_ranks(elapsed, dist)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 15.0, 1: 15.0}


def test_whole_job_value_is_weak_scaling():
    one = bench.whole_job_gbs(16_908_288, 100, 5.0, 1)
    two = bench.whole_job_gbs(16_908_288, 100, 5.0, 2)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(16_908_288 * 100 / 5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    class A:
        impl = "ours"
    os.environ.pop("WORLD_SIZE", None)
    world, rank, local, pg = bench.dist_setup(A())
    assert (world, rank, pg) == (1, 0, None)
    assert bench.max_over_ranks(3.5, None) == 3.5


def test_physical_gpu_index(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3,5")
    assert bench.physical_gpu_index(1) == 5
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.physical_gpu_index(2) == 2
