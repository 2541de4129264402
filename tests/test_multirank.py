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


# --------------------------------------------------------------------------- #
# Row split over ranks (row_wise_topk_b200.sharded) on CPU: the real gloo
# all-gather, with the per-rank selection steps done by the oracle and the two
# layout steps restated in numpy, checks the sequencing, the shard-major layout
# of the exchange and the index offsets against the oracle on whole rows.
# --------------------------------------------------------------------------- #
class _OracleBackend:
    def __init__(self, dtype):
        self.dtype = dtype

    def local_topk(self, x_shard, k, nan_mode):
        import numpy as np
        import torch
        import oracle.topk_oracle as O
        bits = x_shard.numpy().view(np.uint16 if self.dtype == "bf16" else np.uint32)
        res = O.oracle_topk(bits, self.dtype, k, sorted_index=1, return_value=1, index_dtype="i64",
                            nan_mode=nan_mode)
        signed = res.values.view(np.int16 if self.dtype == "bf16" else np.int32)
        return torch.from_numpy(signed.copy()), torch.from_numpy(res.indices.astype(np.int64))

    def all_gather(self, values, indices, group):
        import torch
        import torch.distributed as dist
        world = dist.get_world_size(group)
        wide = values.to(torch.int32)                 # gloo has no int16 all-gather
        vg = [torch.empty_like(wide) for _ in range(world)]
        ig = [torch.empty_like(indices) for _ in range(world)]
        dist.all_gather(vg, wide.contiguous(), group=group)
        dist.all_gather(ig, indices.contiguous(), group=group)
        return torch.stack(vg).to(values.dtype), torch.stack(ig)

    def stack(self, vals_g, idx_g, k, shard_len, out_stride):
        import numpy as np
        import torch
        g, rows = vals_g.shape[0], vals_g.shape[1]
        neg_inf = -128 if self.dtype == "bf16" else -8388608       # 0xFF80 / 0xFF800000 as signed
        vs = np.full((rows, out_stride), neg_inf, dtype=vals_g.numpy().dtype)
        ix = np.full((rows, out_stride), -1, dtype=np.int64)
        for s in range(g):
            vs[:, s * k:(s + 1) * k] = vals_g[s].numpy()
            idx = idx_g[s].numpy()
            ix[:, s * k:(s + 1) * k] = np.where(idx >= 0, idx + s * shard_len, idx)
        return torch.from_numpy(vs), torch.from_numpy(ix)

    def final_topk(self, stacked, k, sorted_index, return_value, nan_mode):
        import numpy as np
        import torch
        import oracle.topk_oracle as O
        bits = stacked.numpy().view(np.uint16 if self.dtype == "bf16" else np.uint32)
        res = O.oracle_topk(bits, self.dtype, k, sorted_index=1, return_value=1, index_dtype="i64",
                            nan_mode=nan_mode)
        signed = res.values.view(np.int16 if self.dtype == "bf16" else np.int32)
        return torch.from_numpy(signed.copy()), torch.from_numpy(res.indices)

    def take(self, table, pos, index_dtype):
        import numpy as np
        import torch
        t, p = table.numpy(), pos.numpy()
        out = np.where(p >= 0, np.take_along_axis(t, np.maximum(p, 0), axis=1), p)
        return torch.from_numpy(out.astype(np.int64))


def _split_worker(rank, world, port, q, dtype, rows, n, k):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np
    import torch
    import torch.distributed as dist
    import workloads as W
    from row_wise_topk_b200.sharded import topk_row_split
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = W.random_small(77, dtype, rows, n, k, dist="ties")
        shard = n // world
        mine = w.x[:, rank * shard:(rank + 1) * shard]
        signed = mine.view(np.int16 if dtype == "bf16" else np.int32)
        vals, idx = topk_row_split(torch.from_numpy(np.ascontiguousarray(signed)), k, shard_len=shard,
                                   backend=_OracleBackend(dtype))
        q.put((rank, vals.numpy().tobytes(), idx.numpy().tobytes()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dtype,rows,n,k", [("f32", 3, 4096, 100), ("bf16", 2, 2048, 700)])
def test_row_split_over_two_ranks_gloo(dtype, rows, n, k):
    import numpy as np
    import oracle.topk_oracle as O
    import workloads as W
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q, dtype, rows, n, k)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict((r, (v, i)) for r, v, i in (q.get(timeout=180) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0] == got[1]                         # every rank ends with the same result
    w = W.random_small(77, dtype, rows, n, k, dist="ties")
    exp = O.oracle_topk(w.x, dtype, k, sorted_index=1, return_value=1, index_dtype="i64")
    idx = np.frombuffer(got[0][1], dtype=np.int64).reshape(rows, k)
    vals = np.frombuffer(got[0][0], dtype=np.uint16 if dtype == "bf16" else np.uint32).reshape(rows, k)
    assert np.array_equal(idx, exp.indices)
    assert np.array_equal(vals, exp.values)


def test_roofline_launch_time():
    # one launch per step: the timed region's average; two (stream + merge): the isolated mean
    assert bench.roofline_launch_ms(0.0225, 1, [0.0286, 0.0290]) == 0.0225
    assert abs(bench.roofline_launch_ms(0.5, 2, [0.2, 0.4]) - 0.3) < 1e-12


def test_recorded_traffic_follows_the_kernel_sources(monkeypatch):
    """roofline.traffic comes from the committed ncu record only while the kernel
    sources hash to the ones it was captured on; any other hash reports null."""
    import json
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for name, e in rec.items():
        assert name in ("indexer", "indexer_varlen", "sampler_256_1024", "long_16_4096"), name
        assert e["dram_bytes_per_launch"] > 0 and os.path.exists(os.path.join(bench.ROOT, "profiles", e["source"]))
        want = e["dram_bytes_per_launch"] if e["kernel_hash"] == bench.kernel_hash() else None
        assert bench.recorded_traffic(name) == want
    monkeypatch.setattr(bench, "kernel_hash", lambda: "0000000000000000")
    assert all(bench.recorded_traffic(name) is None for name in rec)
    assert bench.recorded_traffic("no_such_workload") is None


def test_torch_topk_context_skips_what_it_has_no_counterpart_for():
    # per-row end and the sampling step have no torch.topk counterpart: skipped without
    # touching a device
    import numpy as np

    class Wk:
        end = np.zeros(2, dtype=np.int32)
        elem_bytes = 2
        k = 4
    assert "skipped" in bench.torch_topk_context(None, Wk(), [], None, 1, 1.0, sampling=False)
    Wk.end = None
    assert "skipped" in bench.torch_topk_context(None, Wk(), [], None, 1, 1.0, sampling=True)
