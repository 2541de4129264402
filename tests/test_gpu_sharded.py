"""GPU parity of the row split over ranks (row_wise_topk_b200.sharded) on one GPU.

The ranks are emulated in one process: each shard's TopK runs through the
library, the all-gather is replaced by stacking the shards' results shard-major
(test code), and the library's stack / select / index-map kernels finish; the
result must equal the oracle's TopK of the whole rows, bit for bit."""
import numpy as np
import pytest
import torch

import oracle.topk_oracle as O
import workloads as W
from row_wise_topk_b200.sharded import CudaBackend, _round_up

pytestmark = pytest.mark.gpu


def split_topk_emulated(w, shards, sorted_index=1, index_dtype=torch.int64, nan_mode="trap"):
    be = CudaBackend()
    n = w.row_stride
    shard = n // shards
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    signed = w.x.view(np.int16 if w.dtype == "bf16" else np.int32)
    full = torch.from_numpy(np.ascontiguousarray(signed)).cuda().view(tdt)
    vals, idxs = [], []
    for s in range(shards):
        part = full[:, s * shard:(s + 1) * shard].contiguous()
        v, i = be.local_topk(part, w.k, nan_mode)
        vals.append(v)
        idxs.append(i)
    vg, ig = torch.stack(vals), torch.stack(idxs)           # what the all-gather delivers
    stacked, table = be.stack(vg, ig, w.k, shard, _round_up(shards * w.k, 16))
    fv, pos = be.final_topk(stacked, w.k, sorted_index, True, nan_mode)
    fi = be.take(table, pos, index_dtype)
    torch.cuda.synchronize()
    bits_t = np.uint16 if w.dtype == "bf16" else np.uint32
    fbits = fv.view(torch.int16 if w.dtype == "bf16" else torch.int32)
    return fi.cpu().numpy(), fbits.cpu().numpy().view(bits_t)


@pytest.mark.parametrize("dtype,rows,n,k,shards,dist", [
    ("f32", 2, 1 << 20, 1000, 2, "normal"),
    ("f32", 1, 1 << 22, 4096, 4, "ties"),
    ("bf16", 3, 1 << 18, 512, 4, "ties"),
    ("bf16", 1, 1 << 16, 2000, 8, "ascending"),
    ("f32", 4, 1 << 16, 64, 8, "equal"),
])
def test_split_matches_whole_row(dtype, rows, n, k, shards, dist):
    w = W.random_small(31, dtype, rows, n, k, dist=dist)
    idx, vals = split_topk_emulated(w, shards)
    exp = O.oracle_topk(w.x, dtype, k, sorted_index=1, return_value=1, index_dtype="i64")
    assert np.array_equal(idx, exp.indices)
    assert np.array_equal(vals, exp.values)


def test_split_value_order_and_int32():
    w = W.sampler_logits(2, 1024)      # rows of 129,280 (stride 129,280), 4 shards of 32,320
    idx, vals = split_topk_emulated(w, 4, sorted_index=2, index_dtype=torch.int32)
    exp = O.oracle_topk(w.x, "f32", w.k, end=w.end, sorted_index=1, return_value=1, index_dtype="i64")
    for r in range(w.rows):
        dec = O.decode(exp.values[r], "f32")
        perm = np.lexsort((exp.indices[r], -dec))
        assert np.array_equal(idx[r].astype(np.int64), exp.indices[r][perm])
        assert np.array_equal(vals[r], exp.values[r][perm])


def test_split_nan_row_flagged():
    w = W.long_rows(2, 1 << 18, 500, "uniform", inject_nan=True)   # NaN in row 1
    idx, _ = split_topk_emulated(w, 4, nan_mode="flag")
    assert np.all(idx[1] == O.IDX_NAN)
    exp = O.oracle_topk(w.x[:1], "f32", w.k, sorted_index=1, return_value=1, index_dtype="i64")
    assert np.array_equal(idx[0], exp.indices[0])
