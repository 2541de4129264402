"""GPU test of dsel_topk_noalloc, the entry point for callers that cannot let the
library allocate device memory (engines with their own allocator and budget,
hosts that forbid side allocations, loops where cudaMalloc/cudaFree and their
implicit synchronisation are not acceptable).

The variant must give exactly what dsel_topk gives, and both must equal the CPU
oracle.  The shapes below are split-row plans (one row over several thread-block
clusters), the only plans that use scratch memory, so the static scratch is really
exercised.  Two calls in a row on different inputs show that stale scratch contents
from the previous call do not leak into the next one; a flag-mode call with NaN rows
and more rows x groups, followed by a clean call of another shape, shows that a
leftover NaN mark or a larger count from a bigger plan does not either.  A plan that
needs more than the static scratch must be refused before any launch.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle.topk_oracle as O
import row_wise_topk_b200 as T
import workloads as W
from gpu_util import compare, to_device_bits

pytestmark = pytest.mark.gpu


def _run(fn, w, order, x_dev):
    itorch = torch.int32 if w.index_dtype == "i32" else torch.int64
    vtorch = torch.int16 if w.dtype == "bf16" else torch.int32
    idx = torch.full((w.rows, w.k), 7, dtype=itorch, device="cuda")
    val = torch.full((w.rows, w.k), 7, dtype=vtorch, device="cuda") if w.return_value else None
    st = fn(x_dev.data_ptr(), T.DSEL_BF16 if w.dtype == "bf16" else T.DSEL_F32, w.rows, w.row_stride,
            None, w.k, order, w.return_value, T.DSEL_I32 if w.index_dtype == "i32" else T.DSEL_I64,
            T.DSEL_NAN_FLAG, None if val is None else val.data_ptr(), idx.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
    assert st == 0, T.dsel_status_string(st)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), None if val is None else val.cpu().numpy()


CASES = [
    # (dtype, rows, row_stride, k, order): every one a split-row plan (groups > 1)
    ("f32", 1, 1 << 22, 512, T.DSEL_ORDER_INDEX),
    ("bf16", 1, 1 << 22, 512, T.DSEL_ORDER_NONE),
    ("f32", 2, 1 << 20, 1000, T.DSEL_ORDER_VALUE),
    ("bf16", 3, 1 << 21, 2000, T.DSEL_ORDER_INDEX),
]


def _workload(seed, dtype, rows, stride, k, nan_rows=None):
    return W.random_small(seed, dtype, rows, stride, k, dist="normal", sorted_index=1, return_value=1,
                          index_dtype="i64", nan_rows=nan_rows, nan_mode="flag")


def _split_plan(dtype, rows, stride, k, order):
    st, plan = T.dsel_plan_for(T.DSEL_BF16 if dtype == "bf16" else T.DSEL_F32, rows, stride, k, order,
                               num_sms=torch.cuda.get_device_properties(0).multi_processor_count)
    assert st == 0 and plan["groups"] > 1, "the case must use the split-row scratch"
    assert plan["workspace_bytes"] <= T.DSEL_NOALLOC_SCRATCH_BYTES
    return plan


def _check_both(w, order):
    """dsel_topk_noalloc against dsel_topk bit for bit, and both against the oracle."""
    x = to_device_bits(w.x)
    want_idx, want_val = _run(T.dsel_topk, w, order, x)
    got_idx, got_val = _run(T.dsel_topk_noalloc, w, order, x)
    exp = O.oracle_topk(w.x, w.dtype, w.k, sorted_index=1, return_value=1, index_dtype="i64", nan_mode="flag")
    compare(w, got_idx, got_val, exp, order)
    compare(w, want_idx, want_val, exp, order)
    if order == T.DSEL_ORDER_NONE:   # order unspecified: compare as sets (values alongside)
        pw, pg = np.argsort(want_idx, axis=1), np.argsort(got_idx, axis=1)
        want_idx, got_idx = np.take_along_axis(want_idx, pw, 1), np.take_along_axis(got_idx, pg, 1)
        want_val, got_val = np.take_along_axis(want_val, pw, 1), np.take_along_axis(got_val, pg, 1)
    assert np.array_equal(got_idx, want_idx)
    assert np.array_equal(got_val, want_val)


@pytest.mark.parametrize("dtype,rows,stride,k,order", CASES)
def test_noalloc_matches_topk_on_two_calls_in_a_row(dtype, rows, stride, k, order):
    _split_plan(dtype, rows, stride, k, order)
    for seed in (41, 42):   # two calls in a row, different data
        _check_both(_workload(seed, dtype, rows, stride, k), order)


def test_noalloc_stale_nan_marks_and_counts_do_not_leak():
    # a bigger split plan in flag mode with NaN rows: leaves NaN marks and large
    # counts in the scratch ...
    big = ("bf16", 3, 1 << 21, 2000, T.DSEL_ORDER_INDEX)
    small = ("f32", 1, 1 << 22, 512, T.DSEL_ORDER_INDEX)
    pb, ps = _split_plan(*big), _split_plan(*small)
    assert pb["workspace_bytes"] > ps["workspace_bytes"]   # the first call writes more of the scratch
    w = _workload(51, "bf16", 3, 1 << 21, 2000, nan_rows=np.array([0, 2]))
    _check_both(w, T.DSEL_ORDER_INDEX)
    # ... then a clean call of another shape must not see them
    _check_both(_workload(52, "f32", 1, 1 << 22, 512), T.DSEL_ORDER_INDEX)


def test_noalloc_without_split_uses_no_scratch():
    w = W.indexer_drift(rows=8, n=8192, k=64, sorted_index=1, return_value=1)
    x = to_device_bits(w.x)
    a = _run(T.dsel_topk, w, 1, x)
    b = _run(T.dsel_topk_noalloc, w, 1, x)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_noalloc_refuses_plans_beyond_its_scratch():
    rows, stride, k = 1, 1 << 24, 4096
    st, plan = T.dsel_plan(T.DSEL_F32, rows, stride, k,
                           num_sms=torch.cuda.get_device_properties(0).multi_processor_count)
    assert st == 0 and plan["workspace_bytes"] > T.DSEL_NOALLOC_SCRATCH_BYTES
    # the call plans as dsel_plan does, so it is refused before any launch; the
    # buffers still have the full shape, so that a launch would read valid memory
    x = torch.zeros(rows * stride, dtype=torch.int32, device="cuda")
    idx = torch.zeros(rows * k, dtype=torch.int64, device="cuda")
    st = T.dsel_topk_noalloc(x.data_ptr(), T.DSEL_F32, rows, stride, None, k, 1, 0, T.DSEL_I64,
                             T.DSEL_NAN_FLAG, None, idx.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == T.DSEL_ERR_SCRATCH_LIMIT
    assert "static scratch" in T.dsel_status_string(st)
    assert T.dsel_device_status() == 0
