"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Integer and bit results are compared exactly: indices, value bits, sentinel
slots.  With ``sorted_index=0`` the order is unspecified, so index sets are
compared after sorting (values permuted alongside); with value order the
sequence must match the oracle's set sorted by (value desc, index asc)."""
import numpy as np
import pytest
import torch

import oracle.topk_oracle as O
import row_wise_topk_b200 as T
import workloads as W
from gpu_util import check, expected, compare, run_gpu, to_device_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert T.dsel_device_status() == 0


# --------------------------------------------------------------------------- #
# small and medium cases: several tiles, ragged tails, every option
# --------------------------------------------------------------------------- #
SMALL = []
_seed = 100
for dtype in ("bf16", "f32"):
    for rows, stride in ((1, 4096), (3, 40960), (5, 2048), (200, 1024), (37, 20480)):
        for k in (1, 7, 64, 512, 2000):
            for dist in ("normal", "ties"):
                _seed += 1
                SMALL.append((_seed, dtype, rows, stride, k, dist))


@pytest.mark.parametrize("seed,dtype,rows,stride,k,dist", SMALL)
def test_small_cases(seed, dtype, rows, stride, k, dist):
    w = W.random_small(seed, dtype, rows, stride, k, dist=dist, with_end=(seed % 2 == 0),
                       end_lo=0, sorted_index=1, return_value=1, index_dtype="i64")
    order = [T.DSEL_ORDER_INDEX, T.DSEL_ORDER_NONE][seed % 2]
    check(w, order=order)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("order", [0, 1, 2])
@pytest.mark.parametrize("rv", [0, 1])
@pytest.mark.parametrize("idt", ["i32", "i64"])
def test_option_grid(dtype, order, rv, idt):
    if order == 2 and dtype == "bf16":
        pytest.skip("value order is float32 only")
    w = W.random_small(7, dtype, 9, 24576, 300, dist="ties", with_end=True, end_lo=100)
    check(w, order=order, return_value=rv, index_dtype=idt)


SPLIT = [
    # (dtype, rows, row_stride, k): rows longer than one cluster's slices; the longest
    # span several clusters whose partial results the merge kernel combines
    ("f32", 1, 1 << 20, 4096),
    ("f32", 2, 1 << 19, 1000),
    ("f32", 1, 1 << 22, 512),
    ("bf16", 1, 1 << 22, 512),
    ("bf16", 3, 1 << 21, 2000),
]


@pytest.mark.parametrize("dist", ["ascending", "equal", "ties"])
@pytest.mark.parametrize("dtype,rows,stride,k", SPLIT)
def test_split_rows(dist, dtype, rows, stride, k):
    """few long rows: cluster split and, for the longest, several clusters + merge"""
    w = W.random_small(11, dtype, rows, stride, k, dist=dist, sorted_index=1)
    check(w, order=T.DSEL_ORDER_INDEX)
    if dtype == "f32":   # value order is float32 only
        check(w, order=T.DSEL_ORDER_VALUE)
    check(w, order=T.DSEL_ORDER_NONE)


@pytest.mark.parametrize("dtype,rows,stride,k", [("f32", 1, 1 << 22, 512), ("bf16", 1, 1 << 22, 512),
                                                  ("bf16", 3, 1 << 21, 2000)])
def test_plans_cover_split_and_merge(dtype, rows, stride, k):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    dt = T.DSEL_BF16 if dtype == "bf16" else T.DSEL_F32
    for order in (T.DSEL_ORDER_INDEX, T.DSEL_ORDER_NONE):
        st, p = T.dsel_plan_for(dt, rows, stride, k, order, num_sms=sms)
        assert st == 0 and p["kernel"] == T.DSEL_KERNEL_STREAM and p["groups"] > 1


@pytest.mark.parametrize("rows", [10, 14, 16])
def test_split_rows_wide_clusters(rows):
    """rows too long for the slice kernel, split over the streaming kernel's clusters:
    the device plan takes the cluster size and groups with the most CTAs whose
    clusters the device holds in one wave (clusters above the portable 8 included)"""
    st, p = T.dsel_plan_device(T.DSEL_F32, rows, 1 << 20, 1024, T.DSEL_ORDER_INDEX)
    assert st == 0 and p["kernel"] == T.DSEL_KERNEL_STREAM and 2 <= p["cluster"] <= 16
    assert rows * p["cluster"] * p["groups"] <= torch.cuda.get_device_properties(0).multi_processor_count
    w = W.random_small(23 + rows, "f32", rows, 1 << 20, 1024, dist="ties", sorted_index=1)
    check(w, order=T.DSEL_ORDER_INDEX)
    check(w, order=T.DSEL_ORDER_VALUE)


def test_device_plan_matches_host_plan_below_eight():
    """the device plan differs from the host planner only in how a row split over the
    streaming kernel's clusters is sized (clusters and groups that fit one wave) and
    in the slice kernel's cluster limit"""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for args in [(T.DSEL_BF16, 64, 131072, 512, 1), (T.DSEL_F32, 256, 129280, 1024, 2),
                 (T.DSEL_BF16, 4096, 16384, 512, 1), (T.DSEL_F32, 1, 1 << 28, 1000, 1)]:
        st, dp = T.dsel_plan_device(*args)
        hst, hp = T.dsel_plan_for(*args, num_sms=sms, max_cluster=8)
        assert st == 0 and hst == 0
        assert (dp["kernel"], dp["threads"]) == (hp["kernel"], hp["threads"])
        if hp["kernel"] != T.DSEL_KERNEL_SLICE and hp["cluster"] * hp["groups"] == 1:
            assert dp == hp
        if dp["kernel"] == T.DSEL_KERNEL_STREAM and dp["cluster"] * dp["groups"] > 1:
            assert dp["cluster"] * dp["groups"] >= hp["cluster"] * hp["groups"] // 2


def test_all_rows_short():
    w = W.random_small(3, "bf16", 10, 16, 4096, dist="normal")
    check(w, order=1)
    w = W.random_small(4, "f32", 10, 64, 64, dist="normal", with_end=True, end_lo=0)
    check(w, order=0)


def test_k_equals_row_length_and_empty_rows():
    w = W.random_small(5, "f32", 6, 1024, 1024, dist="normal")
    check(w)
    w = W.random_small(6, "bf16", 6, 1024, 8, dist="normal", with_end=True)
    w.end[:] = [0, 8, 9, 1024, 1, 16]
    check(w)


def test_nan_rows_flag_mode():
    rows = 12
    nan_rows = np.array([1, 4, 5, 11])
    w = W.random_small(8, "bf16", rows, 8192, 100, dist="normal", with_end=True, end_lo=50,
                       nan_rows=nan_rows, nan_mode="flag")
    gi, gv = check(w, order=1)
    lens = w.valid_lengths()
    for r in nan_rows:
        if lens[r] > w.k:
            assert (gi[r] == T.DSEL_IDX_NAN).all() and (gv[r] == 0x7FC0).all()
    w32 = W.random_small(9, "f32", rows, 4096, 4096, dist="ties", nan_rows=nan_rows, nan_mode="flag")
    check(w32, order=0)


def test_nan_in_split_rows_flag_mode():
    w = W.long_rows(4, 1 << 21, 1000, "uniform", inject_nan=True)
    check(w, order=1)


def test_bad_end_flag_and_trap():
    w = W.random_small(10, "f32", 4, 2048, 16, dist="normal", with_end=True, nan_mode="flag")
    w.end[:] = [-1, 2049, 2048, 17]
    check(w, order=1)
    w.nan_mode = "trap"                     # trap mode clamps an invalid end
    check(w, order=1)


def test_signed_zero_and_inf_ties():
    x = np.zeros((2, 256), dtype=np.float32)
    x[0, ::2] = -0.0
    x[1, :] = np.where(np.arange(256) % 3 == 0, np.inf, -0.0)
    w = W.Workload("zeros", "f32", x.view(np.uint32), None, 100, 1, 1, "i64")
    check(w)
    wb = W.Workload("zeros_bf16", "bf16", W.bf16_bits_rne(x), None, 100, 1, 1, "i32")
    check(wb)


def test_deterministic_repeat():
    w = W.indexer_drift(rows=16, n=65536, k=512, sorted_index=0, return_value=1)
    x = to_device_bits(w.x)
    a = run_gpu(w, x_dev=x)
    b = run_gpu(w, x_dev=x)
    assert np.array_equal(np.sort(a[0], 1), np.sort(b[0], 1))


def test_torch_wrapper_bf16():
    w = W.indexer_varlen(rows=32, stride=4096, k=128)
    x = to_device_bits(w.x).view(torch.bfloat16)
    end = torch.from_numpy(w.end).cuda()
    vals, idx = T.topk(x, w.k, end=end, sorted_index=1, return_value=True, index_dtype=torch.int64)
    exp = expected(w, return_value=1, index_dtype="i64")
    compare(w, idx.cpu().numpy(), vals.view(torch.int16).cpu().numpy().view(np.uint16), exp, 1)


# --------------------------------------------------------------------------- #
# the workload families at full size (the bench's launch configuration)
# --------------------------------------------------------------------------- #
# --------------------------------------------------------------------------- #
# up to one wave of rows of 32-64 KB: one slice per row (no cluster)
# --------------------------------------------------------------------------- #
SHORT = [
    # (seed, dtype, rows, stride, k, dist, order): bf16 rows above 32 KB (shorter ones
    # go to the row-resident kernel), each one slice of the slice kernel, one CTA per SM
    (301, "bf16", 148, 32768, 1, "normal", 1),
    (302, "bf16", 140, 32768, 512, "ties", 0),
    (303, "bf16", 100, 16400, 4096, "normal", 1),
    (304, "bf16", 120, 20480, 512, "ties", 1),
    (305, "bf16", 148, 24576, 64, "ascending", 0),
    (306, "bf16", 97, 30000 // 16 * 16, 2000, "equal", 1),
]


@pytest.mark.parametrize("seed,dtype,rows,stride,k,dist,order", SHORT)
def test_one_slice_rows(seed, dtype, rows, stride, k, dist, order):
    st, plan = T.dsel_plan_for(T.DSEL_BF16 if dtype == "bf16" else T.DSEL_F32, rows, stride, k, order,
                               num_sms=torch.cuda.get_device_properties(0).multi_processor_count)
    assert st == 0 and plan["kernel"] == T.DSEL_KERNEL_SLICE and plan["cluster"] == 1, \
        "the case must use one slice per row"
    w = W.random_small(seed, dtype, rows, stride, k, dist=dist, with_end=(seed % 2 == 0),
                       end_lo=0, sorted_index=1, return_value=1, index_dtype="i64")
    check(w, order=order)


MID = [
    # (seed, dtype, rows, stride, k, dist, order): value order takes the streaming kernel's
    # 256-thread shape (two CTAs per SM); index order and no order the slice kernel, a
    # cluster per row, one wave of CTAs
    (401, "f32", 70, 65536, 1024, "normal", 2),
    (402, "f32", 72, 40960, 50, "ties", 2),
    (403, "bf16", 64, 131072, 512, "ascending", 1),
    (404, "f32", 49, 16400, 700, "equal", 2),
    (405, "f32", 70, 65536, 1024, "normal", 1),
    (406, "f32", 74, 40960, 50, "ties", 0),
    (407, "f32", 37, 129280, 1024, "ties", 1),
    (408, "bf16", 9, 131072, 2000, "normal", 0),
]


@pytest.mark.parametrize("seed,dtype,rows,stride,k,dist,order", MID)
def test_mid_row_shape(seed, dtype, rows, stride, k, dist, order):
    st, plan = T.dsel_plan_for(T.DSEL_BF16 if dtype == "bf16" else T.DSEL_F32, rows, stride, k, order,
                               num_sms=torch.cuda.get_device_properties(0).multi_processor_count)
    if order == T.DSEL_ORDER_VALUE:
        assert st == 0 and plan["kernel"] == T.DSEL_KERNEL_STREAM, "value order takes the streaming kernel"
    else:
        assert st == 0 and plan["kernel"] == T.DSEL_KERNEL_SLICE and plan["cluster"] >= 2
        assert rows * plan["cluster"] <= torch.cuda.get_device_properties(0).multi_processor_count
    w = W.random_small(seed, dtype, rows, stride, k, dist=dist, with_end=(seed % 2 == 0),
                       end_lo=0, sorted_index=1, return_value=1, index_dtype="i64")
    check(w, order=order)


def test_pr1_duplicates_full():
    check(W.pr1_duplicates())


def test_indexer_drift_full():
    w = W.indexer_drift()
    check(w)                                  # sorted 0, no values, int32 (as benchmarked)
    check(w, order=1, return_value=1)


@pytest.mark.parametrize("rv", [0, 1])
def test_indexer_varlen_full(rv):
    w = W.indexer_varlen(return_value=rv)
    check(w)


@pytest.mark.parametrize("batch", [1, 8, 64, 256])
@pytest.mark.parametrize("k", [50, 1024, 4096])
def test_sampler_full(batch, k):
    check(W.sampler_logits(batch, k))


@pytest.mark.parametrize("dist", ["ascending", "equal"])
def test_slice_lists_hold_a_sorted_top_k(dist):
    """64 sampler-sized rows at k = 4096 on the slice kernel, whose lists hold k + 2000
    entries or more: with ascending rows the last slice holds the whole top k; with
    equal keys every list overflows and the exact selection takes over"""
    st, p = T.dsel_plan_device(T.DSEL_F32, 64, 129280, 4096, T.DSEL_ORDER_INDEX)
    assert st == 0 and p["kernel"] == T.DSEL_KERNEL_SLICE and p["capacity"] >= 4096 + 2000
    w = W.random_small(31, "f32", 64, 129280, 4096, dist=dist, sorted_index=1)
    check(w, order=T.DSEL_ORDER_INDEX)
    check(w, order=T.DSEL_ORDER_NONE)


@pytest.mark.parametrize("rows,n", [(1, 1 << 28), (16, 1 << 24)])
@pytest.mark.parametrize("k", [1000, 4096])
def test_long_rows_uniform_full(rows, n, k):
    check(W.long_rows(rows, n, k, "uniform"))


@pytest.mark.parametrize("variant", ["desc", "equal"])
@pytest.mark.parametrize("rows,n", [(1, 1 << 28), (16, 1 << 24)])
def test_long_rows_closed_forms_full(variant, rows, n):
    """sorted-descending and all-equal rows: the answer is indices 0..k-1 (any size)."""
    k = 4096
    w = W.long_rows(rows, n, k, variant)
    gi, gv = run_gpu(w)
    assert (gi == np.arange(k)[None, :]).all()
    assert (gv == w.x[:, :k]).all()


@pytest.mark.parametrize("rows,n", [(1, 1 << 28), (16, 1 << 24)])
def test_long_rows_nan_flag_full(rows, n):
    w = W.long_rows(rows, n, 1000, "uniform", inject_nan=True)
    gi, _ = run_gpu(w)
    flagged = np.flatnonzero((gi == T.DSEL_IDX_NAN).all(axis=1))
    assert flagged.tolist() == w.nan_rows.tolist()
    clean = [r for r in range(rows) if r not in set(w.nan_rows.tolist())][:2]
    if clean:
        exp = expected(w, np.array(clean))
        compare(w, gi, None, O.OracleResult(exp.indices, None, exp.status, False), 1, clean)


@pytest.mark.parametrize("rows", [6, 160])
def test_value_order_short_rows(rows):
    """Rows no longer than k in value order come back sorted by value, like the
    selected rows (the oracle's value_order), padding last; they skip the NaN check,
    so a NaN is listed at its totalOrder place.  6 rows: the streaming kernel; 160
    rows of 256 B: the row-resident kernel."""
    rng = np.random.default_rng(31)
    k, stride = 64, 64
    pool = np.array([-np.inf, -1.5, -0.0, 0.0, 0.25, 0.25, 3.0, np.inf], dtype=np.float32)
    f = pool[rng.integers(0, len(pool), size=(rows, stride))]
    bits = f.view(np.uint32).copy()
    bits[0, 5] = 0x7FC00000      # +NaN: first in value order
    bits[1, 9] = 0xFFC00001      # -NaN: last among the real entries
    end = rng.integers(0, stride + 1, size=rows).astype(np.int32)
    end[0], end[1] = 40, 64
    w = W.Workload("short_value_order", "f32", bits, end, k, 2, 1, "i64", nan_mode="flag")
    st, plan = T.dsel_plan_for(T.DSEL_F32, rows, stride, k, T.DSEL_ORDER_VALUE,
                               num_sms=torch.cuda.get_device_properties(0).multi_processor_count)
    assert st == 0 and plan["kernel"] == (T.DSEL_KERNEL_RESIDENT if rows >= 148 else T.DSEL_KERNEL_STREAM)
    gi, gv = check(w, order=T.DSEL_ORDER_VALUE)
    assert gi[0, 0] == 5 and gv[0, 0] == 0x7FC00000
    assert gi[1, 63] == 9 and gv[1, 63] == 0xFFC00001
    for r in range(rows):
        assert (gi[r, end[r]:] == T.DSEL_IDX_PAD).all()
