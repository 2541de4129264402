"""GPU parity of the row-resident kernel (at least as many rows as SMs, rows of at
most 32 KB held whole in shared memory) against the CPU oracle.

The cases reach every branch of its selection: the vector-maximum seed and rows
with fewer vectors than k (no seed), one histogram level of single keys, deeper
levels over wide key ranges (f32, +-inf with heavy ties), the small-bucket
ranking, partial chunks and partial vectors (ragged ``end``), rows no longer than
k, NaN and invalid-``end`` rows in the flag mode, every output order and index
type, and the sampling step on top of it."""
import numpy as np
import pytest
import torch

import oracle.topk_oracle as O
import row_wise_topk_b200 as T
import workloads as W
from gpu_util import check, compare, expected, run_gpu

pytestmark = pytest.mark.gpu

F32, BF16 = "f32", "bf16"


def n_sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def assert_resident(dtype, rows, stride, k):
    st, plan = T.dsel_plan(T.DSEL_BF16 if dtype == BF16 else T.DSEL_F32, rows, stride, k, num_sms=n_sms())
    assert st == 0 and plan["kernel"] == T.DSEL_KERNEL_RESIDENT, "the case must use the row-resident kernel"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert T.dsel_device_status() == 0


CASES = [
    # (seed, dtype, rows, stride, k, dist, order, with_end)
    (501, BF16, 150, 16384, 512, "normal", 1, True),
    (502, BF16, 150, 16384, 512, "ties", 1, False),
    (503, BF16, 160, 16384, 4096, "normal", 0, True),
    (504, BF16, 148, 8208, 1, "normal", 1, False),        # a partial last chunk (32 B)
    (505, BF16, 200, 2048, 512, "ascending", 1, True),    # no seed (fewer vectors than k)
    (506, BF16, 300, 1024, 2000, "ties", 0, True),        # every row no longer than k
    (507, BF16, 149, 16384, 7, "equal", 1, False),
    (508, BF16, 150, 12304, 64, "ties", 0, True),
    (511, F32, 150, 8192, 1024, "normal", 2, True),       # value order
    (512, F32, 150, 8192, 4096, "normal", 1, False),
    (513, F32, 160, 8192, 50, "ties", 1, True),           # levels of 32-bit keys down to one key
    (514, F32, 148, 4112, 4096, "normal", 0, False),      # n barely above k
    (515, F32, 200, 6144, 700, "ascending", 2, True),
    (516, F32, 150, 1040, 1, "equal", 1, True),
    (517, F32, 150, 16, 4, "normal", 1, True),            # tiny rows
]


@pytest.mark.parametrize("seed,dtype,rows,stride,k,dist,order,with_end", CASES)
def test_resident_cases(seed, dtype, rows, stride, k, dist, order, with_end):
    assert_resident(dtype, rows, stride, k)
    w = W.random_small(seed, dtype, rows, stride, k, dist=dist, with_end=with_end, end_lo=0,
                       sorted_index=1, return_value=1, index_dtype="i64")
    check(w, order=order)


@pytest.mark.parametrize("dtype", [BF16, F32])
@pytest.mark.parametrize("rv", [0, 1])
@pytest.mark.parametrize("idt", ["i32", "i64"])
def test_resident_options(dtype, rv, idt):
    stride = 16384 if dtype == BF16 else 8192
    assert_resident(dtype, 150, stride, 300)
    w = W.random_small(21, dtype, 150, stride, 300, dist="normal", with_end=True, end_lo=100)
    check(w, order=1, return_value=rv, index_dtype=idt)


def test_resident_dense_cluster_levels():
    """f32 rows whose k-th value sits in a dense run of consecutive floats, with
    outliers stretching the key range to nearly all 2^32 keys: the histogram has to
    descend several levels (bins of 2^22, 2^12, 2^2 keys, then one key, or ranking)."""
    rng = np.random.default_rng(77)
    rows, n, k = 150, 8192, 1000
    base = np.float32(1.0)
    run = base + np.arange(3000, dtype=np.float32) * np.finfo(np.float32).eps   # consecutive floats
    x = np.empty((rows, n), dtype=np.float32)
    for r in range(rows):
        v = np.concatenate([rng.permutation(run), rng.uniform(-1e30, 0.5, n - 3000 - 2).astype(np.float32),
                            np.array([3e38, -3e38], dtype=np.float32)])
        x[r] = v[rng.permutation(n)]
    w = W.Workload("dense_cluster", F32, W.f32_bits(x), None, k, sorted_index=1, return_value=1,
                   index_dtype="i64")
    assert_resident(F32, rows, n, k)
    check(w)


def test_resident_quantised_varlen():
    w = W.indexer_varlen(rows=300, stride=16384, return_value=1)
    assert_resident(BF16, 300, 16384, 512)
    check(w)


@pytest.mark.parametrize("dtype", [BF16, F32])
def test_resident_nan_and_bad_end_rows(dtype):
    stride = 4096
    rows = 160
    nan_rows = np.arange(3, rows, 7)
    w = W.random_small(33, dtype, rows, stride, 100, dist="normal", with_end=True, end_lo=0, nan_rows=nan_rows,
                       nan_mode="flag")
    end = w.end.copy()
    end[5] = stride + 16      # past the stride: flagged
    end[6] = -1               # negative: flagged
    w.end[:] = end
    assert_resident(dtype, rows, stride, 100)
    gi, gv = run_gpu(w, order=1)
    exp = expected(w)
    compare(w, gi, gv, exp, 1)
    assert (gi[5] == T.DSEL_IDX_BAD_END).all() and (gi[6] == T.DSEL_IDX_BAD_END).all()
    lens = w.end
    flagged = [r for r in nan_rows if 0 <= lens[r] <= stride and lens[r] > w.k]
    assert flagged and all((gi[r] == T.DSEL_IDX_NAN).all() for r in flagged)


def test_resident_sampling_step():
    from test_gpu_sample import check_sample

    rng = np.random.default_rng(9)
    rows, n, k = 160, 8192, 256
    x = (3.0 * rng.standard_normal((rows, n))).astype(np.float32)
    w = W.Workload("resident_sample", F32, W.f32_bits(x), None, k, sorted_index=1, return_value=1,
                   index_dtype="i64")
    assert_resident(F32, rows, n, k)
    u = W.uniforms(rows, seed=11)
    check_sample(w, 0.8, 0.9, u)
    check_sample(w, 0.0, 1.0, u, return_topk=False)

