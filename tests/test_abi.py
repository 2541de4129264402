"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates arguments on the host before touching CUDA, and the
host-side planner returns consistent plans."""
import ctypes
import os
import re

import pytest

import row_wise_topk_b200 as T

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dsel.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"DSEL_API\s+[\w\s\*]+?\b(dsel_\w+)\s*\(", text)


def header_define(name):
    m = re.search(r"#define\s+%s\s+\(?(-?\d+)\)?" % name, open(HEADER).read())
    return int(m.group(1))


def test_every_declared_symbol_is_exported():
    syms = declared_symbols()
    assert "dsel_topk" in syms and len(syms) >= 6
    lib = ctypes.CDLL(T.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), s


def test_python_constants_match_header():
    for name in ["DSEL_BF16", "DSEL_F32", "DSEL_I32", "DSEL_I64", "DSEL_NAN_TRAP", "DSEL_NAN_FLAG",
                 "DSEL_ORDER_NONE", "DSEL_ORDER_INDEX", "DSEL_ORDER_VALUE", "DSEL_IDX_PAD",
                 "DSEL_IDX_NAN", "DSEL_IDX_BAD_END", "DSEL_OK"]:
        assert getattr(T, name) == header_define(name), name


def test_stride_requirement_and_strings():
    assert T.dsel_stride_requirement(T.DSEL_BF16) == 16
    assert T.dsel_stride_requirement(T.DSEL_F32) == 16
    assert T.dsel_stride_requirement(7) == -1
    for code in range(0, -17, -1):
        s = T.dsel_status_string(code)
        assert s and s != "unknown status", code
    assert T.dsel_status_string(-99) == "unknown status"
    assert "sm_100a" in T.dsel_version()


def call(**kw):
    a = dict(x=0x1000, dtype=T.DSEL_F32, rows=4, row_stride=8192, end=None, k=64, sorted_index=1,
             return_value=1, index_dtype=T.DSEL_I64, nan_mode=T.DSEL_NAN_TRAP, values_out=0x2000,
             indices_out=0x3000, stream=None)
    a.update(kw)
    return T.dsel_topk(**a)


@pytest.mark.parametrize("kw,err", [
    (dict(dtype=2), "DSEL_ERR_DTYPE"),
    (dict(k=0), "DSEL_ERR_K"),
    (dict(k=4097), "DSEL_ERR_K"),
    (dict(rows=-1), "DSEL_ERR_ROWS"),
    (dict(row_stride=8190), "DSEL_ERR_STRIDE"),
    (dict(row_stride=0), "DSEL_ERR_STRIDE"),
    (dict(row_stride=1 << 32), "DSEL_ERR_STRIDE"),
    (dict(index_dtype=3), "DSEL_ERR_INDEX_DTYPE"),
    (dict(nan_mode=2), "DSEL_ERR_NAN_MODE"),
    (dict(sorted_index=3), "DSEL_ERR_ORDER"),
    (dict(sorted_index=2, dtype=T.DSEL_BF16), "DSEL_ERR_ORDER"),
    (dict(x=None), "DSEL_ERR_NULL"),
    (dict(indices_out=None), "DSEL_ERR_NULL"),
    (dict(values_out=None), "DSEL_ERR_VALUES"),
    (dict(return_value=0), "DSEL_ERR_VALUES"),
    (dict(return_value=2), "DSEL_ERR_VALUES"),
    (dict(x=0x1004), "DSEL_ERR_ALIGN"),
])
def test_host_argument_checks(kw, err):
    assert call(**kw) == header_define(err)


@pytest.mark.parametrize("kw,err", [
    (dict(dtype=2), "DSEL_ERR_DTYPE"),
    (dict(k=4097), "DSEL_ERR_K"),
    (dict(rows=-1), "DSEL_ERR_ROWS"),
    (dict(row_stride=8200), "DSEL_ERR_STRIDE"),
    (dict(index_dtype=2), "DSEL_ERR_INDEX_DTYPE"),
    (dict(nan_mode=-1), "DSEL_ERR_NAN_MODE"),
    (dict(sorted_index=2, dtype=T.DSEL_BF16), "DSEL_ERR_ORDER"),
    (dict(x=None), "DSEL_ERR_NULL"),
    (dict(values_out=None), "DSEL_ERR_VALUES"),
    (dict(x=0x1002), "DSEL_ERR_ALIGN"),
])
def test_noalloc_host_argument_checks(kw, err):
    assert call_noalloc(**kw) == header_define(err)


def call_noalloc(**kw):
    a = dict(x=0x1000, dtype=T.DSEL_F32, rows=4, row_stride=8192, end=None, k=64, sorted_index=1,
             return_value=1, index_dtype=T.DSEL_I64, nan_mode=T.DSEL_NAN_TRAP, values_out=0x2000,
             indices_out=0x3000, stream=None)
    a.update(kw)
    return T.dsel_topk_noalloc(**a)


def test_noalloc_zero_rows_is_a_noop():
    assert call_noalloc(rows=0, x=None, indices_out=None, values_out=None, return_value=0) == 0


def _stack(**kw):
    a = dict(vals_in=0x1000, idx_in=0x2000, dtype=T.DSEL_F32, rows=3, k=64, shards=2, shard_len=4096,
             out_stride=128, vals_out=0x3000, idx_out=0x4000, stream=None)
    a.update(kw)
    return T.lib.dsel_shard_stack(*a.values())


def _take(**kw):
    a = dict(table=0x1000, table_stride=128, pos=0x2000, pos_dtype=T.DSEL_I64, rows=3, k=64,
             index_dtype=T.DSEL_I32, indices_out=0x3000, stream=None)
    a.update(kw)
    return T.lib.dsel_take_index(*a.values())


@pytest.mark.parametrize("kw,err", [
    (dict(dtype=5), "DSEL_ERR_DTYPE"),
    (dict(k=0), "DSEL_ERR_K"),
    (dict(shards=0), "DSEL_ERR_K"),
    (dict(shard_len=63), "DSEL_ERR_K"),                 # every shard must give k real candidates
    (dict(rows=-2), "DSEL_ERR_ROWS"),
    (dict(out_stride=112), "DSEL_ERR_STRIDE"),          # < shards * k
    (dict(out_stride=136), "DSEL_ERR_STRIDE"),          # not a multiple of 16
    (dict(idx_out=None), "DSEL_ERR_NULL"),
])
def test_shard_stack_host_argument_checks(kw, err):
    assert _stack(**kw) == header_define(err)


@pytest.mark.parametrize("kw,err", [
    (dict(k=4097), "DSEL_ERR_K"),
    (dict(table_stride=0), "DSEL_ERR_K"),
    (dict(rows=-1), "DSEL_ERR_ROWS"),
    (dict(pos_dtype=2), "DSEL_ERR_INDEX_DTYPE"),
    (dict(index_dtype=7), "DSEL_ERR_INDEX_DTYPE"),
    (dict(pos=None), "DSEL_ERR_NULL"),
])
def test_take_index_host_argument_checks(kw, err):
    assert _take(**kw) == header_define(err)


def test_shard_steps_with_zero_rows_are_noops():
    assert _stack(rows=0, vals_in=None, idx_in=None, vals_out=None, idx_out=None) == 0
    assert _take(rows=0, table=None, pos=None, indices_out=None) == 0


def call_sample(**kw):
    a = dict(x=0x1000, rows=4, row_stride=8192, end=None, k=64, temperature=1.0, top_p=0.9, u=0x4000,
             nan_mode=T.DSEL_NAN_FLAG, values_out=0x2000, indices_out=0x3000, token_out=0x5000, prob_out=None,
             stream=None)
    a.update(kw)
    return T.dsel_topk_sample(**a)


@pytest.mark.parametrize("kw,err", [
    (dict(k=0), "DSEL_ERR_K"),
    (dict(k=4097), "DSEL_ERR_K"),
    (dict(rows=-1), "DSEL_ERR_ROWS"),
    (dict(row_stride=8190), "DSEL_ERR_STRIDE"),
    (dict(nan_mode=5), "DSEL_ERR_NAN_MODE"),
    (dict(x=None), "DSEL_ERR_NULL"),
    (dict(u=None), "DSEL_ERR_NULL"),
    (dict(token_out=None), "DSEL_ERR_NULL"),
    (dict(values_out=None), "DSEL_ERR_VALUES"),
    (dict(indices_out=None), "DSEL_ERR_VALUES"),
    (dict(x=0x1008), "DSEL_ERR_ALIGN"),
])
def test_sample_host_argument_checks(kw, err):
    assert call_sample(**kw) == header_define(err)


def test_sample_zero_rows_is_a_noop():
    assert call_sample(rows=0, x=None, u=None, token_out=None) == 0


def test_zero_rows_is_a_noop():
    assert call(rows=0, x=None, indices_out=None, values_out=None, return_value=0) == 0


PEAK = dict(num_sms=148, smem_optin=232448, max_cluster=8)


@pytest.mark.parametrize("dtype,rows,stride,k", [
    (T.DSEL_F32, 4, 8192, 64),
    (T.DSEL_BF16, 64, 131072, 512),
    (T.DSEL_BF16, 4096, 16384, 512),
    (T.DSEL_F32, 1, 129280, 50), (T.DSEL_F32, 8, 129280, 1024), (T.DSEL_F32, 64, 129280, 4096),
    (T.DSEL_F32, 256, 129280, 4096), (T.DSEL_F32, 256, 129280, 1024), (T.DSEL_BF16, 300, 131072, 512),
    (T.DSEL_F32, 1, 1 << 28, 1000), (T.DSEL_F32, 16, 1 << 24, 4096),
    (T.DSEL_BF16, 3, 16, 4096), (T.DSEL_F32, 1, 16, 1),
    (T.DSEL_BF16, 4096, 16400, 512), (T.DSEL_F32, 300, 8192, 4096), (T.DSEL_F32, 300, 8208, 64),
    (T.DSEL_BF16, 148, 16, 4096), (T.DSEL_F32, 200, 4096, 1),
    (T.DSEL_BF16, 100, 65536, 512), (T.DSEL_F32, 37, 131072, 1000), (T.DSEL_BF16, 20, 1 << 19, 64),
    (T.DSEL_F32, 73, 32768, 64), (T.DSEL_BF16, 147, 16400, 4096),
])
def test_plan_invariants(dtype, rows, stride, k):
    st, p = T.dsel_plan(dtype, rows, stride, k, **PEAK)
    assert st == 0
    check_plan(dtype, rows, stride, k, p)


def check_plan(dtype, rows, stride, k, p, fit=None):
    """What a plan must hold for its kernel's buffers and launch (fit: the cluster
    capacity a fitted plan was made for, else None for the host plan)."""
    eb = 2 if dtype == T.DSEL_BF16 else 4
    assert p["smem_bytes"] <= PEAK["smem_optin"]
    assert p["kernel"] in (T.DSEL_KERNEL_STREAM, T.DSEL_KERNEL_RESIDENT, T.DSEL_KERNEL_SLICE)
    if p["kernel"] == T.DSEL_KERNEL_SLICE:
        # rows cut into `cluster` slices, each held whole in one CTA's shared memory as
        # chunks of 16 KB, plus the CTA's candidate lists; 512 threads from 4 chunks
        assert p["threads"] == (512 if p["stages"] >= 4 else 256)
        assert p["groups"] == 1 and 1 <= p["cluster"] <= 16
        assert p["round"] % 16 == 0 and p["round"] * p["cluster"] >= stride
        assert p["block"] * eb == 16384 and p["stages"] == -(-p["round"] // p["block"]) <= 8
        assert p["capacity"] >= k + 2000 and p["capacity"] % 32 == 0          # candidate list
        assert p["smem_bytes"] >= p["stages"] * (16384 + 2048) + p["capacity"] * (eb + 4) + 5 * 4096
        assert p["b2"] == 0 and p["workspace_bytes"] == 0
        assert (1 << p["idx_bits"]) >= stride
        # as few slices as fit (8 chunks and a list of k + 2000), or more while the
        # batch leaves SMs idle (but no slice under 8192 elements)
        def fits(c):
            sl = (-(-stride // c) + 15) // 16 * 16
            ch = -(-sl * eb // 16384)
            fixed = ch * (16384 + 2048) + -(-ch * 8 // 16) * 16 + 5632 * 4 + 1024 + 64
            lcap = min(16384, (PEAK["smem_optin"] - fixed) // (eb + 6)) // 32 * 32
            return ch <= 8 and lcap >= k + 2000
        assert fits(p["cluster"])
        assert p["cluster"] == 1 or not fits(p["cluster"] - 1) or \
            (rows * p["cluster"] <= PEAK["num_sms"] and p["cluster"] <= min(8, -(-stride // 8192)))
        return
    if rows >= PEAK["num_sms"] and stride * eb <= 32 * 1024:
        # rows that fit in shared memory: one 256-thread CTA per row holds the whole row
        assert p["kernel"] == T.DSEL_KERNEL_RESIDENT
        assert (p["threads"], p["cluster"], p["groups"], p["b2"]) == (256, 1, 1, 0)
        assert p["block"] * eb == 4096 and p["round"] == stride
        assert p["stages"] == -(-(stride * eb) // 4096) <= 8
        assert p["capacity"] == 1 << (k - 1).bit_length()          # value order sorts k entries in place
        assert p["smem_bytes"] >= stride * eb + 3 * 4096 + p["capacity"] * (eb + 4)
        assert (1 << p["idx_bits"]) >= stride and p["workspace_bytes"] == 0
        return
    assert p["kernel"] == T.DSEL_KERNEL_STREAM
    slack = 1024 if p["threads"] != 512 else (4096 if k <= 1024 else 2048)
    assert p["capacity"] >= k + p["b2"] + slack
    assert p["capacity"] >= 1 << (k - 1).bit_length()          # room for the bitonic padding
    assert p["capacity"] >= 4096                                 # the round-0 seed histograms
    q = p["round"] // p["block"]
    slice_ = -(-(-(-stride // (p["cluster"] * p["groups"]))) // 16) * 16
    nb_max = -(-slice_ // p["block"])
    assert p["stages"] == nb_max or (p["stages"] % q == 0 and p["stages"] < nb_max)
    assert p["threads"] in (128, 256, 512)
    assert p["round"] == p["threads"] * (16 if dtype == T.DSEL_BF16 else 8) * (16 // eb)
    if p["threads"] == 128:   # short rows: one CTA per row, one round in flight, several CTAs per SM
        assert rows >= PEAK["num_sms"] and stride <= 2 * p["round"]
        assert (p["cluster"], p["groups"]) == (1, 1) and p["stages"] <= q
        assert p["smem_bytes"] <= 232448 // 2
    if p["threads"] == 256:   # long rows, k <= 1024: one CTA per row, two CTAs per SM
        assert rows >= PEAK["num_sms"] and k <= 1024
        assert (p["cluster"], p["groups"]) == (1, 1)
        assert 2 * (p["smem_bytes"] + 1024) <= PEAK["smem_optin"] + 1024
    assert p["round"] % p["block"] == 0 and (p["block"] * eb) % 16 == 0
    assert 1 <= p["cluster"] <= (PEAK["max_cluster"] if fit is None else 16)
    assert p["groups"] >= 1 and p["groups"] * k <= 8 * p["capacity"]
    if fit is not None and p["cluster"] > PEAK["max_cluster"]:
        assert rows * p["groups"] <= fit[p["cluster"]]          # non-portable sizes only where they fit
    assert (1 << p["idx_bits"]) >= stride
    assert p["idx_bits"] + 8 * eb <= 63
    if p["groups"] > 1:
        assert p["workspace_bytes"] >= rows * p["groups"] * k * 8
    else:
        assert p["workspace_bytes"] == 0
    # the row is split at most once per SM
    assert rows * p["cluster"] * p["groups"] <= max(rows, PEAK["num_sms"])


def test_plan_splits():
    # many rows of at most 32 KB: the row-resident kernel; a little longer: the
    # streaming kernel's 128-thread shape
    p = T.dsel_plan(T.DSEL_BF16, 4096, 16384, 512, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_RESIDENT and p["threads"] == 256
    p = T.dsel_plan(T.DSEL_BF16, 4096, 16400, 512, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_STREAM and p["threads"] == 128
    # the slice kernel only while at most four waves of slices cover the batch
    p = T.dsel_plan(T.DSEL_BF16, 64, 131072, 512, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_SLICE and p["cluster"] * 64 <= PEAK["num_sms"]
    p = T.dsel_plan(T.DSEL_F32, 64, 129280, 4096, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_SLICE and p["cluster"] * 64 <= 4 * PEAK["num_sms"]
    p = T.dsel_plan(T.DSEL_F32, 256, 129280, 1024, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_STREAM
    # value order never takes the slice kernel
    p = T.dsel_plan_for(T.DSEL_F32, 256, 129280, 1024, T.DSEL_ORDER_VALUE, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_STREAM and p["threads"] == 256
    assert T.dsel_plan_for(T.DSEL_F32, 256, 129280, 1024, T.DSEL_ORDER_INDEX, **PEAK)[1] == \
        T.dsel_plan(T.DSEL_F32, 256, 129280, 1024, **PEAK)[1]
    assert T.dsel_plan_for(T.DSEL_F32, 4, 8192, 64, 3, **PEAK)[0] == header_define("DSEL_ERR_ORDER")
    # fewer rows than SMs: never resident
    assert T.dsel_plan(T.DSEL_BF16, 147, 16384, 512, **PEAK)[1]["kernel"] == T.DSEL_KERNEL_SLICE
    # rows longer than sixteen 128 KB slices: the streaming kernel
    assert T.dsel_plan(T.DSEL_F32, 256, 1 << 20, 4096, **PEAK)[1]["kernel"] == T.DSEL_KERNEL_STREAM
    # long rows, k <= 1024, at least as many rows as SMs: 256 threads, two CTAs per SM
    assert T.dsel_plan(T.DSEL_F32, 256, 1 << 20, 1024, **PEAK)[1]["threads"] == 256
    # 64 indexer rows: two slices per row, each held in one CTA's shared memory
    p = T.dsel_plan(T.DSEL_BF16, 64, 131072, 512, **PEAK)[1]
    assert (p["kernel"], p["cluster"], p["groups"]) == (T.DSEL_KERNEL_SLICE, 2, 1)
    # one or eight sampler rows: eight slices per row (spreading a row further only to
    # fill idle SMs stops at the portable cluster size); 256 rows (several waves of
    # slices): the streaming kernel
    assert T.dsel_plan(T.DSEL_F32, 1, 129280, 50, **PEAK)[1]["cluster"] == 8
    assert T.dsel_plan(T.DSEL_F32, 8, 129280, 1024, **PEAK)[1]["cluster"] == 8
    # a row that needs more than eight slices to fit still takes a larger cluster
    p = T.dsel_plan(T.DSEL_F32, 1, 393216, 512, **PEAK)[1]   # 1.5 MB: twelve slices of 128 KB
    assert (p["kernel"], p["cluster"]) == (T.DSEL_KERNEL_SLICE, 12)
    p = T.dsel_plan(T.DSEL_F32, 256, 129280, 1024, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_STREAM
    # a single 2^28 row uses several clusters
    p = T.dsel_plan(T.DSEL_F32, 1, 1 << 28, 1000, **PEAK)[1]
    assert p["groups"] > 1 and p["cluster"] == 8


def test_plan_rejects_bad_args():
    assert T.dsel_plan(T.DSEL_F32, 4, 8191, 64, **PEAK)[0] == header_define("DSEL_ERR_STRIDE")
    assert T.dsel_plan(T.DSEL_F32, 4, 8192, 5000, **PEAK)[0] == header_define("DSEL_ERR_K")


def test_resident_plan_fits_four_ctas_per_sm():
    # the varlen indexer batch: 16,384-element bf16 rows, k = 512; a B200 SM has 228 KB of
    # shared memory and reserves 1 KB per CTA
    p = T.dsel_plan(T.DSEL_BF16, 4096, 16384, 512, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_RESIDENT
    assert 4 * (p["smem_bytes"] + 1024) <= 228 * 1024
    # value order with the largest k on f32 rows still fits one CTA's opt-in limit
    p = T.dsel_plan(T.DSEL_F32, 4096, 8192, 4096, **PEAK)[1]
    assert p["kernel"] == T.DSEL_KERNEL_RESIDENT and p["smem_bytes"] <= PEAK["smem_optin"]


def _best_split(rows, stride, k, capacity, fit, sms=148):
    """The largest number of CTAs over the (cluster, groups) splits of a row whose
    clusters all fit at once, and the fewest groups reaching it (the rule stated for
    dsel_plan_fit); None when no size fits."""
    splits = max(1, min(sms // max(rows, 1), stride // 8192))
    max_groups = min(255, max(1, 8 * capacity // k))
    best = None
    for c in range(2, min(splits, 16) + 1):
        if fit[c] < 1:
            continue
        g = min(max(1, splits // c), max_groups)
        if rows * g > fit[c]:
            g = fit[c] // rows
        if g >= 1 and (best is None or (c * g, -g) > (best[0] * best[1], -best[1])):
            best = (c, g)
    return best


@pytest.mark.parametrize("fit", [
    [0] + [148 // c for c in range(1, 17)],                                   # every SM usable by any cluster
    [0, 148, 74, 49, 36, 29, 24, 21, 12, 9, 8, 8, 8, 8, 8, 8, 8],             # large clusters scarce (GPC bound)
    [0, 148, 70, 45, 32, 24, 20, 16, 14, 0, 0, 0, 0, 0, 0, 0, 0],             # no cluster above the portable 8
])
@pytest.mark.parametrize("rows,stride,k", [(16, 1 << 24, 4096), (16, 1 << 24, 1000), (1, 1 << 28, 1000),
                                           (1, 1 << 28, 4096), (10, 1 << 20, 1024), (3, 1 << 21, 2000),
                                           (2, 1 << 20, 64)])
def test_fitted_split_keeps_every_cluster_in_one_wave(fit, rows, stride, k):
    st, p = T.dsel_plan_fit(T.DSEL_F32, rows, stride, k, T.DSEL_ORDER_INDEX, fit)
    assert st == 0 and p["kernel"] == T.DSEL_KERNEL_STREAM
    c, g = p["cluster"], p["groups"]
    assert rows * g <= fit[c]                                   # every cluster of the launch at once
    assert (c, g) == _best_split(rows, stride, k, p["capacity"], fit)
    assert p["workspace_bytes"] == (rows * g * (k * 8 + 8) if g > 1 else 0)


def test_fitted_split_when_sixteen_clusters_of_eight_do_not_fit():
    # a capacity in which sixteen clusters of 8 (or 9) do not fit at once, nor 48 of
    # 3: two groups of clusters of 4 (128 CTAs) beat one of 7 (112)
    fit = [0, 148, 74, 40, 36, 28, 24, 21, 12, 9, 8, 8, 8, 8, 8, 8, 8]
    p = T.dsel_plan_fit(T.DSEL_F32, 16, 1 << 24, 4096, T.DSEL_ORDER_INDEX, fit)[1]
    assert (p["cluster"], p["groups"]) == (4, 2)
    # the host planner, with no capacity to go by, keeps the portable split
    h = T.dsel_plan_for(T.DSEL_F32, 16, 1 << 24, 4096, T.DSEL_ORDER_INDEX, **PEAK)[1]
    assert (h["cluster"], h["groups"]) == (8, 1)


def test_fitted_plan_is_the_host_plan_without_a_split():
    fit = [0] + [148 // c for c in range(1, 17)]
    for args in [(T.DSEL_BF16, 64, 131072, 512, 0), (T.DSEL_F32, 256, 129280, 1024, 1),
                 (T.DSEL_BF16, 4096, 16384, 512, 1), (T.DSEL_F32, 8, 129280, 50, 1),
                 (T.DSEL_F32, 256, 129280, 1024, T.DSEL_ORDER_VALUE)]:
        assert T.dsel_plan_fit(*args, fit) == T.dsel_plan_for(*args, **PEAK)
    # no cluster size fits at all: the portable split
    none = [0, 148] + [0] * 15
    assert T.dsel_plan_fit(T.DSEL_F32, 16, 1 << 24, 4096, 1, none) == \
        T.dsel_plan_for(T.DSEL_F32, 16, 1 << 24, 4096, 1, **PEAK)
    assert T.dsel_plan_fit(T.DSEL_F32, 16, 1 << 24, 4096, 3, none)[0] == header_define("DSEL_ERR_ORDER")


FITS = [
    [0] + [148 // c for c in range(1, 17)],
    [0, 148, 74, 49, 36, 29, 24, 21, 12, 9, 8, 8, 8, 8, 8, 8, 8],
    [0, 148, 70, 45, 32, 24, 20, 16, 14, 0, 0, 0, 0, 0, 0, 0, 0],
]


def _random_shapes(seed, n):
    """Seeded shapes spread log-uniformly: 1..8192 rows, row strides of 16..2^28
    elements (multiples of 16), k = 1..4096, both dtypes."""
    import numpy as np
    rng = np.random.default_rng(seed)
    for _ in range(n):
        dtype = T.DSEL_BF16 if rng.random() < 0.5 else T.DSEL_F32
        rows = int(np.exp(rng.uniform(0, np.log(8192))))
        stride = 16 * max(1, int(np.exp(rng.uniform(0, np.log(1 << 24)))))
        k = max(1, min(4096, int(np.exp(rng.uniform(0, np.log(4097))))))
        yield dtype, rows, stride, k


@pytest.mark.parametrize("seed", [11, 12, 13])
def test_random_shapes_plan_within_their_buffers(seed):
    # every valid shape gets a plan, in every order, on the host and on each fitted
    # capacity, and each plan holds what its kernel's buffers and launch need
    orders = [T.DSEL_ORDER_NONE, T.DSEL_ORDER_INDEX, T.DSEL_ORDER_VALUE]
    for dtype, rows, stride, k in _random_shapes(seed, 200):
        for order in orders:
            if order == T.DSEL_ORDER_VALUE and dtype == T.DSEL_BF16:
                continue
            st, h = T.dsel_plan_for(dtype, rows, stride, k, order, **PEAK)
            assert st == 0, (dtype, rows, stride, k, order)
            check_plan(dtype, rows, stride, k, h)
            if order == T.DSEL_ORDER_VALUE:
                assert h["kernel"] != T.DSEL_KERNEL_SLICE
            for fit in FITS:
                st, f = T.dsel_plan_fit(dtype, rows, stride, k, order, fit)
                assert st == 0, (dtype, rows, stride, k, order, fit)
                check_plan(dtype, rows, stride, k, f, fit=fit)
                # the capacity only moves a long row's split over clusters and groups
                assert (f["kernel"], f["threads"], f["round"], f["block"], f["b2"]) == \
                    (h["kernel"], h["threads"], h["round"], h["block"], h["b2"])
                if (f["cluster"], f["groups"]) != (h["cluster"], h["groups"]):
                    assert f["kernel"] == T.DSEL_KERNEL_STREAM and rows < PEAK["num_sms"]
                    assert rows * f["groups"] <= fit[f["cluster"]]
                    assert (f["cluster"], f["groups"]) == \
                        _best_split(rows, stride, k, f["capacity"], fit)


def test_binding_fails_loudly_without_the_library():
    # no CPU fallback: importing the binding with its library absent raises
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, ROW_WISE_TOPK_LIB="libdsel_not_built.so")
    res = subprocess.run([sys.executable, "-c", "import row_wise_topk_b200"], cwd=root, env=env,
                         capture_output=True, text=True, timeout=120)
    assert res.returncode != 0
    assert "ImportError" in res.stderr and "no fallback" in res.stderr
