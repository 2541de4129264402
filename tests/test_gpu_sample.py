"""GPU parity of dsel_topk_sample (TopK + sampling draw) against the CPU oracles.

The draw decides an integer from float32 arithmetic on the GPU and float64 in
the oracle, so a token may differ only where the oracle's prefix sums put the
target u * E_c, or the top-p cut, within rounding distance of a boundary; such
rows are accepted when the GPU token is a valid draw under that rounding, and
there must be few of them.  Row codes, the TopK part of the result (value order,
bit-exact) and the reported probability are compared directly."""
import numpy as np
import pytest
import torch

import oracle.sample_oracle as S
import oracle.topk_oracle as O
import row_wise_topk_b200 as T
import workloads as W
from gpu_util import compare, to_device_bits

pytestmark = pytest.mark.gpu

REL = 2e-5          # float32 rounding allowance on prefix sums, relative to the total weight


def run_sample(w, t, top_p, u, *, nan_mode="flag", return_topk=True):
    x = to_device_bits(w.x)
    end = None if w.end is None else torch.from_numpy(w.end.astype(np.int32)).cuda()
    ud = torch.from_numpy(u.astype(np.float32)).cuda()
    token = torch.full((w.rows,), 999, dtype=torch.int64, device="cuda")
    prob = torch.full((w.rows,), -5.0, dtype=torch.float32, device="cuda")
    val = idx = None
    if return_topk:
        val = torch.full((w.rows, w.k), 77, dtype=torch.int32, device="cuda")
        idx = torch.full((w.rows, w.k), 12345, dtype=torch.int64, device="cuda")
    st = T.dsel_topk_sample(x.data_ptr(), w.rows, w.row_stride, None if end is None else end.data_ptr(), w.k,
                            t, top_p, ud.data_ptr(), T.DSEL_NAN_FLAG if nan_mode == "flag" else T.DSEL_NAN_TRAP,
                            None if val is None else val.data_ptr(), None if idx is None else idx.data_ptr(),
                            token.data_ptr(), prob.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, T.dsel_status_string(st)
    torch.cuda.synchronize()
    out = (token.cpu().numpy(), prob.cpu().numpy())
    if return_topk:
        out += (idx.cpu().numpy(), val.cpu().numpy().view(np.uint32))
    return out


def valid_near_boundary(res, r, pos_g, u):
    """True when position pos_g is a draw that float32 rounding can produce: for
    a cut c within one of the oracle's (c itself, or a neighbour whose prefix sum
    lies within rounding of the top-p threshold), u * E_c lies within rounding of
    the interval [E_{pos_g - 1}, E_{pos_g}]."""
    pre = res.prefix[r]
    tot = pre[-1]
    eps = REL * tot
    c0 = int(res.kept[r])
    for c in (c0 - 1, c0, c0 + 1):
        if c < 1 or c > len(pre) or pos_g >= c:
            continue
        target = u * pre[c - 1]
        lo = pre[pos_g - 1] if pos_g > 0 else 0.0
        if lo - eps <= target <= pre[pos_g] + eps:
            return True
    return False


def check_sample(w, t, top_p, u, *, nan_mode="flag", return_topk=True, max_boundary_frac=0.01):
    res = S.oracle_sample(w.x, w.k, t, top_p, u, end=w.end, nan_mode=nan_mode)
    out = run_sample(w, t, top_p, u, nan_mode=nan_mode, return_topk=return_topk)
    token, prob = out[0], out[1]
    boundary = 0
    for r in range(w.rows):
        if res.token[r] < 0:
            assert token[r] == res.token[r], (r, token[r], res.token[r])
            assert np.isnan(prob[r])
            continue
        if token[r] == res.token[r]:
            assert prob[r] == pytest.approx(res.prob[r], rel=1e-4, abs=1e-7), (r, prob[r], res.prob[r])
            continue
        order = res.order[r]
        hit = np.flatnonzero(order == token[r])
        assert len(hit) == 1, f"row {r}: token {token[r]} is not a candidate"
        assert valid_near_boundary(res, r, int(hit[0]), float(u[r])), (r, token[r], res.token[r])
        boundary += 1
    assert boundary <= max(1, max_boundary_frac * w.rows), boundary
    if return_topk:
        idx, val = out[2], out[3]
        exp = O.oracle_topk(w.x, "f32", w.k, end=w.end, sorted_index=1, return_value=1, index_dtype="i64",
                            nan_mode=nan_mode)
        compare(w, idx, val, exp, T.DSEL_ORDER_VALUE)


@pytest.mark.parametrize("batch,k", [(1, 50), (8, 1024), (64, 4096), (256, 50), (256, 1024)])
@pytest.mark.parametrize("t,top_p", [(1.0, 1.0), (0.7, 0.9), (2.5, 0.5)])
def test_sampler_workload(batch, k, t, top_p):
    w = W.sampler_logits(batch, k)
    check_sample(w, t, top_p, W.uniforms(batch, seed=batch * 7 + k))


def test_greedy_and_degenerate_cuts():
    w = W.sampler_logits(16, 512)
    u = W.uniforms(16, seed=1)
    check_sample(w, 0.0, 0.9, u)            # greedy
    check_sample(w, 1.0, 1e-9, u)           # the cut keeps one candidate
    check_sample(w, 1e4, 1.0, u)            # nearly uniform weights


def test_row_shapes_and_codes():
    # short rows (end <= k), an empty row, a NaN row, an invalid end, ragged ends,
    # across the 512-thread plan
    rng = np.random.default_rng(21)
    rows, stride, k = 12, 8192, 300
    x = (rng.standard_normal((rows, stride)) * 2).astype(np.float32)
    x[3, 4000] = np.nan                      # long row with a NaN: code -2
    x[5, 10] = np.nan                        # short row with a NaN: code -2 (the draw checks it)
    end = np.array([8192, 100, 0, 8192, 7000, 200, 8192 + 16, 299, 300, 301, 8000, 1], dtype=np.int32)
    w = W.Workload("sample_shapes", "f32", W.f32_bits(x), end, k, sorted_index=2, return_value=1,
                   index_dtype="i64", nan_mode="flag")
    check_sample(w, 1.3, 0.8, W.uniforms(rows, seed=3))


@pytest.mark.parametrize("rows,stride,k", [(1, 1 << 22, 512), (3, 1 << 20, 2000), (200, 4096, 700)])
def test_plans(rows, stride, k):
    """split rows with a merge launch, clusters, and the 128-thread shape"""
    rng = np.random.default_rng(rows + k)
    x = (rng.standard_normal((rows, stride)) * 3).astype(np.float32)
    w = W.Workload("sample_plans", "f32", W.f32_bits(x), None, k, sorted_index=2, return_value=1,
                   index_dtype="i64", nan_mode="flag")
    check_sample(w, 0.9, 0.95, W.uniforms(rows, seed=k))


def test_token_only_call_matches():
    w = W.sampler_logits(8, 1024)
    u = W.uniforms(8, seed=9)
    a = run_sample(w, 0.8, 0.9, u)
    b = run_sample(w, 0.8, 0.9, u, return_topk=False)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
