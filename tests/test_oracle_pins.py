"""Pins for the CPU oracle: checks against things other than the oracle itself.

* hand-worked cases (tests/golden/hand_cases.json) for ties, signed zeros,
  infinities, subnormals, short rows, NaN rows and ``end``;
* an exhaustive bfloat16 decode against torch's own bfloat16 conversion, and
  float32 edge patterns against ``struct``;
* the partition-based selection against a full sort (brute force) on many small
  rows with heavy ties;
* closed forms (ascending, descending, all-equal rows);
* the invariants every result must satisfy, on small versions of every workload;
* torch.topk's sorted values (a library routine) on NaN-free rows.

The mutation tests at the end plant one plausible mistake at a time in the
oracle and check that some pin above catches it.
"""
import json
import os
import struct

import numpy as np
import pytest
import torch

import oracle.topk_oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _load_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def hand_case_failures(oracle_fn):
    bad = []
    for c in _load_cases():
        bits_t = np.uint16 if c["dtype"] == "bf16" else np.uint32
        row = np.array([int(h, 16) for h in c["row"]], dtype=bits_t)[None, :]
        end = None if "end" not in c else np.array([c["end"]], dtype=np.int32)
        res = oracle_fn(row, c["dtype"], c["k"], end=end, sorted_index=1, return_value=1,
                        index_dtype="i64", nan_mode=c.get("nan_mode", "trap"))
        got_idx = res.indices[0].tolist()
        got_val = ["%0*x" % (4 if c["dtype"] == "bf16" else 8, int(v)) for v in res.values[0]]
        if got_idx != c["indices"] or got_val != c["values"] or int(res.status[0]) != c["status"]:
            bad.append((c["name"], got_idx, got_val, int(res.status[0])))
    return bad


def brute_force_failures(select_fn, trials=400, seed=11):
    rng = np.random.default_rng(seed)
    pool = np.array([-np.inf, -3.0, -1.0, -0.0, 0.0, 0.25, 1.0, 7.0, np.inf])
    bad = []
    for t in range(trials):
        n = int(rng.integers(2, 41))
        if t % 3 == 0:
            v = rng.standard_normal(n)
        else:
            v = pool[rng.integers(0, len(pool), size=n)]
        for k in range(1, n):
            got = select_fn(v.copy(), k).tolist()
            want = O.brute_force_row(v, k)
            if got != want:
                bad.append((v.tolist(), k, got, want))
                break
    return bad


# --------------------------------------------------------------------------- #
def test_hand_cases():
    assert hand_case_failures(O.oracle_topk) == []


def test_decode_bf16_exhaustive_vs_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = O.decode_bf16(bits)
    theirs = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan_o, nan_t = np.isnan(ours), np.isnan(theirs)
    assert (nan_o == nan_t).all()
    assert nan_o.sum() == 2 * 127  # all-ones exponent, 127 non-zero mantissas, two signs
    assert (ours[~nan_o] == theirs[~nan_t]).all()
    # signed zeros decode with their sign
    assert np.signbit(ours[0x8000]) and not np.signbit(ours[0x0000])


def test_decode_f32_edges_vs_struct():
    rng = np.random.default_rng(5)
    edge = [0, 0x80000000, 1, 0x80000001, 0x007FFFFF, 0x00800000, 0x3F800000, 0xBF800000,
            0x7F7FFFFF, 0xFF7FFFFF, 0x7F800000, 0xFF800000]
    pats = np.array(edge + rng.integers(0, 2**32, size=20000, dtype=np.uint64).tolist(),
                    dtype=np.uint64).astype(np.uint32)
    ours = O.decode_f32(pats)
    for b, o in zip(pats.tolist(), ours.tolist()):
        ref = struct.unpack("<f", struct.pack("<I", b))[0]
        if ref != ref:
            assert o != o
        else:
            assert o == ref and (np.signbit(o) == np.signbit(ref))


def test_select_matches_brute_force():
    assert brute_force_failures(O.select_row) == []


def test_brute_force_closed_forms():
    n = 17
    asc = np.arange(n, dtype=np.float64)
    for k in range(1, n):
        assert O.brute_force_row(asc, k) == list(range(n - k, n))
        assert O.brute_force_row(asc[::-1].copy(), k) == list(range(k))
        assert O.brute_force_row(np.full(n, 2.5), k) == list(range(k))


def test_closed_forms_large():
    n, k = 200_000, 777
    asc = np.arange(n, dtype=np.float64)
    assert O.select_row(asc, k).tolist() == list(range(n - k, n))
    assert O.select_row(asc[::-1].copy(), k).tolist() == list(range(k))
    assert O.select_row(np.full(n, -0.0), k).tolist() == list(range(k))


# --------------------------------------------------------------------------- #
def check_invariants(w: W.Workload, res: O.OracleResult):
    lens = w.valid_lengths()
    for r in range(w.rows):
        n = int(lens[r])
        idx = res.indices[r].astype(np.int64)
        if res.status[r] == O.ROW_NAN:
            assert (idx == O.IDX_NAN).all()
            continue
        if n <= w.k:
            assert res.status[r] == O.ROW_SHORT
            assert idx[:n].tolist() == list(range(n)) and (idx[n:] == O.IDX_PAD).all()
            continue
        assert res.status[r] == O.ROW_SELECTED
        assert len(idx) == w.k and len(set(idx.tolist())) == w.k        # exactly k, unique
        assert idx.min() >= 0 and idx.max() < n                          # inside [0, end)
        assert (np.diff(idx) > 0).all()                                  # ascending index
        v = O.decode(w.x[r, :n], w.dtype)
        mask = np.zeros(n, bool)
        mask[idx] = True
        lo = v[mask].min()
        if (~mask).any():
            hi = v[~mask].max()
            assert lo >= hi                                              # selected >= unselected
            # tie rule: unselected entries equal to the boundary value sit after every
            # selected entry with that value
            tie_un = np.flatnonzero((~mask) & (v == lo))
            tie_sel = np.flatnonzero(mask & (v == lo))
            if len(tie_un):
                assert tie_un.min() > tie_sel.max()
        if res.values is not None:
            assert (res.values[r] == w.x[r, idx]).all()                  # original bits


SMALL_WORKLOADS = [
    lambda: W.pr1_duplicates(),
    lambda: W.indexer_drift(rows=4, n=8192, k=512),
    lambda: W.indexer_varlen(rows=64, stride=2048, k=512),
    lambda: W.sampler_logits(batch=2, k=50),
    lambda: W.sampler_logits(batch=1, k=4096),
    lambda: W.long_rows(2, 1 << 16, 1000, "uniform"),
    lambda: W.long_rows(2, 1 << 15, 4096, "desc"),
    lambda: W.long_rows(2, 1 << 15, 1000, "equal"),
    lambda: W.random_small(7, "bf16", 16, 512, 37, dist="ties", with_end=True),
    lambda: W.random_small(8, "f32", 16, 512, 100, dist="ties", with_end=True),
]


@pytest.mark.parametrize("make", SMALL_WORKLOADS)
def test_invariants(make):
    w = make()
    res = O.oracle_topk(w.x, w.dtype, w.k, end=w.end, sorted_index=1, return_value=1,
                        index_dtype=w.index_dtype, nan_mode="flag")
    check_invariants(w, res)


@pytest.mark.parametrize("make", SMALL_WORKLOADS[:6])
def test_values_match_torch_topk(make):
    """torch.topk (CPU) returns the same multiset of values, sorted descending."""
    w = make()
    res = O.oracle_topk(w.x, w.dtype, w.k, end=w.end, nan_mode="flag")
    lens = w.valid_lengths()
    for r in range(w.rows):
        n = int(lens[r])
        if n <= w.k:
            continue
        v = torch.from_numpy(O.decode(w.x[r, :n], w.dtype))
        ref = torch.topk(v, w.k, sorted=True).values.numpy()
        ours = -np.sort(-O.decode(res.values[r], w.dtype))
        assert (ours == ref).all()


def test_nan_rows_flagged_exactly():
    w = W.long_rows(6, 4096, 100, "uniform", inject_nan=True)
    res = O.oracle_topk(w.x, w.dtype, w.k, nan_mode="flag")
    assert np.flatnonzero(res.status == O.ROW_NAN).tolist() == w.nan_rows.tolist()
    assert not res.would_trap
    res_t = O.oracle_topk(w.x, w.dtype, w.k, nan_mode="trap")
    assert res_t.would_trap


def test_short_rows_skip_nan_check():
    w = W.random_small(3, "bf16", 8, 64, 64, dist="normal", nan_rows=np.arange(8))
    res = O.oracle_topk(w.x, w.dtype, w.k, nan_mode="trap")
    assert not res.would_trap and (res.status == O.ROW_SHORT).all()


def test_index_dtypes():
    w = W.pr1_duplicates()
    a = O.oracle_topk(w.x, w.dtype, w.k, index_dtype="i32")
    b = O.oracle_topk(w.x, w.dtype, w.k, index_dtype="i64")
    assert a.indices.dtype == np.int32 and b.indices.dtype == np.int64
    assert (a.indices == b.indices).all()


# --------------------------------------------------------------------------- #
# Mutation tests: one planted mistake at a time must be caught by a pin above.
# --------------------------------------------------------------------------- #
def _select_ties_largest_index(v, k):
    n = v.shape[0]
    t = np.partition(v, n - k)[n - k]
    above = np.flatnonzero(v > t)
    need = k - above.shape[0]
    tied = np.flatnonzero(v == t)[-need:]
    return np.sort(np.concatenate([above, tied]))


def _select_wrong_end(v, k):
    # partitions from the wrong end (k-th smallest instead of k-th largest)
    t = np.partition(v, k)[k]
    above = np.flatnonzero(v > t)[:k]
    tied = np.flatnonzero(v == t)[: max(k - above.shape[0], 0)]
    return np.sort(np.concatenate([above, tied]))


def _select_by_bits(v, k):
    # orders -0.0 below +0.0 (compares sign bits instead of values)
    key = np.where(np.signbit(v) & (v == 0), -1e-300, v)
    return O.select_row(key, k)


@pytest.mark.parametrize("mutant", [_select_ties_largest_index, _select_wrong_end, _select_by_bits])
def test_mutant_selection_is_caught(monkeypatch, mutant):
    caught = bool(brute_force_failures(mutant, trials=200))
    monkeypatch.setattr(O, "select_row", mutant)
    caught = caught or bool(hand_case_failures(O.oracle_topk))
    assert caught


def test_mutant_decode_is_caught():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):     # the shifted patterns include NaNs
        wrong = (bits.astype(np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)
    theirs = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    ok = np.isnan(theirs)
    assert not (wrong[~ok] == theirs[~ok]).all()


def test_mutant_short_rule_is_caught(monkeypatch):
    real = O.oracle_topk

    def strict_short(x_bits, dtype, k, **kw):
        # treats n == k as a normal row (should be a short row)
        kw2 = dict(kw)
        res = real(x_bits, dtype, k, **kw2)
        end = kw.get("end")
        n = x_bits.shape[1] if end is None else int(end[0])
        if n == k and res.status[0] == O.ROW_SHORT:
            res.status[0] = O.ROW_SELECTED
        return res

    assert hand_case_failures(strict_short)


def _rows_ignore_end(real):
    return lambda x_bits, dtype, k, **kw: real(x_bits, dtype, k, **{**kw, "end": None})


def _bad_end_clamped_in_flag_mode(real):
    def f(x_bits, dtype, k, **kw):
        end = kw.get("end")
        if end is not None:
            kw = {**kw, "end": np.clip(np.asarray(end), 0, x_bits.shape[1])}
        return real(x_bits, dtype, k, **kw)
    return f


def _padding_zero(real):
    def f(x_bits, dtype, k, **kw):
        res = real(x_bits, dtype, k, **kw)
        res.indices[res.indices == O.IDX_PAD] = 0
        return res
    return f


def _end_one_past(real):
    # reads one entry past the valid range (end + 1, where that stays inside the row)
    def f(x_bits, dtype, k, **kw):
        end = kw.get("end")
        if end is not None:
            end = np.asarray(end)
            kw = {**kw, "end": np.where((end >= 0) & (end < x_bits.shape[1]), end + 1, end)}
        return real(x_bits, dtype, k, **kw)
    return f


@pytest.mark.parametrize("mutant", [_rows_ignore_end, _bad_end_clamped_in_flag_mode, _padding_zero, _end_one_past])
def test_mutant_row_rule_is_caught(mutant):
    assert not hand_case_failures(O.oracle_topk)
    assert hand_case_failures(mutant(O.oracle_topk))


def nan_flag_failures(oracle_fn):
    w = W.long_rows(6, 2048, 10, "uniform", inject_nan=True)
    res = oracle_fn(w.x, w.dtype, w.k, nan_mode="flag")
    return np.flatnonzero(res.status == O.ROW_NAN).tolist() != w.nan_rows.tolist()


def test_mutant_nan_ignored_is_caught(monkeypatch):
    assert not nan_flag_failures(O.oracle_topk)
    real_decode = O.decode
    monkeypatch.setattr(O, "decode", lambda b, d: np.nan_to_num(real_decode(b, d)))
    assert nan_flag_failures(O.oracle_topk)


# --------------------------------------------------------------------------- #
# value order (sorted_index = 2) and its reading for short rows with NaN
# --------------------------------------------------------------------------- #
def test_value_order_matches_a_stable_library_sort():
    """NaN-free rows: value descending, ties by index, is numpy's stable sort of -v
    (a library routine); -0.0 and +0.0 compare equal there too."""
    rng = np.random.default_rng(21)
    pool = np.array([-np.inf, -2.0, -0.0, 0.0, 0.5, 3.0, np.inf], dtype=np.float32)
    for t in range(200):
        n = int(rng.integers(1, 60))
        f = pool[rng.integers(0, len(pool), size=n)] if t % 2 else rng.standard_normal(n).astype(np.float32)
        idx = np.sort(rng.choice(1000, size=n, replace=False))
        got = O.value_order(f.view(np.uint32), idx, "f32")
        want = np.argsort(-f.astype(np.float64), kind="stable")
        assert got.tolist() == want.tolist()


def test_value_order_hand_case_with_nan():
    """A worked case: +NaN payloads rank above +inf (larger payload first), -NaN
    payloads below -inf (larger payload last), -0.0 == +0.0 tied by index."""
    f = np.array([1.0, -0.0, 0.0, np.inf, -np.inf, 2.0, 1.0], dtype=np.float32)
    b = np.concatenate([f.view(np.uint32), np.array([0x7FC00000, 0x7FC00001, 0xFFC00000, 0xFFC00001],
                                                    dtype=np.uint32)])
    assert O.value_order(b, np.arange(11), "f32").tolist() == [8, 7, 3, 5, 0, 6, 1, 2, 4, 9, 10]
    # the index breaks ties, whatever the positions
    assert O.value_order(b[[6, 0]], np.array([3, 9]), "f32").tolist() == [0, 1]
    assert O.value_order(b[[6, 0]], np.array([9, 3]), "f32").tolist() == [1, 0]
