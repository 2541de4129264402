"""Pins for the sampling oracle (oracle/sample_oracle.py), checked against closed
forms and brute force rather than against itself.  CPU only."""
import math

import numpy as np
import pytest

import oracle.sample_oracle as S
from oracle.topk_oracle import IDX_BAD_END, IDX_NAN, IDX_PAD


def f32_bits(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


def test_greedy_and_tiny_top_p_pick_the_argmax():
    rng = np.random.default_rng(5)
    x = rng.normal(size=(6, 300)).astype(np.float32) * 3
    u = rng.random(6)
    for t, p in ((0.0, 0.9), (1.0, 1e-12)):
        res = S.oracle_sample(f32_bits(x), 40, t, p, u)
        # argmax, ties to the lower index
        want = [int(np.flatnonzero(row == row.max())[0]) for row in x]
        assert res.token.tolist() == want
        assert np.all(res.kept == 1) and np.allclose(res.prob, 1.0)


def test_all_equal_row_is_a_uniform_draw_over_the_lowest_indices():
    # top-k of an all-equal row is indices 0..k-1 (ties by index); weights all 1
    k = 50
    x = np.full((1, 1000), 0.25, dtype=np.float32)
    for u in (0.0, 0.013, 0.5, 0.999):
        res = S.oracle_sample(f32_bits(x), k, 0.7, 1.0, np.array([u]))
        assert res.token[0] == math.floor(u * k)
        assert res.prob[0] == pytest.approx(1.0 / k)


def test_two_candidates_closed_form():
    a, b, t = 2.0, 1.25, 0.5
    x = np.full((1, 64), -100.0, dtype=np.float32)
    x[0, 7], x[0, 3] = a, b
    p_first = 1.0 / (1.0 + math.exp((b - a) / t))
    for u, want in ((p_first - 1e-6, 7), (p_first + 1e-6, 3), (0.0, 7), (0.999999, 3)):
        res = S.oracle_sample(f32_bits(x), 2, t, 1.0, np.array([u]))
        assert res.token[0] == want
    res = S.oracle_sample(f32_bits(x), 2, t, 1.0, np.array([0.1]))
    assert res.prob[0] == pytest.approx(p_first, rel=1e-6)


def test_top_p_cut_worked_example():
    # probabilities 0.5, 0.3, 0.2 at temperature 1; top_p 0.75 keeps two, renormalised
    # to 0.625 / 0.375
    x = np.full((1, 32), -80.0, dtype=np.float32)
    x[0, 10], x[0, 20], x[0, 5] = math.log(0.5), math.log(0.3), math.log(0.2)
    for u, want in ((0.6, 10), (0.7, 20), (0.0, 10), (0.99, 20)):
        res = S.oracle_sample(f32_bits(x), 3, 1.0, 0.75, np.array([u]))
        assert res.kept[0] == 2
        assert res.token[0] == want
    res = S.oracle_sample(f32_bits(x), 3, 1.0, 0.75, np.array([0.9]))
    assert res.prob[0] == pytest.approx(0.375, rel=1e-6)
    # top_p just above 0.8 keeps the third candidate too
    res = S.oracle_sample(f32_bits(x), 3, 1.0, 0.81, np.array([0.95]))
    assert res.kept[0] == 3 and res.token[0] == 5


def test_draw_frequencies_match_the_probabilities():
    """Brute force over a fine grid of u: each candidate is drawn for a share of the
    grid equal to its renormalised probability."""
    z = np.array([3.0, 2.2, 2.2, 1.0, -0.5, -3.0])
    t, top_p = 0.8, 0.95
    e = np.exp((z - z[0]) / t)
    c = int(np.argmax(np.cumsum(e) >= top_p * e.sum())) + 1
    want = e[:c] / e[:c].sum()
    grid = (np.arange(200000) + 0.5) / 200000
    counts = np.zeros(len(z))
    for u in grid:
        pos, _, cc, _ = S.sample_row(z, t, top_p, u)
        assert cc == c
        counts[pos] += 1
    assert np.allclose(counts[:c] / len(grid), want, atol=1e-5)
    assert counts[c:].sum() == 0


def test_ties_are_ordered_by_index_and_high_temperature_flattens():
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, [9, 2, 14]] = 5.0            # three equal leaders: value order 2, 9, 14
    res = S.oracle_sample(f32_bits(x), 3, 1e6, 1.0, np.array([0.0]))
    assert res.order[0].tolist() == [2, 9, 14]
    assert res.token[0] == 2
    res = S.oracle_sample(f32_bits(x), 3, 1e6, 1.0, np.array([0.5]))
    assert res.token[0] == 9 and res.prob[0] == pytest.approx(1 / 3)


def test_row_rules():
    x = np.ones((4, 32), dtype=np.float32)
    x[1, 7] = np.nan
    end = np.array([32, 32, 40, 0], dtype=np.int32)   # row 2: invalid end; row 3: empty
    res = S.oracle_sample(f32_bits(x), 8, 1.0, 1.0, np.full(4, 0.3), end=end, nan_mode="flag")
    assert res.token[1] == IDX_NAN and res.token[2] == IDX_BAD_END and res.token[3] == IDX_PAD
    assert 0 <= res.token[0] < 8
    # a short row (n <= k) samples among its n entries
    xs = np.array([[1.0, -2.0, 3.0, 2.0] + [0.0] * 12], dtype=np.float32)
    res = S.oracle_sample(f32_bits(xs), 8, 0.0, 1.0, np.array([0.2]), end=np.array([4], dtype=np.int32))
    assert res.token[0] == 2 and res.kept[0] == 4   # greedy; top_p = 1 keeps all four
    # ... and the draw checks it for NaN, which TopK skips on short rows
    xs[0, 1] = np.nan
    res = S.oracle_sample(f32_bits(xs), 8, 1.0, 1.0, np.array([0.2]), end=np.array([4], dtype=np.int32))
    assert res.token[0] == IDX_NAN and not res.would_trap
    res = S.oracle_sample(f32_bits(xs), 8, 1.0, 1.0, np.array([0.2]), end=np.array([4], dtype=np.int32),
                          nan_mode="trap")
    assert res.would_trap


def test_token_is_always_in_the_top_k():
    rng = np.random.default_rng(11)
    x = (rng.normal(size=(20, 2000)) * 3).astype(np.float32)
    k = 64
    res = S.oracle_sample(f32_bits(x), k, 1.3, 0.9, rng.random(20))
    for r in range(20):
        top = set(np.argsort(-x[r], kind="stable")[:k].tolist())
        assert int(res.token[r]) in top
        assert 0 < res.prob[r] <= 1


def test_infinite_logits():
    # +inf leaders share all the mass; a row of -inf draws uniformly among them
    x = np.full((2, 16), -np.inf, dtype=np.float32)
    x[0, [4, 11]] = np.inf
    x[0, 2] = 7.0
    res = S.oracle_sample(f32_bits(x), 3, 1.0, 1.0, np.array([0.75, 0.7]))
    assert res.token[0] == 11 and res.prob[0] == pytest.approx(0.5)
    assert res.token[1] == 2 and res.prob[1] == pytest.approx(1 / 3)   # candidates 0, 1, 2


def test_top_p_reached_exactly_keeps_the_shortest_prefix():
    # an all-equal row of k = 50 candidates: weights all 1, E_c = c, E_m = 50; top_p = 0.5
    # is reached exactly at c = 25 (0.5 * 50 = 25, exact in binary), and top_p = 0.02 at c = 1
    x = np.full((1, 400), -1.5, dtype=np.float32)
    for top_p, c in ((0.5, 25), (0.02, 1), (0.5 + 1e-9, 26)):
        res = S.oracle_sample(f32_bits(x), 50, 1.0, top_p, np.array([0.999]))
        assert res.kept[0] == c
        assert res.token[0] == c - 1 and res.prob[0] == pytest.approx(1.0 / c)


# Mutants of the draw: each changes one step of the reading in a way a careless
# restatement could, and at least one pin above must fail on it.

def _mutant_temperature_multiplies(z, temperature, top_p, u):
    return _with_weights(z, top_p, u, lambda: np.where(z == z[0], 1.0, np.exp((z - z[0]) * temperature))
                         if temperature > 0 else _greedy(len(z)))


def _mutant_top_p_one_short(z, temperature, top_p, u):
    pos, p, c, pre = _REAL_SAMPLE_ROW(z, temperature, top_p, u)
    if c <= 1 or top_p >= 1.0:
        return pos, p, c, pre
    c -= 1
    target = u * pre[c - 1]
    pos = min(int(np.searchsorted(pre[:c], target, side="right")), c - 1)
    e = np.diff(np.concatenate([[0.0], pre]))
    return pos, float(e[pos] / pre[c - 1]), c, pre


def _mutant_top_p_strict(z, temperature, top_p, u):
    e = _weights(z, temperature)
    pre = np.cumsum(e)
    c = m = len(z)
    if top_p < 1.0:
        c = min(max(int(np.searchsorted(pre, top_p * pre[-1], side="right")) + 1, 1), m)
    pos = min(int(np.searchsorted(pre[:c], u * pre[c - 1], side="right")), c - 1)
    return pos, float(e[pos] / pre[c - 1]), c, pre


def _mutant_draw_at_or_above(z, temperature, top_p, u):
    pos, p, c, pre = _REAL_SAMPLE_ROW(z, temperature, top_p, u)
    e = np.diff(np.concatenate([[0.0], pre]))
    pos = min(int(np.searchsorted(pre[:c], u * pre[c - 1], side="left")), c - 1)
    return pos, float(e[pos] / pre[c - 1]), c, pre


def _mutant_probability_not_renormalised(z, temperature, top_p, u):
    pos, p, c, pre = _REAL_SAMPLE_ROW(z, temperature, top_p, u)
    return pos, p * pre[c - 1] / pre[-1], c, pre


def _mutant_leaders_not_forced_to_one(z, temperature, top_p, u):
    return _with_weights(z, top_p, u, lambda: np.exp((z - z[0]) / temperature) if temperature > 0
                         else _greedy(len(z)))


def _greedy(m):
    e = np.zeros(m)
    e[0] = 1.0
    return e


def _weights(z, temperature):
    if temperature <= 0.0:
        return _greedy(len(z))
    with np.errstate(invalid="ignore", over="ignore"):
        return np.where(z == z[0], 1.0, np.exp((z - z[0]) / temperature))


def _with_weights(z, top_p, u, make):
    with np.errstate(invalid="ignore", over="ignore"):
        e = make()
    pre = np.cumsum(e)
    c = m = len(z)
    if top_p < 1.0:
        c = min(max(int(np.searchsorted(pre, top_p * pre[-1], side="left")) + 1, 1), m)
    pos = min(int(np.searchsorted(pre[:c], u * pre[c - 1], side="right")), c - 1)
    return pos, float(e[pos] / pre[c - 1]), c, pre


_REAL_SAMPLE_ROW = S.sample_row
_PINS = [test_greedy_and_tiny_top_p_pick_the_argmax, test_all_equal_row_is_a_uniform_draw_over_the_lowest_indices,
         test_two_candidates_closed_form, test_top_p_cut_worked_example, test_ties_are_ordered_by_index_and_high_temperature_flattens,
         test_row_rules, test_token_is_always_in_the_top_k, test_infinite_logits,
         test_top_p_reached_exactly_keeps_the_shortest_prefix]


def _pins_fail():
    for pin in _PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


def test_the_mutants_stand_apart_from_the_oracle():
    # each mutant really differs from the oracle somewhere, so catching it means something
    z = np.array([np.inf, 2.0, 2.0, 1.0, 0.5, -1.0, -1.0, -4.0])
    zf = np.array([3.0, 2.0, 2.0, 1.0, 0.5, -1.0, -1.0, -4.0])
    for mutant in _MUTANTS:
        differs = False
        for zz in (z, zf, np.zeros(50)):
            for t in (0.5, 1.0, 2.0):
                for tp in (0.3, 0.5, 0.9, 1.0):
                    for u in (0.0, 0.25, 0.5, 0.77, 0.999):
                        with np.errstate(all="ignore"):
                            a = _REAL_SAMPLE_ROW(zz, t, tp, u)
                            b = mutant(zz, t, tp, u)
                        if a[0] != b[0] or a[2] != b[2] or not (a[1] == b[1] or (np.isnan(a[1]) and np.isnan(b[1]))):
                            differs = True
        assert differs, mutant.__name__


_MUTANTS = [_mutant_temperature_multiplies, _mutant_top_p_one_short, _mutant_top_p_strict,
            _mutant_draw_at_or_above, _mutant_probability_not_renormalised, _mutant_leaders_not_forced_to_one]


@pytest.mark.parametrize("mutant", _MUTANTS, ids=lambda f: f.__name__[len("_mutant_"):])
def test_sample_mutants_are_caught(monkeypatch, mutant):
    assert not _pins_fail()                     # the pins pass on the oracle itself
    monkeypatch.setattr(S, "sample_row", mutant)
    assert _pins_fail()
