"""Pins for the oracle's drift step (E6).

The page fixes two hard properties ([news] "Drift: Bending Variable Back to
Fixed"): a drifted symbol moves to a nearby lower-cost symbol, and no symbol
moves by more than one reconstruction level; the result fits the container.
The greedy ranking (least added squared error per bit saved, ties to the
lowest index) is a reading where the page is silent; it is pinned here against an
independent restatement that sorts every candidate move once and applies them
in order (the same rule, written as a sort rather than a repeated arg-min),
which checks the procedure and its tie order on small strings.
"""
import numpy as np
import pytest

from oracle import oracle as o


def _sorted_rule(st, u, q0, budget):
    n = len(q0)
    cands = []
    for i in range(n):
        s = int(q0[i])
        for j in (s - 1, s + 1):
            if 0 <= j < st.n and st.cost[j] < st.cost[s]:
                dn = np.float32(u[i]) - st.yf[j]
                d0 = np.float32(u[i]) - st.yf[s]
                key = np.float32(np.float32(dn * dn) - np.float32(d0 * d0)) / np.float32(st.cost[s] - st.cost[j])
                cands.append((float(np.float32(key)), i, j))
    cands.sort()
    q = q0.copy()
    moved = set()
    length, _ = o.rans_encode(st, q)
    for key, i, j in cands:
        if length <= budget:
            break
        if i in moved:
            continue
        q[i] = j
        moved.add(i)
        length, _ = o.rans_encode(st, q)
    return length, q, moved


@pytest.mark.parametrize("n_levels,n_syms", [(8, 8), (6, 8), (8, 16), (6, 12)])
def test_greedy_matches_sorted_restatement(n_levels, n_syms):
    st = o.Stream(n_levels, 36)
    rng = np.random.default_rng(n_levels * 31 + n_syms)
    checked = 0
    for trial in range(400):
        u = (rng.standard_normal(n_syms) * 1.8).astype(np.float32)
        if trial % 5 == 0:  # force exact key ties between equal values
            u[n_syms // 2:] = u[: n_syms - n_syms // 2]
        q0 = o.quantize(st, u)
        full, _ = o.rans_encode(st, q0)
        budget = full - int(rng.integers(1, 3))
        if budget < 3:
            continue
        ln, q, moved, moves, fb = o.drift_fit(st, u, q0, budget)
        rl, rq, rmoved = _sorted_rule(st, u, q0, budget)
        if fb:
            continue  # candidates ran out; covered by the fallback test
        assert ln == rl and ln <= budget
        np.testing.assert_array_equal(q, rq)
        assert set(np.nonzero(moved)[0]) == rmoved and moves == len(rmoved)
        checked += 1
    assert checked > 100


def test_drift_invariants_full_vectors():
    st = o.Stream(8, 36)
    rng = np.random.default_rng(11)
    total_moves = 0
    for trial in range(300):
        u = (rng.standard_normal(128) * (1.0 + 0.3 * (trial % 3))).astype(np.float32)
        q0 = o.quantize(st, u)
        full, _ = o.rans_encode(st, q0)
        budget = min(st.payload_bytes, full - 1)
        ln, q, moved, moves, fb = o.drift_fit(st, u, q0, budget)
        if fb:
            continue
        d = q.astype(int) - q0.astype(int)
        assert np.all(np.abs(d) <= 1)                      # at most one level
        assert np.all((d != 0) == moved)                   # only marked symbols moved
        assert np.all(st.cost[q[moved]] < st.cost[q0[moved]])  # each to a cheaper level
        assert ln <= budget
        total_moves += moves
    assert total_moves > 0


def test_fallback_when_candidates_run_out():
    st = o.Stream(8, 36)
    rng = np.random.default_rng(5)
    u = (rng.standard_normal(128) * 3).astype(np.float32)
    q0 = o.quantize(st, u)
    ln, q, moved, moves, fb = o.drift_fit(st, u, q0, 12)
    assert fb
    assert set(np.unique(q)) <= {3, 4}
    np.testing.assert_array_equal(q >= 4, q0 >= 4)  # keeps each symbol's side
    assert ln == o.rans_encode(st, q)[0]


def test_standard_budget_never_falls_back_on_gaussian_data():
    tab = o.Tables(2)
    rng = np.random.default_rng(6)
    X = rng.standard_normal((2000, 128)).astype(np.float32) * np.float32(2.0)
    for st in (tab.k, tab.v):
        cont, syms, stats, bad = o.encode_vectors(st, tab.signs, X, np.zeros(2000, np.int32))
        assert bad == 0 and stats.overflow_fallbacks == 0
        assert 0 < stats.syms_drifted < 0.01 * 2000 * 128
