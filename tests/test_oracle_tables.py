"""Pins for the oracle's table design (T1-T5).

Each check is against something other than the oracle's own formula: Max's
1960 table, numerical integration of the Gaussian (scipy.integrate.quad), the
Gaussian CDF from scipy.stats, the defining optimality conditions of
Lloyd-Max and ECSQ quantisers, and the numbers the D-Quant pages state.
"""
import math
import os

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows.setdefault(int(parts[0]), {})[parts[1]] = [float(v) for v in parts[2:]]
    return rows


def _page_facts():
    facts = {}
    with open(os.path.join(GOLDEN, "page_facts.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split()[:2]
                facts[k] = float(v)
    return facts


@pytest.mark.parametrize("n", [4, 6, 8])
def test_lloyd_max_matches_max_1960(n):
    g = _read_golden("lloyd_max_gaussian.txt")[n]
    y, t, p = o.lloyd_max(n)
    half_y = y[n // 2:]
    half_t = t[n // 2 - 1:]
    np.testing.assert_allclose(half_y, g["levels"], atol=1e-3)
    np.testing.assert_allclose(half_t, g["thresholds"], atol=1e-3)
    mse = 1.0 - float(np.sum(p * y * y))
    assert abs(mse - g["mse"][0]) < 2e-4
    assert abs(o.load().dqo_entropy(n, p.ctypes.data_as(o.C.c_void_p)) - g["entropy"][0]) < 2e-3


def _cells_scipy(t):
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    p = stats.norm.cdf(edges[1:]) - stats.norm.cdf(edges[:-1])
    # tail-accurate for upper cells
    up = edges[:-1] >= 0
    p[up] = stats.norm.sf(edges[:-1][up]) - stats.norm.sf(edges[1:][up])
    return p


def _centroid_quad(a, b):
    num = integrate.quad(lambda u: u * stats.norm.pdf(u), a, b, epsabs=1e-14, epsrel=1e-13, limit=200)[0]
    den = integrate.quad(lambda u: stats.norm.pdf(u), a, b, epsabs=1e-16, epsrel=1e-13, limit=200)[0]
    return num / den


@pytest.mark.parametrize("n", [4, 6, 8])
def test_lloyd_max_optimality_conditions(n):
    y, t, p = o.lloyd_max(n)
    np.testing.assert_allclose(t, 0.5 * (y[:-1] + y[1:]), atol=1e-12)
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    for i in range(n):
        assert abs(_centroid_quad(edges[i], edges[i + 1]) - y[i]) < 1e-9


BUDGETS = [(8, 36), (6, 36), (8, 31), (6, 31), (8, 48), (6, 48)]


@pytest.mark.parametrize("n,cb", BUDGETS)
def test_stream_design_conditions(n, cb):
    st = o.Stream(n, cb)
    r = (8 * (cb - 2) - 24) / 128
    assert st.rate == pytest.approx(r, abs=0)
    # levels and thresholds strictly increasing, odd-symmetric, middle t = 0
    assert np.all(np.diff(st.y) > 0) and np.all(np.diff(st.t) > 0)
    np.testing.assert_allclose(st.y, -st.y[::-1], atol=1e-15)
    assert st.t[n // 2 - 1] == 0.0
    # cell probabilities from scipy's CDF; entropy meets the rate
    p = _cells_scipy(st.t)
    np.testing.assert_allclose(p, st.p, rtol=1e-9, atol=1e-15)
    H = -np.sum(p * np.log2(p))
    if st.is_lloyd_max:
        assert H <= r
    else:
        assert abs(H - r) < 1e-9
    # centroid condition by numerical integration
    edges = np.concatenate([[-np.inf], st.t, [np.inf]])
    for i in range(n):
        assert abs(_centroid_quad(edges[i], edges[i + 1]) - st.y[i]) < 1e-9
    # decision boundaries: neighbouring Lagrangian costs are equal at t_i
    l = -np.log2(p)
    for i in range(n - 1):
        ci = (st.t[i] - st.y[i]) ** 2 + st.lam * l[i]
        cj = (st.t[i] - st.y[i + 1]) ** 2 + st.lam * l[i + 1]
        assert abs(ci - cj) < 1e-9
    # mse: E[(u - y_q)^2] by integration
    mse = sum(integrate.quad(lambda u, yy=st.y[i]: (u - yy) ** 2 * stats.norm.pdf(u),
                             edges[i], edges[i + 1], limit=200)[0] for i in range(n))
    assert abs(mse - st.mse) < 1e-9


def test_design_choice_per_budget():
    # 2.26 bit -> 36 B; both streams are entropy-constrained there (the
    # Lloyd-Max designs need 2.82 / 2.44 bits/value, above the 1.94 left)
    k, v = o.Stream(8, 36), o.Stream(6, 36)
    assert not k.is_lloyd_max and not v.is_lloyd_max
    assert k.lam > 0 and v.lam > 0
    # 3.0 bit -> 48 B: the 6-level Lloyd-Max fits (2.44 <= 2.6875)
    assert o.Stream(6, 48).is_lloyd_max
    assert not o.Stream(8, 48).is_lloyd_max
    # lambda = 0 reproduces Lloyd-Max exactly
    y, t, p = o.lloyd_max(8)
    res = o.ecsq(8, 0.0, y)
    np.testing.assert_allclose(res[0], y, atol=1e-12)
    # entropy decreases as lambda grows
    hs = [-np.sum(o.ecsq(8, lam, y)[2] * np.log2(o.ecsq(8, lam, y)[2])) for lam in (0.0, 0.05, 0.1, 0.15)]
    assert all(a > b for a, b in zip(hs, hs[1:]))


@pytest.mark.parametrize("n,cb", BUDGETS)
def test_integer_frequencies(n, cb):
    st = o.Stream(n, cb)
    f = st.freq.astype(np.int64)
    assert f.sum() == 4096 and f.min() >= 1
    np.testing.assert_array_equal(f, f[::-1])
    np.testing.assert_array_equal(st.cum, np.concatenate([[0], np.cumsum(f)]))
    quota = 4096 * st.p
    # quota property of largest-remainder apportionment (floor at 1)
    for fi, qi in zip(f, quota):
        if qi >= 1:
            assert abs(fi - qi) < 1.0
        else:
            assert fi == 1
    # cross-entropy of the integer model within 0.5% of H(p) (+ the cost of
    # the floor-at-1 cells, which the ideal model gives < 1/4096)
    ce = -np.sum(st.p * np.log2(f / 4096.0))
    assert ce <= st.entropy * 1.005 + 1e-3
    # costs are fp32(12 - log2 f)
    np.testing.assert_allclose(2.0 ** (12.0 - st.cost.astype(np.float64)), f, rtol=1e-6)


def test_page_numbers():
    facts = _page_facts()
    # 2.26 bits/value -> 36-byte container for 128 values (36*8/128 = 2.25)
    assert o.container_bytes(facts["budget_bits_per_value"]) == 36
    assert o.container_bytes(facts["low_budget_bits_per_value"]) == 31
    assert o.container_bytes(3.0) == 48
    # "roughly 7x" less KV memory than BF16
    assert round(facts["bf16_bits"] / facts["budget_bits_per_value"]) == facts["kv_memory_saving"]
    # 8 levels for keys, 6 for values, at that budget
    tab = o.Tables(8, k_levels=int(facts["key_levels"]), v_levels=int(facts["value_levels"]))
    assert tab.k.n == 8 and tab.v.n == 6
    assert tab.k.container_bytes == 36 and tab.v.container_bytes == 36


def test_infeasible_budget_rejected():
    with pytest.raises(ValueError):
        o.Stream(8, 12)  # not even the all-innermost fallback fits
    with pytest.raises(ValueError):
        o.Stream(7, 36)  # odd level counts are not symmetric


def test_entropy_coding_beats_fixed_width_at_same_bytes():
    # [news] "Why Fixed Width Is a Ceiling": at the same storage, entropy
    # coding fits more levels and less distortion than fixed width. 36 B of
    # container holds 2 bits/value fixed width (4 Lloyd-Max levels) plus the
    # norm; the 8-level entropy-constrained design has lower MSE.
    y4, t4, p4 = o.lloyd_max(4)
    mse4 = 1.0 - np.sum(p4 * y4 * y4)
    assert o.Stream(8, 36).mse < mse4
    assert o.Stream(6, 36).mse < mse4
    assert math.isclose(mse4, 0.1175, abs_tol=2e-4)
