"""The pass-based order of the rate-distortion fill equals the one-at-a-time
order (CPU, oracle only).

The GPU fills test several candidates per encode pass: from the next
untested candidate, each of the next W candidates is applied alone to the
current string. The first that fits is kept, the ones before it are
dropped, and the ones after it are tested again on the new string in the
next pass. W is 4 in the drift kernel's fill phase and 32 in the
warp-per-vector kernel. The argument that this gives the oracle's
one-at-a-time result (each candidate, in key order, kept if the string with
it and every earlier kept candidate fits): the keys and their order do not
change while candidates are kept, and a candidate dropped in a pass was
tested on exactly the string the one-at-a-time order tests it on (nothing
was kept between). This restates the pass-based order in numpy over the
oracle's exact coded lengths and checks it against oracle.rd_fill on random
strings at several budgets, for W = 1 (the one-at-a-time order itself), 4
and 32.
"""
import numpy as np
import pytest

from oracle import oracle as o


def _candidates(st, u, q0, qd):
    """(key, index, target) of the fill candidates in key order (ties to the
    lower index), fp32 as the fill rule states."""
    u = u.astype(np.float32)
    y = st.yf.astype(np.float32)
    cost = st.cost.astype(np.float32)
    err = (u[:, None] - y[None, :]) ** 2
    near = np.argmin(err, axis=1)
    out = []
    for i in range(len(u)):
        j, s = int(near[i]), int(qd[i])
        if j == s or abs(j - s) != 1 or abs(j - int(q0[i])) > 1:
            continue
        dd = np.float32(err[i, j] - err[i, s])
        dr = np.float32(cost[j] - cost[s])
        if dd < 0 and dr > 0:
            out.append((np.float32(dd / dr), i, j))
    out.sort(key=lambda c: (c[0], c[1]))
    return out


def _fill_in_passes(st, u, q0, qd, budget, width):
    base = qd.copy()
    queue = _candidates(st, u, q0, qd)
    kept = 0
    while queue:
        window = queue[:width]
        first = None
        for m, (_, i, j) in enumerate(window):
            trial = base.copy()
            trial[i] = j
            if o.rans_encode(st, trial)[0] <= budget:
                first = m
                break
        if first is None:
            queue = queue[width:]
        else:
            _, i, j = window[first]
            base[i] = j
            kept += 1
            queue = queue[first + 1:]
    return base, kept


@pytest.mark.parametrize("C", [31, 36, 48])
def test_pass_order_equals_one_at_a_time(C):
    rng = np.random.default_rng(C)
    tab = o.Tables(1, k_container_bytes=C, v_container_bytes=C)
    n_kept = 0
    for st in (tab.k, tab.v):
        for _ in range(40):
            u = (rng.standard_normal(128) * rng.choice([0.8, 1.0, 1.3])).astype(np.float32)
            q0 = o.quantize(st, u)
            ln, qd, _, _, fb = o.drift_fit(st, u, q0, st.payload_bytes)
            if fb:
                continue
            _, qf, ups = o.rd_fill(st, u, q0, qd, st.payload_bytes)
            for width in (1, 4, 32):
                got, kept = _fill_in_passes(st, u, q0, qd, st.payload_bytes, width)
                np.testing.assert_array_equal(got, qf)
                assert kept == ups
            n_kept += ups
    assert n_kept > 0


def test_pass_order_with_more_room():
    # A budget a few bytes above the container's keeps many candidates, so
    # passes keep one and re-test the rest many times.
    rng = np.random.default_rng(7)
    st = o.Tables(1).k
    for extra in (1, 3, 8):
        for _ in range(15):
            u = rng.standard_normal(128).astype(np.float32)
            q0 = o.quantize(st, u)
            ln, qd, _, _, fb = o.drift_fit(st, u, q0, st.payload_bytes)
            _, qf, ups = o.rd_fill(st, u, q0, qd, st.payload_bytes + extra)
            for width in (4, 32):
                got, kept = _fill_in_passes(st, u, q0, qd, st.payload_bytes + extra, width)
                np.testing.assert_array_equal(got, qf)
                assert kept == ups
