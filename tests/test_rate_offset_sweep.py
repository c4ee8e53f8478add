"""The drift-against-distortion sweep of oracle/rate_offset_sweep.py (CPU).

Pins: the design entropy equals the container's target rate plus the offset
(the tables solve H(p) = r + offset whenever the Lloyd-Max design is above
it); drift grows monotonically with the offset (finer levels overflow more
containers); offset 0 reproduces the default tables' drift; and around the
pages' key drift rate (0.75 % of symbols, at about +0.05 bit/value here) the
rotated coordinates' mean squared error is lower than at offset 0.
"""
import pytest

from oracle import oracle as o
from oracle import rate_offset_sweep as rs


@pytest.fixture(scope="module")
def res():
    return rs.sweep(rows=6, tokens=256, offsets=(-0.1, 0.0, 0.05, 0.1, 0.2))


def test_entropy_is_rate_plus_offset(res):
    base = (8 * (36 - 2) - 24) / 128.0  # the 36-byte container's target rate
    for r in res:
        for s in ("k", "v"):
            d = r[s]
            assert abs(d["rate"] - (base + r["offset"])) < 1e-12
            if d["lam"] > 0:  # entropy-constrained design: H = r + offset
                assert abs(d["entropy"] - d["rate"]) < 1e-6
            else:            # Lloyd-Max already below the target
                assert d["entropy"] <= d["rate"] + 1e-9


def test_drift_grows_with_offset(res):
    for s in ("k", "v"):
        rates = [r[s]["drift_syms"] for r in res]
        assert all(a <= b for a, b in zip(rates, rates[1:])), rates
        assert rates[-1] > 10 * max(rates[1], 1e-4)


def test_offset_zero_is_the_default_design(res):
    default = o.Tables(8)
    r0 = [r for r in res if r["offset"] == 0.0][0]
    assert abs(r0["k"]["entropy"] - default.k.entropy) < 1e-12
    assert abs(r0["v"]["entropy"] - default.v.entropy) < 1e-12


def test_small_positive_offset_lowers_mse(res):
    by = {r["offset"]: r for r in res}
    for s in ("k", "v"):
        assert by[0.05][s]["mse_u"] < by[0.0][s]["mse_u"]
        assert by[0.05][s]["drift_syms"] > by[0.0][s]["drift_syms"]
