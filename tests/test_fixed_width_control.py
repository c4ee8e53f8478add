"""The fixed-width control of oracle/fixed_width_control.py (CPU).

Pins: the control's quantiser is the Gaussian Lloyd-Max quantiser of Max
(1960) with the D-Quant tie rule (a value on a threshold goes up); the
reconstruction is the exact inverse of the rotation when the levels equal the
rotated coordinates; and on a small sample the measured distortions order as
rate-distortion theory says (more bits, less error; entropy coding at 36
bytes below the 4-level fixed-width code at 34 bytes on both streams; the
rate-distortion fill of drift mode 1 never raises the error and lowers it at
2.26 bits).
"""
import numpy as np
import pytest

from oracle import fixed_width_control as fw
from oracle import oracle as o


def test_control_quantiser_is_max_1960_with_ties_up():
    syms, y = fw.fixed_width_codes(np.array([-2.0, -0.9816, -0.5, 0.0, 0.5, 0.9815, 2.0], np.float32), 2)
    _, t, _ = o.lloyd_max(4)
    assert np.allclose(np.abs(y), [1.510, 0.4528, 0.4528, 1.510], atol=1e-3)
    assert np.allclose(t, [-0.9816, 0.0, 0.9816], atol=1e-3)
    # thresholds at about -0.9816 / 0 / 0.9816; a value equal to a threshold goes up
    expect = np.searchsorted(t, np.array([-2.0, -0.9816, -0.5, 0.0, 0.5, 0.9815, 2.0]), side="right")
    np.testing.assert_array_equal(syms, expect)
    assert syms[3] == 2  # u = 0 sits on the middle threshold: upper cell


def test_reconstruct_inverts_the_rotation():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 128)).astype(np.float32)
    sg = o.signs(0, 1)[0]
    u, nh = fw.rotate_all(x, sg)
    xh = fw.reconstruct(u.astype(np.float64), nh, sg)
    # only the fp16 norm and the fp32 rotation round
    assert np.max(np.abs(xh - x) / np.linalg.norm(x, axis=1, keepdims=True)) < 2e-3


def test_distortion_orders_as_expected_on_a_small_sample():
    res = fw.measure(rows=4, tokens=64)
    mse = {(r["stream"], r["coder"].split()[0], round(r["bits"], 2), "RD fill" in r["coder"]): r["mse_u"]
           for r in res}
    for s in ("K", "V"):
        assert mse[(s, "D-Quant", 1.96, False)] > mse[(s, "D-Quant", 2.26, False)] > mse[(s, "D-Quant", 3.0, False)]
        fixed = [v for (st, c, _, _), v in mse.items() if st == s and c == "fixed"][0]
        assert mse[(s, "D-Quant", 2.26, False)] < fixed
        # the fill spends unused bytes on accuracy: never worse, better below 3 bits
        for b in (1.96, 2.26, 3.0):
            assert mse[(s, "D-Quant", b, True)] <= mse[(s, "D-Quant", b, False)]
        assert mse[(s, "D-Quant", 2.26, True)] < 0.99 * mse[(s, "D-Quant", 2.26, False)]
    for r in res:
        assert r["attn"] >= 0 and np.isfinite(r["attn"])


if __name__ == "__main__":
    pytest.main([__file__])
