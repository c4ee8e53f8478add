"""Pins for the oracle's encode steps E1-E4, E7 and dequantisation.

Checks use properties fixed by the mathematics: ||u||^2 = 128 after
normalisation, the stored norm equals ||x|| to fp16 rounding, the inverse
rotation recovers x exactly up to the fp16 norm, the symbol of a value is the
count of thresholds at or below it (numpy.searchsorted), and the measured
distortion over Gaussian data matches the design MSE.
"""
import numpy as np
import pytest

from oracle import oracle as o

F16_EPS = 2.0 ** -11


def _rng(seed=0):
    return np.random.default_rng(seed)


def test_rotate_normalize_unit_rms_and_norm():
    rng = _rng(0)
    sg = o.signs(5, 1)[0]
    for k in range(200):
        x = (rng.standard_normal(128) * np.exp(rng.normal(0, 1, 128))).astype(np.float32)
        u, nh, nf = o.rotate_normalize(x, sg)
        assert nf == 0
        assert abs(float(np.dot(u.astype(np.float64), u)) / 128.0 - 1.0) < 1e-5
        nrm = np.linalg.norm(x.astype(np.float64))
        got = o.f16_to_f64(np.array([nh]))[0]
        assert abs(got - nrm) <= nrm * (F16_EPS + 1e-6)


def test_inverse_rotation_recovers_input():
    # x = ||x|| * D H u / 128 exactly (H H = 128 I, D D = I, u = H D x sqrt(128)/||Hx||)
    rng = _rng(1)
    sg = o.signs(9, 1)[0]
    H = o.hadamard(128)
    for _ in range(50):
        x = rng.standard_normal(128).astype(np.float32) * 3
        u, nh, _ = o.rotate_normalize(x, sg)
        nrm = o.f16_to_f64(np.array([nh]))[0]
        xr = nrm * sg * (H @ u.astype(np.float64)) / 128.0
        assert np.max(np.abs(xr - x)) <= (F16_EPS + 1e-5) * np.linalg.norm(x) + 1e-6
    # and it matches the dequantiser when the levels are the values themselves
    st = o.Stream(8, 36)
    syms = np.zeros((1, 128), dtype=np.uint8)
    dq = o.dequantize(st, syms, np.array([0x3C00], dtype=np.uint16), sg)  # norm 1.0
    np.testing.assert_allclose(dq[0], sg * (H @ np.full(128, float(st.yf[0]))) / 128.0)


def test_zero_and_nonfinite_vectors():
    st = o.Stream(8, 36)
    sg = o.signs(0, 1)
    for x, flagged in ((np.zeros(128, np.float32), 0),
                       (np.full(128, np.nan, np.float32), 1),
                       (np.where(np.arange(128) == 7, np.inf, 1.0).astype(np.float32), 1),
                       (np.full(128, 3.0e38, np.float32), 1)):  # sum of squares overflows
        u, nh, nf = o.rotate_normalize(x, sg[0])
        assert nf == flagged and nh == 0 and not u.any()
        cont, syms, stats, bad = o.encode_vectors(st, sg, x[None], np.zeros(1, np.int32))
        assert bad == 0 and stats.nonfinite_inputs == flagged
        assert (syms == 4).all()  # u = 0 sits on the middle threshold: upper-inner level
        d, nh2, status = o.decode_containers(st, cont)
        assert status[0] == 0 and nh2[0] == 0 and (d == 4).all()


def test_quantize_counts_thresholds():
    rng = _rng(2)
    for n, cb in ((8, 36), (6, 36), (8, 31), (6, 48)):
        st = o.Stream(n, cb)
        u = (rng.standard_normal(50000) * 1.5).astype(np.float32)
        u[:len(st.tf)] = st.tf  # exact ties go to the upper cell
        np.testing.assert_array_equal(o.quantize(st, u), np.searchsorted(st.tf, u, side="right"))


def test_container_layout_and_round_trip():
    rng = _rng(3)
    tab = o.Tables(4)
    K = (rng.standard_normal((4, 64, 128)) * np.exp(rng.normal(0, 1, 128))).astype(np.float32)
    ho = np.repeat(np.arange(4, dtype=np.int32), 64)
    for st in (tab.k, tab.v):
        cont, syms, stats, bad = o.encode_vectors(st, tab.signs, K.reshape(-1, 128), ho)
        assert bad == 0 and cont.shape == (256, 36)
        d, nh, status = o.decode_containers(st, cont)
        assert not status.any()
        np.testing.assert_array_equal(d, syms)
        for v in range(256):
            u, n16, _ = o.rotate_normalize(K.reshape(-1, 128)[v], tab.signs[ho[v]])
            assert nh[v] == n16 == (int(cont[v, 0]) | (int(cont[v, 1]) << 8))
            x = int(cont[v, 2]) | (int(cont[v, 3]) << 8) | (int(cont[v, 4]) << 16)
            assert 65536 <= x < (1 << 24)


@pytest.mark.parametrize("n,cb", [(8, 36), (6, 36), (8, 48)])
def test_distortion_matches_design(n, cb):
    # Gaussian coordinates after rotation: the measured E[(u - y_q)^2] over
    # many vectors agrees with the design MSE from integration (drift adds a
    # little on top; the pages call it a sparse local correction).
    rng = _rng(4)
    st = o.Stream(n, cb)
    sg = o.signs(1, 1)
    X = rng.standard_normal((3000, 128)).astype(np.float32)
    cont, syms, stats, bad = o.encode_vectors(st, sg, X, np.zeros(3000, np.int32))
    err = []
    for v in range(0, 3000, 3):
        u, _, _ = o.rotate_normalize(X[v], sg[0])
        err.append(np.mean((u.astype(np.float64) - st.yf[syms[v]]) ** 2))
    assert abs(np.mean(err) - st.mse) < 0.05 * st.mse
