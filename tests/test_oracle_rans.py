"""Pins for the oracle's rANS coder.

Round trips on random strings (including frequency-1 symbols and constant
strings), the decoder's final state returning to L, the code length of a
long stream within 1% of the information-theoretic cross-entropy of the
integer model, and a 128-symbol string's pushed bits within [-8.5, +1] of
its ideal length.
"""
import numpy as np
import pytest

from oracle import oracle as o


@pytest.mark.parametrize("n,cb", [(8, 36), (6, 36), (8, 31), (6, 48)])
def test_round_trip_random_strings(n, cb):
    st = o.Stream(n, cb)
    rng = np.random.default_rng(n * 100 + cb)
    p = st.freq / 4096.0
    for trial in range(3000):
        ln = int(rng.integers(1, 300))
        mode = trial % 4
        if mode == 0:
            q = rng.choice(n, size=ln, p=p)
        elif mode == 1:
            q = rng.integers(0, n, ln)  # rare symbols often
        elif mode == 2:
            q = np.full(ln, rng.integers(0, n))  # constant strings
        else:
            q = np.where(rng.random(ln) < 0.5, 0, n - 1)  # only the freq-1 extremes
        q = q.astype(np.uint8)
        length, buf = o.rans_encode(st, q)
        assert buf is not None and len(buf) == length
        rc, dq, xf, used = o.rans_decode(st, buf, ln)
        assert rc == 0, (trial, rc)
        assert xf == 65536 and used == length
        np.testing.assert_array_equal(dq, q)


def test_empty_string_is_just_the_state():
    st = o.Stream(8, 36)
    length, buf = o.rans_encode(st, np.zeros(0, dtype=np.uint8))
    assert length == 3 and list(buf) == [0, 0, 1]  # x = L = 2^16, little-endian


def test_long_stream_length_matches_cross_entropy():
    st = o.Stream(8, 36)
    rng = np.random.default_rng(7)
    n = 1_000_000
    q = rng.choice(8, size=n, p=st.p).astype(np.uint8)
    length, buf = o.rans_encode(st, q, cap=n)
    ideal_bits = float(np.sum(12.0 - np.log2(st.freq[q].astype(np.float64))))
    assert abs(8.0 * length - ideal_bits) / ideal_bits < 0.01
    rc, dq, xf, used = o.rans_decode(st, buf, n)
    assert rc == 0 and np.array_equal(dq, q)


def test_decoder_flags_corruption():
    st = o.Stream(8, 36)
    rng = np.random.default_rng(3)
    q = rng.choice(8, size=128, p=st.p).astype(np.uint8)
    length, buf = o.rans_encode(st, q)
    # truncated stream: the decoder runs out of bytes
    rc, *_ = o.rans_decode(st, buf[:max(3, length - 2)], 128)
    assert rc == 2
    # a state below L is rejected up front
    bad = buf.copy(); bad[2] = 0
    rc, *_ = o.rans_decode(st, bad, 128)
    assert rc == 1
    # flipped payload bits: almost always a wrong final state or an overrun
    flagged = 0
    for k in range(200):
        b2 = buf.copy()
        pos = 3 + int(rng.integers(0, max(1, length - 3)))
        b2[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        rc, dq, xf, used = o.rans_decode(st, b2, 128)
        flagged += (rc != 0) or (not np.array_equal(dq, q))
    assert flagged == 200


@pytest.mark.parametrize("n,cb", [(8, 36), (6, 36), (8, 31), (6, 48)])
def test_pushed_bits_track_the_ideal_length(n, cb):
    # A 128-symbol string's pushed bytes carry its ideal length, the sum of
    # the symbols' costs -log2(f / 4096), less what stays in the final state
    # (up to 8 bits above the initial 2^16) and at most a fraction of a bit
    # more (the integer model's rounding). The decode-step append uses the
    # upper bound to rank moves before the first encode of a string that may
    # not fit; its result does not depend on it.
    st = o.Stream(n, cb)
    rng = np.random.default_rng(n * 1000 + cb)
    p = st.freq / 4096.0
    for trial in range(1500):
        mode = trial % 3
        if mode == 0:
            q = rng.choice(n, size=128, p=p)
        elif mode == 1:
            q = rng.integers(0, n, 128)  # rare symbols often
        else:
            q = np.where(rng.random(128) < 0.5, 0, n - 1)
        q = q.astype(np.uint8)
        length, _ = o.rans_encode(st, q)
        resid = (length - 3) * 8 - float(st.cost[q].astype(np.float64).sum())
        assert -8.5 <= resid <= 1.0, (trial, resid)
