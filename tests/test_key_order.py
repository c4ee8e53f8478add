"""The integer form of the drift and fill keys keeps the float order (CPU).

The GPU ranks move keys as unsigned integers: the float's bits with all
bits flipped when the sign bit is set, else with the sign bit set, after
-0 is made +0 (k + 0 in round-to-nearest). Two warp minimum reductions then
give the least key and the lowest index holding it. The drift rule orders
candidates by the fp32 key with ties to the lower index, and the float
order holds -0 and +0 equal. This restates the mapping in numpy and checks,
on random keys with many ties, both signed zeros, tiny and huge magnitudes
and +inf (no candidate), that ordering by (integer, index) equals ordering
by (float key, index), and that +inf maps above every finite key.
"""
import numpy as np


def order_bits(k):
    k = (np.asarray(k, dtype=np.float32) + np.float32(0.0)).astype(np.float32)  # -0 -> +0
    b = k.view(np.uint32)
    flip = np.where((b >> np.uint32(31)) != 0, np.uint32(0xFFFFFFFF), np.uint32(0x80000000))
    return b ^ flip


def test_integer_order_equals_float_order():
    rng = np.random.default_rng(0)
    for _ in range(200):
        n = 128
        pool = np.array([0.0, -0.0, 1e-38, -1e-38, 1e-45, -1e-45, 3.5, -3.5, 1e30, -1e30, np.inf],
                        dtype=np.float32)
        k = np.where(rng.random(n) < 0.5, rng.choice(pool, n),
                     (rng.standard_normal(n) * rng.choice([1e-3, 1.0, 1e3], n)).astype(np.float32))
        k = k.astype(np.float32)
        idx = np.arange(n)
        by_float = np.lexsort((idx, k))  # float order: -0 == +0
        ib = order_bits(k)
        by_int = np.lexsort((idx, ib))
        np.testing.assert_array_equal(by_int, by_float)


def test_signed_zeros_tie_and_inf_is_largest():
    assert order_bits(np.float32(-0.0)) == order_bits(np.float32(0.0))
    finite = np.array([-3.4e38, -1.0, -1e-45, 0.0, 1e-45, 1.0, 3.4e38], dtype=np.float32)
    inf_bits = order_bits(np.float32(np.inf))
    assert inf_bits == 0xFF800000
    assert np.all(order_bits(finite) < inf_bits)
    assert np.all(np.diff(order_bits(finite).astype(np.int64)) > 0)
