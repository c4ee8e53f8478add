"""Pins for the fp64 attention oracle.

The oracle's attention over the dequantised cache is compared with PyTorch's
fp64 scaled_dot_product_attention on the explicitly dequantised matrices, and
the rotated-domain identity the kernels use (score = scale * ||k|| * <H D q /
128, y_hat>) is checked against the explicit form to 1e-12.
"""
import math

import numpy as np
import torch

from oracle import oracle as o


def _small_case(seed=0, B=2, Hkv=2, G=2, T=40):
    rng = np.random.default_rng(seed)
    tab = o.Tables(Hkv)
    K = (rng.standard_normal((B, Hkv, T, 128)) * np.exp(rng.normal(0, 1, 128))).astype(np.float32)
    V = rng.standard_normal((B, Hkv, T, 128)).astype(np.float32)
    q = rng.standard_normal((B, Hkv * G, 128))
    kc, vc, ks, vs, _, _ = o.encode_cache(tab, K, V)
    return tab, q, kc, vc, ks, vs, K, V


def test_attention_matches_torch_sdpa():
    tab, q, kc, vc, ks, vs, K, V = _small_case()
    B, Hq, _ = q.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    seq = [40, 17]
    out = o.attention_fp64(tab, q, kc, vc, seq)
    for b in range(B):
        for h in range(Hkv):
            T = seq[b]
            d, nh, _ = o.decode_containers(tab.k, kc[b, h, :T])
            kh = o.dequantize(tab.k, d, nh, tab.signs[h])
            d, nh, _ = o.decode_containers(tab.v, vc[b, h, :T])
            vh = o.dequantize(tab.v, d, nh, tab.signs[h])
            qq = torch.from_numpy(q[b, h * G:(h + 1) * G])[None, :, None, :]
            kk = torch.from_numpy(kh)[None, None].expand(1, G, T, 128)
            vv = torch.from_numpy(vh)[None, None].expand(1, G, T, 128)
            ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[0, :, 0].numpy()
            np.testing.assert_allclose(out[b, h * G:(h + 1) * G], ref, rtol=1e-12, atol=1e-12)


def test_rotated_domain_identity():
    tab, q, kc, vc, ks, vs, K, V = _small_case(seed=1, B=1, Hkv=1, G=1, T=30)
    H = o.hadamard(128)
    d, nh, _ = o.decode_containers(tab.k, kc[0, 0])
    kh = o.dequantize(tab.k, d, nh, tab.signs[0])
    scale = 1.0 / math.sqrt(128)
    explicit = scale * kh @ q[0, 0]
    qt = H @ (tab.signs[0] * q[0, 0]) / 128.0
    rotated = scale * o.f16_to_f64(nh) * (tab.k.yf.astype(np.float64)[d] @ qt)
    np.testing.assert_allclose(rotated, explicit, rtol=1e-12, atol=1e-12)


def test_empty_and_single_token_sequences():
    tab, q, kc, vc, ks, vs, K, V = _small_case(seed=2, B=2, Hkv=1, G=1, T=8)
    out = o.attention_fp64(tab, q, kc, vc, [0, 1])
    assert np.all(out[0] == 0.0)
    d, nh, _ = o.decode_containers(tab.v, vc[1, 0, :1])
    np.testing.assert_allclose(out[1, 0], o.dequantize(tab.v, d, nh, tab.signs[0])[0], rtol=1e-14)


def test_dequantised_scores_track_exact_scores():
    # The whole lossy path against the unquantised keys: with Gaussian
    # coordinates the relative error of q.k over many keys is about
    # sqrt(design MSE) (the quantisation error is near-independent of the
    # level), and the correlation is about sqrt(1 - MSE). A sign, permutation
    # or scale mistake in rotation/dequantisation breaks both.
    rng = np.random.default_rng(3)
    tab = o.Tables(1)
    K = rng.standard_normal((1, 1, 4000, 128)).astype(np.float32)
    kc, vc, ks, vs, _, _ = o.encode_cache(tab, K, K)
    d, nh, _ = o.decode_containers(tab.k, kc[0, 0])
    kh = o.dequantize(tab.k, d, nh, tab.signs[0])
    q = rng.standard_normal(128)
    exact = K[0, 0].astype(np.float64) @ q
    approx = kh @ q
    rel = np.linalg.norm(approx - exact) / np.linalg.norm(exact)
    assert abs(rel - np.sqrt(tab.k.mse)) < 0.15 * np.sqrt(tab.k.mse)
    assert np.corrcoef(exact, approx)[0, 1] > np.sqrt(1 - tab.k.mse) - 0.02
