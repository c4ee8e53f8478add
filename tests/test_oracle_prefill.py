"""Pins for the fp64 chunked-prefill attention oracle (CPU).

The oracle (attention_prefill_fp64) is compared with
  - PyTorch's fp64 scaled_dot_product_attention on the explicitly
    dequantised matrices with a boolean causal mask built from the query
    positions (a library routine, not the oracle's own arithmetic);
  - the already pinned decode-attention oracle: query token i of a chunk at
    position p is decode attention with seq_len = p + 1 (one row at a time);
  - closed forms: a query at position 0 sees token 0 only, so its output is
    that token's dequantised V exactly; positions outside [0, T_cap) give 0;
  - causality: changing the cache after position p leaves row p unchanged.
An off-by-one in the mask, a transposed head mapping or a wrong scale fails
one of these.
"""
import numpy as np
import torch

from oracle import oracle as o


def _case(seed=0, B=2, Hkv=2, G=2, T=96, n_q=7):
    rng = np.random.default_rng(seed)
    tab = o.Tables(Hkv)
    K = (rng.standard_normal((B, Hkv, T, 128)) * np.exp(rng.normal(0, 1, 128))).astype(np.float32)
    V = rng.standard_normal((B, Hkv, T, 128)).astype(np.float32)
    q = rng.standard_normal((B, n_q, Hkv * G, 128))
    kc, vc, _, _, _, _ = o.encode_cache(tab, K, V)
    return tab, q, kc, vc, K, V


def test_prefill_matches_torch_sdpa_with_causal_mask():
    tab, q, kc, vc, K, V = _case()
    B, n_q, Hq, _ = q.shape
    Hkv, T = kc.shape[1], kc.shape[2]
    G = Hq // Hkv
    q_start = [40, 89]
    out = o.attention_prefill_fp64(tab, q, kc, vc, q_start)
    for b in range(B):
        for h in range(Hkv):
            d, nh, _ = o.decode_containers(tab.k, kc[b, h])
            kh = o.dequantize(tab.k, d, nh, tab.signs[h])
            d, nh, _ = o.decode_containers(tab.v, vc[b, h])
            vh = o.dequantize(tab.v, d, nh, tab.signs[h])
            pos = q_start[b] + np.arange(n_q)
            mask = torch.from_numpy(np.arange(T)[None, :] <= pos[:, None])  # [n_q, T]
            qq = torch.from_numpy(np.ascontiguousarray(q[b, :, h * G:(h + 1) * G].transpose(1, 0, 2)))[None]
            kk = torch.from_numpy(kh)[None, None].expand(1, G, T, 128)
            vv = torch.from_numpy(vh)[None, None].expand(1, G, T, 128)
            ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask)[0].numpy()
            ok = pos < T
            got = out[b, :, h * G:(h + 1) * G].transpose(1, 0, 2)
            np.testing.assert_allclose(got[:, ok], ref[:, ok], rtol=1e-12, atol=1e-12)


def test_each_row_is_decode_attention_at_its_position():
    tab, q, kc, vc, K, V = _case(seed=1, B=2, Hkv=2, G=4, T=64, n_q=5)
    q_start = [0, 50]
    out = o.attention_prefill_fp64(tab, q, kc, vc, q_start)
    for i in range(q.shape[1]):
        seq = [q_start[b] + i + 1 for b in range(q.shape[0])]
        ref = o.attention_fp64(tab, q[:, i], kc, vc, seq)
        np.testing.assert_allclose(out[:, i], ref, rtol=1e-12, atol=1e-12)


def test_position_zero_sees_only_token_zero_and_out_of_range_is_zero():
    tab, q, kc, vc, K, V = _case(seed=2, B=3, Hkv=1, G=2, T=32, n_q=3)
    out = o.attention_prefill_fp64(tab, q, kc, vc, [0, 31, -2])
    d, nh, _ = o.decode_containers(tab.v, vc[0, 0, :1])
    v0 = o.dequantize(tab.v, d, nh, tab.signs[0])[0]
    for g in range(2):
        np.testing.assert_allclose(out[0, 0, g], v0, rtol=1e-13, atol=1e-15)
    # sequence 1: positions 31 (valid), 32 and 33 (past T_cap = 32)
    assert np.all(out[1, 1:] == 0.0) and np.any(out[1, 0] != 0.0)
    # sequence 2: positions -2, -1 (invalid), 0 (valid: token 0 only)
    assert np.all(out[2, :2] == 0.0)
    d, nh, _ = o.decode_containers(tab.v, vc[2, 0, :1])
    np.testing.assert_allclose(out[2, 2, 0], o.dequantize(tab.v, d, nh, tab.signs[0])[0], rtol=1e-13)


def test_later_tokens_do_not_change_earlier_rows():
    tab, q, kc, vc, K, V = _case(seed=3, B=1, Hkv=1, G=1, T=64, n_q=10)
    out = o.attention_prefill_fp64(tab, q, kc, vc, [20])
    K2, V2 = K.copy(), V.copy()
    K2[:, :, 25:] *= -3.0
    V2[:, :, 25:] += 1.0
    kc2, vc2, _, _, _, _ = o.encode_cache(tab, K2, V2)
    out2 = o.attention_prefill_fp64(tab, q, kc2, vc2, [20])
    np.testing.assert_array_equal(out[:, :5], out2[:, :5])  # positions 20..24
    assert not np.allclose(out[:, 5:], out2[:, 5:])
