"""CPU checks of the seeded synthetic inputs (shapes, determinism, recipe)."""
import numpy as np
import torch

from decode_attention_dq_b200 import synth


def test_rows_are_deterministic_and_independent():
    w = synth.WORKLOADS["qwen3_8b_b16_t8k"]
    a = synth.kv_row(w, "k", 3, 5, n=64)
    b = synth.kv_row(w, "k", 3, 5, n=64)
    c = synth.kv_row(w, "k", 3, 6, n=64)
    assert a.shape == (64, 128) and a.dtype == np.float32
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)
    # a longer draw starts with the same tokens (prefix-stable rows)
    np.testing.assert_array_equal(synth.kv_row(w, "v", 1, 2, n=100)[:64], synth.kv_row(w, "v", 1, 2, n=64))
    # step tokens differ from the context
    assert not np.array_equal(synth.kv_row(w, "k", 3, 5, n=1, step=0), a[:1])
    blk = synth.kv_block(w, "k", [(3, 5), (3, 6)], n=64, threads=2)
    np.testing.assert_array_equal(blk[0], a)
    np.testing.assert_array_equal(blk[1], c)


def test_values_are_exact_in_workload_dtype():
    w = synth.WORKLOADS["qwen3_8b_b16_t8k"]
    x = synth.kv_row(w, "k", 0, 0, n=32)
    np.testing.assert_array_equal(torch.from_numpy(x).to(torch.bfloat16).float().numpy(), x)
    q = synth.q_block(synth.scaled(w, B=2))
    assert q.shape == (2, 32, 128)
    np.testing.assert_array_equal(torch.from_numpy(q).to(torch.bfloat16).float().numpy(), q)
    t = synth.WORKLOADS["tiny_b1_t256"]
    assert synth.kv_row(t, "k", 0, 0).shape == (256, 128)


def test_recipe_statistics():
    w = synth.WORKLOADS["qwen3_8b_b16_t8k"]
    k = synth.kv_row(w, "k", 0, 0, n=8192).astype(np.float64)
    v = synth.kv_row(w, "v", 0, 0, n=8192).astype(np.float64)
    s = synth.channel_scales(w, "k", 0).astype(np.float64)
    # K: per-channel std ~ scale (plus the 0.2 shift), 4 outliers x10
    ratio = k.std(axis=0) / np.sqrt(s ** 2 + 0.04)
    assert np.all(np.abs(ratio - 1) < 0.1)
    assert (s > 10 * np.exp(-2.5)).sum() >= 4
    # per-token shift: the per-token mean over channels has std ~0.2
    assert abs((k - 0).mean(axis=1).std() - np.sqrt(0.04 + (s ** 2).sum() / 128 ** 2)) < 0.05
    # V ~ N(0, 1)
    assert abs(v.std() - 1.0) < 0.02 and abs(v.mean()) < 0.02
    t = synth.WORKLOADS["tiny_b1_t256"]
    st = synth.channel_scales(t, "k", 0)
    assert st.shape == (128,) and (st > 3).sum() >= 2
