"""Parity at the benchmark's full sizes, in the launch configuration bench.py
times.

The whole batch is prefilled through dq_append_kv (context tokens 0..T-2),
then one decode step appends token T-1 for every sequence and runs
dq_decode_attention over the T tokens with the whole batch, as bench.py does.
For a few sampled sequences the oracle encodes the same seeded K/V: their
containers must be bit-identical and their attention rows (all query heads)
within max-abs 2e-3 x RMS of the oracle's fp64 attention. The serving shape
(128 x 8K), the Qwen3-8B-shaped decode step (16 x 8K), the long context
(4 x 128K) and all three budgets of the 32 x 32K sweep are covered.
"""
import numpy as np
import pytest
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from oracle import oracle as o
from tests import _common as cm

pytestmark = pytest.mark.gpu

FULL_CASES = [
    ("serve_b128_t8k", [0, 77, 127]),
    ("qwen3_8b_b16_t8k", [3, 15]),
    ("long_b4_t128k", [2]),
    ("llama_b32_t32k_1p96", [5]),
    ("llama_b32_t32k_2p26", [17]),
    ("llama_b32_t32k_3p0", [30]),
]


def _oracle_rows(w, ref_t, b, T):
    """K, V float32 [1, Hkv, T, 128] of sequence b: the prefilled context
    (T-1 tokens) then the token of decode step 0."""
    K = np.empty((1, w.Hkv, T, 128), np.float32)
    V = np.empty_like(K)
    for h in range(w.Hkv):
        K[0, h, :T - 1] = synth.kv_row(w, "k", b, h, n=T - 1)
        V[0, h, :T - 1] = synth.kv_row(w, "v", b, h, n=T - 1)
        K[0, h, T - 1] = synth.kv_row(w, "k", b, h, n=1, step=0)[0]
        V[0, h, T - 1] = synth.kv_row(w, "v", b, h, n=1, step=0)[0]
    return K, V


@pytest.mark.parametrize("wname,sample", FULL_CASES)
def test_fullsize_step_matches_oracle_on_sampled_sequences(wname, sample):
    w = synth.WORKLOADS[wname]
    T = w.T
    tab = dq.dq_build_tables(n_kv_heads=w.Hkv, k_bits_per_value=w.k_bits, v_bits_per_value=w.v_bits)
    ck, cv = tab.k.container_bytes, tab.v.container_bytes
    T_cap = (T + 31) // 32 * 32
    kc = dq.new_cache(w.B, w.Hkv, T_cap, ck)
    vc = dq.new_cache(w.B, w.Hkv, T_cap, cv)
    stats = dq.new_stats()
    synth.prefill_cache(tab, w, kc, vc, T - 1, stats=stats, threads=16)

    rows = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    k_new = torch.from_numpy(synth.kv_block(w, "k", rows, n=1, step=0, threads=16)).to(
        "cuda", w.torch_dtype).view(w.B, w.Hkv, 1, 128)
    v_new = torch.from_numpy(synth.kv_block(w, "v", rows, n=1, step=0, threads=16)).to(
        "cuda", w.torch_dtype).view(w.B, w.Hkv, 1, 128)
    start = torch.full((w.B,), T - 1, dtype=torch.int32, device="cuda")
    dq.dq_append_kv(tab, k_new, v_new, start, kc, vc, stats=stats)
    q = synth.q_block(w, step=0)
    qt = torch.from_numpy(q).to("cuda", w.torch_dtype)
    seq = torch.full((w.B,), T, dtype=torch.int32, device="cuda")
    ws = torch.empty(dq.dq_decode_workspace_bytes(tab, w.B, w.Hq, w.Hkv, T), dtype=torch.uint8, device="cuda")
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device="cuda")
    dq.dq_decode_attention(tab, qt, kc, vc, seq, T, out, ws, stats=stats)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    s = dq.stats_dict(stats)
    assert s["integrity_errors"] == 0 and s["nonfinite_inputs"] == 0 and s["dropped_writes"] == 0

    ref_t = o.Tables(w.Hkv, k_container_bytes=ck, v_container_bytes=cv)
    for b in sample:
        K, V = _oracle_rows(w, ref_t, b, T)
        rk, rv, _, _, _, _ = o.encode_cache(ref_t, K, V)
        np.testing.assert_array_equal(dq.containers_of(kc[b:b + 1])[:, :, :T].cpu().numpy(), rk)
        np.testing.assert_array_equal(dq.containers_of(vc[b:b + 1])[:, :, :T].cpu().numpy(), rv)
        ref = o.attention_fp64(ref_t, q[b:b + 1], rk, rv, [T])
        cm.assert_attention_close(got[b:b + 1], ref, what="%s b=%d" % (wname, b))
