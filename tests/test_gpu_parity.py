"""GPU parity: the CUDA path (through the C-ABI) against the CPU oracle.

Containers, symbols, norms and drift counters must be bit-identical; attention
must be within max-abs 2e-3 x RMS of the oracle's fp64 attention over the same
containers. Sizes span several 32-token tiles with ragged tails, warp ranges
that start and end inside a (sequence, head), every supported GQA group size
and both input dtypes.
"""
import numpy as np
import pytest
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from oracle import oracle as o
from tests import _common as cm

pytestmark = pytest.mark.gpu


def test_tables_and_signs_match_oracle():
    for kb, vb, seed in ((2.26, 2.26, 0), (1.96, 1.96, 7), (3.0, 2.26, 123)):
        lib = cm.lib_tables(8, kb, vb, seed)
        ref = cm.oracle_tables(8, kb, vb, seed)
        for ls, rs in ((lib.k, ref.k), (lib.v, ref.v)):
            assert ls.n_levels == rs.n and ls.container_bytes == rs.container_bytes
            assert ls.freq == [int(v) for v in rs.freq] and ls.cum == [int(v) for v in rs.cum]
            np.testing.assert_array_equal(np.float32(ls.levels), rs.yf)
            np.testing.assert_array_equal(np.float32(ls.thresholds), rs.tf)
            np.testing.assert_array_equal(np.float32(ls.cost), rs.cost)
        np.testing.assert_array_equal(lib.signs().numpy(), ref.signs)


def _decode_on_gpu(tab, kind, cont):
    c = torch.from_numpy(np.ascontiguousarray(cont)).cuda()
    n = cont.shape[0]
    syms = torch.empty((n, 128), dtype=torch.uint8, device="cuda")
    nh = torch.empty(n, dtype=torch.int16, device="cuda")
    status = torch.empty(n, dtype=torch.int32, device="cuda")
    stats = dq.new_stats()
    dq.dq_decode_symbols(tab, c, kind, syms, nh, status, stats)
    torch.cuda.synchronize()
    return (syms.cpu().numpy(), nh.cpu().numpy().view(np.uint16), status.cpu().numpy(),
            dq.stats_dict(stats))


@pytest.mark.parametrize("wname,T", [("tiny_b1_t256", 256), ("qwen3_8b_b16_t8k", 200)])
def test_decode_symbols_bit_exact(wname, T):
    w = synth.WORKLOADS[wname]
    w = synth.scaled(w, B=min(w.B, 2), T=T)
    K, V, _ = cm.inputs(w)
    ref = cm.oracle_tables(w.Hkv)
    lib = cm.lib_tables(w.Hkv)
    kc, vc, ks, vs, _, _ = o.encode_cache(ref, K, V)
    for kind, cont, syms in ((dq.DQ_STREAM_K, kc, ks), (dq.DQ_STREAM_V, vc, vs)):
        flat = cont.reshape(-1, cont.shape[-1])
        g_syms, g_nh, g_st, stats = _decode_on_gpu(lib, kind, flat)
        np.testing.assert_array_equal(g_syms, syms.reshape(-1, 128))
        np.testing.assert_array_equal(g_nh, flat[:, 0].astype(np.uint16) | (flat[:, 1].astype(np.uint16) << 8))
        assert not g_st.any() and stats["integrity_errors"] == 0


def test_decode_symbols_flags_corruption_like_oracle():
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=1, Hkv=1, Hq=4, T=600)
    K, V, _ = cm.inputs(w)
    ref = cm.oracle_tables(1)
    lib = cm.lib_tables(1)
    kc, vc, ks, vs, _, _ = o.encode_cache(ref, K, V)
    flat = kc.reshape(-1, kc.shape[-1]).copy()
    rng = np.random.default_rng(0)
    for i in range(flat.shape[0]):
        mode = i % 4
        if mode == 0:
            flat[i, rng.integers(5, flat.shape[1])] ^= np.uint8(1 << rng.integers(0, 8))
        elif mode == 1:
            flat[i, 4] = 0  # initial state below L
        elif mode == 2:
            flat[i, flat.shape[1] - 1] = 0xA5  # trailing byte: padding or payload
        # mode 3 left intact
    r_syms, r_nh, r_st = o.decode_containers(ref.k, flat)
    g_syms, g_nh, g_st, stats = _decode_on_gpu(lib, dq.DQ_STREAM_K, flat)
    np.testing.assert_array_equal(g_st, r_st)
    np.testing.assert_array_equal(g_nh, r_nh)
    np.testing.assert_array_equal(g_syms, r_syms)
    assert stats["integrity_errors"] == int((r_st != 0).sum()) > 0
    assert set(np.unique(r_st)) >= {0, 1, 3}


# Appends of up to ~38K vectors per stream run the warp-per-vector kernel on a
# 148-SM B200, larger ones the lane-per-vector kernel: both are covered, for
# fp32 (tiny) and bf16 inputs and every budget.
APPEND_CASES = [
    ("tiny_b1_t256", 256, 2.26, 2.26),
    ("qwen3_8b_b16_t8k", 300, 2.26, 2.26),
    ("llama_b32_t32k_1p96", 160, 1.96, 1.96),
    ("llama_b32_t32k_3p0", 160, 3.0, 3.0),
    ("tiny_b1_t256", 65536, 2.26, 2.26),
    ("qwen3_8b_b16_t8k", 4096, 2.26, 2.26),
    ("llama_b32_t32k_1p96", 4096, 1.96, 1.96),
    ("llama_b32_t32k_3p0", 4096, 3.0, 3.0),
    # asymmetric budgets (48-byte K, 31-byte V) and the largest container (64 bytes)
    ("qwen3_8b_b16_t8k", 300, 3.0, 1.96),
    ("qwen3_8b_b16_t8k", 4096, 1.96, 3.0),
    ("qwen3_8b_b16_t8k", 300, 4.0, 4.0),
]


@pytest.mark.parametrize("inline_drift", [False, True])
@pytest.mark.parametrize("wname,T,kb,vb", APPEND_CASES)
def test_append_bit_exact(wname, T, kb, vb, inline_drift):
    w = synth.WORKLOADS[wname]
    w = synth.scaled(w, B=min(w.B, 2), T=T)
    K, V, _ = cm.inputs(w)
    ref = cm.oracle_tables(w.Hkv, kb, vb)
    lib = cm.lib_tables(w.Hkv, kb, vb)
    rk, rv, _, _, kst, vst = o.encode_cache(ref, K, V)
    stats = dq.new_stats()
    # inline_drift: dq_append_kv without a workspace (drift inside the encode
    # kernel); otherwise large appends list their over-long containers for
    # the separate drift kernel.
    kc, vc = cm.gpu_append_all(lib, K, V, w.torch_dtype, stats=stats,
                               workspace=False if inline_drift else None)
    torch.cuda.synchronize()
    kf, vf = cm.flat(kc), cm.flat(vc)
    np.testing.assert_array_equal(kf[:, :, :T], rk)
    np.testing.assert_array_equal(vf[:, :, :T], rv)
    assert not kf[:, :, T:].any() and not vf[:, :, T:].any()
    s = dq.stats_dict(stats)
    assert s["k_syms_drifted"] == kst.syms_drifted and s["v_syms_drifted"] == vst.syms_drifted
    assert s["k_cont_drifted"] == kst.cont_drifted and s["v_cont_drifted"] == vst.cont_drifted
    assert s["overflow_fallbacks"] == kst.overflow_fallbacks + vst.overflow_fallbacks
    assert s["nonfinite_inputs"] == 0 and s["dropped_writes"] == 0


def test_append_incremental_positions_and_drops():
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=3, Hkv=2, Hq=8, T=80)
    K, V, _ = cm.inputs(w)
    ref = cm.oracle_tables(2)
    lib = cm.lib_tables(2)
    rk, rv, _, _, _, _ = o.encode_cache(ref, K, V)
    T_cap = 96
    kc = dq.new_cache(3, 2, T_cap, 36)
    vc = dq.new_cache(3, 2, T_cap, 36)
    stats = dq.new_stats()
    # three appends of 40, 1 and 39 tokens; sequence 2 starts 21 positions
    # late so its last 5 tokens fall past T_cap and are dropped.
    shift = np.array([0, 0, 21])
    done = 0
    for n in (40, 1, 39):
        kt = torch.from_numpy(K[:, :, done:done + n]).to("cuda", torch.bfloat16).contiguous()
        vt = torch.from_numpy(V[:, :, done:done + n]).to("cuda", torch.bfloat16).contiguous()
        start = torch.tensor(done + shift, dtype=torch.int32, device="cuda")
        dq.dq_append_kv(lib, kt, vt, start, kc, vc, stats=stats)
        done += n
    torch.cuda.synchronize()
    kn, vn = cm.flat(kc), cm.flat(vc)
    np.testing.assert_array_equal(kn[:2, :, :80], rk[:2])
    np.testing.assert_array_equal(vn[:2, :, :80], rv[:2])
    assert not kn[:2, :, 80:].any() and not vn[:2, :, 80:].any()
    np.testing.assert_array_equal(kn[2, :, 21:], rk[2, :, :75])
    np.testing.assert_array_equal(vn[2, :, 21:], rv[2, :, :75])
    assert not kn[2, :, :21].any() and not vn[2, :, :21].any()
    assert dq.stats_dict(stats)["dropped_writes"] == 2 * 2 * 5  # K and V, 2 heads, 5 tokens


def test_append_nonfinite_and_zero_vectors():
    w = synth.scaled(synth.WORKLOADS["tiny_b1_t256"], T=64)
    K, V, _ = cm.inputs(w)
    K[0, 0, 3, 7] = np.nan
    K[0, 0, 9, :] = 0.0
    V[0, 0, 11, 0] = np.inf
    V[0, 0, 12, :] = 3.0e38
    ref = cm.oracle_tables(1)
    lib = cm.lib_tables(1)
    rk, rv, _, _, kst, vst = o.encode_cache(ref, K, V)
    stats = dq.new_stats()
    kc, vc = cm.gpu_append_all(lib, K, V, torch.float32, stats=stats)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cm.flat(kc)[:, :, :64], rk)
    np.testing.assert_array_equal(cm.flat(vc)[:, :, :64], rv)
    assert dq.stats_dict(stats)["nonfinite_inputs"] == kst.nonfinite_inputs + vst.nonfinite_inputs == 3


ATTN_CASES = [
    # workload, B, Hkv, G, T, seq_lens
    ("tiny_b1_t256", 1, 1, 1, 256, [256]),
    ("qwen3_8b_b16_t8k", 3, 2, 4, 400, [400, 1, 267]),
    ("qwen3_8b_b16_t8k", 2, 2, 2, 130, [33, 130]),
    ("qwen3_8b_b16_t8k", 2, 1, 8, 96, [64, 95]),
    ("qwen3_8b_b16_t8k", 1, 2, 4, 3000, [2999]),
    # more token groups than warps in the grid: warp ranges cross (b, h) edges
    ("qwen3_8b_b16_t8k", 8, 8, 4, 3001, [3000, 33, 2900, 0, 2600, 2500, 40, 3001]),
    ("long_b4_t64k", 2, 8, 4, 20000, [20000, 12345]),
    # far fewer token groups than warps: most warps are empty and the combine
    # walks the few segments of each (b, h)
    ("qwen3_8b_b16_t8k", 1, 1, 4, 64, [64]),
    ("qwen3_8b_b16_t8k", 1, 8, 4, 64, [64]),
]


@pytest.mark.parametrize("wname,B,Hkv,G,T,seq", ATTN_CASES)
@pytest.mark.parametrize("q_dtype", [torch.float32, torch.bfloat16])
def test_attention_parity(wname, B, Hkv, G, T, seq, q_dtype):
    w = synth.scaled(synth.WORKLOADS[wname], B=B, Hkv=Hkv, Hq=Hkv * G, T=T)
    K, V, q = cm.inputs(w)
    if q_dtype == torch.bfloat16:
        q = torch.from_numpy(q).to(torch.bfloat16).float().numpy()
    ref_t = cm.oracle_tables(Hkv)
    lib = cm.lib_tables(Hkv)
    rk, rv, _, _, _, _ = o.encode_cache(ref_t, K, V)
    kc, vc = cm.gpu_append_all(lib, K, V, w.torch_dtype)
    ref = o.attention_fp64(ref_t, q, rk, rv, seq)
    stats = dq.new_stats()
    got = cm.gpu_attention(lib, q, kc, vc, seq, q_dtype=q_dtype, stats=stats)
    cm.assert_attention_close(got, ref, what=str((wname, B, Hkv, G, T)))
    assert dq.stats_dict(stats)["integrity_errors"] == 0


@pytest.mark.parametrize("kb,vb", [(3.0, 1.96), (1.96, 3.0), (4.0, 4.0)])
def test_attention_parity_other_budgets(kb, vb):
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=3, Hkv=2, Hq=8, T=700)
    K, V, q = cm.inputs(w)
    ref_t = cm.oracle_tables(2, kb, vb)
    lib = cm.lib_tables(2, kb, vb)
    rk, rv, _, _, _, _ = o.encode_cache(ref_t, K, V)
    kc, vc = cm.gpu_append_all(lib, K, V, w.torch_dtype)
    np.testing.assert_array_equal(cm.flat(kc)[:, :, :700], rk)
    np.testing.assert_array_equal(cm.flat(vc)[:, :, :700], rv)
    seq = [700, 255, 1]
    ref = o.attention_fp64(ref_t, q, rk, rv, seq)
    stats = dq.new_stats()
    got = cm.gpu_attention(lib, q, kc, vc, seq, stats=stats)
    cm.assert_attention_close(got, ref, what="budgets %s/%s" % (kb, vb))
    assert dq.stats_dict(stats)["integrity_errors"] == 0


def test_attention_bf16_output_and_scale():
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=2, Hkv=2, Hq=8, T=200)
    K, V, q = cm.inputs(w)
    ref_t = cm.oracle_tables(2)
    lib = cm.lib_tables(2)
    rk, rv, _, _, _, _ = o.encode_cache(ref_t, K, V)
    kc, vc = cm.gpu_append_all(lib, K, V, torch.bfloat16)
    ref = o.attention_fp64(ref_t, q, rk, rv, [200, 150], sm_scale=0.05)
    got = cm.gpu_attention(lib, q, kc, vc, [200, 150], out_dtype=torch.bfloat16, sm_scale=0.05)
    cm.assert_attention_close(got, ref, extra_rel=2.0 ** -8, what="bf16 out")


def test_attention_edges_and_clamping():
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=3, Hkv=1, Hq=4, T=64)
    K, V, q = cm.inputs(w)
    ref_t = cm.oracle_tables(1)
    lib = cm.lib_tables(1)
    rk, rv, _, _, _, _ = o.encode_cache(ref_t, K, V)
    kc, vc = cm.gpu_append_all(lib, K, V, torch.bfloat16)
    stats = dq.new_stats()
    # sequence 0 empty; sequence 2 claims 80 tokens but T_max is 48: clamped.
    got = cm.gpu_attention(lib, q, kc, vc, [0, 40, 80], T_max=48, stats=stats)
    assert np.all(got[0] == 0.0)
    ref = o.attention_fp64(ref_t, q, rk, rv, [0, 40, 48])
    cm.assert_attention_close(got, ref, what="clamped")
    assert dq.stats_dict(stats)["clamped_lengths"] == 1


def test_argument_errors():
    lib = cm.lib_tables(2)
    kc = torch.zeros((1, 2, 32, 36), dtype=torch.uint8, device="cuda")
    q = torch.zeros((1, 8, 128), device="cuda")
    out = torch.zeros_like(q)
    seq = torch.ones(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")

    def code(fn):
        with pytest.raises(dq.DqError) as e:
            fn()
        return e.value.code

    assert code(lambda: dq.dq_decode_attention(lib, torch.zeros((1, 6, 128), device="cuda"), kc, kc,
                                               seq, 1, torch.zeros((1, 6, 128), device="cuda"), ws)) == -4
    assert code(lambda: dq.dq_decode_attention(lib, q, kc, kc, seq, 64, out, ws)) == -4  # T_max > T_cap
    bad_cap = torch.zeros((1, 2, 24, 36), dtype=torch.uint8, device="cuda")
    assert code(lambda: dq.dq_decode_attention(lib, q, bad_cap, bad_cap, seq, 1, out, ws)) == -6
    assert code(lambda: dq.dq_decode_attention(lib, q, kc, kc, seq, 32, out, ws[:16])) == -5
    with pytest.raises(TypeError):
        dq.dq_decode_attention(lib, q.half(), kc, kc, seq, 1, out, ws)
    k = torch.zeros((1, 3, 1, 128), device="cuda")
    assert code(lambda: dq.dq_append_kv(lib, k, k, seq, kc, kc)) == -4  # Hkv mismatch
    k2 = torch.zeros((1, 2, 1, 128), device="cuda")
    assert code(lambda: dq.dq_append_kv(lib, k2, k2, seq, bad_cap, bad_cap)) == -6  # T_cap % 32
    with pytest.raises(dq.DqError):
        dq.dq_build_tables(n_kv_heads=2, head_dim=64)
