"""Drift mode 1 (drift, then the rate-distortion fill) on the GPU against the
oracle: containers bit-identical to attention's input definition, the same
drift and fill counts, at 1.96, 2.26 and 3.0 bits per value, for a small
append (one token per sequence, the warp-per-vector kernel with its fill), a
large one (the lane-per-vector kernel, then the drift kernel's fill phase for
every container) and paged pools; attention over the filled caches matches
the fp64 oracle, and the fill lowers the reconstruction error of the
synthetic rows as the oracle says it does.
"""
import numpy as np
import pytest
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from oracle import oracle as o
from tests import _common as cm

pytestmark = pytest.mark.gpu


def _tables(Hkv, bits):
    lib = dq.dq_build_tables(n_kv_heads=Hkv, k_bits_per_value=bits, v_bits_per_value=bits, drift_mode=1)
    ref = o.Tables(Hkv, k_container_bytes=o.container_bytes(bits), v_container_bytes=o.container_bytes(bits),
                   drift_mode=1)
    return lib, ref


@pytest.mark.parametrize("bits,B,T,dtype", [(2.26, 2, 300, torch.bfloat16), (1.96, 3, 100, torch.float32),
                                            (3.0, 2, 64, torch.bfloat16), (2.26, 2, 4096, torch.bfloat16),
                                            (1.96, 2, 4096, torch.float32), (3.0, 2, 4096, torch.bfloat16)])
def test_fill_containers_bit_exact(bits, B, T, dtype):
    Hkv = 8 if T == 4096 else 2
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=B, Hkv=Hkv, Hq=4 * Hkv, T=T)
    K, V, _ = cm.inputs(w)
    if dtype == torch.float32:
        K = K + np.float32(1e-3) * np.sin(np.arange(K.size, dtype=np.float32)).reshape(K.shape)
    lib, ref = _tables(Hkv, bits)
    stats = dq.new_stats()
    kc, vc = cm.gpu_append_all(lib, K, V, dtype, stats=stats)
    rk, rv, _, _, kst, vst = o.encode_cache(ref, K, V)
    np.testing.assert_array_equal(cm.flat(kc)[:, :, :T], rk)
    np.testing.assert_array_equal(cm.flat(vc)[:, :, :T], rv)
    s = dq.stats_dict(stats)
    assert s["k_syms_filled"] == kst.syms_filled and s["v_syms_filled"] == vst.syms_filled
    assert s["k_syms_drifted"] == kst.syms_drifted and s["v_syms_drifted"] == vst.syms_drifted
    if bits < 3.0:
        assert kst.syms_filled > 0 and vst.syms_filled > 0


def test_fill_one_token_steps_and_attention():
    B, Hkv, G, T = 3, 2, 4, 160
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=B, Hkv=Hkv, Hq=Hkv * G, T=T)
    K, V, q = cm.inputs(w)
    lib, ref = _tables(Hkv, 2.26)
    T_cap = cm.t_cap_for(T)
    kc = dq.new_cache(B, Hkv, T_cap, 36)
    vc = dq.new_cache(B, Hkv, T_cap, 36)
    # one token per call (the decode-step append)
    for t in range(T):
        kt = torch.from_numpy(np.ascontiguousarray(K[:, :, t:t + 1])).to("cuda", torch.bfloat16)
        vt = torch.from_numpy(np.ascontiguousarray(V[:, :, t:t + 1])).to("cuda", torch.bfloat16)
        dq.dq_append_kv(lib, kt, vt, torch.full((B,), t, dtype=torch.int32, device="cuda"), kc, vc)
    rk, rv, _, _, _, _ = o.encode_cache(ref, K, V)
    np.testing.assert_array_equal(cm.flat(kc)[:, :, :T], rk)
    np.testing.assert_array_equal(cm.flat(vc)[:, :, :T], rv)
    lens = [T, 97, 1]
    got = cm.gpu_attention(lib, q, kc, vc, lens)
    cm.assert_attention_close(got, o.attention_fp64(ref, q, rk, rv, lens), what="attention over filled caches")


@pytest.mark.parametrize("B,Hkv,T", [(2, 2, 256), (4, 8, 1280)])
def test_fill_paged_matches_contiguous(B, Hkv, T):
    # (4, 8, 1280): 40,960 vectors per stream take the lane kernel and the
    # drift kernel's fill, writing through the page table.
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=B, Hkv=Hkv, Hq=4 * Hkv, T=T)
    K, V, _ = cm.inputs(w)
    lib, ref = _tables(Hkv, 2.26)
    n_pages = T // 32
    num_pages = B * n_pages + 1
    ids = np.random.default_rng(5).permutation(num_pages)[:B * n_pages].reshape(B, n_pages).astype(np.int32)
    pt = torch.from_numpy(ids).cuda()
    kp = dq.new_pool(num_pages, Hkv, 36)
    vp = dq.new_pool(num_pages, Hkv, 36)
    kt = torch.from_numpy(K).to("cuda", torch.bfloat16).contiguous()
    vt = torch.from_numpy(V).to("cuda", torch.bfloat16).contiguous()
    dq.dq_append_kv_paged(lib, kt, vt, torch.zeros(B, dtype=torch.int32, device="cuda"), kp, vp, pt)
    torch.cuda.synchronize()
    rk, rv, _, _, _, _ = o.encode_cache(ref, K, V)
    t = torch.arange(T, device="cuda")
    for pool, r in ((kp, rk), (vp, rv)):
        g = pool[pt[:, t // 32].long()]                       # [B, T, Hkv, C, 32]
        g = g[torch.arange(B)[:, None], t[None, :], :, :, (t % 32)[None, :]].permute(0, 2, 1, 3)
        np.testing.assert_array_equal(g.cpu().numpy(), r)


def test_fill_lowers_reconstruction_error():
    B, Hkv, T = 2, 2, 512
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=B, Hkv=Hkv, Hq=4 * Hkv, T=T)
    K, V, _ = cm.inputs(w)
    errs = {}
    for mode in (0, 1):
        lib = dq.dq_build_tables(n_kv_heads=Hkv, drift_mode=mode)
        ref = o.Tables(Hkv, drift_mode=mode)
        kc, vc = cm.gpu_append_all(lib, K, V, torch.bfloat16)
        syms, nh, st = o.decode_containers(ref.k, cm.flat(kc)[:, :, :T].reshape(-1, 36))
        assert not st.any()
        xh = np.stack([o.dequantize(ref.k, syms.reshape(B, Hkv, T, 128)[b, h], nh.reshape(B, Hkv, T)[b, h],
                                    ref.signs[h]) for b in range(B) for h in range(Hkv)])
        errs[mode] = float(np.sum((xh - K.reshape(B * Hkv, T, 128).astype(np.float64)) ** 2))
    assert errs[1] < errs[0] * 0.99, errs
