"""Paged caches: dq_append_kv_paged and dq_decode_attention_paged.

Pages of 32 tokens are handed out in a shuffled order from a pool larger
than needed. Containers gathered through the page table must be bit-identical
to the oracle's, attention must match the oracle within 2e-3 x RMS and be
bit-identical to the contiguous-cache call on the same tokens, and page-table
entries out of range must be counted without being dereferenced.
"""
import numpy as np
import pytest
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from oracle import oracle as o
from tests import _common as cm

pytestmark = pytest.mark.gpu


def _page_table(lens, max_pages, num_pages, seed):
    """int32 [B, max_pages]: distinct pages in a shuffled order for the pages a
    sequence uses, -1 elsewhere."""
    rng = np.random.default_rng(seed)
    need = [(n + 31) // 32 for n in lens]
    assert sum(need) <= num_pages
    ids = rng.permutation(num_pages)[:sum(need)]
    pt = np.full((len(lens), max_pages), -1, np.int32)
    k = 0
    for b, m in enumerate(need):
        pt[b, :m] = ids[k:k + m]
        k += m
    return torch.from_numpy(pt).cuda()


def _gather(pool, pt, T):
    """Flat containers [B, Hkv, T, C] of a pool through a page table."""
    B = pt.shape[0]
    t = torch.arange(T, device=pool.device)
    pages = pt[:, t // 32].long().clamp(min=0)                  # [B, T]
    g = pool[pages]                                               # [B, T, Hkv, C, 32]
    g = g[torch.arange(B)[:, None], t[None, :], :, :, (t % 32)[None, :]]  # [B, T, Hkv, C]
    return g.permute(0, 2, 1, 3).contiguous().cpu().numpy()


def _inputs(B, Hkv, G, T, wname="qwen3_8b_b16_t8k"):
    w = synth.scaled(synth.WORKLOADS[wname], B=B, Hkv=Hkv, Hq=Hkv * G, T=T)
    K, V, q = cm.inputs(w)
    return w, K, V, q


def test_paged_append_and_decode_match_oracle_and_contiguous():
    B, Hkv, G, T = 3, 2, 4, 700
    lens = [700, 33, 433]
    w, K, V, q = _inputs(B, Hkv, G, T)
    lib = cm.lib_tables(Hkv)
    ref_t = cm.oracle_tables(Hkv)
    rk, rv, _, _, _, _ = o.encode_cache(ref_t, K, V)
    max_pages, num_pages = (T + 31) // 32, 60
    pt = _page_table(lens, max_pages, num_pages, seed=7)
    kp = dq.new_pool(num_pages, Hkv, 36)
    vp = dq.new_pool(num_pages, Hkv, 36)
    stats = dq.new_stats()
    # two appends (600 tokens, then 100) of every sequence; tokens past a
    # sequence's own pages (page -1) are dropped
    done = 0
    for n in (600, 100):
        kt = torch.from_numpy(K[:, :, done:done + n]).to("cuda", torch.bfloat16).contiguous()
        vt = torch.from_numpy(V[:, :, done:done + n]).to("cuda", torch.bfloat16).contiguous()
        start = torch.full((B,), done, dtype=torch.int32, device="cuda")
        dq.dq_append_kv_paged(lib, kt, vt, start, kp, vp, pt, stats=stats)
        done += n
    torch.cuda.synchronize()
    kf, vf = _gather(kp, pt, T), _gather(vp, pt, T)
    for b, n in enumerate(lens):
        np.testing.assert_array_equal(kf[b, :, :n], rk[b, :, :n])
        np.testing.assert_array_equal(vf[b, :, :n], rv[b, :, :n])
    s = dq.stats_dict(stats)
    # tokens past a sequence's mapped pages, K and V of every head
    unmapped = sum(max(0, T - 32 * ((n + 31) // 32)) for n in lens) * Hkv * 2
    assert s["bad_pages"] == unmapped and s["dropped_writes"] == unmapped

    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(dq.dq_decode_workspace_bytes(lib, B, w.Hq, Hkv, T), dtype=torch.uint8, device="cuda")
    qt = torch.from_numpy(q).cuda()
    out_p = torch.empty((B, w.Hq, 128), device="cuda")
    st2 = dq.new_stats()
    dq.dq_decode_attention_paged(lib, qt, kp, vp, pt, seq, T, out_p, ws, stats=st2)
    # the same tokens in a contiguous cache
    kc, vc = cm.gpu_append_all(lib, K, V, torch.bfloat16)
    out_c = torch.empty_like(out_p)
    dq.dq_decode_attention(lib, qt, kc, vc, seq, T, out_c, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out_c)
    ref = o.attention_fp64(ref_t, q, rk, rv, lens)
    cm.assert_attention_close(out_p.cpu().numpy().astype(np.float64), ref, what="paged")
    s2 = dq.stats_dict(st2)
    assert s2["bad_pages"] == 0 and s2["integrity_errors"] == 0


def test_paged_large_append_uses_the_lane_kernel_bit_exact():
    # 2 x 8 x 4096 = 65536 vectors per stream: lane-per-vector encode and the
    # separate drift kernel.
    B, Hkv, T = 2, 8, 4096
    w, K, V, _ = _inputs(B, Hkv, 4, T)
    lib = cm.lib_tables(Hkv)
    ref_t = cm.oracle_tables(Hkv)
    rk, rv, _, _, kst, vst = o.encode_cache(ref_t, K, V)
    max_pages, num_pages = T // 32, 2 * (T // 32) + 5
    pt = _page_table([T, T], max_pages, num_pages, seed=3)
    kp = dq.new_pool(num_pages, Hkv, 36)
    vp = dq.new_pool(num_pages, Hkv, 36)
    stats = dq.new_stats()
    kt = torch.from_numpy(K).to("cuda", torch.bfloat16).contiguous()
    vt = torch.from_numpy(V).to("cuda", torch.bfloat16).contiguous()
    dq.dq_append_kv_paged(lib, kt, vt, torch.zeros(B, dtype=torch.int32, device="cuda"), kp, vp, pt,
                          stats=stats)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_gather(kp, pt, T), rk)
    np.testing.assert_array_equal(_gather(vp, pt, T), rv)
    s = dq.stats_dict(stats)
    assert s["k_syms_drifted"] == kst.syms_drifted and s["v_syms_drifted"] == vst.syms_drifted
    assert s["bad_pages"] == 0 and s["dropped_writes"] == 0


def test_out_of_range_pages_are_counted_not_read():
    B, Hkv, G, T = 2, 1, 4, 96
    w, K, V, q = _inputs(B, Hkv, G, T)
    lib = cm.lib_tables(Hkv)
    num_pages, max_pages = 8, 3
    pt = torch.tensor([[0, 1, 2], [3, 99, -5]], dtype=torch.int32, device="cuda")
    kp = dq.new_pool(num_pages, Hkv, 36)
    vp = dq.new_pool(num_pages, Hkv, 36)
    stats = dq.new_stats()
    kt = torch.from_numpy(K).to("cuda", torch.bfloat16).contiguous()
    vt = torch.from_numpy(V).to("cuda", torch.bfloat16).contiguous()
    dq.dq_append_kv_paged(lib, kt, vt, torch.zeros(B, dtype=torch.int32, device="cuda"), kp, vp, pt,
                          stats=stats)
    torch.cuda.synchronize()
    s = dq.stats_dict(stats)
    # sequence 1: tokens 32..95 map to pages 99 and -5 -> dropped, K and V
    assert s["bad_pages"] == 2 * 64 and s["dropped_writes"] == 2 * 64
    seq = torch.tensor([96, 96], dtype=torch.int32, device="cuda")
    ws = torch.empty(dq.dq_decode_workspace_bytes(lib, B, w.Hq, Hkv, T), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, w.Hq, 128), device="cuda")
    st2 = dq.new_stats()
    dq.dq_decode_attention_paged(lib, torch.from_numpy(q).cuda(), kp, vp, pt, seq, T, out, ws, stats=st2)
    torch.cuda.synchronize()
    assert dq.stats_dict(st2)["bad_pages"] > 0
    # sequence 0 is untouched by sequence 1's bad entries
    ref_t = cm.oracle_tables(Hkv)
    rk, rv, _, _, _, _ = o.encode_cache(ref_t, K[:1], V[:1])
    ref = o.attention_fp64(ref_t, q[:1], rk, rv, [96])
    cm.assert_attention_close(out[:1].cpu().numpy().astype(np.float64), ref, what="page-table errors")
