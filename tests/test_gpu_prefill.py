"""Chunked-prefill attention over the compressed cache (dq_prefill_attention)
against the fp64 oracle (attention_prefill_fp64).

Caches are filled through dq_append_kv (containers bit-identical to the
oracle's, checked here too). Cases span several 128-row query blocks with a
ragged last block, several 32-token groups with a ragged causal diagonal,
G = 1, 2, 4, 8, fp32 and bf16 operands, rows whose positions fall outside the
cache, a single-token chunk (which is decode attention), paged pools,
31- and 48-byte containers, a full-size chunk of 512 tokens at the end of an
8K context and one of 256 tokens at the end of a 64K context (sampled (b, h)
rows). The bar is max |gpu - oracle| <= 2e-3 * RMS(oracle).
"""
import numpy as np
import pytest
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from oracle import oracle as o
from tests import _common as cm

pytestmark = pytest.mark.gpu


def _setup(B, Hkv, G, T, wname="qwen3_8b_b16_t8k", dtype=torch.bfloat16):
    w = synth.scaled(synth.WORKLOADS[wname], B=B, Hkv=Hkv, Hq=Hkv * G, T=T)
    K, V, _ = cm.inputs(w)
    lib = cm.lib_tables(Hkv)
    ref_t = cm.oracle_tables(Hkv)
    kc, vc = cm.gpu_append_all(lib, K, V, dtype)
    rk, rv, _, _, _, _ = o.encode_cache(ref_t, K, V)
    return w, lib, ref_t, kc, vc, rk, rv


def _pad(rc, T_cap):
    """Oracle containers padded to the cache capacity (zero containers)."""
    if rc.shape[2] == T_cap:
        return rc
    pad = np.zeros(rc.shape[:2] + (T_cap - rc.shape[2], rc.shape[3]), rc.dtype)
    return np.concatenate([rc, pad], axis=2)


def _prefill(lib, q, kc, vc, q_start, q_dtype=torch.float32, out_dtype=torch.float32, stats=None):
    qt = torch.from_numpy(np.ascontiguousarray(q, dtype=np.float32)).to(device="cuda", dtype=q_dtype)
    out = torch.full(q.shape, float("nan"), dtype=out_dtype, device="cuda")
    qs = torch.tensor(q_start, dtype=torch.int32, device="cuda")
    dq.dq_prefill_attention(lib, qt, kc, vc, qs, out, stats=stats)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("G,q_dtype", [(4, torch.float32), (4, torch.bfloat16), (1, torch.float32),
                                       (2, torch.bfloat16), (8, torch.float32)])
def test_prefill_matches_oracle(G, q_dtype):
    B, Hkv, T = 2, 2, 400
    w, lib, ref_t, kc, vc, rk, rv = _setup(B, Hkv, G, T)
    np.testing.assert_array_equal(cm.flat(kc)[:, :, :T], rk)
    np.testing.assert_array_equal(cm.flat(vc)[:, :, :T], rv)
    n_q = 150  # 128 / G query tokens per block: ragged last block for every G
    q_start = [0, T - n_q]
    q = synth.q_chunk(w, n_q)
    if q_dtype == torch.bfloat16:
        q = torch.from_numpy(q).to(torch.bfloat16).float().numpy()
    stats = dq.new_stats()
    got = _prefill(lib, q, kc, vc, q_start, q_dtype=q_dtype, stats=stats)
    ref = o.attention_prefill_fp64(ref_t, q, _pad(rk, kc.shape[2]), _pad(rv, vc.shape[2]), q_start)
    cm.assert_attention_close(got, ref, what="prefill G=%d" % G)
    s = dq.stats_dict(stats)
    assert s["wait_timeouts"] == 0 and s["integrity_errors"] == 0 and s["clamped_lengths"] == 0


def test_prefill_bf16_output_and_unaligned_start():
    B, Hkv, G, T = 3, 1, 4, 300
    w, lib, ref_t, kc, vc, rk, rv = _setup(B, Hkv, G, T)
    n_q = 37
    q_start = [5, 263, 100]
    q = synth.q_chunk(w, n_q)
    got = _prefill(lib, q, kc, vc, q_start, out_dtype=torch.bfloat16)
    ref = o.attention_prefill_fp64(ref_t, q, _pad(rk, kc.shape[2]), _pad(rv, vc.shape[2]), q_start)
    # bf16 output: add the output rounding (2^-9 of the largest value)
    cm.assert_attention_close(got, ref, extra_rel=2.0 ** -8, what="prefill bf16 out")


def test_single_token_chunk_is_decode_attention():
    B, Hkv, G, T = 2, 2, 4, 333
    w, lib, ref_t, kc, vc, rk, rv = _setup(B, Hkv, G, T)
    q1 = synth.q_block(w)  # [B, Hq, 128]
    lens = [T, 200]
    got = _prefill(lib, q1[:, None], kc, vc, [lens[0] - 1, lens[1] - 1])[:, 0]
    dec = cm.gpu_attention(lib, q1, kc, vc, lens)
    ref = o.attention_fp64(ref_t, q1, rk, rv, lens)
    cm.assert_attention_close(got, ref, what="prefill n_q=1")
    cm.assert_attention_close(dec, ref, what="decode")
    cm.assert_attention_close(got, dec, what="prefill vs decode")


def test_rows_outside_the_cache_are_zero_and_counted():
    B, Hkv, G, T = 5, 1, 2, 96
    w, lib, ref_t, kc, vc, rk, rv = _setup(B, Hkv, G, T)
    T_cap = kc.shape[2]
    n_q = 10
    # 4 rows below 0; 7 rows at or past T_cap; all valid; all past the cache;
    # all below 0 (whole query blocks with nothing to attend)
    q_start = [-4, T_cap - 3, 40, T_cap + 5, -1000]
    q = synth.q_chunk(w, n_q)
    stats = dq.new_stats()
    got = _prefill(lib, q, kc, vc, q_start, stats=stats)
    ref = o.attention_prefill_fp64(ref_t, q, _pad(rk, T_cap), _pad(rv, T_cap), q_start)
    assert np.all(got[0, :4] == 0.0) and np.all(got[1, 3:] == 0.0)
    assert np.all(got[3] == 0.0) and np.all(got[4] == 0.0)
    cm.assert_attention_close(got, ref, what="prefill out-of-range rows")
    s = dq.stats_dict(stats)
    assert s["clamped_lengths"] == (4 + 7 + 10 + 10) * G and s["wait_timeouts"] == 0


def test_paged_prefill_equals_contiguous():
    B, Hkv, G, T = 2, 2, 4, 256
    w, lib, ref_t, kc, vc, rk, rv = _setup(B, Hkv, G, T)
    n_pages = T // 32
    num_pages = B * n_pages + 3
    rng = np.random.default_rng(11)
    ids = rng.permutation(num_pages)[:B * n_pages].reshape(B, n_pages)
    pt = torch.from_numpy(ids.astype(np.int32)).cuda()
    kp = dq.new_pool(num_pages, Hkv, 36)
    vp = dq.new_pool(num_pages, Hkv, 36)
    # copy the contiguous caches' 32-token blocks into their pages
    kb = kc.view(B, Hkv, n_pages, -1)
    vb = vc.view(B, Hkv, n_pages, -1)
    for b in range(B):
        for j in range(n_pages):
            kp.view(num_pages, Hkv, -1)[ids[b, j]] = kb[b, :, j]
            vp.view(num_pages, Hkv, -1)[ids[b, j]] = vb[b, :, j]
    n_q = 70
    q_start = [T - n_q, 100]
    q = synth.q_chunk(w, n_q)
    qt = torch.from_numpy(q).cuda()
    qs = torch.tensor(q_start, dtype=torch.int32, device="cuda")
    out_c = torch.empty_like(qt)
    out_p = torch.empty_like(qt)
    stats = dq.new_stats()
    dq.dq_prefill_attention(lib, qt, kc, vc, qs, out_c)
    dq.dq_prefill_attention_paged(lib, qt, kp, vp, pt, qs, out_p, stats=stats)
    torch.cuda.synchronize()
    assert torch.equal(out_c, out_p)
    s = dq.stats_dict(stats)
    assert s["bad_pages"] == 0 and s["wait_timeouts"] == 0


def test_full_size_chunk_at_end_of_8k_context_sampled():
    w = synth.WORKLOADS["qwen3_8b_b16_t8k"]
    lib = cm.lib_tables(w.Hkv)
    ref_t = cm.oracle_tables(w.Hkv)
    kc = dq.new_cache(w.B, w.Hkv, w.T, 36)
    vc = dq.new_cache(w.B, w.Hkv, w.T, 36)
    synth.prefill_cache(lib, w, kc, vc, w.T)
    n_q = 512
    q_start = [w.T - n_q] * w.B
    q = synth.q_chunk(w, n_q)
    stats = dq.new_stats()
    got = _prefill(lib, q, kc, vc, q_start, stats=stats)
    kf, vf = cm.flat(kc), cm.flat(vc)
    rows = [(0, 0), (7, 5), (15, 7)]
    ref = o.attention_prefill_fp64(ref_t, q, kf, vf, q_start, rows=rows)
    G = w.Hq // w.Hkv
    for b, h in rows:
        cm.assert_attention_close(got[b, :, h * G:(h + 1) * G], ref[b, :, h * G:(h + 1) * G],
                                  what="8K chunk row (%d,%d)" % (b, h))
    s = dq.stats_dict(stats)
    assert s["wait_timeouts"] == 0 and s["integrity_errors"] == 0


@pytest.mark.parametrize("bits", [1.96, 3.0])
def test_prefill_other_budgets(bits):
    # 31- and 48-byte containers (other decode tables, the two-byte K step at
    # 1.96 bits)
    B, Hkv, G, T = 2, 2, 4, 300
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=B, Hkv=Hkv, Hq=Hkv * G, T=T)
    K, V, _ = cm.inputs(w)
    lib = cm.lib_tables(Hkv, k_bits=bits, v_bits=bits)
    ref_t = cm.oracle_tables(Hkv, k_bits=bits, v_bits=bits)
    kc, vc = cm.gpu_append_all(lib, K, V, torch.bfloat16)
    rk, rv, _, _, _, _ = o.encode_cache(ref_t, K, V)
    n_q = 90
    q_start = [T - n_q, 17]
    q = synth.q_chunk(w, n_q)
    stats = dq.new_stats()
    got = _prefill(lib, q, kc, vc, q_start, stats=stats)
    ref = o.attention_prefill_fp64(ref_t, q, _pad(rk, kc.shape[2]), _pad(rv, vc.shape[2]), q_start)
    cm.assert_attention_close(got, ref, what="prefill %.2f bits" % bits)
    s = dq.stats_dict(stats)
    assert s["wait_timeouts"] == 0 and s["integrity_errors"] == 0


def test_long_context_chunk_sampled():
    # The last 256 tokens of a 65536-token context (one (b, h) row checked).
    w = synth.WORKLOADS["long_b4_t64k"]
    lib = cm.lib_tables(w.Hkv)
    ref_t = cm.oracle_tables(w.Hkv)
    kc = dq.new_cache(w.B, w.Hkv, w.T, 36)
    vc = dq.new_cache(w.B, w.Hkv, w.T, 36)
    synth.prefill_cache(lib, w, kc, vc, w.T)
    n_q = 256
    q_start = [w.T - n_q] * w.B
    q = synth.q_chunk(w, n_q)
    stats = dq.new_stats()
    got = _prefill(lib, q, kc, vc, q_start, out_dtype=torch.bfloat16, stats=stats)
    G = w.Hq // w.Hkv
    b, h = 2, 5
    ref = o.attention_prefill_fp64(ref_t, q, cm.flat(kc), cm.flat(vc), q_start, rows=[(b, h)])
    cm.assert_attention_close(got[b, :, h * G:(h + 1) * G], ref[b, :, h * G:(h + 1) * G], extra_rel=2.0 ** -8,
                              what="64K chunk row (%d,%d)" % (b, h))
    s = dq.stats_dict(stats)
    assert s["wait_timeouts"] == 0 and s["integrity_errors"] == 0


def test_small_workspace_runs_in_waves_identically():
    # A workspace with room for 3 (b, KV head) rows: 2 x 4 rows run in 3
    # waves and give the same bits as one wave; below one row is refused.
    B, Hkv, G, T = 2, 4, 4, 300
    w, lib, ref_t, kc, vc, rk, rv = _setup(B, Hkv, G, T)
    T_cap = kc.shape[2]
    n_q = 64
    q_start = [T - n_q, 40]
    qt = torch.from_numpy(synth.q_chunk(w, n_q)).cuda()
    qs = torch.tensor(q_start, dtype=torch.int32, device="cuda")
    full = torch.empty(dq.dq_prefill_workspace_bytes(lib, B, Hkv, T_cap), dtype=torch.uint8, device="cuda")
    row = dq.dq_prefill_workspace_bytes(lib, 1, 1, T_cap)
    small = torch.empty(3 * row + 100, dtype=torch.uint8, device="cuda")
    out_a = torch.empty_like(qt)
    out_b = torch.empty_like(qt)
    stats = dq.new_stats()
    dq.dq_prefill_attention(lib, qt, kc, vc, qs, out_a, workspace=full)
    dq.dq_prefill_attention(lib, qt, kc, vc, qs, out_b, workspace=small, stats=stats)
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
    assert dq.stats_dict(stats)["wait_timeouts"] == 0
    with pytest.raises(dq.DqError):
        dq.dq_prefill_attention(lib, qt, kc, vc, qs, out_b, workspace=small[:row - 16])
