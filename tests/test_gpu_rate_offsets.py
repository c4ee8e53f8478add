"""Tables designed above the container's nominal rate (dq_config rate
offsets) on the GPU: at +0.05 bit/value for K and +0.14 for V the drift rates
are near the pages' 0.75 % and 5 % ([news] "Drift: Bending Variable Back to
Fixed"), so drift runs for a third to nearly all containers. Containers and
drift counts must still be bit-identical to the oracle, in the
warp-per-vector path (small appends) and the lane-per-vector path with the
separate drift kernel (large appends), and decode and prefill attention over
those caches must match the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from oracle import oracle as o
from tests import _common as cm

pytestmark = pytest.mark.gpu

K_OFF, V_OFF = 0.05, 0.14


def _tables(Hkv):
    lib = dq.dq_build_tables(n_kv_heads=Hkv, k_rate_offset=K_OFF, v_rate_offset=V_OFF)
    ref = o.Tables(Hkv, k_rate_offset=K_OFF, v_rate_offset=V_OFF)
    return lib, ref


@pytest.mark.parametrize("B,Hkv,T", [(2, 2, 500), (2, 8, 4096)])
def test_offset_tables_bit_exact(B, Hkv, T):
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=B, Hkv=Hkv, Hq=4 * Hkv, T=T)
    K, V, q = cm.inputs(w)
    lib, ref = _tables(Hkv)
    stats = dq.new_stats()
    kc, vc = cm.gpu_append_all(lib, K, V, torch.bfloat16, stats=stats)
    rk, rv, _, _, kst, vst = o.encode_cache(ref, K, V)
    np.testing.assert_array_equal(cm.flat(kc)[:, :, :T], rk)
    np.testing.assert_array_equal(cm.flat(vc)[:, :, :T], rv)
    s = dq.stats_dict(stats)
    assert s["k_syms_drifted"] == kst.syms_drifted and s["v_syms_drifted"] == vst.syms_drifted
    assert s["k_cont_drifted"] == kst.cont_drifted and s["v_cont_drifted"] == vst.cont_drifted
    assert s["overflow_fallbacks"] == kst.overflow_fallbacks + vst.overflow_fallbacks
    # drift near the pages' rates: several tenths of a percent of K symbols,
    # a few percent of V symbols
    n = B * Hkv * T * 128
    assert 0.003 < kst.syms_drifted / n < 0.02 and 0.02 < vst.syms_drifted / n < 0.09
    if T <= 500:
        lens = [T, T - 123]
        got = cm.gpu_attention(lib, q, kc, vc, lens)
        cm.assert_attention_close(got, o.attention_fp64(ref, q, rk, rv, lens), what="decode, offset tables")
        n_q = 64
        qc = synth.q_chunk(w, n_q)
        qt = torch.from_numpy(qc).cuda()
        out = torch.empty_like(qt)
        starts = [T - n_q, 100]
        dq.dq_prefill_attention(lib, qt, kc, vc, torch.tensor(starts, dtype=torch.int32, device="cuda"), out)
        torch.cuda.synchronize()
        pad = np.zeros((B, Hkv, kc.shape[2] - T, 36), np.uint8)
        refp = o.attention_prefill_fp64(ref, qc, np.concatenate([rk, pad], 2), np.concatenate([rv, pad], 2), starts)
        cm.assert_attention_close(out.cpu().numpy().astype(np.float64), refp, what="prefill, offset tables")
