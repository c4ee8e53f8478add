"""dq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (for example a plugin handed only input and output
pointers, or a serving loop that must not call cudaMalloc once running). It
takes no workspace and uses the library's fixed device scratch array instead.

Checked through the C-ABI against dq_decode_attention (which is given a
caller-allocated workspace) on two calls in a row with different queries, so a
second call that reuses the scratch left by the first must still be right.
This file is collected last so a failure here does not hide other tests.
"""
import numpy as np
import pytest
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from tests import _common as cm

pytestmark = pytest.mark.gpu


def _case():
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=3, Hkv=2, Hq=8, T=700)
    K, V, q = cm.inputs(w)
    tab = cm.lib_tables(w.Hkv)
    kc, vc = cm.gpu_append_all(tab, K, V, w.torch_dtype)
    return w, tab, kc, vc


def test_noalloc_matches_workspace_entry_on_two_calls():
    w, tab, kc, vc = _case()
    seq_lens = [700, 1, 433]
    seq = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    T_max = 700
    for call in range(2):
        q = torch.from_numpy(synth.q_block(w, step=call)).cuda()
        ws = torch.empty(dq.dq_decode_workspace_bytes(tab, w.B, w.Hq, w.Hkv, T_max),
                         dtype=torch.uint8, device="cuda")
        ref = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device="cuda")
        dq.dq_decode_attention(tab, q, kc, vc, seq, T_max, ref, ws)
        got = torch.full((w.B, w.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        stats = dq.new_stats()
        dq.dq_decode_attention_noalloc(tab, q, kc, vc, seq, T_max, got, stats=stats)
        torch.cuda.synchronize()
        r = ref.cpu().numpy().astype(np.float64)
        g = got.cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all()
        cm.assert_attention_close(g, r, what="noalloc call %d" % call)
        assert dq.stats_dict(stats)["integrity_errors"] == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    tab = cm.lib_tables(8)
    B, Hq, Hkv, T_cap = 256, 64, 8, 32  # 2048 (b, h) slots of 8 heads > the 8 MiB scratch
    assert dq.dq_decode_workspace_bytes(tab, B, Hq, Hkv, T_cap) > (8 << 20)
    kc = torch.zeros((B, Hkv, T_cap, 36), dtype=torch.uint8, device="cuda")
    q = torch.zeros((B, Hq, 128), dtype=torch.float32, device="cuda")
    out = torch.zeros_like(q)
    seq = torch.full((B,), T_cap, dtype=torch.int32, device="cuda")
    with pytest.raises(dq.DqError) as e:
        dq.dq_decode_attention_noalloc(tab, q, kc, kc, seq, T_cap, out)
    assert e.value.code == -5  # DQ_ERR_WORKSPACE
