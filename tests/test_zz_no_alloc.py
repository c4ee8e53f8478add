"""dq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (for example a plugin handed only input and output
pointers, or a serving loop that must not call cudaMalloc once running). It
takes no workspace and uses the library's fixed device scratch array instead.

Checked through the C-ABI against dq_decode_attention (which is given a
caller-allocated workspace). Both run the same kernels on the same inputs, so
the outputs must be bit-identical. The calls go large first, then smaller, so
the second call runs over slots and prefix sums that the first left in the
shared scratch array; stale contents must never reach an output.
This file is collected last so a failure here does not hide other tests.
"""
import pytest
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from tests import _common as cm

pytestmark = pytest.mark.gpu


def _case():
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=4, Hkv=2, Hq=8, T=1500)
    K, V, q = cm.inputs(w)
    tab = cm.lib_tables(w.Hkv)
    kc, vc = cm.gpu_append_all(tab, K, V, w.torch_dtype)
    return w, tab, kc, vc


def _both(tab, w, q, kc, vc, seq_lens):
    B = len(seq_lens)
    seq = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    T_max = max(seq_lens)
    ws = torch.empty(dq.dq_decode_workspace_bytes(tab, B, w.Hq, w.Hkv, T_max), dtype=torch.uint8,
                     device="cuda")
    ref = torch.empty((B, w.Hq, 128), dtype=torch.float32, device="cuda")
    dq.dq_decode_attention(tab, q[:B], kc[:B], vc[:B], seq, T_max, ref, ws)
    got = torch.full((B, w.Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
    stats = dq.new_stats()
    dq.dq_decode_attention_noalloc(tab, q[:B], kc[:B], vc[:B], seq, T_max, got, stats=stats)
    torch.cuda.synchronize()
    return ref, got, dq.stats_dict(stats)


def test_noalloc_matches_workspace_entry_on_two_calls():
    w, tab, kc, vc = _case()
    # A large call (4 sequences, long contexts), then a smaller one (2
    # sequences, short and ragged) with other queries.
    for call, seq_lens in enumerate([[1500, 1500, 1201, 1499], [37, 1]]):
        q = torch.from_numpy(synth.q_block(w, step=call)).cuda()
        ref, got, st = _both(tab, w, q, kc, vc, seq_lens)
        assert torch.isfinite(got).all()
        assert torch.equal(got, ref), "noalloc call %d differs from dq_decode_attention" % call
        assert st["integrity_errors"] == 0


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
