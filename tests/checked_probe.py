"""Run by tests/test_gpu_checked.py in a child process (DQ_LIBRARY selects
the library): a small cache of valid containers, then the same cache with a
few containers corrupted on the host so that their decoders read past their
bytes. Prints one JSON line with the stats of each call. Runs nothing when
imported."""
import json
import sys

import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth


def main():
    w = synth.scaled(synth.WORKLOADS["qwen3_8b_b16_t8k"], B=2, Hkv=2, Hq=8, T=256)
    tab = dq.dq_build_tables(n_kv_heads=w.Hkv)
    B, Hkv, T, C = w.B, w.Hkv, w.T, tab.k.container_bytes
    rows = [(b, h) for b in range(B) for h in range(Hkv)]
    k = torch.from_numpy(synth.kv_block(w, "k", rows, n=T)).cuda().view(B, Hkv, T, 128)
    v = torch.from_numpy(synth.kv_block(w, "v", rows, n=T)).cuda().view(B, Hkv, T, 128)
    kc = dq.new_cache(B, Hkv, T, C)
    vc = dq.new_cache(B, Hkv, T, tab.v.container_bytes)
    st = dq.new_stats()
    dq.dq_append_kv(tab, k, v, torch.zeros(B, dtype=torch.int32, device="cuda"), kc, vc, stats=st)
    q = torch.from_numpy(synth.q_block(w, 0)).cuda().view(B, w.Hq, 128)
    seq = torch.full((B,), T, dtype=torch.int32, device="cuda")
    out = torch.empty((B, w.Hq, 128), dtype=torch.float32, device="cuda")
    ws = torch.empty(dq.dq_decode_workspace_bytes(tab, B, w.Hq, Hkv, T), dtype=torch.uint8, device="cuda")
    res = {"append": dq.stats_dict(st)}

    def decode(tag):
        s = dq.new_stats()
        dq.dq_decode_attention(tab, q, kc, vc, seq, T, out, ws, stats=s)
        torch.cuda.synchronize()
        res[tag] = dq.stats_dict(s)
        res[tag + "_finite"] = bool(torch.isfinite(out).all())

    def prefill(tag):
        n_q = 40
        qc = torch.from_numpy(synth.q_chunk(w, n_q)).cuda()
        o = torch.empty((B, n_q, w.Hq, 128), dtype=torch.float32, device="cuda")
        qs = torch.full((B,), T - n_q, dtype=torch.int32, device="cuda")
        pw = torch.empty(dq.dq_prefill_workspace_bytes(tab, B, Hkv, T), dtype=torch.uint8, device="cuda")
        s = dq.new_stats()
        dq.dq_prefill_attention(tab, qc, kc, vc, qs, o, workspace=pw, stats=s)
        torch.cuda.synchronize()
        res[tag] = dq.stats_dict(s)

    decode("decode_valid")
    prefill("prefill_valid")
    # Corrupt 5 K and 3 V containers: state x = 2^16 (bytes 2..4 of the
    # interleaved layout [T/32][C][32]) and a zero payload, so that every
    # decode step takes at least one byte and the decoder runs past byte C.
    for cache, toks in ((kc, [(0, 0, 3), (0, 1, 40), (1, 0, 100), (1, 1, 200), (1, 1, 255)]),
                        (vc, [(0, 0, 7), (1, 0, 64), (1, 1, 129)])):
        for b, h, t in toks:
            g, lane = t // 32, t % 32
            blk = cache[b, h].view(T // 32, cache.shape[3], 32)
            blk[g, 2:5, lane] = torch.tensor([0, 0, 1], dtype=torch.uint8, device="cuda")
            blk[g, 5:, lane] = 0
    decode("decode_corrupt")
    prefill("prefill_corrupt")
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    sys.exit(main())
