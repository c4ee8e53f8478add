"""Drift against distortion as the level design's target rate moves (TEST
INFRASTRUCTURE).

[news] "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits", "Drift:
Bending Variable Back to Fixed": drift changes 0.75 % of key symbols and
5.00 % of value symbols, none by more than one level. How often drift fires
depends on how far the level design's entropy sits above what the container
holds: the tables target r = (8 (C - 2) - 24) / 128 bits per value plus a
per-stream rate offset (dq_config.k_rate_offset / v_rate_offset). A higher
target gives finer levels (less quantisation error) and more over-long
containers (more drift error); this module measures that trade with the
oracle only (CPU) on the synthetic workload rows: per offset and stream, the
design entropy, the drift rates, the mean squared error of the rotated
coordinates after drift, the relative error of the reconstructed vectors and
the relative RMS error of decode attention against fp64 attention over the
unquantised K and V.

    python -m oracle.rate_offset_sweep [--rows 48] [--tokens 512] [--bits 2.26]
"""
from __future__ import annotations

import argparse
import math
import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from oracle import fixed_width_control as fw  # noqa: E402
from oracle import oracle as o  # noqa: E402

OFFSETS = (-0.1, 0.0, 0.05, 0.1, 0.15, 0.2)


def sweep(workload: str = "qwen3_8b_b16_t8k", rows: int = 48, tokens: int = 512, bits: float = 2.26,
          offsets=OFFSETS):
    """One result per offset (same offset for K and V): dict with per-stream
    entropy, drift rates, MSE of the rotated coordinates and relative error
    of x, plus the attention error of the pair."""
    from decode_attention_dq_b200 import synth

    w = synth.WORKLOADS[workload]
    G = w.Hq // w.Hkv
    C = o.container_bytes(bits)
    picks = [(b % w.B, (b * 3) % w.Hkv) for b in range(rows)]
    data = {s: [synth.kv_row(w, s, b, h, n=tokens) for b, h in picks] for s in ("k", "v")}
    qs = [synth.q_rows(w, b)[h * G:(h + 1) * G].astype(np.float64) for b, h in picks]
    ref = [fw.attention(qs[r], data["k"][r].astype(np.float64), data["v"][r].astype(np.float64))
           for r in range(rows)]
    out = []
    for off in offsets:
        tab = o.Tables(w.Hkv, k_container_bytes=C, v_container_bytes=C, k_rate_offset=off, v_rate_offset=off)
        res = {"offset": off}
        recon = {}
        for s in ("k", "v"):
            st = tab.k if s == "k" else tab.v
            y = st.yf.astype(np.float64)
            mse = rel = 0.0
            moved = cont = fb = 0
            recon[s] = []
            for r in range(rows):
                h = picks[r][1]
                x = data[s][r]
                cnt, syms, stt, bad = o.encode_vectors(st, tab.signs, x, np.full(tokens, h, np.int32))
                assert bad == 0
                u = np.stack([o.rotate_normalize(v, tab.signs[h])[0] for v in x]).astype(np.float64)
                mse += float(np.sum((u - y[syms]) ** 2))
                d, nh, status = o.decode_containers(st, cnt)
                assert not status.any()
                xh = fw.reconstruct(y[d.astype(np.int64)], nh, tab.signs[h])
                recon[s].append(xh)
                rel += float(np.sum((xh - x) ** 2)) / float(np.sum(x.astype(np.float64) ** 2))
                moved += stt.syms_drifted
                cont += stt.cont_drifted
                fb += stt.overflow_fallbacks
            n = rows * tokens
            res[s] = dict(entropy=st.entropy, rate=st.rate, lam=st.lam, mse_u=mse / (n * o.D), rel_x=rel / rows,
                          drift_syms=moved / (n * o.D), drift_cont=cont / n, fallbacks=fb)
        num = sum(float(np.sum((fw.attention(qs[r], recon["k"][r], recon["v"][r]) - ref[r]) ** 2))
                  for r in range(rows))
        den = sum(float(np.sum(ref[r] ** 2)) for r in range(rows))
        res["attn"] = math.sqrt(num / den)
        out.append(res)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="qwen3_8b_b16_t8k")
    ap.add_argument("--rows", type=int, default=48)
    ap.add_argument("--tokens", type=int, default=512)
    ap.add_argument("--bits", type=float, default=2.26)
    args = ap.parse_args()
    res = sweep(args.workload, args.rows, args.tokens, args.bits)
    print("| rate offset (bit/value) | stream | design entropy | symbols drifted | containers drifted | "
          "MSE of rotated coords | rel. error of x | attention rel. RMS error |")
    print("|---|---|---|---|---|---|---|---|")
    for r in res:
        for s in ("k", "v"):
            d = r[s]
            print("| %+.2f | %s | %.3f | %.2f %% | %.1f %% | %.4f | %.4f | %.4f |" % (
                r["offset"], s.upper(), d["entropy"], 100 * d["drift_syms"], 100 * d["drift_cont"],
                d["mse_u"], d["rel_x"], r["attn"]))


if __name__ == "__main__":
    main()
