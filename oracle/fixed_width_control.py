"""Fixed width against entropy coding at the same bytes (TEST INFRASTRUCTURE).

[news] "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits", "Why Fixed
Width Is a Ceiling": a fixed-width code spends the same bits on every
coordinate, while the rotated coordinates are close to N(0,1), so most of them
sit near zero; entropy coding the quantised symbols spends fewer bits there
and can afford finer levels in the same bytes ("Drift: Bending Variable Back
to Fixed" gives 8 levels for K and 6 for V at 2.26 bits per value).

This module measures that claim on the synthetic workloads with the oracle
only (CPU, fp64 where it matters): D-Quant containers (rANS + drift, and with
the rate-distortion fill of drift mode 1) against a
fixed-width control that quantises the same rotated, normalised coordinates
with the Gaussian Lloyd-Max quantiser of 2^b levels at b bits per value (b = 2:
4 levels, 32 bytes of codes + the 2-byte fp16 norm = 34 bytes, within the
36-byte D-Quant container). Reported per stream and budget: the mean squared
error of the rotated coordinates, the relative error of the reconstructed
vectors, and the relative RMS error of decode-attention outputs against fp64
attention over the unquantised K and V.

    python -m oracle.fixed_width_control [--rows 64] [--tokens 512]
"""
from __future__ import annotations

import argparse
import math
import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from oracle import oracle as o  # noqa: E402


def rotate_all(x: np.ndarray, sg: np.ndarray):
    """u [N,128] (rotated, normalised, fp32) and fp16 norm bits [N] of rows x."""
    n = x.shape[0]
    u = np.zeros((n, o.D), np.float32)
    nh = np.zeros(n, np.uint16)
    for i in range(n):
        u[i], nh[i], _ = o.rotate_normalize(x[i], sg)
    return u, nh


def fixed_width_codes(u: np.ndarray, bits: int):
    """Gaussian Lloyd-Max quantiser with 2^bits levels: symbols (count of
    thresholds <= u, as the D-Quant quantiser) and the levels."""
    y, t, _ = o.lloyd_max(2 ** bits)
    syms = np.searchsorted(t, u, side="right")
    return syms, y


def reconstruct(y_hat: np.ndarray, norm16: np.ndarray, sg: np.ndarray) -> np.ndarray:
    """x_hat = ||x|| * D * (H * y_hat) / 128 in fp64 (rows of y_hat)."""
    z = y_hat.astype(np.float64) @ o.hadamard(o.D)
    return o.f16_to_f64(norm16)[:, None] * sg.astype(np.float64) * z / o.D


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(128)) v in fp64 for query rows q [G,128]."""
    a = (q @ k.T) / math.sqrt(o.D)
    a -= a.max(axis=1, keepdims=True)
    p = np.exp(a)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


def measure(workload: str = "qwen3_8b_b16_t8k", rows: int = 64, tokens: int = 512,
            budgets=(1.96, 2.26, 3.0), fixed_bits=(2,), drift_modes=(0, 1)):
    """Rows of results: one per (stream, coder, budget); D-Quant once per
    drift mode (0: drift only; 1: drift, then the rate-distortion fill)."""
    from decode_attention_dq_b200 import synth

    w = synth.WORKLOADS[workload]
    G = w.Hq // w.Hkv
    picks = [(b % w.B, (b * 3) % w.Hkv) for b in range(rows)]
    sg_all = o.signs(0, w.Hkv)
    data = {}
    for stream in ("k", "v"):
        xs = [synth.kv_row(w, stream, b, h, n=tokens) for b, h in picks]
        data[stream] = xs
    qs = [synth.q_rows(w, b)[h * G:(h + 1) * G].astype(np.float64) for b, h in picks]
    ref_out = [attention(qs[r], data["k"][r].astype(np.float64), data["v"][r].astype(np.float64))
               for r in range(rows)]

    def stats_for(recon):  # recon[stream][r] -> x_hat rows
        out = []
        for r in range(rows):
            out.append(attention(qs[r], recon["k"][r], recon["v"][r]))
        err = math.sqrt(sum(float(np.sum((out[r] - ref_out[r]) ** 2)) for r in range(rows)) /
                        sum(float(np.sum(ref_out[r] ** 2)) for r in range(rows)))
        return err

    results = []
    rotated = {s: [rotate_all(data[s][r], sg_all[picks[r][1]]) for r in range(rows)] for s in ("k", "v")}

    # D-Quant at each budget (same budget for K and V) and drift mode.
    for bits, mode in [(b_, m_) for b_ in budgets for m_ in drift_modes]:
        C = o.container_bytes(bits)
        tab = o.Tables(w.Hkv, k_container_bytes=C, v_container_bytes=C, drift_mode=mode)
        recon = {}
        for s in ("k", "v"):
            st = tab.k if s == "k" else tab.v
            mse_u, rel_x, moved = 0.0, 0.0, 0
            recon[s] = []
            for r in range(rows):
                h = picks[r][1]
                x = data[s][r]
                cont, syms, stt, bad = o.encode_vectors(st, tab.signs, x, np.full(x.shape[0], h, np.int32),
                                                        drift_mode=mode)
                assert bad == 0
                u, _ = rotated[s][r]
                y_hat = st.yf.astype(np.float64)[syms.astype(np.int64)]
                mse_u += float(np.sum((u.astype(np.float64) - y_hat) ** 2))
                dsyms, dn, status = o.decode_containers(st, cont)
                assert not status.any()
                xh = reconstruct(st.yf.astype(np.float64)[dsyms.astype(np.int64)], dn, tab.signs[h])
                recon[s].append(xh)
                rel_x += float(np.sum((xh - x) ** 2)) / float(np.sum(x.astype(np.float64) ** 2))
                moved += stt.syms_drifted
            n = rows * tokens
            results.append(dict(stream=s.upper(),
                                coder="D-Quant %d levels (rANS + drift%s)" % (st.n, " + RD fill" if mode else ""),
                                bits=bits, bytes=C, mse_u=mse_u / (n * o.D), rel_x=rel_x / rows,
                                drift=moved / (n * o.D)))
        err = stats_for(recon)
        for rrow in results[-2:]:
            rrow["attn"] = err

    # Fixed-width control.
    for b in fixed_bits:
        recon = {}
        for s in ("k", "v"):
            mse_u, rel_x = 0.0, 0.0
            recon[s] = []
            for r in range(rows):
                h = picks[r][1]
                x = data[s][r]
                u, nh = rotated[s][r]
                syms, y = fixed_width_codes(u, b)
                y_hat = y[syms]
                mse_u += float(np.sum((u.astype(np.float64) - y_hat) ** 2))
                xh = reconstruct(y_hat, nh, sg_all[h])
                recon[s].append(xh)
                rel_x += float(np.sum((xh - x) ** 2)) / float(np.sum(x.astype(np.float64) ** 2))
            n = rows * tokens
            results.append(dict(stream=s.upper(), coder="fixed width, Lloyd-Max %d levels" % (2 ** b),
                                bits=b + 16 / o.D, bytes=(o.D * b + 7) // 8 + 2, mse_u=mse_u / (n * o.D),
                                rel_x=rel_x / rows, drift=0.0))
        err = stats_for(recon)
        for rrow in results[-2:]:
            rrow["attn"] = err
    return results


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="qwen3_8b_b16_t8k")
    ap.add_argument("--rows", type=int, default=64)
    ap.add_argument("--tokens", type=int, default=512)
    args = ap.parse_args()
    res = measure(args.workload, args.rows, args.tokens)
    print("| stream | coder | bit/value | bytes | MSE of rotated coords | rel. error of x | "
          "attention rel. RMS error | symbols drifted |")
    print("|---|---|---|---|---|---|---|---|")
    for r in res:
        print("| %s | %s | %.2f | %d | %.4f | %.4f | %.4f | %.3f %% |" % (
            r["stream"], r["coder"], r["bits"], r["bytes"], r["mse_u"], r["rel_x"], r["attn"],
            100 * r["drift"]))


if __name__ == "__main__":
    main()
