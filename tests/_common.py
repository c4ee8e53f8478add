"""Helpers shared by the GPU parity tests: run the same seeded inputs through
the CUDA path (via the C-ABI binding) and through the CPU oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

import decode_attention_dq_b200 as dq
from decode_attention_dq_b200 import synth
from oracle import oracle as o

ATOL_REL_RMS = 2e-3  # attention parity: max |gpu - oracle| <= 2e-3 * RMS(oracle)


def lib_tables(n_kv_heads, k_bits=2.26, v_bits=2.26, seed=0, k_levels=8, v_levels=6):
    return dq.dq_build_tables(n_kv_heads=n_kv_heads, k_bits_per_value=k_bits,
                              v_bits_per_value=v_bits, sign_seed=seed, k_levels=k_levels,
                              v_levels=v_levels)


def oracle_tables(n_kv_heads, k_bits=2.26, v_bits=2.26, seed=0, k_levels=8, v_levels=6):
    return o.Tables(n_kv_heads, k_levels=k_levels, v_levels=v_levels,
                    k_container_bytes=o.container_bytes(k_bits),
                    v_container_bytes=o.container_bytes(v_bits), sign_seed=seed)


def inputs(w: synth.Workload, T: int | None = None):
    """K, V float32 [B, Hkv, T, 128] and q float32 [B, Hq, 128] for a workload."""
    T = w.T if T is None else T
    rows = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    K = synth.kv_block(w, "k", rows, n=T).reshape(w.B, w.Hkv, T, 128)
    V = synth.kv_block(w, "v", rows, n=T).reshape(w.B, w.Hkv, T, 128)
    q = synth.q_block(w)
    return K, V, q


def t_cap_for(T):
    return max(32, (T + 31) // 32 * 32)


def flat(cache):
    """Flat containers (numpy [B, Hkv, T_cap, C]) of a GPU cache."""
    return dq.containers_of(cache).cpu().numpy()


def gpu_append_all(tab, K, V, dtype, T_cap=None, stats=None, workspace=None):
    """Append all T tokens of K, V (numpy float32) through dq_append_kv."""
    B, H, T, _ = K.shape
    T_cap = t_cap_for(T) if T_cap is None else T_cap
    kt = torch.from_numpy(K).to(device="cuda", dtype=dtype).contiguous()
    vt = torch.from_numpy(V).to(device="cuda", dtype=dtype).contiguous()
    kc = torch.zeros((B, H, T_cap, tab.k.container_bytes), dtype=torch.uint8, device="cuda")
    vc = torch.zeros((B, H, T_cap, tab.v.container_bytes), dtype=torch.uint8, device="cuda")
    start = torch.zeros(B, dtype=torch.int32, device="cuda")
    dq.dq_append_kv(tab, kt, vt, start, kc, vc, stats=stats, workspace=workspace)
    return kc, vc


def gpu_attention(tab, q, kc, vc, seq_lens, T_max=None, q_dtype=torch.float32,
                  out_dtype=torch.float32, stats=None, sm_scale=None):
    B, Hq, _ = q.shape
    Hkv = kc.shape[1]
    seq = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    T_max = int(max(seq_lens)) if T_max is None else T_max
    nbytes = dq.dq_decode_workspace_bytes(tab, B, Hq, Hkv, T_max)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    qt = torch.from_numpy(np.ascontiguousarray(q, dtype=np.float32)).to(device="cuda", dtype=q_dtype)
    out = torch.empty((B, Hq, 128), dtype=out_dtype, device="cuda")
    dq.dq_decode_attention(tab, qt, kc, vc, seq, T_max, out, ws, sm_scale=sm_scale, stats=stats)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def assert_attention_close(got, ref, extra_rel=0.0, what=""):
    ref = np.asarray(ref, dtype=np.float64)
    mask = ~np.isnan(ref)
    rms = math.sqrt(float(np.mean(ref[mask] ** 2)))
    err = float(np.max(np.abs(got[mask] - ref[mask])))
    tol = ATOL_REL_RMS * rms + extra_rel * float(np.max(np.abs(ref[mask])))
    assert err <= tol, "%s max|d|=%.3e tol=%.3e (rms %.3e)" % (what, err, tol, rms)
    return err / rms if rms > 0 else 0.0
