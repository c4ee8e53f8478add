"""Drift with exactly tied move keys, GPU against the oracle.

The rotation is z = H (s * x) with H the unnormalised Sylvester matrix and
H H = 128 I, so x = s * (H v) / 128 gives z = v exactly whenever the
butterfly sums are exact in fp32. Here v takes two or three power-of-two
magnitudes (over 16) with random signs, every partial sum is a small
multiple of 1/2048, and the rotated, normalised coordinates fall into a few
classes of identical |u|. The levels are mirrored, so every coordinate of a
class that sits on the same symbol has the same move key ([news] "D-Quant:
Entropy Coding Meets KV Cache at 2.26 Bits", "Drift: Bending Variable Back
to Fixed": moves go to a cheaper neighbour; the pages do not order equal
keys, and the lowest symbol index goes first). With magnitudes 1 and
3 about 89 % of the containers drift by about 8 moves each, so the ties are
resolved many times per container, across several of the drift kernel's
4-count windows and the warp kernel's 32-count passes. Containers and drift
counts must be bit-identical to the oracle's, for the warp-per-vector path
(small appends), the lane-per-vector path with the drift kernel (large
appends) and the rate-distortion fill (drift mode 1).
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import decode_attention_dq_b200 as dq
from oracle import oracle as o
from tests import _common as cm

_H = scipy.linalg.hadamard(128).astype(np.float64)


def _tied_inputs(tab, B, Hkv, T, mags, probs, seed):
    """K, V [B, Hkv, T, 128] float32 with rotated coordinates in a few exact
    magnitude classes (signs of the oracle's tables)."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(2):
        m = rng.choice(np.asarray(mags, dtype=np.float64) / 16.0, size=(B, Hkv, T, 128), p=probs)
        v = m * rng.choice([-1.0, 1.0], size=m.shape)
        x = (v @ _H.T) / 128.0 * tab.signs.astype(np.float64)[None, :, None, :]
        x32 = x.astype(np.float32)
        assert np.array_equal(x32.astype(np.float64), x)  # exact in fp32
        out.append(x32)
    return out


def _check(lib, ref, K, V, dtype, drift_mode=0):
    stats = dq.new_stats()
    kc, vc = cm.gpu_append_all(lib, K, V, dtype, stats=stats)
    torch.cuda.synchronize()
    # The oracle encodes exactly what the kernels read.
    Kr = torch.from_numpy(K).to(dtype).float().numpy()
    Vr = torch.from_numpy(V).to(dtype).float().numpy()
    rk, rv, _, _, kst, vst = o.encode_cache(ref, Kr, Vr)
    T = K.shape[2]
    np.testing.assert_array_equal(cm.flat(kc)[:, :, :T], rk)
    np.testing.assert_array_equal(cm.flat(vc)[:, :, :T], rv)
    s = dq.stats_dict(stats)
    assert s["k_syms_drifted"] == kst.syms_drifted and s["v_syms_drifted"] == vst.syms_drifted
    assert s["k_cont_drifted"] == kst.cont_drifted and s["v_cont_drifted"] == vst.cont_drifted
    assert s["overflow_fallbacks"] == kst.overflow_fallbacks + vst.overflow_fallbacks
    if drift_mode == 1:
        assert s["k_syms_filled"] == kst.syms_filled and s["v_syms_filled"] == vst.syms_filled
    return kst, vst


def test_construction_gives_exact_magnitude_classes():
    """CPU: the inputs really have two exact |u| classes after the oracle's
    rotation and normalisation."""
    ref = o.Tables(2)
    K, _ = _tied_inputs(ref, 1, 2, 4, (1, 3), (0.6, 0.4), seed=1)
    for h in range(2):
        for t in range(4):
            u, _, _ = o.rotate_normalize(K[0, h, t], ref.signs[h])
            assert len(np.unique(np.abs(u))) == 2


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("mags,probs", [((1, 3), (0.6, 0.4)), ((1, 2, 8), (0.6, 0.3, 0.1))])
def test_tied_keys_warp_kernel(dtype, mags, probs):
    lib, ref = cm.lib_tables(2), o.Tables(2)
    K, V = _tied_inputs(ref, 2, 2, 300, mags, probs, seed=2)
    kst, vst = _check(lib, ref, K, V, dtype)
    assert kst.cont_drifted > 100 and vst.cont_drifted > 100


@pytest.mark.gpu
@pytest.mark.parametrize("mags,probs", [((1, 3), (0.6, 0.4)), ((1, 2, 8), (0.6, 0.3, 0.1))])
def test_tied_keys_lane_and_drift_kernels(mags, probs):
    # Large enough for the lane-per-vector kernel (two full 128-vector CTAs
    # per SM and stream), whose over-long containers go to the drift kernel.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, Hkv = 4, 2
    T = -(-(sms * 128 * 2 + 64) // (B * Hkv))
    lib, ref = cm.lib_tables(Hkv), o.Tables(Hkv)
    K, V = _tied_inputs(ref, B, Hkv, T, mags, probs, seed=3)
    kst, vst = _check(lib, ref, K, V, torch.float32)
    n = B * Hkv * T
    assert kst.cont_drifted > n // 10 and vst.cont_drifted > n // 10


@pytest.mark.gpu
def test_tied_keys_rate_distortion_fill():
    lib = dq.dq_build_tables(n_kv_heads=2, drift_mode=1)
    ref = o.Tables(2, drift_mode=1)
    K, V = _tied_inputs(ref, 2, 2, 200, (1, 2, 8), (0.6, 0.3, 0.1), seed=4)
    kst, vst = _check(lib, ref, K, V, torch.float32, drift_mode=1)
    assert kst.cont_drifted > 50 and kst.syms_filled + vst.syms_filled > 0


@pytest.mark.gpu
def test_tied_keys_rate_distortion_fill_large():
    # The lane-per-vector kernel, then the drift kernel's fill phase.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, Hkv = 4, 2
    T = -(-(sms * 128 * 2 + 64) // (B * Hkv))
    lib = dq.dq_build_tables(n_kv_heads=Hkv, drift_mode=1)
    ref = o.Tables(Hkv, drift_mode=1)
    K, V = _tied_inputs(ref, B, Hkv, T, (1, 2, 8), (0.6, 0.3, 0.1), seed=5)
    kst, vst = _check(lib, ref, K, V, torch.float32, drift_mode=1)
    assert kst.cont_drifted > B * Hkv * T // 10 and kst.syms_filled + vst.syms_filled > 0
