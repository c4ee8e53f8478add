"""ctypes wrapper around the plain-C oracle plus the fp64 attention oracle.

TEST INFRASTRUCTURE: only tests/, ``__graft_entry__.smoke()`` and bench.py's
cpu_baseline/reference legs may import this module. It shares nothing with the
product library.

Sources: [news] "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits",
sections "Why Fixed Width Is a Ceiling" and "Drift: Bending Variable Back to
Fixed"; [abstract] "D-Quant: Driftable Entropy Coding for KV Cache
Quantization", Abstract. The attention over the compressed cache
(``attention_fp64``) is textbook softmax attention over the dequantised keys
and values: the pages put dequantisation "within attention kernels"
([abstract]) and say nothing else about the attention itself.
"""
from __future__ import annotations

import ctypes as C
import math
from dataclasses import dataclass

import numpy as np

from . import build as _build

D = 128
MAX_LEVELS = 16
HEADER_BYTES = 5


class _Stream(C.Structure):
    _fields_ = [
        ("n_levels", C.c_int32),
        ("container_bytes", C.c_int32),
        ("payload_bytes", C.c_int32),
        ("is_lloyd_max", C.c_int32),
        ("rate", C.c_double),
        ("lam", C.c_double),
        ("entropy", C.c_double),
        ("mse", C.c_double),
        ("y", C.c_double * MAX_LEVELS),
        ("t", C.c_double * MAX_LEVELS),
        ("p", C.c_double * MAX_LEVELS),
        ("yf", C.c_float * MAX_LEVELS),
        ("tf", C.c_float * MAX_LEVELS),
        ("cost", C.c_float * MAX_LEVELS),
        ("freq", C.c_uint32 * MAX_LEVELS),
        ("cum", C.c_uint32 * (MAX_LEVELS + 1)),
    ]


class _Stats(C.Structure):
    _fields_ = [
        ("syms_drifted", C.c_uint64),
        ("cont_drifted", C.c_uint64),
        ("overflow_fallbacks", C.c_uint64),
        ("nonfinite_inputs", C.c_uint64),
        ("syms_filled", C.c_uint64),
    ]


_lib = None


def load():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        lib = C.CDLL(path)
        P = C.POINTER
        vp = C.c_void_p
        lib.dqo_lloyd_max.argtypes = [C.c_int, vp, vp, vp, P(C.c_int)]
        lib.dqo_ecsq.argtypes = [C.c_int, C.c_double, vp, vp, vp, vp, P(C.c_int)]
        lib.dqo_entropy.argtypes = [C.c_int, vp]
        lib.dqo_entropy.restype = C.c_double
        lib.dqo_int_freqs.argtypes = [C.c_int, vp, vp]
        lib.dqo_container_bytes.argtypes = [C.c_double]
        lib.dqo_build_stream.argtypes = [C.c_int, C.c_int, C.c_double, P(_Stream)]
        lib.dqo_splitmix64_next.argtypes = [P(C.c_uint64)]
        lib.dqo_splitmix64_next.restype = C.c_uint64
        lib.dqo_signs.argtypes = [C.c_uint64, C.c_int, vp]
        lib.dqo_f32_to_f16_rn.argtypes = [C.c_float]
        lib.dqo_f32_to_f16_rn.restype = C.c_uint16
        lib.dqo_f16_to_f32.argtypes = [C.c_uint16]
        lib.dqo_f16_to_f32.restype = C.c_float
        lib.dqo_bf16_to_f32.argtypes = [C.c_uint16]
        lib.dqo_bf16_to_f32.restype = C.c_float
        lib.dqo_wht_f32.argtypes = [vp, C.c_int]
        lib.dqo_rotate_normalize.argtypes = [vp, vp, vp, P(C.c_uint16)]
        lib.dqo_quantize.argtypes = [P(_Stream), vp, C.c_int, vp]
        lib.dqo_rans_encode.argtypes = [P(_Stream), vp, C.c_int, vp, C.c_int]
        lib.dqo_drift_fit.argtypes = [P(_Stream), vp, vp, C.c_int, C.c_int,
                                      P(C.c_int), vp, P(C.c_int)]
        lib.dqo_encode_vector.argtypes = [P(_Stream), vp, vp, vp, vp, P(_Stats)]
        lib.dqo_rans_decode.argtypes = [P(_Stream), vp, C.c_int, vp, C.c_int,
                                        P(C.c_uint32), P(C.c_int)]
        lib.dqo_decode_container.argtypes = [P(_Stream), vp, vp, P(C.c_uint16)]
        lib.dqo_encode_batch.argtypes = [P(_Stream), vp, vp, vp, C.c_int64, vp,
                                         vp, P(_Stats)]
        lib.dqo_decode_batch.argtypes = [P(_Stream), vp, C.c_int64, vp, vp, vp]
        lib.dqo_encode_batch_mode.argtypes = [P(_Stream), vp, vp, vp, C.c_int64, vp,
                                              vp, P(_Stats), C.c_int]
        lib.dqo_rd_fill.argtypes = [P(_Stream), vp, vp, vp, C.c_int, C.c_int, P(C.c_int)]
        lib.dqo_decode_batch.restype = C.c_int64
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


@dataclass
class Stats:
    syms_drifted: int = 0
    cont_drifted: int = 0
    overflow_fallbacks: int = 0
    nonfinite_inputs: int = 0
    syms_filled: int = 0

    def add(self, s: _Stats):
        self.syms_drifted += int(s.syms_drifted)
        self.cont_drifted += int(s.cont_drifted)
        self.overflow_fallbacks += int(s.overflow_fallbacks)
        self.nonfinite_inputs += int(s.nonfinite_inputs)
        self.syms_filled += int(s.syms_filled)


class Stream:
    """One stream's table (K or V), as the oracle designs it."""

    def __init__(self, n_levels: int, container_bytes: int, rate_offset: float = 0.0):
        self._s = _Stream()
        rc = load().dqo_build_stream(n_levels, container_bytes, rate_offset,
                                     C.byref(self._s))
        if rc != 0:
            raise ValueError("oracle table build failed (rc=%d) for n=%d C=%d"
                             % (rc, n_levels, container_bytes))
        n = n_levels
        s = self._s
        self.n = n
        self.container_bytes = int(s.container_bytes)
        self.payload_bytes = int(s.payload_bytes)
        self.is_lloyd_max = bool(s.is_lloyd_max)
        self.rate = float(s.rate)
        self.lam = float(s.lam)
        self.entropy = float(s.entropy)
        self.mse = float(s.mse)
        self.y = np.array(s.y[:n], dtype=np.float64)
        self.t = np.array(s.t[:n - 1], dtype=np.float64)
        self.p = np.array(s.p[:n], dtype=np.float64)
        self.yf = np.array(s.yf[:n], dtype=np.float32)
        self.tf = np.array(s.tf[:n - 1], dtype=np.float32)
        self.cost = np.array(s.cost[:n], dtype=np.float32)
        self.freq = np.array(s.freq[:n], dtype=np.uint32)
        self.cum = np.array(s.cum[:n + 1], dtype=np.uint32)

    @property
    def ref(self):
        return C.byref(self._s)


def container_bytes(bits_per_value: float) -> int:
    return int(load().dqo_container_bytes(float(bits_per_value)))


def lloyd_max(n: int):
    y = np.zeros(MAX_LEVELS); t = np.zeros(MAX_LEVELS); p = np.zeros(MAX_LEVELS)
    it = C.c_int(0)
    rc = load().dqo_lloyd_max(n, _ptr(y), _ptr(t), _ptr(p), C.byref(it))
    assert rc == 0
    return y[:n].copy(), t[:n - 1].copy(), p[:n].copy()


def ecsq(n: int, lam: float, y_init: np.ndarray):
    yi = np.zeros(MAX_LEVELS); yi[:n] = y_init
    y = np.zeros(MAX_LEVELS); t = np.zeros(MAX_LEVELS); p = np.zeros(MAX_LEVELS)
    it = C.c_int(0)
    rc = load().dqo_ecsq(n, float(lam), _ptr(yi), _ptr(y), _ptr(t), _ptr(p), C.byref(it))
    if rc != 0:
        return None
    return y[:n].copy(), t[:n - 1].copy(), p[:n].copy()


def int_freqs(p: np.ndarray) -> np.ndarray:
    n = len(p)
    pp = np.zeros(MAX_LEVELS); pp[:n] = p
    f = np.zeros(MAX_LEVELS, dtype=np.uint32)
    rc = load().dqo_int_freqs(n, _ptr(pp), _ptr(f))
    assert rc == 0
    return f[:n].copy()


def splitmix64(seed: int, count: int):
    st = C.c_uint64(seed)
    return [int(load().dqo_splitmix64_next(C.byref(st))) for _ in range(count)]


def signs(seed: int, n_heads: int) -> np.ndarray:
    out = np.zeros((n_heads, D), dtype=np.int8)
    for h in range(n_heads):
        row = np.zeros(D, dtype=np.int8)
        load().dqo_signs(C.c_uint64(seed), h, _ptr(row))
        out[h] = row
    return out


def f32_to_f16_bits(v: float) -> int:
    return int(load().dqo_f32_to_f16_rn(C.c_float(v)))


def f16_bits_to_f32(h: int) -> float:
    return float(load().dqo_f16_to_f32(C.c_uint16(h)))


def wht_f32(z: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(z, dtype=np.float32).copy()
    load().dqo_wht_f32(_ptr(a), a.shape[0])
    return a


def rotate_normalize(x: np.ndarray, sg: np.ndarray):
    x = np.ascontiguousarray(x, dtype=np.float32)
    sg = np.ascontiguousarray(sg, dtype=np.int8)
    u = np.zeros(D, dtype=np.float32)
    nh = C.c_uint16(0)
    nf = load().dqo_rotate_normalize(_ptr(x), _ptr(sg), _ptr(u), C.byref(nh))
    return u, int(nh.value), int(nf)


def quantize(st: Stream, u: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(u, dtype=np.float32)
    q = np.zeros(u.shape[0], dtype=np.uint8)
    load().dqo_quantize(st.ref, _ptr(u), u.shape[0], _ptr(q))
    return q


def rans_encode(st: Stream, q: np.ndarray, cap: int | None = None):
    """Returns (length, bytes or None)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    n = q.shape[0]
    if cap is None:
        cap = 2 * n + 8
    out = np.zeros(cap, dtype=np.uint8)
    ln = load().dqo_rans_encode(st.ref, _ptr(q), n, _ptr(out), cap)
    return ln, (out[:ln].copy() if ln <= cap else None)


def rans_decode(st: Stream, buf: np.ndarray, n: int):
    buf = np.ascontiguousarray(buf, dtype=np.uint8)
    q = np.zeros(n, dtype=np.uint8)
    xf = C.c_uint32(0)
    used = C.c_int(0)
    rc = load().dqo_rans_decode(st.ref, _ptr(buf), buf.shape[0], _ptr(q), n,
                                C.byref(xf), C.byref(used))
    return rc, q, int(xf.value), int(used.value)


def drift_fit(st: Stream, u: np.ndarray, q: np.ndarray, budget: int):
    u = np.ascontiguousarray(u, dtype=np.float32)
    q = np.ascontiguousarray(q, dtype=np.uint8).copy()
    n = q.shape[0]
    moved = np.zeros(n, dtype=np.uint8)
    moves = C.c_int(0)
    fb = C.c_int(0)
    ln = load().dqo_drift_fit(st.ref, _ptr(u), _ptr(q), n, budget, C.byref(moves),
                              _ptr(moved), C.byref(fb))
    return ln, q, moved.astype(bool), int(moves.value), bool(fb.value)


def rd_fill(st: Stream, u: np.ndarray, q0: np.ndarray, q: np.ndarray, budget: int):
    """Rate-distortion fill of one symbol string (drift mode 1): returns
    (length, filled symbols, number of symbols moved up)."""
    u = np.ascontiguousarray(u, dtype=np.float32)
    q0 = np.ascontiguousarray(q0, dtype=np.uint8)
    q = np.ascontiguousarray(q, dtype=np.uint8).copy()
    ups = C.c_int(0)
    ln = load().dqo_rd_fill(st.ref, _ptr(u), _ptr(q0), _ptr(q), q.shape[0], budget, C.byref(ups))
    return ln, q, int(ups.value)


def encode_vectors(st: Stream, sg_per_head: np.ndarray, x: np.ndarray,
                   head_of: np.ndarray, drift_mode: int = 0):
    """Encode N vectors x[N,128] (float32) with sign rows sg_per_head[head_of[v]].
    drift_mode 0: drift only; 1: drift, then the rate-distortion fill.

    Returns (containers [N,C] uint8, symbols [N,128] uint8, Stats, n_bad)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n = x.shape[0]
    sg = np.ascontiguousarray(sg_per_head, dtype=np.int8)
    ho = np.ascontiguousarray(head_of, dtype=np.int32)
    cont = np.zeros((n, st.container_bytes), dtype=np.uint8)
    syms = np.zeros((n, D), dtype=np.uint8)
    s = _Stats()
    bad = load().dqo_encode_batch_mode(st.ref, _ptr(sg), _ptr(x), _ptr(ho), n,
                                       _ptr(cont), _ptr(syms), C.byref(s), int(drift_mode))
    stats = Stats()
    stats.add(s)
    return cont, syms, stats, int(bad)


def decode_containers(st: Stream, cont: np.ndarray):
    """Decode containers [N,C] -> (symbols [N,128], norm16 [N], status [N])."""
    cont = np.ascontiguousarray(cont, dtype=np.uint8)
    n = cont.shape[0]
    syms = np.zeros((n, D), dtype=np.uint8)
    nh = np.zeros(n, dtype=np.uint16)
    status = np.zeros(n, dtype=np.int32)
    load().dqo_decode_batch(st.ref, _ptr(cont), n, _ptr(syms), _ptr(nh), _ptr(status))
    return syms, nh, status


class Tables:
    """K and V stream tables plus per-head rotation signs."""

    def __init__(self, n_kv_heads: int, k_levels: int = 8, v_levels: int = 6,
                 k_container_bytes: int = 36, v_container_bytes: int = 36,
                 sign_seed: int = 0, k_rate_offset: float = 0.0,
                 v_rate_offset: float = 0.0, drift_mode: int = 0):
        self.drift_mode = drift_mode
        self.k = Stream(k_levels, k_container_bytes, k_rate_offset)
        self.v = Stream(v_levels, v_container_bytes, v_rate_offset)
        self.n_kv_heads = n_kv_heads
        self.sign_seed = sign_seed
        self.signs = signs(sign_seed, n_kv_heads)


def encode_cache(tab: Tables, K: np.ndarray, V: np.ndarray):
    """Encode K, V [B,Hkv,T,128] (float32 values) into caches [B,Hkv,T,C]."""
    B, H, T, d = K.shape
    assert d == D and V.shape == K.shape and H == tab.n_kv_heads
    head_of = np.broadcast_to(np.arange(H, dtype=np.int32)[None, :, None], (B, H, T)).reshape(-1)
    kc, ks, kst, kbad = encode_vectors(tab.k, tab.signs, K.reshape(-1, D), head_of, tab.drift_mode)
    vc, vs, vst, vbad = encode_vectors(tab.v, tab.signs, V.reshape(-1, D), head_of, tab.drift_mode)
    assert kbad == 0 and vbad == 0
    return (kc.reshape(B, H, T, -1), vc.reshape(B, H, T, -1),
            ks.reshape(B, H, T, D), vs.reshape(B, H, T, D), kst, vst)


def hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix (unnormalised), fp64."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def dequantize(st: Stream, syms: np.ndarray, norm16: np.ndarray, sg: np.ndarray) -> np.ndarray:
    """x_hat = ||x|| * D * (H * y_hat) / 128 in fp64, with y_hat = y[symbol]
    (the inverse of E1-E3: H H = 128 I and D D = I)."""
    y = st.yf.astype(np.float64)[np.asarray(syms, dtype=np.int64)]
    z = y @ hadamard(D)  # H symmetric
    nrm = f16_to_f64(norm16)
    return nrm[..., None] * sg.astype(np.float64) * z / D


def attention_fp64(tab: Tables, q: np.ndarray, kcache: np.ndarray, vcache: np.ndarray,
                   seq_lens, sm_scale: float | None = None, rows=None) -> np.ndarray:
    """Textbook softmax attention in fp64 over the dequantised cache.

    q [B,Hq,128]; caches [B,Hkv,T_cap,C]; query head hq reads KV head
    hq // (Hq/Hkv). Returns out [B,Hq,128]; a sequence of length 0 gives 0.
    ``rows`` optionally limits the work to a list of (b, h_kv) pairs (other
    outputs are left as NaN)."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = kcache.shape[1]
    G = Hq // Hkv
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    out = np.full((B, Hq, D), np.nan)
    if rows is None:
        rows = [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in rows:
        T = int(seq_lens[b])
        if T == 0:
            out[b, h * G:(h + 1) * G] = 0.0
            continue
        ks, kn, kstat = decode_containers(tab.k, kcache[b, h, :T])
        vs, vn, vstat = decode_containers(tab.v, vcache[b, h, :T])
        assert not kstat.any() and not vstat.any(), "corrupt container in oracle input"
        kh = dequantize(tab.k, ks, kn, tab.signs[h])
        vh = dequantize(tab.v, vs, vn, tab.signs[h])
        for g in range(G):
            a = sm_scale * (kh @ q[b, h * G + g])
            a = a - a.max()
            p = np.exp(a)
            p /= p.sum()
            out[b, h * G + g] = p @ vh
    return out


def attention_prefill_fp64(tab: Tables, q: np.ndarray, kcache: np.ndarray, vcache: np.ndarray,
                           q_start, sm_scale: float | None = None, rows=None) -> np.ndarray:
    """Causal attention of a prompt chunk over the dequantised cache, fp64.

    [news] "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits", "The
    Numbers": long prompts are processed chunk by chunk; the chunk's own K
    and V are in the cache before it attends. q [B, n_q, Hq, 128]; query
    token i of sequence b sits at position p = q_start[b] + i and attends to
    cache positions 0 .. p (softmax(sm_scale q K^T) V over those rows of the
    dequantised cache). A position outside [0, T_cap) gives 0. Query head hq
    reads KV head hq // (Hq / Hkv). ``rows`` optionally limits the work to a
    list of (b, h_kv) pairs (other outputs are NaN)."""
    q = np.asarray(q, dtype=np.float64)
    B, n_q, Hq, _ = q.shape
    Hkv, T_cap = kcache.shape[1], kcache.shape[2]
    G = Hq // Hkv
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    out = np.full((B, n_q, Hq, D), np.nan)
    if rows is None:
        rows = [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in rows:
        pos = int(q_start[b]) + np.arange(n_q)
        ok = (pos >= 0) & (pos < T_cap)
        out[b, :, h * G:(h + 1) * G] = 0.0
        if not ok.any():
            continue
        T = int(pos[ok].max()) + 1
        ks, kn, kstat = decode_containers(tab.k, kcache[b, h, :T])
        vs, vn, vstat = decode_containers(tab.v, vcache[b, h, :T])
        assert not kstat.any() and not vstat.any(), "corrupt container in oracle input"
        kh = dequantize(tab.k, ks, kn, tab.signs[h])
        vh = dequantize(tab.v, vs, vn, tab.signs[h])
        qi = np.nonzero(ok)[0]                            # query tokens with a valid position
        mask = np.arange(T)[None, :] <= pos[qi, None]     # [rows, T]: key t visible to query i
        for g in range(G):
            a = sm_scale * (q[b, qi, h * G + g] @ kh.T)  # [rows, T]
            a = np.where(mask, a, -np.inf)
            a = a - a.max(axis=1, keepdims=True)
            p = np.exp(a)                                  # exp(-inf) = 0 outside the mask
            p /= p.sum(axis=1, keepdims=True)
            out[b, qi, h * G + g] = p @ vh
    return out
