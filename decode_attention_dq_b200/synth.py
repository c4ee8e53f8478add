"""Seeded synthetic K/V/q inputs shaped like the D-Quant pages' workloads.

No step of the method lives here: this module only draws random numbers. It
is shared by the tests (to feed both the CUDA path and the CPU oracle the same
inputs) and by bench.py. Every row (sequence b, KV head h) is drawn from its
own numpy PCG64 stream, seeded from (workload seed, stream id, b, h), so any
row can be regenerated on its own, in any process.

Recipes (the pages measure on Qwen3-8B / Llama-3.1-8B activations, which are
not available here; these stand in for them):
  tiny  -- K, V fp32 = N(0,1) x per-channel lognormal(0, 0.5) scales with
           2 channels x 8 (separate scales for K and V); q ~ N(0,1) fp32.
  llm   -- bf16. K = N(0,1) x per-(KV head, channel) lognormal(0, 1) scales,
           4 outlier channels per head x 10, plus a per-(b, h, t) scalar shift
           ~ N(0, 0.2^2) added to every channel; V ~ N(0,1); q ~ N(0,1).
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

_K, _V, _Q, _SCALE, _KNEW, _VNEW, _QSTEP = 1, 2, 3, 4, 5, 6, 7


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hkv: int
    Hq: int
    T: int
    dtype: str            # "f32" or "bf16"
    recipe: str           # "tiny" or "llm"
    seed: int
    k_bits: float = 2.26
    v_bits: float = 2.26
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny_b1_t256": Workload("tiny_b1_t256", 1, 1, 1, 256, "f32", "tiny", 0),
    "qwen3_8b_b16_t8k": Workload("qwen3_8b_b16_t8k", 16, 8, 32, 8192, "bf16", "llm", 1),
    "serve_b128_t8k": Workload("serve_b128_t8k", 128, 8, 32, 8192, "bf16", "llm", 2),
    # a quarter of the serving batch: same kernel and per-sequence work, a
    # cache (151 MB) still larger than L2, small enough for profiler captures
    "serve_b32_t8k": Workload("serve_b32_t8k", 32, 8, 32, 8192, "bf16", "llm", 2),
    "long_b4_t64k": Workload("long_b4_t64k", 4, 8, 32, 65536, "bf16", "llm", 3),
    "long_b4_t128k": Workload("long_b4_t128k", 4, 8, 32, 131072, "bf16", "llm", 3),
    "llama_b32_t32k_1p96": Workload("llama_b32_t32k_1p96", 32, 8, 32, 32768, "bf16", "llm", 4,
                                    1.96, 1.96),
    "llama_b32_t32k_2p26": Workload("llama_b32_t32k_2p26", 32, 8, 32, 32768, "bf16", "llm", 4),
    "llama_b32_t32k_3p0": Workload("llama_b32_t32k_3p0", 32, 8, 32, 32768, "bf16", "llm", 4,
                                   3.0, 3.0),
}


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def channel_scales(w: Workload, stream: str, h: int) -> np.ndarray:
    """Per-channel scale vector [128] for a KV head (K: outliers; V: ones)."""
    if w.recipe == "tiny":
        g = _rng(w.seed, _SCALE, 0 if stream == "k" else 1, h)
        s = np.exp(g.normal(0.0, 0.5, 128))
        s[g.choice(128, 2, replace=False)] *= 8.0
        return s.astype(np.float32)
    if stream == "v":
        return np.ones(128, dtype=np.float32)
    g = _rng(w.seed, _SCALE, 0, h)
    s = np.exp(g.normal(0.0, 1.0, 128))
    s[g.choice(128, 4, replace=False)] *= 10.0
    return s.astype(np.float32)


def _round(a: np.ndarray, w: Workload) -> np.ndarray:
    if w.dtype == "f32":
        return a.astype(np.float32)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def kv_row(w: Workload, stream: str, b: int, h: int, n: int | None = None, step: int | None = None
           ) -> np.ndarray:
    """K or V of one (b, h) row: float32 [n, 128] holding values exactly
    representable in the workload dtype. step=None gives the prefilled context
    (n defaults to w.T); step=s gives the token appended at decode step s."""
    n = w.T if n is None else n
    sid = {"k": _K, "v": _V}[stream] if step is None else {"k": _KNEW, "v": _VNEW}[stream]
    g = _rng(w.seed, sid, b, h) if step is None else _rng(w.seed, sid, b, h, step)
    x = g.standard_normal((n, 128), dtype=np.float32)
    x *= channel_scales(w, stream, h)[None, :]
    if stream == "k" and w.recipe == "llm":
        x += g.normal(0.0, 0.2, (n, 1)).astype(np.float32)
    return _round(x, w)


def q_rows(w: Workload, b: int, step: int = 0) -> np.ndarray:
    """q of one sequence: float32 [Hq, 128] (values in the workload dtype)."""
    g = _rng(w.seed, _QSTEP, b, step)
    return _round(g.standard_normal((w.Hq, 128), dtype=np.float32), w)


def kv_block(w: Workload, stream: str, rows, n: int | None = None, step: int | None = None,
             threads: int = 8) -> np.ndarray:
    """Stack kv_row over a list of (b, h) rows: float32 [len(rows), n, 128]."""
    n = w.T if n is None else n
    out = np.empty((len(rows), n, 128), dtype=np.float32)

    def one(i):
        b, h = rows[i]
        out[i] = kv_row(w, stream, b, h, n=n, step=step)

    if threads > 1 and len(rows) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(len(rows))))
    else:
        for i in range(len(rows)):
            one(i)
    return out


def q_block(w: Workload, step: int = 0) -> np.ndarray:
    """q for the whole batch: float32 [B, Hq, 128]."""
    return np.stack([q_rows(w, b, step) for b in range(w.B)])


def q_chunk(w: Workload, n_q: int, first_step: int = 0) -> np.ndarray:
    """Queries of a prompt chunk: float32 [B, n_q, Hq, 128]; query token i of
    sequence b is q_rows(w, b, first_step + i)."""
    return np.stack([np.stack([q_rows(w, b, first_step + i) for i in range(n_q)]) for b in range(w.B)])


def scaled(w: Workload, **changes) -> Workload:
    """The same recipe at other sizes (for tests at sizes the oracle finishes)."""
    d = dict(name=w.name + "_small", B=w.B, Hkv=w.Hkv, Hq=w.Hq, T=w.T, dtype=w.dtype,
             recipe=w.recipe, seed=w.seed, k_bits=w.k_bits, v_bits=w.v_bits)
    d.update(changes)
    return Workload(**d)


def prefill_cache(tab, w: Workload, kcache, vcache, n_tokens: int, seqs_per_call: int = 8,
                  threads: int = 16, stats=None, timings: list | None = None, page_table=None):
    """Fill positions [0, n_tokens) of every sequence's cache with the
    workload's seeded K/V, appended through dq_append_kv in batches of
    sequences (the inputs are drawn on the host, then copied to the device).
    With `timings`, each dq_append_kv call is bracketed by CUDA events on the
    current stream and (start event, end event, vectors per stream) is
    appended to the list; the first call is then made twice and only its
    second run is timed (the first also loads the kernels). With `page_table`
    (int32 [B, max_pages]) kcache and vcache are page pools and the tokens go
    through dq_append_kv_paged."""
    from ._native import dq_append_kv, dq_append_kv_paged  # local import: synth itself needs no GPU

    def append(kt, vt, start, b0, b1, st):
        if page_table is None:
            dq_append_kv(tab, kt, vt, start, kcache[b0:b1], vcache[b0:b1], stats=st)
        else:
            dq_append_kv_paged(tab, kt, vt, start, kcache, vcache, page_table[b0:b1], stats=st)

    for b0 in range(0, w.B, seqs_per_call):
        b1 = min(w.B, b0 + seqs_per_call)
        rows = [(b, h) for b in range(b0, b1) for h in range(w.Hkv)]
        K = kv_block(w, "k", rows, n=n_tokens, threads=threads)
        V = kv_block(w, "v", rows, n=n_tokens, threads=threads)
        kt = torch.from_numpy(K).to(device=kcache.device, dtype=w.torch_dtype).view(
            b1 - b0, w.Hkv, n_tokens, 128)
        vt = torch.from_numpy(V).to(device=kcache.device, dtype=w.torch_dtype).view(
            b1 - b0, w.Hkv, n_tokens, 128)
        start = torch.zeros(b1 - b0, dtype=torch.int32, device=kcache.device)
        if timings is not None:
            if b0 == 0:  # untimed first run (same inputs, same containers)
                append(kt, vt, start, b0, b1, None)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
        append(kt, vt, start, b0, b1, stats)
        if timings is not None:
            e1.record()
            timings.append((e0, e1, (b1 - b0) * w.Hkv * n_tokens))
