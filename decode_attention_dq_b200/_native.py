"""ctypes binding of libdq (include/dq.h): the same entry points, argument
marshalling only. PyTorch supplies device memory and streams; every step of
the path runs in libdq's CUDA kernels. There is no CPU fallback: if libdq.so
is missing, loading raises.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# DQ_LIBRARY selects another build of the same ABI (lib/libdq_checked.so:
# the attention kernels also count containers decoded past their bytes).
LIB_PATH = os.environ.get("DQ_LIBRARY") or os.path.join(HERE, "lib", "libdq.so")

DQ_OK = 0
DQ_F32, DQ_BF16 = 0, 1
DQ_STREAM_K, DQ_STREAM_V = 0, 1
STATS_FIELDS = ("k_syms_drifted", "v_syms_drifted", "k_cont_drifted", "v_cont_drifted",
                "overflow_fallbacks", "integrity_errors", "nonfinite_inputs",
                "dropped_writes", "clamped_lengths", "bad_pages", "wait_timeouts",
                "k_syms_filled", "v_syms_filled", "overreads")
EXPORTED = ("dq_config_default", "dq_build_tables", "dq_free_tables", "dq_get_stream_table",
            "dq_get_stream_design", "dq_get_signs", "dq_append_kv", "dq_decode_workspace_bytes",
            "dq_decode_attention", "dq_decode_symbols", "dq_error_string", "dq_last_cuda_error",
            "dq_design_stream", "dq_decode_attention_noalloc", "dq_append_workspace_bytes",
            "dq_append_kv_ws", "dq_append_kv_paged", "dq_decode_attention_paged",
            "dq_prefill_attention", "dq_prefill_attention_paged", "dq_prefill_workspace_bytes")


class DqConfig(C.Structure):
    _fields_ = [
        ("head_dim", C.c_int32), ("k_levels", C.c_int32), ("v_levels", C.c_int32),
        ("prob_bits", C.c_int32), ("k_container_bytes", C.c_int32),
        ("v_container_bytes", C.c_int32), ("k_bits_per_value", C.c_float),
        ("v_bits_per_value", C.c_float), ("n_kv_heads", C.c_int32), ("drift_mode", C.c_int32),
        ("sign_seed", C.c_uint64), ("k_rate_offset", C.c_float), ("v_rate_offset", C.c_float),
    ]


class DqError(RuntimeError):
    def __init__(self, fn, code):
        lib = load()
        msg = lib.dq_error_string(code).decode()
        if code == -8:
            msg += " (cuda error %d)" % lib.dq_last_cuda_error()
        super().__init__("%s failed: %s [%d]" % (fn, msg, code))
        self.code = code


_lib = None


def load():
    """Load libdq.so; raises if it has not been built (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libdq.so not built at %s; run `python -m decode_attention_dq_b200.build`"
                          % LIB_PATH)
    lib = C.CDLL(LIB_PATH)
    vp, i32, i64, P = C.c_void_p, C.c_int32, C.c_int64, C.POINTER
    lib.dq_config_default.argtypes = [P(DqConfig)]
    lib.dq_config_default.restype = None
    lib.dq_build_tables.argtypes = [P(DqConfig), P(vp)]
    lib.dq_free_tables.argtypes = [vp]
    lib.dq_free_tables.restype = None
    lib.dq_get_stream_table.argtypes = [vp, C.c_int, vp, vp, vp, vp, vp, vp, vp]
    lib.dq_get_stream_design.argtypes = [vp, C.c_int, vp, vp, vp, vp, vp]
    lib.dq_get_signs.argtypes = [vp, vp]
    lib.dq_append_kv.argtypes = [vp, vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, vp, vp, vp,
                                 i64, vp, vp]
    lib.dq_append_workspace_bytes.argtypes = [vp, C.c_int, C.c_int, C.c_int]
    lib.dq_append_workspace_bytes.restype = C.c_size_t
    lib.dq_append_kv_ws.argtypes = [vp, vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, vp, vp, vp,
                                    i64, vp, C.c_size_t, vp, vp]
    lib.dq_append_kv_paged.argtypes = [vp, vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, vp, vp, vp,
                                       i64, vp, i64, vp, C.c_size_t, vp, vp]
    lib.dq_decode_attention_paged.argtypes = [vp, vp, C.c_int, vp, vp, i64, vp, i64, vp, C.c_int,
                                              C.c_int, C.c_int, i64, C.c_float, vp, C.c_int, vp,
                                              C.c_size_t, vp, vp]
    lib.dq_decode_workspace_bytes.argtypes = [vp, C.c_int, C.c_int, C.c_int, i64]
    lib.dq_decode_workspace_bytes.restype = C.c_size_t
    lib.dq_decode_attention.argtypes = [vp, vp, C.c_int, vp, vp, vp, C.c_int, C.c_int, C.c_int,
                                        i64, i64, C.c_float, vp, C.c_int, vp, C.c_size_t, vp, vp]
    lib.dq_decode_symbols.argtypes = [vp, vp, C.c_int, i64, vp, vp, vp, vp, vp]
    lib.dq_decode_attention_noalloc.argtypes = [vp, vp, C.c_int, vp, vp, vp, C.c_int, C.c_int,
                                                C.c_int, i64, i64, C.c_float, vp, C.c_int, vp, vp]
    lib.dq_prefill_workspace_bytes.argtypes = [vp, C.c_int, C.c_int, i64]
    lib.dq_prefill_workspace_bytes.restype = C.c_size_t
    lib.dq_prefill_attention.argtypes = [vp, vp, C.c_int, vp, vp, vp, C.c_int, C.c_int, C.c_int,
                                         C.c_int, i64, C.c_float, vp, C.c_int, vp, C.c_size_t, vp, vp]
    lib.dq_prefill_attention_paged.argtypes = [vp, vp, C.c_int, vp, vp, i64, vp, i64, vp, C.c_int,
                                               C.c_int, C.c_int, C.c_int, C.c_float, vp, C.c_int, vp,
                                               C.c_size_t, vp, vp]
    lib.dq_error_string.argtypes = [C.c_int]
    lib.dq_error_string.restype = C.c_char_p
    lib.dq_last_cuda_error.argtypes = []
    lib.dq_design_stream.argtypes = [i32, i32, C.c_double, vp, vp, vp, vp, vp, vp, vp, vp]
    _lib = lib
    return lib


def _check(fn, code):
    if code != DQ_OK:
        raise DqError(fn, code)


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DQ_F32
    if t.dtype == torch.bfloat16:
        return DQ_BF16
    raise TypeError("dtype must be float32 or bfloat16, got %s" % t.dtype)


def dq_config_default(**overrides) -> DqConfig:
    cfg = DqConfig()
    load().dq_config_default(C.byref(cfg))
    for k, v in overrides.items():
        setattr(cfg, k, v)
    return cfg


@dataclass
class StreamTable:
    n_levels: int
    container_bytes: int
    levels: list
    thresholds: list
    freq: list
    cum: list
    cost: list


class Tables:
    """Owns a dq_tables handle (built on the current CUDA device)."""

    def __init__(self, cfg: DqConfig):
        self._h = C.c_void_p()
        _check("dq_build_tables", load().dq_build_tables(C.byref(cfg), C.byref(self._h)))
        self.cfg = cfg
        self.n_kv_heads = cfg.n_kv_heads
        self.k = self.stream_table(DQ_STREAM_K)
        self.v = self.stream_table(DQ_STREAM_V)

    @property
    def handle(self):
        return self._h

    def stream_table(self, kind: int) -> StreamTable:
        n = C.c_int32(); cb = C.c_int32()
        lev = (C.c_float * 8)(); thr = (C.c_float * 7)(); f = (C.c_uint32 * 8)()
        cum = (C.c_uint32 * 9)(); cost = (C.c_float * 8)()
        _check("dq_get_stream_table", load().dq_get_stream_table(
            self._h, kind, C.byref(n), C.byref(cb), lev, thr, f, cum, cost))
        nl = n.value
        return StreamTable(nl, cb.value, list(lev)[:nl], list(thr)[:nl - 1], list(f)[:nl],
                           list(cum)[:nl + 1], list(cost)[:nl])

    def design(self, kind: int) -> dict:
        lam = C.c_double(); ent = C.c_double(); rate = C.c_double(); mse = C.c_double()
        lm = C.c_int32()
        _check("dq_get_stream_design", load().dq_get_stream_design(
            self._h, kind, C.byref(lam), C.byref(ent), C.byref(rate), C.byref(mse), C.byref(lm)))
        return dict(lam=lam.value, entropy=ent.value, rate=rate.value, mse=mse.value,
                    is_lloyd_max=bool(lm.value))

    def signs(self):
        buf = (C.c_int8 * (self.n_kv_heads * 128))()
        _check("dq_get_signs", load().dq_get_signs(self._h, buf))
        return torch.tensor(list(buf), dtype=torch.int8).reshape(self.n_kv_heads, 128)

    def close(self):
        if self._h:
            load().dq_free_tables(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def dq_build_tables(cfg: DqConfig | None = None, **overrides) -> Tables:
    if cfg is None:
        cfg = dq_config_default(**overrides)
    return Tables(cfg)


def new_stats(device=None) -> torch.Tensor:
    """A zeroed device dq_stats (one uint64 per field of STATS_FIELDS)."""
    return torch.zeros(len(STATS_FIELDS), dtype=torch.int64, device=device or "cuda")


def stats_dict(stats: torch.Tensor) -> dict:
    vals = stats.cpu().tolist()
    return dict(zip(STATS_FIELDS, vals))


def new_cache(B: int, Hkv: int, T_cap: int, C: int, device=None) -> torch.Tensor:
    """Zeroed uint8 cache of shape [B, Hkv, T_cap, C] (T_cap a multiple of 32).
    The bytes are in the library's interleaved layout; use containers_of()
    to read flat containers."""
    assert T_cap % 32 == 0, "T_cap must be a multiple of 32"
    return torch.zeros((B, Hkv, T_cap, C), dtype=torch.uint8, device=device or "cuda")


def containers_of(cache: torch.Tensor) -> torch.Tensor:
    """Flat containers [B, Hkv, T_cap, C] (a copy) of a cache whose bytes are in
    the interleaved layout [B][Hkv][T_cap/32][C][32]."""
    B, H, T_cap, C = cache.shape
    return cache.reshape(B, H, T_cap // 32, C, 32).transpose(-1, -2).reshape(B, H, T_cap, C).contiguous()


def dq_append_workspace_bytes(tab: Tables, B: int, Hkv: int, n_new: int) -> int:
    return int(load().dq_append_workspace_bytes(tab.handle, B, Hkv, n_new))


def dq_append_kv(tab: Tables, k: torch.Tensor, v: torch.Tensor, start_pos: torch.Tensor,
                 kcache: torch.Tensor, vcache: torch.Tensor, stats: torch.Tensor | None = None,
                 stream=None, workspace: torch.Tensor | None = None) -> None:
    """k, v: [B, Hkv, n_new, 128] (f32/bf16, contiguous, CUDA); start_pos int32 [B];
    caches uint8 [B, Hkv, T_cap, C] holding the interleaved layout (see new_cache).
    Calls dq_append_kv_ws; without `workspace` one is taken from PyTorch's
    allocator on the caches' device. workspace=False calls dq_append_kv (drift
    inside the encode kernel)."""
    B, Hkv, n_new, d = k.shape
    assert d == 128 and v.shape == k.shape and k.dtype == v.dtype
    assert k.is_contiguous() and v.is_contiguous() and kcache.is_contiguous() and vcache.is_contiguous()
    assert start_pos.dtype == torch.int32 and kcache.dtype == torch.uint8
    T_cap = kcache.shape[2]
    if workspace is False:
        _check("dq_append_kv", load().dq_append_kv(
            tab.handle, _ptr(k), _ptr(v), _dtype_code(k), B, Hkv, n_new, _ptr(start_pos),
            _ptr(kcache), _ptr(vcache), T_cap, _ptr(stats), _stream(stream)))
        return
    if workspace is None:
        nbytes = dq_append_workspace_bytes(tab, B, Hkv, n_new)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=kcache.device)
    _check("dq_append_kv_ws", load().dq_append_kv_ws(
        tab.handle, _ptr(k), _ptr(v), _dtype_code(k), B, Hkv, n_new, _ptr(start_pos),
        _ptr(kcache), _ptr(vcache), T_cap, _ptr(workspace), workspace.numel(), _ptr(stats),
        _stream(stream)))


def dq_decode_workspace_bytes(tab: Tables, B: int, Hq: int, Hkv: int, T_max: int) -> int:
    return int(load().dq_decode_workspace_bytes(tab.handle, B, Hq, Hkv, T_max))


def dq_decode_attention(tab: Tables, q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor,
                        seq_lens: torch.Tensor, T_max: int, out: torch.Tensor,
                        workspace: torch.Tensor, sm_scale: float | None = None,
                        stats: torch.Tensor | None = None, stream=None) -> None:
    """q [B, Hq, 128]; caches uint8 [B, Hkv, T_cap, C]; seq_lens int32 [B];
    out [B, Hq, 128] (f32/bf16); workspace uint8 with dq_decode_workspace_bytes."""
    B, Hq, d = q.shape
    Hkv, T_cap = kcache.shape[1], kcache.shape[2]
    assert d == 128 and q.is_contiguous() and out.is_contiguous() and seq_lens.dtype == torch.int32
    if sm_scale is None:
        sm_scale = 128 ** -0.5
    _check("dq_decode_attention", load().dq_decode_attention(
        tab.handle, _ptr(q), _dtype_code(q), _ptr(kcache), _ptr(vcache), _ptr(seq_lens), B, Hq,
        Hkv, T_cap, T_max, float(sm_scale), _ptr(out), _dtype_code(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(stats), _stream(stream)))


def dq_decode_attention_noalloc(tab: Tables, q: torch.Tensor, kcache: torch.Tensor,
                                vcache: torch.Tensor, seq_lens: torch.Tensor, T_max: int,
                                out: torch.Tensor, sm_scale: float | None = None,
                                stats: torch.Tensor | None = None, stream=None) -> None:
    """dq_decode_attention for callers that cannot allocate: no workspace
    argument; the library's fixed 8 MiB device scratch array is used instead
    (shared by all calls on a device, so overlapping calls must be ordered)."""
    B, Hq, d = q.shape
    Hkv, T_cap = kcache.shape[1], kcache.shape[2]
    assert d == 128 and q.is_contiguous() and out.is_contiguous() and seq_lens.dtype == torch.int32
    if sm_scale is None:
        sm_scale = 128 ** -0.5
    _check("dq_decode_attention_noalloc", load().dq_decode_attention_noalloc(
        tab.handle, _ptr(q), _dtype_code(q), _ptr(kcache), _ptr(vcache), _ptr(seq_lens), B, Hq,
        Hkv, T_cap, T_max, float(sm_scale), _ptr(out), _dtype_code(out), _ptr(stats),
        _stream(stream)))


def dq_prefill_workspace_bytes(tab: Tables, B: int, Hkv: int, T_cap: int) -> int:
    """Bytes of the dq_prefill_attention workspace (decoded tiles)."""
    return int(load().dq_prefill_workspace_bytes(tab.handle, B, Hkv, T_cap))


def _prefill_ws(tab, workspace, B, Hkv, T_cap, device):
    need = dq_prefill_workspace_bytes(tab, B, Hkv, T_cap)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    return workspace


def dq_prefill_attention(tab: Tables, q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor,
                         q_start: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor | None = None,
                         sm_scale: float | None = None, stats: torch.Tensor | None = None,
                         stream=None) -> None:
    """Chunked-prefill attention: q [B, n_q, Hq, 128] (query token i of
    sequence b at position q_start[b] + i, causal over the cache); caches
    uint8 [B, Hkv, T_cap, C]; q_start int32 [B]; out [B, n_q, Hq, 128];
    workspace uint8 of dq_prefill_workspace_bytes (allocated if None)."""
    B, n_q, Hq, d = q.shape
    Hkv, T_cap = kcache.shape[1], kcache.shape[2]
    assert d == 128 and q.is_contiguous() and out.is_contiguous() and q_start.dtype == torch.int32
    assert out.shape == q.shape
    if sm_scale is None:
        sm_scale = 128 ** -0.5
    workspace = _prefill_ws(tab, workspace, B, Hkv, T_cap, q.device)
    _check("dq_prefill_attention", load().dq_prefill_attention(
        tab.handle, _ptr(q), _dtype_code(q), _ptr(kcache), _ptr(vcache), _ptr(q_start), B, n_q, Hq,
        Hkv, T_cap, float(sm_scale), _ptr(out), _dtype_code(out), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(stats), _stream(stream)))


def dq_prefill_attention_paged(tab: Tables, q: torch.Tensor, kpool: torch.Tensor, vpool: torch.Tensor,
                               page_table: torch.Tensor, q_start: torch.Tensor, out: torch.Tensor,
                               workspace: torch.Tensor | None = None, sm_scale: float | None = None,
                               stats: torch.Tensor | None = None, stream=None) -> None:
    """Chunked-prefill attention over page pools (see dq_prefill_attention)."""
    B, n_q, Hq, d = q.shape
    Hkv = kpool.shape[1]
    assert d == 128 and q.is_contiguous() and out.is_contiguous() and q_start.dtype == torch.int32
    assert page_table.dtype == torch.int32 and page_table.is_contiguous() and out.shape == q.shape
    if sm_scale is None:
        sm_scale = 128 ** -0.5
    workspace = _prefill_ws(tab, workspace, B, Hkv, 32 * page_table.shape[1], q.device)
    _check("dq_prefill_attention_paged", load().dq_prefill_attention_paged(
        tab.handle, _ptr(q), _dtype_code(q), _ptr(kpool), _ptr(vpool), kpool.shape[0],
        _ptr(page_table), page_table.shape[1], _ptr(q_start), B, n_q, Hq, Hkv, float(sm_scale),
        _ptr(out), _dtype_code(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(stats), _stream(stream)))


def dq_decode_symbols(tab: Tables, cache: torch.Tensor, kind: int, syms: torch.Tensor,
                      norm16: torch.Tensor, status: torch.Tensor | None = None,
                      stats: torch.Tensor | None = None, stream=None) -> None:
    """cache uint8 [..., C] (flat containers); syms uint8 [n, 128]; norm16 int16/uint16 [n]."""
    n = syms.shape[0]
    _check("dq_decode_symbols", load().dq_decode_symbols(
        tab.handle, _ptr(cache), kind, n, _ptr(syms), _ptr(norm16), _ptr(status), _ptr(stats),
        _stream(stream)))


def dq_error_string(code: int) -> str:
    return load().dq_error_string(code).decode()


def dq_design_stream(n_levels: int, container_bytes: int, rate_offset: float = 0.0) -> dict:
    """Host-only table design of one stream (no device needed)."""
    lev = (C.c_float * 8)(); thr = (C.c_float * 7)(); f = (C.c_uint32 * 8)()
    cum = (C.c_uint32 * 9)(); cost = (C.c_float * 8)()
    lam = C.c_double(); ent = C.c_double(); mse = C.c_double()
    _check("dq_design_stream", load().dq_design_stream(
        n_levels, container_bytes, rate_offset, lev, thr, f, cum, cost, C.byref(lam),
        C.byref(ent), C.byref(mse)))
    n = n_levels
    return dict(levels=list(lev)[:n], thresholds=list(thr)[:n - 1], freq=list(f)[:n],
                cum=list(cum)[:n + 1], cost=list(cost)[:n], lam=lam.value, entropy=ent.value,
                mse=mse.value)


def new_pool(num_pages: int, Hkv: int, C: int, device=None) -> torch.Tensor:
    """Zeroed uint8 page pool [num_pages, Hkv, C, 32] (pages of 32 tokens)."""
    return torch.zeros((num_pages, Hkv, C, 32), dtype=torch.uint8, device=device or "cuda")


def dq_append_kv_paged(tab: Tables, k: torch.Tensor, v: torch.Tensor, start_pos: torch.Tensor,
                       kpool: torch.Tensor, vpool: torch.Tensor, page_table: torch.Tensor,
                       stats: torch.Tensor | None = None, stream=None,
                       workspace: torch.Tensor | None = None) -> None:
    """Append into page pools [num_pages, Hkv, C, 32] through page_table
    int32 [B, max_pages] (see dq_append_kv for the other arguments)."""
    B, Hkv, n_new, d = k.shape
    assert d == 128 and v.shape == k.shape and k.dtype == v.dtype
    assert k.is_contiguous() and v.is_contiguous() and kpool.is_contiguous() and vpool.is_contiguous()
    assert page_table.dtype == torch.int32 and page_table.is_contiguous() and page_table.shape[0] == B
    if workspace is None:
        nbytes = dq_append_workspace_bytes(tab, B, Hkv, n_new)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=kpool.device)
    _check("dq_append_kv_paged", load().dq_append_kv_paged(
        tab.handle, _ptr(k), _ptr(v), _dtype_code(k), B, Hkv, n_new, _ptr(start_pos),
        _ptr(kpool), _ptr(vpool), kpool.shape[0], _ptr(page_table), page_table.shape[1],
        _ptr(workspace), workspace.numel(), _ptr(stats), _stream(stream)))


def dq_decode_attention_paged(tab: Tables, q: torch.Tensor, kpool: torch.Tensor, vpool: torch.Tensor,
                              page_table: torch.Tensor, seq_lens: torch.Tensor, T_max: int,
                              out: torch.Tensor, workspace: torch.Tensor, sm_scale: float | None = None,
                              stats: torch.Tensor | None = None, stream=None) -> None:
    """Decode attention over page pools (see dq_decode_attention)."""
    B, Hq, d = q.shape
    Hkv = kpool.shape[1]
    assert d == 128 and q.is_contiguous() and out.is_contiguous() and seq_lens.dtype == torch.int32
    assert page_table.dtype == torch.int32 and page_table.is_contiguous()
    if sm_scale is None:
        sm_scale = 128 ** -0.5
    _check("dq_decode_attention_paged", load().dq_decode_attention_paged(
        tab.handle, _ptr(q), _dtype_code(q), _ptr(kpool), _ptr(vpool), kpool.shape[0],
        _ptr(page_table), page_table.shape[1], _ptr(seq_lens), B, Hq, Hkv, T_max, float(sm_scale),
        _ptr(out), _dtype_code(out), _ptr(workspace), workspace.numel(), _ptr(stats),
        _stream(stream)))
