"""CPU checks of the C-ABI boundary (no GPU needed).

libdq.so (and the DQ_CHECKED build, libdq_checked.so) loads and exports
every function include/dq.h declares; the binding's stats fields are the
header's; the host-side table design (dq_design_stream, the same code
dq_build_tables uploads) is byte-identical to the oracle's independently
written design.
"""
import ctypes
import os
import re

import numpy as np
import pytest

from decode_attention_dq_b200 import _native as N
from oracle import oracle as o

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "dq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(dq_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = N.load()
    declared = _declared_functions()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)
    assert set(declared) == set(N.EXPORTED)


def _stats_fields():
    text = open(os.path.join(ROOT, "include", "dq.h")).read()
    body = re.search(r"typedef struct \{([^}]*)\} dq_stats;", text, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    return tuple(re.findall(r"unsigned long long (\w+);", body))


def test_stats_fields_match_the_header():
    # new_stats() allocates one uint64 per STATS_FIELDS entry: the binding's
    # names and order must be the C struct's.
    assert _stats_fields() == N.STATS_FIELDS


def test_checked_library_exports_every_declared_symbol():
    from decode_attention_dq_b200 import build

    path = build.build(checked=True)  # no-op when up to date
    lib = ctypes.CDLL(path)
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_error_strings():
    for code in range(-9, 1):
        assert N.dq_error_string(code)
    assert N.dq_error_string(-100) == "unknown status"


BUDGETS = [(8, 36), (6, 36), (8, 31), (6, 31), (8, 48), (6, 48), (4, 36), (2, 36), (8, 64)]


@pytest.mark.parametrize("n,cb", BUDGETS)
def test_host_design_equals_oracle(n, cb):
    lib = N.dq_design_stream(n, cb)
    ref = o.Stream(n, cb)
    assert lib["freq"] == [int(v) for v in ref.freq]
    assert lib["cum"] == [int(v) for v in ref.cum]
    np.testing.assert_array_equal(np.array(lib["levels"], np.float32), ref.yf)
    np.testing.assert_array_equal(np.array(lib["thresholds"], np.float32), ref.tf)
    np.testing.assert_array_equal(np.array(lib["cost"], np.float32), ref.cost)
    assert lib["lam"] == pytest.approx(ref.lam, abs=1e-12)
    assert lib["entropy"] == pytest.approx(ref.entropy, abs=1e-12)
    assert lib["mse"] == pytest.approx(ref.mse, abs=1e-12)


@pytest.mark.parametrize("off", [-0.1, 0.05, 0.2])
def test_host_design_equals_oracle_with_rate_offsets(off):
    for n in (8, 6):
        lib = N.dq_design_stream(n, 36, off)
        ref = o.Stream(n, 36, off)
        assert lib["freq"] == [int(v) for v in ref.freq]
        np.testing.assert_array_equal(np.array(lib["levels"], np.float32), ref.yf)
        np.testing.assert_array_equal(np.array(lib["thresholds"], np.float32), ref.tf)


def test_host_design_rejects_bad_configs():
    with pytest.raises(N.DqError) as e:
        N.dq_design_stream(8, 12)
    assert e.value.code == -3
    with pytest.raises(N.DqError) as e:
        N.dq_design_stream(7, 36)
    assert e.value.code == -2
    with pytest.raises(N.DqError):
        N.dq_design_stream(10, 36)  # the decoder supports at most 8 levels


def test_argument_errors_are_codes_before_any_device_work():
    # Host-side fault injection: null pointers and invalid configurations
    # come back as error codes from the argument checks, which run before
    # any CUDA call (so this needs no GPU), and size queries without tables
    # return 0.
    lib = N.load()
    vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    null_calls = {
        "dq_append_kv": ([vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, i64, vp, vp],
                         [None, None, None, 0, 1, 1, 1, None, None, None, 32, None, None]),
        "dq_decode_attention": ([vp, vp, i32, vp, vp, vp, i32, i32, i32, i64, i64, f32, vp, i32, vp, sz, vp, vp],
                                [None, None, 0, None, None, None, 1, 4, 1, 32, 32, 0.0, None, 0, None, 0, None, None]),
        "dq_prefill_attention": ([vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i64, f32, vp, i32, vp, sz, vp, vp],
                                 [None, None, 0, None, None, None, 1, 1, 4, 1, 32, 0.0, None, 0, None, 0, None, None]),
        "dq_get_signs": ([vp, vp], [None, None]),
        "dq_build_tables": ([vp, vp], [None, None]),
    }
    for name, (argt, args) in null_calls.items():
        f = getattr(lib, name)
        f.argtypes, f.restype = argt, ctypes.c_int
        assert f(*args) == -1, name  # DQ_ERR_NULL
    for name, argt, args in (("dq_decode_workspace_bytes", [vp, i32, i32, i32, i64], [None, 1, 4, 1, 32]),
                             ("dq_prefill_workspace_bytes", [vp, i32, i32, i64], [None, 1, 1, 32]),
                             ("dq_append_workspace_bytes", [vp, i32, i32, i32], [None, 1, 1, 1])):
        f = getattr(lib, name)
        f.argtypes, f.restype = argt, sz
        assert f(*args) == 0, name
    out = ctypes.c_void_p()
    for fields, code in (({"head_dim": 64}, -2), ({"prob_bits": 11}, -2), ({"k_levels": 9}, -2),
                         ({"n_kv_heads": 0}, -2), ({"k_container_bytes": 8}, -3)):
        cfg = N.DqConfig()
        lib.dq_config_default(ctypes.byref(cfg))
        for k, v in fields.items():
            setattr(cfg, k, v)
        assert lib.dq_build_tables(ctypes.byref(cfg), ctypes.byref(out)) == code, fields
