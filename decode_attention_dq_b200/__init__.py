"""B200 (sm_100a) implementation of the D-Quant compressed-KV hot path.

The compute runs in libdq (include/dq.h): an append/encode kernel that
rotates, normalises, quantises, rANS-codes and drifts each K/V head vector
into a fixed-size container, a decode-attention kernel (every warp takes
an equal share of all token groups) plus a combine kernel that decode the
containers inside attention, and chunked-prefill attention: a kernel that
decodes each attended 32-token block once into fp16 tiles and one that runs
the scores and P.V on the tensor cores (tcgen05) over those tiles. This package is a
thin ctypes binding (argument marshalling only) plus seeded synthetic inputs.
"""
from ._native import (DQ_BF16, DQ_F32, DQ_STREAM_K, DQ_STREAM_V, DqConfig, DqError,  # noqa: F401
                      Tables, containers_of, dq_append_kv, dq_append_workspace_bytes, dq_build_tables, dq_config_default,
                      dq_append_kv_paged, dq_decode_attention, dq_decode_attention_noalloc,
                      dq_decode_attention_paged, dq_prefill_attention, dq_prefill_attention_paged,
                      dq_prefill_workspace_bytes,
                      new_pool,
                      dq_decode_symbols, dq_decode_workspace_bytes,
                      dq_design_stream, dq_error_string, load, new_cache, new_stats,
                      stats_dict)
