/*
 * dq.h -- C-ABI of libdq, the B200 (sm_100a) D-Quant compressed-KV hot path.
 *
 * D-Quant stores each token's K or V head vector as a fixed-size byte
 * container: the vector is rotated and normalised so its coordinates are close
 * to N(0,1), quantised to a few levels, entropy-coded with rANS, and "drift"
 * moves a few symbols one level to a cheaper neighbour until the stream fits.
 * Attention then decodes the containers inside the attention kernel.
 *   [news] "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits", sections
 *          "Why Fixed Width Is a Ceiling" and "Drift: Bending Variable Back to
 *          Fixed" (8 levels for K, 6 for V at 2.26 bits; no symbol moves more
 *          than one level; analytic, calibration-free probability model).
 *   [abstract] "D-Quant: Driftable Entropy Coding for KV Cache Quantization",
 *          Abstract (fixed-size bitstreams; regular memory access and parallel
 *          dequantisation within attention kernels).
 *
 * Conventions for every entry point:
 *   - Pointers named d_* and the k/v/q/out buffers are DEVICE pointers on the
 *     device the tables were built on; everything else is host memory.
 *   - The caller owns every device buffer (inputs, caches, workspace, stats,
 *     outputs). The library owns only what dq_build_tables allocates.
 *   - Device work is enqueued on `stream` (a cudaStream_t, or NULL for the
 *     legacy default stream) and is asynchronous; nothing is allocated and
 *     nothing synchronises inside dq_append_kv, dq_decode_attention and
 *     dq_decode_symbols.
 *   - Return value: DQ_OK (0) or a negative DQ_ERR_* code. Argument errors are
 *     detected on the host before anything is enqueued. Errors in the data
 *     (a corrupt container, a non-finite input, a position past the cache)
 *     never fault or hang a kernel: they are counted in the caller's dq_stats.
 *   - No C++ exception crosses this boundary. There is no CPU fallback.
 *
 * Layouts (row-major, contiguous):
 *   K/V new tokens   [B][Hkv][n_new][128]           fp32 or bf16
 *   K cache          [B][Hkv][T_cap/32][C_k][32]    uint8, T_cap % 32 == 0
 *   V cache          [B][Hkv][T_cap/32][C_v][32]    uint8, T_cap % 32 == 0
 *   q                [B][Hq][128]                   fp32 or bf16
 *   out              [B][Hq][128]                   fp32 or bf16
 * Query head hq attends with KV head hq / (Hq / Hkv) (grouped-query
 * attention). Container layout: bytes 0-1 the fp16 norm ||x||
 * (little-endian), bytes 2-4 the final rANS state (little-endian), then the
 * renormalisation bytes in decode order, then zero padding to C.
 * Cache layout: the containers of each block of 32 consecutive tokens are
 * byte-interleaved, byte j of token t at index [t / 32][j][t % 32]; a cache
 * is the same number of bytes (T_cap * C per (b, h)) as flat containers. The
 * decoder's 32 lanes (one per token) then read their next bytes from 32
 * different shared-memory banks. dq_decode_symbols takes flat containers.
 */
#ifndef DQ_H
#define DQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum dq_status {
  DQ_OK = 0,
  DQ_ERR_NULL = -1,      /* a required pointer is NULL                       */
  DQ_ERR_CONFIG = -2,    /* head_dim != 128, prob_bits != 12, level counts    */
  DQ_ERR_BUDGET = -3,    /* container too small for the level design          */
  DQ_ERR_SHAPE = -4,     /* B, Hkv, Hq, n_new, T_cap, T_max out of range       */
  DQ_ERR_WORKSPACE = -5, /* workspace smaller than dq_decode_workspace_bytes  */
  DQ_ERR_ALIGN = -6,     /* pointer or T_cap alignment (see each call)        */
  DQ_ERR_DTYPE = -7,     /* unknown dtype code                                */
  DQ_ERR_CUDA = -8,      /* a CUDA runtime call or launch failed              */
  DQ_ERR_DEVICE = -9     /* not an sm_100 device, or not the tables' device   */
};

enum dq_dtype { DQ_F32 = 0, DQ_BF16 = 1 };
enum dq_stream_kind { DQ_STREAM_K = 0, DQ_STREAM_V = 1 };

/* Table configuration. Container size C = round-half-up(bits * 128 / 8)
 * when *_container_bytes is 0 (2.26 -> 36 B, 1.96 -> 31 B, 3.0 -> 48 B). */
typedef struct {
  int32_t head_dim;          /* must be 128                                  */
  int32_t k_levels;          /* even, 2..8 (default 8)                       */
  int32_t v_levels;          /* even, 2..8 (default 6)                       */
  int32_t prob_bits;         /* must be 12 (M = 4096)                        */
  int32_t k_container_bytes; /* 0: derive from k_bits_per_value              */
  int32_t v_container_bytes; /* 0: derive from v_bits_per_value              */
  float k_bits_per_value;    /* default 2.26                                 */
  float v_bits_per_value;    /* default 2.26                                 */
  int32_t n_kv_heads;        /* >= 1; one rotation-sign vector per KV head   */
  int32_t drift_mode;        /* 0: drift only (default); 1: drift, then the  */
                             /* rate-distortion fill (see dq_append_kv)      */
  uint64_t sign_seed;        /* rotation signs: splitmix64 from this seed    */
  float k_rate_offset;       /* added to the target rate, bits/value (0)     */
  float v_rate_offset;       /* added to the target rate, bits/value (0)     */
} dq_config;

/* Device counters, caller-owned (cudaMemset to 0 before use; may be NULL in
 * every call that takes one). Updated with atomics. */
typedef struct {
  unsigned long long k_syms_drifted;     /* K symbols moved by drift         */
  unsigned long long v_syms_drifted;     /* V symbols moved by drift         */
  unsigned long long k_cont_drifted;     /* K containers with >= 1 move      */
  unsigned long long v_cont_drifted;     /* V containers with >= 1 move      */
  unsigned long long overflow_fallbacks; /* containers that took the fallback */
  unsigned long long integrity_errors;   /* corrupt containers decoded       */
  unsigned long long nonfinite_inputs;   /* input vectors treated as zero    */
  unsigned long long dropped_writes;     /* append positions >= T_cap        */
  unsigned long long clamped_lengths;    /* seq_len > T_max or > T_cap       */
  unsigned long long bad_pages;          /* page-table entries out of range  */
  unsigned long long wait_timeouts;      /* bounded in-kernel waits given up */
  unsigned long long k_syms_filled;      /* K symbols moved up by the fill   */
  unsigned long long v_syms_filled;      /* V symbols moved up by the fill   */
  unsigned long long overreads;          /* checked builds only (libdq_checked.so,
                                          * compiled with DQ_CHECKED): containers
                                          * whose decoder inside the attention
                                          * kernels consumed bytes past the
                                          * container (a corrupt container; the
                                          * read stays in the kernel's shared
                                          * memory and is counted, never
                                          * trapped). Always 0 in libdq.so. */
} dq_stats;

typedef struct dq_tables dq_tables; /* opaque, library-owned */

/* Fills *cfg with the defaults: head_dim 128, K 8 levels, V 6 levels,
 * prob_bits 12, 2.26 bits/value for both streams (36-byte containers),
 * n_kv_heads 8, sign_seed 0, no rate offsets. */
void dq_config_default(dq_config *cfg);

/* Designs the K and V tables ([news] "Drift..." 3rd paragraph: the
 * probability model comes analytically from the normal distribution, no
 * calibration data) and uploads them to the CURRENT device.
 *   Level design: Lloyd-Max for N(0,1) when its entropy fits the target rate
 *   r = (8(C-2) - 24)/128 + rate_offset, else the entropy-constrained scalar
 *   quantiser whose entropy equals r. Integer frequencies sum to 4096.
 * Returns DQ_ERR_CONFIG / DQ_ERR_BUDGET / DQ_ERR_DEVICE / DQ_ERR_CUDA on
 * failure (and *out is left NULL). Ownership of *out passes to the caller,
 * who releases it with dq_free_tables. Not asynchronous (one-time set-up). */
int dq_build_tables(const dq_config *cfg, dq_tables **out);

/* Releases the tables (host and device memory). NULL is allowed. Must not be
 * called while work that uses the tables is still running on the device. */
void dq_free_tables(dq_tables *t);

/* Host copies of one stream's table (for inspection and tests). Arrays must
 * hold 8 entries (levels, freq, cost), 9 (cum), 7 (thresholds). Any output
 * pointer may be NULL. */
int dq_get_stream_table(const dq_tables *t, int stream_kind, int32_t *n_levels,
                        int32_t *container_bytes, float *levels,
                        float *thresholds, uint32_t *freq, uint32_t *cum,
                        float *cost);

/* Design summary of one stream: ECSQ multiplier (0 for Lloyd-Max), entropy
 * and target rate in bits/value, design MSE for N(0,1). */
int dq_get_stream_design(const dq_tables *t, int stream_kind, double *lambda,
                         double *entropy, double *rate, double *mse,
                         int32_t *is_lloyd_max);

/* Host-only design of one stream's table (no device is touched): the same
 * design dq_build_tables uploads. Arrays: levels, freq, cost 8 entries;
 * thresholds 7; cum 9 (entries past n_levels are 0, or 4096 for cum). Any
 * output pointer may be NULL. Returns DQ_ERR_CONFIG / DQ_ERR_BUDGET like
 * dq_build_tables. */
int dq_design_stream(int32_t n_levels, int32_t container_bytes, double rate_offset,
                     float *levels, float *thresholds, uint32_t *freq, uint32_t *cum,
                     float *cost, double *lambda, double *entropy, double *mse);

/* Host copy of the rotation signs, int8 [n_kv_heads][128], values +-1. */
int dq_get_signs(const dq_tables *t, int8_t *signs);

/* Appends n_new tokens per sequence ([news] "Drift: Bending Variable Back to
 * Fixed": each token's K or V goes into a fixed-size container; when the
 * entropy-coded stream is too long, a few symbols drift one level to a
 * cheaper neighbour until it fits).
 *   k, v        device, [B][Hkv][n_new][128], dtype DQ_F32 or DQ_BF16,
 *               16-byte aligned
 *   d_start_pos device int32 [B]: token j of sequence b is written at
 *               position d_start_pos[b] + j; positions outside [0, T_cap)
 *               are skipped and counted in dropped_writes
 *   d_kcache    device cache of C_k-byte containers, d_vcache of C_v-byte
 *               ones, both in the interleaved cache layout above;
 *               T_cap % 32 == 0 (else DQ_ERR_ALIGN)
 *   d_stats     device dq_stats or NULL
 *   stream      cudaStream_t
 * Hkv must equal the tables' n_kv_heads. Containers are bit-identical to the
 * reference definition (fp32 rotation/normalisation in a fixed order, greedy
 * drift, zero padding).
 * With drift_mode 1 in the tables' configuration, a rate-distortion fill
 * follows drift ([news] "So What": the rate-distortion toolbox of video
 * coding carries over): a container's unused bytes are spent on accuracy by
 * moving symbols one level up to their nearest level (at most one level from
 * the quantiser's symbol), best error reduction per bit first, each kept
 * only if the exact coded length still fits (none after a fallback). The
 * decoder is unchanged; encoding is about 15 times slower. Large appends
 * with a workspace (dq_append_kv_ws) run the fill in the drift kernel, one
 * launch per stream; the others run a warp per vector. */
int dq_append_kv(const dq_tables *t, const void *k, const void *v, int dtype,
                 int B, int Hkv, int n_new, const int32_t *d_start_pos,
                 uint8_t *d_kcache, uint8_t *d_vcache, int64_t T_cap,
                 dq_stats *d_stats, void *stream);

/* Bytes of the optional workspace of dq_append_kv_ws for these shapes:
 * 256 + 8 * B * Hkv * n_new (a list of the over-long containers of each
 * stream). Returns 0 on invalid shapes. */
size_t dq_append_workspace_bytes(const dq_tables *t, int B, int Hkv, int n_new);

/* dq_append_kv with a caller-provided device workspace (16-byte aligned, at
 * least dq_append_workspace_bytes; contents need not be initialised). Large
 * appends then list their over-long containers there (with drift_mode 1,
 * every container) and drift them ([news] "Drift: Bending Variable Back to
 * Fixed") in a separate kernel that runs at higher occupancy than the encode
 * kernel; the containers are the same bytes as with dq_append_kv. d_workspace NULL gives dq_append_kv. Calls
 * sharing a workspace must not overlap on the GPU. DQ_ERR_WORKSPACE if
 * ws_bytes is too small, DQ_ERR_ALIGN if the workspace is misaligned. */
int dq_append_kv_ws(const dq_tables *t, const void *k, const void *v, int dtype,
                    int B, int Hkv, int n_new, const int32_t *d_start_pos,
                    uint8_t *d_kcache, uint8_t *d_vcache, int64_t T_cap,
                    void *d_workspace, size_t ws_bytes, dq_stats *d_stats,
                    void *stream);

/* Bytes of device workspace dq_decode_attention needs for these shapes
 * (token-group prefix sums and the warps' partial softmax states: about
 * (B*Hkv + SMs*warps_per_SM) * G * 520 bytes, G = Hq/Hkv). Depends only on
 * its arguments, the tables' container sizes and the tables' device; T_max
 * does not change it. Returns 0 on invalid shapes. */
size_t dq_decode_workspace_bytes(const dq_tables *t, int B, int Hq, int Hkv,
                                 int64_t T_max);

/* Decode attention over the compressed cache ([abstract]: regular memory
 * access and parallel dequantisation within attention kernels). For every
 * (b, hq): out = softmax(sm_scale * q K^T) V over the first d_seq_lens[b]
 * tokens of the cache, with K and V dequantised from their containers
 * inside the kernel. Runs as a prefix kernel (token groups per sequence), a
 * split kernel (every warp takes an equal share of all 32-token groups of
 * all (b, h): rANS decode of K and V, q.K^T, online softmax, P.V) and a
 * combine kernel (log-sum-exp merge of the partial states and the inverse
 * rotation).
 *   q           device [B][Hq][128], q_dtype DQ_F32 or DQ_BF16
 *   d_kcache, d_vcache  device caches (interleaved layout), 16-byte
 *               aligned, T_cap % 32 == 0
 *   d_seq_lens  device int32 [B]; a length above T_max or T_cap is clamped
 *               and counted in clamped_lengths; length 0 gives out = 0
 *   T_max       host bound on max(d_seq_lens), 0 <= T_max <= T_cap
 *   sm_scale    softmax scale (1/sqrt(128) is the usual choice)
 *   out         device [B][Hq][128], out_dtype DQ_F32 or DQ_BF16
 *   d_workspace device, >= dq_decode_workspace_bytes(...) bytes, 16-byte
 *               aligned; contents need not be initialised
 *   d_stats     device dq_stats or NULL (integrity_errors counts containers
 *               whose decoder did not end in the initial state)
 * Hq must be a multiple of Hkv with Hq/Hkv in {1, 2, 4, 8}; Hkv must equal
 * the tables' n_kv_heads. */
int dq_decode_attention(const dq_tables *t, const void *q, int q_dtype,
                        const uint8_t *d_kcache, const uint8_t *d_vcache,
                        const int32_t *d_seq_lens, int B, int Hq, int Hkv,
                        int64_t T_cap, int64_t T_max, float sm_scale,
                        void *out, int out_dtype, void *d_workspace,
                        size_t ws_bytes, dq_stats *d_stats, void *stream);

/* Paged caches. The pages' serving results ([news] "The Numbers": batch 128
 * at an 8K prompt on one GPU) come from a serving engine, and such engines
 * hand out KV memory in fixed-size pages through a per-sequence page table;
 * the D-Quant pages describe no page table themselves. A page here is one
 * 32-token block of every KV head: a pool of num_pages pages is laid out
 * [num_pages][Hkv][C][32] (the 32 containers of a block byte-interleaved as
 * in the contiguous cache), and token t of sequence b lives in page
 * d_page_table[b * max_pages + t / 32], at lane t % 32 of its blocks.
 *   d_kpool, d_vpool  device pools of C_k- and C_v-byte containers, 16-byte
 *                     aligned (DQ_ERR_ALIGN)
 *   num_pages         pages in each pool, 1 .. 2^31
 *   d_page_table      device int32 [B][max_pages], 4-byte aligned; entries
 *                     outside [0, num_pages) are never dereferenced: they
 *                     are counted in bad_pages (an append drops the token,
 *                     the decoder reads page 0 instead)
 *   max_pages         pages per sequence; a sequence holds up to
 *                     32 * max_pages tokens (the T_cap of the contiguous calls)
 * Everything else is as in dq_append_kv_ws and dq_decode_attention (the
 * decode workspace is dq_decode_workspace_bytes, the append workspace is
 * optional); containers and outputs are the same as with a contiguous cache
 * holding the same tokens. */
int dq_append_kv_paged(const dq_tables *t, const void *k, const void *v, int dtype,
                       int B, int Hkv, int n_new, const int32_t *d_start_pos,
                       uint8_t *d_kpool, uint8_t *d_vpool, int64_t num_pages,
                       const int32_t *d_page_table, int64_t max_pages,
                       void *d_workspace, size_t ws_bytes, dq_stats *d_stats,
                       void *stream);
int dq_decode_attention_paged(const dq_tables *t, const void *q, int q_dtype,
                              const uint8_t *d_kpool, const uint8_t *d_vpool,
                              int64_t num_pages, const int32_t *d_page_table,
                              int64_t max_pages, const int32_t *d_seq_lens,
                              int B, int Hq, int Hkv, int64_t T_max, float sm_scale,
                              void *out, int out_dtype, void *d_workspace,
                              size_t ws_bytes, dq_stats *d_stats, void *stream);

/* Decode attention without a caller-provided workspace. The D-Quant pages
 * have no counterpart to this call: it exists for callers that cannot
 * allocate device memory -- a host application or plugin that is handed only
 * input and output device pointers, or a serving loop that must not call
 * cudaMalloc once it is running (an allocation can synchronise the device and
 * compete with a caching allocator that owns the memory). It computes exactly
 * what dq_decode_attention computes, with the same arguments minus the
 * workspace, and allocates nothing.
 *   Scratch: the partial results go to a fixed 8 MiB array in the
 *   library's own device memory (held by every GPU that loads the library
 *   until the process exits). Shapes whose workspace is above 8 MiB (see
 *   dq_decode_workspace_bytes; on a 148-SM B200 with 36-byte containers
 *   that is B*Hkv above about 1650 for G = 4, above about 250 for G = 8)
 *   are rejected with DQ_ERR_WORKSPACE before anything is enqueued.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, no allocation) with that device current; make that
 *   first call before any stream capture. The address is kept per device with
 *   the id of its CUDA context; a call in a new context on that device (after
 *   cudaDeviceReset, for example) looks the address up again, so that first
 *   call after the reset should also come before any stream capture.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents; nothing in it needs to start at zero. Calls whose work
 *   overlaps on the GPU (for example on two streams) race on the array and
 *   must be ordered by the caller. */
int dq_decode_attention_noalloc(const dq_tables *t, const void *q, int q_dtype,
                                const uint8_t *d_kcache, const uint8_t *d_vcache,
                                const int32_t *d_seq_lens, int B, int Hq, int Hkv,
                                int64_t T_cap, int64_t T_max, float sm_scale,
                                void *out, int out_dtype, dq_stats *d_stats,
                                void *stream);

/* Chunked-prefill attention over the compressed cache ([news] "D-Quant:
 * Entropy Coding Meets KV Cache at 2.26 Bits", "The Numbers": long prompts
 * of 8K to 128K tokens; [abstract]: dequantisation within attention
 * kernels). A prompt processed in chunks first appends the chunk's K and V
 * (dq_append_kv with n_new = n_q) and then attends: query token i of
 * sequence b sits at position p = d_q_start[b] + i and
 *   out[b][i][hq] = softmax(sm_scale * q[b][i][hq] K^T) V
 * over cache positions 0 .. p (causal), K and V dequantised from their
 * containers on the GPU. Query head hq reads KV head hq / (Hq/Hkv).
 * Two kernels: every 32-token block that the chunk attends to is rANS-
 * decoded once per (b, KV head) into fp16 tiles in the workspace; then one
 * CTA per (b, KV head, block of 128 / G query tokens) streams the tiles in
 * and runs the scores and P.V on the tensor cores (tcgen05, fp16 operands
 * split into hi + lo halves where fp32 precision matters, fp32 accumulation
 * in tensor memory) with the online softmax in between.
 *   q           device [B][n_q][Hq][128], q_dtype DQ_F32 or DQ_BF16
 *   d_kcache, d_vcache  device caches (interleaved layout), 16-byte aligned,
 *               T_cap % 32 == 0
 *   d_q_start   device int32 [B]; a query row whose position is outside
 *               [0, T_cap) gets out = 0 and is counted in clamped_lengths
 *   out         device [B][n_q][Hq][128], out_dtype DQ_F32 or DQ_BF16
 *   d_workspace device, 16-byte aligned, contents need not be
 *               initialised: the decoded tiles (521 bytes per token and KV
 *               head of the cache). dq_prefill_workspace_bytes(...) bytes
 *               hold the whole batch; any size down to one (b, KV head)
 *               row, dq_prefill_workspace_bytes(t, 1, 1, T_cap), works:
 *               the call then runs in waves of as many rows as fit
 *               (DQ_ERR_WORKSPACE below one row)
 *   d_stats     device dq_stats or NULL (integrity_errors: corrupt
 *               containers in the attended range; wait_timeouts: should
 *               stay 0)
 * Hq / Hkv must be 1, 2, 4 or 8 and Hkv the tables' n_kv_heads; n_q >= 0
 * (0 does nothing). Calls sharing a workspace must not overlap on the GPU. */
size_t dq_prefill_workspace_bytes(const dq_tables *t, int B, int Hkv,
                                  int64_t T_cap);
int dq_prefill_attention(const dq_tables *t, const void *q, int q_dtype,
                         const uint8_t *d_kcache, const uint8_t *d_vcache,
                         const int32_t *d_q_start, int B, int n_q, int Hq,
                         int Hkv, int64_t T_cap, float sm_scale, void *out,
                         int out_dtype, void *d_workspace, size_t ws_bytes,
                         dq_stats *d_stats, void *stream);
/* The same over paged pools (layout and page-table rules as in
 * dq_decode_attention_paged; T_cap is 32 * max_pages for the workspace). */
int dq_prefill_attention_paged(const dq_tables *t, const void *q, int q_dtype,
                               const uint8_t *d_kpool, const uint8_t *d_vpool,
                               int64_t num_pages, const int32_t *d_page_table,
                               int64_t max_pages, const int32_t *d_q_start, int B,
                               int n_q, int Hq, int Hkv, float sm_scale,
                               void *out, int out_dtype, void *d_workspace,
                               size_t ws_bytes, dq_stats *d_stats, void *stream);

/* Test hook: decodes n flat containers of one stream.
 *   d_cache   device [n][C]; d_syms device uint8 [n][128]; d_norm16 device
 *             uint16 [n]; d_status device int32 [n] (may be NULL)
 * Status per container: 0 ok, 1 initial state below 2^16, 2 the decoder ran
 * past the container, 3 final state != 2^16, 4 non-zero padding. Symbols
 * after the point of failure are 0. Corrupt containers are also counted in
 * d_stats->integrity_errors. */
int dq_decode_symbols(const dq_tables *t, const uint8_t *d_cache,
                      int stream_kind, int64_t n_containers, uint8_t *d_syms,
                      uint16_t *d_norm16, int32_t *d_status, dq_stats *d_stats,
                      void *stream);

/* Static description of a status code. Never NULL. */
const char *dq_error_string(int status);

/* The last CUDA error code seen by the library on this thread (0 if none). */
int dq_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DQ_H */
