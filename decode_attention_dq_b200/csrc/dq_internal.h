// dq_internal.h -- shared declarations of libdq (host design, device tables,
// kernel launchers). Not part of the public C-ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include "dq.h"

namespace dqi {

constexpr int kD = 128;            // head dimension
constexpr int kMaxLevels = 8;      // decoder supports up to 8 levels
constexpr int kProbBits = 12;      // M = 2^12
constexpr uint32_t kM = 4096u;
constexpr uint32_t kL = 65536u;    // rANS lower bound (32-bit state)
constexpr int kHeaderBytes = 5;    // fp16 norm + 3-byte final state
constexpr int kMaxContainer = 64;  // bytes; kernels stage at most this

// Host-side design of one stream (K or V).
struct StreamDesign {
  int n_levels = 0;
  int container_bytes = 0;
  int payload_bytes = 0;
  bool lloyd_max = false;
  double rate = 0, lambda = 0, entropy = 0, mse = 0;
  double y[kMaxLevels] = {}, t[kMaxLevels] = {}, p[kMaxLevels] = {};
  float levels[kMaxLevels] = {};
  float thresholds[kMaxLevels] = {};
  float cost[kMaxLevels] = {};
  uint32_t freq[kMaxLevels] = {};
  uint32_t cum[kMaxLevels + 1] = {};
};

// Returns DQ_OK, DQ_ERR_CONFIG or DQ_ERR_BUDGET.
int design_stream(int n_levels, int container_bytes, double rate_offset,
                  StreamDesign *out);
int container_bytes_for(double bits_per_value);
void rotation_signs(uint64_t seed, int n_heads, int8_t *out /*[n][128]*/);

// Device-resident table of one stream. Kernels copy `lut` with 16-byte
// loads, so the struct keeps a 16-byte multiple size inside DevTables.
struct alignas(16) DevStream {
  // Decode look-up: slot -> (slot - cum[s]) | s << 11 | f_s << 20
  // (slot - cum[s] < f_s <= 2048 fits 11 bits; f_s fits 12 bits).
  uint32_t lut[kM];
  float levels[kMaxLevels];
  float thresholds[kMaxLevels];  // n-1 used, the rest +inf
  float cost[kMaxLevels];
  uint32_t freq[kMaxLevels];
  uint32_t cum[kMaxLevels];
  // Levels for fp16 tensor-core operands: level16[s] holds the fp16 bits of
  // tile_scale * levels[s]; tile_scale in [1, 2) is chosen on the host so that
  // these fp16 values are as close as possible (relatively) to the scaled
  // fp32 levels; tile_rel_err is the largest relative error left.
  uint32_t level16[kMaxLevels];
  float tile_scale, tile_rel_err;
  int32_t n_levels, container_bytes, payload_bytes, pad;
  // Levels for the fp16 K operand of the prefill score MMA: score16[s] holds
  // the fp16 bits of score_scale * levels[s], with score_scale in [1, 2)
  // chosen to minimise the frequency-weighted absolute error of the levels
  // (the frequent inner levels come out exact to about 1e-6); score_err is
  // the largest relative error left (on a rare outer level).
  uint32_t score16[kMaxLevels];
  float score_scale, score_err;
};

struct DevTables {
  DevStream k, v;
};
static_assert(sizeof(DevStream) % 16 == 0, "DevStream must keep 16-byte alignment of the v table");

// Kernel launchers (defined in the .cu files). All return cudaError_t as int.
struct AppendArgs {
  const DevTables *tabs;
  const uint32_t *sign_bits;  // [Hkv][4]
  const void *k, *v;
  int dtype, B, Hkv, n_new;
  const int32_t *start_pos;
  uint8_t *kcache, *vcache;
  int64_t T_cap;
  int ck, cv;       // container bytes
  int nk, nv;       // levels
  bool two_k, two_v;  // the stream's table has a symbol with f < 16 (two pushes per step)
  int drift_mode;     // 0: drift only; 1: drift, then the rate-distortion fill
  dq_stats *stats;
  // Optional drift list (workspace): over-long containers of the
  // lane-per-vector kernel are listed here ([2][list_cap] vector indices, K
  // then V; counts in drift_count[2]) and drifted by a separate kernel.
  // nullptr: drift runs inside the encode kernel.
  uint32_t *drift_list;
  uint32_t *drift_count;
  int64_t list_cap;
  // Paged caches (nullptr: contiguous caches of T_cap tokens per row): token
  // t of sequence b is in page page_table[b * max_pages + t / 32] of a pool
  // laid out [num_pages][Hkv][C][32]; T_cap = 32 max_pages.
  const int32_t *page_table;
  int64_t max_pages, num_pages;
};
// Bytes of the optional append workspace for nvec vectors per stream.
size_t append_workspace_bytes(int64_t nvec);
int launch_append(const AppendArgs &a, void *stream);

struct DecodeArgs {
  const DevTables *tabs;
  const uint32_t *sign_bits;
  const void *q;
  int q_dtype;
  const uint8_t *kcache, *vcache;
  const int32_t *seq_lens;
  int B, Hq, Hkv, G;
  int64_t T_cap, T_max;
  float sm_scale;
  void *out;
  int out_dtype;
  int64_t *prefix;     // [B + 1] token-group prefix sums (written by the prefix kernel)
  float *ws_o;         // [slots][G][128] partial o_rot per (b, h) segment of a warp
  float *ws_ml;        // [slots][G][2]   partial (max, sum)
  int grid;            // CTAs of the split kernel (one per SM)
  int64_t total_warps;  // grid * decode_warps_per_cta(G, ck, cv); slots = B * Hkv + total_warps
  int ck, cv;
  bool two_k, two_v;  // the stream's table has a symbol with f < 16
  dq_stats *stats;
  // Paged caches, as in AppendArgs (nullptr: contiguous).
  const int32_t *page_table;
  int64_t max_pages, num_pages;
};
int launch_decode_attention(const DecodeArgs &a, void *stream);
// Warps per CTA of the split kernel for these shapes (0 if unsupported).
int decode_warps_per_cta(int G, int ck, int cv);

// Chunked-prefill attention (dq_prefill.cu).
struct PrefillArgs {
  const DevTables *tabs;
  const uint32_t *sign_bits;
  const void *q;       // [B][n_q][Hq][128]
  int q_dtype;
  const uint8_t *kcache, *vcache;
  const int32_t *q_start;  // [B]: position of query token 0 of each sequence
  int B, n_q, Hq, Hkv, G;
  int64_t T_cap;
  float sm_scale;
  void *out;           // [B][n_q][Hq][128]
  int out_dtype;
  int ck, cv;
  bool two_k, two_v;
  uint8_t *tiles;      // workspace: decoded slots of rows bh0 .. bh0 + nbh - 1, [nbh][ceil(T_cap / 128)]
  int64_t bh0, nbh;    // the wave of (b, KV head) rows (flat index b Hkv + h) this launch handles
  int nslots;          // ring depth of the attention kernel (prefill_ring_slots)
  int tile_grid;       // CTAs of the tile kernel
  dq_stats *stats;
  const int32_t *page_table;  // paged caches as in AppendArgs (nullptr: contiguous)
  int64_t max_pages, num_pages;
};
int launch_prefill_attention(const PrefillArgs &a, void *stream);
int prefill_ring_slots();
// CTAs of the attention kernel for nbh rows: nbh * ceil(n_q / (128 / G)).
int64_t prefill_grid(int64_t nbh, int G, int n_q);
// Bytes of decoded slots for B x Hkv rows of T_cap tokens.
size_t prefill_workspace_bytes(int B, int Hkv, int64_t T_cap);
bool prefill_supported(int ck, int cv);

struct SymbolsArgs {
  const DevStream *tab;
  const uint8_t *cache;
  int64_t n;
  int c;
  uint8_t *syms;
  uint16_t *norm16;
  int32_t *status;
  dq_stats *stats;
};
int launch_decode_symbols(const SymbolsArgs &a, void *stream);

}  // namespace dqi
