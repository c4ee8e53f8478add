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

// Device-resident table of one stream.
struct DevStream {
  // Decode look-up: slot -> (slot - cum[s]) | s << 11 | f_s << 20
  // (slot - cum[s] < f_s <= 2048 fits 11 bits; f_s fits 12 bits).
  uint32_t lut[kM];
  float levels[kMaxLevels];
  float thresholds[kMaxLevels];  // n-1 used, the rest +inf
  float cost[kMaxLevels];
  uint32_t freq[kMaxLevels];
  uint32_t cum[kMaxLevels];
  int32_t n_levels, container_bytes, payload_bytes, pad;
};

struct DevTables {
  DevStream k, v;
};

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
  dq_stats *stats;
};
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
  float *ws_o;   // [B*Hq][S][128]
  float *ws_ml;  // [B*Hq][S][2]
  int splits;
  int64_t chunk;  // tokens per split (multiple of 32)
  int ck, cv;
  bool two_k, two_v;  // the stream's table has a symbol with f < 16
  dq_stats *stats;
};
int launch_decode_attention(const DecodeArgs &a, void *stream);

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
