// dq_abi.cpp -- the C-ABI of libdq: argument checks, table upload, workspace
// sizing and kernel launches. Every entry point catches C++ exceptions and
// reports a DQ_ERR_* code; nothing here allocates per call except
// dq_build_tables.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "dq_internal.h"

struct dq_tables {
  dq_config cfg{};
  int device = -1;
  int sm_count = 0;
  dqi::StreamDesign k, v;
  std::vector<int8_t> signs;
  void *d_block = nullptr;
  dqi::DevTables *d_tabs = nullptr;
  uint32_t *d_sign_bits = nullptr;
};

namespace {

thread_local int g_last_cuda = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda = static_cast<int>(e);
  return DQ_ERR_CUDA;
}

// Same device as the tables? (Device pointers from another device would be
// read through peer mappings at best; refuse instead.)
int check_device(const dq_tables *t) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  return dev == t->device ? DQ_OK : DQ_ERR_DEVICE;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// IEEE binary32 -> binary16, round to nearest even (overflow to infinity).
uint16_t f32_to_f16_rn(float f) {
  uint32_t x;
  std::memcpy(&x, &f, 4);
  const uint32_t sign = (x >> 16) & 0x8000u;
  x &= 0x7FFFFFFFu;
  if (x >= 0x7F800000u) return static_cast<uint16_t>(sign | (x > 0x7F800000u ? 0x7E00u : 0x7C00u));
  if (x >= 0x477FF000u) return static_cast<uint16_t>(sign | 0x7C00u);  // rounds to >= 65520
  if (x < 0x38800000u) {  // below 2^-14: subnormal half, units of 2^-24
    float a;
    std::memcpy(&a, &x, 4);
    return static_cast<uint16_t>(sign | static_cast<uint32_t>(std::nearbyint(static_cast<double>(a) * 16777216.0)));
  }
  uint32_t h = ((((x >> 23) - 127u + 15u) << 10) | ((x & 0x7FFFFFu) >> 13));
  const uint32_t rem = x & 0x1FFFu;
  if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) ++h;
  return static_cast<uint16_t>(sign | h);
}

double f16_to_double(uint16_t h) {
  const int e = (h >> 10) & 0x1F;
  const int m = h & 0x3FF;
  double v = e == 0 ? std::ldexp(static_cast<double>(m), -24) : std::ldexp(1024.0 + m, e - 25);
  return (h & 0x8000u) ? -v : v;
}

// Scale kappa in [1, 2) (steps of 2^-16) that minimises the largest relative
// error of fp16(kappa * level) over the non-zero levels; the smallest such
// kappa on ties.
void choose_tile_scale(const dqi::StreamDesign &d, dqi::DevStream *s) {
  double best_err = INFINITY;
  double best_k = 1.0;
  for (int j = 0; j < 65536; ++j) {
    const double kappa = 1.0 + j / 65536.0;
    double err = 0.0;
    for (int i = 0; i < d.n_levels; ++i) {
      const double y = static_cast<double>(d.levels[i]);
      if (y == 0.0) continue;
      const double h = f16_to_double(f32_to_f16_rn(static_cast<float>(kappa * y)));
      err = std::max(err, std::fabs(h - kappa * y) / std::fabs(kappa * y));
    }
    if (err < best_err) {
      best_err = err;
      best_k = kappa;
    }
  }
  s->tile_scale = static_cast<float>(best_k);
  s->tile_rel_err = static_cast<float>(best_err);
  for (int i = 0; i < dqi::kMaxLevels; ++i)
    s->level16[i] = i < d.n_levels ? f32_to_f16_rn(static_cast<float>(best_k * static_cast<double>(d.levels[i]))) : 0u;
}

// Scale kappa in [1, 2) (steps of 2^-16) for the prefill score operand:
// minimises sum_s f_s |fp16(kappa y_s) / kappa - y_s|, the expected absolute
// error of a coordinate's level, so the frequent inner levels are the exact
// ones; the smallest such kappa on ties.
void choose_score_scale(const dqi::StreamDesign &d, dqi::DevStream *s) {
  double best_err = INFINITY;
  double best_k = 1.0;
  for (int j = 0; j < 65536; ++j) {
    const double kappa = 1.0 + j / 65536.0;
    double err = 0.0;
    for (int i = 0; i < d.n_levels; ++i) {
      const double y = static_cast<double>(d.levels[i]);
      const double h = f16_to_double(f32_to_f16_rn(static_cast<float>(kappa * y)));
      err += static_cast<double>(d.freq[i]) * std::fabs(h / kappa - y);
    }
    if (err < best_err) {
      best_err = err;
      best_k = kappa;
    }
  }
  double worst = 0.0;
  for (int i = 0; i < dqi::kMaxLevels; ++i) {
    s->score16[i] = 0u;
    if (i >= d.n_levels) continue;
    const double y = static_cast<double>(d.levels[i]);
    s->score16[i] = f32_to_f16_rn(static_cast<float>(best_k * y));
    if (y != 0.0) worst = std::max(worst, std::fabs(f16_to_double(static_cast<uint16_t>(s->score16[i])) - best_k * y) /
                                              std::fabs(best_k * y));
  }
  s->score_scale = static_cast<float>(best_k);
  s->score_err = static_cast<float>(worst);
}

void fill_dev_stream(const dqi::StreamDesign &d, dqi::DevStream *s) {
  std::memset(s, 0, sizeof(*s));
  for (int sym = 0; sym < d.n_levels; ++sym)
    for (uint32_t slot = d.cum[sym]; slot < d.cum[sym + 1]; ++slot)
      s->lut[slot] = (slot - d.cum[sym]) | (static_cast<uint32_t>(sym) << 11) | (d.freq[sym] << 20);
  for (int i = 0; i < dqi::kMaxLevels; ++i) {
    s->levels[i] = i < d.n_levels ? d.levels[i] : 0.0f;
    s->thresholds[i] = d.thresholds[i];
    s->cost[i] = i < d.n_levels ? d.cost[i] : INFINITY;
    s->freq[i] = i < d.n_levels ? d.freq[i] : 0u;
    s->cum[i] = i < d.n_levels ? d.cum[i] : dqi::kM;
  }
  choose_tile_scale(d, s);
  choose_score_scale(d, s);
  s->n_levels = d.n_levels;
  s->container_bytes = d.container_bytes;
  s->payload_bytes = d.payload_bytes;
}

// A symbol with f < 16 can make one coding step move two bytes.
bool has_small_freq(const dqi::StreamDesign &d) {
  for (int s = 0; s < d.n_levels; ++s)
    if (d.freq[s] < 16) return true;
  return false;
}

const dqi::StreamDesign *stream_of(const dq_tables *t, int kind) {
  if (!t) return nullptr;
  if (kind == DQ_STREAM_K) return &t->k;
  if (kind == DQ_STREAM_V) return &t->v;
  return nullptr;
}

// Workspace of dq_decode_attention: the token-group prefix sums, then one
// partial-state slot per (b, h) segment of a warp's range. Slot (b Hkv + h) +
// warp is unique, so B Hkv + (total warps) slots cover every case.
struct WsLayout {
  int grid = 0;
  int64_t total_warps = 0;
  size_t prefix_off = 0, o_off = 0, ml_off = 0, total = 0;
};

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

WsLayout ws_layout(const dq_tables *t, int B, int Hkv, int G) {
  WsLayout w;
  const int nw = dqi::decode_warps_per_cta(G, t->k.container_bytes, t->v.container_bytes);
  if (nw <= 0) return w;
  w.grid = t->sm_count;
  w.total_warps = static_cast<int64_t>(w.grid) * nw;
  const size_t slots = static_cast<size_t>(B) * Hkv + static_cast<size_t>(w.total_warps);
  w.prefix_off = 0;
  w.o_off = round256((static_cast<size_t>(B) + 1) * sizeof(int64_t));
  w.ml_off = w.o_off + round256(slots * G * dqi::kD * sizeof(float));
  w.total = w.ml_off + slots * G * 2 * sizeof(float);
  return w;
}

}  // namespace

extern "C" {

void dq_config_default(dq_config *cfg) {
  if (!cfg) return;
  std::memset(cfg, 0, sizeof(*cfg));
  cfg->head_dim = 128;
  cfg->k_levels = 8;
  cfg->v_levels = 6;
  cfg->prob_bits = 12;
  cfg->k_bits_per_value = 2.26f;
  cfg->v_bits_per_value = 2.26f;
  cfg->n_kv_heads = 8;
  cfg->sign_seed = 0;
}

const char *dq_error_string(int status) {
  switch (status) {
    case DQ_OK: return "ok";
    case DQ_ERR_NULL: return "a required pointer is NULL";
    case DQ_ERR_CONFIG: return "invalid configuration (head_dim, prob_bits or level counts)";
    case DQ_ERR_BUDGET: return "container too small (or too large) for the level design";
    case DQ_ERR_SHAPE: return "invalid shape argument";
    case DQ_ERR_WORKSPACE: return "workspace too small";
    case DQ_ERR_ALIGN: return "misaligned pointer or T_cap not a multiple of 16";
    case DQ_ERR_DTYPE: return "unknown dtype";
    case DQ_ERR_CUDA: return "CUDA runtime error (see dq_last_cuda_error)";
    case DQ_ERR_DEVICE: return "not an sm_100 device or not the device of the tables";
    default: return "unknown status";
  }
}

int dq_last_cuda_error(void) { return g_last_cuda; }

// Host-only design of one stream (no device needed); arrays of 8 (9 for cum).
int dq_design_stream(int32_t n_levels, int32_t container_bytes, double rate_offset,
                     float *levels, float *thresholds, uint32_t *freq, uint32_t *cum,
                     float *cost, double *lambda, double *entropy, double *mse) {
  try {
    dqi::StreamDesign d;
    int rc = dqi::design_stream(n_levels, container_bytes, rate_offset, &d);
    if (rc != DQ_OK) return rc;
    for (int i = 0; i < dqi::kMaxLevels; ++i) {
      if (levels) levels[i] = i < n_levels ? d.levels[i] : 0.0f;
      if (thresholds && i < dqi::kMaxLevels - 1) thresholds[i] = d.thresholds[i];
      if (freq) freq[i] = d.freq[i];
      if (cost) cost[i] = i < n_levels ? d.cost[i] : 0.0f;
    }
    if (cum)
      for (int i = 0; i <= dqi::kMaxLevels; ++i) cum[i] = i <= n_levels ? d.cum[i] : dqi::kM;
    if (lambda) *lambda = d.lambda;
    if (entropy) *entropy = d.entropy;
    if (mse) *mse = d.mse;
    return DQ_OK;
  } catch (...) {
    return DQ_ERR_CONFIG;
  }
}

int dq_build_tables(const dq_config *cfg, dq_tables **out) {
  if (!cfg || !out) return DQ_ERR_NULL;
  *out = nullptr;
  if (cfg->head_dim != dqi::kD || cfg->prob_bits != dqi::kProbBits || cfg->n_kv_heads < 1 ||
      cfg->n_kv_heads > 4096 || (cfg->drift_mode != 0 && cfg->drift_mode != 1))
    return DQ_ERR_CONFIG;
  dq_tables *t = nullptr;
  try {
    t = new dq_tables();
    t->cfg = *cfg;
    const int ck = cfg->k_container_bytes ? cfg->k_container_bytes
                                          : dqi::container_bytes_for(cfg->k_bits_per_value);
    const int cv = cfg->v_container_bytes ? cfg->v_container_bytes
                                          : dqi::container_bytes_for(cfg->v_bits_per_value);
    int rc = dqi::design_stream(cfg->k_levels, ck, cfg->k_rate_offset, &t->k);
    if (rc == DQ_OK) rc = dqi::design_stream(cfg->v_levels, cv, cfg->v_rate_offset, &t->v);
    if (rc != DQ_OK) {
      delete t;
      return rc;
    }
    t->signs.resize(static_cast<size_t>(cfg->n_kv_heads) * dqi::kD);
    dqi::rotation_signs(cfg->sign_seed, cfg->n_kv_heads, t->signs.data());

    cudaError_t e = cudaGetDevice(&t->device);
    if (e != cudaSuccess) { delete t; return cuda_fail(e); }
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, t->device);
    if (e != cudaSuccess) { delete t; return cuda_fail(e); }
    if (prop.major != 10) { delete t; return DQ_ERR_DEVICE; }
    t->sm_count = prop.multiProcessorCount;

    std::vector<uint8_t> host(sizeof(dqi::DevTables) + t->signs.size() / 8);
    auto *dt = reinterpret_cast<dqi::DevTables *>(host.data());
    fill_dev_stream(t->k, &dt->k);
    fill_dev_stream(t->v, &dt->v);
    auto *bits = reinterpret_cast<uint32_t *>(host.data() + sizeof(dqi::DevTables));
    for (int h = 0; h < cfg->n_kv_heads; ++h)
      for (int w = 0; w < 4; ++w) {
        uint32_t word = 0;
        for (int l = 0; l < 32; ++l)
          if (t->signs[h * dqi::kD + w * 32 + l] < 0) word |= 1u << l;
        bits[h * 4 + w] = word;
      }
    e = cudaMalloc(&t->d_block, host.size());
    if (e != cudaSuccess) { delete t; return cuda_fail(e); }
    e = cudaMemcpy(t->d_block, host.data(), host.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { cudaFree(t->d_block); delete t; return cuda_fail(e); }
    t->d_tabs = reinterpret_cast<dqi::DevTables *>(t->d_block);
    t->d_sign_bits = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(t->d_block) + sizeof(dqi::DevTables));
    *out = t;
    return DQ_OK;
  } catch (const std::bad_alloc &) {
    delete t;
    return DQ_ERR_CONFIG;
  } catch (...) {
    delete t;
    return DQ_ERR_CONFIG;
  }
}

void dq_free_tables(dq_tables *t) {
  if (!t) return;
  if (t->d_block) cudaFree(t->d_block);
  delete t;
}

int dq_get_stream_table(const dq_tables *t, int stream_kind, int32_t *n_levels,
                        int32_t *container_bytes, float *levels, float *thresholds,
                        uint32_t *freq, uint32_t *cum, float *cost) {
  const dqi::StreamDesign *d = stream_of(t, stream_kind);
  if (!d) return t ? DQ_ERR_CONFIG : DQ_ERR_NULL;
  if (n_levels) *n_levels = d->n_levels;
  if (container_bytes) *container_bytes = d->container_bytes;
  for (int i = 0; i < dqi::kMaxLevels; ++i) {
    if (levels) levels[i] = i < d->n_levels ? d->levels[i] : 0.0f;
    if (thresholds && i < dqi::kMaxLevels - 1) thresholds[i] = d->thresholds[i];
    if (freq) freq[i] = d->freq[i];
    if (cost) cost[i] = i < d->n_levels ? d->cost[i] : 0.0f;
  }
  if (cum)
    for (int i = 0; i <= dqi::kMaxLevels; ++i) cum[i] = i <= d->n_levels ? d->cum[i] : dqi::kM;
  return DQ_OK;
}

int dq_get_stream_design(const dq_tables *t, int stream_kind, double *lambda, double *entropy,
                         double *rate, double *mse, int32_t *is_lloyd_max) {
  const dqi::StreamDesign *d = stream_of(t, stream_kind);
  if (!d) return t ? DQ_ERR_CONFIG : DQ_ERR_NULL;
  if (lambda) *lambda = d->lambda;
  if (entropy) *entropy = d->entropy;
  if (rate) *rate = d->rate;
  if (mse) *mse = d->mse;
  if (is_lloyd_max) *is_lloyd_max = d->lloyd_max ? 1 : 0;
  return DQ_OK;
}

int dq_get_signs(const dq_tables *t, int8_t *signs) {
  if (!t || !signs) return DQ_ERR_NULL;
  std::memcpy(signs, t->signs.data(), t->signs.size());
  return DQ_OK;
}

size_t dq_append_workspace_bytes(const dq_tables *t, int B, int Hkv, int n_new) {
  if (!t || B < 0 || Hkv < 1 || n_new < 0) return 0;
  return dqi::append_workspace_bytes(static_cast<int64_t>(B) * Hkv * n_new);
}

int dq_append_kv(const dq_tables *t, const void *k, const void *v, int dtype, int B, int Hkv,
                 int n_new, const int32_t *d_start_pos, uint8_t *d_kcache, uint8_t *d_vcache,
                 int64_t T_cap, dq_stats *d_stats, void *stream) {
  return dq_append_kv_ws(t, k, v, dtype, B, Hkv, n_new, d_start_pos, d_kcache, d_vcache, T_cap, nullptr, 0,
                         d_stats, stream);
}

// Shared by dq_append_kv_ws (page_table NULL) and dq_append_kv_paged.
static int append_core(const dq_tables *t, const void *k, const void *v, int dtype, int B, int Hkv, int n_new,
                       const int32_t *d_start_pos, uint8_t *d_kcache, uint8_t *d_vcache, int64_t T_cap,
                       void *d_workspace, size_t ws_bytes, dq_stats *d_stats, void *stream,
                       const int32_t *page_table, int64_t max_pages, int64_t num_pages) {
  try {
    if (!t || !k || !v || !d_start_pos || !d_kcache || !d_vcache) return DQ_ERR_NULL;
    if (dtype != DQ_F32 && dtype != DQ_BF16) return DQ_ERR_DTYPE;
    if (B < 0 || n_new < 0 || T_cap < 0 || Hkv != t->cfg.n_kv_heads) return DQ_ERR_SHAPE;
    if (!aligned(k, 16) || !aligned(v, 16) || T_cap % 32) return DQ_ERR_ALIGN;
    int rc = check_device(t);
    if (rc != DQ_OK) return rc;
    if (B == 0 || n_new == 0) return DQ_OK;
    dqi::AppendArgs a{};
    a.tabs = t->d_tabs;
    a.sign_bits = t->d_sign_bits;
    a.k = k;
    a.v = v;
    a.dtype = dtype;
    a.B = B;
    a.Hkv = Hkv;
    a.n_new = n_new;
    a.start_pos = d_start_pos;
    a.kcache = d_kcache;
    a.vcache = d_vcache;
    a.T_cap = T_cap;
    a.ck = t->k.container_bytes;
    a.cv = t->v.container_bytes;
    a.nk = t->k.n_levels;
    a.nv = t->v.n_levels;
    a.drift_mode = t->cfg.drift_mode;
    a.two_k = has_small_freq(t->k);
    a.two_v = has_small_freq(t->v);
    a.stats = d_stats;
    const int64_t nvec = static_cast<int64_t>(B) * Hkv * n_new;
    if (d_workspace) {
      if (!aligned(d_workspace, 16)) return DQ_ERR_ALIGN;
      if (ws_bytes < dqi::append_workspace_bytes(nvec)) return DQ_ERR_WORKSPACE;
      a.drift_count = static_cast<uint32_t *>(d_workspace);
      a.drift_list = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(d_workspace) + 256);
      a.list_cap = nvec;
    }
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.num_pages = num_pages;
    int e = dqi::launch_append(a, stream);
    return e == 0 ? DQ_OK : cuda_fail(static_cast<cudaError_t>(e));
  } catch (...) {
    return DQ_ERR_CUDA;
  }
}

int dq_append_kv_ws(const dq_tables *t, const void *k, const void *v, int dtype, int B, int Hkv, int n_new,
                    const int32_t *d_start_pos, uint8_t *d_kcache, uint8_t *d_vcache, int64_t T_cap,
                    void *d_workspace, size_t ws_bytes, dq_stats *d_stats, void *stream) {
  return append_core(t, k, v, dtype, B, Hkv, n_new, d_start_pos, d_kcache, d_vcache, T_cap, d_workspace, ws_bytes,
                     d_stats, stream, nullptr, 0, 0);
}

int dq_append_kv_paged(const dq_tables *t, const void *k, const void *v, int dtype, int B, int Hkv, int n_new,
                       const int32_t *d_start_pos, uint8_t *d_kpool, uint8_t *d_vpool, int64_t num_pages,
                       const int32_t *d_page_table, int64_t max_pages, void *d_workspace, size_t ws_bytes,
                       dq_stats *d_stats, void *stream) {
  if (!d_page_table) return DQ_ERR_NULL;
  if (num_pages < 1 || max_pages < 1 || max_pages > (int64_t(1) << 40) || num_pages > (int64_t(1) << 31))
    return DQ_ERR_SHAPE;
  if (!aligned(d_page_table, 4)) return DQ_ERR_ALIGN;
  return append_core(t, k, v, dtype, B, Hkv, n_new, d_start_pos, d_kpool, d_vpool, 32 * max_pages, d_workspace,
                     ws_bytes, d_stats, stream, d_page_table, max_pages, num_pages);
}

size_t dq_decode_workspace_bytes(const dq_tables *t, int B, int Hq, int Hkv, int64_t T_max) {
  if (!t || B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || T_max < 0) return 0;
  return ws_layout(t, B, Hkv, Hq / Hkv).total;
}

// Shared by dq_decode_attention (page_table NULL) and dq_decode_attention_paged.
static int decode_core(const dq_tables *t, const void *q, int q_dtype, const uint8_t *d_kcache,
                       const uint8_t *d_vcache, const int32_t *d_seq_lens, int B, int Hq, int Hkv,
                       int64_t T_cap, int64_t T_max, float sm_scale, void *out, int out_dtype,
                       void *d_workspace, size_t ws_bytes, dq_stats *d_stats, void *stream,
                       const int32_t *page_table, int64_t max_pages, int64_t num_pages) {
  try {
    if (!t || !q || !d_kcache || !d_vcache || !d_seq_lens || !out || !d_workspace) return DQ_ERR_NULL;
    if ((q_dtype != DQ_F32 && q_dtype != DQ_BF16) || (out_dtype != DQ_F32 && out_dtype != DQ_BF16))
      return DQ_ERR_DTYPE;
    if (B < 0 || Hkv != t->cfg.n_kv_heads || Hq < Hkv || Hq % Hkv) return DQ_ERR_SHAPE;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return DQ_ERR_SHAPE;
    if (T_cap < 0 || T_max < 0 || T_max > T_cap) return DQ_ERR_SHAPE;
    if (T_cap % 32 || !aligned(d_kcache, 16) || !aligned(d_vcache, 16) || !aligned(d_workspace, 16) ||
        !aligned(q, 4) || !aligned(out, 4))
      return DQ_ERR_ALIGN;
    if (!std::isfinite(sm_scale)) return DQ_ERR_SHAPE;
    const WsLayout wl = ws_layout(t, B, Hkv, G);
    if (wl.total == 0) return DQ_ERR_SHAPE;
    if (ws_bytes < wl.total) return DQ_ERR_WORKSPACE;
    int rc = check_device(t);
    if (rc != DQ_OK) return rc;
    if (B == 0) return DQ_OK;
    dqi::DecodeArgs a{};
    a.tabs = t->d_tabs;
    a.sign_bits = t->d_sign_bits;
    a.q = q;
    a.q_dtype = q_dtype;
    a.kcache = d_kcache;
    a.vcache = d_vcache;
    a.seq_lens = d_seq_lens;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = G;
    a.T_cap = T_cap;
    a.T_max = T_max;
    a.sm_scale = sm_scale;
    a.out = out;
    a.out_dtype = out_dtype;
    uint8_t *ws = static_cast<uint8_t *>(d_workspace);
    a.prefix = reinterpret_cast<int64_t *>(ws + wl.prefix_off);
    a.ws_o = reinterpret_cast<float *>(ws + wl.o_off);
    a.ws_ml = reinterpret_cast<float *>(ws + wl.ml_off);
    a.grid = wl.grid;
    a.total_warps = wl.total_warps;
    a.ck = t->k.container_bytes;
    a.cv = t->v.container_bytes;
    a.two_k = has_small_freq(t->k);
    a.two_v = has_small_freq(t->v);
    a.stats = d_stats;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.num_pages = num_pages;
    int e = dqi::launch_decode_attention(a, stream);
    return e == 0 ? DQ_OK : cuda_fail(static_cast<cudaError_t>(e));
  } catch (...) {
    return DQ_ERR_CUDA;
  }
}

int dq_decode_attention(const dq_tables *t, const void *q, int q_dtype, const uint8_t *d_kcache,
                        const uint8_t *d_vcache, const int32_t *d_seq_lens, int B, int Hq, int Hkv,
                        int64_t T_cap, int64_t T_max, float sm_scale, void *out, int out_dtype,
                        void *d_workspace, size_t ws_bytes, dq_stats *d_stats, void *stream) {
  return decode_core(t, q, q_dtype, d_kcache, d_vcache, d_seq_lens, B, Hq, Hkv, T_cap, T_max, sm_scale, out,
                     out_dtype, d_workspace, ws_bytes, d_stats, stream, nullptr, 0, 0);
}

int dq_decode_attention_paged(const dq_tables *t, const void *q, int q_dtype, const uint8_t *d_kpool,
                              const uint8_t *d_vpool, int64_t num_pages, const int32_t *d_page_table,
                              int64_t max_pages, const int32_t *d_seq_lens, int B, int Hq, int Hkv,
                              int64_t T_max, float sm_scale, void *out, int out_dtype, void *d_workspace,
                              size_t ws_bytes, dq_stats *d_stats, void *stream) {
  if (!d_page_table) return DQ_ERR_NULL;
  if (num_pages < 1 || max_pages < 1 || max_pages > (int64_t(1) << 40) || num_pages > (int64_t(1) << 31))
    return DQ_ERR_SHAPE;
  if (!aligned(d_page_table, 4)) return DQ_ERR_ALIGN;
  return decode_core(t, q, q_dtype, d_kpool, d_vpool, d_seq_lens, B, Hq, Hkv, 32 * max_pages, T_max, sm_scale,
                     out, out_dtype, d_workspace, ws_bytes, d_stats, stream, d_page_table, max_pages, num_pages);
}

static int prefill_core(const dq_tables *t, const void *q, int q_dtype, const uint8_t *d_kcache,
                        const uint8_t *d_vcache, const int32_t *d_q_start, int B, int n_q, int Hq, int Hkv,
                        int64_t T_cap, float sm_scale, void *out, int out_dtype, void *d_workspace,
                        size_t ws_bytes, dq_stats *d_stats, void *stream, const int32_t *page_table,
                        int64_t max_pages, int64_t num_pages) {
  try {
    if (!t || !q || !d_kcache || !d_vcache || !d_q_start || !out || !d_workspace) return DQ_ERR_NULL;
    if ((q_dtype != DQ_F32 && q_dtype != DQ_BF16) || (out_dtype != DQ_F32 && out_dtype != DQ_BF16))
      return DQ_ERR_DTYPE;
    if (B < 0 || n_q < 0 || Hkv != t->cfg.n_kv_heads || Hq < Hkv || Hq % Hkv) return DQ_ERR_SHAPE;
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return DQ_ERR_SHAPE;
    if (T_cap < 0) return DQ_ERR_SHAPE;
    if (T_cap % 32 || !aligned(d_kcache, 16) || !aligned(d_vcache, 16) || !aligned(q, 4) || !aligned(out, 4) ||
        !aligned(d_q_start, 4) || !aligned(d_workspace, 16))
      return DQ_ERR_ALIGN;
    if (!std::isfinite(sm_scale)) return DQ_ERR_SHAPE;
    if (!dqi::prefill_supported(t->k.container_bytes, t->v.container_bytes)) return DQ_ERR_SHAPE;
    // The workspace holds the decoded tiles of a wave of (b, KV head) rows:
    // at least one row; a smaller workspace than the whole batch's runs the
    // call in several waves.
    const int64_t rows = static_cast<int64_t>(B) * Hkv;
    const size_t row_bytes = dqi::prefill_workspace_bytes(1, 1, T_cap);
    if (T_cap > 0 && ws_bytes < row_bytes) return DQ_ERR_WORKSPACE;
    const int64_t per_wave = row_bytes ? std::min<int64_t>(rows, static_cast<int64_t>(ws_bytes / row_bytes)) : rows;
    if (per_wave > 0 && dqi::prefill_grid(per_wave, G, n_q) > 0x7FFFFFFF) return DQ_ERR_SHAPE;
    int rc = check_device(t);
    if (rc != DQ_OK) return rc;
    if (B == 0 || n_q == 0 || T_cap == 0) {
      if (B > 0 && n_q > 0) {  // no cache: every row is outside it, out = 0
        const size_t n = static_cast<size_t>(B) * n_q * Hq * dqi::kD * (out_dtype == DQ_F32 ? 4 : 2);
        cudaError_t e = cudaMemsetAsync(out, 0, n, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e);
      }
      return DQ_OK;
    }
    dqi::PrefillArgs a{};
    a.tabs = t->d_tabs;
    a.sign_bits = t->d_sign_bits;
    a.q = q;
    a.q_dtype = q_dtype;
    a.kcache = d_kcache;
    a.vcache = d_vcache;
    a.q_start = d_q_start;
    a.B = B;
    a.n_q = n_q;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = G;
    a.T_cap = T_cap;
    a.sm_scale = sm_scale;
    a.out = out;
    a.out_dtype = out_dtype;
    a.ck = t->k.container_bytes;
    a.cv = t->v.container_bytes;
    a.two_k = has_small_freq(t->k);
    a.two_v = has_small_freq(t->v);
    a.tiles = static_cast<uint8_t *>(d_workspace);
    a.nslots = dqi::prefill_ring_slots();
    a.stats = d_stats;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.num_pages = num_pages;
    for (int64_t bh0 = 0; bh0 < rows; bh0 += per_wave) {
      a.bh0 = bh0;
      a.nbh = std::min<int64_t>(per_wave, rows - bh0);
      const int64_t groups = a.nbh * (T_cap / 32);
      a.tile_grid = static_cast<int>(std::min<int64_t>(t->sm_count, (groups + 19) / 20));
      int e = dqi::launch_prefill_attention(a, stream);
      if (e != 0) return cuda_fail(static_cast<cudaError_t>(e));
    }
    return DQ_OK;
  } catch (...) {
    return DQ_ERR_CUDA;
  }
}

size_t dq_prefill_workspace_bytes(const dq_tables *t, int B, int Hkv, int64_t T_cap) {
  if (!t || B < 0 || Hkv < 1 || T_cap < 0 || T_cap % 32) return 0;
  return std::max<size_t>(16, dqi::prefill_workspace_bytes(B, Hkv, T_cap));
}

int dq_prefill_attention(const dq_tables *t, const void *q, int q_dtype, const uint8_t *d_kcache,
                         const uint8_t *d_vcache, const int32_t *d_q_start, int B, int n_q, int Hq, int Hkv,
                         int64_t T_cap, float sm_scale, void *out, int out_dtype, void *d_workspace,
                         size_t ws_bytes, dq_stats *d_stats, void *stream) {
  return prefill_core(t, q, q_dtype, d_kcache, d_vcache, d_q_start, B, n_q, Hq, Hkv, T_cap, sm_scale, out,
                      out_dtype, d_workspace, ws_bytes, d_stats, stream, nullptr, 0, 0);
}

int dq_prefill_attention_paged(const dq_tables *t, const void *q, int q_dtype, const uint8_t *d_kpool,
                               const uint8_t *d_vpool, int64_t num_pages, const int32_t *d_page_table,
                               int64_t max_pages, const int32_t *d_q_start, int B, int n_q, int Hq, int Hkv,
                               float sm_scale, void *out, int out_dtype, void *d_workspace, size_t ws_bytes,
                               dq_stats *d_stats, void *stream) {
  if (!d_page_table) return DQ_ERR_NULL;
  if (num_pages < 1 || max_pages < 1 || max_pages > (int64_t(1) << 40) || num_pages > (int64_t(1) << 31))
    return DQ_ERR_SHAPE;
  if (!aligned(d_page_table, 4)) return DQ_ERR_ALIGN;
  return prefill_core(t, q, q_dtype, d_kpool, d_vpool, d_q_start, B, n_q, Hq, Hkv, 32 * max_pages, sm_scale, out,
                      out_dtype, d_workspace, ws_bytes, d_stats, stream, d_page_table, max_pages, num_pages);
}

int dq_decode_symbols(const dq_tables *t, const uint8_t *d_cache, int stream_kind,
                      int64_t n_containers, uint8_t *d_syms, uint16_t *d_norm16, int32_t *d_status,
                      dq_stats *d_stats, void *stream) {
  try {
    if (!t || !d_cache || !d_syms || !d_norm16) return DQ_ERR_NULL;
    if (stream_kind != DQ_STREAM_K && stream_kind != DQ_STREAM_V) return DQ_ERR_CONFIG;
    if (n_containers < 0) return DQ_ERR_SHAPE;
    if (!aligned(d_cache, 4)) return DQ_ERR_ALIGN;
    int rc = check_device(t);
    if (rc != DQ_OK) return rc;
    if (n_containers == 0) return DQ_OK;
    dqi::SymbolsArgs a{};
    a.tab = stream_kind == DQ_STREAM_K ? &t->d_tabs->k : &t->d_tabs->v;
    a.cache = d_cache;
    a.n = n_containers;
    a.c = stream_kind == DQ_STREAM_K ? t->k.container_bytes : t->v.container_bytes;
    a.syms = d_syms;
    a.norm16 = d_norm16;
    a.status = d_status;
    a.stats = d_stats;
    int e = dqi::launch_decode_symbols(a, stream);
    return e == 0 ? DQ_OK : cuda_fail(static_cast<cudaError_t>(e));
  } catch (...) {
    return DQ_ERR_CUDA;
  }
}

}  // extern "C"
