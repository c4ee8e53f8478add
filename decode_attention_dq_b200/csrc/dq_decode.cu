// dq_decode.cu -- decode attention over the compressed KV cache.
//
// [abstract] "D-Quant: Driftable Entropy Coding for KV Cache Quantization":
// fixed-size bitstreams give regular memory access and parallel
// dequantisation within attention kernels. [news] "D-Quant: Entropy Coding
// Meets KV Cache at 2.26 Bits", intro: rANS decoding runs inside the attention
// kernel; "The Numbers" 2nd paragraph: entropy decoding adds computation.
//
// Split kernel, one CTA per (sequence b, KV head h, token chunk):
//   D1  q~ = H D q / 128 for the G query heads of h (scaled by sm_scale log2 e)
//   D2  stage each warp's 32 K and 32 V containers into shared memory with
//       16-byte cp.async, double-buffered
//   D3  one lane per token: rANS-decode K (table look-up, multiply-add,
//       byte renormalisation) and accumulate q~ . y_hat for the G heads
//   D5  the same lane decodes V into a per-warp tile of levels
//   D4  online softmax per head across the warp (score * ||k||)
//   D5' coordinate-parallel P.V from the tile (weights p * ||v||)
//   D6  merge the warps and write (m, l, o_rot) per head to the workspace
// Combine kernel, one warp per (b, query head):
//   D7  log-sum-exp merge of the splits, o = D H o_rot / (128 l)
#include "dq_device.cuh"

namespace dqi {
namespace {

constexpr int kWarps = 8;
constexpr int kTile = 32;          // tokens per warp group (one per lane)
constexpr int kYStride = kD + 1;   // y tile row stride (floats), conflict-free
constexpr float kLog2e = 1.4426950408889634f;

struct SplitSmem {
  size_t lut_k, lut_v, lev, qt, warp0, warp_bytes, stage_k, stage_v, ytile, wbuf, total;
};

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

__host__ __device__ inline SplitSmem split_smem_layout(int G, int ck, int cv) {
  SplitSmem s;
  s.lut_k = 0;
  s.lut_v = s.lut_k + kM * 4;
  s.lev = s.lut_v + kM * 4;
  s.qt = s.lev + 2 * kMaxLevels * 4;
  s.warp0 = align16(s.qt + static_cast<size_t>(kD) * G * 4);
  s.stage_k = 0;
  s.stage_v = align16(2 * static_cast<size_t>(kTile) * ck);
  s.ytile = s.stage_v + align16(2 * static_cast<size_t>(kTile) * cv);
  s.wbuf = s.ytile + static_cast<size_t>(kTile) * kYStride * 4;
  s.warp_bytes = align16(s.wbuf + static_cast<size_t>(kTile) * G * 4);
  // 256 bytes of slack: a corrupt container can make its decoder read up
  // to 2 bytes per symbol past its start; those reads stay inside the CTA's
  // shared memory and only produce garbage (flagged by the final-state check).
  s.total = s.warp0 + kWarps * s.warp_bytes + 256;
  return s;
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Copies the containers of tokens [t0, t0 + n) of one cache row (n is 16 or 32,
// so n * C is a multiple of 16) into shared memory, 16 bytes per lane-step.
__device__ __forceinline__ void stage_group(uint8_t *dst, const uint8_t *row, int64_t t0, int n, int C,
                                            int lane) {
  const int chunks = (n * C) >> 4;
  const uint8_t *src = row + t0 * C;
  for (int c = lane; c < chunks; c += 32) cp_async16(dst + c * 16, src + c * 16);
}

struct RansLane {
  uint32_t x;
  const uint8_t *p;
};

// One decode step: returns the symbol's table entry (level index in bits
// 24..26) and advances the state, shifting in at most two bytes.
__device__ __forceinline__ uint32_t rans_step(RansLane &r, const uint32_t *lut) {
  const uint32_t e = lut[r.x & (kM - 1)];
  r.x = ((e >> 12) & 0xFFFu) * (r.x >> kProbBits) + (e & 0xFFFu);
  if (r.x < kL) {
    r.x = (r.x << 8) | *r.p++;
    if (r.x < kL) r.x = (r.x << 8) | *r.p++;
  }
  return e;
}

template <int G>
__global__ void __launch_bounds__(kWarps * 32, 1) decode_split_kernel(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const SplitSmem L = split_smem_layout(G, a.ck, a.cv);
  uint32_t *lut_k = reinterpret_cast<uint32_t *>(smem + L.lut_k);
  uint32_t *lut_v = reinterpret_cast<uint32_t *>(smem + L.lut_v);
  float *lev = reinterpret_cast<float *>(smem + L.lev);  // [0..7] K, [8..15] V
  float *qt = reinterpret_cast<float *>(smem + L.qt);    // [128][G]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t *wsm = smem + L.warp0 + warp * L.warp_bytes;
  uint8_t *stage_k = wsm + L.stage_k;
  uint8_t *stage_v = wsm + L.stage_v;
  float *ytile = reinterpret_cast<float *>(wsm + L.ytile);
  float *wbuf = reinterpret_cast<float *>(wsm + L.wbuf);

  const int bh = blockIdx.x;
  const int b = bh / a.Hkv, h = bh % a.Hkv;
  const int split = blockIdx.y;
  int64_t len = a.seq_lens[b];
  if (len < 0) len = 0;
  const int64_t cap = a.T_max < a.T_cap ? a.T_max : a.T_cap;
  if (len > cap) len = cap;
  const int64_t c0 = static_cast<int64_t>(split) * a.chunk;
  const int64_t c1 = (c0 + a.chunk) < len ? (c0 + a.chunk) : len;

  // Tables into shared memory.
  {
    const uint4 *sk = reinterpret_cast<const uint4 *>(a.tabs->k.lut);
    const uint4 *sv = reinterpret_cast<const uint4 *>(a.tabs->v.lut);
    uint4 *dk = reinterpret_cast<uint4 *>(lut_k);
    uint4 *dv = reinterpret_cast<uint4 *>(lut_v);
    for (int i = threadIdx.x; i < static_cast<int>(kM / 4); i += blockDim.x) {
      dk[i] = __ldg(sk + i);
      dv[i] = __ldg(sv + i);
    }
    if (threadIdx.x < kMaxLevels) {
      lev[threadIdx.x] = a.tabs->k.levels[threadIdx.x];
      lev[kMaxLevels + threadIdx.x] = a.tabs->v.levels[threadIdx.x];
    }
  }
  // D1: q~ for the G query heads of KV head h.
  {
    uint32_t sw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) sw[k] = __ldg(a.sign_bits + h * 4 + k);
    const float qscale = a.sm_scale * kLog2e / static_cast<float>(kD);
    for (int g = warp; g < G; g += kWarps) {
      const int64_t qbase = (static_cast<int64_t>(b) * a.Hq + h * G + g) * kD;
      float v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = apply_sign(load_elem(a.q, qbase + lane + 32 * k, a.q_dtype), sw[k], lane);
      wht128_warp(v, lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) qt[(lane + 32 * k) * G + g] = v[k] * qscale;
    }
  }
  __syncthreads();

  const uint8_t *krow = a.kcache + static_cast<int64_t>(bh) * a.T_cap * a.ck;
  const uint8_t *vrow = a.vcache + static_cast<int64_t>(bh) * a.T_cap * a.cv;

  float m_run[G], l_run[G], o_acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    l_run[g] = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) o_acc[g][k] = 0.0f;
  }
  unsigned bad_count = 0;

  // Groups of 32 tokens handled by this warp: c0 + (warp + j * kWarps) * 32.
  const int64_t ngroups = (c1 > c0) ? (c1 - c0 + kTile - 1) / kTile : 0;
  int64_t gidx = warp;
  auto issue = [&](int64_t gi, int buf) {
    if (gi < ngroups) {
      const int64_t t0 = c0 + gi * kTile;
      const int n = (a.T_cap - t0) < kTile ? static_cast<int>(a.T_cap - t0) : kTile;
      stage_group(stage_k + buf * kTile * a.ck, krow, t0, n, a.ck, lane);
      stage_group(stage_v + buf * kTile * a.cv, vrow, t0, n, a.cv, lane);
    }
    cp_async_commit();
  };
  issue(gidx, 0);
  int buf = 0;
  for (; gidx < ngroups; gidx += kWarps, buf ^= 1) {
    issue(gidx + kWarps, buf ^ 1);
    cp_async_wait_1();
    __syncwarp();
    const int64_t t = c0 + gidx * kTile + lane;
    const bool valid = t < c1;
    const uint8_t *kb = stage_k + buf * kTile * a.ck + lane * a.ck;
    const uint8_t *vb = stage_v + buf * kTile * a.cv + lane * a.cv;
    const float nk = __half2float(__ushort_as_half(static_cast<unsigned short>(kb[0] | (kb[1] << 8))));
    const float nv = __half2float(__ushort_as_half(static_cast<unsigned short>(vb[0] | (vb[1] << 8))));
    RansLane rk{static_cast<uint32_t>(kb[2]) | (static_cast<uint32_t>(kb[3]) << 8) |
                    (static_cast<uint32_t>(kb[4]) << 16),
                kb + kHeaderBytes};
    RansLane rv{static_cast<uint32_t>(vb[2]) | (static_cast<uint32_t>(vb[3]) << 8) |
                    (static_cast<uint32_t>(vb[4]) << 16),
                vb + kHeaderBytes};
    float sc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) sc[g] = 0.0f;
    float *yrow = ytile + lane * kYStride;
#pragma unroll 2
    for (int i = 0; i < kD; ++i) {
      const uint32_t ek = rans_step(rk, lut_k);
      const uint32_t ev = rans_step(rv, lut_v);
      const float yk = lev[ek >> 24];
      const float yv = lev[kMaxLevels + (ev >> 24)];
      const float *qi = qt + i * G;
#pragma unroll
      for (int g = 0; g < G; ++g) sc[g] = fmaf(qi[g], yk, sc[g]);
      yrow[i] = yv;
    }
    bad_count += __popc(__ballot_sync(kFull, valid && (rk.x != kL || rv.x != kL)));

    // D4: online softmax across the warp, per head.
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float s = valid ? sc[g] * nk : -INFINITY;
      const float m_new = fmaxf(m_run[g], warp_max(s));
      float p = 0.0f, alpha = 1.0f;
      if (m_new != -INFINITY) {
        p = exp2f(s - m_new);
        alpha = exp2f(m_run[g] - m_new);
      }
      l_run[g] = l_run[g] * alpha + warp_sum(p);
#pragma unroll
      for (int k = 0; k < 4; ++k) o_acc[g][k] *= alpha;
      m_run[g] = m_new;
      wbuf[lane * G + g] = valid ? p * nv : 0.0f;
    }
    __syncwarp();
    // D5': coordinates lane + 32 k accumulate over the 32 tokens.
    for (int tt = 0; tt < kTile; ++tt) {
      float w[G];
#pragma unroll
      for (int g = 0; g < G; ++g) w[g] = wbuf[tt * G + g];
      const float *yr = ytile + tt * kYStride;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float y = yr[lane + 32 * k];
#pragma unroll
        for (int g = 0; g < G; ++g) o_acc[g][k] = fmaf(w[g], y, o_acc[g][k]);
      }
    }
    __syncwarp();
  }
  asm volatile("cp.async.wait_all;\n" ::: "memory");
  if (a.stats && lane == 0 && bad_count) atomicAdd(&a.stats->integrity_errors, static_cast<unsigned long long>(bad_count));

  // D6: merge the warps' partial softmax states.
  __syncthreads();
  float *mrg_m = reinterpret_cast<float *>(smem + L.warp0);  // [kWarps][G]
  float *mrg_l = mrg_m + kWarps * G;                          // [kWarps][G]
  float *mrg_o = mrg_l + kWarps * G;                          // [kWarps][G][128]
  if (lane == 0)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mrg_m[warp * G + g] = m_run[g];
      mrg_l[warp * G + g] = l_run[g];
    }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int k = 0; k < 4; ++k) mrg_o[(warp * G + g) * kD + lane + 32 * k] = o_acc[g][k];
  __syncthreads();
  const int S = gridDim.y;
  for (int idx = threadIdx.x; idx < G * kD; idx += blockDim.x) {
    const int g = idx / kD, c = idx % kD;
    float M = -INFINITY;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mrg_m[w * G + g]);
    float o = 0.0f, l = 0.0f;
    if (M != -INFINITY)
      for (int w = 0; w < kWarps; ++w) {
        const float mw = mrg_m[w * G + g];
        if (mw == -INFINITY) continue;
        const float sc = exp2f(mw - M);
        o = fmaf(sc, mrg_o[(w * G + g) * kD + c], o);
        l = fmaf(sc, mrg_l[w * G + g], l);
      }
    const int64_t row = (static_cast<int64_t>(b) * a.Hq + h * G + g) * S + split;
    a.ws_o[row * kD + c] = o;
    if (c == 0) {
      a.ws_ml[row * 2] = M;
      a.ws_ml[row * 2 + 1] = l;
    }
  }
}

__global__ void __launch_bounds__(128) combine_kernel(const DecodeArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);  // b * Hq + hq
  if (row >= static_cast<int64_t>(a.B) * a.Hq) return;
  const int b = static_cast<int>(row / a.Hq), hq = static_cast<int>(row % a.Hq);
  const int h = hq / a.G;
  const int S = a.splits;
  if (hq == 0 && lane == 0 && a.stats) {
    const int64_t len = a.seq_lens[b];
    const int64_t cap = a.T_max < a.T_cap ? a.T_max : a.T_cap;
    if (len < 0 || len > cap) atomicAdd(&a.stats->clamped_lengths, 1ull);
  }
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, a.ws_ml[(row * S + s) * 2]);
  float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  float Ls = 0.0f;
  if (M != -INFINITY)
    for (int s = 0; s < S; ++s) {
      const float ms = a.ws_ml[(row * S + s) * 2];
      if (ms == -INFINITY) continue;
      const float sc = exp2f(ms - M);
      Ls = fmaf(sc, a.ws_ml[(row * S + s) * 2 + 1], Ls);
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = fmaf(sc, a.ws_o[(row * S + s) * kD + lane + 32 * k], v[k]);
    }
  const float inv = (Ls > 0.0f) ? 1.0f / (Ls * static_cast<float>(kD)) : 0.0f;
  wht128_warp(v, lane);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t sw = __ldg(a.sign_bits + h * 4 + k);
    const float o = apply_sign(v[k] * inv, sw, lane);
    store_elem(a.out, row * kD + lane + 32 * k, o, a.out_dtype);
  }
}

template <int G>
int launch_split(const DecodeArgs &a, cudaStream_t st) {
  const SplitSmem L = split_smem_layout(G, a.ck, a.cv);
  static bool configured[kMaxContainer + 1][kMaxContainer + 1] = {};
  if (!configured[a.ck][a.cv]) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(L.total));
    if (e != cudaSuccess) return static_cast<int>(e);
    configured[a.ck][a.cv] = true;
  }
  dim3 grid(static_cast<unsigned>(a.B * a.Hkv), static_cast<unsigned>(a.splits));
  decode_split_kernel<G><<<grid, kWarps * 32, L.total, st>>>(a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_decode_attention(const DecodeArgs &a, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a.ck > kMaxContainer || a.cv > kMaxContainer) return static_cast<int>(cudaErrorInvalidValue);
  int e = 0;
  switch (a.G) {
    case 1: e = launch_split<1>(a, st); break;
    case 2: e = launch_split<2>(a, st); break;
    case 4: e = launch_split<4>(a, st); break;
    case 8: e = launch_split<8>(a, st); break;
    default: return static_cast<int>(cudaErrorInvalidValue);
  }
  if (e) return e;
  const int64_t rows = static_cast<int64_t>(a.B) * a.Hq;
  combine_kernel<<<static_cast<unsigned>((rows + 3) / 4), 128, 0, st>>>(a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dqi
