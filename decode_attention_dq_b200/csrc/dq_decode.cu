// dq_decode.cu -- decode attention over the compressed KV cache.
//
// [abstract] "D-Quant: Driftable Entropy Coding for KV Cache Quantization":
// fixed-size bitstreams give regular memory access and parallel
// dequantisation within attention kernels. [news] "D-Quant: Entropy Coding
// Meets KV Cache at 2.26 Bits", intro: rANS decoding runs inside the attention
// kernel; "The Numbers" 2nd paragraph: entropy decoding adds computation.
//
// Split kernel: one persistent CTA per SM (as many warps as shared memory
// allows) walks over work items (sequence b, KV head h, token chunk); all
// warps of the CTA share the decode tables and q~ of the current item.
//   D1  q~ = H D q / 128 for the G query heads of h (times sm_scale log2 e)
//   D2  each warp stages 32 K and 32 V containers at a time into shared
//       memory with 16-byte cp.async, one group ahead
//   D3  one lane per token: rANS-decode K (table look-up, multiply-add, byte
//       renormalisation) and accumulate q~ . y_hat for the G heads
//   D5  in the same loop the lane decodes V of the PREVIOUS group (whose
//       softmax weights are known) into a half-width tile of levels, so every
//       lane runs two independent rANS chains
//   D4  online softmax per head across the warp (score * ||k||)
//   D5' P.V from the tile: each lane accumulates 4 coordinates x G heads
//       over 16 tokens with packed fp32 multiply-adds
//   D6  at the end of an item the warps' (m, l, o_rot) are merged and written
//       to the workspace
// Combine kernel, one warp per (b, query head):
//   D7  log-sum-exp merge of the splits, o = D H o_rot / (128 l)
#include <type_traits>

#include "dq_device.cuh"

namespace dqi {
namespace {

constexpr int kMaxWarps = 16;      // warps per CTA (one persistent CTA per SM)
constexpr int kTile = 32;          // tokens per warp group (one per lane)
constexpr int kHalf = 64;          // coordinates per V tile half
constexpr int kTStride = kHalf + 4;  // V tile row stride (floats): conflict-free 128-bit access
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

// Shared-memory layout of the split kernel. Everything a CTA shares (decode
// tables, q~) comes first; each warp then owns its staging slots, V tile and
// softmax-weight buffer.
struct SplitSmem {
  size_t lut_k, lut_v, lev, qt, warp0, warp_bytes;
  size_t kst, vst, tile, wbuf;  // offsets inside a warp's area
  size_t total;
  int nwarps;
};

__host__ __device__ inline SplitSmem split_smem_layout(int G, int ck, int cv, int nwarps) {
  SplitSmem s;
  s.lut_k = 0;
  s.lut_v = s.lut_k + kM * 4;
  s.lev = s.lut_v + kM * 4;
  s.qt = s.lev + 2 * kMaxLevels * 4;
  s.warp0 = align16(s.qt + static_cast<size_t>(kD) * G * 4);
  s.kst = 0;                                                        // 2 slots of 32 K containers
  s.vst = align16(2 * static_cast<size_t>(kTile) * ck);             // 2 slots of 32 V containers
  s.tile = s.vst + align16(2 * static_cast<size_t>(kTile) * cv);    // [32][kTStride] floats
  s.wbuf = s.tile + static_cast<size_t>(kTile) * kTStride * 4;      // [32][G] floats
  s.warp_bytes = align16(s.wbuf + static_cast<size_t>(kTile) * G * 4);
  s.nwarps = nwarps;
  // 256 bytes of slack: a corrupt container can make its decoder read up to
  // 2 bytes per symbol past its start; those reads stay inside the CTA's
  // shared memory and only produce garbage (flagged by the final-state check).
  s.total = s.warp0 + static_cast<size_t>(nwarps) * s.warp_bytes + 256;
  return s;
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Copies the containers of tokens [t0, t0 + n) of one cache row (n is 16 or
// 32, so n * C is a multiple of 16) into shared memory, 16 bytes per copy.
__device__ __forceinline__ void stage_group(uint8_t *dst, const uint8_t *row, int64_t t0, int n, int C,
                                            int lane) {
  const int chunks = (n * C) >> 4;
  const uint8_t *src = row + t0 * C;
  for (int c = lane; c < chunks; c += 32) cp_async16(dst + c * 16, src + c * 16);
}

// rANS decoder state of one lane: the 32-bit state and the shared-memory
// offset (from the kernel's shared base) of the next container byte.
struct RansLane {
  uint32_t x;
  uint32_t p;
};

__device__ __forceinline__ RansLane rans_open(const uint8_t *smem, uint32_t off) {
  RansLane r;
  r.x = static_cast<uint32_t>(smem[off + 2]) | (static_cast<uint32_t>(smem[off + 3]) << 8) |
        (static_cast<uint32_t>(smem[off + 4]) << 16);
  r.p = off + kHeaderBytes;
  return r;
}

// One decode step. Table entry layout: bits 0..10 slot - c_s, bits 11..13 the
// symbol s, bits 20..31 f_s. The state advances as x = f (x >> 12) + (slot -
// c_s). Renormalisation is arithmetic, without branches or selects: with
// n = 1 exactly when x < 2^16 (the top bit of x - 2^16), x += n (255 x + b)
// shifts in the next byte b and the cursor moves by n. A second byte can only
// be needed after a symbol with f < 16 (x >= 16 f after the step); kTwo
// enables that step for tables that have such a symbol. The byte reads never
// leave the staged shared memory (the cursor moves at most 2 bytes per
// symbol; 256 bytes of slack follow the last staged container). Returns the
// byte offset 4 s of the symbol's level.
template <bool kTwo>
__device__ __forceinline__ uint32_t rans_step(RansLane &r, const uint32_t *lut, const uint8_t *smem) {
  const uint32_t e = lut[r.x & (kM - 1)];
  uint32_t x = (e >> 20) * (r.x >> kProbBits) + (e & 0x7FFu);
  const uint32_t b0 = smem[r.p];
  const uint32_t b1 = kTwo ? static_cast<uint32_t>(smem[r.p + 1]) : 0u;
  const uint32_t n0 = __umulhi(x - kL, 2u);
  x += n0 * (x * 255u + b0);
  uint32_t adv = n0;
  if constexpr (kTwo) {
    const uint32_t n1 = __umulhi(x - kL, 2u);
    x += n1 * (x * 255u + b1);
    adv += n1;
  }
  r.p += adv;
  r.x = x;
  return (e >> 9) & 0x1Cu;
}

__device__ __forceinline__ float norm_of(const uint8_t *cb) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(cb[0] | (cb[1] << 8))));
}

// sc[g] += q~[i][g] * y for the G heads, two heads per packed fp32 FMA.
template <int G>
__device__ __forceinline__ void score_fma(float (&sc)[G], const float *qi, float y) {
  if constexpr (G % 2 == 0) {
    const float2 yy = make_float2(y, y);
#pragma unroll
    for (int g = 0; g < G; g += 2) {
      const float2 q2 = *reinterpret_cast<const float2 *>(qi + g);
      const float2 r = __ffma2_rn(q2, yy, make_float2(sc[g], sc[g + 1]));
      sc[g] = r.x;
      sc[g + 1] = r.y;
    }
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) sc[g] = fmaf(qi[g], y, sc[g]);
  }
}

// Per-warp state of one work item's online softmax and P.V accumulators.
// Lane l accumulates coordinates 4 (l & 15) .. +3 of each 64-coordinate half
// over the tokens of its half-group (l >> 4); the two half-groups are summed
// at the end of the item.
template <int G>
struct WarpAcc {
  float m[G], l[G];
  float2 o[2][G][2];  // [half][head][coordinate pair]: coordinates 4q + {0,1} and 4q + {2,3}
};

template <int G, int half>
__device__ __forceinline__ void pv_half(WarpAcc<G> &acc, const float *tile, const float *wbuf, int lane) {
  const int th = lane >> 4, q = lane & 15;
#pragma unroll 4
  for (int kk = 0; kk < 16; ++kk) {
    const int t = th * 16 + kk;
    const float4 y = *reinterpret_cast<const float4 *>(tile + t * kTStride + 4 * q);
    float w[G];
    if constexpr (G % 4 == 0) {
#pragma unroll
      for (int g4 = 0; g4 < G; g4 += 4) {
        const float4 ww = *reinterpret_cast<const float4 *>(wbuf + t * G + g4);
        w[g4] = ww.x; w[g4 + 1] = ww.y; w[g4 + 2] = ww.z; w[g4 + 3] = ww.w;
      }
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) w[g] = wbuf[t * G + g];
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float2 wg = make_float2(w[g], w[g]);
      acc.o[half][g][0] = __ffma2_rn(make_float2(y.x, y.y), wg, acc.o[half][g][0]);
      acc.o[half][g][1] = __ffma2_rn(make_float2(y.z, y.w), wg, acc.o[half][g][1]);
    }
  }
}

// Online-softmax update for one group's scores (lane = token); keeps the
// probabilities p (without the V norm) in `p` for the caller.
template <int G>
__device__ __forceinline__ void softmax_update(WarpAcc<G> &acc, const float (&sc)[G], float nk, bool valid,
                                               float (&p)[G]) {
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float s = valid ? sc[g] * nk : -INFINITY;
    const float m_new = fmaxf(acc.m[g], warp_max(s));
    float alpha = 1.0f;
    p[g] = 0.0f;
    if (m_new != -INFINITY) {
      p[g] = exp2f(s - m_new);
      alpha = exp2f(acc.m[g] - m_new);
    }
    acc.l[g] = acc.l[g] * alpha + warp_sum(p[g]);
    acc.m[g] = m_new;
    const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      acc.o[h][g][0] = __fmul2_rn(acc.o[h][g][0], a2);
      acc.o[h][g][1] = __fmul2_rn(acc.o[h][g][1], a2);
    }
  }
}

// Warps per CTA: as many as shared memory allows, capped so that G = 8 keeps
// enough registers for its larger accumulators.
__host__ __device__ constexpr int max_warps_for(int G) { return G >= 8 ? 12 : kMaxWarps; }

template <int G, bool kTwoK, bool kTwoV>
__global__ void __launch_bounds__(max_warps_for(G) * 32, 1) decode_split_kernel(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int nwarps = blockDim.x >> 5;
  const SplitSmem L = split_smem_layout(G, a.ck, a.cv, nwarps);
  uint32_t *lut_k = reinterpret_cast<uint32_t *>(smem + L.lut_k);
  uint32_t *lut_v = reinterpret_cast<uint32_t *>(smem + L.lut_v);
  float *lev = reinterpret_cast<float *>(smem + L.lev);  // [0..7] K, [8..15] V
  float *qt = reinterpret_cast<float *>(smem + L.qt);    // [128][G]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t *wsm = smem + L.warp0 + warp * L.warp_bytes;
  uint8_t *kst = wsm + L.kst;
  uint8_t *vst = wsm + L.vst;
  float *tile = reinterpret_cast<float *>(wsm + L.tile);
  float *wbuf = reinterpret_cast<float *>(wsm + L.wbuf);
  const int ck = a.ck, cv = a.cv;

  // Decode tables into shared memory (once per CTA).
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
  const int S = a.splits;
  const int64_t n_items = static_cast<int64_t>(a.B) * a.Hkv * S;
  const int64_t cap = a.T_max < a.T_cap ? a.T_max : a.T_cap;
  unsigned bad_count = 0;

  for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int bh = static_cast<int>(item / S);
    const int split = static_cast<int>(item % S);
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    int64_t len = a.seq_lens[b];
    if (len < 0) len = 0;
    if (len > cap) len = cap;
    const int64_t c0 = static_cast<int64_t>(split) * a.chunk;
    const int64_t c1 = (c0 + a.chunk) < len ? (c0 + a.chunk) : len;
    const int64_t ngroups = (c1 > c0) ? (c1 - c0 + kTile - 1) / kTile : 0;

    __syncthreads();  // previous item's merge area and q~ are no longer in use
    // D1: q~ = H D q / 128 for the G query heads of KV head h, times sm_scale log2 e.
    {
      uint32_t sw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) sw[k] = __ldg(a.sign_bits + h * 4 + k);
      const float qscale = a.sm_scale * kLog2e / static_cast<float>(kD);
      for (int g = warp; g < G; g += nwarps) {
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

    const uint8_t *krow = a.kcache + static_cast<int64_t>(bh) * a.T_cap * ck;
    const uint8_t *vrow = a.vcache + static_cast<int64_t>(bh) * a.T_cap * cv;
    auto group_t0 = [&](int64_t j) { return c0 + (warp + j * nwarps) * kTile; };
    const int64_t nmine = (ngroups > warp) ? (ngroups - warp + nwarps - 1) / nwarps : 0;
    auto ncopy = [&](int64_t t0) { return (a.T_cap - t0) < kTile ? static_cast<int>(a.T_cap - t0) : kTile; };

    WarpAcc<G> acc;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      acc.m[g] = -INFINITY;
      acc.l[g] = 0.0f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        acc.o[hh][g][0] = make_float2(0.0f, 0.0f);
        acc.o[hh][g][1] = make_float2(0.0f, 0.0f);
      }
    }

    if (nmine > 0) {
      // Prologue: K(0), V(0) into slot 0 and K(1) into K slot 1. Invariant at
      // the top of iteration j: V(j) sits in V slot j%2 and K(j+1) in K slot
      // (j+1)%2, both complete; iteration j prefetches K(j+2) and V(j+1).
      {
        const int64_t t0 = group_t0(0);
        stage_group(kst, krow, t0, ncopy(t0), ck, lane);
        stage_group(vst, vrow, t0, ncopy(t0), cv, lane);
        if (nmine > 1) {
          const int64_t t1 = group_t0(1);
          stage_group(kst + kTile * ck, krow, t1, ncopy(t1), ck, lane);
        }
        cp_async_commit();
        cp_async_wait_0();
        __syncwarp();
      }
      // K pass of group 0 on its own.
      float sc[G], p[G];
      {
        const uint8_t *kb = kst + lane * ck;
        RansLane rk = rans_open(smem, static_cast<uint32_t>(kb - smem));
#pragma unroll
        for (int g = 0; g < G; ++g) sc[g] = 0.0f;
#pragma unroll 4
        for (int i = 0; i < kD; ++i) {
          const uint32_t ek = rans_step<kTwoK>(rk, lut_k, smem);
          const float yk = *reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(lev) + ek);
          score_fma<G>(sc, qt + i * G, yk);
        }
        const bool valid = group_t0(0) + lane < c1;
        bad_count += __popc(__ballot_sync(kFull, valid && rk.x != kL));
        softmax_update(acc, sc, norm_of(kb), valid, p);
      }
      for (int64_t j = 0; j < nmine; ++j) {
        const int cur = static_cast<int>(j & 1), nxt = cur ^ 1;
        const bool has_next = j + 1 < nmine;
        // V(j) is in slot cur, K(j+1) in slot nxt (both staged). Weights of group j:
        {
          const uint8_t *vb = vst + cur * kTile * cv + lane * cv;
          const bool valid = group_t0(j) + lane < c1;
          const float nv = norm_of(vb);
#pragma unroll
          for (int g = 0; g < G; ++g) wbuf[lane * G + g] = valid ? p[g] * nv : 0.0f;
        }
        __syncwarp();
        // Prefetch K(j+2) into slot cur and V(j+1) into slot nxt.
        if (j + 2 < nmine) {
          const int64_t t2 = group_t0(j + 2);
          stage_group(kst + cur * kTile * ck, krow, t2, ncopy(t2), ck, lane);
        }
        if (has_next) {
          const int64_t t1 = group_t0(j + 1);
          stage_group(vst + nxt * kTile * cv, vrow, t1, ncopy(t1), cv, lane);
        }
        cp_async_commit();

        const uint8_t *kb = kst + nxt * kTile * ck + lane * ck;
        const uint8_t *vb = vst + cur * kTile * cv + lane * cv;
        RansLane rk = rans_open(smem, static_cast<uint32_t>(kb - smem));
        RansLane rv = rans_open(smem, static_cast<uint32_t>(vb - smem));
#pragma unroll
        for (int g = 0; g < G; ++g) sc[g] = 0.0f;
        float *trow = tile + lane * kTStride;
        auto run_half = [&](auto half_c) {
          constexpr int half = decltype(half_c)::value;
          if (has_next) {
#pragma unroll 2
            for (int i4 = 0; i4 < kHalf; i4 += 4) {
              float yv[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int i = half * kHalf + i4 + u;
                const uint32_t ek = rans_step<kTwoK>(rk, lut_k, smem);
                const uint32_t ev = rans_step<kTwoV>(rv, lut_v, smem);
                const float yk = *reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(lev) + ek);
                yv[u] = *reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(lev + kMaxLevels) + ev);
                score_fma<G>(sc, qt + i * G, yk);
              }
              *reinterpret_cast<float4 *>(trow + i4) = make_float4(yv[0], yv[1], yv[2], yv[3]);
            }
          } else {
#pragma unroll 2
            for (int i4 = 0; i4 < kHalf; i4 += 4) {
              float yv[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const uint32_t ev = rans_step<kTwoV>(rv, lut_v, smem);
                yv[u] = *reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(lev + kMaxLevels) + ev);
              }
              *reinterpret_cast<float4 *>(trow + i4) = make_float4(yv[0], yv[1], yv[2], yv[3]);
            }
          }
          __syncwarp();
          pv_half<G, half>(acc, tile, wbuf, lane);
          __syncwarp();
        };
        run_half(std::integral_constant<int, 0>{});
        run_half(std::integral_constant<int, 1>{});
        {
          const bool vvalid = group_t0(j) + lane < c1;
          bad_count += __popc(__ballot_sync(kFull, vvalid && rv.x != kL));
        }
        if (has_next) {
          const bool valid = group_t0(j + 1) + lane < c1;
          bad_count += __popc(__ballot_sync(kFull, valid && rk.x != kL));
          softmax_update(acc, sc, norm_of(kb), valid, p);
          // The next iteration needs V(j+1) (slot nxt) and K(j+2) (slot cur).
          cp_async_wait_0();
          __syncwarp();
        }
      }
      cp_async_wait_0();
    }
    // Sum the two half-groups of tokens.
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          acc.o[hh][g][c2].x += __shfl_xor_sync(kFull, acc.o[hh][g][c2].x, 16);
          acc.o[hh][g][c2].y += __shfl_xor_sync(kFull, acc.o[hh][g][c2].y, 16);
        }

    // D6: merge the warps' partial softmax states.
    __syncthreads();
    float *mrg_m = reinterpret_cast<float *>(smem + L.warp0);  // [nwarps][G]
    float *mrg_l = mrg_m + nwarps * G;                          // [nwarps][G]
    float *mrg_o = mrg_l + nwarps * G;                          // [nwarps][G][128]
    if (lane == 0)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        mrg_m[warp * G + g] = acc.m[g];
        mrg_l[warp * G + g] = acc.l[g];
      }
    if (lane < 16)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int g = 0; g < G; ++g)
          *reinterpret_cast<float4 *>(mrg_o + (warp * G + g) * kD + hh * kHalf + 4 * lane) =
              make_float4(acc.o[hh][g][0].x, acc.o[hh][g][0].y, acc.o[hh][g][1].x, acc.o[hh][g][1].y);
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * kD; idx += blockDim.x) {
      const int g = idx / kD, c = idx % kD;
      float M = -INFINITY;
      for (int w = 0; w < nwarps; ++w) M = fmaxf(M, mrg_m[w * G + g]);
      float o = 0.0f, l = 0.0f;
      if (M != -INFINITY)
        for (int w = 0; w < nwarps; ++w) {
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
  if (a.stats && lane == 0 && bad_count) atomicAdd(&a.stats->integrity_errors, static_cast<unsigned long long>(bad_count));
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

int warps_for(int G, int ck, int cv) {
  int nw = max_warps_for(G);
  while (nw > 1 && split_smem_layout(G, ck, cv, nw).total > 227 * 1024) --nw;
  return nw;
}

template <int G, bool kTwoK, bool kTwoV>
int launch_split(const DecodeArgs &a, cudaStream_t st) {
  const int nw = warps_for(G, a.ck, a.cv);
  const SplitSmem L = split_smem_layout(G, a.ck, a.cv, nw);
  auto kern = decode_split_kernel<G, kTwoK, kTwoV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
  if (e != cudaSuccess) return static_cast<int>(e);
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return static_cast<int>(e);
  const int64_t items = static_cast<int64_t>(a.B) * a.Hkv * a.splits;
  const int grid = static_cast<int>(items < sms ? items : sms);
  if (grid <= 0) return 0;
  kern<<<grid, nw * 32, L.total, st>>>(a);
  return static_cast<int>(cudaGetLastError());
}

template <int G>
int launch_split_g(const DecodeArgs &a, cudaStream_t st) {
  if (a.two_k && a.two_v) return launch_split<G, true, true>(a, st);
  if (a.two_k) return launch_split<G, true, false>(a, st);
  if (a.two_v) return launch_split<G, false, true>(a, st);
  return launch_split<G, false, false>(a, st);
}

}  // namespace

int launch_decode_attention(const DecodeArgs &a, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a.ck > kMaxContainer || a.cv > kMaxContainer) return static_cast<int>(cudaErrorInvalidValue);
  int e = 0;
  switch (a.G) {
    case 1: e = launch_split_g<1>(a, st); break;
    case 2: e = launch_split_g<2>(a, st); break;
    case 4: e = launch_split_g<4>(a, st); break;
    case 8: e = launch_split_g<8>(a, st); break;
    default: return static_cast<int>(cudaErrorInvalidValue);
  }
  if (e) return e;
  const int64_t rows = static_cast<int64_t>(a.B) * a.Hq;
  combine_kernel<<<static_cast<unsigned>((rows + 3) / 4), 128, 0, st>>>(a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dqi
