// dq_decode.cu -- decode attention over the compressed KV cache.
//
// [abstract] "D-Quant: Driftable Entropy Coding for KV Cache Quantization":
// fixed-size bitstreams give regular memory access and parallel
// dequantisation within attention kernels. [news] "D-Quant: Entropy Coding
// Meets KV Cache at 2.26 Bits", intro: rANS decoding runs inside the attention
// kernel; "The Numbers" 2nd paragraph: entropy decoding adds computation.
//
// Work split. The cache of sequence b, KV head h is cut into groups of 32
// tokens (one token per lane). All groups of all (b, h) are numbered in one
// flat order (b, then h, then token group) and every warp of the grid takes
// an equal contiguous range of that order, so the work is balanced to one
// group whatever the batch's lengths are. Where a warp's range crosses from
// one (b, h) to the next it writes the partial softmax state of the first
// and starts the next; partial states go to slot (b Hkv + h) + warp, which is
// unique because the warps' ranges are ordered. Warps never wait on each
// other: one persistent CTA per SM only shares the decode tables.
//
// Prefix kernel (one CTA): token groups per sequence and their prefix sums.
// Split kernel, per warp and per (b, h) segment of its range:
//   D1  q~ = H D q / 128 for the G query heads of h (times sm_scale log2 e)
//   D2  the warp stages 32 K and 32 V containers at a time (one 32-token
//       block of the cache, whose containers are byte-interleaved) into
//       shared memory with 16-byte cp.async, one group ahead; lane l reads
//       byte j of its container at offset 32 j + l, so the 32 lanes' byte
//       reads fall into different banks even after their cursors drift apart
//   D3  one lane per token: rANS-decode K (table look-up, multiply-add, byte
//       renormalisation) and accumulate q~ . y_hat for the G heads
//   D5  in the same loop the lane decodes V of the PREVIOUS group (whose
//       softmax weights are known) into a half-width (64-coordinate) fp16
//       tile of scaled levels, so every lane runs two independent rANS chains
//   D4  online softmax per head across the warp (score * ||k||)
//   D5' P.V on the tensor cores: o_rot^T[128 x G] += Y^T[128 x 32] w[32 x G]
//       per group with warp-level m16n8k16 fp16 MMAs, fp32 accumulation.
//       Y^T comes from the tile with ldmatrix.trans; w = p ||v|| is split
//       into two fp16 halves (hi + lo) so it keeps fp32 precision; the
//       levels are stored as fp16(kappa y) with a per-table kappa that makes
//       them exact to a few 1e-5 (relative), undone in the combine
//   D6  at the end of a segment the warp writes (m, l, o_rot) to its slot
// Combine kernel, one CTA per (b, query head), of 16 warps for small batches
// (hundreds of slots per row) and 4 otherwise:
//   D7  log-sum-exp merge of the slots of (b, h), o = D H o_rot / (128 l)
#include <type_traits>

#include "dq_device.cuh"

namespace dqi {
namespace {

constexpr int kMaxWarps = 16;      // warps per CTA (one persistent CTA per SM)
constexpr int kTile = 32;          // tokens per warp group (one per lane)
constexpr int kHalf = 64;          // coordinates per V tile pass
constexpr int kTileRow = kHalf * 2;  // bytes per token row of the fp16 V tile
constexpr int kWhStride = 40;      // halves per head row of the weight buffer
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

// Shared-memory layout of the split kernel: the decode tables shared by the
// CTA, then one area per warp with its staging slots, V tile, softmax-weight
// buffer (fp16 hi and lo, [2][8 heads][kWhStride]) and q~.
struct SplitSmem {
  size_t lut_k, lut_v, lev, warp0, warp_bytes;
  size_t kst, vst, tile, wbuf, qt;  // offsets inside a warp's area
  size_t total;
};

__host__ __device__ inline SplitSmem split_smem_layout(int G, int ck, int cv, int nwarps) {
  SplitSmem s;
  s.lut_k = 0;
  s.lut_v = s.lut_k + kM * 4;
  s.lev = s.lut_v + kM * 4;
  s.warp0 = align16(s.lev + 2 * kMaxLevels * 4);
  s.kst = 0;                                                        // 2 slots of 32 K containers
  s.vst = align16(2 * static_cast<size_t>(kTile) * ck);             // 2 slots of 32 V containers
  s.tile = s.vst + align16(2 * static_cast<size_t>(kTile) * cv);    // [32 tokens][64] fp16, swizzled
  s.wbuf = s.tile + static_cast<size_t>(kTile) * kTileRow;          // [2][8][kWhStride] fp16
  s.qt = s.wbuf + 2 * 8 * kWhStride * 2;                            // [128][G] floats
  s.warp_bytes = align16(s.qt + static_cast<size_t>(kD) * G * 4);
  // A corrupt container can make its decoder's cursor run past the
  // container, by at most 2 bytes per symbol (byte 5 + 2 * 128 at most),
  // i.e. 32 * 261 bytes from the staged block in the interleaved layout.
  // Those reads only produce garbage (flagged by the final-state check); the
  // slack keeps the last warp's reads inside the CTA's shared memory.
  const size_t reach = s.vst + static_cast<size_t>(kTile) * cv + static_cast<size_t>(kTile) * (kHeaderBytes + 2 * kD + 1);
  const size_t slack = reach > s.warp_bytes ? align16(reach - s.warp_bytes) + 256 : 256;
  s.total = s.warp0 + static_cast<size_t>(nwarps) * s.warp_bytes + slack;
  return s;
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Copies one 32-token block (32 C bytes, a multiple of 16) of a cache into
// shared memory, 16 bytes per copy.
__device__ __forceinline__ void stage_block(uint8_t *dst, const uint8_t *src, int C, int lane) {
  const int chunks = (kTile * C) >> 4;
  for (int c = lane; c < chunks; c += 32) cp_async16(dst + c * 16, src + c * 16);
}

// rANS decoder state of one lane: the 32-bit state and the shared-memory
// offset (from the kernel's shared base) of the next container byte; byte j
// of the lane's container is 32 j past byte 0.
struct RansLane {
  uint32_t x;
  uint32_t p;
};

__device__ __forceinline__ RansLane rans_open(const uint8_t *smem, uint32_t off) {
  RansLane r;
  r.x = static_cast<uint32_t>(smem[off + 2 * kTile]) | (static_cast<uint32_t>(smem[off + 3 * kTile]) << 8) |
        (static_cast<uint32_t>(smem[off + 4 * kTile]) << 16);
  r.p = off + kHeaderBytes * kTile;
  return r;
}

#ifdef DQ_CHECKED
// Whether a lane's decoder consumed bytes past its container of C bytes at
// cb (the cursor starts at byte 5 and moves 32 per byte consumed). Counted in
// dq_stats.overreads by DQ_CHECKED builds.
__device__ __forceinline__ bool overread(const RansLane &r, const uint8_t *cb, const uint8_t *smem, int C) {
  return r.p > static_cast<uint32_t>(cb - smem) + static_cast<uint32_t>(C) * kTile;
}
#endif

// One decode step. Table entry layout: bits 0..10 slot - c_s, bits 11..13 the
// symbol s, bits 20..31 f_s. The state advances as x = f (x >> 12) + (slot -
// c_s). Renormalisation has no branches: while x < 2^16 the next byte b is
// shifted in (x = 256 x + b) and the cursor moves, both as selects (fewer
// instructions than an arithmetic 0/1 multiplier, which measured 3-6 %
// slower). A second byte can only be needed after a symbol with f < 16
// (x >= 16 f after the step); kTwo enables that step for tables that have
// such a symbol. The byte reads never
// leave the kernel's shared memory (the cursor moves at most 2 bytes per
// symbol and the layout leaves room for that). Returns the byte offset 4 s
// of the symbol's level.
template <bool kTwo>
__device__ __forceinline__ uint32_t rans_step(RansLane &r, const uint32_t *lut, const uint8_t *smem) {
  const uint32_t e = lut[r.x & (kM - 1)];
  uint32_t x = (e >> 20) * (r.x >> kProbBits) + (e & 0x7FFu);
  const uint32_t b0 = smem[r.p];
  const uint32_t b1 = kTwo ? static_cast<uint32_t>(smem[r.p + kTile]) : 0u;
  uint32_t p = r.p;
  const bool lo0 = x < kL;
  x = lo0 ? (x * 256u + b0) : x;
  p = lo0 ? p + kTile : p;
  if constexpr (kTwo) {
    const bool lo1 = x < kL;
    x = lo1 ? (x * 256u + b1) : x;
    p = lo1 ? p + kTile : p;
  }
  r.p = p;
  r.x = x;
  return (e >> 9) & 0x1Cu;
}

// fp16 norm in bytes 0 and 1 of a staged (interleaved) container.
__device__ __forceinline__ float norm_of(const uint8_t *cb) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(cb[0] | (cb[kTile] << 8))));
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

// Byte offset in the V tile of token t's 16-byte chunk c (8 coordinates):
// chunks are XOR-swizzled by t & 7, so a lane's 128-bit store of its own row
// and an 8-row ldmatrix both touch 8 different 16-byte bank groups.
__device__ __forceinline__ uint32_t tile_off(int t, int c) {
  return static_cast<uint32_t>(t * kTileRow + ((c ^ (t & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr)
               : "memory");
}

// d += a b for one m16n8k16 tile: fp16 operands, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Per-warp state of one segment's online softmax and P.V accumulators. The
// accumulators are the m16n8 C fragments of o_rot^T: c[mt] covers
// coordinates 16 mt .. 16 mt + 15; lane l holds coordinates 16 mt + l / 4
// (+ 8) of heads 2 (l % 4) and 2 (l % 4) + 1 (heads >= G stay zero).
template <int G>
struct WarpAcc {
  float m[G], l[G];
  float c[kD / 16][4];
};

// P.V for one 64-coordinate half of the current group: A = Y^T (16
// coordinates x 16 tokens) by ldmatrix.trans from the tile, B = the group's
// weights (16 tokens x 8 heads) as fp16 hi and lo fragments.
template <int half>
__device__ __forceinline__ void pv_mma_half(float (&c)[kD / 16][4], uint32_t tile_s, const uint32_t (&bh)[2][2],
                                            const uint32_t (&bl)[2][2], int lane) {
  const int r = (lane & 7) + ((lane >> 4) & 1) * 8;  // token row within a 16-token step
  const int cadd = (lane >> 3) & 1;                   // second 8 coordinates of the m-tile
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      uint32_t a[4];
      ldsm_x4_trans(a, tile_s + tile_off(ks * 16 + r, 2 * mt + cadd));
      mma_16816(c[half * 4 + mt], a, bh[ks][0], bh[ks][1]);
      mma_16816(c[half * 4 + mt], a, bl[ks][0], bl[ks][1]);
    }
  }
}

// Online-softmax update for one group's scores (lane = token); keeps the
// probabilities p (without the V norm) in `p` for the caller.
template <int G>
__device__ __forceinline__ void softmax_update(WarpAcc<G> &acc, const float (&sc)[G], float nk, bool valid,
                                               float (&p)[G], int lane) {
  float alpha[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float s = valid ? sc[g] * nk : -INFINITY;
    const float m_new = fmaxf(acc.m[g], warp_max(s));
    alpha[g] = 1.0f;
    p[g] = 0.0f;
    if (m_new != -INFINITY) {
      p[g] = exp2f(s - m_new);
      alpha[g] = exp2f(acc.m[g] - m_new);
    }
    acc.l[g] = acc.l[g] * alpha[g] + warp_sum(p[g]);
    acc.m[g] = m_new;
  }
  // This lane's accumulators belong to heads 2 (lane % 4) and 2 (lane % 4) + 1.
  float aa = 1.0f, ab = 1.0f;
  const int cq = lane & 3;
#pragma unroll
  for (int g2 = 0; 2 * g2 < G; ++g2)
    if (cq == g2) {
      aa = alpha[2 * g2];
      ab = (2 * g2 + 1 < G) ? alpha[2 * g2 + 1] : 1.0f;
    }
  const float2 a2 = make_float2(aa, ab);
#pragma unroll
  for (int mt = 0; mt < kD / 16; ++mt) {
    const float2 lo = __fmul2_rn(make_float2(acc.c[mt][0], acc.c[mt][1]), a2);
    const float2 hi = __fmul2_rn(make_float2(acc.c[mt][2], acc.c[mt][3]), a2);
    acc.c[mt][0] = lo.x; acc.c[mt][1] = lo.y; acc.c[mt][2] = hi.x; acc.c[mt][3] = hi.y;
  }
}

__device__ __forceinline__ int64_t clamp_len(int32_t len, int64_t cap) {
  int64_t v = len;
  if (v < 0) v = 0;
  if (v > cap) v = cap;
  return v;
}

// First flat group index of warp w out of W over N groups (warp w owns
// [first(w), first(w + 1))).
__host__ __device__ __forceinline__ int64_t warp_first(int64_t w, int64_t W, int64_t N) { return (w * N) / W; }

// Warps that split N groups out of the grid's `total`: min(total, N). With
// W <= N every warp owns at least one group, so the warps whose ranges meet
// a (b, h) form one contiguous run with no empty warp in it; with W = N warp
// w owns exactly group w.
__host__ __device__ __forceinline__ int64_t active_warps(int64_t total, int64_t N) { return total < N ? total : N; }

// Token groups per sequence and their prefix sums: prefix[b] = groups of
// sequences 0..b-1, prefix[B] = total. One CTA of kPrefixThreads threads;
// also counts the sequence lengths that had to be clamped.
constexpr int kPrefixThreads = 1024;

__global__ void __launch_bounds__(kPrefixThreads) prefix_kernel(const DecodeArgs a) {
  __shared__ int64_t warp_tot[kPrefixThreads / 32];
  __shared__ int64_t carry_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t cap = a.T_max < a.T_cap ? a.T_max : a.T_cap;
  if (threadIdx.x == 0) {
    carry_s = 0;
    a.prefix[0] = 0;
  }
  unsigned clamped = 0;
  __syncthreads();
  for (int base = 0; base < a.B; base += kPrefixThreads) {
    const int i = base + static_cast<int>(threadIdx.x);
    int64_t v = 0;
    if (i < a.B) {
      const int32_t len = a.seq_lens[i];
      if (len < 0 || len > cap) ++clamped;
      v = (clamp_len(len, cap) + kTile - 1) / kTile;
    }
    int64_t inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t nb = __shfl_up_sync(kFull, inc, o);
      if (lane >= o) inc += nb;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int64_t before = carry_s;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    if (i < a.B) a.prefix[i + 1] = before + inc;
    __syncthreads();  // everyone has read carry_s and warp_tot
    if (threadIdx.x == kPrefixThreads - 1) carry_s = before + inc;
    __syncthreads();
  }
  if (a.stats) {
    const unsigned c = static_cast<unsigned>(warp_sum(static_cast<float>(clamped)));
    if (lane == 0 && c) atomicAdd(&a.stats->clamped_lengths, static_cast<unsigned long long>(c));
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
  float *lev = reinterpret_cast<float *>(smem + L.lev);  // [0..7] K levels, [8..15] V fp16 bits
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t *wsm = smem + L.warp0 + warp * L.warp_bytes;
  uint8_t *kst = wsm + L.kst;
  uint8_t *vst = wsm + L.vst;
  const uint32_t tile_s = static_cast<uint32_t>(__cvta_generic_to_shared(wsm + L.tile));
  uint16_t *wh = reinterpret_cast<uint16_t *>(wsm + L.wbuf);  // [hi, lo][8 heads][kWhStride]
  const uint32_t *whw = reinterpret_cast<const uint32_t *>(wh);
  float *qt = reinterpret_cast<float *>(wsm + L.qt);  // [128][G]
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
      reinterpret_cast<uint32_t *>(lev)[kMaxLevels + threadIdx.x] = a.tabs->v.level16[threadIdx.x];
    }
  }
  __syncthreads();

  const int64_t cap = a.T_max < a.T_cap ? a.T_max : a.T_cap;
  const int64_t Hkv = a.Hkv;
  const int64_t N = a.prefix[a.B] * Hkv;  // total token groups
  // Warps that take part: all of them, or one per group when there are
  // fewer groups than warps, so that no participating warp is empty.
  const int64_t W = active_warps(static_cast<int64_t>(gridDim.x) * nwarps, N);
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * nwarps + warp;
  if (wid >= W) return;
  int64_t g = warp_first(wid, W, N);
  const int64_t g_end = warp_first(wid + 1, W, N);
  if (g >= g_end) return;
  unsigned bad_count = 0;
#ifdef DQ_CHECKED
  unsigned over_count = 0;
#endif
  unsigned bad_pages = 0;

  // Sequence holding flat group g: the largest b with prefix[b] * Hkv <= g
  // (it has tokens, since g < prefix[b + 1] * Hkv).
  int b = 0;
  {
    int lo = 0, hi = a.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.prefix[mid] * Hkv <= g) lo = mid;
      else hi = mid - 1;
    }
    b = lo;
  }
  int64_t gb = a.prefix[b + 1] - a.prefix[b];  // token groups per head of sequence b
  int h = static_cast<int>((g - a.prefix[b] * Hkv) / gb);
  int64_t j0 = (g - a.prefix[b] * Hkv) % gb;

  while (true) {
    const int64_t n = (g_end - g) < (gb - j0) ? (g_end - g) : (gb - j0);  // groups in this segment
    const int64_t len = clamp_len(a.seq_lens[b], cap);
    const int64_t bh = static_cast<int64_t>(b) * Hkv + h;

    // D1: q~ = H D q / 128 for the G query heads of KV head h, times sm_scale log2 e.
    {
      uint32_t sw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) sw[k] = __ldg(a.sign_bits + h * 4 + k);
      const float qscale = a.sm_scale * kLog2e / static_cast<float>(kD);
#pragma unroll 1
      for (int gg = 0; gg < G; ++gg) {
        const int64_t qbase = (static_cast<int64_t>(b) * a.Hq + h * G + gg) * kD;
        float v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = apply_sign(load_elem(a.q, qbase + lane + 32 * k, a.q_dtype), sw[k], lane);
        wht128_warp(v, lane);
#pragma unroll
        for (int k = 0; k < 4; ++k) qt[(lane + 32 * k) * G + gg] = v[k] * qscale;
      }
    }

    const int64_t tseg = j0 * kTile;
    auto group_t0 = [&](int64_t j) { return tseg + j * kTile; };
    // Cache block (32 tokens of one KV head) holding group j of the segment:
    // block b of a cache sits at byte 32 C b. Contiguous caches: row bh,
    // token block t / 32. Paged caches: page_table[b][t / 32] * Hkv + h; an
    // entry out of range is counted and read as page 0 (garbage, no fault).
    auto block_of = [&](int64_t j) -> int64_t {
      const int64_t tb = (tseg >> 5) + j;
      if (a.page_table) {
        int64_t pg = a.page_table[static_cast<int64_t>(b) * a.max_pages + tb];
        if (pg < 0 || pg >= a.num_pages) {
          ++bad_pages;
          pg = 0;
        }
        return pg * Hkv + h;
      }
      return bh * (a.T_cap / kTile) + tb;
    };
    auto kblock = [&](int64_t blk) { return a.kcache + blk * kTile * ck; };
    auto vblock = [&](int64_t blk) { return a.vcache + blk * kTile * cv; };

    WarpAcc<G> acc;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      acc.m[gg] = -INFINITY;
      acc.l[gg] = 0.0f;
    }
#pragma unroll
    for (int mt = 0; mt < kD / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc.c[mt][e] = 0.0f;

    // Prologue: K(0), V(0) into slot 0 and K(1) into K slot 1. Invariant at
    // the top of iteration j: V(j) sits in V slot j%2 and K(j+1) in K slot
    // (j+1)%2, both complete; iteration j prefetches K(j+2) and V(j+1).
    // Block ids run one iteration ahead of their use: bj1 = block of group
    // j+1, bj2 = block of group j+2 at the top of iteration j.
    int64_t bj1 = 0, bj2 = 0;
    {
      const int64_t b0 = block_of(0);
      stage_block(kst, kblock(b0), ck, lane);
      stage_block(vst, vblock(b0), cv, lane);
      if (n > 1) {
        bj1 = block_of(1);
        stage_block(kst + kTile * ck, kblock(bj1), ck, lane);
      }
      if (n > 2) bj2 = block_of(2);
      cp_async_commit();
      cp_async_wait_0();
      __syncwarp();  // staged bytes and q~ visible to the whole warp
    }
    // K pass of group 0 on its own.
    float sc[G], p[G];
    {
      const uint8_t *kb = kst + lane;
      RansLane rk = rans_open(smem, static_cast<uint32_t>(kb - smem));
#pragma unroll
      for (int gg = 0; gg < G; ++gg) sc[gg] = 0.0f;
#pragma unroll 4
      for (int i = 0; i < kD; ++i) {
        const uint32_t ek = rans_step<kTwoK>(rk, lut_k, smem);
        const float yk = *reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(lev) + ek);
        score_fma<G>(sc, qt + i * G, yk);
      }
      const bool valid = group_t0(0) + lane < len;
      bad_count += __popc(__ballot_sync(kFull, valid && rk.x != kL));
#ifdef DQ_CHECKED
      over_count += __popc(__ballot_sync(kFull, valid && overread(rk, kb, smem, ck)));
#endif
      softmax_update(acc, sc, norm_of(kb), valid, p, lane);
    }
    for (int64_t j = 0; j < n; ++j) {
      const int cur = static_cast<int>(j & 1), nxt = cur ^ 1;
      const bool has_next = j + 1 < n;
      // V(j) is in slot cur, K(j+1) in slot nxt (both staged). Weights of
      // group j, w = p ||v||, as fp16 hi + lo, then this lane's B fragments:
      // b[ks][0] holds tokens 16 ks + 2 (lane % 4) + {0, 1} of head lane / 4,
      // b[ks][1] the same tokens + 8 (zero for heads >= G).
      uint32_t fb_hi[2][2], fb_lo[2][2];
      {
        const uint8_t *vb = vst + cur * kTile * cv + lane;
        const bool valid = group_t0(j) + lane < len;
        const float nv = norm_of(vb);
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          const float w = valid ? p[gg] * nv : 0.0f;
          const __half hi = __float2half_rn(w);
          const __half lo = __float2half_rn(w - __half2float(hi));
          wh[gg * kWhStride + lane] = __half_as_ushort(hi);
          wh[(8 + gg) * kWhStride + lane] = __half_as_ushort(lo);
        }
        __syncwarp();
        const int n_head = lane >> 2, cq = lane & 3;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int word = n_head * (kWhStride / 2) + ks * 8 + r * 4 + cq;
            fb_hi[ks][r] = n_head < G ? whw[word] : 0u;
            fb_lo[ks][r] = n_head < G ? whw[8 * (kWhStride / 2) + word] : 0u;
          }
      }
      // Prefetch K(j+2) into slot cur and V(j+1) into slot nxt.
      if (j + 2 < n) stage_block(kst + cur * kTile * ck, kblock(bj2), ck, lane);
      if (has_next) stage_block(vst + nxt * kTile * cv, vblock(bj1), cv, lane);
      cp_async_commit();
      bj1 = bj2;
      if (j + 3 < n) bj2 = block_of(j + 3);

      const uint8_t *kb = kst + nxt * kTile * ck + lane;
      const uint8_t *vb = vst + cur * kTile * cv + lane;
      RansLane rk = rans_open(smem, static_cast<uint32_t>(kb - smem));
      RansLane rv = rans_open(smem, static_cast<uint32_t>(vb - smem));
#pragma unroll
      for (int gg = 0; gg < G; ++gg) sc[gg] = 0.0f;
      const uint32_t *lev16 = reinterpret_cast<const uint32_t *>(lev + kMaxLevels);
      auto run_half = [&](auto half_c) {
        constexpr int half = decltype(half_c)::value;
#pragma unroll 1
        for (int i8 = 0; i8 < kHalf; i8 += 8) {
          uint32_t hv[8];
          if (has_next) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = half * kHalf + i8 + u;
              const uint32_t ek = rans_step<kTwoK>(rk, lut_k, smem);
              const uint32_t ev = rans_step<kTwoV>(rv, lut_v, smem);
              const float yk = *reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(lev) + ek);
              hv[u] = *reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint8_t *>(lev16) + ev);
              score_fma<G>(sc, qt + i * G, yk);
            }
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const uint32_t ev = rans_step<kTwoV>(rv, lut_v, smem);
              hv[u] = *reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint8_t *>(lev16) + ev);
            }
          }
          const uint4 pk = make_uint4(__byte_perm(hv[0], hv[1], 0x5410), __byte_perm(hv[2], hv[3], 0x5410),
                                      __byte_perm(hv[4], hv[5], 0x5410), __byte_perm(hv[6], hv[7], 0x5410));
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(tile_s + tile_off(lane, i8 >> 3)),
                       "r"(pk.x), "r"(pk.y), "r"(pk.z), "r"(pk.w)
                       : "memory");
        }
        __syncwarp();
        pv_mma_half<half>(acc.c, tile_s, fb_hi, fb_lo, lane);
        __syncwarp();
      };
      run_half(std::integral_constant<int, 0>{});
      run_half(std::integral_constant<int, 1>{});
      {
        const bool vvalid = group_t0(j) + lane < len;
        bad_count += __popc(__ballot_sync(kFull, vvalid && rv.x != kL));
#ifdef DQ_CHECKED
        over_count += __popc(__ballot_sync(kFull, vvalid && overread(rv, vb, smem, cv)));
#endif
      }
      if (has_next) {
        const bool valid = group_t0(j + 1) + lane < len;
        bad_count += __popc(__ballot_sync(kFull, valid && rk.x != kL));
#ifdef DQ_CHECKED
        over_count += __popc(__ballot_sync(kFull, valid && overread(rk, kb, smem, ck)));
#endif
        softmax_update(acc, sc, norm_of(kb), valid, p, lane);
        // The next iteration needs V(j+1) (slot nxt) and K(j+2) (slot cur).
        cp_async_wait_0();
        __syncwarp();
      }
    }
    cp_async_wait_0();
    __syncwarp();  // staging and q~ areas are free for the next segment

    // D6: write this segment's state (o_rot in units of the V tile scale).
    const int64_t slot = bh + wid;
    if (lane == 0)
#pragma unroll
      for (int gg = 0; gg < G; ++gg)
        *reinterpret_cast<float2 *>(a.ws_ml + (slot * G + gg) * 2) = make_float2(acc.m[gg], acc.l[gg]);
    {
      const int row = lane >> 2, head0 = 2 * (lane & 3);
#pragma unroll
      for (int mt = 0; mt < kD / 16; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int head = head0 + (e & 1);
          if (head < G) a.ws_o[(slot * G + head) * kD + 16 * mt + row + 8 * (e >> 1)] = acc.c[mt][e];
        }
    }

    g += n;
    if (g >= g_end) break;
    // Next segment: the following head of b, else the next sequence with tokens.
    j0 = 0;
    if (++h == a.Hkv) {
      h = 0;
      do {
        ++b;
      } while (a.prefix[b + 1] == a.prefix[b]);
      gb = a.prefix[b + 1] - a.prefix[b];
    }
  }
  if (a.stats && lane == 0 && bad_count) atomicAdd(&a.stats->integrity_errors, static_cast<unsigned long long>(bad_count));
  if (a.stats && lane == 0 && bad_pages) atomicAdd(&a.stats->bad_pages, static_cast<unsigned long long>(bad_pages));
#ifdef DQ_CHECKED
  if (a.stats && lane == 0 && over_count) atomicAdd(&a.stats->overreads, static_cast<unsigned long long>(over_count));
#endif
}

// Combine: one CTA of kCombWarps warps per (b, query head). The warps split
// the row's slots into contiguous chunks; a warp takes its chunk 32 slots at
// a time (lane i reads slot i's (m, l), so the batch's weights come from one
// load per lane and one max/sum over the warp; the partial o vectors of the
// batch are then read with independent loads), merging batch after batch
// with an online rescale. The warps' results meet in shared memory. With a
// small batch a row has hundreds of slots (one per split warp) and few rows
// run at once, so the host takes 16 warps per CTA there (the merge is a
// chain of load batches, latency-bound), 4 otherwise.
template <int kCombWarps>
__global__ void __launch_bounds__(kCombWarps * 32) combine_kernel(const DecodeArgs a) {
  __shared__ float sh_m[kCombWarps], sh_l[kCombWarps];
  __shared__ float sh_o[kCombWarps][kD];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = blockIdx.x;  // b * Hq + hq
  const int b = static_cast<int>(row / a.Hq), hq = static_cast<int>(row % a.Hq);
  const int G = a.G;
  const int h = hq / G, gg = hq % G;
  const int64_t Hkv = a.Hkv;
  const int64_t gb = a.prefix[b + 1] - a.prefix[b];
  const int64_t bh = static_cast<int64_t>(b) * Hkv + h;
  float M = -INFINITY, Ls = 0.0f;
  float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (gb > 0) {
    // The warps whose ranges meet groups [g0, g1) of (b, h) are the
    // contiguous run from the owner of g0 to the owner of g1 - 1 (owner(g) =
    // the largest w with first(w) <= g); none of them is empty (W <= N), and
    // each wrote its partial state of (b, h) to slot bh + w.
    const int64_t N = a.prefix[a.B] * Hkv;
    const int64_t W = active_warps(a.total_warps, N);
    const int64_t g0 = a.prefix[b] * Hkv + h * gb, g1 = g0 + gb;
    const int64_t w_lo = ((g0 + 1) * W - 1) / N;
    const int64_t w_hi = (g1 * W - 1) / N;
    const int64_t S = w_hi - w_lo + 1;
    const int64_t cs = (S + kCombWarps - 1) / kCombWarps;
    const int64_t c0 = w_lo + warp * cs;
    const int64_t c1 = (c0 + cs < w_hi + 1) ? c0 + cs : w_hi + 1;
    const float2 *ml = reinterpret_cast<const float2 *>(a.ws_ml);
    for (int64_t base = c0; base < c1; base += 32) {
      const int64_t w = base + lane;
      float2 s = make_float2(-INFINITY, 0.0f);
      if (w < c1) s = ml[(bh + w) * G + gg];
      const float bm = warp_max(s.x);
      if (bm == -INFINITY) continue;  // all segments of the batch empty
      const float m_new = fmaxf(M, bm);
      const float r = exp2f(M - m_new);  // 0 while M is -inf
      Ls *= r;
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] *= r;
      M = m_new;
      const float sc = exp2f(s.x - M);  // 0 for lanes past the chunk or empty segments
      Ls += warp_sum(sc * s.y);
      const int nb = static_cast<int>((c1 - base) < 32 ? (c1 - base) : 32);
#pragma unroll 8
      for (int i = 0; i < nb; ++i) {
        const float si = __shfl_sync(kFull, sc, i);
        const float *o = a.ws_o + ((bh + base + i) * G + gg) * kD + lane;
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = fmaf(si, o[32 * k], v[k]);
      }
    }
  }
  if (lane == 0) {
    sh_m[warp] = M;
    sh_l[warp] = Ls;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) sh_o[warp][lane + 32 * k] = v[k];
  __syncthreads();
  if (warp != 0) return;
  float Mt = -INFINITY;
#pragma unroll
  for (int w = 0; w < kCombWarps; ++w) Mt = fmaxf(Mt, sh_m[w]);
  float Lt = 0.0f;
  float o[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  if (Mt != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kCombWarps; ++w) {
      const float r = exp2f(sh_m[w] - Mt);  // 0 for a warp without slots
      Lt = fmaf(r, sh_l[w], Lt);
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] = fmaf(r, sh_o[w][lane + 32 * k], o[k]);
    }
  }
  const float inv = (Lt > 0.0f) ? 1.0f / (Lt * static_cast<float>(kD) * a.tabs->v.tile_scale) : 0.0f;
  wht128_warp(o, lane);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t sw = __ldg(a.sign_bits + h * 4 + k);
    const float y = apply_sign(o[k] * inv, sw, lane);
    store_elem(a.out, row * kD + lane + 32 * k, y, a.out_dtype);
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
  if (static_cast<int64_t>(a.grid) * nw != a.total_warps) return static_cast<int>(cudaErrorInvalidValue);
  const SplitSmem L = split_smem_layout(G, a.ck, a.cv, nw);
  constexpr auto kern = decode_split_kernel<G, kTwoK, kTwoV>;
  const cudaError_t e = ensure_max_dynamic_smem<kern>(static_cast<int>(L.total));
  if (e != cudaSuccess) return static_cast<int>(e);
  kern<<<a.grid, nw * 32, L.total, st>>>(a);
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

int decode_warps_per_cta(int G, int ck, int cv) {
  if (G != 1 && G != 2 && G != 4 && G != 8) return 0;
  if (ck < 1 || cv < 1 || ck > kMaxContainer || cv > kMaxContainer) return 0;
  return warps_for(G, ck, cv);
}

int launch_decode_attention(const DecodeArgs &a, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a.ck > kMaxContainer || a.cv > kMaxContainer || a.grid < 1) return static_cast<int>(cudaErrorInvalidValue);
  prefix_kernel<<<1, kPrefixThreads, 0, st>>>(a);
  const cudaError_t ce = cudaGetLastError();
  if (ce != cudaSuccess) return static_cast<int>(ce);
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
  if (rows > 0x7FFFFFFF) return static_cast<int>(cudaErrorInvalidValue);
  // At least 64 slots per (b, KV head) possible: wide CTAs.
  if (a.total_warps >= static_cast<int64_t>(64) * a.B * a.Hkv)
    combine_kernel<16><<<static_cast<unsigned>(rows), 16 * 32, 0, st>>>(a);
  else
    combine_kernel<4><<<static_cast<unsigned>(rows), 4 * 32, 0, st>>>(a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dqi
