// dq_append.cu -- append/encode path: rotate, normalise, quantise, rANS-encode
// and drift each new K/V head vector into its fixed-size container.
//
// [news] "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits":
//   "Why Fixed Width Is a Ceiling" -- after rotation and normalisation the
//   coordinates are close to N(0,1);
//   "Drift: Bending Variable Back to Fixed" -- each token's K or V goes into a
//   fixed-size byte container, rANS-coded; an over-long stream has a few
//   symbols drift from high-cost to nearby lower-cost symbols until it fits,
//   none by more than one level.
// [abstract] "D-Quant: Driftable Entropy Coding for KV Cache Quantization".
//
// Every fp32 operation uses an explicitly rounded intrinsic (__fadd_rn,
// __fmul_rn, __fdiv_rn, __fsqrt_rn) so no multiply-add is contracted: the
// containers are bit-identical to the format's definition.
//
// Work split: one warp takes `vpw` (1..32) vectors of one stream.
//   phase 1 (warp per vector): E1 sign flip, E2 Walsh-Hadamard transform
//     (shuffles for stages 1..16, registers for 32 and 64), E3 norm in a fixed
//     tree, scale, fp16 norm, E4 quantisation; u and symbols to shared memory.
//   phase 2 (lane per vector): E5 rANS encode last-to-first; containers that
//     fit are stored at once.
//   phase 3 (warp per over-long container): E6 drift. The greedy rule (least
//     key first, ties to the lower index) applies moves in a fixed order, so
//     the warp ranks the candidate moves by repeated arg-min and lane m
//     encodes the string with the first m+1 moves applied; the smallest m that
//     fits is the greedy result. 32 move counts are tried per pass.
#include "dq_device.cuh"

namespace dqi {
namespace {

constexpr int kAW = 4;  // warps per CTA
constexpr int kUStride = kD + 1;
constexpr int kQStride = kD + 4;
constexpr int kStack = kMaxContainer;
constexpr float kSqrtD = 11.3137084989847604f;  // fl32(sqrt(128))
constexpr uint8_t kNoRank = 255;

struct AppendTables {
  float lev[kMaxLevels], thr[kMaxLevels], cost[kMaxLevels];
  uint32_t freq[kMaxLevels], cum[kMaxLevels];
  unsigned long long rcp[kMaxLevels];  // ceil(2^40 / f)
};

// Per-warp shared-memory area; vpw vectors per warp.
struct WarpArea {
  float *u;           // [vpw][kUStride]
  uint8_t *q;         // [vpw][kQStride]
  uint8_t *stack;     // [32][kStack]
  uint8_t *rank;      // [128] move rank of each symbol, kNoRank if none yet
  uint8_t *tgt;       // [128] level a drifted symbol moves to
  uint16_t *norm16;   // [vpw]
  uint8_t *nonfinite; // [vpw]
};

__host__ __device__ inline size_t warp_area_bytes(int vpw) {
  size_t b = static_cast<size_t>(vpw) * kUStride * 4;
  b += static_cast<size_t>(vpw) * kQStride;
  b += 32 * kStack + 128 + 128;
  b += static_cast<size_t>(vpw) * 2 + vpw;
  return (b + 15) & ~size_t(15);
}

__device__ inline WarpArea warp_area(uint8_t *base, int vpw) {
  WarpArea w;
  uint8_t *p = base;
  w.u = reinterpret_cast<float *>(p);
  p += static_cast<size_t>(vpw) * kUStride * 4;
  w.q = p;
  p += static_cast<size_t>(vpw) * kQStride;
  w.stack = p;
  p += 32 * kStack;
  w.rank = p;
  p += 128;
  w.tgt = p;
  p += 128;
  w.norm16 = reinterpret_cast<uint16_t *>(p);
  p += static_cast<size_t>(vpw) * 2;
  w.nonfinite = p;
  return w;
}

// Exact x / f and x mod f for x < 2^24 and 1 <= f <= 4096 with M = ceil(2^40 / f):
// x M / 2^40 = x / f + d with 0 <= d < x / 2^40 < 2^-16 < 1 / f, so the floor
// is x / f.
__device__ __forceinline__ uint32_t div_rcp(uint32_t x, unsigned long long M) {
  return static_cast<uint32_t>((static_cast<unsigned long long>(x) * M) >> 40);
}

// E5: rANS-encode 128 symbols, coded 127 -> 0, starting from x = 2^16.
// sym(i) gives symbol i. Pushed bytes go to `stack` in push order. Returns the
// total length 3 + #pushed, or cap + 1 as soon as it exceeds `cap`.
template <typename SymFn>
__device__ __forceinline__ int rans_encode(SymFn sym, const AppendTables &T, uint8_t *stack, int cap,
                                           uint32_t *x_out) {
  uint32_t x = kL;
  int np = 0;
  const int max_push = cap - 3;
  for (int i = kD - 1; i >= 0; --i) {
    const uint32_t s = sym(i);
    const uint32_t f = T.freq[s];
    const uint32_t xmax = ((kL >> kProbBits) << 8) * f;
    while (x >= xmax) {
      if (np >= max_push) return cap + 1;
      stack[np++] = static_cast<uint8_t>(x & 0xFFu);
      x >>= 8;
    }
    const uint32_t qf = div_rcp(x, T.rcp[s]);
    x = qf * kM + (x - qf * f) + T.cum[s];
  }
  *x_out = x;
  return 3 + np;
}

// Writes one container; byte k goes to dst[32 k] (the cache interleaves the
// bytes of the 32 tokens of a block).
__device__ __forceinline__ void store_container(uint8_t *dst, int C, uint16_t n16, uint32_t x, const uint8_t *stack,
                                                int len) {
  const int np = len - 3;
  for (int k = 0; k < C; ++k) {
    uint8_t byte;
    if (k == 0) byte = static_cast<uint8_t>(n16 & 0xFFu);
    else if (k == 1) byte = static_cast<uint8_t>(n16 >> 8);
    else if (k < 5) byte = static_cast<uint8_t>((x >> (8 * (k - 2))) & 0xFFu);
    else if (k - 5 < np) byte = stack[np - 1 - (k - 5)];
    else byte = 0;
    dst[32 * k] = byte;
  }
}

// Best drift move of symbol i (one level toward a strictly cheaper neighbour):
// key = ((u - y_j)^2 - (u - y_q)^2) / (cost_q - cost_j) in fp32, ties to the
// lower j. Returns +inf when the symbol has no candidate.
__device__ __forceinline__ float best_move(const AppendTables &T, int nl, int s, float ui, int *tj) {
  float best = INFINITY;
  *tj = s;
#pragma unroll
  for (int dj = -1; dj <= 1; dj += 2) {
    const int j = s + dj;
    if (j < 0 || j >= nl) continue;
    if (!(T.cost[j] < T.cost[s])) continue;
    const float dn = __fsub_rn(ui, T.lev[j]);
    const float d0 = __fsub_rn(ui, T.lev[s]);
    const float num = __fsub_rn(__fmul_rn(dn, dn), __fmul_rn(d0, d0));
    const float key = __fdiv_rn(num, __fsub_rn(T.cost[s], T.cost[j]));
    if (*tj == s || key < best) {
      best = key;
      *tj = j;
    }
  }
  return best;
}

__global__ void __launch_bounds__(kAW * 32) append_kernel(const AppendArgs a, int vpw) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  AppendTables &T = *reinterpret_cast<AppendTables *>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  WarpArea W = warp_area(smem_raw + ((sizeof(AppendTables) + 15) & ~size_t(15)) + warp * warp_area_bytes(vpw), vpw);
  const bool is_v = blockIdx.y == 1;
  const DevStream &tab = is_v ? a.tabs->v : a.tabs->k;
  const int nl = is_v ? a.nv : a.nk;
  const int C = is_v ? a.cv : a.ck;
  const int P = C - 2;
  const void *src = is_v ? a.v : a.k;
  uint8_t *cache = is_v ? a.vcache : a.kcache;
  if (threadIdx.x < kMaxLevels) {
    const int s = threadIdx.x;
    T.lev[s] = tab.levels[s];
    T.thr[s] = tab.thresholds[s];
    T.cost[s] = tab.cost[s];
    T.freq[s] = tab.freq[s];
    T.cum[s] = tab.cum[s];
    const unsigned long long f = tab.freq[s] ? tab.freq[s] : 1u;
    T.rcp[s] = ((1ull << 40) + f - 1) / f;
  }
  __syncthreads();

  const int64_t per_seq = static_cast<int64_t>(a.Hkv) * a.n_new;
  const int64_t nvec = static_cast<int64_t>(a.B) * per_seq;
  const int64_t v0 = (static_cast<int64_t>(blockIdx.x) * kAW + warp) * vpw;
  if (v0 >= nvec) return;
  const int nmine = static_cast<int>((nvec - v0) < vpw ? (nvec - v0) : vpw);

  // ---- phase 1: warp per vector ----
  for (int vv = 0; vv < nmine; ++vv) {
    const int64_t v = v0 + vv;
    const int h = static_cast<int>((v % per_seq) / a.n_new);
    float z[4];
    bool nf = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float xv = load_elem(src, v * kD + lane + 32 * k, a.dtype);
      nf |= !isfinite(xv);
      z[k] = apply_sign(xv, __ldg(a.sign_bits + h * 4 + k), lane);
    }
    nf = __any_sync(kFull, nf);
    float u[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    uint16_t n16 = 0;
    if (!nf) {
      wht128_warp(z, lane);
      float part = __fadd_rn(__fadd_rn(__fmul_rn(z[0], z[0]), __fmul_rn(z[1], z[1])),
                             __fadd_rn(__fmul_rn(z[2], z[2]), __fmul_rn(z[3], z[3])));
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) part = __fadd_rn(part, __shfl_xor_sync(kFull, part, off));
      if (!isfinite(part)) {
        nf = true;
      } else {
        const float r = __fsqrt_rn(part);
        const float sigma = (r == 0.0f) ? 0.0f : __fdiv_rn(kSqrtD, r);
        if (r != 0.0f && isfinite(sigma)) {
#pragma unroll
          for (int k = 0; k < 4; ++k) u[k] = __fmul_rn(z[k], sigma);
        }
        float nv = __fdiv_rn(r, kSqrtD);
        if (nv > 65504.0f) nv = 65504.0f;
        n16 = __half_as_ushort(__float2half_rn(nv));
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int c = 0;
      for (int j = 0; j < nl - 1; ++j) c += (T.thr[j] <= u[k]) ? 1 : 0;
      W.u[vv * kUStride + lane + 32 * k] = u[k];
      W.q[vv * kQStride + lane + 32 * k] = static_cast<uint8_t>(c);
    }
    if (lane == 0) {
      W.norm16[vv] = n16;
      W.nonfinite[vv] = nf ? 1 : 0;
    }
  }
  __syncwarp();

  auto dst_of = [&](int vv, bool *dropped) -> uint8_t * {
    const int64_t v = v0 + vv;
    const int b = static_cast<int>(v / per_seq);
    const int h = static_cast<int>((v % per_seq) / a.n_new);
    const int j = static_cast<int>(v % a.n_new);
    const int64_t pos = static_cast<int64_t>(a.start_pos[b]) + j;
    *dropped = pos < 0 || pos >= a.T_cap;
    if (*dropped) return nullptr;
    // Byte 0 of the container: block pos / 32 of row (b, h), lane pos % 32.
    return cache + ((static_cast<int64_t>(b) * a.Hkv + h) * a.T_cap + (pos & ~int64_t(31))) * C + (pos & 31);
  };

  // ---- phase 2: lane per vector, first encode ----
  bool dropped = false, too_long = false;
  if (lane < nmine) {
    const uint8_t *q = W.q + lane * kQStride;
    uint8_t *stack = W.stack + lane * kStack;
    uint32_t x = 0;
    const int len = rans_encode([&](int i) { return static_cast<uint32_t>(q[i]); }, T, stack, P, &x);
    too_long = len > P;
    uint8_t *dst = dst_of(lane, &dropped);
    if (!too_long && dst) store_container(dst, C, W.norm16[lane], x, stack, len);
  }
  unsigned drift_mask = __ballot_sync(kFull, too_long);
  unsigned moves_total = 0, cont_drifted = 0, fallbacks = 0;
  unsigned drops = __ballot_sync(kFull, dropped);

  // ---- phase 3: warp per over-long container (E6 drift) ----
  while (drift_mask) {
    const int vv = __ffs(drift_mask) - 1;
    drift_mask &= drift_mask - 1;
    uint8_t *q = W.q + vv * kQStride;
    const float *uu = W.u + vv * kUStride;
    // Best move and key of the 4 symbols this lane owns (i = lane + 32 k).
    float key[4];
    int tj[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = lane + 32 * k;
      key[k] = best_move(T, nl, q[i], uu[i], &tj[k]);
      W.rank[i] = kNoRank;
      W.tgt[i] = static_cast<uint8_t>(tj[k]);
    }
    __syncwarp();
    int ranked = 0;       // moves ranked so far
    int applied = -1;     // number of moves in the result
    bool exhausted = false;
    while (applied < 0 && !exhausted) {
      // Rank the next (up to) 32 moves: repeated arg-min over (key, index).
      int added = 0;
      for (; added < 32; ++added) {
        float bk = key[0];
        int bi = lane;
#pragma unroll
        for (int k = 1; k < 4; ++k)
          if (key[k] < bk) { bk = key[k]; bi = lane + 32 * k; }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          const float ok = __shfl_xor_sync(kFull, bk, off);
          const int oi = __shfl_xor_sync(kFull, bi, off);
          if (ok < bk || (ok == bk && oi < bi)) { bk = ok; bi = oi; }
        }
        if (bk == INFINITY) break;  // no candidate left
        if ((bi & 31) == lane) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (bi == lane + 32 * k) key[k] = INFINITY;
          W.rank[bi] = static_cast<uint8_t>(ranked + added);
        }
      }
      __syncwarp();
      // Lane m (m < added) encodes the string with moves 0 .. ranked + m applied.
      const int m_moves = ranked + lane;  // highest rank applied by this lane
      int len = P + 1;
      uint32_t x = 0;
      uint8_t *stack = W.stack + lane * kStack;
      if (lane < added)
        len = rans_encode(
            [&](int i) {
              const uint32_t r = W.rank[i];
              return (r != kNoRank && static_cast<int>(r) <= m_moves) ? static_cast<uint32_t>(W.tgt[i])
                                                                      : static_cast<uint32_t>(q[i]);
            },
            T, stack, P, &x);
      const unsigned fit = __ballot_sync(kFull, lane < added && len <= P);
      if (fit) {
        const int win = __ffs(fit) - 1;
        applied = ranked + win + 1;
        if (lane == win) {
          bool dr = false;
          uint8_t *dst = dst_of(vv, &dr);
          if (dst) store_container(dst, C, W.norm16[vv], x, stack, len);
        }
      } else {
        ranked += added;
        exhausted = added < 32;
      }
      __syncwarp();
    }
    if (applied < 0) {
      // Fallback (candidates exhausted): every symbol to the innermost level
      // of its side, with the moves made so far counted.
      const int hlf = nl / 2;
      if (lane == 0) {
        uint32_t x = 0;
        uint8_t *stack = W.stack;
        const int len = rans_encode(
            [&](int i) {
              const uint32_t r = W.rank[i];
              const uint32_t s = (r != kNoRank) ? W.tgt[i] : q[i];
              return static_cast<uint32_t>(s >= static_cast<uint32_t>(hlf) ? hlf : hlf - 1);
            },
            T, stack, P, &x);
        bool dr = false;
        uint8_t *dst = dst_of(vv, &dr);
        if (dst && len <= P) store_container(dst, C, W.norm16[vv], x, stack, len);
      }
      applied = ranked;
      ++fallbacks;
    }
    moves_total += static_cast<unsigned>(applied);
    cont_drifted += applied > 0 ? 1u : 0u;
    __syncwarp();
  }

  if (a.stats && lane == 0) {
    const unsigned nfs = [&]() {
      unsigned c = 0;
      for (int vv = 0; vv < nmine; ++vv) c += W.nonfinite[vv];
      return c;
    }();
    if (moves_total) atomicAdd(is_v ? &a.stats->v_syms_drifted : &a.stats->k_syms_drifted, (unsigned long long)moves_total);
    if (cont_drifted) atomicAdd(is_v ? &a.stats->v_cont_drifted : &a.stats->k_cont_drifted, (unsigned long long)cont_drifted);
    if (fallbacks) atomicAdd(&a.stats->overflow_fallbacks, (unsigned long long)fallbacks);
    if (nfs) atomicAdd(&a.stats->nonfinite_inputs, (unsigned long long)nfs);
    if (drops) atomicAdd(&a.stats->dropped_writes, (unsigned long long)__popc(drops));
  }
}

}  // namespace

int launch_append(const AppendArgs &a, void *stream) {
  if (a.ck > kMaxContainer || a.cv > kMaxContainer) return static_cast<int>(cudaErrorInvalidValue);
  const int64_t nvec = static_cast<int64_t>(a.B) * a.Hkv * a.n_new;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Vectors per warp: 32 when there is enough work for every SM, fewer (down
  // to 1) for small appends such as one decode step, so the work still
  // spreads over all SMs.
  int vpw = 32;
  while (vpw > 1 && nvec < static_cast<int64_t>(vpw) * kAW * sms * 4) vpw >>= 1;
  const int64_t per_cta = static_cast<int64_t>(kAW) * vpw;
  const int64_t gx = (nvec + per_cta - 1) / per_cta;
  if (gx > 0x7FFFFFFF) return static_cast<int>(cudaErrorInvalidConfiguration);
  const size_t smem = ((sizeof(AppendTables) + 15) & ~size_t(15)) + kAW * warp_area_bytes(vpw);
  cudaError_t e = cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return static_cast<int>(e);
  dim3 grid(static_cast<unsigned>(gx), 2);
  append_kernel<<<grid, kAW * 32, smem, static_cast<cudaStream_t>(stream)>>>(a, vpw);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dqi
