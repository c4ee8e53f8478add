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
// Work split: one warp takes 32 vectors of one stream.
//   phase 1 (warp per vector): E1 sign flip, E2 Walsh-Hadamard transform
//     (shuffles for stages 1..16, registers for 32 and 64), E3 norm in a
//     fixed tree, scale, fp16 norm, E4 quantisation; u and symbols to smem.
//   phase 2 (lane per vector): E5 rANS encode last-to-first, E6 greedy drift
//     with re-encoding, E7 container store.
#include "dq_device.cuh"

namespace dqi {
namespace {

constexpr int kAW = 4;          // warps per CTA
constexpr int kUStride = kD + 1;
constexpr int kQStride = kD + 4;
constexpr int kStack = kMaxContainer;
constexpr float kSqrtD = 11.3137084989847604f;  // fl32(sqrt(128))

struct AppendSmem {
  float u[kAW][32][kUStride];
  uint8_t q[kAW][32][kQStride];
  uint8_t stack[kAW][32][kStack];
  uint16_t norm16[kAW][32];
  uint8_t nonfinite[kAW][32];
  float lev[kMaxLevels], thr[kMaxLevels], cost[kMaxLevels];
  uint32_t freq[kMaxLevels], cum[kMaxLevels];
};

// E5: rANS-encode q[0..127] (coded 127 -> 0) into `stack` (pushed order).
// Returns the total length 3 + #pushed, or cap + 1 as soon as it is known to
// exceed `cap` bytes (the pushed bytes are then incomplete).
__device__ __forceinline__ int rans_encode(const uint8_t *q, const AppendSmem &S, uint8_t *stack, int cap,
                                           uint32_t *x_out) {
  uint32_t x = kL;
  int np = 0;
  const int max_push = cap - 3;
  for (int i = kD - 1; i >= 0; --i) {
    const uint32_t s = q[i];
    const uint32_t f = S.freq[s];
    const uint32_t xmax = ((kL >> kProbBits) << 8) * f;
    while (x >= xmax) {
      if (np >= max_push) return cap + 1;
      stack[np++] = static_cast<uint8_t>(x & 0xFFu);
      x >>= 8;
    }
    x = (x / f) * kM + (x % f) + S.cum[s];
  }
  *x_out = x;
  return 3 + np;
}

__global__ void __launch_bounds__(kAW * 32) append_kernel(const AppendArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  AppendSmem &S = *reinterpret_cast<AppendSmem *>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool is_v = blockIdx.y == 1;
  const DevStream &tab = is_v ? a.tabs->v : a.tabs->k;
  const int nl = is_v ? a.nv : a.nk;
  const int C = is_v ? a.cv : a.ck;
  const int P = C - 2;
  const void *src = is_v ? a.v : a.k;
  uint8_t *cache = is_v ? a.vcache : a.kcache;
  if (threadIdx.x < kMaxLevels) {
    S.lev[threadIdx.x] = tab.levels[threadIdx.x];
    S.thr[threadIdx.x] = tab.thresholds[threadIdx.x];
    S.cost[threadIdx.x] = tab.cost[threadIdx.x];
    S.freq[threadIdx.x] = tab.freq[threadIdx.x];
    S.cum[threadIdx.x] = tab.cum[threadIdx.x];
  }
  __syncthreads();

  const int64_t per_seq = static_cast<int64_t>(a.Hkv) * a.n_new;
  const int64_t nvec = static_cast<int64_t>(a.B) * per_seq;
  const int64_t v0 = (static_cast<int64_t>(blockIdx.x) * kAW + warp) * 32;

  // ---- phase 1: warp per vector ----
  for (int vv = 0; vv < 32; ++vv) {
    const int64_t v = v0 + vv;
    if (v >= nvec) break;
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
      for (int j = 0; j < nl - 1; ++j) c += (S.thr[j] <= u[k]) ? 1 : 0;
      S.u[warp][vv][lane + 32 * k] = u[k];
      S.q[warp][vv][lane + 32 * k] = static_cast<uint8_t>(c);
    }
    if (lane == 0) {
      S.norm16[warp][vv] = n16;
      S.nonfinite[warp][vv] = nf ? 1 : 0;
    }
  }
  __syncwarp();

  // ---- phase 2: lane per vector ----
  const int64_t v = v0 + lane;
  const bool valid = v < nvec;
  unsigned moves = 0, fb = 0;
  bool dropped = false;
  if (valid) {
    uint8_t *q = S.q[warp][lane];
    const float *uu = S.u[warp][lane];
    uint8_t *stack = S.stack[warp][lane];
    uint32_t moved[4] = {0u, 0u, 0u, 0u};
    uint32_t x = 0;
    int len = rans_encode(q, S, stack, P, &x);
    while (len > P) {  // E6 drift
      int bi = -1, bj = -1;
      float bkey = 0.0f;
      for (int i = 0; i < kD; ++i) {
        if ((moved[i >> 5] >> (i & 31)) & 1u) continue;
        const int s = q[i];
        const float ui = uu[i];
#pragma unroll
        for (int dj = -1; dj <= 1; dj += 2) {
          const int j = s + dj;
          if (j < 0 || j >= nl) continue;
          if (!(S.cost[j] < S.cost[s])) continue;
          const float dn = __fsub_rn(ui, S.lev[j]);
          const float d0 = __fsub_rn(ui, S.lev[s]);
          const float num = __fsub_rn(__fmul_rn(dn, dn), __fmul_rn(d0, d0));
          const float key = __fdiv_rn(num, __fsub_rn(S.cost[s], S.cost[j]));
          if (bi < 0 || key < bkey) {
            bi = i;
            bj = j;
            bkey = key;
          }
        }
      }
      if (bi < 0) break;
      q[bi] = static_cast<uint8_t>(bj);
      moved[bi >> 5] |= 1u << (bi & 31);
      ++moves;
      len = rans_encode(q, S, stack, P, &x);
    }
    if (len > P) {  // fallback: innermost level of each symbol's side
      const int hlf = nl / 2;
      for (int i = 0; i < kD; ++i) q[i] = static_cast<uint8_t>(q[i] >= hlf ? hlf : hlf - 1);
      len = rans_encode(q, S, stack, P, &x);
      fb = 1;
    }
    const int64_t per = a.n_new;
    const int b = static_cast<int>(v / per_seq);
    const int h = static_cast<int>((v % per_seq) / per);
    const int j = static_cast<int>(v % per);
    const int64_t pos = static_cast<int64_t>(a.start_pos[b]) + j;
    if (pos < 0 || pos >= a.T_cap || len > P) {
      dropped = true;
    } else {
      uint8_t *dst = cache + ((static_cast<int64_t>(b) * a.Hkv + h) * a.T_cap + pos) * C;
      const uint16_t n16 = S.norm16[warp][lane];
      const int np = len - 3;
      for (int k = 0; k < C; ++k) {
        uint8_t byte;
        if (k == 0) byte = static_cast<uint8_t>(n16 & 0xFFu);
        else if (k == 1) byte = static_cast<uint8_t>(n16 >> 8);
        else if (k < 5) byte = static_cast<uint8_t>((x >> (8 * (k - 2))) & 0xFFu);
        else if (k - 5 < np) byte = stack[np - 1 - (k - 5)];
        else byte = 0;
        dst[k] = byte;
      }
    }
  }
  if (a.stats) {
    const unsigned drifted = __ballot_sync(kFull, moves > 0);
    unsigned tot_moves = moves;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) tot_moves += __shfl_xor_sync(kFull, tot_moves, o);
    const unsigned fbs = __ballot_sync(kFull, fb != 0);
    const unsigned nfs = __ballot_sync(kFull, valid && S.nonfinite[warp][lane]);
    const unsigned drops = __ballot_sync(kFull, dropped);
    if (lane == 0) {
      if (tot_moves) atomicAdd(is_v ? &a.stats->v_syms_drifted : &a.stats->k_syms_drifted, (unsigned long long)tot_moves);
      if (drifted) atomicAdd(is_v ? &a.stats->v_cont_drifted : &a.stats->k_cont_drifted, (unsigned long long)__popc(drifted));
      if (fbs) atomicAdd(&a.stats->overflow_fallbacks, (unsigned long long)__popc(fbs));
      if (nfs) atomicAdd(&a.stats->nonfinite_inputs, (unsigned long long)__popc(nfs));
      if (drops) atomicAdd(&a.stats->dropped_writes, (unsigned long long)__popc(drops));
    }
  }
}

}  // namespace

int launch_append(const AppendArgs &a, void *stream) {
  if (a.ck > kMaxContainer || a.cv > kMaxContainer) return static_cast<int>(cudaErrorInvalidValue);
  const int64_t nvec = static_cast<int64_t>(a.B) * a.Hkv * a.n_new;
  const int64_t per_cta = kAW * 32;
  const int64_t gx = (nvec + per_cta - 1) / per_cta;
  if (gx > 0x7FFFFFFF) return static_cast<int>(cudaErrorInvalidConfiguration);
  const size_t smem = sizeof(AppendSmem);
  cudaError_t e = cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return static_cast<int>(e);
  dim3 grid(static_cast<unsigned>(gx), 2);
  append_kernel<<<grid, kAW * 32, smem, static_cast<cudaStream_t>(stream)>>>(a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dqi
