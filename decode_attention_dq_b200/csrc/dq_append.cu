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
// Work split: one warp takes 32 consecutive vectors of one stream.
//   phase 1 (four lanes per vector, 32 coordinates each in registers, four
//     passes of 8 vectors): E1 sign flip, E2 Walsh-Hadamard transform (the
//     seven butterfly stages in order, two of them between lanes), E3 norm
//     in the fixed tree (the 32 partial sums of four squares, then pairwise
//     over offsets 16, 8, 4, 2, 1), scale, fp16 norm, E4 quantisation by a
//     three-step search over the sorted thresholds; symbols packed 4 per
//     word in shared memory.
//   phase 2 (lane per vector): E5 rANS encode last-to-first without branches
//     (a renormalisation push is written every step and kept only when
//     needed; the division by f is an exact multiply-shift); containers that
//     fit are stored at once.
//   phase 3 (warp per over-long container, a few percent): E6 drift. The warp
//     recomputes the vector's rotated coordinates (4 per lane, the same
//     arithmetic), ranks the candidate moves by repeated arg-min (least key
//     first, ties to the lower index), and lane m encodes the string with the
//     first m+1 moves applied; the smallest m that fits is the greedy result.
//     The warp-per-vector kernel (small appends) tries up to 32 move counts
//     per pass; a string whose symbol costs add up to near the budget is
//     ranked before its first encode, so that one pass tries 0 .. 31 moves
//     (lane m: m moves) instead of an encode that fails and a second one;
//     it stores a container with the whole warp, a byte per lane. The separate
//     drift kernel (lane-per-vector appends) keeps 8 containers per warp in
//     flight and tries 4 move counts of each per encode pass, ranking 4 more
//     moves of a container only when its window had no fit; in drift mode 1
//     it also runs the rate-distortion fill of every container.
#include "dq_device.cuh"

namespace dqi {
namespace {

constexpr int kAW = 4;                  // warps per CTA
constexpr int kStackSlots = 64;         // bytes of push stack per lane
constexpr float kSqrtD = 11.3137084989847604f;  // fl32(sqrt(128))
constexpr uint8_t kNoRank = 255;

// Division by f for the encoder: q = floor(x / f) = (x * m) >> k for every
// x < 4096 f, with k = 12 + ceil(log2 f^2) and m = ceil(2^k / f). (x m / 2^k
// = x / f + x e / (f 2^k) with e = m f - 2^k < f, and x e < 4096 f^2 <= 2^k,
// so the excess stays below 1 / f and the floor is exact.)
struct EncSym {
  uint32_t m, k, xmax, cum;  // xmax = 4096 f: push while x >= xmax
  uint32_t g, f, pad0, pad1; // g = 4096 - f: x' = x + q g + cum
};

struct AppendTables {
  EncSym es[kMaxLevels];
  float thr[kMaxLevels];  // thresholds, padded with +inf
  float lev[kMaxLevels], cost[kMaxLevels];
  uint32_t freq[kMaxLevels], cum[kMaxLevels];
};

// Per-warp shared memory: push stacks (byte j of lane l at [j][l]), the
// lanes' packed symbols (word w of lane l at [w][l]) and the symbols, move
// ranks and targets of the container being drifted.
struct WarpArea {
  uint8_t stack[kStackSlots * 32];
  uint32_t syms[kD / 4][32];
  uint8_t q[kD], rank[kD], tgt[kD];
  int32_t head[32];  // KV head of the warp's vector l (lane-per-vector kernel)
  uint16_t n16[32];  // fp16 norm of the warp's vector l
  uint8_t nf[32];    // vector l was non-finite
};

// Writes one container; byte k goes to dst[32 k] (the cache interleaves the
// bytes of the 32 tokens of a block). stk[32 j] holds push j.
__device__ __forceinline__ void store_container(uint8_t *dst, int C, uint16_t n16, uint32_t x, const uint8_t *stk,
                                                int len) {
  const int np = len - 3;
  for (int k = 0; k < C; ++k) {
    uint8_t byte;
    if (k == 0) byte = static_cast<uint8_t>(n16 & 0xFFu);
    else if (k == 1) byte = static_cast<uint8_t>(n16 >> 8);
    else if (k < 5) byte = static_cast<uint8_t>((x >> (8 * (k - 2))) & 0xFFu);
    else if (k - 5 < np) byte = stk[32 * (np - 1 - (k - 5))];
    else byte = 0;
    dst[32 * k] = byte;
  }
}

// store_container by a whole converged warp, one byte per lane: the string
// is the one lane `src` encoded (its pushes at stack[src + 32 j]); every lane
// passes that lane's x and len.
__device__ __forceinline__ void store_container_warp(uint8_t *dst, int C, uint16_t n16, uint32_t x,
                                                     const uint8_t *stack, int src, int len, int lane) {
  const int np = len - 3;
#pragma unroll
  for (int k0 = 0; k0 < kMaxContainer; k0 += 32) {
    const int k = k0 + lane;
    if (k < C) {
      uint8_t byte;
      if (k == 0) byte = static_cast<uint8_t>(n16 & 0xFFu);
      else if (k == 1) byte = static_cast<uint8_t>(n16 >> 8);
      else if (k < 5) byte = static_cast<uint8_t>((x >> (8 * (k - 2))) & 0xFFu);
      else if (k - 5 < np) byte = stack[src + 32 * (np - 1 - (k - 5))];
      else byte = 0;
      dst[32 * k] = byte;
    }
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

// A float key as an unsigned integer with the same order (sign bit set:
// all bits flipped; clear: the sign bit set). -0 is first made +0 (k + 0 in
// round-to-nearest; the float order holds them equal), keys are never NaN,
// so equal integers are equal keys; +inf (no candidate) maps to 0xFF800000,
// above every finite key.
__device__ __forceinline__ uint32_t order_bits(float k) {
  const uint32_t b = __float_as_uint(__fadd_rn(k, 0.0f));
  return b ^ (static_cast<uint32_t>(static_cast<int32_t>(b) >> 31) | 0x80000000u);
}
constexpr uint32_t kNoKey = 0xFF800000u;      // order_bits(+inf)
constexpr uint32_t kRankedKey = 0xFFFFFFFFu;  // above kNoKey

// Warp arg-min over the 128 keys of a vector (symbol lane + 32 k in key[k],
// as order_bits): the least key, ties to the lowest symbol index. Returns
// that index, or -1 when no key is below kNoKey (no candidate left).
__device__ __forceinline__ int warp_argmin(const uint32_t (&key)[4], int lane) {
  const uint32_t bk = __reduce_min_sync(kFull, min(min(key[0], key[1]), min(key[2], key[3])));
  if (bk >= kNoKey) return -1;
  const uint32_t mine = key[0] == bk   ? static_cast<uint32_t>(lane)
                        : key[1] == bk ? static_cast<uint32_t>(lane + 32)
                        : key[2] == bk ? static_cast<uint32_t>(lane + 64)
                        : key[3] == bk ? static_cast<uint32_t>(lane + 96)
                                       : 0xFFFFFFFFu;
  return static_cast<int>(__reduce_min_sync(kFull, mine));
}

// E4: symbol = number of thresholds <= u (ties go up), by a three-step
// search over the 7 sorted thresholds t0..t6 (padded with +inf).
__device__ __forceinline__ uint32_t quantize7(float u, const float (&t)[7]) {
  const bool p1 = t[3] <= u;
  const float ta = p1 ? t[5] : t[1];
  const bool p2 = ta <= u;
  const float tb = p1 ? (p2 ? t[6] : t[4]) : (p2 ? t[2] : t[0]);
  const bool p3 = tb <= u;
  return (p1 ? 4u : 0u) + (p2 ? 2u : 0u) + (p3 ? 1u : 0u);
}

// Sign word bit `b` moved to the float sign position.
__device__ __forceinline__ uint32_t sign_bit(uint32_t word, int b) { return (word << (31 - b)) & 0x80000000u; }

// E5 without branches: rANS-encode 128 symbols (sym(i) gives symbol i),
// coded 127 -> 0 from x = 2^16. A renormalisation push writes the low byte of
// x to the lane's stack every step and keeps it only when x >= 4096 f; pushes
// go to stk[32 j]. Returns the total length 3 + #pushed; above `cap` the
// container is too long (pushes past the stack wrap around and are never
// stored). No lane branches, so all 32 lanes of a warp stay converged. kTwo:
// the table has a symbol with f < 16, so a step can push two bytes. kStk:
// push-stack slots per lane (a power of two, at least C - 4).
//
// A push is st.shared.u8 without a memory clobber, so that the compiler can
// move the next steps' symbol and table loads ahead of it (as a C++ store it
// could not tell the push stack from the tables and held every load back
// behind the previous step's store). The stack is not read during the
// encode; encode_bf has compiler barriers before and after the pushes.
__device__ __forceinline__ void push_byte(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u8 [%0], %1;\n" ::"r"(a), "r"(v));
}

// One encode step of encode_bf (stk_s: the lane's stack as a shared-memory
// address).
template <bool kTwo, int kStk = kStackSlots>
__device__ __forceinline__ void encode_step(uint32_t s, const uint8_t *esb, uint32_t stk_s, uint32_t &x, uint32_t &np) {
  const uint4 e0 = *reinterpret_cast<const uint4 *>(esb + s * sizeof(EncSym));  // {m, k, xmax, cum}
  const uint32_t g = *reinterpret_cast<const uint32_t *>(esb + s * sizeof(EncSym) + 16);
  bool push = x >= e0.z;
  push_byte(stk_s + 32 * (np & (kStk - 1)), x & 0xFFu);
  np += push ? 1u : 0u;
  x = push ? (x >> 8) : x;
  if constexpr (kTwo) {
    push = x >= e0.z;
    push_byte(stk_s + 32 * (np & (kStk - 1)), x & 0xFFu);
    np += push ? 1u : 0u;
    x = push ? (x >> 8) : x;
  }
  const uint32_t q = static_cast<uint32_t>((static_cast<unsigned long long>(x) * e0.x) >> e0.y);
  x = (x + e0.w) + q * g;
}

// kRegs: symbols come from registers (the loop is unrolled completely so
// that sym(i) indexes them statically); otherwise from shared memory.
template <bool kTwo, bool kRegs, typename SymFn, int kStk = kStackSlots>
__device__ __forceinline__ int encode_bf(SymFn sym, const EncSym *es, uint8_t *stk, uint32_t *x_out) {
  uint32_t x = kL;
  uint32_t np = 0;
  const uint8_t *esb = reinterpret_cast<const uint8_t *>(es);
  asm volatile("" ::: "memory");  // earlier stores (of the stack too) come before the pushes
  const uint32_t stk_s = static_cast<uint32_t>(__cvta_generic_to_shared(stk));
  if constexpr (kRegs) {
#pragma unroll
    for (int i = kD - 1; i >= 0; --i) encode_step<kTwo, kStk>(sym(i), esb, stk_s, x, np);
  } else {
#pragma unroll 8
    for (int i = kD - 1; i >= 0; --i) encode_step<kTwo, kStk>(sym(i), esb, stk_s, x, np);
  }
  asm volatile("" ::: "memory");  // the pushes above come before any read of the stack
  *x_out = x;
  return 3 + static_cast<int>(np);
}

// Phase-1 arithmetic for one vector spread over the warp (coordinate
// lane + 32 k in u[k]): same operations, same order, so the same u, symbols
// and norm as quad_prepare. Returns the symbols of this lane's coordinates in
// qk[], the fp16 norm and whether the vector was non-finite.
__device__ __forceinline__ void warp_prepare_regs(const AppendArgs &a, const void *src, int64_t v, int h,
                                                  const float (&t)[7], int lane, float (&u)[4], uint32_t (&qk)[4],
                                                  uint16_t *n16_out, bool *nf_out) {
  float z[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    z[k] = apply_sign(load_elem(src, v * kD + lane + 32 * k, a.dtype), __ldg(a.sign_bits + h * 4 + k), lane);
  wht128_warp(z, lane);
  float part = __fadd_rn(__fadd_rn(__fmul_rn(z[0], z[0]), __fmul_rn(z[1], z[1])),
                         __fadd_rn(__fmul_rn(z[2], z[2]), __fmul_rn(z[3], z[3])));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) part = __fadd_rn(part, __shfl_xor_sync(kFull, part, off));
  const bool nf = !isfinite(part);
  float sigma = 0.0f;
  uint16_t n16 = 0;
  if (!nf) {
    const float r = __fsqrt_rn(part);
    sigma = (r == 0.0f) ? 0.0f : __fdiv_rn(kSqrtD, r);
    if (!(r != 0.0f && isfinite(sigma))) sigma = 0.0f;
    float nv = __fdiv_rn(r, kSqrtD);
    if (nv > 65504.0f) nv = 65504.0f;
    n16 = __half_as_ushort(__float2half_rn(nv));
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    u[k] = nf ? 0.0f : __fmul_rn(z[k], sigma);
    qk[k] = quantize7(u[k], t);
  }
  *n16_out = n16;
  *nf_out = nf;
}

// warp_prepare_regs with the symbols written to q[lane + 32 k].
__device__ __forceinline__ void warp_prepare(const AppendArgs &a, const void *src, int64_t v, int h,
                                             const float (&t)[7], int lane, float (&u)[4], uint8_t *q,
                                             uint16_t *n16_out, bool *nf_out) {
  uint32_t qk[4];
  warp_prepare_regs(a, src, v, h, t, lane, u, qk, n16_out, nf_out);
#pragma unroll
  for (int k = 0; k < 4; ++k) q[lane + 32 * k] = static_cast<uint8_t>(qk[k]);
}

// v / d, with v % d in *rem, for 0 <= v and 0 < d; in 32-bit arithmetic
// when both fit (the same quotient, far fewer instructions than a 64-bit
// division).
__device__ __forceinline__ int64_t div_rem(int64_t v, int64_t d, int64_t *rem) {
  if (((v | d) >> 32) == 0) {
    const uint32_t q = static_cast<uint32_t>(v) / static_cast<uint32_t>(d);
    *rem = v - static_cast<int64_t>(q) * d;
    return q;
  }
  const int64_t q = v / d;
  *rem = v - q * d;
  return q;
}

// Where the vectors of one append call come from and go to (one stream).
struct StreamCtx {
  const void *src;
  uint8_t *cache;
  int nl, C, P;
  int64_t per_seq, nvec;
  float t[7];

  // Sequence b, KV head h and new-token index j of vector v
  // (v = (b Hkv + h) n_new + j).
  __device__ void split(const AppendArgs &a, int64_t v, int *b, int *h, int64_t *j) const {
    int64_t rem, jj;
    *b = static_cast<int>(div_rem(v, per_seq, &rem));
    *h = static_cast<int>(div_rem(rem, a.n_new, &jj));
    *j = jj;
  }
  __device__ int head_of(const AppendArgs &a, int64_t v) const {
    int b, h;
    int64_t j;
    split(a, v, &b, &h, &j);
    return h;
  }
  // Byte 0 of the container of token j of sequence b, KV head h (lane
  // pos % 32 of the 32-token block holding position pos), or null when the
  // position is outside the cache (dropped) or its page-table entry is out of
  // range (also *bad_page).
  __device__ uint8_t *dst_at(const AppendArgs &a, int b, int h, int64_t j, bool *dropped,
                             bool *bad_page = nullptr) const {
    const int64_t pos = static_cast<int64_t>(a.start_pos[b]) + j;
    *dropped = pos < 0 || pos >= a.T_cap;
    if (*dropped) return nullptr;
    int64_t block;
    if (a.page_table) {
      const int32_t pg = a.page_table[static_cast<int64_t>(b) * a.max_pages + (pos >> 5)];
      if (pg < 0 || pg >= a.num_pages) {
        *dropped = true;
        if (bad_page) *bad_page = true;
        return nullptr;
      }
      block = static_cast<int64_t>(pg) * a.Hkv + h;
    } else {
      block = (static_cast<int64_t>(b) * a.Hkv + h) * (a.T_cap >> 5) + (pos >> 5);
    }
    return cache + block * 32 * C + (pos & 31);
  }
  __device__ uint8_t *dst_of(const AppendArgs &a, int64_t v, bool *dropped, bool *bad_page = nullptr) const {
    int b, h;
    int64_t j;
    split(a, v, &b, &h, &j);
    return dst_at(a, b, h, j, dropped, bad_page);
  }
};

// Copies one stream's tables into shared memory (the threads with filler
// index 0..7) and fills the stream context. Callers synchronise before using T.
__device__ __forceinline__ StreamCtx stream_setup(const AppendArgs &a, AppendTables &T, bool is_v, int filler) {
  const DevStream &tab = is_v ? a.tabs->v : a.tabs->k;
  StreamCtx c;
  c.nl = is_v ? a.nv : a.nk;
  c.C = is_v ? a.cv : a.ck;
  c.P = c.C - 2;
  c.src = is_v ? a.v : a.k;
  c.cache = is_v ? a.vcache : a.kcache;
  c.per_seq = static_cast<int64_t>(a.Hkv) * a.n_new;
  c.nvec = static_cast<int64_t>(a.B) * c.per_seq;
  if (filler < kMaxLevels) {
    const int s = filler;
    T.lev[s] = tab.levels[s];
    T.thr[s] = (s < c.nl - 1) ? tab.thresholds[s] : INFINITY;
    T.cost[s] = tab.cost[s];
    const uint32_t f = tab.freq[s] ? tab.freq[s] : 1u;
    T.freq[s] = tab.freq[s];
    T.cum[s] = tab.cum[s];
    EncSym e;
    const uint32_t lg = 32 - __clz(f * f - 1u);  // ceil(log2 f^2); 0 for f = 1
    e.k = 12 + (f == 1 ? 0u : lg);
    e.m = static_cast<uint32_t>(((1ull << e.k) + f - 1) / f);
    e.xmax = f << 12;
    e.cum = tab.cum[s];
    e.g = 4096u - f;
    e.f = f;
    e.pad0 = e.pad1 = 0;
    T.es[s] = e;
  }
#pragma unroll
  for (int j = 0; j < 7; ++j) c.t[j] = (j < c.nl - 1) ? tab.thresholds[j] : INFINITY;
  return c;
}

// Norm and scale from the sum of squares ss (E3): sigma = sqrt(128) / r with
// r = sqrt(ss) (0 for the zero vector), the fp16 norm r / sqrt(128)
// (clamped to the largest finite half), and whether the vector is
// non-finite (then u = 0 and the norm is 0).
__device__ __forceinline__ void norm_scale(float ss, float *sigma_out, uint16_t *n16_out, bool *nf_out) {
  const bool nf = !isfinite(ss);
  uint16_t n16 = 0;
  float sigma = 0.0f;
  if (!nf) {
    const float r = __fsqrt_rn(ss);
    sigma = (r == 0.0f) ? 0.0f : __fdiv_rn(kSqrtD, r);
    if (!(r != 0.0f && isfinite(sigma))) sigma = 0.0f;
    float nv = __fdiv_rn(r, kSqrtD);
    if (nv > 65504.0f) nv = 65504.0f;
    n16 = __half_as_ushort(__float2half_rn(nv));
  }
  *sigma_out = sigma;
  *n16_out = n16;
  *nf_out = nf;
}

// One butterfly stage of E2 between the lanes j and j ^ o of a quad: the
// lane whose bit is clear holds a and keeps a + b, its partner holds b and
// keeps a - b, computed as (-b) + a (IEEE subtraction is addition of the
// negated operand, so the result is the same); neg is the sign bit for the
// partner, 0 for the lane whose bit is clear.
__device__ __forceinline__ float cross_butterfly(float z, int o, uint32_t neg) {
  const float p = __shfl_xor_sync(kFull, z, o);
  return __fadd_rn(__uint_as_float(__float_as_uint(z) ^ neg), p);
}

// Phase 1 for the 32 vectors of a warp (v0 .. v0 + 31), four lanes per
// vector: in pass p the quad g = lane / 4 takes vector l = 8 p + g, and its
// lane j holds the coordinates 32 m + 8 j + e in z[m][e]. E1 sign flip, E2
// with the stages h = 1, 2, 4 in-lane, h = 8 and 16 between lanes j ^ 1 and
// j ^ 2, h = 32 and 64 in-lane again (the seven stages in order, so the same
// sums as a transform in one lane); E3 with the 32 partial sums of four
// squares in-lane (lane j holds p_l for l = 8 j + e), offsets 16 and 8 from
// lanes j ^ 2 and j ^ 1, then 4, 2, 1 in-lane; E4 by the three-step search.
// Symbol i of vector l goes to byte i % 4 of W.syms[i / 4][l]; the norm and
// the non-finite flag to W.n16[l] and W.nf[l]. W.head[l] holds the vector's
// KV head on entry.
template <bool kBF16>
__device__ __forceinline__ void quad_prepare(const AppendArgs &a, const StreamCtx &c, WarpArea &W, int64_t v0,
                                             int lane) {
  const int g = lane >> 2, j = lane & 3;
#pragma unroll 1
  for (int p = 0; p < 4; ++p) {
    const int l = 8 * p + g;
    const int64_t v = v0 + l;
    const bool valid = v < c.nvec;  // quad-uniform
    float z[4][8];
    if (valid) {
      const int h = W.head[l];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t sb = __ldg(a.sign_bits + h * 4 + m) >> (8 * j);
        const int64_t e0 = v * kD + 32 * m + 8 * j;
        if constexpr (kBF16) {
          const uint4 w = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(c.src) + e0));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            z[m][2 * t] = __uint_as_float((ww[t] << 16) ^ sign_bit(sb, 2 * t));
            z[m][2 * t + 1] = __uint_as_float((ww[t] & 0xFFFF0000u) ^ sign_bit(sb, 2 * t + 1));
          }
        } else {
          const uint4 *src4 = reinterpret_cast<const uint4 *>(static_cast<const float *>(c.src) + e0);
          const uint4 w0 = __ldg(src4), w1 = __ldg(src4 + 1);
          const uint32_t ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) z[m][e] = __uint_as_float(ww[e] ^ sign_bit(sb, e));
        }
      }
    } else {
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int e = 0; e < 8; ++e) z[m][e] = 0.0f;
    }
    // E2, h = 1, 2, 4 (bits of e).
#pragma unroll
    for (int st = 0; st < 3; ++st) {
      const int hh = 1 << st;
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
          const int e = ((pr >> st) << (st + 1)) | (pr & (hh - 1));
          const float a0 = z[m][e], b0 = z[m][e + hh];
          z[m][e] = __fadd_rn(a0, b0);
          z[m][e + hh] = __fsub_rn(a0, b0);
        }
    }
    // h = 8, 16 (bits of j).
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int e = 0; e < 8; ++e) z[m][e] = cross_butterfly(z[m][e], 1, (j & 1) ? 0x80000000u : 0u);
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int e = 0; e < 8; ++e) z[m][e] = cross_butterfly(z[m][e], 2, (j & 2) ? 0x80000000u : 0u);
    // h = 32, 64 (bits of m).
#pragma unroll
    for (int st = 0; st < 2; ++st) {
      const int hm = 1 << st;
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int m = ((pr >> st) << (st + 1)) | (pr & (hm - 1));
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a0 = z[m][e], b0 = z[m + hm][e];
          z[m][e] = __fadd_rn(a0, b0);
          z[m + hm][e] = __fsub_rn(a0, b0);
        }
      }
    }
    // E3.
    float pp[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      pp[e] = __fadd_rn(__fadd_rn(__fmul_rn(z[0][e], z[0][e]), __fmul_rn(z[1][e], z[1][e])),
                        __fadd_rn(__fmul_rn(z[2][e], z[2][e]), __fmul_rn(z[3][e], z[3][e])));
#pragma unroll
    for (int e = 0; e < 8; ++e) pp[e] = __fadd_rn(pp[e], __shfl_xor_sync(kFull, pp[e], 2));  // lanes j = 0, 1
#pragma unroll
    for (int e = 0; e < 8; ++e) pp[e] = __fadd_rn(pp[e], __shfl_xor_sync(kFull, pp[e], 1));  // lane j = 0
#pragma unroll
    for (int o = 4; o >= 1; o >>= 1)
#pragma unroll
      for (int e = 0; e < o; ++e) pp[e] = __fadd_rn(pp[e], pp[e + o]);
    const float ss = __shfl_sync(kFull, pp[0], lane & ~3);
    float sigma;
    uint16_t n16;
    bool nf;
    norm_scale(ss, &sigma, &n16, &nf);
    // E4 (u = 0 for the zero and the non-finite vector).
    if (valid) {
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float u = nf ? 0.0f : __fmul_rn(z[m][4 * hf + e], sigma);
            word |= quantize7(u, c.t) << (8 * e);
          }
          W.syms[8 * m + 2 * j + hf][l] = word;
        }
      if (j == 0) {
        W.n16[l] = n16;
        W.nf[l] = nf ? 1 : 0;
      }
    }
  }
}

// Drift counters of one warp.
struct DriftCount {
  unsigned moves = 0, containers = 0, fallbacks = 0, filled = 0;
};

// E6 for one over-long container, by the whole warp. On entry q[] holds the
// symbols and u[k] this lane's coordinates lane + 32 k; rank[] and tgt[] are
// scratch, stack the warp's push stacks. Returns the number of moves applied
// (the ranked moves 0 .. n - 1, in rank[] / tgt[]), or -1 after a fallback.
template <bool kTwo>
// zero_first: the string without moves has not been encoded yet; the first
// pass ranks 31 moves and lane m encodes the string with m of them (lane 0:
// none), so that the first count that fits, zero included, comes out of one
// encode pass. Later passes are as without it.
__device__ __forceinline__ int drift_one(const AppendArgs &a, const StreamCtx &c, const AppendTables &T,
                                          uint8_t *stack, const uint8_t *q, uint8_t *rank, uint8_t *tgt, int64_t vd,
                                          uint16_t n16v, const float (&u)[4], int lane, int first_batch,
                                          DriftCount &dc, bool zero_first = false) {
  uint8_t *stk = stack + lane;
  // Best move and key of the 4 symbols this lane owns (i = lane + 32 k).
  uint32_t key[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = lane + 32 * k;
    int tj;
    key[k] = order_bits(best_move(T, c.nl, q[i], u[k], &tj));
    rank[i] = kNoRank;
    tgt[i] = static_cast<uint8_t>(tj);
  }
  __syncwarp();
  int ranked = 0;    // moves ranked so far
  int applied = -1;  // number of moves in the result
  bool exhausted = false;
  while (applied < 0 && !exhausted) {
    // Rank the next moves by repeated arg-min over (key, index):
    // first_batch on the first pass, then up to 32 per pass.
    const bool zf = zero_first && ranked == 0;  // this pass includes the string without moves
    const int batch = zf ? 31 : (ranked == 0 ? first_batch : 32);
    int added = 0;
    for (; added < batch; ++added) {
      const int bi = warp_argmin(key, lane);
      if (bi < 0) break;  // no candidate left
      if ((bi & 31) == lane) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (bi == lane + 32 * k) key[k] = kRankedKey;
        rank[bi] = static_cast<uint8_t>(ranked + added);
      }
    }
    __syncwarp();
    // Lane m encodes the string with moves 0 .. ranked + m applied (lanes
    // m >= added too, with all ranked moves; their result is not used); in
    // a zero-first pass, moves 0 .. m - 1 (lanes m > added: not used).
    const int m_moves = zf ? lane - 1 : ranked + lane;  // highest rank applied by this lane
    uint32_t x = 0;
    const int len = encode_bf<kTwo, false>(
        [&](int i) {
          const uint32_t r = rank[i];
          return (r != kNoRank && static_cast<int>(r) <= m_moves) ? static_cast<uint32_t>(tgt[i])
                                                                  : static_cast<uint32_t>(q[i]);
        },
        T.es, stk, &x);
    const unsigned fit = __ballot_sync(kFull, (zf ? lane <= added : lane < added) && len <= c.P);
    if (fit) {
      const int win = __ffs(fit) - 1;
      applied = zf ? win : ranked + win + 1;
      const uint32_t xw = __shfl_sync(kFull, x, win);
      const int lw = __shfl_sync(kFull, len, win);
      __syncwarp();  // lane win's pushes before the other lanes read them
      bool dr = false;
      uint8_t *dst = c.dst_of(a, vd, &dr);
      if (dst) store_container_warp(dst, c.C, n16v, xw, stack, win, lw, lane);
    } else {
      ranked += added;
      exhausted = added < batch;
    }
    __syncwarp();
  }
  if (applied < 0) {
    // Fallback (candidates exhausted): every symbol to the innermost level
    // of its side, with the moves made so far counted.
    const int hlf = c.nl / 2;
    uint32_t x = 0;
    const int len = encode_bf<kTwo, false>(
        [&](int i) {
          const uint32_t r = rank[i];
          const uint32_t s = (r != kNoRank) ? tgt[i] : q[i];
          return static_cast<uint32_t>(s >= static_cast<uint32_t>(hlf) ? hlf : hlf - 1);
        },
        T.es, stk, &x);
    if (lane == 0) {
      bool dr = false;
      uint8_t *dst = c.dst_of(a, vd, &dr);
      if (dst && len <= c.P) store_container(dst, c.C, n16v, x, stk, len);
    }
    applied = ranked;
    ++dc.fallbacks;
    dc.moves += static_cast<unsigned>(applied);
    dc.containers += applied > 0 ? 1u : 0u;
    __syncwarp();
    return -1;
  }
  dc.moves += static_cast<unsigned>(applied);
  dc.containers += applied > 0 ? 1u : 0u;
  __syncwarp();
  return applied;
}

// Rate-distortion fill (drift mode 1) of one container that fits, by the
// whole warp: qd[] holds the symbols after drift, q0[] the quantiser's, u[k]
// this lane's coordinates lane + 32 k. A candidate is a symbol whose nearest
// level j (least (u - y_j)^2 in fp32, ties to the lower level) is one level
// from qd and at most one from q0, with dD = (u - y_j)^2 - (u - y_qd)^2 < 0 and
// dR = cost_j - cost_qd > 0; candidates go in order of dD / dR (fp32, ties to
// the lower index), each kept if the string with it and every earlier kept
// candidate still fits. Stores the container; returns the number of symbols
// moved.
//
// The keys do not change while candidates are kept, so a pass tests 32 at
// once: from the next untested rank p, lane m encodes the current string with
// candidate p + m alone applied. Candidates p .. p + m* - 1 before the first
// one that fits (m*) do not fit on the string they are tested on in the
// one-at-a-time order either (nothing was kept between), so they are
// dropped; p + m* is kept, lane m* stores its string (the container as
// stored before the fill stands when nothing is kept) and the next pass
// starts after it. cand[] (128 entries) holds the ranked candidates (symbol
// index | target << 8).
template <bool kTwo>
__device__ __forceinline__ int rd_fill(const AppendArgs &a, const StreamCtx &c, const AppendTables &T,
                                       uint8_t *stack, const uint8_t *q0, uint8_t *qd, uint16_t *cand, int64_t v,
                                       uint16_t n16, const float (&u)[4], int lane) {
  uint32_t key[4];
  uint8_t jn[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = lane + 32 * k;
    int j = 0;
    float best = 0.0f;
    for (int l = 0; l < c.nl; ++l) {
      const float d = __fsub_rn(u[k], T.lev[l]);
      const float e = __fmul_rn(d, d);
      if (l == 0 || e < best) {
        best = e;
        j = l;
      }
    }
    const int s = qd[i];
    jn[k] = static_cast<uint8_t>(j);
    key[k] = kNoKey;
    if (j != s && abs(j - s) == 1 && abs(j - static_cast<int>(q0[i])) <= 1) {
      const float dj = __fsub_rn(u[k], T.lev[j]);
      const float ds = __fsub_rn(u[k], T.lev[s]);
      const float dd = __fsub_rn(__fmul_rn(dj, dj), __fmul_rn(ds, ds));
      const float dr = __fsub_rn(T.cost[j], T.cost[s]);
      if (dd < 0.0f && dr > 0.0f) key[k] = order_bits(__fdiv_rn(dd, dr));
    }
  }
  uint8_t *stk = stack + lane;
  bool dropped = false;
  uint8_t *dst = c.dst_of(a, v, &dropped);
  int ups = 0, ranked = 0, p = 0;
  bool exhausted = false;
  for (;;) {
    // Ranks p .. p + 31 (as far as there are candidates).
    while (!exhausted && ranked < p + 32) {
      const int bi = warp_argmin(key, lane);
      if (bi < 0) {
        exhausted = true;
        break;
      }
      if ((bi & 31) == lane) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (bi == lane + 32 * k) {
            key[k] = kRankedKey;
            cand[ranked] = static_cast<uint16_t>(bi | (jn[k] << 8));
          }
      }
      ++ranked;
    }
    if (p >= ranked) break;
    __syncwarp();
    const bool has = p + lane < ranked;
    const uint32_t cw = has ? cand[p + lane] : 0xFFFFu;
    const int ci = static_cast<int>(cw & 0xFFu);  // 255: no candidate (matches no symbol)
    const uint32_t ct = cw >> 8;
    uint32_t x = 0;
    const int len = encode_bf<kTwo, false>(
        [&](int i) { return i == ci ? ct : static_cast<uint32_t>(qd[i]); }, T.es, stk, &x);
    const unsigned fit = __ballot_sync(kFull, has && len <= c.P);
    __syncwarp();
    if (fit) {
      const int m = __ffs(fit) - 1;
      if (lane == m) {
        qd[ci] = static_cast<uint8_t>(ct);
        if (dst) store_container(dst, c.C, n16, x, stk, len);
      }
      ++ups;
      p += m + 1;
    } else {
      p += 32;
    }
    __syncwarp();
  }
  return ups;
}

__device__ __forceinline__ void add_stats(const AppendArgs &a, bool is_v, const DriftCount &dc, unsigned nf,
                                          unsigned drops, unsigned bad_pages = 0) {
  if (!a.stats) return;
  if (bad_pages) atomicAdd(&a.stats->bad_pages, (unsigned long long)bad_pages);
  if (dc.moves) atomicAdd(is_v ? &a.stats->v_syms_drifted : &a.stats->k_syms_drifted, (unsigned long long)dc.moves);
  if (dc.containers)
    atomicAdd(is_v ? &a.stats->v_cont_drifted : &a.stats->k_cont_drifted, (unsigned long long)dc.containers);
  if (dc.fallbacks) atomicAdd(&a.stats->overflow_fallbacks, (unsigned long long)dc.fallbacks);
  if (dc.filled)
    atomicAdd(is_v ? &a.stats->v_syms_filled : &a.stats->k_syms_filled, (unsigned long long)dc.filled);
  if (nf) atomicAdd(&a.stats->nonfinite_inputs, (unsigned long long)nf);
  if (drops) atomicAdd(&a.stats->dropped_writes, (unsigned long long)drops);
}

// Lane-per-vector body: 32 consecutive vectors per warp.
template <bool kBF16, bool kTwo>
__device__ __forceinline__ void lane_body(const AppendArgs &a, AppendTables &T, WarpArea &W, bool is_v) {
  const int lane = threadIdx.x & 31;
  const StreamCtx c = stream_setup(a, T, is_v, static_cast<int>(threadIdx.x));
  __syncthreads();
  const int64_t v0 = (static_cast<int64_t>(blockIdx.x) * kAW + (threadIdx.x >> 5)) * 32;
  if (v0 >= c.nvec) return;
  const int64_t v = v0 + lane;
  const bool valid = v < c.nvec;

  // ---- phases 1 and 2: lane per vector ----
  uint8_t *stk = W.stack + lane;
  uint16_t n16 = 0;
  bool nf = false, dropped = false, too_long = false, bad_page = false;
  int vb = 0, vh = 0;
  int64_t vj = 0;
  if (valid) c.split(a, v, &vb, &vh, &vj);
  W.head[lane] = vh;
  __syncwarp();
  quad_prepare<kBF16>(a, c, W, v0, lane);
  __syncwarp();
  if (valid) {
    n16 = W.n16[lane];
    nf = W.nf[lane] != 0;
    // The encode loop reads the symbols from shared memory so that it can
    // stay rolled (a fully unrolled loop adds ~40 KB of code).
    const uint8_t *sy = reinterpret_cast<const uint8_t *>(&W.syms[0][lane]);
    uint32_t x = 0;
    const int len = encode_bf<kTwo, false>([&](int i) { return static_cast<uint32_t>(sy[(i >> 2) * 128 + (i & 3)]); },
                                           T.es, stk, &x);
    too_long = len > c.P;
    uint8_t *dst = c.dst_at(a, vb, vh, vj, &dropped, &bad_page);
    if (!too_long && dst) store_container(dst, c.C, n16, x, stk, len);
  }
  unsigned drift_mask = __ballot_sync(kFull, too_long);
  const unsigned nf_mask = __ballot_sync(kFull, valid && nf);
  const unsigned drops = __ballot_sync(kFull, dropped);
  const unsigned bads = __ballot_sync(kFull, bad_page);
  DriftCount dc;

  if (a.drift_list) {
    // List the over-long containers for the drift kernel (one atomic per
    // warp); in drift mode 1 every vector, over-long ones with bit 31 set,
    // for the drift kernel's fill.
    const bool listed = a.drift_mode == 1 ? valid : too_long;
    const unsigned list_mask = __ballot_sync(kFull, listed);
    uint32_t base = 0;
    if (lane == 0 && list_mask) base = atomicAdd(&a.drift_count[is_v ? 1 : 0], static_cast<uint32_t>(__popc(list_mask)));
    base = __shfl_sync(kFull, base, 0);
    if (listed)
      a.drift_list[(is_v ? a.list_cap : 0) + base + __popc(list_mask & ((1u << lane) - 1u))] =
          static_cast<uint32_t>(v) | (a.drift_mode == 1 && too_long ? 0x80000000u : 0u);
    drift_mask = 0;
  }

  // ---- phase 3: warp per over-long container (E6 drift) ----
  while (drift_mask) {
    const int vv = __ffs(drift_mask) - 1;
    drift_mask &= drift_mask - 1;
    const int64_t vd = v0 + vv;
    float u[4];
    uint16_t n16v;
    bool nfv;
    warp_prepare(a, c.src, vd, c.head_of(a, vd), c.t, lane, u, W.q, &n16v, &nfv);
    __syncwarp();
    // Most containers need a few moves: rank 8 first (throughput).
    drift_one<kTwo>(a, c, T, W.stack, W.q, W.rank, W.tgt, vd, n16v, u, lane, 8, dc);
  }
  if (lane == 0) add_stats(a, is_v, dc, __popc(nf_mask), __popc(drops), __popc(bads));
}

// Warp-per-vector body for small appends (a decode step): many warps with
// one vector each, so drift and latency spread over the whole GPU.
template <bool kTwo>
__device__ __forceinline__ void warp_body(const AppendArgs &a, AppendTables &T, WarpArea &W, bool is_v) {
  const int lane = threadIdx.x & 31;
  const StreamCtx c = stream_setup(a, T, is_v, static_cast<int>(threadIdx.x));
  __syncthreads();
  const int64_t v = static_cast<int64_t>(blockIdx.x) * kAW + (threadIdx.x >> 5);
  if (v >= c.nvec) return;
  float u[4];
  uint16_t n16;
  bool nf;
  warp_prepare(a, c.src, v, c.head_of(a, v), c.t, lane, u, W.q, &n16, &nf);
  __syncwarp();
  bool dropped = false, bad_page = false;
  uint8_t *dst = c.dst_of(a, v, &dropped, &bad_page);
  DriftCount dc;
  int applied = 0;
  // The string's ideal length, the sum of its symbols' costs in bits. An
  // encoded string pushes at most that + a fraction of a bit, so a string
  // that ends up too long (more than P - 3 pushes) costs nearly 8 (P - 2)
  // bits or more. Above 8 (P - 3) + 4 bits the warp ranks its moves before
  // encoding and tries 0 .. 31 moves in one pass (the greedy result as
  // before, without a first encode that would fail); below it, one encode,
  // and drift after it in the rare case that the string is still too long.
  float cbits = 0.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k) cbits += T.cost[W.q[lane + 32 * k]];
  cbits = warp_sum(cbits);
  const bool spec = __shfl_sync(kFull, cbits > 8.0f * static_cast<float>(c.P - 3) + 4.0f, 0);
  bool drifted = spec;
  int len = 0;
  if (spec) {
    applied = drift_one<kTwo>(a, c, T, W.stack, W.q, W.rank, W.tgt, v, n16, u, lane, 32, dc, true);
  } else {
    uint8_t *stk = W.stack + lane;
    uint32_t x = 0;
    len = encode_bf<kTwo, false>([&](int i) { return static_cast<uint32_t>(W.q[i]); }, T.es, stk, &x);
    if (len <= c.P) {
      // Every lane encoded the same string: lane k stores byte k from its own stack.
      if (dst) store_container_warp(dst, c.C, n16, x, W.stack, lane, len, lane);
    } else {
      __syncwarp();
      drifted = true;
      applied = drift_one<kTwo>(a, c, T, W.stack, W.q, W.rank, W.tgt, v, n16, u, lane, 16, dc);
    }
  }
  if (a.drift_mode == 1 && applied >= 0) {
    // The symbols after drift (the first `applied` ranked moves) go to tgt[].
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = lane + 32 * k;
      const uint32_t r = drifted ? W.rank[i] : kNoRank;
      W.tgt[i] = (r != kNoRank && static_cast<int>(r) < applied) ? W.tgt[i] : W.q[i];
    }
    __syncwarp();
    const int ups = rd_fill<kTwo>(a, c, T, W.stack, W.q, W.tgt, reinterpret_cast<uint16_t *>(&W.syms[0][0]), v, n16,
                                  u, lane);
    if (lane == 0 && ups && a.stats)
      atomicAdd(is_v ? &a.stats->v_syms_filled : &a.stats->k_syms_filled, static_cast<unsigned long long>(ups));
  }
  if (lane == 0) add_stats(a, is_v, dc, nf ? 1u : 0u, dropped ? 1u : 0u, bad_page ? 1u : 0u);
}

// Drift kernel: each warp keeps kSlots listed containers in flight. One
// encode pass tries kWin consecutive move counts of every one of them (lane
// kWin c + j: container c with its ranked moves 0 .. win_c + j applied); the
// first count that fits is the greedy result, the container is stored and
// its slot takes the next list entry. A container with no fitting count in
// its window ranks kWin more moves (the keys of the moves not yet ranked stay
// in shared memory) and is tried again in the next pass; one whose candidates
// run out tries the fallback string on the last lane of its window.
constexpr int kSlots = 8;
constexpr int kWin = 4;
static_assert(kSlots * kWin == 32, "one trial per lane");
constexpr int kDriftWarps = 4;  // warps per drift CTA
constexpr int kDriftCtas = 7;   // drift CTAs per SM the register budget is set for

// kStk push-stack slots per lane: 32 when both containers hold at most 36
// bytes (a string that fits pushes at most C - 5 <= 31 bytes; longer trials
// wrap around and are never stored), else 64.
template <int kStk>
struct DriftArea {
  uint8_t stack[kStk * 32];
  uint16_t sw[kD][kSlots];      // symbol i of slot c: q | tgt << 3 | rank << 6 (kNoRank: not ranked)
  uint32_t key[kSlots][4][32];  // order_bits of the move key of symbol l + 32 k; kRankedKey once ranked
  int64_t vd[kSlots];
  int32_t ranked[kSlots], win[kSlots];
  uint16_t pend[kSlots][kWin];  // fill phase: ranked, untested candidates (index | target << 8)
  int32_t npend[kSlots];
  uint16_t n16[kSlots];
  AppendTables T;
};

// Rate-distortion fill keys of the symbols this lane owns in slot s (drift
// mode 1; the rule of rd_fill): q0 are the quantiser's symbols, qd the
// symbols after drift. The slot's words become qd | nearest level << 3.
template <int kStk>
__device__ __forceinline__ void fill_keys(DriftArea<kStk> &A, int nl, int s, const float (&u)[4],
                                          const uint32_t (&q0)[4], const uint32_t (&qd)[4], int lane) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int j = 0;
    float best = 0.0f;
    for (int l = 0; l < nl; ++l) {
      const float d = __fsub_rn(u[k], A.T.lev[l]);
      const float e = __fmul_rn(d, d);
      if (l == 0 || e < best) {
        best = e;
        j = l;
      }
    }
    const int sd = static_cast<int>(qd[k]);
    uint32_t key = kNoKey;
    if (j != sd && abs(j - sd) == 1 && abs(j - static_cast<int>(q0[k])) <= 1) {
      const float dj = __fsub_rn(u[k], A.T.lev[j]);
      const float ds = __fsub_rn(u[k], A.T.lev[sd]);
      const float dd = __fsub_rn(__fmul_rn(dj, dj), __fmul_rn(ds, ds));
      const float dr = __fsub_rn(A.T.cost[j], A.T.cost[sd]);
      if (dd < 0.0f && dr > 0.0f) key = order_bits(__fdiv_rn(dd, dr));
    }
    A.key[s][k][lane] = key;
    A.sw[lane + 32 * k][s] =
        static_cast<uint16_t>(qd[k] | (static_cast<uint32_t>(j) << 3) | (static_cast<uint32_t>(kNoRank) << 6));
  }
}

// E6 (and, with kFill, the rate-distortion fill of drift mode 1) for one
// stream's list: entries first, first + stride, ... . With kFill the list
// holds every vector (bit 31: over-long); an over-long one drifts first and
// goes on to the fill from its drifted symbols, the others go straight to
// the fill. A fill pass tests up to kWin ranked candidates of a slot, each
// applied alone to the current string (lane kWin c + j: candidate j of the
// slot's queue); the first that fits is kept and stored by its lane, the
// ones before it are dropped and the ones after it stay queued. The keys do
// not change while candidates are kept, so this is the one-at-a-time order's
// result.
template <bool kTwo, int kStk, bool kFill>
__device__ __forceinline__ void drift_stream(const AppendArgs &a, DriftArea<kStk> &A, bool is_v, int lane,
                                             uint32_t first, uint32_t stride, DriftCount &dc) {
  __syncwarp();
  const StreamCtx c = stream_setup(a, A.T, is_v, lane);
  if (lane < kSlots) {
    A.ranked[lane] = 0;
    A.win[lane] = 0;
    A.npend[lane] = 0;
  }
  __syncwarp();
  const uint32_t n = a.drift_count[is_v ? 1 : 0];
  const uint32_t *list = a.drift_list + (is_v ? a.list_cap : 0);
  uint8_t *stk = A.stack + lane;
  const int cs = lane / kWin, jw = lane % kWin;
  const uint32_t hlf = static_cast<uint32_t>(c.nl / 2);
  uint64_t cursor = first;
  // Warp-uniform slot masks: holds a container; candidates ran out; in the
  // fill phase; drifted to a fit and waiting for its fill keys.
  uint32_t live = 0, exh = 0, fil = 0, fsu = 0;
  for (;;) {
    if constexpr (kFill) {
      // Slots that drifted to a fit: fill keys from the drifted symbols
      // (the first A.win[s] ranked moves applied).
#pragma unroll 1
      for (int s = 0; s < kSlots; ++s) {
        if (!((fsu >> s) & 1u)) continue;
        const int64_t v = A.vd[s];
        const int applied = A.win[s];
        float u[4];
        uint32_t q0[4], qd[4];
        uint16_t n16v;
        bool nf;
        warp_prepare_regs(a, c.src, v, c.head_of(a, v), c.t, lane, u, q0, &n16v, &nf);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t w = A.sw[lane + 32 * k][s];
          qd[k] = (static_cast<int>(w >> 6) < applied) ? ((w >> 3) & 7u) : (w & 7u);
        }
        __syncwarp();
        fill_keys(A, c.nl, s, u, q0, qd, lane);
        if (lane == 0) A.npend[s] = 0;
        fsu &= ~(1u << s);
        fil |= 1u << s;
        exh &= ~(1u << s);
      }
    }
    // Free slots take the next list entries.
#pragma unroll 1
    for (int s = 0; s < kSlots && cursor < n; ++s) {
      if ((live >> s) & 1u) continue;
      const uint32_t e = list[cursor];
      cursor += stride;
      const int64_t v = kFill ? static_cast<int64_t>(e & 0x7FFFFFFFu) : static_cast<int64_t>(e);
      const bool over = kFill ? (e >> 31) != 0 : true;
      float u[4];
      uint32_t qk[4];
      uint16_t n16v;
      bool nf;
      warp_prepare_regs(a, c.src, v, c.head_of(a, v), c.t, lane, u, qk, &n16v, &nf);
      if (over) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          int tj;
          A.key[s][k][lane] = order_bits(best_move(A.T, c.nl, static_cast<int>(qk[k]), u[k], &tj));
          A.sw[lane + 32 * k][s] = static_cast<uint16_t>(qk[k] | (static_cast<uint32_t>(tj) << 3) |
                                                         (static_cast<uint32_t>(kNoRank) << 6));
        }
        fil &= ~(1u << s);
      } else {
        fill_keys(A, c.nl, s, u, qk, qk, lane);
        fil |= 1u << s;
      }
      if (lane == 0) {
        A.vd[s] = v;
        A.n16[s] = n16v;
        A.ranked[s] = 0;
        A.win[s] = 0;
        A.npend[s] = 0;
      }
      live |= 1u << s;
      exh &= ~(1u << s);
    }
    if (!live) break;
    __syncwarp();
    // Ranking by repeated arg-min over (key, index): the least key over the
    // warp, then the lowest index holding it. Drift slots rank their moves up
    // to win + kWin; fill slots top their queue up to kWin candidates.
#pragma unroll 1
    for (int s = 0; s < kSlots; ++s) {
      if (!(((live & ~exh) >> s) & 1u)) continue;
      const bool fs = kFill && ((fil >> s) & 1u);
      int r = fs ? A.npend[s] : A.ranked[s];
      const int target = fs ? kWin : A.win[s] + kWin;
      if (r >= target) continue;
      uint32_t key[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) key[k] = A.key[s][k][lane];
      for (; r < target; ++r) {
        const int bi = warp_argmin(key, lane);
        if (bi < 0) {
          exh |= 1u << s;
          break;
        }
        if ((bi & 31) == lane) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (bi == lane + 32 * k) key[k] = kRankedKey;
          const uint32_t w = A.sw[bi][s];
          if (fs) A.pend[s][r] = static_cast<uint16_t>(bi | (((w >> 3) & 7u) << 8));
          else A.sw[bi][s] = static_cast<uint16_t>((w & 0x3Fu) | (static_cast<uint32_t>(r) << 6));
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) A.key[s][k][lane] = key[k];
      if (lane == 0) {
        if (fs) A.npend[s] = r;
        else A.ranked[s] = r;
      }
    }
    __syncwarp();
    // One encode pass. An exhausted drift slot has ranked < win + kWin, so the
    // last lane of its window is free for the fallback string (all ranked
    // moves, then every symbol to the innermost level of its side).
    const bool mine = (live >> cs) & 1u;
    // A lane whose slot is empty encodes a live slot's string (its words
    // were all written at refill, every symbol below nl); its result is
    // not used.
    const int cr = mine ? cs : __ffs(live) - 1;
    const uint16_t *swc = &A.sw[0][cr];
    const bool lf = kFill && ((fil >> cr) & 1u);
    const int win = A.win[cs], ranked = A.ranked[cs];
    const int km = win + jw;
    const bool trial = mine && !lf && km < ranked;
    const bool fb = mine && !lf && ((exh >> cs) & 1u) && jw == kWin - 1;
    const bool has = mine && lf && jw < A.npend[cs];
    const uint32_t cw = has ? A.pend[cs][jw] : 0xFFFFu;
    const int ci = static_cast<int>(cw & 0xFFu);  // 255 (no candidate) matches no symbol
    const uint32_t ct = cw >> 8;
    uint32_t x = 0;
    int len;
    if (__any_sync(kFull, fb)) {
      const uint32_t kmx = fb ? 254u : static_cast<uint32_t>(km);
      auto sym = [&](int i) {
        const uint32_t w = swc[i * kSlots];
        uint32_t sy = ((w >> 6) <= kmx) ? ((w >> 3) & 7u) : (w & 7u);
        if constexpr (kFill) {
          if (lf) sy = (i == ci) ? ct : (w & 7u);
        }
        if (fb) sy = sy >= hlf ? hlf : hlf - 1u;
        return sy;
      };
      len = encode_bf<kTwo, false, decltype(sym), kStk>(sym, A.T.es, stk, &x);
    } else {
      const uint32_t kmx = static_cast<uint32_t>(km);
      auto sym = [&](int i) {
        const uint32_t w = swc[i * kSlots];
        uint32_t sy = ((w >> 6) <= kmx) ? ((w >> 3) & 7u) : (w & 7u);
        if constexpr (kFill) {
          if (lf) sy = (i == ci) ? ct : (w & 7u);
        }
        return sy;
      };
      len = encode_bf<kTwo, false, decltype(sym), kStk>(sym, A.T.es, stk, &x);
    }
    const bool ok = len <= c.P;
    const unsigned fit = __ballot_sync(kFull, (trial || has) && ok);
    const unsigned fc = (fit >> (kWin * cs)) & ((1u << kWin) - 1u);
    const bool store = fc ? (jw == __ffs(fc) - 1) : (fb && ok);
    __syncwarp();  // every lane has read the slot words of this pass
    if (store) {
      bool dr = false;
      uint8_t *dst = c.dst_of(a, A.vd[cs], &dr);
      if (dst) store_container(dst, c.C, A.n16[cs], x, stk, len);
      if (kFill && lf) A.sw[ci][cs] = static_cast<uint16_t>((A.sw[ci][cs] & ~7u) | ct);  // kept: new string
    }
    // Slot bookkeeping (warp-uniform).
    uint32_t drifting = 0;  // drift slots that go on to their next window
#pragma unroll 1
    for (int s = 0; s < kSlots; ++s) {
      if (!((live >> s) & 1u)) continue;
      const unsigned f = (fit >> (kWin * s)) & ((1u << kWin) - 1u);
      if (kFill && ((fil >> s) & 1u)) {
        const int np = A.npend[s];
        const int used = f ? __ffs(f) : np;  // tested candidates resolved by this pass
        if (f) dc.filled += 1;
        __syncwarp();
        if (lane == 0) {
          for (int t = used; t < np; ++t) A.pend[s][t - used] = A.pend[s][t];
          A.npend[s] = np - used;
        }
        if (np - used == 0 && ((exh >> s) & 1u)) {
          live &= ~(1u << s);
          fil &= ~(1u << s);
        }
      } else if (f) {
        dc.moves += static_cast<unsigned>(A.win[s] + __ffs(f));
        dc.containers += 1;
        if constexpr (kFill) {
          __syncwarp();
          if (lane == 0) A.win[s] = A.win[s] + __ffs(f);  // moves applied
          fsu |= 1u << s;
        } else {
          live &= ~(1u << s);
        }
      } else if ((exh >> s) & 1u) {
        const int r = A.ranked[s];
        dc.fallbacks += 1;
        dc.moves += static_cast<unsigned>(r);
        dc.containers += r > 0 ? 1u : 0u;
        live &= ~(1u << s);
      } else {
        drifting |= 1u << s;
      }
    }
    __syncwarp();
    if (lane < kSlots && ((drifting >> lane) & 1u)) A.win[lane] += kWin;
    __syncwarp();
  }
}

// Every warp walks its share of the K list, then of the V list, so the two
// streams' lists (often of very different lengths) spread over all warps.
// kWhich 0 or 1: the K or the V list only (drift mode 1, whose lists hold
// every vector and so have equal lengths: one launch per stream keeps each
// launch's code to one stream's body, which the fill phase makes large).
template <bool kTwoK, bool kTwoV, int kStk, bool kFill, int kWhich>
__global__ void __launch_bounds__(kDriftWarps * 32, kDriftCtas) append_drift_kernel(const AppendArgs a) {
  __shared__ DriftArea<kStk> A[kDriftWarps];
  const int lane = threadIdx.x & 31;
  DriftArea<kStk> &w = A[threadIdx.x >> 5];
  const uint32_t first = blockIdx.x * kDriftWarps + (threadIdx.x >> 5);
  const uint32_t stride = gridDim.x * kDriftWarps;
  DriftCount dk, dv;
  if constexpr (kWhich != 1) drift_stream<kTwoK, kStk, kFill>(a, w, false, lane, first, stride, dk);
  if constexpr (kWhich != 0) drift_stream<kTwoV, kStk, kFill>(a, w, true, lane, first, stride, dv);
  if (lane == 0) {
    add_stats(a, false, dk, 0u, 0u);
    add_stats(a, true, dv, 0u, 0u);
  }
}

// One CTA = kAW warps of one stream (blockIdx.y: 0 = K, 1 = V).
template <bool kBF16, bool kTwoK, bool kTwoV>
__global__ void __launch_bounds__(kAW * 32, 8) append_lane_kernel(const AppendArgs a) {
  __shared__ AppendTables T;
  __shared__ WarpArea W[kAW];
  const bool is_v = blockIdx.y == 1;
  WarpArea &w = W[threadIdx.x >> 5];
  if constexpr (kTwoK == kTwoV) {
    lane_body<kBF16, kTwoK>(a, T, w, is_v);
  } else {
    if (is_v) lane_body<kBF16, kTwoV>(a, T, w, true);
    else lane_body<kBF16, kTwoK>(a, T, w, false);
  }
}

template <bool kTwoK, bool kTwoV>
__global__ void __launch_bounds__(kAW * 32) append_warp_kernel(const AppendArgs a) {
  __shared__ AppendTables T;
  __shared__ WarpArea W[kAW];
  const bool is_v = blockIdx.y == 1;
  WarpArea &w = W[threadIdx.x >> 5];
  if constexpr (kTwoK == kTwoV) {
    warp_body<kTwoK>(a, T, w, is_v);
  } else {
    if (is_v) warp_body<kTwoV>(a, T, w, true);
    else warp_body<kTwoK>(a, T, w, false);
  }
}

template <bool kTwoK, bool kTwoV, int kStk, bool kFill, int kWhich>
int launch_drift_one(const AppendArgs &a, int sms, cudaStream_t st) {
  static int per_sm = 0;
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, append_drift_kernel<kTwoK, kTwoV, kStk, kFill, kWhich>,
                                                      kDriftWarps * 32, 0) != cudaSuccess ||
        n < 1)
      n = 1;
    per_sm = n;
  }
  append_drift_kernel<kTwoK, kTwoV, kStk, kFill, kWhich>
      <<<static_cast<unsigned>(per_sm * sms), kDriftWarps * 32, 0, st>>>(a);
  return static_cast<int>(cudaGetLastError());
}

template <bool kTwoK, bool kTwoV, int kStk, bool kFill>
int launch_drift(const AppendArgs &a, int sms, cudaStream_t st) {
  if constexpr (!kFill) return launch_drift_one<kTwoK, kTwoV, kStk, false, -1>(a, sms, st);
  const int e = launch_drift_one<kTwoK, kTwoV, kStk, true, 0>(a, sms, st);
  if (e != 0) return e;
  return launch_drift_one<kTwoK, kTwoV, kStk, true, 1>(a, sms, st);
}

template <bool kBF16, bool kTwoK, bool kTwoV>
int launch_two(const AppendArgs &a, bool lanes, int64_t nvec, int sms, cudaStream_t st) {
  const int64_t per_cta = lanes ? static_cast<int64_t>(kAW) * 32 : kAW;
  const int64_t gx = (nvec + per_cta - 1) / per_cta;
  if (gx > 0x7FFFFFFF) return static_cast<int>(cudaErrorInvalidConfiguration);
  const dim3 grid(static_cast<unsigned>(gx), 2);
  if (!lanes) {
    append_warp_kernel<kTwoK, kTwoV><<<grid, kAW * 32, 0, st>>>(a);
    return static_cast<int>(cudaGetLastError());
  }
  if (a.drift_list) {
    const cudaError_t e = cudaMemsetAsync(a.drift_count, 0, 2 * sizeof(uint32_t), st);
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  append_lane_kernel<kBF16, kTwoK, kTwoV><<<grid, kAW * 32, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !a.drift_list) return static_cast<int>(e);
  // Drift: a persistent grid, as many CTAs as fit on the SMs at once.
  const bool small = a.ck <= 36 && a.cv <= 36;
  if (a.drift_mode == 1)
    return small ? launch_drift<kTwoK, kTwoV, 32, true>(a, sms, st) : launch_drift<kTwoK, kTwoV, 64, true>(a, sms, st);
  return small ? launch_drift<kTwoK, kTwoV, 32, false>(a, sms, st) : launch_drift<kTwoK, kTwoV, 64, false>(a, sms, st);
}

template <bool kBF16>
int launch_dtype(const AppendArgs &a, bool lanes, int64_t nvec, int sms, cudaStream_t st) {
  if (a.two_k && a.two_v) return launch_two<kBF16, true, true>(a, lanes, nvec, sms, st);
  if (a.two_k) return launch_two<kBF16, true, false>(a, lanes, nvec, sms, st);
  if (a.two_v) return launch_two<kBF16, false, true>(a, lanes, nvec, sms, st);
  return launch_two<kBF16, false, false>(a, lanes, nvec, sms, st);
}

}  // namespace

int launch_append(const AppendArgs &a, void *stream) {
  if (a.ck > kMaxContainer || a.cv > kMaxContainer) return static_cast<int>(cudaErrorInvalidValue);
  const int64_t nvec = static_cast<int64_t>(a.B) * a.Hkv * a.n_new;
  if (nvec == 0) return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Lane per vector once every SM gets a few full CTAs of 128 vectors per
  // stream; below that, a warp per vector spreads the work wider.
  bool lanes = nvec >= static_cast<int64_t>(sms) * kAW * 32 * 2;
  AppendArgs b = a;
  // The drift list holds 32-bit vector indices, one slot per vector.
  if (!lanes || b.list_cap < nvec || nvec > 0xFFFFFFFFll) b.drift_list = nullptr;
  // Drift mode 1 needs the list (its fill runs in the drift kernel, with the
  // over-long flag in bit 31); without it, the warp-per-vector kernel fills.
  if (a.drift_mode == 1 && (!b.drift_list || nvec > 0x7FFFFFFFll)) {
    lanes = false;
    b.drift_list = nullptr;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return b.dtype == DQ_BF16 ? launch_dtype<true>(b, lanes, nvec, sms, st) : launch_dtype<false>(b, lanes, nvec, sms, st);
}

size_t append_workspace_bytes(int64_t nvec) {
  return 256 + 2 * static_cast<size_t>(nvec) * sizeof(uint32_t);
}

}  // namespace dqi
