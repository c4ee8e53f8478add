// dq_prefill.cu -- chunked-prefill attention over the compressed KV cache,
// on the sm_100 tensor cores (tcgen05, accumulators in tensor memory).
//
// [abstract] "D-Quant: Driftable Entropy Coding for KV Cache Quantization":
// fixed-size bitstreams give regular memory access and parallel
// dequantisation within attention kernels. [news] "D-Quant: Entropy Coding
// Meets KV Cache at 2.26 Bits", "The Numbers": the method is evaluated on
// long prompts (8K to 128K); a prompt processed in chunks attends, chunk by
// chunk, over the compressed cache that already holds the chunk's own keys
// and values. Query token i of sequence b sits at position q_start[b] + i and
// attends causally to cache positions 0 .. q_start[b] + i.
//
// Two kernels.
//
// prefill_tiles_kernel decodes every 32-token block of K and V that the chunk
// attends to, once per (b, KV head), into the workspace: one slot per block
// holds a K tile and a V tile (32 tokens x 128 coordinates, fp16 levels in the
// tensor cores' no-swizzle core-matrix layout: token t, coordinate i at byte
// (t/8)*128 + (i/8)*512 + (t%8)*16 + (i%8)*2) and the tokens' K and V norms.
// K levels are kappa_K y with kappa_K chosen to minimise the frequency-
// weighted level error, V levels kappa_V y as in decode attention. Every warp
// of a persistent grid takes blocks in a strided order; a lane decodes one
// token's K and V (two interleaved rANS chains) from the byte-interleaved
// containers staged in shared memory with cp.async, one block ahead.
//
// prefill_kernel: one CTA per (b, KV head h, block of 128 query rows); a row is
// one query token of the chunk with one of the G query heads of h (row r =
// token r / G, head r % G). The CTAs of one (b, h) are launched together (the
// longest causal ranges first) so that its tiles are read from L2. Warps:
//   0-15 softmax: the four warps w, w + 4, w + 8, w + 12 share rows
//        32 (w % 4) .. + 31 (thread = row = lane of tensor memory); warp
//        w + 4 q takes tokens 32 q .. 32 q + 31 of every block. The row's
//        four threads rotate its query (q~ = H D q in fp32, times a power of
//        two; stages h = 1 .. 16 on 32 coordinates each in registers, h = 32
//        and 64 after an exchange through tensor memory), split it into fp16
//        hi + lo and store both into tensor memory; per block j each reads
//        its 32 scores, applies the key norms, the scale and the causal
//        mask, and the four meet (shared memory, a named barrier per row
//        group) on the row maximum; the online softmax rescales the row's O
//        in tensor memory (32 columns per thread) when the running maximum
//        grows, and each thread stores its tokens' weights w = p ||v|| as fp16
//        hi + lo into tensor memory. At the end the four apply 1 / (128 l
//        kappa_V), the inverse rotation D H (split as for q~) and write the
//        output row.
//   16   owns the tensor memory and issues the score MMAs
//          S_j = q~hi K_j^T + q~lo K_j^T        (M 128, N 128, K 128)
//   17   issues the P.V MMAs
//          O  += W_j,hi V_j + W_j,lo V_j         (M 128, N 128, K 128)
//        kind::f16 with fp32 accumulators, A from tensor memory, B (K tile
//        K-major, V tile MN-major) from shared memory. Two issuing warps on
//        two schedulers: each shares its scheduler with four softmax warps,
//        and one warp issuing all 32 MMAs of a block fell behind the tensor
//        core. The barriers order the two streams.
//   18   one lane streams the slots into a ring in shared memory with bulk
//        copies counted on mbarriers.
// The softmax arithmetic runs in packed fp32x2 operations (two tokens per
// instruction) and three-input maxima.
// Every wait is bounded; a CTA that gives up counts it in wait_timeouts,
// skips the rest of its work and still frees its tensor memory after its MMAs
// and copies have drained.
#include <type_traits>

#include "dq_device.cuh"

namespace dqi {
namespace {

constexpr int kRows = 128;          // query rows per CTA (the MMA's M)
constexpr int kGrp = 32;            // tokens per cache block (one decoder warp)
constexpr int kBlk = 128;           // tokens per workspace slot / attention block (the score MMA's N)
constexpr int kSoftWarps = 16;      // warps 0..15: warps w, w + 4, w + 8, w + 12 share rows 32 (w % 4) ..
constexpr int kQuads = kSoftWarps / 4;  // softmax warps per row (each takes 32 tokens of a block)
constexpr int kMmaWarp = 16;        // warp 16: score MMAs; allocates tensor memory
constexpr int kPvWarp = 17;         // warp 17: P.V MMAs
constexpr int kLoadWarp = 18;       // warp 18: slot loader
constexpr int kAttnThreads = 32 * 19;
constexpr int kMaxSlots = 3;        // ring depth of prefill_kernel
constexpr int kTileWarps = 20;      // warps per CTA of prefill_tiles_kernel
constexpr uint32_t kTmemCols = 512;
// Tensor-memory columns (32-bit each; 128 lanes = rows).
constexpr uint32_t kColO = 0;       // O: 128 fp32 columns
constexpr uint32_t kColQh = 128;    // q~ hi: 64 columns of packed fp16 pairs
constexpr uint32_t kColQl = 192;    // q~ lo: 64 columns
constexpr uint32_t kColS = 256;     // 2 buffers x 128 columns: the scores S (fp32), then in place the
                                    // weights W: per 32-token quarter, 16 columns of fp16 hi pairs,
                                    // then 16 of lo pairs
constexpr int kTileBytes = kBlk * kD * 2;                  // one fp16 tile: 128 tokens x 128 coordinates
constexpr int kQmaxOff = 2 * kTileBytes + 2 * kBlk * 4;    // after K tile, V tile, K norms, V norms: the
                                                           // largest V norm of each 32-token quarter
constexpr int kSlotBytes = kQmaxOff + 128;                 // (padded to 128 bytes)
constexpr int kChunkStride = kBlk / 8 * 128;               // bytes between 8-coordinate chunks of a tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kSpin = 1u << 24;  // bound on each mbarrier wait loop
constexpr float kLazyLog2 = 8.0f;      // lazy rescaling: largest growth (log2) of the row maximum kept stale
// Barrier slots of prefill_kernel.
constexpr int kBarFull = 0, kBarEmpty = kMaxSlots, kBarSFull = 2 * kMaxSlots, kBarWFull = kBarSFull + 2,
              kBarPvDone = kBarSFull + 4, kBarQFull = kBarSFull + 6, kBarDrain = kBarSFull + 7,
              kBarDrainPv = kBarSFull + 8, kNumBars = kBarSFull + 9;
static_assert(kSlotBytes % 16 == 0, "bulk copies move multiples of 16 bytes");

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared memory of prefill_tiles_kernel: decode tables, then per warp two
// staging slots for K and two for V.
struct TilesSmem {
  size_t lut_k, lut_v, lev, stage, kslot, vslot, stage_bytes, total;
};

__host__ __device__ inline TilesSmem tiles_smem_layout(int ck, int cv) {
  TilesSmem s;
  s.lut_k = 0;
  s.lut_v = s.lut_k + kM * 4;
  s.lev = s.lut_v + kM * 4;  // [0..7] K score levels, [8..15] V tile levels (fp16 bits)
  s.stage = align_up(s.lev + 2 * kMaxLevels * 4, 128);
  s.kslot = align_up(static_cast<size_t>(kGrp) * ck, 16);
  s.vslot = align_up(static_cast<size_t>(kGrp) * cv, 16);
  s.stage_bytes = 2 * s.kslot + 2 * s.vslot;
  const size_t end = s.stage + static_cast<size_t>(kTileWarps) * s.stage_bytes;
  // A corrupt container moves its decoder's cursor by at most 2 bytes per
  // symbol (byte 5 + 2 * 128 at most), 32 bytes apart in the interleaved
  // layout: reads from the last V slot stay inside the allocation.
  const size_t reach = end - s.vslot + static_cast<size_t>(kGrp) * (kHeaderBytes + 2 * kD + 1);
  s.total = (reach > end ? align_up(reach, 16) : end) + 256;
  return s;
}

// Shared memory of prefill_kernel: barriers, tensor-memory base and abort
// flag, the row-max and go-on exchanges [2 blocks][4 quarters][128 rows],
// the row-sum exchange [4 quarters][128 rows] of the softmax warps of a row,
// then the ring.
struct AttnSmem {
  size_t bars, misc, pmax, lsum, pgo, ring, total;
};

__host__ __device__ inline AttnSmem attn_smem_layout(int nslots) {
  AttnSmem s;
  s.bars = 0;
  s.misc = s.bars + kNumBars * 8;
  s.pmax = align_up(s.misc + 16, 16);
  s.lsum = s.pmax + 2 * kQuads * kRows * 4;
  s.pgo = s.lsum + kQuads * kRows * 4;
  s.ring = align_up(s.pgo + 2 * kQuads * kRows * 4, 128);
  s.total = s.ring + static_cast<size_t>(nslots) * kSlotBytes;
  return s;
}

// Last attended position of sequence b (-1: none) and its 32-token blocks.
__host__ __device__ __forceinline__ int64_t last_position(int64_t qs, int n_q, int64_t T_cap) {
  if (qs > T_cap - 1 || qs + n_q - 1 < 0) return -1;
  return qs + n_q - 1 < T_cap - 1 ? qs + n_q - 1 : T_cap - 1;
}

// ---- PTX wrappers -------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(smem_u32(bar)) : "memory");
}
// Waits for the phase with the given parity to complete. Gives up after
// kSpin polls, or as soon as another thread of the CTA has given up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t it = 0; it < kSpin; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred P;\nmbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\nselp.u32 %0, 1, 0, P;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((it & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Bulk copy (no tensor map, no multicast) of `bytes` (a multiple of 16, both
// addresses 16-byte aligned) from global to this CTA's shared memory;
// completion is counted on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
// d (+)= a b^T: A (M 128 x K 16 fp16) from tensor memory, B from a shared
// memory descriptor, fp32 accumulators in tensor memory. Called by a whole
// converged warp: every lane computes the operands and one elected lane (the
// same one on every call, lane 0) issues, so the operands stay warp-uniform.
// The issuing warp shares its scheduler with four softmax warps, and this
// form issues an MMA in fewer slots than a lane-0 branch.
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p, e;\n.reg .b32 r;\nsetp.ne.b32 p, %4, 0;\nelect.sync r|e, 0xffffffff;\n"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// Commit of the elected lane's MMAs to an mbarrier (called by the same
// converged warp as mma_ts).
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "{\n.reg .pred e;\n.reg .b32 r;\nelect.sync r|e, 0xffffffff;\n"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(smem_u32(bar))
      : "memory");
}
// Shared-memory matrix descriptor, no swizzle: start address, leading and
// stride byte offsets (16-byte units), version 1 (bits 46-47).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Instruction descriptor, kind f16: fp32 accumulators (bit 4), A and B fp16,
// A K-major, B K-major (0) or MN-major (1) at bit 16, N / 8 at bits 17-22,
// M / 16 at bits 24-28.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, int b_mn) {
  return (1u << 4) | (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// 32 consecutive fp32 columns of this warp's 32 lanes (one row per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 8 consecutive fp32 columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// 2^x with the hardware approximation (relative error about 2^-22; x <= 0
// here, results below 2^-126 flush to 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Largest of 32 values: 16 three-input maxima, depth 4.
__device__ __forceinline__ float max32(const float (&v)[32]) {
  float m[12];
#pragma unroll
  for (int i = 0; i < 10; ++i) m[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  m[10] = v[30];
  m[11] = v[31];
  const float a = fmax3(m[0], m[1], m[2]), b = fmax3(m[3], m[4], m[5]), c = fmax3(m[6], m[7], m[8]),
              d = fmax3(m[9], m[10], m[11]);
  return fmaxf(fmax3(a, b, c), d);
}
// fp16 hi + lo of a pair of non-negative fp32 values below 65504: hi is the
// value with its 13 low mantissa bits cleared (exact in fp16 from 2^-14 up),
// lo = w - hi (exact in fp32) rounded to fp16. Packed, first value low.
__device__ __forceinline__ void split_pair_trunc(float2 w, uint32_t &hi, uint32_t &lo) {
  const float2 hf = make_float2(__uint_as_float(__float_as_uint(w.x) & 0xFFFFE000u),
                                __uint_as_float(__float_as_uint(w.y) & 0xFFFFE000u));
  const float2 lf = __ffma2_rn(hf, make_float2(-1.0f, -1.0f), w);
  const __half2 h = __floats2half2_rn(hf.x, hf.y);
  const __half2 l = __floats2half2_rn(lf.x, lf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// fp16 hi + lo of a pair of fp32 values, packed (first value in the low half).
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// 32 consecutive elements base[idx .. idx + 31] (fp32 or bf16) into v. With
// vec (base 16-byte aligned; idx is a multiple of 32) as 16-byte loads: the
// 32 lanes of a warp read 32 different rows, so every load instruction
// touches 32 cache lines, and 4 (bf16) or 8 (fp32) of them replace 32.
__device__ __forceinline__ void load_row32(const void *base, int64_t idx, int dtype, bool vec, float (&v)[32]) {
  if (vec && dtype == DQ_BF16) {
    const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(base) + idx);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 u = __ldg(p + k);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * k + 2 * e] = __uint_as_float(w[e] << 16);
        v[8 * k + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  } else if (vec) {
    const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + idx);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 f = __ldg(p + k);
      v[4 * k] = f.x;
      v[4 * k + 1] = f.y;
      v[4 * k + 2] = f.z;
      v[4 * k + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = load_elem(base, idx + c, dtype);
  }
}
// 8 consecutive elements base[idx .. idx + 7] = z (fp32, or bf16 rounded to
// nearest even); with vec (base 16-byte aligned, idx a multiple of 8) as one
// (bf16) or two (fp32) 16-byte stores.
__device__ __forceinline__ void store_row8(void *base, int64_t idx, const float (&z)[8], int dtype, bool vec) {
  if (vec && dtype == DQ_BF16) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(z[2 * e], z[2 * e + 1]);
      w[e] = *reinterpret_cast<const uint32_t *>(&h);
    }
    *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(base) + idx) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (vec) {
    float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(base) + idx);
    p[0] = make_float4(z[0], z[1], z[2], z[3]);
    p[1] = make_float4(z[4], z[5], z[6], z[7]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) store_elem(base, idx + i, z[i], dtype);
  }
}

// ---- rANS decoding (one lane per token of a staged 32-token block) ------

struct RansLane {
  uint32_t x;
  uint32_t p;  // shared-memory offset of the next byte
};

__device__ __forceinline__ RansLane rans_open(const uint8_t *smem, uint32_t off) {
  RansLane r;
  r.x = static_cast<uint32_t>(smem[off + 2 * kGrp]) | (static_cast<uint32_t>(smem[off + 3 * kGrp]) << 8) |
        (static_cast<uint32_t>(smem[off + 4 * kGrp]) << 16);
  r.p = off + kHeaderBytes * kGrp;
  return r;
}

// One decode step (table entry: bits 0..10 slot - c_s, 11..13 s, 20..31 f_s):
// x = f (x >> 12) + slot - c_s, then byte renormalisation by selects (one
// byte, or two for tables with a symbol of f < 16). Returns 4 s.
template <bool kTwo>
__device__ __forceinline__ uint32_t rans_step(RansLane &r, const uint32_t *lut, const uint8_t *smem) {
  const uint32_t e = lut[r.x & (kM - 1)];
  uint32_t x = (e >> 20) * (r.x >> kProbBits) + (e & 0x7FFu);
  const uint32_t b0 = smem[r.p];
  const uint32_t b1 = kTwo ? static_cast<uint32_t>(smem[r.p + kGrp]) : 0u;
  uint32_t p = r.p;
  const bool lo0 = x < kL;
  x = lo0 ? (x * 256u + b0) : x;
  p = lo0 ? p + kGrp : p;
  if constexpr (kTwo) {
    const bool lo1 = x < kL;
    x = lo1 ? (x * 256u + b1) : x;
    p = lo1 ? p + kGrp : p;
  }
  r.p = p;
  r.x = x;
  return (e >> 9) & 0x1Cu;
}

__device__ __forceinline__ float norm_of(const uint8_t *cb) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(cb[0] | (cb[kGrp] << 8))));
}


template <bool kTwoK, bool kTwoV>
__global__ void __launch_bounds__(kTileWarps * 32, 1) prefill_tiles_kernel(const PrefillArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const TilesSmem L = tiles_smem_layout(a.ck, a.cv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t *lut_k = reinterpret_cast<uint32_t *>(smem + L.lut_k);
  uint32_t *lut_v = reinterpret_cast<uint32_t *>(smem + L.lut_v);
  uint32_t *lev = reinterpret_cast<uint32_t *>(smem + L.lev);
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
      lev[threadIdx.x] = a.tabs->k.score16[threadIdx.x];
      lev[kMaxLevels + threadIdx.x] = a.tabs->v.level16[threadIdx.x];
    }
  }
  __syncthreads();

  const int ck = a.ck, cv = a.cv;
  const int64_t gslots = (a.T_cap + kBlk - 1) / kBlk;  // slots per (b, h)
  constexpr int kQuarters = kBlk / kGrp;
  // Work unit u = ((row - bh0) gslots + slot) * 4 + quarter, row = b Hkv + h
  // of this wave: one 32-token group of one slot.
  const int64_t total = a.nbh * gslots * kQuarters;  // this wave's units
  const int64_t W = static_cast<int64_t>(gridDim.x) * kTileWarps;
  uint8_t *stg = smem + L.stage + static_cast<size_t>(warp) * L.stage_bytes;
  auto kslot = [&](int s) { return stg + s * L.kslot; };
  auto vslot = [&](int s) { return stg + 2 * L.kslot + s * L.vslot; };
  unsigned bad = 0, bad_pages = 0;
#ifdef DQ_CHECKED
  unsigned over = 0;  // containers decoded past their C bytes
#endif
  auto last_of = [&](int64_t u) -> int64_t {
    return last_position(a.q_start[(a.bh0 + u / (gslots * kQuarters)) / a.Hkv], a.n_q, a.T_cap);
  };
  // Next unit >= u (in steps of W) inside a slot the chunk attends to.
  auto next_valid = [&](int64_t u) -> int64_t {
    for (; u < total; u += W) {
      const int64_t hi = last_of(u);
      if (hi >= 0 && (u / kQuarters) % gslots <= hi / kBlk) return u;
    }
    return total;
  };
  // Cache block (32 tokens) of group j of the unit's (b, h).
  auto block_of = [&](int64_t u, int64_t j) -> int64_t {
    const int64_t bh = a.bh0 + u / (gslots * kQuarters);
    if (a.page_table) {
      int64_t pg = a.page_table[(bh / a.Hkv) * a.max_pages + j];
      if (pg < 0 || pg >= a.num_pages) {
        ++bad_pages;
        pg = 0;
      }
      return pg * a.Hkv + bh % a.Hkv;
    }
    return bh * (a.T_cap / kGrp) + j;
  };
  auto group_of = [&](int64_t u) -> int64_t { return ((u / kQuarters) % gslots) * kQuarters + u % kQuarters; };
  // Units whose group holds an attended token are decoded; the others (past
  // the last attended position, possibly past the cache) are zero-filled.
  auto decoded = [&](int64_t u) { return group_of(u) * kGrp <= last_of(u); };
  auto stage = [&](int sl, int64_t u) {
    const int64_t blk = block_of(u, group_of(u));
    const uint8_t *ks = a.kcache + blk * kGrp * ck;
    const uint8_t *vs = a.vcache + blk * kGrp * cv;
    for (int c = lane; c < (kGrp * ck) >> 4; c += 32) cp_async16(kslot(sl) + c * 16, ks + c * 16);
    for (int c = lane; c < (kGrp * cv) >> 4; c += 32) cp_async16(vslot(sl) + c * 16, vs + c * 16);
  };

  int64_t u = next_valid(static_cast<int64_t>(blockIdx.x) * kTileWarps + warp);
  if (u < total && decoded(u)) stage(0, u);
  cp_async_commit();
  for (int k = 0; u < total; ++k) {
    const int sl = k & 1;
    const int64_t u_next = next_valid(u + W);
    if (u_next < total && decoded(u_next)) stage(sl ^ 1, u_next);
    cp_async_commit();
    cp_async_wait_1();
    __syncwarp();
    const int q4 = static_cast<int>(u % kQuarters);
    uint8_t *dst = a.tiles + (u / kQuarters) * static_cast<int64_t>(kSlotBytes);
    float *nrm = reinterpret_cast<float *>(dst + 2 * kTileBytes);
    const int tl = q4 * kGrp + lane;  // token within the slot
    if (decoded(u)) {
      const uint8_t *kb = kslot(sl) + lane;
      const uint8_t *vb = vslot(sl) + lane;
      RansLane rk = rans_open(smem, static_cast<uint32_t>(kb - smem));
      RansLane rv = rans_open(smem, static_cast<uint32_t>(vb - smem));
#pragma unroll 1
      for (int i8 = 0; i8 < kD; i8 += 8) {
        uint32_t hk[8], hv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t ek = rans_step<kTwoK>(rk, lut_k, smem);
          const uint32_t ev = rans_step<kTwoV>(rv, lut_v, smem);
          hk[e] = *reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint8_t *>(lev) + ek);
          hv[e] = *reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint8_t *>(lev) + 4 * kMaxLevels + ev);
        }
        // 8 coordinates of this lane's token: 16 bytes in chunk i8 / 8.
        const size_t off = static_cast<size_t>((i8 >> 3) * kChunkStride + tl * 16);
        *reinterpret_cast<uint4 *>(dst + off) =
            make_uint4(__byte_perm(hk[0], hk[1], 0x5410), __byte_perm(hk[2], hk[3], 0x5410),
                       __byte_perm(hk[4], hk[5], 0x5410), __byte_perm(hk[6], hk[7], 0x5410));
        *reinterpret_cast<uint4 *>(dst + kTileBytes + off) =
            make_uint4(__byte_perm(hv[0], hv[1], 0x5410), __byte_perm(hv[2], hv[3], 0x5410),
                       __byte_perm(hv[4], hv[5], 0x5410), __byte_perm(hv[6], hv[7], 0x5410));
      }
      const int64_t hi = last_of(u);
      const int64_t tok = group_of(u) * kGrp + lane;
      // Tokens past the last attended position keep zero norms: their bytes
      // may be anything, and the softmax multiplies the weights by them.
      nrm[tl] = tok <= hi ? norm_of(kb) : 0.0f;
      const float nvt = tok <= hi ? norm_of(vb) : 0.0f;
      nrm[kBlk + tl] = nvt;
      // The quarter's largest V norm (bounds the softmax weights of a block).
      const float qm = warp_max(nvt);
      if (lane == 0) reinterpret_cast<float *>(dst + kQmaxOff)[q4] = qm;
      if (tok <= hi) bad += (rk.x != kL) + (rv.x != kL);
#ifdef DQ_CHECKED
      // The cursor starts at byte 5 and moves 32 per byte consumed.
      if (tok <= hi)
        over += (rk.p > static_cast<uint32_t>(kb - smem) + static_cast<uint32_t>(ck) * kGrp) +
                (rv.p > static_cast<uint32_t>(vb - smem) + static_cast<uint32_t>(cv) * kGrp);
#endif
    } else {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
      for (int c = 0; c < kD / 8; ++c) {
        *reinterpret_cast<uint4 *>(dst + c * kChunkStride + tl * 16) = z;
        *reinterpret_cast<uint4 *>(dst + kTileBytes + c * kChunkStride + tl * 16) = z;
      }
      nrm[tl] = 0.0f;
      nrm[kBlk + tl] = 0.0f;
      if (lane == 0) reinterpret_cast<float *>(dst + kQmaxOff)[q4] = 0.0f;
    }
    __syncwarp();  // the staging slot is refilled next iteration
    u = u_next;
  }
  cp_async_wait_0();
  if (a.stats) {
#ifdef DQ_CHECKED
    const unsigned o_w = __reduce_add_sync(kFull, over);
    if (lane == 0 && o_w) atomicAdd(&a.stats->overreads, static_cast<unsigned long long>(o_w));
#endif
    const unsigned b_w = __reduce_add_sync(kFull, bad);
    const unsigned p_w = __reduce_add_sync(kFull, bad_pages);
    if (lane == 0 && b_w) atomicAdd(&a.stats->integrity_errors, static_cast<unsigned long long>(b_w));
    if (lane == 0 && p_w) atomicAdd(&a.stats->bad_pages, static_cast<unsigned long long>(p_w));
  }
}

// Barrier of the kQuads softmax warps that share a row group (ids 1..4).
__device__ __forceinline__ void quad_sync(int id) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(32 * kQuads) : "memory");
}

// Stages h = 1, 2, 4, 8, 16 of the unnormalised Walsh-Hadamard transform on
// 32 consecutive coordinates held in registers (butterfly (a, b) -> (a + b,
// a - b), stages in that order).
__device__ __forceinline__ void wht32_regs(float (&v)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1)
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if ((i & h) == 0) {
        const float a0 = v[i], a1 = v[i + h];
        v[i] = __fadd_rn(a0, a1);
        v[i + h] = __fsub_rn(a0, a1);
      }
}

// Stages h = 32 and 64 on the four coordinates i, i + 32, i + 64, i + 96
// (z[m] is coordinate i + 32 m).
__device__ __forceinline__ void wht_4(float (&z)[4]) {
  const float a0 = __fadd_rn(z[0], z[1]), a1 = __fsub_rn(z[0], z[1]);
  const float a2 = __fadd_rn(z[2], z[3]), a3 = __fsub_rn(z[2], z[3]);
  z[0] = __fadd_rn(a0, a2);
  z[2] = __fsub_rn(a0, a2);
  z[1] = __fadd_rn(a1, a3);
  z[3] = __fsub_rn(a1, a3);
}

__global__ void __launch_bounds__(kAttnThreads, 1) prefill_kernel(const PrefillArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int ns = kMaxSlots;  // the host checks a.nslots against it
  const AttnSmem L = attn_smem_layout(ns);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + L.misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 4);
  float *pmax = reinterpret_cast<float *>(smem + L.pmax);  // [2][kQuads][128]
  float *lsum = reinterpret_cast<float *>(smem + L.lsum);  // [kQuads][128]
  int *pgo = reinterpret_cast<int *>(smem + L.pgo);        // [2][kQuads][128]: the warp's waits succeeded
  auto slot_base = [&](int d) { return smem + L.ring + static_cast<size_t>(d) * kSlotBytes; };

  // Work item: the query blocks of one (b, h) are consecutive, latest first.
  const int G = a.G, Mt = kRows / G;
  const int nqb = (a.n_q + Mt - 1) / Mt;
  const int64_t bid = blockIdx.x;
  const int64_t bh = a.bh0 + bid / nqb;
  const int qb = nqb - 1 - static_cast<int>(bid % nqb);
  const int b = static_cast<int>(bh / a.Hkv), h = static_cast<int>(bh % a.Hkv);
  const int64_t qs = a.q_start[b];
  const int i_lo = qb * Mt;
  const int i_hi = min(i_lo + Mt, a.n_q) - 1;
  const int64_t lo_pos = max(qs + i_lo, int64_t(0));
  const int64_t hi_pos = min(qs + i_hi, a.T_cap - 1);
  const int nB = lo_pos <= hi_pos ? static_cast<int>(hi_pos / kBlk) + 1 : 0;  // 128-token blocks to attend
  const int64_t gslots = (a.T_cap + kBlk - 1) / kBlk;

  // A softmax thread's query row (thread = row r of the block). Its loads
  // start before the set-up barrier, so that their latency overlaps the
  // tensor-memory allocation and the barrier initialisation.
  const int qt = warp >> 2;  // token quarter of a softmax warp
  const int r = (warp & 3) * 32 + lane;
  const int ti = i_lo + r / G, g = r % G;
  const bool in_chunk = warp < kSoftWarps && ti <= i_hi;
  const int64_t qbase = ((static_cast<int64_t>(b) * a.n_q + (in_chunk ? ti : 0)) * a.Hq + h * G + g) * kD;
  float qrow[32];
  if (in_chunk) {
    load_row32(a.q, qbase + 32 * qt, a.q_dtype, (reinterpret_cast<uintptr_t>(a.q) & 15u) == 0, qrow);
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) qrow[c] = 0.0f;
  }

  // ---- set-up ----
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tslot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    for (int d = 0; d < ns; ++d) {
      mbar_init(bars + kBarFull + d, 1);
      mbar_init(bars + kBarEmpty + d, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars + kBarSFull + i, 1);
      mbar_init(bars + kBarWFull + i, 32 * kSoftWarps);
      mbar_init(bars + kBarPvDone + i, 1);
    }
    mbar_init(bars + kBarQFull, kRows * kQuads);
    mbar_init(bars + kBarDrain, 1);
    mbar_init(bars + kBarDrainPv, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  unsigned timeouts = 0, clamped = 0;

  if (warp < kSoftWarps) {
    // ===== softmax: warps w, w + 4, w + 8, w + 12 own rows r = 32 (w % 4) +
    // lane; warp w + 4 q takes tokens 32 q .. 32 q + 31 of each block =====
    const uint32_t tl = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);  // this warp's lanes
    const int64_t pos = qs + ti;
    const bool row_ok = in_chunk && pos >= 0 && pos < a.T_cap;
    if (qt == 0 && in_chunk && !row_ok) ++clamped;
    const int quad_id = 1 + (warp & 3);
    // D1: q~ = H D q (unnormalised), times 2^e so that max |q~| is in [2^13,
    // 2^14). The four threads of a row share the work: thread qt rotates
    // coordinates 32 qt .. 32 qt + 31 through stages h = 1 .. 16 in
    // registers, passes them through tensor-memory columns (the score area,
    // unused before the first MMA) and finishes stages h = 32, 64 on the
    // coordinates i + 32 m, i in [8 qt, 8 qt + 8).
    float crow = 0.0f;
    {
      uint32_t sw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) sw[k] = __ldg(a.sign_bits + h * 4 + k);
      float v[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] = ((sw[qt] >> c) & 1u) ? -qrow[c] : qrow[c];
      wht32_regs(v);
      {
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 32; c += 16) {
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(v[c + e]);
          tmem_st16(tl + kColS + 32 * qt + c, w);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      quad_sync(quad_id);
      tc_fence_after();
      float z[4][8];
#pragma unroll
      for (int m = 0; m < 4; ++m) tmem_ld8(tl + kColS + 32 * m + 8 * qt, z[m]);
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float zz[4] = {z[0][i], z[1][i], z[2][i], z[3][i]};
        wht_4(zz);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          z[m][i] = zz[m];
          amax = fmaxf(amax, fabsf(zz[m]));
        }
      }
      pmax[qt * kRows + r] = amax;
      quad_sync(quad_id);
#pragma unroll
      for (int q2 = 0; q2 < kQuads; ++q2) amax = fmaxf(amax, pmax[q2 * kRows + r]);
      float sc = 1.0f;
      if (amax > 0.0f && amax < INFINITY) {
        int ex;
        frexpf(amax, &ex);
        sc = ldexpf(1.0f, 14 - ex);
      }
      // logit (log2 units) = S * ||k|| * crow, with S = sum (q~ sc)(kappa_K y)
      crow = row_ok ? a.sm_scale * kLog2e / (static_cast<float>(kD) * sc * a.tabs->k.score_scale) : 0.0f;
      // Coordinates 32 m + 8 qt + 2 p, + 1 are packed fp16 column 16 m + 4 qt + p.
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int p2 = 0; p2 < 4; ++p2) split_pair(z[m][2 * p2] * sc, z[m][2 * p2 + 1] * sc, hi[p2], lo[p2]);
        tmem_st4(tl + kColQh + 16 * m + 4 * qt, hi);
        tmem_st4(tl + kColQl + 16 * m + 4 * qt, lo);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars + kBarQFull);
      quad_sync(quad_id);  // pmax is reused below; the score columns are the MMA's from here on
    }

    float m_run = -INFINITY, l_run = 0.0f;
    bool alive = true;
    for (int j = 0; j < nB; ++j) {
      const int sb = static_cast<int>(j & 1);
      const int rb = static_cast<int>(j % ns);
      bool ok = alive && mbar_wait(bars + kBarSFull + sb, static_cast<uint32_t>((j >> 1) & 1), abort_flag) &&
                mbar_wait(bars + kBarFull + rb, static_cast<uint32_t>((j / ns) & 1), abort_flag);
      ok = __all_sync(kFull, ok);
      const uint32_t scol = tl + kColS + 128 * sb + 32 * qt;  // this warp's 32 score columns
      const float *nv = reinterpret_cast<const float *>(slot_base(rb) + 2 * kTileBytes) + kBlk + 32 * qt;
      float u[32];
      float mu0 = -INFINITY, vmax = 0.0f;
      if (ok) {
        tc_fence_after();
        tmem_ld32(scol, u);
        const float *nk = reinterpret_cast<const float *>(slot_base(rb) + 2 * kTileBytes) + 32 * qt;
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          const float4 n4 = *reinterpret_cast<const float4 *>(nk + t);
          const float2 a0 = __fmul2_rn(make_float2(u[t], u[t + 1]), make_float2(n4.x, n4.y));
          const float2 a1 = __fmul2_rn(make_float2(u[t + 2], u[t + 3]), make_float2(n4.z, n4.w));
          u[t] = a0.x;
          u[t + 1] = a0.y;
          u[t + 2] = a1.x;
          u[t + 3] = a1.y;
        }
        // u = S ||k|| (the logit divided by crow > 0); tokens past this row's
        // position are masked, which only happens on the causal diagonal.
        const int64_t rel = pos - static_cast<int64_t>(j) * kBlk - 32 * qt;
        const int lim = (!row_ok || rel < 0) ? -1 : (rel > 31 ? 31 : static_cast<int>(rel));
        if (!__all_sync(kFull, lim >= 31)) {
#pragma unroll
          for (int t = 0; t < 32; ++t) u[t] = t <= lim ? u[t] : -INFINITY;
        }
        mu0 = max32(u);
        // Largest V norm of the block's tokens (bounds the weights below),
        // from the slot's four quarter maxima.
        const float4 qv = *reinterpret_cast<const float4 *>(slot_base(rb) + kQmaxOff);
        vmax = fmaxf(fmax3(qv.x, qv.y, qv.z), qv.w);
      }
      // One exchange per block among the four warps of the row: the row
      // maximum and whether each warp could go on (its waits succeeded).
      // The four leave the loop together when one cannot.
      pmax[(sb * kQuads + qt) * kRows + r] = mu0;
      pgo[(sb * kQuads + qt) * kRows + r] = ok ? 1 : 0;
      quad_sync(quad_id);
      bool go = true;
      float mrow = -INFINITY;
#pragma unroll
      for (int q2 = 0; q2 < kQuads; ++q2) {
        go = go && pgo[(sb * kQuads + q2) * kRows + r] != 0;
        mrow = fmaxf(mrow, pmax[(sb * kQuads + q2) * kRows + r]);
      }
      if (!go) {
        if (alive) ++timeouts;
        alive = false;
        break;
      }
      const float mcand = mrow == -INFINITY ? m_run : fmaxf(m_run, mrow * crow);
      // Lazy rescaling: the running maximum stays while the block's is at most
      // kLazyLog2 above it and the weights p ||v|| <= 2^(mcand - m_run) vmax
      // stay within half the fp16 range; O, l and the weights all use the
      // same maximum, so the result is the same. The four quarters of a row
      // decide alike (same inputs).
      const float mx = (m_run != -INFINITY && mcand - m_run <= kLazyLog2 && ex2(mcand - m_run) * vmax <= 32768.0f)
                           ? m_run
                           : mcand;
      float alpha = 1.0f;
      if (mx != -INFINITY && m_run != -INFINITY && mx != m_run) alpha = ex2(m_run - mx);
      // Rescaling O needs P.V of the previous block done; W goes over this
      // block's own score columns and needs nothing more. (The P.V-done
      // barrier of block j - 1 cannot run a phase further before this warp
      // writes W of block j + 1, so the parity wait is unambiguous.)
      const bool resc = j > 0 && __any_sync(kFull, alpha != 1.0f);
      ok = !resc ||
           mbar_wait(bars + kBarPvDone + ((j - 1) & 1), static_cast<uint32_t>(((j - 1) >> 1) & 1), abort_flag);
      ok = __all_sync(kFull, ok);
      float psum = 0.0f;
      if (ok) {
        tc_fence_after();
        if (resc) {
          // This warp rescales O's coordinate columns 32 qt .. 32 qt + 31.
          float o[32];
          const uint32_t oc = tl + kColO + 32 * qt;
          tmem_ld32(oc, o);
          uint32_t w0[16], w1[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            w0[e] = __float_as_uint(o[e] * alpha);
            w1[e] = __float_as_uint(o[16 + e] * alpha);
          }
          tmem_st16(oc, w0);
          tmem_st16(oc + 16, w1);
        }
        // W in place of this warp's own score columns (the scores were read
        // above), 16 tokens at a time: p = 2^(logit - mx), w = p ||v|| as fp16
        // hi (columns 0..15) and lo (16..31); norms of tokens past the last
        // attended position are 0, so masked tokens give exactly 0.
        if (__all_sync(kFull, mx != -INFINITY)) {
          // Packed pairs: x = u crow - mx, p = 2^x, w = p ||v||.
          const float2 c2 = make_float2(crow, crow), m2 = make_float2(-mx, -mx);
          float2 ps2 = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t wh[8], wl[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
              const int t = 16 * c + 2 * p;
              const float2 x = __ffma2_rn(make_float2(u[t], u[t + 1]), c2, m2);
              const float2 pp = make_float2(ex2(x.x), ex2(x.y));
              ps2 = __fadd2_rn(ps2, pp);
              const float2 nn = *reinterpret_cast<const float2 *>(nv + t);
              split_pair_trunc(__fmul2_rn(pp, nn), wh[p], wl[p]);
            }
            tmem_st8(scol + 8 * c, wh);
            tmem_st8(scol + 16 + 8 * c, wl);
          }
          psum = ps2.x + ps2.y;
        } else {
          float ps[2] = {0.0f, 0.0f};
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t wh[8], wl[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
              const int t = 16 * c + 2 * p;
              float p0 = 0.0f, p1 = 0.0f;
              if (mx != -INFINITY) {
                p0 = ex2(fmaf(u[t], crow, -mx));
                p1 = ex2(fmaf(u[t + 1], crow, -mx));
              }
              ps[p & 1] += p0 + p1;
              split_pair(p0 * nv[t], p1 * nv[t + 1], wh[p], wl[p]);
            }
            tmem_st8(scol + 8 * c, wh);
            tmem_st8(scol + 16 + 8 * c, wl);
          }
          psum = ps[0] + ps[1];
        }
        tmem_wait_st();
      } else {
        ++timeouts;
        alive = false;  // the whole row stops at the next agreement
      }
      if (mx != -INFINITY) m_run = mx;
      l_run = l_run * alpha + psum;
      tc_fence_before();
      mbar_arrive(bars + kBarWFull + sb);  // always, so the MMA warp's count completes
    }
    // D7: o = D H o_rot / 128 with o_rot = O / (l kappa_V); l sums the four
    // quarters. Thread qt takes O's coordinates 32 qt .. 32 qt + 31 through
    // stages h = 1 .. 16, passes them through the (now idle) score columns
    // and finishes stages h = 32, 64 on coordinates i + 32 m, i in [8 qt,
    // 8 qt + 8).
    lsum[qt * kRows + r] = l_run;
    quad_sync(quad_id);
    float l_all = 0.0f;
#pragma unroll
    for (int q2 = 0; q2 < kQuads; ++q2) l_all += lsum[q2 * kRows + r];
    bool have_o = alive && nB > 0;
    if (have_o) {
      const int jl = nB - 1;
      const bool okw = mbar_wait(bars + kBarPvDone + (jl & 1), static_cast<uint32_t>((jl >> 1) & 1), abort_flag);
      if (!__all_sync(kFull, okw)) {
        ++timeouts;
        have_o = false;
      }
    }
    // The row's four threads must agree (they exchange columns below).
    pmax[qt * kRows + r] = have_o ? 0.0f : 1.0f;
    quad_sync(quad_id);
#pragma unroll
    for (int q2 = 0; q2 < kQuads; ++q2) have_o = have_o && pmax[q2 * kRows + r] == 0.0f;
    const float inv =
        (have_o && row_ok && l_all > 0.0f) ? 1.0f / (l_all * static_cast<float>(kD) * a.tabs->v.tile_scale) : 0.0f;
    // have_o is the same for the four warps of the row group (their
    // agreement above), so they meet at the barrier below together. Without
    // O (no block, or a wait that gave up) the output is zero and tensor
    // memory is left alone.
    float z[4][8];
    if (have_o) {
      float v[32];
      tc_fence_after();
      tmem_ld32(tl + kColO + 32 * qt, v);
#pragma unroll
      for (int c = 0; c < 32; ++c) v[c] *= inv;
      wht32_regs(v);
      uint32_t w[16];
#pragma unroll
      for (int c = 0; c < 32; c += 16) {
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(v[c + e]);
        tmem_st16(tl + kColS + 32 * qt + c, w);
      }
      tmem_wait_st();
      tc_fence_before();
      quad_sync(quad_id);
      tc_fence_after();
#pragma unroll
      for (int m = 0; m < 4; ++m) tmem_ld8(tl + kColS + 32 * m + 8 * qt, z[m]);
      uint32_t sw[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) sw[k] = __ldg(a.sign_bits + h * 4 + k);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float zz[4] = {z[0][i], z[1][i], z[2][i], z[3][i]};
        wht_4(zz);
#pragma unroll
        for (int m = 0; m < 4; ++m) z[m][i] = ((sw[m] >> (8 * qt + i)) & 1u) ? -zz[m] : zz[m];
      }
    } else {
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int i = 0; i < 8; ++i) z[m][i] = 0.0f;
    }
    const bool vec = (reinterpret_cast<uintptr_t>(a.out) & 15u) == 0;
    if (have_o && vec) {
      // Through shared memory, so that a store instruction writes one whole
      // output row (a warp's 32 lanes would otherwise write 32 rows). The
      // ring is idle: every block's copies have landed and its MMAs are done
      // (P.V of the last block, waited above). Rows 32 (w % 4) .. + 31 of
      // the quad, 132 floats apart (no bank conflicts).
      float *stg = reinterpret_cast<float *>(slot_base(0));
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float4 *p4 = reinterpret_cast<float4 *>(stg + r * 132 + 32 * m + 8 * qt);
        p4[0] = make_float4(z[m][0], z[m][1], z[m][2], z[m][3]);
        p4[1] = make_float4(z[m][4], z[m][5], z[m][6], z[m][7]);
      }
      quad_sync(quad_id);
      // Warp qt of the quad stores rows 8 qt .. 8 qt + 7 of the quad's 32.
#pragma unroll 2
      for (int k = 0; k < 8; ++k) {
        const int rr = (warp & 3) * 32 + 8 * qt + k;
        const int ti2 = i_lo + rr / G;
        if (ti2 > i_hi) continue;  // past the chunk (same for the whole warp)
        const int64_t base2 = ((static_cast<int64_t>(b) * a.n_q + ti2) * a.Hq + h * G + rr % G) * kD;
        const float4 val = reinterpret_cast<const float4 *>(stg + rr * 132)[lane];
        if (a.out_dtype == DQ_BF16) {
          const __nv_bfloat162 h0 = __floats2bfloat162_rn(val.x, val.y), h1 = __floats2bfloat162_rn(val.z, val.w);
          reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.out) + base2)[lane] =
              make_uint2(*reinterpret_cast<const uint32_t *>(&h0), *reinterpret_cast<const uint32_t *>(&h1));
        } else {
          reinterpret_cast<float4 *>(static_cast<float *>(a.out) + base2)[lane] = val;
        }
      }
    } else if (in_chunk) {
#pragma unroll
      for (int m = 0; m < 4; ++m) store_row8(a.out, qbase + 32 * m + 8 * qt, z[m], a.out_dtype, vec);
    }
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    // ===== MMA issue (one lane of each of two warps) =====
    // Warp kMmaWarp issues the score MMAs, warp kPvWarp the P.V MMAs: two
    // issuing threads on two schedulers. Each commits only its own MMAs;
    // the order between the two streams comes from the barriers (S_j is
    // written only after P.V of block j - 2 is done with its buffer; P.V of
    // block j reads W_j, written after S_j was complete).
    auto drain = [&](int bar) {
      tc_commit(bars + bar);
      const uint32_t da = smem_u32(bars + bar);
      for (uint32_t it = 0; it < kSpin; ++it) {
        uint32_t done;
        asm volatile(
            "{\n.reg .pred P;\nmbarrier.try_wait.parity.shared::cta.b64 P, [%1], 0;\nselp.u32 %0, 1, 0, P;\n}\n"
            : "=r"(done)
            : "r"(da)
            : "memory");
        if (done) break;
      }
    };
    if (warp == kMmaWarp && nB > 0) {
      const uint32_t idS = instr_desc(kRows, kBlk, 0);
      bool alive = __all_sync(kFull, mbar_wait(bars + kBarQFull, 0, abort_flag));
      if (!alive && lane == 0) ++timeouts;
      tc_fence_after();
      for (int j = 0; j < nB && alive; ++j) {
        const int rb = static_cast<int>(j % ns);
        alive = __all_sync(kFull, mbar_wait(bars + kBarFull + rb, static_cast<uint32_t>((j / ns) & 1), abort_flag));
        // The score buffer j & 1 held W of block j - 2: wait until its P.V is done.
        if (alive && j >= 2)
          alive = __all_sync(kFull, mbar_wait(bars + kBarPvDone + (j & 1), static_cast<uint32_t>(((j - 2) >> 1) & 1), abort_flag));
        if (!alive) {
          if (lane == 0) ++timeouts;
          break;
        }
        tc_fence_after();
        // S_j = q~ K_j^T: B = K tile, K-major: token groups of 8 at 128 bytes
        // (SBO), coordinate chunks of 8 at kChunkStride bytes (LBO).
        const uint32_t kt = smem_u32(slot_base(rb));
        const uint32_t sd = tbase + kColS + 128 * static_cast<uint32_t>(j & 1);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t bd = smem_desc(kt + ks * 2 * kChunkStride, kChunkStride, 128);
          mma_ts(sd, tbase + kColQh + ks * 8, bd, idS, ks > 0 ? 1u : 0u);
          mma_ts(sd, tbase + kColQl + ks * 8, bd, idS, 1u);
        }
        tc_commit(bars + kBarSFull + (j & 1));
      }
      // Every MMA issued above has completed before tensor memory is freed.
      drain(kBarDrain);
    } else if (warp == kPvWarp && nB > 0) {
      const uint32_t idO = instr_desc(kRows, kD, 1);
      for (int jj = 0; jj < nB; ++jj) {
        if (!__all_sync(kFull, mbar_wait(bars + kBarWFull + (jj & 1), static_cast<uint32_t>((jj >> 1) & 1), abort_flag))) {
          if (lane == 0) ++timeouts;
          break;
        }
        tc_fence_after();
        // O += W_jj V_jj: A = W (tensor memory; tokens 16 ks .. 16 ks + 15 of
        // the hi or lo half), B = V tile, MN-major: token groups of 8 at 128
        // bytes (LBO), coordinate chunks of 8 at kChunkStride bytes (SBO).
        const uint32_t vt = smem_u32(slot_base(static_cast<int>(jj % ns)) + kTileBytes);
        const uint32_t wb = tbase + kColS + 128 * static_cast<uint32_t>(jj & 1);
#pragma unroll
        for (int ks = 0; ks < kBlk / 16; ++ks) {
          const uint64_t bd = smem_desc(vt + ks * 256, 128, kChunkStride);
          // Tokens 16 ks .. 16 ks + 15 are in quarter ks / 2: fp16 hi pairs at
          // its columns 8 (ks % 2) .., lo pairs 16 columns further.
          const uint32_t wc = wb + 32 * static_cast<uint32_t>(ks >> 1) + (ks & 1) * 8;
          mma_ts(tbase + kColO, wc, bd, idO, (jj > 0 || ks > 0) ? 1u : 0u);
          mma_ts(tbase + kColO, wc + 16, bd, idO, 1u);
        }
        tc_commit(bars + kBarPvDone + (jj & 1));
        // The slot is free once P.V is done: its score MMA completed before
        // W_jj could be written.
        tc_commit(bars + kBarEmpty + static_cast<int>(jj % ns));
      }
      drain(kBarDrainPv);
    }
  } else if (warp == kLoadWarp) {
    // ===== slot loader (one lane) =====
    if (lane == 0 && nB > 0) {
      const uint8_t *src = a.tiles + static_cast<size_t>((bh - a.bh0) * gslots) * kSlotBytes;
      int issued = 0;
      for (int j = 0; j < nB; ++j) {
        const int sl = static_cast<int>(j % ns);
        if (j >= ns && !mbar_wait(bars + kBarEmpty + sl, static_cast<uint32_t>(((j / ns) - 1) & 1), abort_flag)) {
          ++timeouts;
          break;
        }
        mbar_arrive_expect_tx(bars + kBarFull + sl, kSlotBytes);
        bulk_g2s(slot_base(sl), src + static_cast<size_t>(j) * kSlotBytes, kSlotBytes, bars + kBarFull + sl);
        ++issued;
      }
      // Drain: the last copies into each slot have landed before the CTA
      // exits (bounded, whatever the abort flag says).
      for (int j = issued > ns ? issued - ns : 0; j < issued; ++j) {
        const uint32_t fa = smem_u32(bars + kBarFull + static_cast<int>(j % ns));
        const uint32_t par = static_cast<uint32_t>((j / ns) & 1);
        for (uint32_t it = 0; it < kSpin; ++it) {
          uint32_t done;
          asm volatile(
              "{\n.reg .pred P;\nmbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\nselp.u32 %0, 1, 0, P;\n}\n"
              : "=r"(done)
              : "r"(fa), "r"(par)
              : "memory");
          if (done) break;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tbase), "r"(kTmemCols) : "memory");
  }
  if (a.stats) {
    const unsigned t_w = __reduce_add_sync(kFull, timeouts);
    const unsigned c_w = __reduce_add_sync(kFull, clamped);
    if (lane == 0) {
      if (t_w) atomicAdd(&a.stats->wait_timeouts, static_cast<unsigned long long>(t_w));
      if (c_w) atomicAdd(&a.stats->clamped_lengths, static_cast<unsigned long long>(c_w));
    }
  }
}

template <bool kTwoK, bool kTwoV>
int launch_tiles_t(const PrefillArgs &a, cudaStream_t st) {
  const TilesSmem L = tiles_smem_layout(a.ck, a.cv);
  constexpr auto kern = prefill_tiles_kernel<kTwoK, kTwoV>;
  const cudaError_t e = ensure_max_dynamic_smem<kern>(static_cast<int>(L.total));
  if (e != cudaSuccess) return static_cast<int>(e);
  kern<<<a.tile_grid, kTileWarps * 32, L.total, st>>>(a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int prefill_ring_slots() {
  int ns = kMaxSlots;
  while (ns > 2 && attn_smem_layout(ns).total > 227 * 1024) --ns;
  return ns;
}

int64_t prefill_grid(int64_t nbh, int G, int n_q) {
  const int Mt = kRows / G;
  return nbh * ((n_q + Mt - 1) / Mt);
}

size_t prefill_workspace_bytes(int B, int Hkv, int64_t T_cap) {
  return static_cast<size_t>(B) * Hkv * static_cast<size_t>((T_cap + kBlk - 1) / kBlk) * kSlotBytes;
}

bool prefill_supported(int ck, int cv) {
  return ck >= 1 && cv >= 1 && ck <= kMaxContainer && cv <= kMaxContainer &&
         tiles_smem_layout(ck, cv).total <= 227 * 1024;
}

int launch_prefill_attention(const PrefillArgs &a, void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a.nslots != kMaxSlots || a.tile_grid < 1 || (a.G != 1 && a.G != 2 && a.G != 4 && a.G != 8) ||
      a.T_cap / kBlk >= 0x7FFFFFFF)
    return static_cast<int>(cudaErrorInvalidValue);
  const int64_t grid = prefill_grid(a.nbh, a.G, a.n_q);
  if (grid < 1 || grid > 0x7FFFFFFF) return static_cast<int>(cudaErrorInvalidValue);
  int e;
  if (a.two_k && a.two_v) e = launch_tiles_t<true, true>(a, st);
  else if (a.two_k) e = launch_tiles_t<true, false>(a, st);
  else if (a.two_v) e = launch_tiles_t<false, true>(a, st);
  else e = launch_tiles_t<false, false>(a, st);
  if (e) return e;
  const AttnSmem L = attn_smem_layout(a.nslots);
  const cudaError_t ce = ensure_max_dynamic_smem<prefill_kernel>(static_cast<int>(L.total));
  if (ce != cudaSuccess) return static_cast<int>(ce);
  prefill_kernel<<<static_cast<unsigned>(grid), kAttnThreads, L.total, st>>>(a);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dqi
