// dq_symbols.cu -- test hook: decode flat containers of one stream into
// symbols, norms and a per-container integrity status.
//
// rANS decode ([news] "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits",
// "Drift: Bending Variable Back to Fixed": symbols are rANS-coded into a
// fixed-size container). One lane decodes one container: slot = x mod 4096
// selects (symbol, frequency, slot - cumulative) from a shared-memory table,
// x = f (x >> 12) + slot - c, then bytes are shifted in while x < 2^16.
#include "dq_device.cuh"

namespace dqi {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32)
decode_symbols_kernel(const DevStream *__restrict__ tab, const uint8_t *__restrict__ cache,
                      int64_t n, int C, uint8_t *__restrict__ syms, uint16_t *__restrict__ norm16,
                      int32_t *__restrict__ status, dq_stats *__restrict__ stats) {
  __shared__ uint32_t lut[kM];
  __shared__ __align__(16) uint8_t stage[kWarps][32 * kMaxContainer + 16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < static_cast<int>(kM); i += blockDim.x) lut[i] = tab->lut[i];

  const int64_t first = (static_cast<int64_t>(blockIdx.x) * kWarps + warp) * 32;
  const int64_t cidx = first + lane;
  const bool valid = cidx < n;
  // Stage this warp's (contiguous) containers with 4-byte loads.
  const int64_t count = (n - first) < 32 ? (n - first) : 32;
  if (count > 0) {
    const int words = static_cast<int>((count * C + 3) / 4);
    const int64_t byte0 = first * C;
    // The byte range may end mid-word only at the very end of the array;
    // read the last partial word byte by byte.
    const int full_words = static_cast<int>((count * C) / 4);
    const uint32_t *src = reinterpret_cast<const uint32_t *>(cache + byte0);
    uint32_t *dst = reinterpret_cast<uint32_t *>(stage[warp]);
    for (int w = lane; w < full_words; w += 32) dst[w] = __ldg(src + w);
    if (lane == 0)
      for (int64_t b = static_cast<int64_t>(full_words) * 4; b < count * C; ++b)
        stage[warp][b] = cache[byte0 + b];
    (void)words;
  }
  __syncthreads();

  int st = 0;
  if (valid) {
    const uint8_t *cb = stage[warp] + lane * C;
    norm16[cidx] = static_cast<uint16_t>(cb[0] | (cb[1] << 8));
    uint32_t x = static_cast<uint32_t>(cb[2]) | (static_cast<uint32_t>(cb[3]) << 8) |
                 (static_cast<uint32_t>(cb[4]) << 16);
    int pos = kHeaderBytes;
    uint32_t *out = reinterpret_cast<uint32_t *>(syms + cidx * kD);
    if (x < kL) {
      st = 1;
      for (int w = 0; w < kD / 4; ++w) out[w] = 0u;
    } else {
      uint32_t pack = 0;
      int i = 0;
      for (; i < kD && st == 0; ++i) {
        const uint32_t e = lut[x & (kM - 1)];
        const uint32_t s = (e >> 11) & 7u;
        x = (e >> 20) * (x >> kProbBits) + (e & 0x7FFu);
        pack |= s << (8 * (i & 3));
        for (int r = 0; r < 2 && x < kL; ++r) {
          if (pos >= C) { st = 2; break; }
          x = (x << 8) | cb[pos++];
        }
        if ((i & 3) == 3 || st != 0) {
          out[i >> 2] = pack;
          pack = 0;
        }
      }
      for (int w = (i + 3) >> 2; w < kD / 4; ++w) out[w] = 0u;
      if (st == 0 && x != kL) st = 3;
      if (st == 0)
        for (int b = pos; b < C; ++b)
          if (cb[b] != 0) { st = 4; break; }
    }
    if (status) status[cidx] = st;
  }
  const unsigned bad = __ballot_sync(kFull, valid && st != 0);
  if (stats && lane == 0 && bad) atomicAdd(&stats->integrity_errors, static_cast<unsigned long long>(__popc(bad)));
}

}  // namespace

int launch_decode_symbols(const SymbolsArgs &a, void *stream) {
  if (a.c > kMaxContainer) return static_cast<int>(cudaErrorInvalidValue);
  const int64_t per_cta = kWarps * 32;
  const int64_t grid = (a.n + per_cta - 1) / per_cta;
  if (grid > 0x7FFFFFFF) return static_cast<int>(cudaErrorInvalidConfiguration);
  decode_symbols_kernel<<<static_cast<unsigned>(grid), kWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
      a.tab, a.cache, a.n, a.c, a.syms, a.norm16, a.status, a.stats);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dqi
