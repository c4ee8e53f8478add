// dq_device.cuh -- device helpers shared by libdq's kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "dq_internal.h"

namespace dqi {

constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ float load_elem(const void *base, int64_t idx, int dtype) {
  if (dtype == DQ_BF16) {
    const uint16_t b = __ldg(static_cast<const uint16_t *>(base) + idx);
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
  return __ldg(static_cast<const float *>(base) + idx);
}

__device__ __forceinline__ void store_elem(void *base, int64_t idx, float v, int dtype) {
  if (dtype == DQ_BF16)
    static_cast<__nv_bfloat16 *>(base)[idx] = __float2bfloat16_rn(v);
  else
    static_cast<float *>(base)[idx] = v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// In-warp unnormalised Walsh-Hadamard transform of a 128-vector held as
// v[k] = z[lane + 32 k], stages h = 1, 2, ..., 64 in that order with the
// butterfly (a, b) -> (a + b, a - b). Each add/sub is one IEEE fp32 op, so the
// result is identical to the sequential definition.
__device__ __forceinline__ void wht128_warp(float (&v)[4], int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const bool upper = (lane & h) != 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float w = __shfl_xor_sync(kFull, v[k], h);
      v[k] = upper ? __fsub_rn(w, v[k]) : __fadd_rn(v[k], w);
    }
  }
  {  // h = 32: pairs (k=0,k=1), (k=2,k=3)
    const float a0 = v[0], a1 = v[1], a2 = v[2], a3 = v[3];
    v[0] = __fadd_rn(a0, a1);
    v[1] = __fsub_rn(a0, a1);
    v[2] = __fadd_rn(a2, a3);
    v[3] = __fsub_rn(a2, a3);
  }
  {  // h = 64: pairs (k=0,k=2), (k=1,k=3)
    const float a0 = v[0], a1 = v[1], a2 = v[2], a3 = v[3];
    v[0] = __fadd_rn(a0, a2);
    v[2] = __fsub_rn(a0, a2);
    v[1] = __fadd_rn(a1, a3);
    v[3] = __fsub_rn(a1, a3);
  }
}

// Raises kernel Kern's dynamic shared-memory limit to at least `bytes` on
// the current device. The attribute call is made only when a larger size is
// first needed on a device, so a launch sequence that repeats (a serving
// loop, one call per layer) pays the host-side attribute call once.
template <auto Kern>
cudaError_t ensure_max_dynamic_smem(int bytes) {
  constexpr int kDevs = 64;
  static std::atomic<int> set_to[kDevs];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < kDevs;
  if (cached && set_to[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cached) {
    int cur = set_to[dev].load(std::memory_order_relaxed);
    while (cur < bytes && !set_to[dev].compare_exchange_weak(cur, bytes, std::memory_order_release)) {
    }
  }
  return e;
}

// Sign of coordinate lane + 32 k for a KV head: bit `lane` of sign word k.
__device__ __forceinline__ float apply_sign(float v, uint32_t word, int lane) {
  return ((word >> lane) & 1u) ? -v : v;
}

}  // namespace dqi
