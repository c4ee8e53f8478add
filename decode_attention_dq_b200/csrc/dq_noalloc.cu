// dq_noalloc.cu -- decode attention for callers that cannot allocate device
// memory.
//
// dq_decode_attention needs a caller-provided workspace for its split-K
// partial results. Some callers have no way to obtain one: a host application
// or plugin that is handed only input and output device pointers and has no
// access to an allocator, a serving loop that forbids any cudaMalloc after
// start-up (cudaMalloc can synchronise the device and competes with a caching
// allocator that owns the memory), or code running where the device allocator
// is not available at all. dq_decode_attention_noalloc serves them: it uses
// a fixed scratch array that lives in the library's own device memory and
// allocates nothing.
//
// The scratch array is a file-scope __device__ variable: every GPU that loads
// the library holds it (kScratchBytes) until the process exits, and every call
// on a device shares it. Host code cannot use the array's name as a device
// address (on the host it is only a stand-in symbol), so the device address
// is looked up with cudaGetSymbolAddress, with the device current, and cached
// per device together with the id of the CUDA context it belongs to. A new
// context on that device (after cudaDeviceReset, or once the primary context
// has been released and created again) loads the module afresh, possibly at
// another address; the id then differs and the address is looked up again,
// so a stale address is never handed to a kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "dq_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

struct ScratchEntry {
  unsigned long long ctx_id;
  void *ptr;
};

std::mutex g_scratch_mutex;
ScratchEntry g_scratch_entry[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Driver entry points for the current context and its id, resolved once
// through the runtime (the library does not link the driver directly).
bool driver_fns(CtxGetCurrentFn *get_current, CtxGetIdFn *get_id) {
  static CtxGetCurrentFn s_current = nullptr;
  static CtxGetIdFn s_id = nullptr;
  static bool s_tried = false;
  if (!s_tried) {
    s_tried = true;
    void *f0 = nullptr, *f1 = nullptr;
    cudaDriverEntryPointQueryResult q0 = cudaDriverEntryPointSymbolNotFound, q1 = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f0, 12000, cudaEnableDefault, &q0) == cudaSuccess &&
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &f1, 12000, cudaEnableDefault, &q1) == cudaSuccess &&
        q0 == cudaDriverEntryPointSuccess && q1 == cudaDriverEntryPointSuccess) {
      s_current = reinterpret_cast<CtxGetCurrentFn>(f0);
      s_id = reinterpret_cast<CtxGetIdFn>(f1);
    }
  }
  *get_current = s_current;
  *get_id = s_id;
  return s_current && s_id;
}

// Id of the context current on this thread; false if there is none yet.
bool current_ctx_id(CtxGetCurrentFn get_current, CtxGetIdFn get_id, unsigned long long *id) {
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || !c) return false;
  return get_id(c, id) == CUDA_SUCCESS;
}

// Device address of g_scratch in the current context of the current device:
// looked up on the first call per device (with that device current) and
// again whenever the device's context has changed since.
int scratch_address(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return DQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DQ_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
  if (!driver_fns(&get_current, &get_id)) return DQ_ERR_CUDA;
  ScratchEntry &ent = g_scratch_entry[dev];
  unsigned long long id = 0;
  if (ent.ptr && current_ctx_id(get_current, get_id, &id) && id == ent.ctx_id) {
    *out = ent.ptr;
    return DQ_OK;
  }
  void *p = nullptr;
  e = cudaGetSymbolAddress(&p, g_scratch);  // also makes the primary context current if needed
  if (e != cudaSuccess || !p) return DQ_ERR_CUDA;
  if (!current_ctx_id(get_current, get_id, &id)) return DQ_ERR_CUDA;
  ent.ptr = p;
  ent.ctx_id = id;
  *out = p;
  return DQ_OK;
}

}  // namespace

extern "C" int dq_decode_attention_noalloc(const dq_tables *t, const void *q, int q_dtype,
                                           const uint8_t *d_kcache, const uint8_t *d_vcache,
                                           const int32_t *d_seq_lens, int B, int Hq, int Hkv,
                                           int64_t T_cap, int64_t T_max, float sm_scale, void *out,
                                           int out_dtype, dq_stats *d_stats, void *stream) {
  try {
    if (!t) return DQ_ERR_NULL;
    // The partial results this call needs must fit the fixed scratch array.
    const size_t need = dq_decode_workspace_bytes(t, B, Hq, Hkv, T_max);
    if (need > kScratchBytes) return DQ_ERR_WORKSPACE;
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != DQ_OK) return rc;
    // Same kernels and checks as dq_decode_attention; only the workspace
    // comes from the library's scratch array. Every partial result is written
    // before it is read, so the stale contents of earlier calls never matter.
    return dq_decode_attention(t, q, q_dtype, d_kcache, d_vcache, d_seq_lens, B, Hq, Hkv, T_cap,
                               T_max, sm_scale, out, out_dtype, scratch, kScratchBytes, d_stats,
                               stream);
  } catch (...) {
    return DQ_ERR_CUDA;
  }
}
