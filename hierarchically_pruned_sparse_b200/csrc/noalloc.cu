// hip_sparse_attn_noalloc: block-sparse attention on scratch memory that the
// library owns, for callers that cannot allocate device memory (a frozen
// memory pool, or a decode step that must not meet a cudaMalloc). The paper
// has no counterpart to this entry point; the arithmetic is exactly that of
// hip_sparse_attn, only the split-K partials and the status block live in a
// fixed device array here instead of a caller workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "hip_sparse.h"
#include "hips_common.cuh"
#include "hips_kernels.h"

namespace {

constexpr size_t kScratchBytes = HIPS_NOALLOC_SCRATCH_BYTES;
constexpr size_t kStatusBytes = 4096;  // status word + split-merge counters
constexpr size_t kCounterOffset = 256;

// One copy per device that loads the library, alive until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[hips::kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the
// symbol itself is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int scratch_on_current_device(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hips::record_cuda_error(e);
  if (dev < 0 || dev >= hips::kMaxDevices) return HIPS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return hips::record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return HIPS_OK;
}

}  // namespace

extern "C" int hip_sparse_attn_noalloc(const void* q, const void* k, const void* v,
                                       const int32_t* idx, const hips_params* params, void* out) {
  hips::AttnArgs a;
  int smem = 0;
  size_t need = 0;
  bool tensor_core = false;
  int st = hips::plan_sparse_attn_own_scratch(q, k, v, idx, params, out, &a, &smem, &need,
                                              &tensor_core);
  if (st) return st;
  if (need > kScratchBytes) return HIPS_ERR_TOO_LARGE;
  void* base = nullptr;
  st = scratch_on_current_device(&base);
  if (st) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(params->stream);
  // the status word and the split-merge counters must start at zero; the
  // partials are fully overwritten
  cudaError_t e = cudaMemsetAsync(base, 0, kStatusBytes, stream);
  if (e != cudaSuccess) return hips::record_cuda_error(e);
  a.status = static_cast<hips::Status*>(base);
  a.counters = reinterpret_cast<unsigned int*>(static_cast<unsigned char*>(base) + kCounterOffset);
  a.part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kStatusBytes);
  return hips::record_cuda_error(tensor_core ? hips::launch_attn_mma(a, smem, stream)
                                             : hips::launch_attn_fma(a, smem, stream));
}
