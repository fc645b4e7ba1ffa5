// hip_sparse_attn_noalloc: block-sparse attention on scratch memory that the
// library owns, for callers that cannot allocate device memory (a frozen
// memory pool, or a decode step that must not meet a cudaMalloc). The paper
// has no counterpart to this entry point; the arithmetic is exactly that of
// hip_sparse_attn, only the split-K partials and the status block live in a
// fixed device array here instead of a caller workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "hip_sparse.h"
#include "hips_common.cuh"
#include "hips_kernels.h"

namespace {

constexpr size_t kScratchBytes = HIPS_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes > hips::kStatusBytes, "room for the partials after the status block");

// One copy per device that loads the library, alive until the process exits.
// Its head follows the workspace layout of hips_kernels.h (status word,
// split-merge counters, then the partials).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// The current CUDA context, through the driver entry point the runtime
// hands out (the library does not link libcuda itself). Null if unavailable.
CUcontext current_context() {
  using GetCurrent = CUresult (*)(CUcontext*);
  static GetCurrent fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<GetCurrent>(p);
  }();
  CUcontext ctx = nullptr;
  if (fn && fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  return ctx;
}

struct ScratchEntry {
  CUcontext ctx;  // context the address belongs to
  void* addr;
};
std::mutex g_scratch_mutex;
ScratchEntry g_scratch[hips::kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code the
// symbol itself is only a host-side stand-in, so the address is looked up
// with the device current, once per device and context, and cached; after a
// device reset (a new primary context) the next call looks it up again.
int scratch_on_current_device(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hips::record_cuda_error(e);
  if (dev < 0 || dev >= hips::kMaxDevices) return HIPS_ERR_UNSUPPORTED;
  // make sure the device's context exists before asking for it
  e = cudaFree(nullptr);
  if (e != cudaSuccess) return hips::record_cuda_error(e);
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchEntry& ent = g_scratch[dev];
  if (!ent.addr || !ctx || ent.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) return hips::record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    ent.addr = p;
    ent.ctx = ctx;
  }
  *addr = ent.addr;
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
  cudaError_t e = cudaMemsetAsync(base, 0, hips::kStatusBytes, stream);
  if (e != cudaSuccess) return hips::record_cuda_error(e);
  a.status = static_cast<hips::Status*>(base);
  a.counters = reinterpret_cast<unsigned int*>(static_cast<unsigned char*>(base) + hips::kCounterOffset);
  a.part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + hips::kStatusBytes);
  return hips::record_cuda_error(tensor_core ? hips::launch_attn_mma(a, smem, stream)
                                             : hips::launch_attn_fma(a, smem, stream));
}

// Status of the most recent hip_sparse_attn_noalloc call on the current
// device: synchronises `stream`, reads the status word from the fixed array
// and clears it.
extern "C" int hip_noalloc_check_status(void* stream) {
  void* base = nullptr;
  int st = scratch_on_current_device(&base);
  if (st) return st;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return hips::record_cuda_error(e);
  hips::Status host{};
  e = cudaMemcpy(&host, base, sizeof(host), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return hips::record_cuda_error(e);
  if (host.flags == 0) return HIPS_OK;
  e = cudaMemset(base, 0, sizeof(host));
  if (e != cudaSuccess) return hips::record_cuda_error(e);
  return HIPS_ERR_TIMEOUT;
}
