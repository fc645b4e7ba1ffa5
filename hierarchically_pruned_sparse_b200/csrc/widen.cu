// Exact widening of an fp8 e5m2 KV cache to bf16, for the e5m2 shapes that
// no e5m2 kernel plans (see api.cu): the bf16 kernels then run on the
// widened rows. A code is the upper byte of the binary16 encoding of the
// same value, and every e5m2 value is exact in bf16 (hips_common.cuh).
#include <cuda_runtime.h>

#include <algorithm>

#include "hips_common.cuh"
#include "hips_kernels.h"
#include "widen.h"

namespace hips {
namespace {

// Thread per 16 codes (one 16-byte load, two 16-byte stores); rows [0,
// rows) of each of `heads` heads, from a head stride of src_cap rows to a
// compact head stride of `rows`.
__global__ void __launch_bounds__(kThreads) widen_e5m2_kernel(const uint8_t* src, uint16_t* dst,
                                                             int64_t heads, int64_t rows,
                                                             int64_t src_cap) {
  constexpr int kChunks = kD / 16;  // 16-code chunks of a row
  const int64_t total = heads * rows * kChunks;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += step) {
    const int64_t c = i % kChunks, r = (i / kChunks) % rows, h = i / (kChunks * rows);
    const uint4 w = *reinterpret_cast<const uint4*>(src + (h * src_cap + r) * kD + c * 16);
    uint4 c0, c1;
    e5m2x16_to_bf16(w, c0, c1);
    uint4* d = reinterpret_cast<uint4*>(dst + (h * rows + r) * kD + c * 16);
    d[0] = c0;
    d[1] = c1;
  }
}

}  // namespace

cudaError_t launch_widen_e5m2(const void* src, void* dst, int64_t heads, int64_t rows, int64_t src_cap,
                              cudaStream_t stream) {
  const int64_t work = heads * rows * (kD / 16);
  const int64_t blocks = std::min<int64_t>((work + kThreads - 1) / kThreads, 148 * 8);
  if (blocks <= 0) return cudaSuccess;
  widen_e5m2_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      static_cast<const uint8_t*>(src), static_cast<uint16_t*>(dst), heads, rows, src_cap);
  return cudaGetLastError();
}

}  // namespace hips
