// Launch interface of the e5m2 widening kernel (widen.cu), used by the C ABI
// for the e5m2 shapes that no e5m2 kernel plans.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hips {

// Exact widening of e5m2 K or V rows [0, rows) of `heads` heads (head stride
// src_cap rows) into compact bf16 rows (head stride `rows`).
cudaError_t launch_widen_e5m2(const void* src, void* dst, int64_t heads, int64_t rows, int64_t src_cap,
                              cudaStream_t stream);

}  // namespace hips
