// Device helpers shared by the hierarchically pruned attention kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hips {

constexpr int kD = 128;            // head_dim
constexpr int kThreads = 256;      // threads of the CUDA-core kernels
constexpr int kWarps = kThreads / 32;
constexpr int kMaxN0 = 2048;       // topk / block_k
constexpr int kMaxDevices = 64;
constexpr unsigned kStatusTimeout = 1u;  // a bounded wait gave up
constexpr unsigned kStatusBound = 2u;    // a list outgrew its planned capacity
constexpr long long kWaitCycles = 4000000000ll;  // ~2 s at 2 GHz
// values of enum hips_dtype (include/hip_sparse.h)
constexpr int kDtypeF32 = 0, kDtypeBf16 = 1, kDtypeBf16E5m2 = 2;

// Status block at the head of every workspace (sticky error bits), plus the
// number of candidate chunks the mask kernels scored since the block was
// cleared (a work counter: every candidate is scored exactly once).
struct Status {
  unsigned int flags;
  unsigned int where;
  unsigned long long scored;
};

__device__ __forceinline__ void report(Status* st, unsigned bits, unsigned where) {
  if (st) {
    atomicOr(&st->flags, bits);
    atomicExch(&st->where, where);
  }
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity; gives up after kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

// Bulk (non-tensor) async copy global -> this CTA's shared memory, completing
// on an mbarrier. dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte async copy global -> shared through the LSU (many in flight per
// thread); dst and src 16-byte aligned.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}

// Arrive on an mbarrier once every cp.async this thread issued so far has
// landed (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- numbers

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint16_t f2bf16_rn(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7f800000u) == 0x7f800000u) return static_cast<uint16_t>((u >> 16) | ((u & 0xffff) ? 0x40 : 0));
  u += 0x7fffu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

// Two floats to packed bf16x2 (round to nearest even); lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Order-preserving map of a float score onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t score_key(float f) {
  if (f == 0.0f) f = 0.0f;  // -0 and +0 are the same score
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Load the 16 elements a lane owns in the canonical order (slices lane and
// lane + 8 of 8 consecutive elements each) of one 128-element row.
template <typename T>
__device__ __forceinline__ void load_row16(const unsigned char* row, int lane8, float (&x)[16]);

template <>
__device__ __forceinline__ void load_row16<uint16_t>(const unsigned char* row, int lane8,
                                                     float (&x)[16]) {
  const uint4 a = *reinterpret_cast<const uint4*>(row + lane8 * 16);
  const uint4 b = *reinterpret_cast<const uint4*>(row + 128 + lane8 * 16);
  x[0] = bf16lo(a.x); x[1] = bf16hi(a.x); x[2] = bf16lo(a.y); x[3] = bf16hi(a.y);
  x[4] = bf16lo(a.z); x[5] = bf16hi(a.z); x[6] = bf16lo(a.w); x[7] = bf16hi(a.w);
  x[8] = bf16lo(b.x); x[9] = bf16hi(b.x); x[10] = bf16lo(b.y); x[11] = bf16hi(b.y);
  x[12] = bf16lo(b.z); x[13] = bf16hi(b.z); x[14] = bf16lo(b.w); x[15] = bf16hi(b.w);
}

template <>
__device__ __forceinline__ void load_row16<float>(const unsigned char* row, int lane8,
                                                  float (&x)[16]) {
  const float4* p0 = reinterpret_cast<const float4*>(row + lane8 * 32);
  const float4* p1 = reinterpret_cast<const float4*>(row + 256 + lane8 * 32);
  const float4 a = p0[0], b = p0[1], c = p1[0], d = p1[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  x[8] = c.x; x[9] = c.y; x[10] = c.z; x[11] = c.w; x[12] = d.x; x[13] = d.y; x[14] = d.z;
  x[15] = d.w;
}

// fp8 e5m2 (1 sign, 5 exponent bits with bias 15, 2 mantissa bits; the
// OCP 8-bit floating-point format): a code is the upper byte of the binary16
// encoding of the same value, so widening through binary16 is exact, and so
// is narrowing the float to bf16 afterwards (at most 3 significant bits,
// exponents within bf16's range).
__device__ __forceinline__ void e5m2x4_to_f32(uint32_t w, float* x) {
  const uint32_t lo = __byte_perm(w, 0u, 0x1404);  // binary16 halves: byte 0 << 8, byte 1 << 8
  const uint32_t hi = __byte_perm(w, 0u, 0x3424);  // byte 2 << 8, byte 3 << 8
  asm("{\n\t.reg .b16 a, b, c, d;\n\t"
      "mov.b32 {a, b}, %4;\n\t"
      "mov.b32 {c, d}, %5;\n\t"
      "cvt.f32.f16 %0, a;\n\t"
      "cvt.f32.f16 %1, b;\n\t"
      "cvt.f32.f16 %2, c;\n\t"
      "cvt.f32.f16 %3, d;\n\t}"
      : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3])
      : "r"(lo), "r"(hi));
}

// Four e5m2 codes -> four bf16 (two words, element 0 in the low half of .x).
__device__ __forceinline__ uint2 e5m2x4_to_bf16x4(uint32_t w) {
  float f[4];
  e5m2x4_to_f32(w, f);
  return make_uint2(__byte_perm(__float_as_uint(f[0]), __float_as_uint(f[1]), 0x7632),
                    __byte_perm(__float_as_uint(f[2]), __float_as_uint(f[3]), 0x7632));
}

// One 16-byte chunk of e5m2 codes (elements 16c .. 16c + 15 of a key row) as
// the two 16-byte bf16 chunks 2c, 2c + 1 of the row.
__device__ __forceinline__ void e5m2x16_to_bf16(const uint4& w, uint4& c0, uint4& c1) {
  const uint2 a = e5m2x4_to_bf16x4(w.x), b = e5m2x4_to_bf16x4(w.y);
  const uint2 c = e5m2x4_to_bf16x4(w.z), d = e5m2x4_to_bf16x4(w.w);
  c0 = make_uint4(a.x, a.y, b.x, b.y);
  c1 = make_uint4(c.x, c.y, d.x, d.y);
}

template <>
__device__ __forceinline__ void load_row16<uint8_t>(const unsigned char* row, int lane8,
                                                    float (&x)[16]) {
  const uint2 a = *reinterpret_cast<const uint2*>(row + lane8 * 8);
  const uint2 b = *reinterpret_cast<const uint2*>(row + 64 + lane8 * 8);
  e5m2x4_to_f32(a.x, x);
  e5m2x4_to_f32(a.y, x + 4);
  e5m2x4_to_f32(b.x, x + 8);
  e5m2x4_to_f32(b.y, x + 12);
}

template <typename T>
constexpr int row_bytes() { return kD * static_cast<int>(sizeof(T)); }

// A lane's share of one key (or value) row in the canonical order, held raw
// in registers until used: slices l8 and l8 + 8 (elements 8 l8 .. 8 l8 + 7
// and 64 + 8 l8 .. 64 + 8 l8 + 7). load() takes a global or a shared-memory
// row (generic addressing); get() widens to fp32 (exactly, for every type).
template <typename KvT>
struct Row16;

template <>
struct Row16<uint16_t> {  // bf16
  uint4 a, b;
  __device__ __forceinline__ void load(const unsigned char* row, int l8) {
    a = *reinterpret_cast<const uint4*>(row + l8 * 16);
    b = *reinterpret_cast<const uint4*>(row + 128 + l8 * 16);
  }
  __device__ __forceinline__ void zero() { a = b = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void get(float (&x)[16]) const {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[2 * i] = bf16lo(w[i]);
      x[2 * i + 1] = bf16hi(w[i]);
    }
  }
};

template <>
struct Row16<float> {
  float4 a0, a1, b0, b1;
  __device__ __forceinline__ void load(const unsigned char* row, int l8) {
    const float4* p = reinterpret_cast<const float4*>(row + l8 * 32);
    const float4* q = reinterpret_cast<const float4*>(row + 256 + l8 * 32);
    a0 = p[0]; a1 = p[1]; b0 = q[0]; b1 = q[1];
  }
  __device__ __forceinline__ void zero() { a0 = a1 = b0 = b1 = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void get(float (&x)[16]) const {
    x[0] = a0.x; x[1] = a0.y; x[2] = a0.z; x[3] = a0.w; x[4] = a1.x; x[5] = a1.y; x[6] = a1.z;
    x[7] = a1.w; x[8] = b0.x; x[9] = b0.y; x[10] = b0.z; x[11] = b0.w; x[12] = b1.x;
    x[13] = b1.y; x[14] = b1.z; x[15] = b1.w;
  }
};

template <>
struct Row16<uint8_t> {  // fp8 e5m2 codes, widened exactly
  uint2 a, b;
  __device__ __forceinline__ void load(const unsigned char* row, int l8) {
    a = *reinterpret_cast<const uint2*>(row + l8 * 8);
    b = *reinterpret_cast<const uint2*>(row + 64 + l8 * 8);
  }
  __device__ __forceinline__ void zero() { a = b = make_uint2(0, 0); }
  __device__ __forceinline__ void get(float (&x)[16]) const {
    e5m2x4_to_f32(a.x, x);
    e5m2x4_to_f32(a.y, x + 4);
    e5m2x4_to_f32(b.x, x + 8);
    e5m2x4_to_f32(b.y, x + 12);
  }
};

// Canonical-order reduction of RC lane partials over the 8 lanes of a group:
// level 1 adds lanes (l, l^4), level 2 (l, l^2), level 3 (l, l^1), i.e.
// ((p0+p4)+(p2+p6)) + ((p1+p5)+(p3+p7)) for every dot. With RC = 2^r dots a
// lane keeps half of its dots at each of the first r levels, so afterwards
// lane l holds dot (l >> (3 - r)) (the same sum tree, fewer shuffles).
template <int RC>
__device__ __forceinline__ float group_reduce_rows(float (&v)[RC], int lane8) {
  static_assert(RC == 1 || RC == 2 || RC == 4 || RC == 8, "RC");
#pragma unroll
  for (int level = 0; level < 3; ++level) {
    const int off = 4 >> level;
    const int have = (RC >> level) > 1 ? (RC >> level) : 1;  // dots still held
    if (have > 1) {
      const int half = have / 2;
      const bool upper = (lane8 & off) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        const float recv = __shfl_xor_sync(0xffffffffu, send, off);
        v[i] = keep + recv;
      }
    } else {
      v[0] = v[0] + __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
  return v[0];
}

template <int RC>
__device__ __forceinline__ int group_row_of_lane(int lane8) {
  return RC == 8 ? lane8 : RC == 4 ? (lane8 >> 1) : RC == 2 ? (lane8 >> 2) : 0;
}

// Exclusive block-wide prefix sum over kThreads threads; `total` gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = lane < kWarps ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kWarps) scratch[lane] = t;
  }
  __syncthreads();
  const int before = w ? scratch[w - 1] : 0;
  total = scratch[kWarps - 1];
  __syncthreads();
  return before + x - v;
}

__device__ __forceinline__ int block_max_int(int v, int* scratch) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) scratch[w] = v;
  __syncthreads();
  int r = scratch[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) r = max(r, scratch[i]);
  __syncthreads();
  return r;
}

}  // namespace hips
