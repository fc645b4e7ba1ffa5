// Block-sparse (and dense) attention on tensor cores for query blocks (bf16).
//
// Computes, for every query row at position p of a query block, the exact
// softmax attention over the keys of the block's selected key blocks that
// lie at or before p (plus the keys appended since the mask was computed),
// as the sparse attention step of "A Training-free Sub-quadratic Cost
// Transformer Model Serving Framework With Hierarchically Pruned Attention"
// (Author Rebuttal to the Reviewer NLBm, W2: per-row non-zero block indices
// and nnz).
//
// Design: one CTA per (256 query rows of a query block, KV head, sequence);
// the rows are the group's query heads x positions, so all of them share
// every gathered K/V tile. They form two M = 128 halves with their own TMEM
// accumulators (S: 2 x 2 buffers of 64 columns, O: 2 x 128 columns, all 512
// columns of the SM). Warp roles:
//  * warps 8-10 gather the keys of the next tiles (64 keys: K and V rows of
//    the listed blocks) with cp.async into a 3-stage ring, in the tensor-core
//    layout (K-major, 128-byte swizzle);
//  * warp 11 issues the MMAs: S = Q K^T (M = 128 rows, N = 64 keys, K = 128)
//    for each half into one of two TMEM buffers, then O += P V (M = 128,
//    N = 128, K = 64, V read as an MN-major operand); S of tile j+1 is issued
//    before P V of tile j, so the tensor core works while the softmax of
//    tile j runs;
//  * warps 0-7 own one query row per thread (warps 0-3 the first half, 4-7
//    the second): read the row of S from TMEM, mask (causal, invalid slots),
//    keep a reference max and the row sum, write P (bf16) to shared memory.
//    The reference max only moves (and O and the sum are rescaled, through
//    TMEM) when a tile's max exceeds it by more than 2^8, so P stays <= 256
//    and the result is the exact softmax.
// All waits are bounded; a timeout sets the status word.
#include <mutex>

#include "hips_common.cuh"
#include "hips_kernels.h"
#include "hips_tc.cuh"

namespace hips {

namespace {

// 2^x by the SFU's ex2.approx.ftz instruction (relative error about 2^-22;
// results below the normal range flush to 0, and 2^-inf = 0): one
// instruction, where exp2f adds the handling of subnormal results that
// softmax weights (at most 2^8, summed in fp32 and stored as bf16) never need.
__device__ __forceinline__ float fast_exp2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

constexpr int kRows = 128;                 // query rows per MMA (M)
constexpr int kHalves = 2;                 // MMA row halves per CTA
constexpr int kCtaRows = kRows * kHalves;  // query rows per CTA
constexpr int kKeys = 64;                  // keys per tile
constexpr int kStages = 3;
constexpr int kSoftmax = kCtaRows;         // softmax threads (warps 0-7)
constexpr int kLoaderWarp0 = kSoftmax / 32;
constexpr int kLoaders = 96;               // warps 8-10
constexpr int kMmaWarp = kLoaderWarp0 + kLoaders / 32;
// 8 softmax + 3 loader + 1 MMA warps: 3 warps per SM sub-partition, so that
// each thread may hold up to 168 registers
constexpr int kAttnThreads = (kMmaWarp + 1) * 32;
constexpr int kQBytes = kRows * 256;       // 32 KB per half: two 16 KB column halves
constexpr int kKVHalf = kKeys * 128;       // 8 KB
constexpr int kKVBytes = kKeys * 256;      // 16 KB per K (or V) tile
constexpr int kPBytes = kRows * 128;       // 16 KB: one row of 64 keys per query row
constexpr float kRescaleLog2 = 8.0f;

struct AttnMmaSmem {
  int q, k, v, p, bars, kpos, slot, table, total;
};

__host__ __device__ inline int al2(int x, int a) { return (x + a - 1) / a * a; }

__host__ __device__ inline AttnMmaSmem attn_mma_layout(int table_items) {
  AttnMmaSmem L;
  int o = 0;
  L.q = o;     o += kHalves * kQBytes;
  L.k = o;     o += kStages * kKVBytes;
  L.v = o;     o += kStages * kKVBytes;
  L.p = o;     o += kHalves * kPBytes;  // one P tile per half
  L.bars = o;  o += 16 * 8;
  L.kpos = o;  o += 2 * kKeys * 4 + 16;  // key positions of two tiles, then their flags
  L.slot = o;  o += 16;
  L.table = o; o += al2(table_items * 8, 16);
  L.total = o + 1024;
  return L;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__global__ void __launch_bounds__(kAttnThreads, 1) attn_mma_kernel(AttnArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qb = blockIdx.y % a.nqb, g = blockIdx.y / a.nqb, b = blockIdx.z;
  const int i0 = qb * a.block_q;
  const int nrows = min(a.block_q, a.q_len - i0);
  const int R = a.group * nrows;
  const int64_t q_first = a.q_pos0 + i0, q_last = q_first + nrows - 1;
  const int64_t vis = min64(q_last + 1, a.seq_len);
  const int IK = a.item_keys;  // a power of two
  const int lik = __ffs(IK) - 1;
  const int ipt = kKeys >> lik;
  const int row0 = blockIdx.x * kCtaRows;
  const int halves = min(kHalves, (R - row0 + kRows - 1) / kRows);  // halves with rows (>= 1)

  const AttnMmaSmem L = attn_mma_layout(a.table_items);
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  unsigned char* qs = smem + L.q;
  unsigned char* ks = smem + L.k;
  unsigned char* vs = smem + L.v;
  unsigned char* ps = smem + L.p;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* kv_full = bars;        // [kStages] cp.async arrivals of the loader threads
  uint64_t* kv_empty = bars + 3;   // [kStages] P V of the tile in the stage done
  uint64_t* s_full = bars + 6;     // [2] S MMAs (both halves) done
  uint64_t* p_full = bars + 8;     // [2] P written by the softmax threads
  uint64_t* pv_done = bars + 10;   // [2] P V MMA done
  int* kpos = reinterpret_cast<int*>(smem + L.kpos);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + L.slot);
  int2* table = reinterpret_cast<int2*>(smem + L.table);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], kLoaders);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], kSoftmax);
      mbar_init(&pv_done[s], 1);
    }
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 0) tmem_alloc(tslot, 512);
  // query rows of this CTA in the operand layout, one 128-row half after the
  // other (rows >= R are zero)
  const uint16_t* qg = static_cast<const uint16_t*>(a.q);
  for (int i = tid; i < kCtaRows * 16; i += kAttnThreads) {
    const int rq = i >> 4, c = i & 15;
    const int ur = row0 + rq, r = rq & (kRows - 1);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (ur < R) {
      const int h = g * a.group + ur / nrows, qi = i0 + ur % nrows;
      v = *reinterpret_cast<const uint4*>(
          qg + ((static_cast<int64_t>(b) * a.n_qheads + h) * a.q_len + qi) * kD + c * 8);
    }
    *reinterpret_cast<uint4*>(qs + (rq >> 7) * kQBytes + (c >> 3) * (kQBytes / 2) +
                              sw128_offset(r, c & 7)) = v;
  }
  // the idx rows may come from the kernel launched just before this one
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- work items (one key block each): the idx blocks, then the keys
  // appended since the mask (or, dense, every block of the causal range)
  const int64_t unit = (static_cast<int64_t>(b) * a.n_kvheads + g) * a.nqb + qb;
  int nitems;
  if (a.dense) {
    nitems = static_cast<int>((vis + IK - 1) / IK);
    for (int t = tid; t < nitems; t += kAttnThreads) {
      const int64_t j0 = static_cast<int64_t>(t) * IK;
      table[t] = make_int2(static_cast<int>(j0), static_cast<int>(min64(IK, vis - j0)));
    }
  } else {
    const int32_t* idx_row = a.idx + unit * a.row_stride;
    const int cap = static_cast<int>(a.row_stride - 1);
    const int nnz = max(0, min(idx_row[0], cap));
    const int64_t tail_items = (max64(0, a.seq_len - a.mask_len) + IK - 1) / IK;
    nitems = static_cast<int>(min64(nnz + tail_items, a.table_items));
    for (int t = tid; t < nitems; t += kAttnThreads) {
      int64_t j0, n;
      if (t < nnz) {
        const int64_t c = idx_row[1 + t];
        j0 = c * IK;
        n = c < 0 ? 0 : min64(IK, min64(a.mask_len, vis) - j0);
      } else {
        j0 = a.mask_len + static_cast<int64_t>(t - nnz) * IK;
        n = min64(IK, vis - j0);
      }
      table[t] = make_int2(static_cast<int>(max64(j0, 0)), static_cast<int>(max64(n, 0)));
    }
  }
  const int ntiles = (nitems + ipt - 1) / ipt;
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tslot;
  const uint32_t tmem_o = tmem + 256;  // O of half h at columns 256 + 128 h
  bool timed_out = false;

  const size_t plane = (static_cast<size_t>(b) * a.kv_heads + g / a.kv_div) * static_cast<size_t>(a.kv_cap) * 256;
  const unsigned char* kbase = static_cast<const unsigned char*>(a.k) + plane;
  const unsigned char* vbase = static_cast<const unsigned char*>(a.v) + plane;

  if (warp >= kLoaderWarp0 && warp < kMmaWarp) {
    // ---------------- loaders: K and V rows of tile j into stage j % kStages
    const int lt = tid - kSoftmax;
    for (int j = 0; j < ntiles; ++j) {
      const int st = j % kStages;
      if (j >= kStages && !mbar_wait(&kv_empty[st], ((j - kStages) / kStages) & 1)) timed_out = true;
      unsigned char* kd = ks + st * kKVBytes;
      unsigned char* vd = vs + st * kKVBytes;
      // two threads per key row (8 of its 16 chunks each, K and V): one
      // table lookup per row and thread
      for (int kk = lt >> 1; kk < kKeys; kk += kLoaders / 2) {
        const int item = j * ipt + (kk >> lik), kt = kk & (IK - 1);
        int64_t key = -1;
        if (item < nitems) {
          const int2 e = table[item];
          if (kt < e.y) key = static_cast<int64_t>(e.x) + kt;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int ch = (lt & 1) + 2 * q;
          const uint32_t dst = (ch >> 3) * kKVHalf + sw128_offset(kk, ch & 7);
          if (key >= 0) {
            cp_async16(kd + dst, kbase + key * 256 + ch * 16);
            cp_async16(vd + dst, vbase + key * 256 + ch * 16);
          } else {
            // a slot without a key: its P is 0, and 0 x V must stay 0 (the
            // slot's stale contents could hold NaN or inf)
            *reinterpret_cast<uint4*>(vd + dst) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      cp_async_arrive(&kv_full[st]);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issue (one thread)
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kRows, kKeys);
      const uint32_t idesc_o = idesc_bf16_f32_bmn(kRows, kD);
      auto issue_pv = [&](int pj) {
        const int psb = pj & 1, pst = pj % kStages;
        if (!mbar_wait(&p_full[psb], (pj >> 1) & 1)) timed_out = true;
        tc_fence_after_sync();
        for (int h = 0; h < halves; ++h) {
#pragma unroll
          for (int k = 0; k < kKeys / 16; ++k) {
            const uint64_t ad = sw128_desc(smem_u32(ps + h * kPBytes) + k * 32);
            const uint64_t bd = sw128_desc_mn(smem_u32(vs + pst * kKVBytes) + k * 2048, kKVHalf);
            tc_mma_bf16(tmem_o + h * 128, ad, bd, idesc_o, (pj > 0 || k > 0) ? 1u : 0u);
          }
        }
        tc_commit(&pv_done[psb]);
        tc_commit(&kv_empty[pst]);
      };
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % kStages, sb = j & 1;
        if (!mbar_wait(&kv_full[st], (j / kStages) & 1)) timed_out = true;
        tc_fence_after_sync();
        for (int h = 0; h < halves; ++h) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t ad =
                sw128_desc(smem_u32(qs + h * kQBytes + (k >> 2) * (kQBytes / 2)) + (k & 3) * 32);
            const uint64_t bd = sw128_desc(smem_u32(ks + st * kKVBytes + (k >> 2) * kKVHalf) + (k & 3) * 32);
            tc_mma_bf16(tmem + h * 128 + sb * kKeys, ad, bd, idesc_s, k > 0 ? 1u : 0u);
          }
        }
        tc_commit(&s_full[sb]);
        if (j >= 1) issue_pv(j - 1);
      }
      if (ntiles > 0) issue_pv(ntiles - 1);
    }
    __syncwarp();
  } else {
    // ---------------- softmax: thread tid owns query row row0 + tid, of
    // half h = tid / 128 (TMEM lane tid % 128)
    const int hh = tid >> 7, rr = tid & (kRows - 1);
    const uint32_t s_col = tmem + hh * 128;   // S buffers of this half
    const uint32_t o_col = tmem_o + hh * 128;  // O of this half
    const int ur = row0 + tid;
    const bool row_ok = ur < R;
    const int64_t my_pos = q_first + (row_ok ? ur % nrows : 0);
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;  // this warp's TMEM lane quarter
    float m_ref = -INFINITY, lsum = 0.0f;
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      if (tid < kKeys) {
        const int item = j * ipt + (tid >> lik), kt = tid & (IK - 1);
        int kp = -1;
        if (item < nitems) {
          const int2 e = table[item];
          if (kt < e.y) kp = e.x + kt;
        }
        kpos[sb * kKeys + tid] = kp;
        // flag: every key of this half-tile is valid and seen by every row
        const bool seen = __all_sync(0xffffffffu, kp >= 0 && kp <= q_first);
        if (lane == 0) kpos[2 * kKeys + sb * 2 + warp] = seen ? 1 : 0;
      }
      named_sync(1, kSoftmax);
      const bool all_seen = kpos[2 * kKeys + sb * 2] && kpos[2 * kKeys + sb * 2 + 1];
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1)) timed_out = true;
      tc_fence_after_sync();
      __syncwarp();
      float s[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys / 16; ++c) {
        float v[16];
        tc_ld16(s_col + lane_base + sb * kKeys + c * 16, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) s[c * 16 + i] = v[i];
      }
      tc_wait_ld();
      float tmax;
      if (all_seen) {
        // no masking: the max of the raw scores times the (positive) scale
        float m[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = max3f(s[i], s[8 + i], max3f(s[16 + i], s[24 + i], s[32 + i]));
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = max3f(m[i], s[40 + i], max3f(s[48 + i], s[56 + i], m[i]));
        tmax = max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7])) * a.scale_log2;
      } else {
        float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < kKeys; c += 4) {
          const int4 kp4 = *reinterpret_cast<const int4*>(kpos + sb * kKeys + c);
          const int kp[4] = {kp4.x, kp4.y, kp4.z, kp4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const bool ok = row_ok && kp[i] >= 0 && kp[i] <= my_pos;
            s[c + i] = ok ? s[c + i] * a.scale_log2 : -INFINITY;
            m[i] = fmaxf(m[i], s[c + i]);
          }
        }
        tmax = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
      }
      // move the reference max only when this tile exceeds it by > 2^8
      const bool grow = tmax > m_ref + kRescaleLog2;
      const float alpha = (grow && m_ref != -INFINITY) ? exp2f(m_ref - tmax) : 1.0f;
      if (__any_sync(0xffffffffu, grow && m_ref != -INFINITY && j > 0)) {
        // O holds tiles < j: wait for the last P V, then scale the rows in TMEM
        if (!mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) timed_out = true;
        tc_fence_after_sync();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < kD / 16; ++c) {
          float v[16];
          tc_ld16(o_col + lane_base + c * 16, v);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] *= alpha;
          tc_st16(o_col + lane_base + c * 16, v);
        }
        tc_wait_st();
      }
      if (grow) {
        lsum *= alpha;
        m_ref = tmax;
      }
      // P overwrites S in place; four partial sums
      float ps4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (all_seen) {
        const float nm = -m_ref;
#pragma unroll
        for (int i = 0; i < kKeys; ++i) {
          s[i] = fast_exp2(fmaf(s[i], a.scale_log2, nm));
          ps4[i & 3] += s[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < kKeys; ++i) {
          s[i] = fast_exp2(s[i] - m_ref);  // 2^-inf = 0
          ps4[i & 3] += s[i];
        }
      }
      lsum += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
      // P buffer sb is free once P V of tile j - 2 is done
      // the P tile of this half is free once P V of tile j - 1 is done
      if (j >= 1 && !mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) timed_out = true;
      unsigned char* prow = ps + hh * kPBytes;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 w;
        w.x = pack_bf16x2(s[c * 8 + 0], s[c * 8 + 1]);
        w.y = pack_bf16x2(s[c * 8 + 2], s[c * 8 + 3]);
        w.z = pack_bf16x2(s[c * 8 + 4], s[c * 8 + 5]);
        w.w = pack_bf16x2(s[c * 8 + 6], s[c * 8 + 7]);
        *reinterpret_cast<uint4*>(prow + sw128_offset(rr, c)) = w;
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(&p_full[sb]);
    }
    // ---- epilogue: O / sum -> bf16 output rows
    if (ntiles > 0) {
      if (!mbar_wait(&pv_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1)) timed_out = true;
      tc_fence_after_sync();
    }
    __syncwarp();
    const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
    uint16_t* orow = nullptr;
    if (row_ok) {
      const int h = g * a.group + ur / nrows, qi = i0 + ur % nrows;
      orow = static_cast<uint16_t*>(a.out) + ((static_cast<int64_t>(b) * a.n_qheads + h) * a.q_len + qi) * kD;
    }
#pragma unroll
    for (int c = 0; c < kD / 16; ++c) {
      float v[16];
      if (ntiles > 0) {
        tc_ld16(o_col + lane_base + c * 16, v);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.0f;
      }
      if (row_ok) {
        uint4 w0, w1;
        uint32_t* u0 = &w0.x;
        uint32_t* u1 = &w1.x;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          u0[i] = pack_bf16x2(v[2 * i] * inv, v[2 * i + 1] * inv);
          u1[i] = pack_bf16x2(v[8 + 2 * i] * inv, v[8 + 2 * i + 1] * inv);
        }
        *reinterpret_cast<uint4*>(orow + c * 16) = w0;
        *reinterpret_cast<uint4*>(orow + c * 16 + 8) = w1;
      }
    }
  }
  if (timed_out) report(a.status, kStatusTimeout, 4);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

int attn_mma_smem_bytes(int table_items) { return attn_mma_layout(table_items).total; }
int attn_mma_tile_keys() { return kKeys; }
int attn_mma_rows() { return kCtaRows; }

cudaError_t launch_attn_mma(const AttnArgs& a, int smem, cudaStream_t stream) {
  static std::mutex mu;  // host threads may launch concurrently
  std::lock_guard<std::mutex> lock(mu);
  static int smem_set[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  dev %= kMaxDevices;
  if (smem > smem_set[dev]) {
    e = cudaFuncSetAttribute(attn_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    smem_set[dev] = smem;
  }
  cudaLaunchConfig_t cfg = {};
  const int mtiles = (a.rows_max + kCtaRows - 1) / kCtaRows;
  cfg.gridDim = dim3(mtiles, a.nqb * a.n_kvheads, a.batch);
  cfg.blockDim = dim3(kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_mma_kernel, a);
}

}  // namespace hips
