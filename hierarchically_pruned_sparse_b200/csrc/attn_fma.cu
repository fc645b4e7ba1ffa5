// Block-sparse (and dense) attention on CUDA cores for decode-sized query
// groups, split over the key list (flash-decoding) plus a combine kernel.
//
// The sparse attention step consumes, per query block, the ascending list of
// selected key blocks and its nnz ("A Training-free Sub-quadratic Cost
// Transformer Model Serving Framework With Hierarchically Pruned Attention",
// Author Rebuttal to the Reviewer NLBm, W2). A query row at position p
// attends the keys j <= p of those blocks that lie below mask_len, plus every
// key in [mask_len, seq_len) appended since the mask was computed (the mask
// refresh interval r_m of the research-map summary, Limitations).
//
// Design: grid (splits, KV head x query block, sequence). Split s takes the
// work items s, s + splits, ... (one key block each); K and V rows of a
// 64-key tile (128 keys for fp8 e5m2 rows, widened exactly when read) are gathered by all threads with 16-byte cp.async copies into a
// 3-stage ring (all stages requested up front) (completion tracked on one mbarrier per stage), the
// G query heads of the group share every gathered tile, and each of 8 warps
// works on 4 keys at a time with 8 lanes per key (16 head elements per lane).
// Scores go through an fp32 online softmax (exp2 domain); each split writes
// (m, l, unnormalised o) to the workspace and the last split of a unit to
// finish (an atomic ticket; nobody waits) merges them into the output. The
// grid is one wave (splits x units <= SM count). The kernel is launched with
// programmatic stream serialisation: everything before the grid-dependency
// wait (barrier set-up, query loads) overlaps the tail of the mask kernel.
#include <mutex>

#include "hips_common.cuh"
#include "hips_kernels.h"

namespace hips {

namespace {

constexpr int kStages = 3;
constexpr int kTileBytes = 16384;  // one of K or V per stage
constexpr int kPartStride = kD + 4; // m, l, pad, pad, o[128]: o 16-byte aligned

struct AttnSmem {
  int kring, vring, bars, table, s, p, alpha, ml, total;
};

__host__ __device__ inline int align16(int x) { return (x + 15) / 16 * 16; }

__host__ __device__ inline AttnSmem attn_smem_layout(int tile_keys, int rc, int table_items) {
  AttnSmem L;
  int o = 0;
  L.kring = o;  o += kStages * kTileBytes;
  L.vring = o;  o += kStages * kTileBytes;
  L.bars = o;   o += align16(kStages * 8);
  L.table = o;  o += align16(table_items * 8);
  L.s = o;      o += align16(rc * tile_keys * 4);
  L.p = o;      o += align16(rc * tile_keys * 4);
  L.alpha = o;  o += align16(rc * 4);
  L.ml = o;     o += align16((2 * rc + 4) * 4);  // m, l per row; merge flag
  L.total = o;
  return L;
}

// T: element type of q and out (bf16 as uint16_t, or float); KT: of k and v
// (T, or uint8_t for fp8 e5m2 codes with bf16 q and out).
template <typename T, typename KT, int RC>
__global__ void __launch_bounds__(kThreads, 1) attn_fma_kernel(AttnArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kRowB = row_bytes<KT>();
  constexpr int kTileKeys = kTileBytes / kRowB;
  constexpr int kPasses = kTileKeys / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int lane8 = lane & 7, grp = lane >> 3;

  const int split = blockIdx.x;
  const int qb = blockIdx.y % a.nqb;
  const int g = blockIdx.y / a.nqb;
  const int b = blockIdx.z;
  const int i0 = qb * a.block_q;
  const int nrows = min(a.block_q, a.q_len - i0);
  const int R = a.group * nrows;
  const int64_t q_first = a.q_pos0 + i0, q_last = q_first + nrows - 1;
  const int IK = a.item_keys;

  const AttnSmem L = attn_smem_layout(kTileKeys, RC, a.table_items);
  unsigned char* kring = smem + L.kring;
  unsigned char* vring = smem + L.vring;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  int2* table = reinterpret_cast<int2*>(smem + L.table);
  float* s_sm = reinterpret_cast<float*>(smem + L.s);
  float* p_sm = reinterpret_cast<float*>(smem + L.p);
  float* alpha_sm = reinterpret_cast<float*>(smem + L.alpha);
  float* ml_sm = reinterpret_cast<float*>(smem + L.ml);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], kThreads);
    fence_mbar_init();
  }
  // query rows in registers: lane holds 16 elements of each of the RC rows
  float qreg[RC][16];
  {
    const T* qp = static_cast<const T*>(a.q);
#pragma unroll
    for (int r = 0; r < RC; ++r) {
      if (r < R) {
        const int h = g * a.group + r / nrows, i = i0 + r % nrows;
        const unsigned char* row = reinterpret_cast<const unsigned char*>(
            qp + ((static_cast<int64_t>(b) * a.n_qheads + h) * a.q_len + i) * kD);
        load_row16<T>(row, lane8, qreg[r]);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) qreg[r][e] = 0.0f;
      }
    }
  }
  // the idx rows may come from the kernel launched just before this one
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- work items of this split: items split, split + nsplit, ... (strided,
  // so the splits stay balanced whatever nnz is). nnz and this split's block
  // ids are loaded together (one memory latency); ids are range-checked so a
  // malformed row cannot drive reads outside [0, seq_len)
  const int64_t unit = (static_cast<int64_t>(b) * a.n_kvheads + g) * a.nqb + qb;
  const int32_t* idx_row = a.dense ? nullptr : a.idx + unit * a.row_stride;
  const int64_t vis = min64(q_last + 1, a.seq_len);
  int nmine;
  if (a.dense) {
    const int64_t nitems = (vis + IK - 1) / IK;
    nmine = nitems > split ? static_cast<int>((nitems - split + a.nsplit - 1) / a.nsplit) : 0;
  } else {
    const int cap = static_cast<int>(a.row_stride - 1);
    const int64_t tail_items = (max64(0, a.seq_len - a.mask_len) + IK - 1) / IK;
    const int raw_nnz = idx_row[0];
    int raw[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t it = split + static_cast<int64_t>(a.nsplit) * (tid + u * kThreads);
      raw[u] = (tid + u * kThreads < a.table_items && it < cap) ? idx_row[1 + it] : -1;
    }
    const int nnz = max(0, min(raw_nnz, cap));
    const int64_t nitems = nnz + tail_items;
    nmine = nitems > split ? static_cast<int>((nitems - split + a.nsplit - 1) / a.nsplit) : 0;
    nmine = min(nmine, a.table_items);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int t = tid + u * kThreads;
      if (t < nmine) {
        const int64_t it = split + static_cast<int64_t>(a.nsplit) * t;
        int64_t j0, n;
        if (it < nnz) {
          const int64_t c = raw[u];
          j0 = c * IK;
          n = c < 0 ? 0 : min64(IK, min64(a.mask_len, vis) - j0);
        } else {
          j0 = a.mask_len + (it - nnz) * IK;
          n = min64(IK, vis - j0);
        }
        table[t] = make_int2(static_cast<int>(max64(j0, 0)), static_cast<int>(max64(n, 0)));
      }
    }
    for (int t = tid + 2 * kThreads; t < nmine; t += kThreads) {  // long rows (few splits)
      const int64_t it = split + static_cast<int64_t>(a.nsplit) * t;
      int64_t j0, n;
      if (it < nnz) {
        const int64_t c = idx_row[1 + it];
        j0 = c * IK;
        n = c < 0 ? 0 : min64(IK, min64(a.mask_len, vis) - j0);
      } else {
        j0 = a.mask_len + (it - nnz) * IK;
        n = min64(IK, vis - j0);
      }
      table[t] = make_int2(static_cast<int>(max64(j0, 0)), static_cast<int>(max64(n, 0)));
    }
  }
  auto item_at = [&](int t) -> int2 {
    if (!a.dense) return table[t];
    const int64_t j0 = (split + static_cast<int64_t>(a.nsplit) * t) * IK;
    return make_int2(static_cast<int>(j0), static_cast<int>(max64(min64(IK, vis - j0), 0)));
  };
  __syncthreads();

  const size_t plane = (static_cast<size_t>(b) * a.kv_heads + g / a.kv_div) * static_cast<size_t>(a.kv_cap) * kRowB;
  const unsigned char* kbase = static_cast<const unsigned char*>(a.k) + plane;
  const unsigned char* vbase = static_cast<const unsigned char*>(a.v) + plane;
  const int ipt = kTileKeys / IK;
  const int ntiles = (nmine + ipt - 1) / ipt;

  constexpr int kChunks = kRowB / 16;  // 16-byte chunks per key row
  auto issue = [&](int t) {  // all threads
    const int slot = t % kStages;
    const int f = t * ipt, cnt = min(ipt, nmine - f);
    unsigned char* kd = kring + slot * kTileBytes;
    unsigned char* vd = vring + slot * kTileBytes;
    const int nchunks = cnt * IK * kChunks;
    for (int i = tid; i < nchunks; i += kThreads) {
      const int kk = i / kChunks, ch = i - kk * kChunks;
      const int item = kk / IK, kt = kk - item * IK;
      const int2 e = item_at(f + item);
      if (kt < e.y) {
        const size_t src = (static_cast<size_t>(e.x) + kt) * kRowB + ch * 16;
        cp_async16(kd + kk * kRowB + ch * 16, kbase + src);
        cp_async16(vd + kk * kRowB + ch * 16, vbase + src);
      }
    }
    cp_async_arrive(&bars[slot]);
  };

  float acc[RC][16];
#pragma unroll
  for (int r = 0; r < RC; ++r)
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[r][e] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f;  // valid in warp r for row r
  bool timed_out = false;

  for (int t = 0; t < min(kStages, ntiles); ++t) issue(t);

  for (int t = 0; t < ntiles; ++t) {
    const int slot = t % kStages;
    if (!mbar_wait(&bars[slot], (t / kStages) & 1)) timed_out = true;
    const int f = t * ipt, cnt = min(ipt, nmine - f);
    const unsigned char* ktile = kring + slot * kTileBytes;
    const unsigned char* vtile = vring + slot * kTileBytes;

    bool kvalid[kPasses];
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      const int kk = p * 32 + warp * 4 + grp;
      const int item = kk / IK, kt = kk - item * IK;
      int64_t j = -1;
      if (item < cnt) {
        const int2 e = item_at(f + item);
        if (kt < e.y) j = static_cast<int64_t>(e.x) + kt;
      }
      kvalid[p] = j >= 0;
      float kx[16];
      load_row16<KT>(ktile + kk * kRowB, lane8, kx);
      float part[RC];
#pragma unroll
      for (int r = 0; r < RC; ++r) {
        float x = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) x = __fmaf_rn(qreg[r][e], kx[e], x);
        part[r] = x;
      }
      const float dot = group_reduce_rows<RC>(part, lane8);
      const int row = group_row_of_lane<RC>(lane8);
      const bool ok = j >= 0 && row < R && j <= q_first + row % nrows;
      if ((lane8 & ((8 / RC) - 1)) == 0) s_sm[row * kTileKeys + kk] = ok ? dot * a.scale_log2 : -INFINITY;
    }
    __syncthreads();
    // online softmax, one warp per row
    if (warp < RC) {
      const int r = warp;
      float sv[kPasses];
      float tmax = -INFINITY;
#pragma unroll
      for (int p = 0; p < kPasses; ++p) {
        sv[p] = s_sm[r * kTileKeys + p * 32 + lane];
        tmax = fmaxf(tmax, sv[p]);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = m_new == -INFINITY ? 1.0f : exp2f(m_run - m_new);
      float psum = 0.0f;
#pragma unroll
      for (int p = 0; p < kPasses; ++p) {
        const float pv = sv[p] == -INFINITY ? 0.0f : exp2f(sv[p] - m_new);
        p_sm[(p * 32 + lane) * RC + r] = pv;
        psum += pv;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
      l_run = l_run * alpha + psum;
      m_run = m_new;
      if (lane == 0) alpha_sm[r] = alpha;
    }
    __syncthreads();
    float al[RC];
#pragma unroll
    for (int r = 0; r < RC; ++r) al[r] = alpha_sm[r];
#pragma unroll
    for (int r = 0; r < RC; ++r)
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[r][e] *= al[r];
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
      if (!kvalid[p]) continue;
      const int kk = p * 32 + warp * 4 + grp;
      float vx[16];
      load_row16<KT>(vtile + kk * kRowB, lane8, vx);
      float pk[RC];
#pragma unroll
      for (int r = 0; r < RC; ++r) pk[r] = p_sm[kk * RC + r];
#pragma unroll
      for (int r = 0; r < RC; ++r)
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[r][e] = __fmaf_rn(pk[r], vx[e], acc[r][e]);
    }
    __syncthreads();
    if (t + kStages < ntiles) issue(t + kStages);  // into the slot just consumed
  }

  // ---- reduce the 4 key groups of a warp, then the 8 warps
#pragma unroll
  for (int r = 0; r < RC; ++r)
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float x = acc[r][e];
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      x += __shfl_xor_sync(0xffffffffu, x, 16);
      acc[r][e] = x;
    }
  float* red = reinterpret_cast<float*>(kring);  // ring is idle now: [warp][RC][128]
  if (grp == 0) {
#pragma unroll
    for (int r = 0; r < RC; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[(warp * RC + r) * kD + lane8 * 8 + e] = acc[r][e];
        red[(warp * RC + r) * kD + 64 + lane8 * 8 + e] = acc[r][8 + e];
      }
  }
  if (warp < RC && lane == 0) {
    ml_sm[2 * warp] = m_run;
    ml_sm[2 * warp + 1] = l_run;
  }
  __syncthreads();
  for (int x = tid; x < R * kD; x += kThreads) {
    const int r = x / kD, e = x % kD;
    float o = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) o += red[(w * RC + r) * kD + e];
    const int h = g * a.group + r / nrows, i = i0 + r % nrows;
    const int64_t grow = (static_cast<int64_t>(b) * a.n_qheads + h) * a.q_len + i;
    const float m = ml_sm[2 * r], l = ml_sm[2 * r + 1];
    if (a.nsplit == 1) {
      const float val = l > 0.0f ? o / l : 0.0f;
      if (sizeof(T) == 2)
        reinterpret_cast<uint16_t*>(a.out)[grow * kD + e] = f2bf16_rn(val);
      else
        reinterpret_cast<float*>(a.out)[grow * kD + e] = val;
    } else {
      float* pr = a.part + (grow * a.nsplit + split) * kPartStride;
      if (e == 0) {
        pr[0] = m;
        pr[1] = l;
      }
      pr[4 + e] = o;
    }
  }
  if (timed_out) report(a.status, kStatusTimeout, 2);
  if (a.nsplit == 1) return;

  // ---- the last split of this unit to finish merges all splits:
  // o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s
  __threadfence();
  __syncthreads();
  int* flag = reinterpret_cast<int*>(ml_sm + 2 * RC);
  if (tid == 0) *flag = atomicAdd(&a.counters[unit], 1u) == static_cast<unsigned>(a.nsplit - 1);
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  float* wts = reinterpret_cast<float*>(kring) + kWarps * RC * kD;  // [RC][nsplit]
  float* lsum = ml_sm;                                              // [RC]
  if (warp < R) {
    const int r = warp;
    const int h = g * a.group + r / nrows, i = i0 + r % nrows;
    const int64_t grow = (static_cast<int64_t>(b) * a.n_qheads + h) * a.q_len + i;
    const float* base = a.part + grow * a.nsplit * kPartStride;
    float M = -INFINITY;
    for (int s = lane; s < a.nsplit; s += 32) M = fmaxf(M, __ldcg(base + s * kPartStride));
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float Ls = 0.0f;
    for (int s = lane; s < a.nsplit; s += 32) {
      const float ms = __ldcg(base + s * kPartStride);
      const float w = (M == -INFINITY || ms == -INFINITY) ? 0.0f : exp2f(ms - M);
      wts[r * a.nsplit + s] = w;
      Ls = __fmaf_rn(w, __ldcg(base + s * kPartStride + 1), Ls);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    __syncwarp();
    if (lane == 0) lsum[r] = Ls;
  }
  __syncthreads();
  for (int x = tid; x < R * (kD / 4); x += kThreads) {
    const int r = x / (kD / 4), d4 = (x % (kD / 4)) * 4;
    const int h = g * a.group + r / nrows, i = i0 + r % nrows;
    const int64_t grow = (static_cast<int64_t>(b) * a.n_qheads + h) * a.q_len + i;
    const float* base = a.part + grow * a.nsplit * kPartStride + 4 + d4;
    float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 8
    for (int s = 0; s < a.nsplit; ++s) {
      const float w = wts[r * a.nsplit + s];
      const float4 ps = __ldcg(reinterpret_cast<const float4*>(base + s * kPartStride));
      o.x = __fmaf_rn(w, ps.x, o.x);
      o.y = __fmaf_rn(w, ps.y, o.y);
      o.z = __fmaf_rn(w, ps.z, o.z);
      o.w = __fmaf_rn(w, ps.w, o.w);
    }
    const float L = lsum[r];
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    const float v0 = o.x * inv, v1 = o.y * inv, v2 = o.z * inv, v3 = o.w * inv;
    if (sizeof(T) == 2) {
      uint16_t* dst = reinterpret_cast<uint16_t*>(a.out) + grow * kD + d4;
      uint2 pk;
      pk.x = static_cast<uint32_t>(f2bf16_rn(v0)) | (static_cast<uint32_t>(f2bf16_rn(v1)) << 16);
      pk.y = static_cast<uint32_t>(f2bf16_rn(v2)) | (static_cast<uint32_t>(f2bf16_rn(v3)) << 16);
      *reinterpret_cast<uint2*>(dst) = pk;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + grow * kD + d4) =
          make_float4(v0, v1, v2, v3);
    }
  }
  if (tid == 0) a.counters[unit] = 0;  // ready for the next call
}

template <typename T, typename KT, int RC>
cudaError_t launch_attn_t(const AttnArgs& a, int smem, cudaStream_t stream) {
  auto kern = attn_fma_kernel<T, KT, RC>;
  static std::mutex mu;  // host threads may launch concurrently
  std::lock_guard<std::mutex> lock(mu);
  static int smem_set[kMaxDevices] = {};  // once per kernel and device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  dev %= kMaxDevices;
  if (smem > smem_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    smem_set[dev] = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.nsplit, a.nqb * a.n_kvheads, a.batch);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename T, typename KT>
cudaError_t launch_attn_rc(const AttnArgs& a, int smem, cudaStream_t s) {
  const int R = a.rows_max;
  if (R <= 1) return launch_attn_t<T, KT, 1>(a, smem, s);
  if (R <= 2) return launch_attn_t<T, KT, 2>(a, smem, s);
  if (R <= 4) return launch_attn_t<T, KT, 4>(a, smem, s);
  return launch_attn_t<T, KT, 8>(a, smem, s);
}

// bytes of one K (V) row
int kv_row_bytes(int dtype) {
  return dtype == kDtypeBf16E5m2 ? kD : dtype == kDtypeBf16 ? 2 * kD : 4 * kD;
}

}  // namespace

int attn_fma_tile_keys(int dtype) { return kTileBytes / kv_row_bytes(dtype); }

int attn_fma_smem_bytes(int dtype, int rows_max, int table_items) {
  const int rc = rows_max <= 1 ? 1 : rows_max <= 2 ? 2 : rows_max <= 4 ? 4 : 8;
  return attn_smem_layout(attn_fma_tile_keys(dtype), rc, table_items).total;
}

cudaError_t launch_attn_fma(const AttnArgs& a, int smem, cudaStream_t stream) {
  if (a.dtype == kDtypeBf16E5m2) return launch_attn_rc<uint16_t, uint8_t>(a, smem, stream);
  return a.dtype == kDtypeBf16 ? launch_attn_rc<uint16_t, uint16_t>(a, smem, stream)
                               : launch_attn_rc<float, float>(a, smem, stream);
}

}  // namespace hips
