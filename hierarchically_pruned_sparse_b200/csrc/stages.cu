// InfiniteHiP pruning stages that run before the hierarchical iteration of a
// mask: the scoring of a stage's chunks (stage_score_kernel) and the per-row
// selection that keeps the best of them (stage_select_kernel).
//
// Method: "[Feature] Support Efficient Sparse HiP Attention (InfiniteHiP)"
// (SGLang pull request), the stages of the serving command's
// --hip-attention-config (stage_chunk_size, stage_k, stage_block_stride_q;
// second_stage_k is the iteration's budget); "A Training-free Sub-quadratic
// Cost Transformer Model Serving Framework With Hierarchically Pruned
// Attention", Author Rebuttal to the Reviewer T2wK, Q1 (the user sets per
// iteration how many chunks are kept, how chunks are broken down and how
// their representatives are picked). Reading (struct hips_stage in
// hip_sparse.h): stage 1 cuts the key blocks [0, N) into aligned chunks of
// its size, a later stage cuts every survivor of the one before; a chunk
// [s, e) is scored by its centre block s + (e - s) / 2 over the stage's query
// rows (the block's last row and every stride_q-th before it); a stage keeps
// its stage_k / chunk_size best chunks by (score desc, start asc).
//
// Design:
//  * stage_score: one wave of (slices x mask rows) CTAs of 256 threads; an
//    8-lane group scores its chunks' centre blocks: the (chunk, key) pairs
//    run in batches of up to 8 rows that are all requested before the first
//    is used (each lane its 32 bytes of a row, as in the mask kernels), and
//    each row is dotted with the stage's query rows (4 or 8 at a time, held
//    in registers) in the canonical fp32 order of the selection dot (lane l:
//    an fma chain over d-slices l and l + 8, then the fixed add tree across
//    the 8 lanes), so a stage decides on exactly the scores the oracle
//    ranks. Per chunk it reads b_k d-element rows: a gather bound by HBM,
//    spread over every SM.
//  * stage_select: one CTA per mask row, with the row's score keys staged in
//    shared memory (all loads in flight at once). A histogram of 2048
//    buckets linear in the score over [min, max] finds the bucket of the
//    keep-th largest score (a bucket above another holds only larger
//    scores); chunks above it are kept, and its members (a handful) are
//    ranked exactly by (score desc, index asc) -- lists are in start order,
//    so the lowest start wins a tie. A cut bucket of more than 2048 members
//    (heavy ties) falls back to an exact radix select over four 8-bit digits
//    of the order-preserving key. An order-preserving scan (each warp a
//    contiguous run, 32 consecutive chunks at a time) lists the kept chunks
//    in start order; every input chunk but the last has the input
//    granularity, so their pieces (the next stage's chunks) are placed
//    without a scan. A final list is then halved in shared memory for as
//    long as the halves number at most n0 (the iteration's rounds that keep
//    every candidate and so need no scores).
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "hips_common.cuh"
#include "hips_kernels.h"

namespace hips {
namespace {

constexpr int kRowBatch = 32;  // query rows in shared memory at a time
static_assert(kRowBatch % 8 == 0, "rows are dotted 8 at a time");

// The query block, KV head and key range of mask row `unit`
// ((b * mask heads + m) * n_qblocks + qb, as in the mask kernels).
struct RowInfo {
  int b, m, i0, i1;
  int64_t kvh, Tc, N;
};

__device__ __forceinline__ RowInfo row_info(const StageArgs& a, int64_t unit) {
  RowInfo r;
  const int qb = static_cast<int>(unit % a.nqb);
  r.m = static_cast<int>((unit / a.nqb) % a.n_mheads);
  r.b = static_cast<int>(unit / (static_cast<int64_t>(a.nqb) * a.n_mheads));
  r.i0 = qb * a.block_q;
  r.i1 = min(r.i0 + a.block_q, a.q_len);
  r.kvh = static_cast<int64_t>(r.b) * a.kv_heads + r.m / a.kv_div;
  r.Tc = min64(a.q_pos0 + r.i1, a.seq_len);  // one past the block's last row
  r.N = (r.Tc + a.block_k - 1) / a.block_k;
  return r;
}

// Chunks of a mask row's input: the tiling of [0, N) by c_in blocks, or the
// list `in` (count, then starts and ends).
struct Chunks {
  const int32_t* in;
  int c_in, cap;
  int64_t N;
  __device__ __forceinline__ int count() const {
    return in ? in[0] : static_cast<int>((N + c_in - 1) / c_in);
  }
  __device__ __forceinline__ void get(int i, int& s, int& e) const {
    if (in) {
      s = in[4 + i];
      e = in[4 + cap + i];
    } else {
      s = i * c_in;
      e = static_cast<int>(min64(N, static_cast<int64_t>(s) + c_in));
    }
  }
};

__device__ __forceinline__ Chunks row_chunks(const StageArgs& a, int64_t unit, int64_t N) {
  Chunks c;
  c.in = a.c_in > 0 ? nullptr : a.in + unit * a.lstride;
  c.c_in = a.c_in;
  c.cap = a.cap;
  c.N = N;
  return c;
}

// Key rows a group keeps in flight: the raw rows and RC query rows (16
// floats each per lane) share the register budget.
template <typename KvT, int RC>
constexpr int pairs_per_batch() {
  return sizeof(KvT) == 4 ? (RC == 8 ? 2 : 4) : (RC == 8 ? 4 : 8);
}

constexpr int kBoundsTile = 512;  // chunk bounds staged in shared memory at a time

template <typename KvT, int RC>
__global__ void __launch_bounds__(kThreads) stage_score_kernel(const StageArgs a) {
  __shared__ __align__(16) float qs[kRowBatch * kD];
  __shared__ int64_t qpos[kRowBatch];
  __shared__ int bs[kBoundsTile], be[kBoundsTile];
  const int64_t unit = blockIdx.y;
  const RowInfo ri = row_info(a, unit);
  const Chunks ch = row_chunks(a, unit, ri.N);
  const int M = ch.count();
  if (M <= a.keep) return;  // the row keeps every chunk: nothing to rank
  const int per = (M + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  const int lo = static_cast<int>(blockIdx.x) * per, hi = min(M, lo + per);
  if (lo >= hi) return;  // uniform over the CTA
  const int tid = threadIdx.x, l8 = tid & 7;
  const int grp = tid >> 3;  // 8-lane group of the CTA, 0..31
  const int bk = a.block_k, lbk = __ffs(bk) - 1;
  const int npos = (ri.i1 - ri.i0 + a.stride_q - 1) / a.stride_q;
  const int R = a.group * npos;  // rows: head-major, then positions from the last back
  constexpr int kRowB = row_bytes<KvT>();
  constexpr int KB = pairs_per_batch<KvT, RC>();
  const unsigned char* kbase = static_cast<const unsigned char*>(a.k) + ri.kvh * a.kv_cap * kRowB;
  float* out = a.scores + unit * a.cap;
  if (tid == 0 && a.status && blockIdx.x == 0)
    atomicAdd(&a.status->scored, static_cast<unsigned long long>(M));

  for (int r0 = 0; r0 < R; r0 += kRowBatch) {
    const int nr = min(kRowBatch, R - r0);
    const int nrp = (nr + RC - 1) / RC * RC;
    __syncthreads();  // the previous batch's rows are no longer read
    for (int x = tid; x < nrp * kD; x += kThreads) {
      const int r = x / kD, e = x % kD;
      float v = 0.0f;
      int64_t pos = -1;
      if (r < nr) {
        const int rr = r0 + r;
        const int h = ri.m * a.group + rr / npos;
        const int i = ri.i1 - 1 - (rr % npos) * a.stride_q;
        const int64_t off = ((static_cast<int64_t>(ri.b) * a.n_qheads + h) * a.q_len + i) * kD + e;
        if (a.dtype == kDtypeF32)
          v = static_cast<const float*>(a.q)[off];
        else
          v = __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(a.q)[off]) << 16);
        pos = a.q_pos0 + i;
      }
      qs[x] = v;
      if (e == 0) qpos[r] = pos;
    }
    for (int t0 = lo; t0 < hi; t0 += kBoundsTile) {
      const int nt = min(kBoundsTile, hi - t0);
      __syncthreads();  // qs written; the previous tile's bounds are no longer read
      for (int i = tid; i < nt; i += kThreads) ch.get(t0 + i, bs[i], be[i]);
      __syncthreads();
      // group grp scores chunks grp, grp + 32, ... of the tile: its (chunk,
      // key) pairs run in batches of KB rows requested before the first is
      // used. The first group of a warp has the most pairs: its count bounds
      // the loop of the whole warp (the add tree's shuffles need every lane).
      const int npairs = (nt > grp ? (nt - grp + 31) / 32 : 0) << lbk;
      const int gw = grp & ~3;
      const int npw = (nt > gw ? (nt - gw + 31) / 32 : 0) << lbk;
      float run = -INFINITY;  // the current chunk's running max
      for (int p0 = 0; p0 < npw; p0 += KB) {
        Row16<KvT> kr[KB];
        bool jok[KB];
        int64_t jv[KB];
#pragma unroll
        for (int u = 0; u < KB; ++u) {
          const int p = p0 + u;
          const int ci = grp + 32 * (p >> lbk);  // chunk of the tile
          bool ok = p < npairs;
          int64_t j = 0;
          if (ok) {
            const int s = bs[ci], e = be[ci];
            j = (static_cast<int64_t>(s + (e - s) / 2) << lbk) + (p & (bk - 1));  // centre block's key
            ok = j < ri.Tc;
          }
          jok[u] = ok;
          jv[u] = j;
          if (ok) kr[u].load(kbase + j * kRowB, l8);
          else kr[u].zero();
        }
        float best[KB];
#pragma unroll
        for (int u = 0; u < KB; ++u) best[u] = -INFINITY;
        for (int rc = 0; rc < nrp; rc += RC) {
          // RC query rows in registers (this lane's 16 elements of each)
          float qv[RC][16];
#pragma unroll
          for (int w = 0; w < RC; ++w) {
            const float4* qr = reinterpret_cast<const float4*>(qs + (rc + w) * kD);
            const float4 q0 = qr[2 * l8], q1 = qr[2 * l8 + 1];
            const float4 q2 = qr[16 + 2 * l8], q3 = qr[16 + 2 * l8 + 1];
            qv[w][0] = q0.x; qv[w][1] = q0.y; qv[w][2] = q0.z; qv[w][3] = q0.w;
            qv[w][4] = q1.x; qv[w][5] = q1.y; qv[w][6] = q1.z; qv[w][7] = q1.w;
            qv[w][8] = q2.x; qv[w][9] = q2.y; qv[w][10] = q2.z; qv[w][11] = q2.w;
            qv[w][12] = q3.x; qv[w][13] = q3.y; qv[w][14] = q3.z; qv[w][15] = q3.w;
          }
          const int r = rc + group_row_of_lane<RC>(l8);  // the row whose dot this lane ends with
          const bool rok = r < nr;
          const int64_t rpos = qpos[r];
#pragma unroll
          for (int u = 0; u < KB; ++u) {
            float x[16];
            kr[u].get(x);
            float part[RC];
#pragma unroll
            for (int w = 0; w < RC; ++w) {
              float acc = 0.0f;
#pragma unroll
              for (int e = 0; e < 16; ++e) acc = __fmaf_rn(qv[w][e], x[e], acc);
              part[w] = acc;
            }
            const float dot = group_reduce_rows<RC>(part, l8);
            if (jok[u] && rok && jv[u] <= rpos) best[u] = fmaxf(best[u], dot);
          }
        }
#pragma unroll
        for (int u = 0; u < KB; ++u) {
          const int p = p0 + u;
          const int t = p & (bk - 1);
          if (t == 0) run = -INFINITY;
          run = fmaxf(run, best[u]);
          if (t == bk - 1) {  // the chunk's last key: its score (max over the group)
            float m = fmaxf(run, __shfl_xor_sync(0xffffffffu, run, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            const int c = t0 + grp + 32 * (p >> lbk);
            // the same lane writes chunk c in every row batch
            if (p < npairs && l8 == 0) out[c] = r0 == 0 ? m : fmaxf(out[c], m);
          }
        }
      }
    }
  }
}

// Order-preserving placement over elements [0, n): element i asks for
// count(i) slots; emit(i, pos) is called for every element with a nonzero
// count, pos being the sum of the counts of the elements before it. Warp w
// walks the contiguous run [w pw, (w + 1) pw) 32 consecutive elements at a
// time (lane l the l-th: conflict-free shared-memory reads); total gets the
// sum. Every thread of the CTA must call it.
template <typename CountF, typename EmitF>
__device__ __forceinline__ void ordered_emit(int n, CountF count, EmitF emit, int* scratch,
                                             int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int pw = ((n + kWarps - 1) / kWarps + 31) & ~31;
  const int lo = min(n, warp * pw), hi = min(n, lo + pw);
  int wsum = 0;
  for (int b0 = lo; b0 < hi; b0 += 32) {
    const int i = b0 + lane;
    wsum += __reduce_add_sync(0xffffffffu, i < hi ? count(i) : 0);
  }
  if (lane == 0) scratch[warp] = wsum;
  __syncthreads();
  int off = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int v = scratch[w];
    off += w < warp ? v : 0;
    total += v;
  }
  __syncthreads();  // scratch is free again
  for (int b0 = lo; b0 < hi; b0 += 32) {
    const int i = b0 + lane;
    const int c = i < hi ? count(i) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (c) emit(i, off + incl - c);
    off += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// Inverse of score_key: the score a key orders.
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// kept[i] = 1 for the `keep` largest keys of [0, n), ties at the cut to the
// lowest indices (the rule (score desc, start asc) on a start-ordered list).
// Value buckets: 2048 buckets linear in the score over [min, max] (the bucket
// of a score never decreases with the score, so a bucket above another holds
// only larger scores); the bucket of the keep-th largest is found from a
// histogram, and its members are ranked exactly. Returns false, having
// decided nothing, when that bucket holds more than kBand chunks (heavy
// ties): the caller then ranks by digits. hb (2048 ints) and mem (kBand ints)
// are shared-memory scratch.
constexpr int kSelBuckets = 2048;
constexpr int kBand = 2048;

__device__ bool bucket_select(const uint32_t* key, uint8_t* kept, int n, int keep, int* hist256,
                              int* scratch, int* hb, int* mem) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  (void)hist256;
  float mn = INFINITY, mx = -INFINITY;
  for (int i = tid; i < n; i += kThreads) {
    const float f = key_score(key[i]);
    mn = fminf(mn, f);
    mx = fmaxf(mx, f);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  float* fscr = reinterpret_cast<float*>(scratch);
  if (lane == 0) {
    fscr[warp] = mn;
    fscr[kWarps + warp] = mx;
  }
  for (int i = tid; i < kSelBuckets; i += kThreads) hb[i] = 0;
  __syncthreads();
  mn = fscr[0];
  mx = fscr[kWarps];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) {
    mn = fminf(mn, fscr[w]);
    mx = fmaxf(mx, fscr[kWarps + w]);
  }
  const float scale = mx > mn ? static_cast<float>(kSelBuckets - 1) / (mx - mn) : 0.0f;
  auto bucket = [&](uint32_t k) {
    return min(max(static_cast<int>((key_score(k) - mn) * scale), 0), kSelBuckets - 1);
  };
  for (int i = tid; i < n; i += kThreads) atomicAdd(&hb[bucket(key[i])], 1);
  __syncthreads();
  // the cut bucket, from the top: thread t sums buckets 2047 - 8t ... 2040 - 8t
  int c[8], sum = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    c[q] = hb[kSelBuckets - 1 - 8 * tid - q];
    sum += c[q];
  }
  int tot;
  const int excl = block_excl_scan(sum, scratch, tot);
  if (excl < keep && keep <= excl + sum) {
    int acc = excl;
    for (int q = 0; q < 8; ++q) {
      if (acc + c[q] >= keep) {
        scratch[48] = kSelBuckets - 1 - 8 * tid - q;  // the cut bucket
        scratch[49] = keep - acc;                      // kept from it
        scratch[50] = c[q];                            // its members
        scratch[51] = 0;
        break;
      }
      acc += c[q];
    }
  }
  __syncthreads();
  const int cut = scratch[48], need = scratch[49], nmem = scratch[50];
  if (nmem > kBand) return false;  // uniform
  for (int i = tid; i < n; i += kThreads) {
    const int bi = bucket(key[i]);
    kept[i] = bi > cut ? 1 : 0;
    if (bi == cut) mem[atomicAdd(&scratch[51], 1)] = i;
  }
  __syncthreads();
  // exact rank of each member among the members: (key desc, index asc)
  for (int m = tid; m < nmem; m += kThreads) {
    const int i = mem[m];
    const uint32_t ki = key[i];
    int r = 0;
    for (int x = 0; x < nmem; ++x) {
      const int j = mem[x];
      const uint32_t kj = key[j];
      r += (kj > ki || (kj == ki && j < i)) ? 1 : 0;
    }
    kept[i] = r < need ? 1 : 0;
  }
  return true;
}

// The same selection by the digits of the keys (four 8-bit passes, most
// significant first): exact whatever the ties, slower where scores crowd
// into a few digits.
__device__ void radix_select(const uint32_t* key, uint8_t* kept, int n, int keep, int* hist,
                             int* scratch) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0u, pmask = 0u;
  int need = keep;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t k = key[i];
      if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255 - 8l ... 248 - 8l (from the top)
      int c[8], sum = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        c[q] = hist[255 - 8 * lane - q];
        sum += c[q];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - sum;
      if (excl < need && need <= incl) {
        int acc = excl;
        for (int q = 0; q < 8; ++q) {
          if (acc + c[q] >= need) {
            scratch[0] = 255 - 8 * lane - q;
            scratch[1] = need - acc;
            break;
          }
          acc += c[q];
        }
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(scratch[0]) << shift;
    pmask |= 255u << shift;
    need = scratch[1];
    __syncthreads();
  }
  const uint32_t thr = prefix;
  for (int i = tid; i < n; i += kThreads) kept[i] = key[i] > thr ? 1 : 0;
  __syncthreads();
  int neq;
  ordered_emit(
      n, [&](int i) { return key[i] == thr ? 1 : 0; },
      [&](int i, int pos) { kept[i] = pos < need ? 1 : 0; }, scratch, neq);
}

// Selection of one mask row. The score keys of its chunks (4 bytes each) and
// their kept flags (1 byte) sit in shared memory; the chunk bounds are read
// where they lie (computed for a tiling, from the list otherwise) for the
// kept chunks only.
constexpr int kSelStaged = kStageMaxChunks;  // chunks of one selection, at most
constexpr int kSelDyn = 5 * kSelStaged;

__global__ void __launch_bounds__(kThreads) stage_select_kernel(const StageArgs a) {
  extern __shared__ __align__(16) uint32_t skey[];
  uint8_t* kbit = reinterpret_cast<uint8_t*>(skey + kSelStaged);
  __shared__ int hist[256];
  __shared__ int scratch[64];
  __shared__ int fs[2][kMaxN0];
  __shared__ int fe[2][kMaxN0];
  const int64_t unit = blockIdx.x;
  const RowInfo ri = row_info(a, unit);
  const Chunks ch = row_chunks(a, unit, ri.N);
  const int tid = threadIdx.x;
  const int M = ch.count();
  const int n0 = static_cast<int>(min64(a.n0max, ri.N));
  int32_t* o = a.out + unit * a.lstride;
  if (M > kSelStaged) {  // beyond the planned bound: report and write an empty row
    if (tid == 0) {
      report(a.status, kStatusBound, 0x5e0u);
      o[0] = 0; o[1] = 0; o[2] = 0; o[3] = 0;
    }
    return;
  }
  const bool ranked = a.keep > 0 && M > a.keep;
  if (ranked) {
    const float* sc = a.scores + unit * a.cap;
#pragma unroll 4
    for (int i = tid; i < M; i += kThreads) skey[i] = score_key(sc[i]);
    __syncthreads();
    // ---- kept: the keep best keys; ties at the cut go to the lowest indices
    if (!bucket_select(skey, kbit, M, a.keep, hist, scratch, fs[0], fe[0]))
      radix_select(skey, kbit, M, a.keep, hist, scratch);
    __syncthreads();
  }

  // ---- the kept chunks in start order (their indices replace the keys),
  // then their pieces of c_out blocks: every input chunk has c_list blocks
  // but the last one (chunks are aligned pieces of aligned chunks, so only
  // the one that holds block N - 1 can be clipped, and lists are in start
  // order), so kept chunk r's pieces start at r * full
  int* kidx = reinterpret_cast<int*>(skey);
  int nkept;
  ordered_emit(
      M, [&](int i) { return !ranked || kbit[i] ? 1 : 0; },
      [&](int i, int r) { kidx[r] = i; }, scratch, nkept);
  __syncthreads();
  const int co = a.c_out;
  int last_len;
  {
    int s0, e0;
    ch.get(M - 1, s0, e0);
    last_len = e0 - s0;
  }
  const int full = (a.c_list + co - 1) / co, last = (last_len + co - 1) / co;
  const bool last_kept = nkept > 0 && kidx[nkept - 1] == M - 1;
  const int ptot = last_kept ? (nkept - 1) * full + last : nkept * full;
  int* ps = a.final_list ? fs[0] : o + 4;
  int* pe = a.final_list ? fe[0] : o + 4 + a.cap;
  const int lim = a.final_list ? min(a.cap, kMaxN0) : a.cap;
  if (ptot > lim) {  // the planned bound was wrong: report and write an empty row
    if (tid == 0) {
      report(a.status, kStatusBound, 0x5e1u);
      o[0] = 0; o[1] = 0; o[2] = 0; o[3] = 0;
    }
    return;
  }
  __syncthreads();  // fs/fe (the bucket select's scratch) are free again
  for (int r = tid; r < nkept; r += kThreads) {
    int s0, e0;
    ch.get(kidx[r], s0, e0);
    int pos = r * full;
    for (int p = s0; p < e0; p += co, ++pos) {
      ps[pos] = p;
      pe[pos] = min(p + co, e0);
    }
  }
  if (!a.final_list) {
    if (tid == 0) { o[0] = ptot; o[1] = 0; o[2] = 0; o[3] = 0; }
    return;
  }

  // ---- the iteration's rounds that keep every candidate: halve while the
  // halves (one-block chunks stay whole) number at most n0
  int cur = 0, cnt = ptot;
  for (;;) {
    __syncthreads();
    int mine_long = 0;
    for (int i = tid; i < cnt; i += kThreads) mine_long |= fe[cur][i] - fs[cur][i] > 1 ? 1 : 0;
    if (!__syncthreads_or(mine_long)) break;
    int nh;
    const int* cs = fs[cur];
    const int* cz = fe[cur];
    int* ns = fs[cur ^ 1];
    int* nz = fe[cur ^ 1];
    // count first: halving past n0 candidates is a round that ranks
    ordered_emit(
        cnt, [&](int i) { return cz[i] - cs[i] > 1 ? 2 : 1; },
        [&](int i, int pos) {
          const int s0 = cs[i], e0 = cz[i];
          if (pos + 1 < kMaxN0 && e0 - s0 > 1) {
            const int m = s0 + (e0 - s0) / 2;
            ns[pos] = s0; nz[pos] = m;
            ns[pos + 1] = m; nz[pos + 1] = e0;
          } else if (pos < kMaxN0 && e0 - s0 <= 1) {
            ns[pos] = s0; nz[pos] = e0;
          }
        },
        scratch, nh);
    if (nh > n0) break;  // the written halves are discarded: cur keeps the chunks
    cur ^= 1;
    cnt = nh;
  }
  __syncthreads();
  int blocks = 0;
  for (int i = tid; i < cnt; i += kThreads) {
    o[4 + i] = fs[cur][i];
    o[4 + a.cap + i] = fe[cur][i];
    blocks += fe[cur][i] - fs[cur][i];
  }
  int total;
  (void)block_excl_scan(blocks, scratch, total);
  if (tid == 0) {
    o[0] = cnt;
    o[1] = min(n0, total);  // the chunks every round keeps, and the final count
    o[2] = 0;
    o[3] = 0;
  }
}

}  // namespace

template <typename KvT>
void launch_score_t(const StageArgs& a, dim3 grid, cudaStream_t stream) {
  // rows of a stage: the mask's heads at its strided positions
  const int rows = a.group * ((std::min(a.block_q, a.q_len) + a.stride_q - 1) / a.stride_q);
  if (rows <= 4) stage_score_kernel<KvT, 4><<<grid, kThreads, 0, stream>>>(a);
  else stage_score_kernel<KvT, 8><<<grid, kThreads, 0, stream>>>(a);
}

cudaError_t launch_stage_score(const StageArgs& a, cudaStream_t stream) {
  const dim3 grid(a.slices, static_cast<unsigned>(a.units));
  switch (a.dtype) {
    case kDtypeF32: launch_score_t<float>(a, grid, stream); break;
    case kDtypeBf16: launch_score_t<uint16_t>(a, grid, stream); break;
    case kDtypeBf16E5m2: launch_score_t<uint8_t>(a, grid, stream); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_stage_select(const StageArgs& a, cudaStream_t stream) {
  // score keys and kept flags: 5 bytes per chunk (the attribute is set once
  // per device)
  constexpr int kDyn = kSelDyn;
  static std::once_flag done[kMaxDevices];
  static cudaError_t status[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(done[dev], [&] {
    status[dev] = cudaFuncSetAttribute(stage_select_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kDyn);
  });
  if (status[dev] != cudaSuccess) return status[dev];
  stage_select_kernel<<<static_cast<unsigned>(a.units), kThreads, kDyn, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace hips
