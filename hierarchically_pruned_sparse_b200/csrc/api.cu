// C ABI of libhip_sparse.so: argument validation, launch planning, dispatch.
// Every entry point validates on the host before launching anything and
// launches only on params->stream; nothing here allocates device memory.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "hip_sparse.h"
#include "hips_common.cuh"
#include "hips_kernels.h"
#include "widen.h"

static_assert(HIPS_F32 == hips::kDtypeF32 && HIPS_BF16 == hips::kDtypeBf16 &&
                  HIPS_BF16_E5M2 == hips::kDtypeBf16E5m2,
              "kernel dtype codes follow enum hips_dtype");

namespace {

thread_local int g_last_cuda_error = 0;

constexpr int kPlanSMs = 148;         // B200 streaming multiprocessors
using hips::kStatusBytes;             // workspace head layout (hips_kernels.h)
using hips::kCounterOffset;
using hips::kMaxCounters;
constexpr int kMaxSmem = 227 * 1024;

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int validate(const hips_params* p, int op) {
  if (!p) return HIPS_ERR_INVALID_ARG;
  if (p->batch <= 0 || p->n_qheads <= 0 || p->n_kvheads <= 0) return HIPS_ERR_INVALID_ARG;
  if (p->n_qheads % p->n_kvheads) return HIPS_ERR_INVALID_ARG;
  if (p->head_dim != hips::kD) return HIPS_ERR_UNSUPPORTED;
  if (p->dtype != HIPS_F32 && p->dtype != HIPS_BF16 && p->dtype != HIPS_BF16_E5M2)
    return HIPS_ERR_UNSUPPORTED;
  if (p->flags & ~HIPS_FLAG_HEAD_MASKS) return HIPS_ERR_INVALID_ARG;
  if (p->seq_len <= 0 || p->seq_len >= (int64_t{1} << 31)) return HIPS_ERR_INVALID_ARG;
  if (p->kv_capacity < p->seq_len) return HIPS_ERR_INVALID_ARG;
  if (p->q_len <= 0 || p->q_pos0 < 0 || p->q_pos0 + p->q_len > p->seq_len) return HIPS_ERR_INVALID_ARG;
  if (op != HIPS_OP_DENSE) {
    if (p->mask_len <= 0 || p->mask_len > p->seq_len) return HIPS_ERR_INVALID_ARG;
    if (p->block_q <= 0 || !is_pow2(p->block_k)) return HIPS_ERR_INVALID_ARG;
    if (p->topk < p->block_k || p->topk % p->block_k) return HIPS_ERR_INVALID_ARG;
    if (p->sink < 0 || p->window < 0) return HIPS_ERR_INVALID_ARG;
    if (p->topk / p->block_k > hips::kMaxN0) return HIPS_ERR_UNSUPPORTED;
  }
  const double elems = static_cast<double>(p->batch) * p->n_kvheads * p->kv_capacity * p->head_dim;
  if (elems > 4.0e18) return HIPS_ERR_INVALID_ARG;
  if (op == HIPS_OP_MASK || op == HIPS_OP_MASK_SPARSE) {
    // pruning stages (struct hips_stage): sizes in whole blocks, each
    // dividing the one before, kept keys in whole chunks
    if (p->n_stages < 0 || p->n_stages > HIPS_MAX_STAGES) return HIPS_ERR_INVALID_ARG;
    if (p->n_stages > 0 && !p->stages) return HIPS_ERR_INVALID_ARG;
    for (int i = 0; i < p->n_stages; ++i) {
      const hips_stage& g = p->stages[i];
      if (g.chunk_size <= 0 || g.chunk_size % p->block_k || g.stride_q < 1) return HIPS_ERR_INVALID_ARG;
      if (g.stage_k < 0 || g.stage_k % g.chunk_size) return HIPS_ERR_INVALID_ARG;
      if (i > 0 && p->stages[i - 1].chunk_size % g.chunk_size) return HIPS_ERR_INVALID_ARG;
    }
  }
  return HIPS_OK;
}

int64_t row_stride(const hips_params* p) {
  const int64_t bk = p->block_k;
  int64_t cap = p->topk / bk + cdiv(p->sink, bk);
  if (p->window > 0) cap += cdiv(static_cast<int64_t>(p->window) + p->block_q - 1, bk) + 1;
  return 1 + cap;
}

// One mask per query head, or one per KV-head group (the default).
bool head_masks(const hips_params* p) { return (p->flags & HIPS_FLAG_HEAD_MASKS) != 0; }
// Heads that own an idx row, and query heads per such head.
int mask_heads(const hips_params* p) { return head_masks(p) ? p->n_qheads : p->n_kvheads; }
int mask_group(const hips_params* p) { return head_masks(p) ? 1 : p->n_qheads / p->n_kvheads; }
int kv_div(const hips_params* p) { return head_masks(p) ? p->n_qheads / p->n_kvheads : 1; }

int group_rows(const hips_params* p, int block_q) {
  return mask_group(p) * std::min(block_q, p->q_len);
}

// ---------------------------------------------------------------- mask plan

// The pruning stages of a mask call (struct hips_stage): one step per stage
// that ranks (stage_k > 0), each a scoring launch and a selection launch
// per mask row; with no ranking stage, one selection step that only cuts and
// halves. The last step writes the iteration's initial chunk lists.
struct StageStep {
  int c_in;     // > 0: the input is the tiling of [0, N) by c_in blocks; 0: the previous list
  int keep;     // chunks a row keeps (0: all, nothing scored)
  int stride_q;
  int c_out;    // blocks per output piece
  bool final_list;
};

struct StagePlan {
  int nsteps;
  StageStep steps[HIPS_MAX_STAGES + 1];
  int cap;          // entries of a list (and scores per row)
  int64_t lstride;  // int32 per row of a list
  size_t bytes;     // scores, then two lists, each 256-byte aligned
};

struct MaskPlan {
  hips::MaskArgs a;
  int smem;
  size_t ws;
  StagePlan stp;
  size_t st_off;  // workspace offset of the stage buffers
  bool mma;  // tensor-core kernel (bf16 or e5m2 keys) or CUDA-core kernel
  bool norms;  // key-block norm pre-pass into the workspace (many-row masks)
  bool decode;  // the decode kernel (one query position per mask row)
};

// Decode plan: e5m2 keys, one query position per mask row (b_q = 1, or a
// single query row) with at most decode_max_rows() query rows. A cluster
// of C CTAs per mask row (C the largest size with every row resident at once,
// at least 8 candidates per CTA); the attention, when asked for, runs in the
// same launch.
int plan_decode(const hips_params* p, int cluster_cap, bool attend, MaskPlan* plan) {
  hips::MaskArgs& a = plan->a;
  if (p->dtype != HIPS_BF16_E5M2 || !(p->q_len == 1 || p->block_q == 1) ||
      a.rows_max > hips::decode_max_rows() || a.units > 65535)
    return HIPS_ERR_UNSUPPORTED;
  const int64_t ncand = 2 * static_cast<int64_t>(a.n0max);
  int c = 1;
  for (int t = std::min(cluster_cap, 16); t > 1; --t) {
    if (a.units * t <= kPlanSMs && cdiv(ncand, t) >= 8) {
      c = t;
      break;
    }
  }
  a.cluster = c;
  a.per_cta = static_cast<int>(cdiv(cdiv(ncand, c), 8) * 8);
  a.rows_pad = a.rows_max;
  a.stages = 0;
  plan->smem = hips::decode_smem_bytes(a, attend, kMaxSmem);
  if (plan->smem > kMaxSmem) return HIPS_ERR_UNSUPPORTED;
  plan->decode = true;
  plan->mma = false;
  plan->norms = false;
  plan->ws = kStatusBytes;
  return HIPS_OK;
}

// Tensor-core mask plan: bf16 keys with up to 256 query rows per mask, or
// e5m2 keys with up to 16 (one MMA column block); b_k <= 32.
int plan_mask_mma(const hips_params* p, int cluster_cap, MaskPlan* plan) {
  hips::MaskArgs& a = plan->a;
  const int nc = hips::mask_mma_nc(a.rows_max);
  const bool kv8 = p->dtype == HIPS_BF16_E5M2;
  if ((p->dtype != HIPS_BF16 && !kv8) || nc == 0 || p->block_k > 32 || a.units > 65535)
    return HIPS_ERR_UNSUPPORTED;
  if (kv8 && nc != 1) return HIPS_ERR_UNSUPPORTED;  // e5m2 keys: one MMA column block
  const int cpt = hips::mask_mma_tile_keys() / p->block_k;
  const int64_t ncand = 2 * static_cast<int64_t>(a.n0max);
  // the largest cluster (any size up to the cap) with one CTA per SM for all
  // units and at least one full tile of candidates per CTA
  int c = 1;
  for (int t = std::min(cluster_cap, 16); t > 1; --t) {
    if (a.units * t <= kPlanSMs && cdiv(ncand, t) >= cpt) {
      c = t;
      break;
    }
  }
  a.cluster = c;
  a.per_cta = static_cast<int>(cdiv(ncand, c));
  a.rows_pad = nc * 16;
  a.stages = 0;
  plan->smem = hips::mask_mma_smem_bytes(nc, a.n0max, a.per_cta, c, kv8);
  if (plan->smem > kMaxSmem) return HIPS_ERR_UNSUPPORTED;
  plan->mma = true;
  plan->ws = kStatusBytes;
  plan->norms = false;
  if (nc >= 4) {
    // many query rows per mask (prefill): the scoring kernel reads the key
    // norms that bound its tensor-core rounding from a pre-pass over K
    a.knorm_stride = cdiv(p->seq_len, p->block_k);
    const size_t bytes = static_cast<size_t>(p->batch) * p->n_kvheads * a.knorm_stride * sizeof(float);
    plan->ws = kStatusBytes + (bytes + 255) / 256 * 256;
    plan->norms = true;
  }
  return HIPS_OK;
}

int plan_mask_kernel(const hips_params* p, int cluster_cap, MaskPlan* plan, bool attend) {
  hips::MaskArgs& a = plan->a;
  a = hips::MaskArgs{};
  plan->decode = false;
  a.dtype = p->dtype;
  a.n_qheads = p->n_qheads;
  a.n_kvheads = mask_heads(p);
  a.group = mask_group(p);
  a.kv_heads = p->n_kvheads;
  a.kv_div = kv_div(p);
  a.q_len = p->q_len;
  a.block_q = p->block_q;
  a.block_k = p->block_k;
  a.n0max = p->topk / p->block_k;
  a.sink = p->sink;
  a.window = p->window;
  a.nqb = static_cast<int>(cdiv(p->q_len, p->block_q));
  a.units = static_cast<int64_t>(p->batch) * mask_heads(p) * a.nqb;
  a.seq_len = p->seq_len;
  a.kv_cap = p->kv_capacity;
  a.q_pos0 = p->q_pos0;
  a.row_stride = row_stride(p);
  a.rows_max = group_rows(p, p->block_q);
  plan->mma = false;
  plan->norms = false;
  // The tensor-core mask kernel first: it is the faster one wherever it
  // plans (measured at 128k and 1M keys, one and 16 sequences). The decode
  // kernel serves the e5m2 decode shapes it cannot plan (budgets whose
  // candidate lists outgrow its shared memory).
  if (plan_mask_mma(p, cluster_cap, plan) == HIPS_OK) return HIPS_OK;
  if (plan_decode(p, cluster_cap, attend, plan) == HIPS_OK) return HIPS_OK;
  plan->decode = false;
  if (p->dtype == HIPS_BF16_E5M2) return HIPS_ERR_UNSUPPORTED;  // no other e5m2 mask
  if (a.rows_max > 32 || a.units > 65535) return HIPS_ERR_UNSUPPORTED;
  const int rc = hips::mask_fma_rc(a.rows_max);
  a.rows_pad = static_cast<int>(cdiv(a.rows_max, rc) * rc);
  const int tile_keys = hips::mask_fma_tile_keys(p->dtype);
  if (p->block_k > tile_keys) return HIPS_ERR_UNSUPPORTED;
  const int cpt = tile_keys / p->block_k;
  const int64_t ncand = 2 * static_cast<int64_t>(a.n0max);
  int c = 1;
  while (2 * c <= cluster_cap && a.units * (2 * c) <= kPlanSMs && cdiv(ncand, 2 * c) >= cpt) c *= 2;
  a.cluster = c;
  a.per_cta = static_cast<int>(cdiv(ncand, c));
  a.stages = 3;
  plan->smem = hips::mask_fma_smem_bytes(a.n0max, a.rows_pad, a.per_cta, c, a.stages);
  if (plan->smem > kMaxSmem) {
    a.stages = 2;
    plan->smem = hips::mask_fma_smem_bytes(a.n0max, a.rows_pad, a.per_cta, c, a.stages);
  }
  if (plan->smem > kMaxSmem) return HIPS_ERR_UNSUPPORTED;
  plan->ws = kStatusBytes;
  return HIPS_OK;
}

// Steps and buffers of the pruning stages, with bounds taken over every mask
// row: the first ranking stage has at most ceil(N / c) chunks, a later one at
// most (the chunks kept before) x (their size / its size), each at most
// kStageMaxChunks; the iteration must start from at most n0max chunks.
int plan_stages(const hips_params* p, int64_t units, StagePlan* sp) {
  sp->nsteps = 0;
  sp->bytes = 0;
  sp->cap = 0;
  sp->lstride = 0;
  if (p->n_stages == 0) return HIPS_OK;
  const int64_t bk = p->block_k;
  const int64_t nmax = cdiv(std::min<int64_t>(p->q_pos0 + p->q_len, p->seq_len), bk);
  const int64_t n0max = p->topk / bk;
  const hips_stage* st = p->stages;
  const int S = p->n_stages;
  int ranked[HIPS_MAX_STAGES];
  int nr = 0;
  for (int i = 0; i < S; ++i)
    if (st[i].stage_k > 0) ranked[nr++] = i;
  const int64_t c_last = st[S - 1].chunk_size / bk;
  int64_t cap = n0max, kept = 0, kept_c = 1;
  for (int t = 0; t < nr; ++t) {
    const hips_stage& g = st[ranked[t]];
    const int64_t c = g.chunk_size / bk;
    const int64_t cands = t == 0 ? cdiv(nmax, c) : kept * (kept_c / c);
    const int64_t keep = g.stage_k / g.chunk_size;
    if (cands > hips::kStageMaxChunks) return HIPS_ERR_UNSUPPORTED;
    cap = std::max(cap, cands);
    StageStep& step = sp->steps[sp->nsteps++];
    step.c_in = t == 0 ? static_cast<int>(c) : 0;
    step.keep = static_cast<int>(std::min<int64_t>(keep, 1 << 30));
    step.stride_q = g.stride_q;
    step.final_list = t + 1 == nr;
    step.c_out = static_cast<int>(step.final_list ? c_last : st[ranked[t + 1]].chunk_size / bk);
    kept = std::min(keep, cands);
    kept_c = c;
  }
  int64_t pieces;
  if (nr == 0) {
    StageStep& step = sp->steps[sp->nsteps++];
    step = StageStep{static_cast<int>(c_last), 0, 1, static_cast<int>(c_last), true};
    pieces = cdiv(nmax, c_last);
  } else {
    pieces = kept * (kept_c / c_last);
  }
  if (pieces > n0max) return HIPS_ERR_UNSUPPORTED;
  cap = std::max(cap, pieces);
  if (cap > (int64_t{1} << 22)) return HIPS_ERR_UNSUPPORTED;
  sp->cap = static_cast<int>(cap);
  sp->lstride = 4 + 2 * cap;
  const size_t scores = (static_cast<size_t>(units) * cap * sizeof(float) + 255) / 256 * 256;
  const size_t list = (static_cast<size_t>(units) * sp->lstride * sizeof(int32_t) + 255) / 256 * 256;
  sp->bytes = scores + 2 * list;
  return HIPS_OK;
}

int plan_mask(const hips_params* p, int cluster_cap, MaskPlan* plan, bool attend = false) {
  int st = plan_mask_kernel(p, cluster_cap, plan, attend);
  if (st) return st;
  st = plan_stages(p, plan->a.units, &plan->stp);
  if (st) return st;
  plan->st_off = (plan->ws + 255) / 256 * 256;
  if (plan->stp.nsteps) plan->ws = plan->st_off + plan->stp.bytes;
  return HIPS_OK;
}

// Clusters of this plan's shape that fit on the device at once, cached per
// device and shape (queried once, outside any stream capture in practice).
int resident_clusters(const MaskPlan& plan) {
  struct Entry { int dev, dtype, rows, cluster, smem, n; };
  static std::mutex mu;  // host threads may plan concurrently
  std::lock_guard<std::mutex> lock(mu);
  static Entry cache[64];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  const hips::MaskArgs& a = plan.a;
  const int rows = plan.decode ? 200 + a.rows_max
                   : plan.mma  ? 100 + hips::mask_mma_nc(a.rows_max)
                               : hips::mask_fma_rc(a.rows_max);
  for (int i = 0; i < used; ++i) {
    const Entry& e = cache[i];
    if (e.dev == dev && e.dtype == a.dtype && e.rows == rows && e.cluster == a.cluster &&
        e.smem == plan.smem)
      return e.n;
  }
  const int n = plan.decode ? hips::decode_max_active_clusters(a, plan.smem)
                : plan.mma  ? hips::mask_mma_max_active_clusters(a, plan.smem)
                            : hips::mask_fma_max_active_clusters(a, plan.smem);
  if (used < 64) cache[used++] = Entry{dev, a.dtype, rows, a.cluster, plan.smem, n};
  return n;
}

// ---------------------------------------------------------------- attention plan

struct AttnPlan {
  hips::AttnArgs a;
  int smem;
  size_t ws;
  bool mma;  // tensor-core kernel (query blocks, bf16) or CUDA-core split-K kernel
};

// Tensor-core plan: bf16 query blocks of more than 8 rows (a CTA per 128 rows
// of a block, every key of the row list in one CTA).
int plan_attn_mma(const hips_params* p, bool dense, AttnPlan* plan) {
  hips::AttnArgs& a = plan->a;
  if (p->dtype != HIPS_BF16 || a.rows_max <= 8) return HIPS_ERR_UNSUPPORTED;
  a.item_keys = dense ? 16 : p->block_k;
  if (a.item_keys > hips::attn_mma_tile_keys()) return HIPS_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(a.nqb) * a.n_kvheads > 65535 || p->batch > 65535) return HIPS_ERR_UNSUPPORTED;
  int64_t items;
  if (dense) {
    items = cdiv(std::min<int64_t>(p->q_pos0 + p->q_len, p->seq_len), a.item_keys);
  } else {
    items = (a.row_stride - 1) + cdiv(std::max<int64_t>(0, p->seq_len - p->mask_len), a.item_keys);
  }
  if (items > (1 << 20)) return HIPS_ERR_UNSUPPORTED;
  a.table_items = static_cast<int>(items);
  a.nsplit = 1;
  plan->smem = hips::attn_mma_smem_bytes(a.table_items);
  if (plan->smem > kMaxSmem) return HIPS_ERR_UNSUPPORTED;
  plan->mma = true;
  plan->ws = kStatusBytes;
  return HIPS_OK;
}

int plan_attn(const hips_params* p, bool dense, AttnPlan* plan) {
  hips::AttnArgs& a = plan->a;
  a = hips::AttnArgs{};
  plan->mma = false;
  // dense prefill (bf16) runs on the tensor-core kernel in 64-row query blocks
  const bool dense_blocks = dense && p->dtype == HIPS_BF16 && p->q_len >= 64;
  const int block_q = dense ? (dense_blocks ? 64 : 1) : p->block_q;
  a.dtype = p->dtype;
  a.batch = p->batch;
  a.n_qheads = p->n_qheads;
  // a dense call has no masks: its query heads always share their KV head's tiles
  const bool per_head = head_masks(p) && !dense;
  a.n_kvheads = per_head ? p->n_qheads : p->n_kvheads;
  a.group = per_head ? 1 : p->n_qheads / p->n_kvheads;
  a.kv_heads = p->n_kvheads;
  a.kv_div = per_head ? p->n_qheads / p->n_kvheads : 1;
  a.q_len = p->q_len;
  a.block_q = block_q;
  a.nqb = static_cast<int>(cdiv(p->q_len, block_q));
  a.dense = dense ? 1 : 0;
  a.rows_max = a.group * std::min(block_q, p->q_len);
  a.seq_len = p->seq_len;
  a.mask_len = dense ? p->seq_len : p->mask_len;
  a.kv_cap = p->kv_capacity;
  a.q_pos0 = p->q_pos0;
  a.row_stride = dense ? 0 : row_stride(p);
  a.rows_total = static_cast<int64_t>(p->batch) * p->n_qheads * p->q_len;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / 11.313708498984761);  // log2(e)/sqrt(128)
  if (plan_attn_mma(p, dense, plan) == HIPS_OK) return HIPS_OK;
  if (a.rows_max > 8) return HIPS_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(a.nqb) * a.n_kvheads > 65535 || p->batch > 65535) return HIPS_ERR_UNSUPPORTED;
  a.item_keys = dense ? 16 : p->block_k;
  const int tile_keys = hips::attn_fma_tile_keys(p->dtype);
  if (a.item_keys > tile_keys) return HIPS_ERR_UNSUPPORTED;
  const int ipt = tile_keys / a.item_keys;
  int64_t w_max;
  if (dense) {
    w_max = cdiv(std::min<int64_t>(p->q_pos0 + p->q_len, p->seq_len), a.item_keys);
  } else {
    w_max = (a.row_stride - 1) + cdiv(std::max<int64_t>(0, p->seq_len - p->mask_len), a.item_keys);
  }
  const int64_t units = static_cast<int64_t>(p->batch) * a.n_kvheads * a.nqb;
  // one wave: splits x units <= SMs (one CTA per SM), at least a tile per split
  int64_t nsplit = std::min<int64_t>(kPlanSMs / units, cdiv(w_max, ipt));
  nsplit = std::max<int64_t>(1, nsplit);
  if (nsplit > 1 && units > kMaxCounters) nsplit = 1;
  a.nsplit = static_cast<int>(nsplit);
  a.table_items = dense ? 0 : static_cast<int>(cdiv(w_max, nsplit));
  plan->smem = hips::attn_fma_smem_bytes(p->dtype, a.rows_max, a.table_items);
  if (plan->smem > kMaxSmem) return HIPS_ERR_UNSUPPORTED;
  size_t part = 0;
  if (a.nsplit > 1) part = static_cast<size_t>(a.rows_total) * a.nsplit * (hips::kD + 4) * sizeof(float);
  plan->ws = kStatusBytes + (part + 255) / 256 * 256;
  return HIPS_OK;
}

int check_workspace(const hips_params* p, size_t need) {
  if (!p->workspace || !aligned(p->workspace, 256) || p->workspace_bytes < need)
    return HIPS_ERR_WORKSPACE;
  return HIPS_OK;
}

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return HIPS_OK;
  g_last_cuda_error = static_cast<int>(e);
  return HIPS_ERR_CUDA;
}

// Workspace bytes of one call with the kernels' own element types (0: no plan).
size_t native_ws(const hips_params* params, int op) {
  if (op == HIPS_OP_MASK) {
    MaskPlan plan;
    return plan_mask(params, 16, &plan) == HIPS_OK ? plan.ws : 0;
  }
  if (op == HIPS_OP_MASK_SPARSE) {  // either the fused launch or the two calls
    const size_t m = native_ws(params, HIPS_OP_MASK);
    const size_t s = native_ws(params, HIPS_OP_SPARSE);
    return m && s ? std::max(m, s) : 0;
  }
  if (op == HIPS_OP_SPARSE || op == HIPS_OP_DENSE) {
    AttnPlan plan;
    return plan_attn(params, op == HIPS_OP_DENSE, &plan) == HIPS_OK ? plan.ws : 0;
  }
  return 0;
}

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

// ---------------------------------------------------------------- e5m2 by widening
// e5m2 shapes that no e5m2 kernel plans (prefill query blocks, masks of more
// than 16 query rows, attention of more than 8 rows per query block): the
// keys (and values) a call reads, rows [0, seq_len) of every head, are
// widened exactly to bf16 in the workspace, after the bf16 plan's own area,
// and the bf16 kernels run on them. The e5m2 path is defined as the bf16 one
// on the widened values, so the results are the same; the cost is one pass
// over the cache and 2 bytes per element of workspace.
hips_params bf16_view(const hips_params* p) {
  hips_params b = *p;
  b.dtype = HIPS_BF16;
  b.kv_capacity = p->seq_len;  // the widened rows are compact
  return b;
}

size_t widened_bytes(const hips_params* p, bool with_v) {
  const size_t one = round256(static_cast<size_t>(p->batch) * p->n_kvheads * p->seq_len * hips::kD *
                              sizeof(uint16_t));
  return with_v ? 2 * one : one;
}

bool needs_widening(const hips_params* p, int op) {
  return p->dtype == HIPS_BF16_E5M2 && native_ws(p, op) == 0;
}

// Widen k (and v) into the workspace; *b gets the bf16 view whose workspace
// is the area before the widened rows, *kw and *vw the widened tensors.
int widen_inputs(const void* k, const void* v, const hips_params* p, int op, hips_params* b,
                 const void** kw, const void** vw) {
  *b = bf16_view(p);
  const size_t w = native_ws(b, op);
  if (!w) return HIPS_ERR_UNSUPPORTED;
  const bool with_v = v != nullptr;
  const size_t off = round256(w);
  if (!p->workspace || !aligned(p->workspace, 256) || p->workspace_bytes < off + widened_bytes(p, with_v))
    return HIPS_ERR_WORKSPACE;
  unsigned char* base = static_cast<unsigned char*>(p->workspace) + off;
  const size_t one = widened_bytes(p, false);
  cudaStream_t stream = static_cast<cudaStream_t>(p->stream);
  const int64_t heads = static_cast<int64_t>(p->batch) * p->n_kvheads;
  cudaError_t e = hips::launch_widen_e5m2(k, base, heads, p->seq_len, p->kv_capacity, stream);
  if (e != cudaSuccess) return cuda_status(e);
  *kw = base;
  *vw = nullptr;
  if (with_v) {
    e = hips::launch_widen_e5m2(v, base + one, heads, p->seq_len, p->kv_capacity, stream);
    if (e != cudaSuccess) return cuda_status(e);
    *vw = base + one;
  }
  b->workspace_bytes = off;
  return HIPS_OK;
}

int run_attention(const void* q, const void* k, const void* v, const int32_t* idx,
                  const hips_params* p, void* out, bool dense) {
  const int op = dense ? HIPS_OP_DENSE : HIPS_OP_SPARSE;
  int st = validate(p, op);
  if (st) return st;
  if (!q || !k || !v || !out || (!dense && !idx)) return HIPS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (idx && !aligned(idx, 4)))
    return HIPS_ERR_INVALID_ARG;
  if (needs_widening(p, op)) {
    hips_params b;
    const void *kw, *vw;
    st = widen_inputs(k, v, p, op, &b, &kw, &vw);
    if (st) return st;
    return run_attention(q, kw, vw, idx, &b, out, dense);
  }
  AttnPlan plan;
  st = plan_attn(p, dense, &plan);
  if (st) return st;
  st = check_workspace(p, plan.ws);
  if (st) return st;
  hips::AttnArgs& a = plan.a;
  a.q = q; a.k = k; a.v = v; a.idx = idx; a.out = out;
  a.status = static_cast<hips::Status*>(p->workspace);
  a.part = reinterpret_cast<float*>(static_cast<char*>(p->workspace) + kStatusBytes);
  a.counters = reinterpret_cast<unsigned int*>(static_cast<char*>(p->workspace) + kCounterOffset);
  cudaStream_t stream = static_cast<cudaStream_t>(p->stream);
  return cuda_status(plan.mma ? hips::launch_attn_mma(a, plan.smem, stream)
                              : hips::launch_attn_fma(a, plan.smem, stream));
}

// The tensor-core mask kernel also runs the attention of its mask row (one
// launch for a decode step) when the row group is a single MMA column block
// of at most mask_mma_fused_rows() query rows.
bool fusable(const MaskPlan& plan) {
  return plan.decode || (plan.mma && hips::mask_mma_nc(plan.a.rows_max) == 1 &&
                         plan.a.rows_max <= hips::mask_mma_fused_rows());
}

// Launch the pruning stages of a mask call; *init gets the list the
// iteration starts from.
int run_stages(const void* q, const void* k, const hips_params* p, const MaskPlan& plan,
               cudaStream_t stream, const int32_t** init) {
  const StagePlan& sp = plan.stp;
  const hips::MaskArgs& m = plan.a;
  unsigned char* base = static_cast<unsigned char*>(p->workspace) + plan.st_off;
  const size_t scores = (static_cast<size_t>(m.units) * sp.cap * sizeof(float) + 255) / 256 * 256;
  const size_t list = (static_cast<size_t>(m.units) * sp.lstride * sizeof(int32_t) + 255) / 256 * 256;
  int32_t* lists[2] = {reinterpret_cast<int32_t*>(base + scores),
                       reinterpret_cast<int32_t*>(base + scores + list)};
  hips::StageArgs s{};
  s.q = q;
  s.k = k;
  s.status = static_cast<hips::Status*>(p->workspace);
  s.dtype = m.dtype;
  s.n_qheads = m.n_qheads;
  s.n_mheads = m.n_kvheads;
  s.group = m.group;
  s.kv_heads = m.kv_heads;
  s.kv_div = m.kv_div;
  s.q_len = m.q_len;
  s.block_q = m.block_q;
  s.block_k = m.block_k;
  s.nqb = m.nqb;
  s.n0max = m.n0max;
  s.units = m.units;
  s.seq_len = m.seq_len;
  s.kv_cap = m.kv_cap;
  s.q_pos0 = m.q_pos0;
  s.lstride = sp.lstride;
  s.cap = sp.cap;
  s.scores = reinterpret_cast<float*>(base);
  // one wave of scoring CTAs (one per SM; each keeps 32 groups' key rows
  // in flight), at least 32 chunks each
  s.slices = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(kPlanSMs / m.units, cdiv(sp.cap, 32))));
  for (int i = 0; i < sp.nsteps; ++i) {
    const StageStep& step = sp.steps[i];
    s.c_in = step.c_in;
    s.c_list = i ? sp.steps[i - 1].c_out : step.c_in;
    s.in = i ? lists[(i - 1) & 1] : nullptr;
    s.out = lists[i & 1];
    s.keep = step.keep;
    s.stride_q = step.stride_q;
    s.c_out = step.c_out;
    s.final_list = step.final_list ? 1 : 0;
    if (step.keep > 0) {
      const cudaError_t e = hips::launch_stage_score(s, stream);
      if (e != cudaSuccess) return cuda_status(e);
    }
    const cudaError_t e = hips::launch_stage_select(s, stream);
    if (e != cudaSuccess) return cuda_status(e);
  }
  *init = lists[(sp.nsteps - 1) & 1];
  return HIPS_OK;
}

// Plan and launch the mask kernel (with the fused attention when v and out
// are given). A cluster of C CTAs needs C free SMs of one GPC: take the
// largest cluster for which every mask row is resident at once (one wave);
// fall back to smaller clusters if the device refuses the shape.
int launch_mask(const void* q, const void* k, const hips_params* params, int32_t* idx_out,
                const void* v, void* out) {
  MaskPlan plan;
  const bool attend = out != nullptr;
  int st = plan_mask(params, 16, &plan, attend);
  if (st) return st;
  st = check_workspace(params, plan.ws);
  if (st) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(params->stream);
  const int32_t* init = nullptr;
  if (plan.stp.nsteps) {
    st = run_stages(q, k, params, plan, stream, &init);
    if (st) return st;
  }
  for (int cap = 16; cap >= 1; cap = std::min(cap - 1, plan.a.cluster - 1)) {
    st = plan_mask(params, cap, &plan, attend);
    if (st) return st;
    if (plan.a.cluster > cap) continue;
    if (plan.a.cluster > 1 && cap > 1) {
      const int fit = resident_clusters(plan);
      if (fit >= 0 && fit < plan.a.units) continue;
    }
    hips::MaskArgs& a = plan.a;
    a.q = q; a.k = k; a.idx = idx_out;
    a.status = static_cast<hips::Status*>(params->workspace);
    if (init) {
      a.init = init;
      a.init_stride = plan.stp.lstride;
      a.init_cap = plan.stp.cap;
    }
    if (plan.norms) {
      a.knorm = reinterpret_cast<const float*>(static_cast<unsigned char*>(params->workspace) + kStatusBytes);
      const cudaError_t e = hips::launch_key_block_norms(a, params->batch, stream);
      if (e != cudaSuccess) return cuda_status(e);
    }
    if (out) {
      if (!fusable(plan)) return HIPS_ERR_UNSUPPORTED;
      a.v = v;
      a.out = out;
      a.scale_log2 = static_cast<float>(1.4426950408889634 / 11.313708498984761);  // log2(e)/sqrt(128)
    }
    const cudaError_t e = plan.decode ? hips::launch_decode(a, plan.smem, stream)
                          : plan.mma  ? hips::launch_mask_mma(a, plan.smem, stream)
                                      : hips::launch_mask_fma(a, plan.smem, stream);
    if (e == cudaSuccess) return HIPS_OK;
    if ((e == cudaErrorInvalidClusterSize || e == cudaErrorLaunchOutOfResources) && cap > 1) {
      (void)cudaGetLastError();
      continue;
    }
    return cuda_status(e);
  }
  return HIPS_ERR_UNSUPPORTED;
}

}  // namespace

namespace hips {

// Validation and launch plan of a sparse attention call that brings its own
// scratch memory (no caller workspace); *scratch_bytes is what it needs.
int plan_sparse_attn_own_scratch(const void* q, const void* k, const void* v, const int32_t* idx,
                                 const hips_params* p, void* out, AttnArgs* args, int* smem,
                                 size_t* scratch_bytes, bool* tensor_core) {
  int st = validate(p, HIPS_OP_SPARSE);
  if (st) return st;
  if (!q || !k || !v || !out || !idx) return HIPS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(idx, 4))
    return HIPS_ERR_INVALID_ARG;
  AttnPlan plan;
  st = plan_attn(p, false, &plan);
  if (st) return st;
  *args = plan.a;
  args->q = q; args->k = k; args->v = v; args->idx = idx; args->out = out;
  *smem = plan.smem;
  *scratch_bytes = plan.ws;
  *tensor_core = plan.mma;
  return HIPS_OK;
}

int record_cuda_error(cudaError_t e) { return cuda_status(e); }

}  // namespace hips

extern "C" {

int64_t hip_idx_row_stride(const hips_params* params) {
  if (validate(params, HIPS_OP_MASK) != HIPS_OK) return 0;
  return row_stride(params);
}

size_t hip_workspace_size(const hips_params* params, int op) {
  if (validate(params, op) != HIPS_OK) return 0;
  const size_t n = native_ws(params, op);
  if (n || params->dtype != HIPS_BF16_E5M2) return n;
  // e5m2 shapes no e5m2 kernel plans: the bf16 plan on widened rows
  const hips_params b = bf16_view(params);
  const size_t w = native_ws(&b, op);
  if (!w) return 0;
  return round256(w) + widened_bytes(params, op != HIPS_OP_MASK);
}

int hip_workspace_init(const hips_params* params) {
  if (!params || !params->workspace || params->workspace_bytes < kStatusBytes) return HIPS_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(params->workspace, 0, kStatusBytes,
                                     static_cast<cudaStream_t>(params->stream)));
}

int hip_check_status(const hips_params* params) {
  if (!params || !params->workspace || params->workspace_bytes < kStatusBytes) return HIPS_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(params->stream);
  hips::Status host{};
  int st = cuda_status(cudaStreamSynchronize(s));
  if (st) return st;
  st = cuda_status(cudaMemcpy(&host, params->workspace, sizeof(host), cudaMemcpyDeviceToHost));
  if (st) return st;
  if (host.flags == 0) return HIPS_OK;
  st = cuda_status(cudaMemset(params->workspace, 0, kStatusBytes));
  if (st) return st;
  return (host.flags & hips::kStatusTimeout) ? HIPS_ERR_TIMEOUT : HIPS_ERR_INTERNAL;
}

int hip_mask(const void* q, const void* k, const hips_params* params, int32_t* idx_out) {
  int st = validate(params, HIPS_OP_MASK);
  if (st) return st;
  if (!q || !k || !idx_out) return HIPS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(idx_out, 4)) return HIPS_ERR_INVALID_ARG;
  if (needs_widening(params, HIPS_OP_MASK)) {
    hips_params b;
    const void *kw, *vw;
    st = widen_inputs(k, nullptr, params, HIPS_OP_MASK, &b, &kw, &vw);
    if (st) return st;
    return hip_mask(q, kw, &b, idx_out);
  }
  return launch_mask(q, k, params, idx_out, nullptr, nullptr);
}

int hip_mask_sparse_attn(const void* q, const void* k, const void* v, const hips_params* params,
                         int32_t* idx_out, void* out) {
  int st = validate(params, HIPS_OP_MASK_SPARSE);
  if (st) return st;
  if (!q || !k || !v || !idx_out || !out) return HIPS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(idx_out, 4))
    return HIPS_ERR_INVALID_ARG;
  if (params->mask_len != params->seq_len) return HIPS_ERR_INVALID_ARG;  // a fresh mask
  if (needs_widening(params, HIPS_OP_MASK_SPARSE)) {
    hips_params b;
    const void *kw, *vw;
    st = widen_inputs(k, v, params, HIPS_OP_MASK_SPARSE, &b, &kw, &vw);
    if (st) return st;
    return hip_mask_sparse_attn(q, kw, vw, &b, idx_out, out);
  }
  MaskPlan plan;
  st = plan_mask(params, 16, &plan, true);
  if (st) return st;
  if (fusable(plan)) return launch_mask(q, k, params, idx_out, v, out);
  st = launch_mask(q, k, params, idx_out, nullptr, nullptr);
  if (st) return st;
  return run_attention(q, k, v, idx_out, params, out, false);
}

int hip_sparse_attn(const void* q, const void* k, const void* v, const int32_t* idx,
                    const hips_params* params, void* out) {
  return run_attention(q, k, v, idx, params, out, false);
}

int hip_dense_attn(const void* q, const void* k, const void* v, const hips_params* params,
                   void* out) {
  return run_attention(q, k, v, nullptr, params, out, true);
}

int hip_last_cuda_error(void) { return g_last_cuda_error; }

const char* hip_error_string(int status) {
  switch (status) {
    case HIPS_OK: return "ok";
    case HIPS_ERR_INVALID_ARG: return "invalid argument";
    case HIPS_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case HIPS_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case HIPS_ERR_CUDA: return "CUDA launch failed";
    case HIPS_ERR_TIMEOUT: return "a bounded device wait expired";
    case HIPS_ERR_TOO_LARGE: return "request exceeds the library's built-in scratch size";
    case HIPS_ERR_INTERNAL: return "a device-side bound check failed";
    default: return "unknown status";
  }
}

}  // extern "C"
