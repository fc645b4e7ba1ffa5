// Launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

struct hips_params;

namespace hips {

struct Status;

// Layout of the head of every workspace (and of the no-allocation entry
// point's fixed scratch array): bytes [0, 256) hold the sticky status word,
// bytes [256, 4096) one split-merge counter per (sequence, KV head, query
// block) unit of a split attention call; both are zero between calls. The
// split-K partials (or the key-norm table of a many-row mask) follow at 4096.
constexpr size_t kStatusBytes = 4096;
constexpr size_t kCounterOffset = 256;
constexpr int64_t kMaxCounters = static_cast<int64_t>((kStatusBytes - kCounterOffset) / sizeof(unsigned int));
static_assert(kCounterOffset >= 16, "the counters start after the status word");
static_assert(kCounterOffset + kMaxCounters * sizeof(unsigned int) <= kStatusBytes,
              "the counter area of kMaxCounters units lies inside the status block");

struct MaskArgs {
  const void* q;
  const void* k;
  int32_t* idx;
  Status* status;
  int dtype, n_qheads, n_kvheads, group, q_len, block_q, block_k, n0max, sink, window;
  int nqb, cluster, per_cta, rows_max, rows_pad, stages;
  // K (and V) of mask head g live in head g / kv_div of kv_heads (kv_div = 1
  // with one mask per KV-head group, = group size with one mask per query head)
  int kv_heads, kv_div;
  int64_t units, seq_len, kv_cap, q_pos0, row_stride;
  // fused decode (tensor-core mask, few rows): when out is set, the cluster
  // of a mask row also computes the row's sparse attention over v
  const void* v;
  void* out;
  float scale_log2;
  // many-row masks: per (sequence, KV head, key block) an upper bound of the
  // block's key 2-norms, written by key_block_norms before the mask launch
  const float* knorm;
  int64_t knorm_stride;  // key blocks per head (ceil(seq_len / block_k))
  // decode kernel: keep the last round's dots for the attention; bytes of
  // one slot of its staging ring
  int stash_dots;
  int slot_bytes;
  int list_cap;  // entries of its staging list
  // pruning stages ran before: the initial chunks of unit u are the list at
  // init + u * init_stride ([count, n_keep, 0, 0, starts[init_cap],
  // ends[init_cap]]) instead of the n0 uniform chunks; n_keep replaces n0
  const int32_t* init;
  int64_t init_stride;
  int init_cap;
};

// One step of the pruning stages (stages.cu): the chunks of every mask row
// -- the tiling of [0, N) in chunks of c_in blocks (c_in > 0), or the list
// `in` -- are scored (stage_score) and the best `keep` of them (all when
// keep is 0) are cut into pieces of c_out blocks and written to `out`
// (stage_select). With final_list the pieces are then halved for as long as
// the halves number at most n0, the result being the iteration's initial
// chunks. Lists hold per unit lstride int32: [count, n_keep, 0, 0,
// starts[cap], ends[cap]] (n_keep only in a final list).
struct StageArgs {
  const void* q;
  const void* k;
  Status* status;
  int dtype, n_qheads, n_mheads, group, kv_heads, kv_div, q_len, block_q, block_k, nqb, n0max;
  int64_t units, seq_len, kv_cap, q_pos0;
  int c_in;
  int c_list;  // blocks of every input chunk but the last (c_in, or the previous step's c_out)
  const int32_t* in;
  int32_t* out;
  int64_t lstride;
  int cap;
  float* scores;  // per unit cap floats
  int keep;
  int stride_q;
  int c_out;
  int final_list;
  int slices;  // CTAs per unit of the scoring launch
};

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* idx;
  void* out;
  float* part;  // split partials [rows_total][nsplit][4 + 128]
  Status* status;
  unsigned int* counters;  // per unit, zero between calls (split merge tickets)
  int dtype, batch, n_qheads, n_kvheads, group, q_len, block_q, nqb, nsplit, dense, rows_max;
  int item_keys, table_items;
  int kv_heads, kv_div;  // K/V of head g at head g / kv_div of kv_heads (as in MaskArgs)
  int64_t rows_total, seq_len, mask_len, kv_cap, q_pos0, row_stride;
  float scale_log2;
};

// CUDA-core hierarchical top-k mask (mask_fma.cu)
int mask_fma_rc(int rows_max);
int mask_fma_smem_bytes(int n0max, int rows_pad, int per_cta, int cluster, int stages);
int mask_fma_tile_keys(int dtype);
// clusters of a.cluster CTAs that can be resident at once (-1 if unknown)
int mask_fma_max_active_clusters(const MaskArgs& a, int smem);
cudaError_t launch_mask_fma(const MaskArgs& a, int smem, cudaStream_t stream);

// Tensor-core hierarchical top-k mask, bf16 keys or e5m2 keys with one MMA
// column block (mask_mma.cu)
int mask_mma_nc(int rows_max);  // N / 16 of the MMA (0 = too many rows)
int mask_mma_smem_bytes(int nc, int n0max, int per_cta, int cluster, bool kv8);
int mask_mma_tile_keys();
int mask_mma_max_active_clusters(const MaskArgs& a, int smem);
cudaError_t launch_mask_mma(const MaskArgs& a, int smem, cudaStream_t stream);
int mask_mma_fused_rows();  // most query rows of a fused mask + attention launch
// Fill a.knorm (a workspace array of units' heads x knorm_stride floats)
cudaError_t launch_key_block_norms(const MaskArgs& a, int batch, cudaStream_t stream);

// Decode-shaped masks over e5m2 keys (one query position per mask row, at
// most decode_max_rows() query rows) with their attention, on CUDA cores
// (decode.cu). decode_smem_bytes sets a.stash_dots (the last round's dots
// kept for the attention) and a.slot_bytes (staging ring) within smem_cap.
int decode_max_rows();
int decode_smem_bytes(MaskArgs& a, bool attend, int smem_cap);
int decode_max_active_clusters(const MaskArgs& a, int smem);
cudaError_t launch_decode(const MaskArgs& a, int smem, cudaStream_t stream);

// Pruning stages (stages.cu). A stage of a mask row ranks at most
// kStageMaxChunks chunks (the selection keeps their score keys in shared
// memory).
constexpr int kStageMaxChunks = 36864;
cudaError_t launch_stage_score(const StageArgs& a, cudaStream_t stream);
cudaError_t launch_stage_select(const StageArgs& a, cudaStream_t stream);

// Tensor-core attention for query blocks, bf16 (attn_mma.cu)
int attn_mma_smem_bytes(int table_items);
int attn_mma_tile_keys();
int attn_mma_rows();
cudaError_t launch_attn_mma(const AttnArgs& a, int smem, cudaStream_t stream);

// CUDA-core split-K attention with the split merge fused (attn_fma.cu)
int attn_fma_tile_keys(int dtype);
int attn_fma_smem_bytes(int dtype, int rows_max, int table_items);
cudaError_t launch_attn_fma(const AttnArgs& a, int smem, cudaStream_t stream);

// Plan of a sparse attention call that uses scratch memory of its own
// (api.cu); the no-allocation entry point in noalloc.cu launches it.
int plan_sparse_attn_own_scratch(const void* q, const void* k, const void* v, const int32_t* idx,
                                 const hips_params* p, void* out, AttnArgs* args, int* smem,
                                 size_t* scratch_bytes, bool* tensor_core);
int record_cuda_error(cudaError_t e);

}  // namespace hips
