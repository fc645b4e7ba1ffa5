/*
 * hip_sparse.h -- C ABI of the B200 (sm_100a) hierarchically pruned attention
 * library (libhip_sparse.so).
 *
 * The method (HiP, "A Training-Free Sub-quadratic Cost Transformer Model
 * Serving Framework with Hierarchically Pruned Attention") has two steps on
 * its hot path, and this library exposes each as one call:
 *
 *   hip_mask         hierarchical top-k selection of key blocks per query
 *                    block: start from k/b_k chunks that tile the causal key
 *                    range, repeatedly halve every chunk, score each half by
 *                    its centre key block and keep the global top k/b_k halves
 *                    until every chunk is one b_k block; then add the
 *                    always-kept sink and sliding-window blocks and write the
 *                    sorted block list with its nnz.
 *                    (Author Rebuttal to the Reviewer RsGC, Q2, steps 1-4;
 *                    research-map summary, Approach and the "Add V 2k and D 1k"
 *                    row of Measured effects.)
 *   hip_sparse_attn  exact softmax attention of every query row over only the
 *                    keys of its selected blocks ("the block sparse attention
 *                    kernel receives the non-zero entries' indices and the
 *                    number of non-zero entries (nnz) for each row": Author
 *                    Rebuttal to the Reviewer NLBm, W2), plus every key
 *                    appended since the mask was computed when a mask is
 *                    reused for r_m decode steps (summary, Limitations).
 *   hip_dense_attn   exact causal attention over every key; a comparison
 *                    point only (the pages compare against FlashAttention2).
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or keeps them. Calls are asynchronous on params->stream
 *    (a cudaStream_t; NULL is the legacy default stream), allocate nothing,
 *    and never synchronise the device.
 *  - Layouts (row-major, element type = params->dtype; with HIPS_BF16_E5M2
 *    k and v hold 1-byte e5m2 codes and q, out bf16):
 *      q, out   [batch, n_qheads, q_len, head_dim]
 *      k, v     [batch, n_kvheads, kv_capacity, head_dim]
 *      idx      int32 [batch, n_kvheads, n_qblocks, row_stride] (n_qheads in
 *               place of n_kvheads with HIPS_FLAG_HEAD_MASKS) with
 *               n_qblocks = ceil(q_len / block_q) and row_stride =
 *               hip_idx_row_stride(params); entry 0 of a row is nnz, then nnz
 *               ascending key-block ids, then -1 padding.
 *    Query head h reads KV head h / (n_qheads / n_kvheads). Query row i sits
 *    at absolute position q_pos0 + i and sees keys j <= q_pos0 + i.
 *  - head_dim must be 128. k, v, q, out must be 16-byte aligned.
 *  - Every call needs a workspace of at least hip_workspace_size(params, op)
 *    bytes (256-byte aligned, caller-owned). Its first 4096 bytes are a
 *    status block: a sticky error word (kernels only ever set bits there) and
 *    the split-merge counters of the attention, which are zero between
 *    calls. Clear it once after allocating (hip_workspace_init) and read it
 *    with hip_check_status. Calls sharing one workspace must not overlap on
 *    the GPU (issue them on one stream).
 *  - Return value: HIPS_OK (0) or a negative HIPS_ERR_* code. Argument errors
 *    are found on the host before anything is launched. HIPS_ERR_CUDA means
 *    a launch failed; hip_last_cuda_error() gives the cudaError_t.
 */
#ifndef HIP_SPARSE_H_
#define HIP_SPARSE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HIPS_API __attribute__((visibility("default")))
#else
#define HIPS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum hips_status {
  HIPS_OK = 0,
  HIPS_ERR_INVALID_ARG = -1, /* null pointer, bad shape, head ratio, topk % block_k ... */
  HIPS_ERR_UNSUPPORTED = -2, /* head_dim != 128, dtype, a shape no kernel covers */
  HIPS_ERR_WORKSPACE = -3,   /* workspace missing, misaligned or too small */
  HIPS_ERR_CUDA = -4,        /* a CUDA launch failed */
  HIPS_ERR_TIMEOUT = -5,     /* a bounded device wait expired (from hip_check_status) */
  HIPS_ERR_TOO_LARGE = -6,   /* more scratch than hip_sparse_attn_noalloc's fixed array */
  HIPS_ERR_INTERNAL = -7     /* a device-side bound check failed (from hip_check_status) */
};

/* Element types. HIPS_BF16_E5M2 is an fp8 KV cache: k and v hold fp8 e5m2
 * codes (1 byte per element; the OCP 8-bit floating-point format, the KV
 * cache type of "--kv-cache-dtype fp8_e5m2" in the HiP attention serving
 * command of the SGLang pull request "[Feature] Support Efficient Sparse HiP
 * Attention (InfiniteHiP)"), while q and out are bf16. Every code widens
 * exactly to bf16, and the mask and attention are those of bf16 keys and
 * values with the widened values. e5m2 kernels read the codes directly for
 * masks of one query position per mask row (decode, or b_q = 1) with at most
 * 8 query rows, for masks of 9 to 16 query rows with block_k <= 32 and
 * topk / block_k <= 1024, and for attention of at most 8 rows per query
 * block. Every other shape that bf16 supports (prefill query blocks, wider
 * masks and attention) widens the keys (and values) it reads, rows [0,
 * seq_len) of every head, into the workspace first and runs the bf16
 * kernels on them: hip_workspace_size then includes 2 bytes per widened
 * element (B x n_kvheads x seq_len x head_dim, once for a mask, twice when
 * values are read), and the call makes one extra pass over the cache. */
enum hips_dtype { HIPS_F32 = 0, HIPS_BF16 = 1, HIPS_BF16_E5M2 = 2 };

enum hips_op { HIPS_OP_MASK = 0, HIPS_OP_SPARSE = 1, HIPS_OP_DENSE = 2, HIPS_OP_MASK_SPARSE = 3 };

/* hips_params.flags bits.
 * HIPS_FLAG_HEAD_MASKS: one mask per query head instead of one per group of
 *   query heads that share a KV head (the switch the SGLang integration calls
 *   HIP_HEAD_REDUCE, here off). A head's chunks are scored over its own b_q
 *   rows only, against its KV head's keys; idx is then
 *   [batch, n_qheads, n_qblocks, row_stride], and query head h attends the
 *   blocks of its own row. ("[Feature] Support Efficient Sparse HiP Attention
 *   (InfiniteHiP)", the HIP_HEAD_REDUCE environment switch.) Dense calls
 *   ignore it. */
enum hips_flags { HIPS_FLAG_HEAD_MASKS = 1 };

/* One InfiniteHiP pruning stage (the stages of the serving command's
 * --hip-attention-config in "[Feature] Support Efficient Sparse HiP Attention
 * (InfiniteHiP)"; Author Rebuttal to the Reviewer T2wK, Q1: the user sets per
 * iteration how many chunks are kept, how chunks are broken down and how
 * their representatives are picked). Stage 1 cuts the key blocks [0, N) of a
 * mask row into chunks of chunk_size keys aligned at multiples of it (the
 * last one clipped); a later stage cuts every chunk kept by the one before
 * into pieces of its own size. A stage with stage_k > 0 scores each chunk
 * [s, e) (in blocks) by its centre block s + (e - s) / 2 -- the max over
 * the stage's query rows and the block's keys they see of q.k -- and keeps
 * the stage_k / chunk_size best by (score desc, start asc); stage_k = 0 (null
 * on the page) keeps every chunk. The stage's query rows are the mask's
 * query heads at the positions i1-1, i1-1-stride_q, ... of the query block
 * [i0, i1) (the block's last row, which sees every key of the range, always
 * scores). After the stages the hierarchical iteration (hip_mask) runs with
 * k = topk (the page's second_stage_k) from the surviving chunks instead of
 * topk / block_k uniform ones: every round halves each chunk and keeps the
 * topk / block_k best halves (all of them while there are no more). The
 * page's stage_block_size_q is the mask's block_q; its stage_stride (1 in
 * every stage of the page's configuration) has no field. */
typedef struct hips_stage {
  int32_t chunk_size;  /* keys per chunk: a multiple of block_k that divides the
                          previous stage's chunk_size */
  int32_t stage_k;     /* keys kept: a multiple of chunk_size; 0 keeps every chunk */
  int32_t stride_q;    /* query-row stride of the stage's scoring, >= 1 */
  int32_t reserved;    /* 0 */
} hips_stage;

/* Most stages of one schedule. */
#define HIPS_MAX_STAGES 8

typedef struct hips_params {
  int32_t batch;      /* sequences */
  int32_t n_qheads;   /* query heads; a multiple of n_kvheads */
  int32_t n_kvheads;  /* key/value heads (GQA groups) */
  int32_t head_dim;   /* 128 */
  int64_t seq_len;    /* keys present now: T_cur */
  int64_t mask_len;   /* keys present when the mask was computed (== seq_len
                         for a fresh mask; < seq_len when reusing it) */
  int64_t kv_capacity;/* allocated length of the key axis, >= seq_len */
  int32_t q_len;      /* query rows per sequence: 1 for decode, T for prefill */
  int32_t dtype;      /* enum hips_dtype of q, k, v and out (accumulation is fp32) */
                      /* (HIPS_BF16_E5M2: q, out bf16; k, v e5m2) */
  int64_t q_pos0;     /* absolute position of query row 0; q_pos0 + q_len <= seq_len */
  int32_t block_q;    /* query rows sharing one mask (b_q) */
  int32_t block_k;    /* keys per block (b_k), a power of two */
  int32_t topk;       /* key budget k; a multiple of block_k, topk/block_k <= 2048 */
  int32_t sink;       /* leading keys always kept (0 = none) */
  int32_t window;     /* sliding-window keys always kept (0 = none) */
  int32_t flags;      /* HIPS_FLAG_* bits; 0 for the defaults */
  void* workspace;    /* device scratch, see hip_workspace_size */
  size_t workspace_bytes;
  void* stream;       /* cudaStream_t */
  int32_t n_stages;   /* pruning stages before the iteration, 0..HIPS_MAX_STAGES */
  int32_t reserved;   /* 0 */
  const hips_stage* stages; /* HOST array of n_stages entries (NULL when 0),
                          read during each call only. The mask of a schedule
                          needs, per mask row, at most topk / block_k chunks
                          at the last stage's size before the iteration
                          (worst case over the rows, from the bounds that
                          stage_k and the key range give); larger schedules
                          return HIPS_ERR_UNSUPPORTED. Attention-only calls
                          ignore the stages. */
} hips_params;

/* Entries of one idx row: 1 (nnz) + the largest possible nnz. */
HIPS_API int64_t hip_idx_row_stride(const hips_params* params);

/* Workspace bytes needed by one call of `op` (enum hips_op) with these
 * params; 0 if the params are invalid. */
HIPS_API size_t hip_workspace_size(const hips_params* params, int op);

/* Zero the 4096-byte status block of params->workspace (async on params->stream). */
HIPS_API int hip_workspace_init(const hips_params* params);

/* Synchronise params->stream, read and clear the status block. Returns
 * HIPS_OK, HIPS_ERR_TIMEOUT if some kernel gave up a bounded wait since the
 * last check, or HIPS_ERR_INTERNAL if a kernel found a list longer than its
 * planned capacity (the outputs of the calls since are then undefined). */
HIPS_API int hip_check_status(const hips_params* params);

/* Hierarchical top-k mask (see above). q: [B, Hq, q_len, d]; k: [B, Hkv,
 * kv_capacity, d]; keys [0, seq_len) are visible. idx_out: int32 [B, Hkv,
 * n_qblocks, row_stride], fully written (padding included). With
 * params->n_stages > 0 the pruning stages (struct hips_stage) run first, in
 * launches of their own on params->stream, and the iteration starts from
 * their survivors. */
HIPS_API int hip_mask(const void* q, const void* k, const hips_params* params, int32_t* idx_out);

/* Block-sparse attention over idx (as written by hip_mask at mask_len keys)
 * plus the keys [mask_len, seq_len). out: [B, Hq, q_len, d] in dtype. */
HIPS_API int hip_sparse_attn(const void* q, const void* k, const void* v, const int32_t* idx,
                    const hips_params* params, void* out);

/* hip_mask followed by hip_sparse_attn on its idx, for a freshly computed
 * mask (mask_len must equal seq_len, else HIPS_ERR_INVALID_ARG): writes
 * idx_out exactly as hip_mask does and out as hip_sparse_attn does. For
 * decode-shaped groups (at most 4 query rows per mask row, bf16) one launch
 * does both: the thread-block cluster that selects a row's blocks then
 * attends over them, each CTA over a contiguous share of the row, and the
 * CTAs' partial softmax sums are merged through distributed shared memory.
 * Other shapes run the two calls. Workspace: hip_workspace_size(params,
 * HIPS_OP_MASK_SPARSE). This is the sequence of the two steps defined above,
 * (Author Rebuttal to the Reviewer RsGC, Q2, then Reviewer NLBm, W2), in one
 * call. */
HIPS_API int hip_mask_sparse_attn(const void* q, const void* k, const void* v,
                                  const hips_params* params, int32_t* idx_out, void* out);

/* Dense causal attention over keys [0, seq_len); block/topk fields ignored. */
HIPS_API int hip_dense_attn(const void* q, const void* k, const void* v, const hips_params* params,
                   void* out);

/* Same result as hip_sparse_attn, for callers that cannot allocate device
 * memory: for example a serving loop whose memory pool is frozen after
 * start-up, or code that must not let a cudaMalloc (and the device-wide
 * synchronisation it may imply) into a latency-critical decode step. It takes
 * no workspace (params->workspace and workspace_bytes are ignored) and calls
 * no allocator; its split-K scratch is a fixed device array of
 * HIPS_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits. There is no counterpart to this
 * call in the paper; it only changes where the scratch lives.
 *  - Calls needing more scratch than that (hip_workspace_size(params,
 *    HIPS_OP_SPARSE) > HIPS_NOALLOC_SCRATCH_BYTES) return HIPS_ERR_TOO_LARGE
 *    before launching anything.
 *  - The first call on each device looks the array's device address up
 *    (cudaGetSymbolAddress, with that device current) and caches it with the
 *    device's context; the first call after a device reset looks it up
 *    again. Make the first call on a device, and the first after a reset,
 *    before any stream capture.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents; each call clears the part that must start at zero. Calls that
 *    overlap on the GPU (different streams, or other host threads) race on
 *    it: serialise them.
 *  - A bounded device wait that gives up is recorded in the array's status
 *    word, which the next call clears: read it with
 *    hip_noalloc_check_status before the next call. */
#define HIPS_NOALLOC_SCRATCH_BYTES (512u << 10)
HIPS_API int hip_sparse_attn_noalloc(const void* q, const void* k, const void* v,
                                     const int32_t* idx, const hips_params* params, void* out);

/* Status of the most recent hip_sparse_attn_noalloc call on the current
 * device: synchronises `stream` (a cudaStream_t), reads the status word of
 * the library's fixed array and clears it. Returns HIPS_OK, or
 * HIPS_ERR_TIMEOUT if that call's kernel gave up a bounded wait (its output
 * is then undefined), or HIPS_ERR_CUDA. Allocates nothing either. */
HIPS_API int hip_noalloc_check_status(void* stream);

/* cudaError_t of the last failed launch on this thread (0 if none). */
HIPS_API int hip_last_cuda_error(void);

/* Static string for a hips_status code. */
HIPS_API const char* hip_error_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* HIP_SPARSE_H_ */
