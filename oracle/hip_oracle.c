/*
 * Oracle for hierarchically pruned attention (HiP) -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow CPU statement of what the hot path computes. Only the tests,
 * the smoke check and the benchmark's CPU-baseline leg may load it; the
 * product library never links or calls it. It shares no code, header or
 * table with the CUDA path.
 *
 * Sources (cited by page title and section):
 *  [RsGC]    "A Training-free Sub-quadratic Cost Transformer Model Serving
 *            Framework With Hierarchically Pruned Attention", Author Rebuttal
 *            to the Reviewer RsGC, Q2: the iteration (initial uniform chunks,
 *            halving, centre-key scoring, global top-k, stop at b_k).
 *  [NLBm]    same page, Author Rebuttal to the Reviewer NLBm: W2 (the sparse
 *            attention kernel takes per-row non-zero block indices plus nnz),
 *            Q1 (block sizes b_q, b_k).
 *  [Summary] "A Training-Free Sub-quadratic Cost Transformer Model Serving
 *            Framework with Hierarchically Pruned Attention" (research-map
 *            summary): Approach (centre tokens as chunk representatives),
 *            Measured effects ("Add V 2k and D 1k": always-kept sink and
 *            sliding-window blocks), Limitations (mask refresh interval r_m).
 *  [PR]      "[Feature] Support Efficient Sparse HiP Attention (InfiniteHiP)"
 *            (SGLang pull request): the serving commands run HiP attention
 *            over a KV cache stored as fp8 e5m2 (--kv-cache-dtype
 *            fp8_e5m2). The code values follow the published 8-bit
 *            floating-point format (OCP "8-bit Floating Point
 *            Specification", E5M2): 1 sign bit, 5 exponent bits with bias 15,
 *            2 mantissa bits; exponent 0 holds zero and the subnormals
 *            m/4 * 2^-14, exponent 31 the infinities (m = 0) and NaNs.
 *            The same commands configure InfiniteHiP's multi-stage pruning
 *            (--hip-attention-config): per layer a list of stages, each with
 *            stage_chunk_size, stage_k, stage_block_size_q,
 *            stage_block_stride_q and stage_stride, then second_stage_k and
 *            sliding_window_size.
 *  [T2wK]    "A Training-free ... Hierarchically Pruned Attention", Author
 *            Rebuttal to the Reviewer T2wK, Q1 (the latest HiP): the user
 *            sets, per iteration, how many chunks are selected, how each
 *            chunk is broken down and how its representative is chosen.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - chunk i of n0 over N blocks is [floor(iN/n0), floor((i+1)N/n0));
 *  - a chunk [s,e) with L=e-s>1 splits at m = s + floor(L/2); a chunk with
 *    L=1 competes as its own candidate;
 *  - the representative block of [s,e) is s + floor((e-s)/2);
 *  - one mask per (sequence, KV head, query block); the score of a block is
 *    the max over the G*b_q query rows of the group and the b_k keys of the
 *    block of q.k, excluding keys after the row (causal) or past the range;
 *    with per_head set (the SGLang integration's HIP_HEAD_REDUCE switch off,
 *    "[Feature] Support Efficient Sparse HiP Attention (InfiniteHiP)"), one
 *    mask per (sequence, query head, query block) over that head's b_q rows
 *    and its KV head's keys, and query head h reads its own idx row;
 *  - ranking uses the raw dot q.k (a positive 1/sqrt(d) scale cannot change
 *    the order but could merge near-ties after rounding); ties go to the
 *    lower start block;
 *  - the dot that decides the selection is evaluated in fp32 in one fixed
 *    ("canonical") order, the same order the GPU kernels use, so that both
 *    sides take the integer decision in the same precision: d is cut into
 *    slices of 8 consecutive elements, slice s belongs to lane s mod 8, each
 *    lane runs an fma chain from 0 over its slices in increasing order, and
 *    the 8 lane partials are added as ((p0+p4)+(p2+p6)) + ((p1+p5)+(p3+p7));
 *  - sink = key blocks [0, ceil(sink/b_k)); window = the blocks covering keys
 *    [max(0, q_first-window+1), q_last] of the query block;
 *  - stages ([PR], [T2wK]): stage 1 tiles the keys [0, T_c) into chunks of
 *    stage_chunk_size keys aligned at multiples of it (a multiple of b_k,
 *    the last chunk clipped); stage s > 1 cuts every chunk that survived
 *    stage s-1 into pieces of its own chunk size (which divides the
 *    previous one). A stage scores its chunks like the halves of the
 *    iteration (centre block, max of the canonical dot) and keeps the
 *    stage_k / stage_chunk_size best by (score desc, start asc); a stage_k
 *    of 0 (null on the page) keeps every chunk unscored. The stage's query
 *    rows are the mask's (stage_block_size_q read as the mask's b_q) taken
 *    at stride stage_block_stride_q counted back from the block's last row,
 *    which sees every key of the range. stage_stride is 1 throughout the
 *    page's configuration and is not modelled. After the stages the
 *    iteration above runs with k = second_stage_k from the surviving chunks
 *    instead of the n0 uniform ones: halve, keep the top n0 (every candidate
 *    when there are no more than n0), stop at single blocks. Without stages
 *    it is the plain iteration;
 *  - attention of a query at position p uses the keys j of the selected
 *    blocks with j <= p and j < mask_len, plus every key in
 *    [mask_len, seq_len) with j <= p (keys appended since the mask refresh).
 * Attention itself is evaluated in fp64 (two passes: max, then weights).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int32_t batch, n_qheads, n_kvheads, head_dim;
  int64_t seq_len;      /* keys present now */
  int64_t mask_len;     /* keys present when the mask was computed */
  int64_t kv_capacity;  /* allocated length of the key axis (>= seq_len) */
  int32_t q_len;        /* query rows per sequence */
  int32_t pad0;
  int64_t q_pos0;       /* absolute position of query row 0 */
  int32_t block_q, block_k, topk, sink, window;
  int32_t per_head;     /* 1: one mask per query head, not per KV-head group */
  int32_t n_stages;     /* pruning stages before the iteration (0: none) */
  const struct oracle_stage* stages;
} oracle_shape;

/* One pruning stage ([PR], [T2wK]; readings in the header). */
typedef struct oracle_stage {
  int32_t chunk_size;  /* keys per chunk: a multiple of b_k dividing the previous stage's */
  int32_t stage_k;     /* keys kept (a multiple of chunk_size); 0 keeps every chunk */
  int32_t stride_q;    /* query-row stride within the query block, >= 1 */
  int32_t pad;
} oracle_stage;

enum { OR_OK = 0, OR_BAD = -1, OR_NOMEM = -2 };

static int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
static int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }
static int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* Value of one fp8 e5m2 code ([PR]; format definition in the header). */
static double e5m2_value(uint8_t c) {
  const int sign = c >> 7, e = (c >> 2) & 31, m = c & 3;
  double v;
  if (e == 0)
    v = ldexp(m / 4.0, -14);
  else if (e == 31)
    v = m == 0 ? INFINITY : NAN;
  else
    v = ldexp(1.0 + m / 4.0, e - 15);
  return sign ? -v : v;
}

/* Decode n e5m2 codes to float (every finite code is exact in float). An
 * fp8 KV cache is attended with these values: the mask and the attention
 * below then take them like any other keys and values. */
void oracle_decode_e5m2(const uint8_t* codes, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (float)e5m2_value(codes[i]);
}

/* The fp32 dot in the canonical order described in the header. */
float oracle_canonical_dot(const float* q, const float* k, int d) {
  float part[8];
  for (int lane = 0; lane < 8; ++lane) {
    float acc = 0.0f;
    for (int s = lane; s * 8 < d; s += 8)
      for (int e = 0; e < 8; ++e) acc = fmaf(q[s * 8 + e], k[s * 8 + e], acc);
    part[lane] = acc;
  }
  float a0 = part[0] + part[4], a1 = part[1] + part[5];
  float a2 = part[2] + part[6], a3 = part[3] + part[7];
  float b0 = a0 + a2, b1 = a1 + a3;
  return b0 + b1;
}

static int shape_ok(const oracle_shape* s) {
  if (!s || s->batch <= 0 || s->n_qheads <= 0 || s->n_kvheads <= 0) return 0;
  if (s->n_qheads % s->n_kvheads) return 0;
  if (s->head_dim <= 0 || s->head_dim % 64) return 0;
  if (s->seq_len <= 0 || s->mask_len <= 0 || s->mask_len > s->seq_len) return 0;
  if (s->kv_capacity < s->seq_len || s->q_len <= 0) return 0;
  if (s->q_pos0 < 0 || s->q_pos0 + s->q_len > s->seq_len) return 0;
  if (s->block_q <= 0 || s->block_k <= 0 || s->topk < s->block_k) return 0;
  if (s->topk % s->block_k || s->sink < 0 || s->window < 0) return 0;
  if (s->per_head != 0 && s->per_head != 1) return 0;
  if (s->n_stages < 0 || (s->n_stages > 0 && !s->stages)) return 0;
  for (int i = 0; i < s->n_stages; ++i) {
    const oracle_stage* g = &s->stages[i];
    if (g->chunk_size <= 0 || g->chunk_size % s->block_k || g->stride_q < 1) return 0;
    if (g->stage_k < 0 || g->stage_k % g->chunk_size) return 0;
    if (i > 0 && s->stages[i - 1].chunk_size % g->chunk_size) return 0;
  }
  return 1;
}

int64_t oracle_num_qblocks(const oracle_shape* s) { return cdiv64(s->q_len, s->block_q); }

/* Entries of one idx row after the nnz slot. */
int64_t oracle_idx_cap(const oracle_shape* s) {
  int64_t bk = s->block_k;
  int64_t cap = s->topk / bk + cdiv64(s->sink, bk);
  if (s->window > 0) cap += cdiv64((int64_t)s->window + s->block_q - 1, bk) + 1;
  return cap;
}

typedef struct { int64_t s, e; float score; } cand;

/* score desc, then start asc ([RsGC] step 4; tie rule: lower index first). */
static int cand_order(const void* pa, const void* pb) {
  const cand* a = (const cand*)pa;
  const cand* b = (const cand*)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->s > b->s) - (a->s < b->s);
}

/* [RsGC] step 4 (and a stage's selection): rank the nc scored candidates by
 * (score desc, start asc) and keep the best m < nc as the new chunks;
 * *gap takes the smaller of itself and the score gap at the cut, in
 * q.k/sqrt(d) units. Returns m. */
static int64_t rank_and_keep(cand* cands, int64_t nc, int64_t m, cand* chunks, int d, double* gap) {
  qsort(cands, (size_t)nc, sizeof(cand), cand_order);
  const double gp = ((double)cands[m - 1].score - (double)cands[m].score) / sqrt((double)d);
  if (gp < *gap) *gap = gp;
  for (int64_t i = 0; i < m; ++i) chunks[i] = cands[i];
  return m;
}

/* The query rows and the key range of one mask row (unit). */
typedef struct {
  int64_t b, g, h0, i0, i1, q_first, q_last, Tc, N, n0;
  int Gm;
} unit_rows;

static int unit_setup(const oracle_shape* sh, int64_t unit, unit_rows* u) {
  const int G = sh->n_qheads / sh->n_kvheads;
  const int64_t nqb = oracle_num_qblocks(sh), bk = sh->block_k;
  /* the mask's heads: G query heads sharing KV head g, or one query head */
  const int64_t mh = sh->per_head ? sh->n_qheads : sh->n_kvheads;
  const int64_t total = (int64_t)sh->batch * mh * nqb;
  if (unit < 0 || unit >= total) return OR_BAD;
  const int64_t qb = unit % nqb, hm = (unit / nqb) % mh;
  u->b = unit / (nqb * mh);
  u->g = sh->per_head ? hm / G : hm;       /* KV head */
  u->Gm = sh->per_head ? 1 : G;            /* query heads of the mask */
  u->h0 = sh->per_head ? hm : hm * G;      /* first of them */
  u->i0 = qb * sh->block_q;
  u->i1 = min64(u->i0 + sh->block_q, sh->q_len);
  u->q_first = sh->q_pos0 + u->i0;
  u->q_last = sh->q_pos0 + u->i1 - 1;
  u->Tc = min64(u->q_last + 1, sh->seq_len);
  u->N = cdiv64(u->Tc, bk);
  u->n0 = min64(sh->topk / bk, u->N);
  return OR_OK;
}

/* [RsGC] step 3: the score of key block `rep` for the unit's query rows: the
 * max over the rows and the block's keys j < Tc, j <= p (causal) of the
 * canonical dot q.k; -inf when no row sees a key of the block. A stage
 * scores with the rows i1-1, i1-1-stride, ... of the block (stride 1: all). */
static float block_score(const float* q, const float* k, const oracle_shape* sh,
                         const unit_rows* u, int64_t rep, int stride) {
  const int d = sh->head_dim;
  const int64_t bk = sh->block_k;
  float best = -INFINITY;
  for (int h = 0; h < u->Gm; ++h) {
    const int64_t qh = u->h0 + h;
    for (int64_t i = u->i1 - 1; i >= u->i0; i -= stride) {
      const int64_t p = sh->q_pos0 + i;
      const float* qr = q + (((u->b * sh->n_qheads + qh) * sh->q_len + i) * d);
      for (int64_t j = rep * bk; j < min64(rep * bk + bk, u->Tc); ++j) {
        if (j > p) continue;
        const float* kj = k + (((u->b * sh->n_kvheads + u->g) * sh->kv_capacity + j) * d);
        float sc = oracle_canonical_dot(qr, kj, d);
        if (sc > best) best = sc;
      }
    }
  }
  return best;
}

/*
 * Scores of explicit key blocks for one unit (the step-3 score above), so
 * that a test can replay the rounds along another selection path: out[i] is
 * the score of blocks[i] (-inf for a block outside [0, N)).
 */
int oracle_block_scores(const float* q, const float* k, const oracle_shape* sh, int64_t unit,
                        const int64_t* blocks, int64_t n, float* out) {
  if (!q || !k || !out || (n > 0 && !blocks) || !shape_ok(sh)) return OR_BAD;
  unit_rows u;
  if (unit_setup(sh, unit, &u) != OR_OK) return OR_BAD;
  for (int64_t i = 0; i < n; ++i)
    out[i] = (blocks[i] >= 0 && blocks[i] < u.N) ? block_score(q, k, sh, &u, blocks[i], 1) : -INFINITY;
  return OR_OK;
}

/*
 * One mask row: sequence b, KV head g, query block qb ([RsGC] steps 1-4,
 * then the sink/window union of [Summary] and the idx+nnz row of [NLBm] W2).
 */
static int mask_unit(const float* q, const float* k, const oracle_shape* sh, int64_t unit,
                     int32_t* row, double* gap_out, int32_t* rounds_out, int64_t* scored_out) {
  const int d = sh->head_dim;
  const int64_t bk = sh->block_k;
  unit_rows u;
  if (unit_setup(sh, unit, &u) != OR_OK) return OR_BAD;
  const int64_t q_first = u.q_first, q_last = u.q_last;
  const int64_t N = u.N, n0 = u.n0;
  const int64_t cap = oracle_idx_cap(sh);

  /* chunks and candidates never overlap, so N bounds both lists */
  cand* chunks = (cand*)malloc(sizeof(cand) * (size_t)N);
  cand* cands = (cand*)malloc(sizeof(cand) * (size_t)N);
  unsigned char* keep = (unsigned char*)calloc((size_t)N, 1);
  if (!chunks || !cands || !keep) { free(chunks); free(cands); free(keep); return OR_NOMEM; }

  double gap = INFINITY;
  int32_t rounds = 0;
  int64_t scored = 0, nk = 0; /* nk: chunks kept so far */

  if (sh->n_stages == 0) {
    /* step 1: n0 chunks that tile the block range [0, N) */
    for (int64_t i = 0; i < n0; ++i) {
      chunks[i].s = i * N / n0;
      chunks[i].e = (i + 1) * N / n0;
    }
    nk = n0;
  } else {
    /* stage 1 cuts the whole range [0, N) into pieces of its chunk size, a
     * later stage every survivor of the one before; a stage with stage_k > 0
     * keeps its best stage_k / chunk_size pieces */
    chunks[0].s = 0;
    chunks[0].e = N;
    nk = 1;
    for (int st = 0; st < sh->n_stages; ++st) {
      const oracle_stage* g = &sh->stages[st];
      const int64_t cs = g->chunk_size / bk;
      int64_t nc = 0;
      for (int64_t i = 0; i < nk; ++i)
        for (int64_t s0 = chunks[i].s; s0 < chunks[i].e; s0 += cs) {
          cands[nc].s = s0;
          cands[nc].e = min64(s0 + cs, chunks[i].e);
          ++nc;
        }
      const int64_t m = g->stage_k / g->chunk_size;
      if (g->stage_k > 0 && nc > m) {
        for (int64_t c = 0; c < nc; ++c)
          cands[c].score = block_score(q, k, sh, &u, cands[c].s + (cands[c].e - cands[c].s) / 2,
                                       g->stride_q);
        nk = rank_and_keep(cands, nc, m, chunks, d, &gap);
        scored += nc;
        ++rounds;
      } else {
        for (int64_t i = 0; i < nc; ++i) chunks[i] = cands[i];
        nk = nc;
      }
    }
  }
  for (;;) {
    int64_t nc = 0, longest = 0;
    for (int64_t i = 0; i < nk; ++i) longest = max64(longest, chunks[i].e - chunks[i].s);
    /* every chunk is one b_k block, no more of them than n0: stop (stages
     * may leave more single blocks than n0; they are ranked once more) */
    if (longest <= 1 && nk <= n0) break;
    /* step 2: halve every chunk */
    for (int64_t i = 0; i < nk; ++i) {
      int64_t s = chunks[i].s, e = chunks[i].e, L = e - s;
      if (L > 1) {
        int64_t m = s + L / 2;
        cands[nc].s = s; cands[nc].e = m; ++nc;
        cands[nc].s = m; cands[nc].e = e; ++nc;
      } else {
        cands[nc].s = s; cands[nc].e = e; ++nc;
      }
    }
    if (nc <= n0) {
      /* no more candidates than survivors: all are kept, none is ranked */
      for (int64_t i = 0; i < nc; ++i) chunks[i] = cands[i];
      nk = nc;
      continue;
    }
    /* step 3: score each half by its centre block */
    for (int64_t c = 0; c < nc; ++c) {
      int64_t rep = cands[c].s + (cands[c].e - cands[c].s) / 2;
      cands[c].score = block_score(q, k, sh, &u, rep, 1);
    }
    /* step 4: global top-n0 of all candidates */
    nk = rank_and_keep(cands, nc, n0, chunks, d, &gap);
    scored += nc;
    ++rounds;
  }
  for (int64_t i = 0; i < nk; ++i) keep[chunks[i].s] = 1;
  /* always-kept sink and sliding-window blocks */
  for (int64_t c = 0; c < min64(cdiv64(sh->sink, bk), N); ++c) keep[c] = 1;
  if (sh->window > 0) {
    int64_t lo = max64(0, q_first - sh->window + 1);
    for (int64_t c = lo / bk; c <= q_last / bk && c < N; ++c) keep[c] = 1;
  }
  int64_t nnz = 0;
  for (int64_t c = 0; c < N; ++c) nnz += keep[c];
  if (nnz > cap) { free(chunks); free(cands); free(keep); return OR_BAD; }
  nnz = 0;
  for (int64_t c = 0; c < N; ++c)
    if (keep[c]) row[1 + nnz++] = (int32_t)c;
  row[0] = (int32_t)nnz;
  for (int64_t i = nnz; i < cap; ++i) row[1 + i] = -1;
  if (gap_out) *gap_out = gap;
  if (rounds_out) *rounds_out = rounds;
  if (scored_out) *scored_out = scored;
  free(chunks); free(cands); free(keep);
  return OR_OK;
}

/*
 * Masks of the given units (unit = (b * Hkv + g) * n_qblocks + qb), or of all
 * units when units == NULL. idx_out holds one row of 1 + cap int32 per unit:
 * [nnz, ascending block ids..., -1 padding]. gap_out (optional) gets the
 * smallest score gap at the cut over the rounds, in q.k/sqrt(d) units
 * (+inf when no round had more candidates than survivors). rounds_out and
 * scored_out (optional) count the rounds and the candidates scored.
 */
int oracle_mask(const float* q, const float* k, const oracle_shape* sh, const int64_t* units,
                int64_t n_units, int32_t* idx_out, double* gap_out, int32_t* rounds_out,
                int64_t* scored_out) {
  if (!q || !k || !idx_out || !shape_ok(sh)) return OR_BAD;
  const int64_t total = (int64_t)sh->batch * (sh->per_head ? sh->n_qheads : sh->n_kvheads) *
                        oracle_num_qblocks(sh);
  if (!units) n_units = total;
  const int64_t stride = 1 + oracle_idx_cap(sh);
  int status = OR_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < n_units; ++u) {
    int64_t unit = units ? units[u] : u;
    int st = (unit < 0 || unit >= total) ? OR_BAD
             : mask_unit(q, k, sh, unit, idx_out + u * stride, gap_out ? gap_out + u : NULL,
                         rounds_out ? rounds_out + u : NULL, scored_out ? scored_out + u : NULL);
    if (st != OR_OK) {
#pragma omp critical
      status = st;
    }
  }
  return status;
}

/* Softmax attention of one query row over an explicit key list, in fp64. */
static void attend(const float* qr, const float* kbase, const float* vbase, int d,
                   const int64_t* keys, int64_t nkeys, float* out) {
  double* o = (double*)calloc((size_t)d, sizeof(double));
  double* s = (double*)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1));
  const double scale = 1.0 / sqrt((double)d);
  double m = -INFINITY, l = 0.0;
  for (int64_t t = 0; t < nkeys; ++t) {
    const float* kj = kbase + keys[t] * d;
    double acc = 0.0;
    for (int e = 0; e < d; ++e) acc += (double)qr[e] * (double)kj[e];
    s[t] = acc * scale;
    if (s[t] > m) m = s[t];
  }
  for (int64_t t = 0; t < nkeys; ++t) {
    const double w = exp(s[t] - m);
    const float* vj = vbase + keys[t] * d;
    l += w;
    for (int e = 0; e < d; ++e) o[e] += w * (double)vj[e];
  }
  for (int e = 0; e < d; ++e) out[e] = nkeys > 0 ? (float)(o[e] / l) : 0.0f;
  free(o);
  free(s);
}

/* Keys attended by query row i of (b, h) under idx ([NLBm] W2, readings above). */
static int64_t row_keys(const oracle_shape* sh, const int32_t* idx_row, int64_t p, int64_t* keys) {
  int64_t n = 0;
  const int64_t bk = sh->block_k;
  if (idx_row) {
    const int32_t nnz = idx_row[0];
    for (int32_t t = 0; t < nnz; ++t) {
      const int64_t c = idx_row[1 + t];
      for (int64_t j = c * bk; j < c * bk + bk; ++j)
        if (j < sh->mask_len && j <= p) keys[n++] = j;
    }
    for (int64_t j = sh->mask_len; j < sh->seq_len && j <= p; ++j) keys[n++] = j;
  } else {
    for (int64_t j = 0; j < sh->seq_len && j <= p; ++j) keys[n++] = j;
  }
  return n;
}

/*
 * Attention rows (row = (b * Hq + h) * q_len + i), or all rows when
 * rows == NULL; out is [n_rows, d] fp32. idx == NULL gives dense causal
 * attention over every key j <= p, j < seq_len.
 */
int oracle_attention(const float* q, const float* k, const float* v, const int32_t* idx,
                     const oracle_shape* sh, const int64_t* rows, int64_t n_rows, float* out) {
  if (!q || !k || !v || !out || !shape_ok(sh)) return OR_BAD;
  const int64_t total = (int64_t)sh->batch * sh->n_qheads * sh->q_len;
  if (!rows) n_rows = total;
  const int d = sh->head_dim, G = sh->n_qheads / sh->n_kvheads;
  const int64_t nqb = oracle_num_qblocks(sh), stride = 1 + oracle_idx_cap(sh);
  int status = OR_OK;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < n_rows; ++r) {
    const int64_t row = rows ? rows[r] : r;
    if (row < 0 || row >= total) {
#pragma omp critical
      status = OR_BAD;
      continue;
    }
    const int64_t i = row % sh->q_len, h = (row / sh->q_len) % sh->n_qheads;
    const int64_t b = row / ((int64_t)sh->q_len * sh->n_qheads), g = h / G;
    const int64_t p = sh->q_pos0 + i;
    const int64_t mrow = sh->per_head ? b * sh->n_qheads + h : b * sh->n_kvheads + g;  /* idx head row */
    const int32_t* idx_row = idx ? idx + (mrow * nqb + i / sh->block_q) * stride : NULL;
    if (idx_row && (idx_row[0] < 0 || idx_row[0] > stride - 1)) {
#pragma omp critical
      status = OR_BAD;
      continue;
    }
    int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)(sh->seq_len + 1));
    if (!keys) {
#pragma omp critical
      status = OR_NOMEM;
      continue;
    }
    const int64_t nk = row_keys(sh, idx_row, p, keys);
    const int64_t kv_off = (b * sh->n_kvheads + g) * sh->kv_capacity * d;
    attend(q + row * d, k + kv_off, v + kv_off, d, keys, nk, out + r * d);
    free(keys);
  }
  return status;
}
