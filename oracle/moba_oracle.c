/*
 * MoBA (Mixture of Block Attention) causal prefill -- CPU oracle, fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow reference that the
 * GPU library is checked against.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the library never does.  It shares
 * no code, header or table with the GPU path.
 *
 * Sources (web pages about MoBA; cited by page title and section):
 *   [README]  "MoBA: Mixture of Block Attention for Long-Context LLMs", the
 *             project README as mirrored on gittoolsai.com: bullets
 *             "Trainable Block Sparse Attention", "Parameter-less Gating
 *             Mechanism"; section "Implementation Details" (moba_naive is the
 *             attention-mask form); its FAQ answers taken from GitHub issue #27
 *             (top-k minus one for the forced current block; the last chunk is
 *             never a gating candidate) and the FAQ on forcing the current block
 *             (mean pooling over the current block would leak future tokens).
 *   [KIMI]    youleyou.com, "Kimi发布MoBA突破性实现无限上下文", sections
 *             "MoBA：基于块的混合注意力机制" (equal-length blocks, mean-pooled keys,
 *             own block always chosen, causal mask) and "PyTorch实现关键要点"
 *             (pool, score by product with the query, mask future blocks, top-k,
 *             attention on own block and chosen blocks, merge by online softmax).
 *   [GUIDE]   bxzpzcl.cn, "MoBA终极指南…", section "MoBA核心技术原理深度解析"
 *             (rotary embedding, then mean pooling, then top-k gating).
 *   [OVERVIEW] zhuoshang.net, "MoBA是什么？…", section "MoBA的技术原理"
 *             (no attention to future blocks; causal mask in the current block).
 *
 * What it computes, for every query row (token t of sequence s at local position
 * p, query head h, KV head g = h / (Hq/Hkv)), following the mask-based form:
 *   1. Pool: Kbar[b] = mean of the keys of block b (valid tokens only).   [KIMI]
 *   2. Score: s_b = <q, Kbar[b]> for the past blocks b < i = floor(p/bs);
 *      parameter-free, no scale.                           [README], [KIMI]
 *   3. Select: the own block i always; plus the m = min(top_k - 1, i) past
 *      blocks of largest score (descending score, ties to the lower index).
 *      Block i is not a gating candidate and future blocks never are.
 *                                               [README FAQ #27], [KIMI]
 *   4. Materialise the block mask M[b] and the key mask keep[j] =
 *      M[floor(j/bs)] and j <= p.                     [README moba_naive]
 *   5. Masked softmax with scale 1/sqrt(D): LSE = ln sum_keep exp(z_j), O =
 *      sum_keep exp(z_j - LSE) V[j].               [KIMI], [OVERVIEW]
 * Everything in fp64; inputs are fp32 values or bf16 bit patterns widened
 * exactly.  Library primitives used as steps: libm exp/log, qsort.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int32_t num_seqs;
  const int32_t* cu_seqlens; /* num_seqs + 1 token offsets, [0] = 0, nondecreasing */
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;
  int32_t top_k;          /* counts the own block */
  double softmax_scale;   /* 0 => 1/sqrt(head_dim) */
  int32_t dtype;          /* 0: fp32 inputs, 1: bf16 bit patterns */
} oracle_problem;

enum { ORACLE_OK = 0, ORACLE_EINVAL = 1 };

static int check_problem(const oracle_problem* pr) {
  if (!pr || pr->num_seqs < 1 || !pr->cu_seqlens) return ORACLE_EINVAL;
  if (pr->num_q_heads < 1 || pr->num_kv_heads < 1) return ORACLE_EINVAL;
  if (pr->num_q_heads % pr->num_kv_heads) return ORACLE_EINVAL;
  if (pr->head_dim < 1 || pr->block_size < 1 || pr->top_k < 1) return ORACLE_EINVAL;
  if (pr->dtype != 0 && pr->dtype != 1) return ORACLE_EINVAL;
  if (pr->cu_seqlens[0] != 0) return ORACLE_EINVAL;
  for (int s = 0; s < pr->num_seqs; ++s)
    if (pr->cu_seqlens[s + 1] < pr->cu_seqlens[s]) return ORACLE_EINVAL;
  return ORACLE_OK;
}

static inline double widen(const void* base, int dtype, size_t idx) {
  if (dtype == 0) return (double)((const float*)base)[idx];
  uint32_t u = (uint32_t)((const uint16_t*)base)[idx] << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static inline int64_t blocks_in(int64_t len, int32_t bs) { return (len + bs - 1) / bs; }

/* Offsets of each sequence's first block in the sequence-ordered block list. */
int64_t oracle_block_offsets(const oracle_problem* pr, int64_t* blk_off /* num_seqs+1 */) {
  if (check_problem(pr)) return -1;
  int64_t tot = 0;
  for (int s = 0; s < pr->num_seqs; ++s) {
    if (blk_off) blk_off[s] = tot;
    tot += blocks_in(pr->cu_seqlens[s + 1] - pr->cu_seqlens[s], pr->block_size);
  }
  if (blk_off) blk_off[pr->num_seqs] = tot;
  return tot;
}

/* ---------------------------------------------------------------- threads */
typedef void (*range_fn)(void* ctx, int64_t lo, int64_t hi);
typedef struct { range_fn fn; void* ctx; int64_t lo, hi; } range_job;
static void* range_tramp(void* a) {
  range_job* j = (range_job*)a;
  j->fn(j->ctx, j->lo, j->hi);
  return NULL;
}
static void parallel_for(int64_t n, int nthreads, range_fn fn, void* ctx) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > n) nthreads = (int)(n > 0 ? n : 1);
  pthread_t th[256];
  range_job jobs[256];
  for (int i = 0; i < nthreads; ++i) {
    jobs[i].fn = fn; jobs[i].ctx = ctx;
    jobs[i].lo = n * i / nthreads; jobs[i].hi = n * (i + 1) / nthreads;
  }
  for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, range_tramp, &jobs[i]);
  range_tramp(&jobs[0]);
  for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------- 1. pooling */
typedef struct {
  const oracle_problem* pr;
  const void* K;
  double* Kbar;
  const int64_t* blk_off;
} pool_ctx;

static void pool_range(void* c, int64_t lo, int64_t hi) {
  pool_ctx* x = (pool_ctx*)c;
  const oracle_problem* pr = x->pr;
  const int D = pr->head_dim, hkv = pr->num_kv_heads, bs = pr->block_size;
  for (int64_t gb = lo; gb < hi; ++gb) {
    int s = 0;
    while (x->blk_off[s + 1] <= gb) ++s;
    int64_t b = gb - x->blk_off[s];
    int64_t t0 = pr->cu_seqlens[s] + b * bs;
    int64_t t1 = t0 + bs;
    if (t1 > pr->cu_seqlens[s + 1]) t1 = pr->cu_seqlens[s + 1];
    for (int g = 0; g < hkv; ++g) {
      double* out = x->Kbar + ((size_t)gb * hkv + g) * D;
      for (int d = 0; d < D; ++d) out[d] = 0.0;
      for (int64_t t = t0; t < t1; ++t)
        for (int d = 0; d < D; ++d) out[d] += widen(x->K, pr->dtype, ((size_t)t * hkv + g) * D + d);
      for (int d = 0; d < D; ++d) out[d] /= (double)(t1 - t0);
    }
  }
}

/* Kbar [NB, Hkv, D] (sequence-ordered blocks): mean of each block's keys. [KIMI] */
int oracle_pool_keys(const oracle_problem* pr, const void* K, double* Kbar, int nthreads) {
  if (check_problem(pr) || !K || !Kbar) return ORACLE_EINVAL;
  int64_t* off = (int64_t*)malloc(sizeof(int64_t) * (pr->num_seqs + 1));
  int64_t nb = oracle_block_offsets(pr, off);
  pool_ctx c = {pr, K, Kbar, off};
  parallel_for(nb, nthreads, pool_range, &c);
  free(off);
  return ORACLE_OK;
}

/* --------------------------------------------------- 2.-5. per query row */
typedef struct { double score; int32_t idx; } cand;

/* descending score; equal scores keep the lower block index first */
static int cand_cmp(const void* a, const void* b) {
  const cand* x = (const cand*)a;
  const cand* y = (const cand*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

typedef struct {
  const oracle_problem* pr;
  const void* Qrows;      /* [nrows, D] in the problem's dtype */
  const void* K;          /* [T, Hkv, D] */
  const void* V;          /* [T, Hkv, D] */
  const double* Kbar;     /* [NB, Hkv, D] */
  const int64_t* row_t;
  const int32_t* row_h;
  int32_t* sel;           /* [nrows, top_k] */
  double* gap;            /* [nrows] or NULL */
  double* gmax;           /* [nrows] or NULL */
  double* O;              /* [nrows, D] or NULL */
  double* lse;            /* [nrows] or NULL */
  uint8_t* mask_out;      /* [nrows, max_blocks] or NULL: the materialised block mask */
  int64_t max_blocks;
  const int64_t* blk_off;
  int err;
} rows_ctx;

static void rows_range(void* c, int64_t lo, int64_t hi) {
  rows_ctx* x = (rows_ctx*)c;
  const oracle_problem* pr = x->pr;
  const int D = pr->head_dim, hkv = pr->num_kv_heads, bs = pr->block_size, k = pr->top_k;
  const int G = pr->num_q_heads / hkv;
  const double scale = pr->softmax_scale > 0.0 ? pr->softmax_scale : 1.0 / sqrt((double)D);
  double* q = (double*)malloc(sizeof(double) * D);
  double* acc = (double*)malloc(sizeof(double) * D);
  cand* cs = (cand*)malloc(sizeof(cand) * (size_t)(x->max_blocks > 0 ? x->max_blocks : 1));
  uint8_t* M = (uint8_t*)malloc((size_t)(x->max_blocks > 0 ? x->max_blocks : 1));
  size_t zcap = (size_t)k * bs;
  double* z = (double*)malloc(sizeof(double) * zcap);
  for (int64_t r = lo; r < hi; ++r) {
    const int64_t t = x->row_t[r];
    const int h = x->row_h[r];
    int s = 0;
    while (pr->cu_seqlens[s + 1] <= t) ++s;
    const int64_t t_start = pr->cu_seqlens[s];
    const int64_t p = t - t_start;
    const int64_t nb_s = blocks_in(pr->cu_seqlens[s + 1] - t_start, bs);
    const int64_t i = p / bs;
    const int g = h / G;
    for (int d = 0; d < D; ++d) q[d] = widen(x->Qrows, pr->dtype, (size_t)r * D + d);

    /* 2. parameter-free gate scores against the past blocks only */
    double smax = 0.0;
    for (int64_t b = 0; b < i; ++b) {
      const double* kb = x->Kbar + ((size_t)(x->blk_off[s] + b) * hkv + g) * D;
      double sc = 0.0;
      for (int d = 0; d < D; ++d) sc += q[d] * kb[d];
      cs[b].score = sc;
      cs[b].idx = (int32_t)b;
      if (fabs(sc) > smax) smax = fabs(sc);
    }
    /* 3. own block always; top m of the past blocks by (score desc, index asc) */
    qsort(cs, (size_t)i, sizeof(cand), cand_cmp);
    const int64_t m = (k - 1 < i) ? (k - 1) : i;
    memset(M, 0, (size_t)nb_s);
    M[i] = 1;
    int32_t* sr = x->sel + (size_t)r * k;
    sr[0] = (int32_t)i;
    for (int64_t c2 = 0; c2 < m; ++c2) {
      M[cs[c2].idx] = 1;
      sr[1 + c2] = cs[c2].idx;
    }
    for (int64_t c2 = 1 + m; c2 < k; ++c2) sr[c2] = -1;
    if (x->gap) x->gap[r] = (m >= 1 && m < i) ? cs[m - 1].score - cs[m].score : INFINITY;
    if (x->gmax) x->gmax[r] = smax;
    if (x->mask_out) {
      uint8_t* mo = x->mask_out + (size_t)r * x->max_blocks;
      memset(mo, 0, (size_t)x->max_blocks);
      memcpy(mo, M, (size_t)nb_s);
    }
    if (!x->O && !x->lse) continue;

    /* 4.-5. key mask keep[j] = M[j / bs] && j <= p, then a masked softmax */
    size_t nz = 0;
    double zmax = -INFINITY;
    for (int64_t b = 0; b < nb_s; ++b) {
      if (!M[b]) continue;
      for (int64_t j = b * bs; j < (b + 1) * bs && j <= p; ++j) {
        const size_t kb = ((size_t)(t_start + j) * hkv + g) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * widen(x->K, pr->dtype, kb + d);
        if (nz >= zcap) { x->err = 1; break; }
        z[nz++] = scale * dot;
        if (scale * dot > zmax) zmax = scale * dot;
      }
    }
    double sum = 0.0;
    for (size_t n = 0; n < nz; ++n) sum += exp(z[n] - zmax);
    const double lse = zmax + log(sum);
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    nz = 0;
    for (int64_t b = 0; b < nb_s; ++b) {
      if (!M[b]) continue;
      for (int64_t j = b * bs; j < (b + 1) * bs && j <= p; ++j) {
        const double w = exp(z[nz++] - lse);
        const size_t vb = ((size_t)(t_start + j) * hkv + g) * D;
        for (int d = 0; d < D; ++d) acc[d] += w * widen(x->V, pr->dtype, vb + d);
      }
    }
    if (x->O) for (int d = 0; d < D; ++d) x->O[(size_t)r * D + d] = acc[d];
    if (x->lse) x->lse[r] = lse;
  }
  free(q); free(acc); free(cs); free(M); free(z);
}

/*
 * Oracle for a list of query rows (token row_t[r], query head row_h[r]).
 * Qrows holds those rows' query vectors [nrows, D]; K and V are whole
 * [T, Hkv, D] tensors; Kbar comes from oracle_pool_keys.
 * Outputs: sel [nrows, top_k] (slot 0 = own block, then chosen past blocks by
 * descending score, -1 padding; indices local to the sequence), gap (last chosen
 * minus best unchosen score, +inf when the choice is forced), gmax (max |score|
 * over the candidates), O [nrows, D], lse [nrows] (natural log, scaled logits),
 * mask [nrows, max_blocks] (optional).  Any output pointer except sel may be NULL.
 */
int oracle_rows(const oracle_problem* pr, const void* Qrows, const void* K, const void* V,
                const double* Kbar, const int64_t* row_t, const int32_t* row_h, int64_t nrows,
                int32_t* sel, double* gap, double* gmax, double* O, double* lse,
                uint8_t* mask, int nthreads) {
  if (check_problem(pr) || !Qrows || !Kbar || !row_t || !row_h || !sel) return ORACLE_EINVAL;
  if ((O || lse) && (!K || !V)) return ORACLE_EINVAL;
  const int64_t T = pr->cu_seqlens[pr->num_seqs];
  for (int64_t r = 0; r < nrows; ++r)
    if (row_t[r] < 0 || row_t[r] >= T || row_h[r] < 0 || row_h[r] >= pr->num_q_heads)
      return ORACLE_EINVAL;
  int64_t* off = (int64_t*)malloc(sizeof(int64_t) * (pr->num_seqs + 1));
  oracle_block_offsets(pr, off);
  int64_t mb = 0;
  for (int s = 0; s < pr->num_seqs; ++s) {
    int64_t nb = off[s + 1] - off[s];
    if (nb > mb) mb = nb;
  }
  rows_ctx c = {pr, Qrows, K, V, Kbar, row_t, row_h, sel, gap, gmax, O, lse, mask, mb, off, 0};
  parallel_for(nrows, nthreads, rows_range, &c);
  free(off);
  return c.err ? ORACLE_EINVAL : ORACLE_OK;
}
