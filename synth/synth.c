/*
 * Seeded synthetic inputs for MoBA causal prefill: Q, K, V of shape [T, H, D].
 *
 * This file is input preparation only.  It computes none of the attention
 * method's arithmetic (no pooling, gating, selection or softmax); both the
 * CPU oracle's tests and the GPU path's callers read the buffers it fills.
 *
 * Element definition (counter based, so any element can be produced alone):
 *   stream(seed, id)   = splitmix64(splitmix64(seed) ^ (id * 0x9E3779B97F4A7C15))
 *   word(stream, n)    = splitmix64(stream + n)
 *   pair n of a tensor: u1 = ((word(2n) >> 11) + 1) * 2^-53   in (0, 1]
 *                       u2 =  (word(2n+1) >> 11)     * 2^-53   in [0, 1)
 *                       R  = sqrt(-2 ln u1),  a = 2 pi u2       (Box-Muller, fp64)
 *   element e (flat index into [T,H,D]) = (float)(R cos a) if e even, (float)(R sin a) if odd
 *
 *   Rotary embedding (rotate-half form used by Llama-family models), optional:
 *   position p = t - cu_seqlens[s] (restarts at each sequence), for d < D/2,
 *   angle = p * theta^(-2d/D) in fp64, c = (float)cos(angle), s = (float)sin(angle),
 *   x[d] <- x[d]*c - x[d+D/2]*s,  x[d+D/2] <- x[d+D/2]*c + x[d]*s   (fp32, no fused multiply-add).
 *
 *   Planted relevance, optional, added after the rotary step (amplitude A, e.g. 0.5):
 *   u_g = unit vector from normals of stream id 4 (index g*D + d), one per KV head g.
 *   For every sequence s, KV head g and query block i >= 1 a target block
 *   r(s,i,g) = floor(U * i) with U = (word of stream id 5 at (s * 2^20 + i) * Hkv + g >> 11) * 2^-53.
 *   Keys of block r get A * c * u_g where c counts the query blocks targeting r;
 *   queries of block i >= 1 (all query heads of group g) get A * u_g.  V gets none.
 *   The sum is formed in fp64 and rounded to fp32, then (optionally) to bf16 by
 *   round-to-nearest-even.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SYNTH_ID_Q 1u
#define SYNTH_ID_K 2u
#define SYNTH_ID_V 3u
#define SYNTH_ID_U 4u
#define SYNTH_ID_R 5u

typedef struct {
  uint64_t seed;
  int32_t num_seqs;
  const int32_t* cu_seqlens; /* host, num_seqs + 1 entries */
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size; /* used by the plant only */
  double rope_theta;  /* <= 0: no rotary embedding */
  double plant;       /* 0: no planted relevance */
} synth_spec;

static inline uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint32_t id) {
  return splitmix64(splitmix64(seed) ^ ((uint64_t)id * 0x9E3779B97F4A7C15ull));
}

static const double kTwoPi = 6.283185307179586476925286766559;

/* Normal sample number e of the stream (fp64, before rounding). */
static inline double normal_at(uint64_t key, uint64_t e) {
  uint64_t n = e >> 1;
  uint64_t w1 = splitmix64(key + 2 * n);
  uint64_t w2 = splitmix64(key + 2 * n + 1);
  double u1 = (double)((w1 >> 11) + 1) * 0x1.0p-53;
  double u2 = (double)(w2 >> 11) * 0x1.0p-53;
  double r = sqrt(-2.0 * log(u1));
  double a = kTwoPi * u2;
  return (e & 1) ? r * sin(a) : r * cos(a);
}

uint64_t synth_splitmix64(uint64_t x) { return splitmix64(x); }
double synth_normal(uint64_t seed, uint32_t id, uint64_t e) {
  return normal_at(stream_key(seed, id), e);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

static int seq_of_token(const synth_spec* sp, int64_t t) {
  int lo = 0, hi = sp->num_seqs - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (sp->cu_seqlens[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

/* target block of query block i (>= 1) for KV head g of sequence s */
static inline int32_t plant_target(uint64_t rkey, int s, int32_t i, int g, int hkv) {
  uint64_t idx = (((uint64_t)s << 20) + (uint64_t)i) * (uint64_t)hkv + (uint64_t)g;
  double u = (double)(splitmix64(rkey + idx) >> 11) * 0x1.0p-53;
  int32_t r = (int32_t)floor(u * (double)i);
  if (r >= i) r = i - 1;
  return r;
}

typedef struct {
  const synth_spec* sp;
  int which; /* 0 Q, 1 K, 2 V */
  const int64_t* tok; /* row list (NULL: contiguous t0..) */
  const int32_t* head; /* row heads for row lists */
  int64_t t0;
  int64_t n; /* rows (token rows for contiguous mode, (t,h) rows for list mode) */
  int out_kind; /* 0 fp32, 1 bf16 */
  void* out;
  const double* u;          /* [Hkv, D] unit vectors, or NULL */
  const int32_t* kcount;    /* per (s, g, block) plant counts for K, or NULL */
  const int64_t* kcount_off;/* per-sequence offset into kcount */
  int64_t lo, hi;           /* this worker's share */
} job_t;

/* cos/sin of the rotary angles of position p (fp64 angle, rounded to fp32) */
static void rope_table(const synth_spec* sp, int64_t p, float* cosv, float* sinv) {
  const int D = sp->head_dim;
  for (int d = 0; d < D / 2; ++d) {
    double inv = pow(sp->rope_theta, -2.0 * (double)d / (double)D);
    double ang = (double)p * inv;
    cosv[d] = (float)cos(ang);
    sinv[d] = (float)sin(ang);
  }
}

/* Produce one [D] row (token t, head h) into dst; cosv/sinv hold the rotary
 * table of t's position when the spec asks for rotary embedding. */
static void make_row(const job_t* j, int64_t t, int h, const float* cosv, const float* sinv,
                     float* dst) {
  const synth_spec* sp = j->sp;
  const int D = sp->head_dim;
  const int H = (j->which == 0) ? sp->num_q_heads : sp->num_kv_heads;
  const uint32_t id = (j->which == 0) ? SYNTH_ID_Q : (j->which == 1 ? SYNTH_ID_K : SYNTH_ID_V);
  const uint64_t key = stream_key(sp->seed, id);
  const uint64_t base = ((uint64_t)t * (uint64_t)H + (uint64_t)h) * (uint64_t)D;
  float x[512];
  for (int d = 0; d < D; d += 2) {
    /* base and D are even, so each row holds whole Box-Muller pairs */
    uint64_t n = (base + (uint64_t)d) >> 1;
    uint64_t w1 = splitmix64(key + 2 * n);
    uint64_t w2 = splitmix64(key + 2 * n + 1);
    double u1 = (double)((w1 >> 11) + 1) * 0x1.0p-53;
    double u2 = (double)(w2 >> 11) * 0x1.0p-53;
    double r = sqrt(-2.0 * log(u1));
    double a = kTwoPi * u2;
    x[d] = (float)(r * cos(a));
    x[d + 1] = (float)(r * sin(a));
  }
  int s = -1;
  int64_t p = 0;
  if (sp->rope_theta > 0.0 || (sp->plant != 0.0 && j->which != 2)) {
    s = seq_of_token(sp, t);
    p = t - sp->cu_seqlens[s];
  }
  if (sp->rope_theta > 0.0 && j->which != 2) {
    const int half = D / 2;
    for (int d = 0; d < half; ++d) {
      float c = cosv[d], sn = sinv[d];
      float x1 = x[d], x2 = x[d + half];
      float a = x1 * c, b = x2 * sn;
      float e = x2 * c, f = x1 * sn;
      x[d] = a - b;
      x[d + half] = e + f;
    }
  }
  if (sp->plant != 0.0 && j->which != 2) {
    const int G = sp->num_q_heads / sp->num_kv_heads;
    const int g = (j->which == 0) ? h / G : h;
    const int32_t blk = (int32_t)(p / sp->block_size);
    double amp = 0.0;
    if (j->which == 0) {
      amp = (blk >= 1) ? sp->plant : 0.0;
    } else {
      int64_t nb = ((int64_t)(sp->cu_seqlens[s + 1] - sp->cu_seqlens[s]) + sp->block_size - 1) / sp->block_size;
      amp = sp->plant * (double)j->kcount[j->kcount_off[s] + (int64_t)g * nb + blk];
    }
    if (amp != 0.0)
      for (int d = 0; d < D; ++d) x[d] = (float)((double)x[d] + amp * j->u[g * D + d]);
  }
  memcpy(dst, x, sizeof(float) * (size_t)D);
}

static void* worker(void* arg) {
  job_t* j = (job_t*)arg;
  const synth_spec* sp = j->sp;
  const int D = sp->head_dim;
  const int H = (j->which == 0) ? sp->num_q_heads : sp->num_kv_heads;
  float row[512];
  float cosv[256], sinv[256];
  const int rope = sp->rope_theta > 0.0 && j->which != 2;
  for (int64_t r = j->lo; r < j->hi; ++r) {
    if (j->tok == NULL) {
      /* contiguous: r indexes token rows; write all H heads */
      int64_t t = j->t0 + r;
      if (rope) rope_table(sp, t - sp->cu_seqlens[seq_of_token(sp, t)], cosv, sinv);
      for (int h = 0; h < H; ++h) {
        make_row(j, t, h, cosv, sinv, row);
        size_t off = ((size_t)r * (size_t)H + (size_t)h) * (size_t)D;
        if (j->out_kind == 0) memcpy((float*)j->out + off, row, sizeof(float) * (size_t)D);
        else for (int d = 0; d < D; ++d) ((uint16_t*)j->out)[off + d] = f32_to_bf16_rne(row[d]);
      }
    } else {
      int64_t t = j->tok[r];
      if (rope) rope_table(sp, t - sp->cu_seqlens[seq_of_token(sp, t)], cosv, sinv);
      make_row(j, t, j->head[r], cosv, sinv, row);
      size_t off = (size_t)r * (size_t)D;
      if (j->out_kind == 0) memcpy((float*)j->out + off, row, sizeof(float) * (size_t)D);
      else for (int d = 0; d < D; ++d) ((uint16_t*)j->out)[off + d] = f32_to_bf16_rne(row[d]);
    }
  }
  return NULL;
}

static int check_spec(const synth_spec* sp) {
  if (!sp || sp->num_seqs < 1 || !sp->cu_seqlens) return 1;
  if (sp->head_dim < 2 || sp->head_dim > 512 || (sp->head_dim & 1)) return 2;
  if (sp->num_q_heads < 1 || sp->num_kv_heads < 1 || sp->num_q_heads % sp->num_kv_heads) return 3;
  if (sp->block_size < 1) return 4;
  if (sp->cu_seqlens[0] != 0) return 5;
  for (int s = 0; s < sp->num_seqs; ++s)
    if (sp->cu_seqlens[s + 1] < sp->cu_seqlens[s]) return 5;
  return 0;
}

static int run(const synth_spec* sp, int which, const int64_t* tok, const int32_t* head,
               int64_t t0, int64_t n, int out_kind, void* out, int nthreads) {
  int rc = check_spec(sp);
  if (rc) return rc;
  if (which < 0 || which > 2 || n < 0 || !out) return 6;
  const int D = sp->head_dim, hkv = sp->num_kv_heads;
  double* u = NULL;
  int32_t* kcount = NULL;
  int64_t* koff = NULL;
  if (sp->plant != 0.0 && which != 2) {
    u = (double*)malloc(sizeof(double) * (size_t)hkv * (size_t)D);
    const uint64_t ukey = stream_key(sp->seed, SYNTH_ID_U);
    for (int g = 0; g < hkv; ++g) {
      double nrm = 0.0;
      for (int d = 0; d < D; ++d) {
        double v = normal_at(ukey, (uint64_t)g * (uint64_t)D + (uint64_t)d);
        u[g * D + d] = v;
        nrm += v * v;
      }
      nrm = sqrt(nrm);
      for (int d = 0; d < D; ++d) u[g * D + d] /= nrm;
    }
    if (which == 1) {
      koff = (int64_t*)malloc(sizeof(int64_t) * (size_t)(sp->num_seqs + 1));
      int64_t tot = 0;
      for (int s = 0; s < sp->num_seqs; ++s) {
        koff[s] = tot;
        int64_t nb = ((int64_t)(sp->cu_seqlens[s + 1] - sp->cu_seqlens[s]) + sp->block_size - 1) / sp->block_size;
        tot += nb * hkv;
      }
      koff[sp->num_seqs] = tot;
      kcount = (int32_t*)calloc((size_t)(tot > 0 ? tot : 1), sizeof(int32_t));
      const uint64_t rkey = stream_key(sp->seed, SYNTH_ID_R);
      for (int s = 0; s < sp->num_seqs; ++s) {
        int64_t nb = ((int64_t)(sp->cu_seqlens[s + 1] - sp->cu_seqlens[s]) + sp->block_size - 1) / sp->block_size;
        for (int g = 0; g < hkv; ++g)
          for (int32_t i = 1; i < nb; ++i)
            kcount[koff[s] + (int64_t)g * nb + plant_target(rkey, s, i, g, hkv)] += 1;
      }
    }
  }
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > n) nthreads = (int)(n > 0 ? n : 1);
  pthread_t th[256];
  job_t jobs[256];
  for (int i = 0; i < nthreads; ++i) {
    job_t* j = &jobs[i];
    j->sp = sp; j->which = which; j->tok = tok; j->head = head; j->t0 = t0; j->n = n;
    j->out_kind = out_kind; j->out = out; j->u = u; j->kcount = kcount; j->kcount_off = koff;
    j->lo = n * i / nthreads; j->hi = n * (i + 1) / nthreads;
  }
  for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &jobs[i]);
  worker(&jobs[0]);
  for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(u); free(kcount); free(koff);
  return 0;
}

/* Fill token rows [t0, t1) of tensor `which` (0 Q, 1 K, 2 V) as [t1-t0, H, D]. */
int synth_fill(const synth_spec* sp, int which, int64_t t0, int64_t t1, int out_kind,
               void* out, int nthreads) {
  if (t1 < t0 || t0 < 0) return 7;
  if (sp && sp->cu_seqlens && t1 > sp->cu_seqlens[sp->num_seqs]) return 7;
  return run(sp, which, NULL, NULL, t0, t1 - t0, out_kind, out, nthreads);
}

/* Produce n individual (token, head) rows of tensor `which` as [n, D]. */
int synth_rows(const synth_spec* sp, int which, const int64_t* tok, const int32_t* head,
               int64_t n, int out_kind, void* out, int nthreads) {
  if (!tok || !head) return 8;
  return run(sp, which, tok, head, 0, n, out_kind, out, nthreads);
}

/* Target block of query block i for KV head g of sequence s (exposed for tests). */
int32_t synth_plant_target(uint64_t seed, int s, int32_t i, int g, int hkv) {
  if (i < 1) return -1;
  return plant_target(stream_key(seed, SYNTH_ID_R), s, i, g, hkv);
}
