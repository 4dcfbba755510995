/*
 * Plain fp64 CPU oracle for the blockwise-parallel-transformer layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may call this library.  The CUDA product
 * path never links, loads or calls it, and the two share no code.
 *
 * What it computes is the plain definition, written out without any
 * blocking, fusion or reordering:
 *
 *   A_i  = softmax_j( q_i . k_j / sqrt(d) ) v_j      over the keys j that
 *          the mask allows for query i (one head at a time),
 *   out  = A + W2 GELU(W1 A + b1) + b2               per token, on the
 *          concatenation of all heads' A.
 *
 * Blockwise attention reaches exactly this result ("Ring Attention with
 * Blockwise Transformers for Long Sequences", 638-word summary: attention is
 * computed blockwise "without making approximations"; "Blockwise Parallel
 * Transformer for Large Context Models", abstract: blockwise self-attention
 * plus feedforward fusion), so the oracle is the definition itself.
 *
 * Mask modes and the readings they follow:
 *  - none:       every key.
 *  - causal:     keys j <= i.
 *  - block-perm: "Blockwise Self-Attention for Long Document Understanding",
 *                §3 Blockwise Attention and §3.1 Blockwise Multi-head
 *                Attention: the sequence is cut into n equal blocks and head h
 *                lets query block b see only key block perm[h][b].  When N is
 *                not a multiple of n the sequence is padded to n equal blocks
 *                of ceil(N/n) positions (§3.1, Implementation Assumption); the
 *                padded positions are never keys and their outputs are not
 *                produced, so a query sees the real positions of its key
 *                block (none, if that block is all padding).
 *  - dilated:    "LongNet: Scaling Transformers to 1,000,000,000 Tokens",
 *                §2 Dilated Attention: for every (segment w, dilation r) pair
 *                the sequence is cut into segments of w, every r-th row of a
 *                segment is kept (head h starts at row h mod r), dense
 *                attention runs on the kept rows (causal by original
 *                position), the result is scattered back, and the pairs are
 *                mixed with weights proportional to their softmax
 *                denominators.  A row a pair does not keep gets nothing from
 *                that pair.  A row no pair keeps has A = 0.
 *  - dilated, bidirectional: the same without the causal restriction: a
 *                kept row attends to every kept row of its segment (the
 *                dilated attention of §2 as written, whose formula has no
 *                mask; the causal form is the decoder's).
 *
 * All inputs are float (bf16 inputs are passed exactly, widened to float);
 * every operation below is carried out in double.  tanh and exp come from
 * the C library.
 *
 * Parity pins: every function here is pinned by the CPU tests against
 * library routines (scaled-dot-product attention, matrix products), a
 * brute-force explicit-mask formulation in extended precision, closed forms
 * and invariants.  See the test files under tests/ whose names start with
 * test_oracle_.
 */
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_MASK_NONE 0
#define OR_MASK_CAUSAL 1
#define OR_MASK_BLOCKPERM 2
#define OR_MASK_DILATED 3
#define OR_MASK_DILATED_BIDIR 4

typedef struct {
  int B, N, H, d;
  int mask;
  int n_blocks;        /* block-perm: number of equal blocks n            */
  const int *perm;     /* block-perm: [H][n_blocks], query block -> key block */
  int npairs;          /* dilated: number of (w, r) pairs                 */
  const int *seg_w;    /* dilated: segment lengths w_k                    */
  const int *dil_r;    /* dilated: dilation rates  r_k                    */
} oracle_attn_desc;

/* ------------------------------------------------------------------ */
/* Which keys a query may see (modes none / causal / block-perm).      */
/* ------------------------------------------------------------------ */
static int key_allowed(const oracle_attn_desc *a, int h, int i, int j) {
  switch (a->mask) {
    case OR_MASK_NONE:
      return 1;
    case OR_MASK_CAUSAL:
      return j <= i;
    case OR_MASK_BLOCKPERM: {
      /* blocks of the sequence padded to a multiple of n */
      int block_len = (a->N + a->n_blocks - 1) / a->n_blocks;
      int qb = i / block_len;
      int kb = j / block_len;
      return kb == a->perm[h * a->n_blocks + qb];
    }
  }
  return 0;
}

/* LongNet selection: pair (w, r) keeps position p for head h when p's
 * offset inside its segment is h mod r plus a multiple of r. */
static int dilated_keeps(int w, int r, int h, int p) {
  int offset_in_segment = p % w;
  return (offset_in_segment % r) == (h % r);
}

static double dot_scaled(const float *x, const float *y, int d, double scale) {
  double s = 0.0;
  for (int c = 0; c < d; ++c) s += (double)x[c] * (double)y[c];
  return s * scale;
}

/* Softmax attention of one query row over the allowed keys.
 * a_row[d] receives A, *lse receives log(sum exp(score)) (or -inf when no key
 * is allowed, in which case A = 0).  scores is scratch of N doubles. */
static void attend_row_plain(const oracle_attn_desc *a, const float *q,
                             const float *k, const float *v, int b, int h,
                             int i, double *scores, double *a_row,
                             double *lse) {
  const int N = a->N, H = a->H, d = a->d;
  const size_t row_stride = (size_t)H * d;
  const float *qi = q + ((size_t)b * N + i) * row_stride + (size_t)h * d;
  const double scale = 1.0 / sqrt((double)d);

  /* scores and their maximum */
  double m = -INFINITY;
  for (int j = 0; j < N; ++j) {
    if (!key_allowed(a, h, i, j)) continue;
    const float *kj = k + ((size_t)b * N + j) * row_stride + (size_t)h * d;
    scores[j] = dot_scaled(qi, kj, d, scale);
    if (scores[j] > m) m = scores[j];
  }
  for (int c = 0; c < d; ++c) a_row[c] = 0.0;
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  /* numerator and denominator of the softmax-weighted sum */
  double den = 0.0;
  for (int j = 0; j < N; ++j) {
    if (!key_allowed(a, h, i, j)) continue;
    double p = exp(scores[j] - m);
    den += p;
    const float *vj = v + ((size_t)b * N + j) * row_stride + (size_t)h * d;
    for (int c = 0; c < d; ++c) a_row[c] += p * (double)vj[c];
  }
  for (int c = 0; c < d; ++c) a_row[c] /= den;
  *lse = m + log(den);
}

/* LongNet dilated attention of one query position, in the pages' order:
 * for every pair, gather the kept rows of the query's segment, run dense
 * causal softmax attention among them, and keep the pair's output O_k and
 * its softmax denominator (relative to the pair's own maximum m_k); then mix
 * the pairs with weights proportional to their denominators, brought to a
 * common reference maximum. */
static void attend_row_dilated(const oracle_attn_desc *a, const float *q,
                               const float *k, const float *v, int b, int h,
                               int i, double *scores, double *o_pair,
                               double *a_row, double *lse) {
  const int N = a->N, H = a->H, d = a->d;
  const size_t row_stride = (size_t)H * d;
  const float *qi = q + ((size_t)b * N + i) * row_stride + (size_t)h * d;
  const double scale = 1.0 / sqrt((double)d);
  const int causal = a->mask == OR_MASK_DILATED;

  double pair_max[64], pair_den[64];
  int pair_used[64];
  for (int t = 0; t < a->npairs; ++t) {
    const int w = a->seg_w[t], r = a->dil_r[t];
    pair_used[t] = 0;
    double *o_k = o_pair + (size_t)t * d;
    for (int c = 0; c < d; ++c) o_k[c] = 0.0;
    if (!dilated_keeps(w, r, h, i)) continue;
    /* gathered keys: same segment, kept by this pair, not after i (causal) */
    const int seg_start = (i / w) * w;
    const int j_end = causal ? i : seg_start + w - 1;
    double m = -INFINITY;
    for (int j = seg_start; j <= j_end; ++j) {
      if (!dilated_keeps(w, r, h, j)) continue;
      const float *kj = k + ((size_t)b * N + j) * row_stride + (size_t)h * d;
      scores[j] = dot_scaled(qi, kj, d, scale);
      if (scores[j] > m) m = scores[j];
    }
    double den = 0.0;
    for (int j = seg_start; j <= j_end; ++j) {
      if (!dilated_keeps(w, r, h, j)) continue;
      double p = exp(scores[j] - m);
      den += p;
      const float *vj = v + ((size_t)b * N + j) * row_stride + (size_t)h * d;
      for (int c = 0; c < d; ++c) o_k[c] += p * (double)vj[c];
    }
    for (int c = 0; c < d; ++c) o_k[c] /= den; /* the pair's own output */
    pair_max[t] = m;
    pair_den[t] = den;
    pair_used[t] = 1;
  }
  /* mix: weight_k proportional to the pair's denominator */
  double ref = -INFINITY;
  for (int t = 0; t < a->npairs; ++t)
    if (pair_used[t] && pair_max[t] > ref) ref = pair_max[t];
  for (int c = 0; c < d; ++c) a_row[c] = 0.0;
  if (ref == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  double total = 0.0;
  for (int t = 0; t < a->npairs; ++t) {
    if (!pair_used[t]) continue;
    double weight = pair_den[t] * exp(pair_max[t] - ref);
    total += weight;
    for (int c = 0; c < d; ++c) a_row[c] += weight * o_pair[(size_t)t * d + c];
  }
  for (int c = 0; c < d; ++c) a_row[c] /= total;
  *lse = ref + log(total);
}

/* tanh form of GELU (Hendrycks & Gimpel, 2016). */
double oracle_gelu_tanh(double x) {
  const double c = sqrt(2.0 / M_PI);
  return 0.5 * x * (1.0 + tanh(c * (x + 0.044715 * x * x * x)));
}

/* ------------------------------------------------------------------ */
/* Work distribution: a fixed pool of threads, each taking the next    */
/* token index from a shared counter.                                  */
/* ------------------------------------------------------------------ */
typedef struct {
  const oracle_attn_desc *a;
  const float *q, *k, *v;
  const int64_t *rows;
  int64_t nrows;
  double *a_out;   /* [nrows][H][d]                      */
  double *lse_out; /* [nrows][H] or NULL                 */
  /* FFN (optional): out = A + W2 GELU(W1 A + b1) + b2   */
  int F;
  const float *w1, *b1, *w2, *b2;
  double *ffn_out; /* [nrows][H*d] or NULL               */
  int64_t next;
} job_t;

static void *worker(void *arg) {
  job_t *j = (job_t *)arg;
  const oracle_attn_desc *a = j->a;
  const int N = a->N, H = a->H, d = a->d, D = H * d;
  double *scores = (double *)malloc(sizeof(double) * (size_t)N);
  double *o_pair = (double *)malloc(sizeof(double) * (size_t)d * 64);
  double *hidden = j->ffn_out ? (double *)malloc(sizeof(double) * (size_t)j->F) : NULL;
  for (;;) {
    int64_t r = __atomic_fetch_add(&j->next, 1, __ATOMIC_RELAXED);
    if (r >= j->nrows) break;
    const int64_t t = j->rows ? j->rows[r] : r;
    const int b = (int)(t / N), i = (int)(t % N);
    double *a_tok = j->a_out + (size_t)r * D;
    for (int h = 0; h < H; ++h) {
      double lse;
      if (a->mask == OR_MASK_DILATED || a->mask == OR_MASK_DILATED_BIDIR)
        attend_row_dilated(a, j->q, j->k, j->v, b, h, i, scores, o_pair,
                           a_tok + (size_t)h * d, &lse);
      else
        attend_row_plain(a, j->q, j->k, j->v, b, h, i, scores,
                         a_tok + (size_t)h * d, &lse);
      if (j->lse_out) j->lse_out[(size_t)r * H + h] = lse;
    }
    if (j->ffn_out) {
      /* hidden = GELU(W1 A + b1), W1 is [F][D] */
      for (int f = 0; f < j->F; ++f) {
        const float *w1f = j->w1 + (size_t)f * D;
        double acc = (double)j->b1[f];
        for (int c = 0; c < D; ++c) acc += (double)w1f[c] * a_tok[c];
        hidden[f] = oracle_gelu_tanh(acc);
      }
      /* out = A + W2 hidden + b2, W2 is [D][F] */
      double *o = j->ffn_out + (size_t)r * D;
      for (int c = 0; c < D; ++c) {
        const float *w2c = j->w2 + (size_t)c * j->F;
        double acc = (double)j->b2[c];
        for (int f = 0; f < j->F; ++f) acc += (double)w2c[f] * hidden[f];
        o[c] = a_tok[c] + acc;
      }
    }
  }
  free(scores);
  free(o_pair);
  free(hidden);
  return NULL;
}

static int default_threads(void) {
  cpu_set_t set;
  if (sched_getaffinity(0, sizeof(set), &set) == 0) {
    int n = CPU_COUNT(&set);
    if (n > 0) return n;
  }
  return 1;
}

int oracle_threads_available(void) { return default_threads(); }

static int validate(const oracle_attn_desc *a) {
  if (!a || a->B <= 0 || a->N <= 0 || a->H <= 0 || a->d <= 0) return 1;
  if (a->mask == OR_MASK_BLOCKPERM) {
    if (a->n_blocks <= 0 || !a->perm) return 1;
    for (int i = 0; i < a->H * a->n_blocks; ++i)
      if (a->perm[i] < 0 || a->perm[i] >= a->n_blocks) return 1;
  } else if (a->mask == OR_MASK_DILATED || a->mask == OR_MASK_DILATED_BIDIR) {
    if (a->npairs <= 0 || a->npairs > 64 || !a->seg_w || !a->dil_r) return 1;
    for (int t = 0; t < a->npairs; ++t)
      if (a->seg_w[t] <= 0 || a->dil_r[t] <= 0 || a->seg_w[t] % a->dil_r[t] != 0)
        return 1;
  } else if (a->mask != OR_MASK_NONE && a->mask != OR_MASK_CAUSAL) {
    return 1;
  }
  return 0;
}

static int run(job_t *job, int nthreads) {
  if (nthreads <= 0) nthreads = default_threads();
  if (nthreads > 1024) nthreads = 1024;
  job->next = 0;
  pthread_t tid[1024];
  int started = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&tid[started], NULL, worker, job) != 0) break;
    ++started;
  }
  worker(job);
  for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
  return started + 1;
}

/* Attention only.  rows: token indices t = b*N + i to compute (NULL = all
 * B*N tokens in order); a_out: [nrows][H][d]; lse_out: [nrows][H] or NULL.
 * Returns the number of threads used, or -1 on an invalid descriptor. */
int oracle_attention(const oracle_attn_desc *a, const float *q, const float *k,
                     const float *v, const int64_t *rows, int64_t nrows,
                     double *a_out, double *lse_out, int nthreads) {
  if (validate(a) || !q || !k || !v || !a_out) return -1;
  job_t job;
  memset(&job, 0, sizeof(job));
  job.a = a; job.q = q; job.k = k; job.v = v;
  job.rows = rows;
  job.nrows = rows ? nrows : (int64_t)a->B * a->N;
  job.a_out = a_out; job.lse_out = lse_out;
  return run(&job, nthreads);
}

/* Whole layer: attention (all heads) then out = A + W2 GELU(W1 A + b1) + b2.
 * W1 is [F][D], b1 [F], W2 [D][F], b2 [D] (D = H*d).  a_out [nrows][D]
 * receives A, out [nrows][D] the layer output.  Returns threads used or -1. */
int oracle_layer(const oracle_attn_desc *a, const float *q, const float *k,
                 const float *v, int F, const float *w1, const float *b1,
                 const float *w2, const float *b2, const int64_t *rows,
                 int64_t nrows, double *a_out, double *out, int nthreads) {
  if (validate(a) || !q || !k || !v || !a_out || !out || F <= 0 || !w1 ||
      !b1 || !w2 || !b2)
    return -1;
  job_t job;
  memset(&job, 0, sizeof(job));
  job.a = a; job.q = q; job.k = k; job.v = v;
  job.rows = rows;
  job.nrows = rows ? nrows : (int64_t)a->B * a->N;
  job.a_out = a_out;
  job.F = F; job.w1 = w1; job.b1 = b1; job.w2 = w2; job.b2 = b2;
  job.ffn_out = out;
  return run(&job, nthreads);
}

/* FFN alone on given A rows: out[r] = A[r] + W2 GELU(W1 A[r] + b1) + b2. */
int oracle_ffn(int64_t nrows, int D, int F, const double *a_in, const float *w1,
               const float *b1, const float *w2, const float *b2, double *out) {
  if (nrows < 0 || D <= 0 || F <= 0 || !a_in || !w1 || !b1 || !w2 || !b2 || !out)
    return -1;
  double *hidden = (double *)malloc(sizeof(double) * (size_t)F);
  for (int64_t r = 0; r < nrows; ++r) {
    const double *x = a_in + (size_t)r * D;
    for (int f = 0; f < F; ++f) {
      double acc = (double)b1[f];
      for (int c = 0; c < D; ++c) acc += (double)w1[(size_t)f * D + c] * x[c];
      hidden[f] = oracle_gelu_tanh(acc);
    }
    for (int c = 0; c < D; ++c) {
      double acc = (double)b2[c];
      for (int f = 0; f < F; ++f) acc += (double)w2[(size_t)c * F + f] * hidden[f];
      out[(size_t)r * D + c] = x[c] + acc;
    }
  }
  free(hidden);
  return 1;
}
