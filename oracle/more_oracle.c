/*
 * fp64 oracle of the MoRE low-rank router.  TEST INFRASTRUCTURE ONLY: tests,
 * the smoke check and the benchmark's CPU-baseline leg may call it; the
 * routing library never does.  It shares no code with the CUDA path.
 *
 * Source: "MoRE: Scaling mixture of experts with hardware-aware low-rank
 * routing" (arXiv 2609.36301), cited below as [MoRE].
 *
 * What it computes, for every token n (plain definitions, fp64 throughout):
 *   z     = x_n . R1            R1 is h x r             [MoRE §2 "MoRE layer"]
 *   l     = z . R2              R2 is r x M             [MoRE App. F, eq. (5)]
 *   top-k = the k largest logits under the order "larger logit first, lower
 *           expert index first on equal logits"         [MoRE §2; App. F Alg. 1,
 *           the strict comparison of the merge and the first-index argmax]
 *   gates = softmax over the k selected logits          [MoRE §2, App. F Fig. 12]
 *   counts[e] = number of (token, slot) pairs naming e  [MoRE App. F eq. (9), f]
 *   training statistics m_n, Z_n and psum of App. F, Algorithm 2, eqs. (6)-(7)
 *           (oracle_train_stats)
 *   the standard (full-rank) router of the same form, l = x_n . W with W h x M,
 *           which App. H.3 fuses with the same kernel design (oracle_route_fullrank)
 * plus what the parity checks need: the margin l_(k) - l_(k+1) of Def. 1
 * [MoRE §3, Definition 1] (+inf when k = M), the gaps between consecutive
 * selected logits, and the root-mean-square of the token's M logits.
 *
 * The names follow the benchmark's convention: R1 (h x r) is the paper's
 * R_2 transposed and R2 (r x M) is the paper's R_1 transposed, so the paper's
 * l = X R_2^T R_1^T is l = (X R1) R2 here.
 *
 * Readings where the pages leave a step open:
 *   - z is kept in fp64.  The paper's kernel narrows z to bf16 before the
 *     second product (App. F, Alg. 1); the oracle is the exact definition
 *     of §2 and does not.
 *   - the selected experts are returned sorted by the order above.
 *   - the softmax subtracts the largest selected logit before exponentiating
 *     (same value as the plain softmax, computed stably).
 *
 * Every input tensor is bf16 (raw 16-bit patterns), widened exactly to double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double oracle_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* z = x . R1 and l = z . R2 for one token (x has h entries). */
void oracle_token_logits(const uint16_t* x, const uint16_t* R1, const uint16_t* R2, int h, int r,
                         int M, double* z, double* logits) {
  for (int i = 0; i < r; ++i) {
    double s = 0.0;
    for (int t = 0; t < h; ++t) s += oracle_bf16(x[t]) * oracle_bf16(R1[(size_t)t * r + i]);
    z[i] = s;
  }
  for (int e = 0; e < M; ++e) {
    double s = 0.0;
    for (int i = 0; i < r; ++i) s += z[i] * oracle_bf16(R2[(size_t)i * M + e]);
    logits[e] = s;
  }
}

/* l = x . W for one token, W h x M (the standard router of App. H.3).  Each l[e] is summed
   over t in increasing order; the loop runs along W's rows so that W is read in order. */
void oracle_token_logits_full(const uint16_t* x, const uint16_t* W, int h, int M, double* logits) {
  for (int e = 0; e < M; ++e) logits[e] = 0.0;
  for (int t = 0; t < h; ++t) {
    const double xt = oracle_bf16(x[t]);
    const uint16_t* w = W + (size_t)t * M;
    for (int e = 0; e < M; ++e) logits[e] += xt * oracle_bf16(w[e]);
  }
}

/* The routing order: a goes before b iff l_a > l_b, or l_a == l_b and a < b. */
typedef struct {
  const double* l;
  int e;
} oracle_item;

static int oracle_cmp(const void* pa, const void* pb) {
  const oracle_item* a = (const oracle_item*)pa;
  const oracle_item* b = (const oracle_item*)pb;
  double la = a->l[a->e], lb = b->l[b->e];
  if (la > lb) return -1;
  if (la < lb) return 1;
  return (a->e < b->e) ? -1 : (a->e > b->e);
}

/*
 * Route one token whose M logits are given: sorted selection, gates, margin,
 * gaps and rms.  scratch (M items) receives all M experts in routing order.
 */
void oracle_select(const double* logits, int M, int k, int32_t* idx, double* gate,
                   double* sel_logit, double* margin, double* gaps, double* rms,
                   oracle_item* scratch) {
  for (int e = 0; e < M; ++e) scratch[e] = (oracle_item){logits, e};
  qsort(scratch, (size_t)M, sizeof(oracle_item), oracle_cmp);
  for (int j = 0; j < k; ++j) {
    idx[j] = scratch[j].e;
    sel_logit[j] = logits[scratch[j].e];
  }
  double top = sel_logit[0], denom = 0.0;
  for (int j = 0; j < k; ++j) denom += exp(sel_logit[j] - top);
  for (int j = 0; j < k; ++j) gate[j] = exp(sel_logit[j] - top) / denom;
  *margin = (k < M) ? sel_logit[k - 1] - logits[scratch[k].e] : INFINITY;
  for (int j = 0; j < k; ++j)
    gaps[j] = (j + 1 < M) ? logits[scratch[j].e] - logits[scratch[j + 1].e] : INFINITY;
  double ss = 0.0;
  for (int e = 0; e < M; ++e) ss += logits[e] * logits[e];
  *rms = sqrt(ss / (double)M);
}

typedef struct {
  const uint16_t *X, *R1, *R2; /* full rank: R1 is NULL and R2 is W (h x M) */
  int h, r, M, k;
  const int64_t* rows;
  int64_t begin, end;
  int32_t* idx;
  double *gate, *logit, *margin, *gaps, *rms;
  int64_t* counts; /* private per job, length M */
} oracle_job;

static void* oracle_worker(void* arg) {
  oracle_job* jb = (oracle_job*)arg;
  double* z = (double*)malloc(sizeof(double) * (size_t)(jb->r > 0 ? jb->r : 1));
  double* l = (double*)malloc(sizeof(double) * (size_t)jb->M);
  oracle_item* scratch = (oracle_item*)malloc(sizeof(oracle_item) * (size_t)jb->M);
  for (int64_t q = jb->begin; q < jb->end; ++q) {
    int64_t n = jb->rows ? jb->rows[q] : q;
    if (jb->R1)
      oracle_token_logits(jb->X + (size_t)n * jb->h, jb->R1, jb->R2, jb->h, jb->r, jb->M, z, l);
    else
      oracle_token_logits_full(jb->X + (size_t)n * jb->h, jb->R2, jb->h, jb->M, l);
    size_t o = (size_t)q * jb->k;
    oracle_select(l, jb->M, jb->k, jb->idx + o, jb->gate + o, jb->logit + o, jb->margin + q,
                  jb->gaps + o, jb->rms + q, scratch);
    for (int j = 0; j < jb->k; ++j) jb->counts[jb->idx[o + j]] += 1;
  }
  free(z);
  free(l);
  free(scratch);
  return NULL;
}

/*
 * Route the tokens rows[0 .. n_rows) of X (N x h), or tokens 0 .. n_rows-1
 * when rows is NULL.  Outputs are indexed by position in rows: idx, gate,
 * logit and gaps are n_rows x k; margin and rms are n_rows; counts (length M)
 * counts the selections of these tokens.  Returns 0, or 1 on bad arguments.
 */
static int oracle_route_rows(const uint16_t* X, const uint16_t* R1, const uint16_t* R2, int64_t N,
                             int h, int r, int M, int k, const int64_t* rows, int64_t n_rows,
                             int32_t* idx, double* gate, double* logit, double* margin, double* gaps,
                             double* rms, int64_t* counts, int nthreads) {
  if (N < 0 || h < 1 || M < 1 || k < 1 || k > M || n_rows < 0) return 1;
  if (!rows && n_rows > N) return 1;
  if (rows)
    for (int64_t q = 0; q < n_rows; ++q)
      if (rows[q] < 0 || rows[q] >= N) return 1;
  memset(counts, 0, sizeof(int64_t) * (size_t)M);
  if (n_rows == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > n_rows) nthreads = (int)n_rows;
  pthread_t th[256];
  int inline_run[256];
  oracle_job jobs[256];
  int64_t* priv = (int64_t*)calloc((size_t)nthreads * (size_t)M, sizeof(int64_t));
  int64_t per = (n_rows + nthreads - 1) / nthreads;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    int64_t b = (int64_t)t * per, e = b + per;
    if (e > n_rows) e = n_rows;
    if (b >= e) break;
    jobs[t] = (oracle_job){X, R1, R2, h, r, M, k, rows, b, e, idx, gate, logit, margin, gaps, rms,
                           priv + (size_t)t * M};
    inline_run[t] = 0;
    if (pthread_create(&th[t], NULL, oracle_worker, &jobs[t]) != 0) {
      oracle_worker(&jobs[t]);
      inline_run[t] = 1;
    }
    used = t + 1;
  }
  for (int t = 0; t < used; ++t) {
    if (!inline_run[t]) pthread_join(th[t], NULL);
    for (int e = 0; e < M; ++e) counts[e] += priv[(size_t)t * M + e];
  }
  free(priv);
  return 0;
}

int oracle_route(const uint16_t* X, const uint16_t* R1, const uint16_t* R2, int64_t N, int h,
                 int r, int M, int k, const int64_t* rows, int64_t n_rows, int32_t* idx,
                 double* gate, double* logit, double* margin, double* gaps, double* rms,
                 int64_t* counts, int nthreads) {
  if (!R1 || r < 1) return 1;
  return oracle_route_rows(X, R1, R2, N, h, r, M, k, rows, n_rows, idx, gate, logit, margin, gaps,
                           rms, counts, nthreads);
}

/*
 * The standard router of App. H.3 ("Fusing a standard MoE layer"): the same selection,
 * gates, counts and parity statistics as oracle_route, with the logits l = x . W of a
 * full-rank W (h x M) instead of (x . R1) . R2.
 */
int oracle_route_fullrank(const uint16_t* X, const uint16_t* W, int64_t N, int h, int M, int k,
                          const int64_t* rows, int64_t n_rows, int32_t* idx, double* gate,
                          double* logit, double* margin, double* gaps, double* rms, int64_t* counts,
                          int nthreads) {
  return oracle_route_rows(X, NULL, W, N, h, 0, M, k, rows, n_rows, idx, gate, logit, margin, gaps,
                           rms, counts, nthreads);
}

/* Full-rank logit of single (token, expert) pairs, fp64: l = sum_t x_t W[t,e]. */
int oracle_logits_at_fullrank(const uint16_t* X, const uint16_t* W, int64_t N, int h, int M,
                              int64_t n_pairs, const int64_t* rows, const int32_t* experts,
                              double* out) {
  for (int64_t p = 0; p < n_pairs; ++p) {
    int64_t n = rows[p];
    int e = experts[p];
    if (n < 0 || n >= N || e < 0 || e >= M) return 1;
    const uint16_t* x = X + (size_t)n * h;
    double s = 0.0;
    for (int t = 0; t < h; ++t) s += oracle_bf16(x[t]) * oracle_bf16(W[(size_t)t * M + e]);
    out[p] = s;
  }
  return 0;
}

/*
 * Training statistics of App. F, Algorithm 2 and eqs. (6)-(7), for the tokens rows[0 ..
 * n_rows) (or 0 .. n_rows-1): per token the largest logit m_n = max_j l_nj and the
 * softmax normalizer relative to it, Z_n = sum_j exp(l_nj - m_n) (Algorithm 2 keeps Z
 * relative to the running maximum); per expert the column sum of the full softmax over
 * all M experts, psum_i = sum_n exp(l_ni - m_n) / Z_n.  Plain fp64 loops; psum is summed
 * per thread in token order and the thread partials are added in thread order.
 * Returns 0, or 1 on bad arguments.
 */
typedef struct {
  const uint16_t *X, *R1, *R2;
  int h, r, M;
  const int64_t* rows;
  int64_t begin, end;
  double *m, *Z;
  double* psum; /* private per job, length M */
} oracle_stats_job;

static void* oracle_stats_worker(void* arg) {
  oracle_stats_job* jb = (oracle_stats_job*)arg;
  double* z = (double*)malloc(sizeof(double) * (size_t)jb->r);
  double* l = (double*)malloc(sizeof(double) * (size_t)jb->M);
  for (int64_t q = jb->begin; q < jb->end; ++q) {
    int64_t n = jb->rows ? jb->rows[q] : q;
    oracle_token_logits(jb->X + (size_t)n * jb->h, jb->R1, jb->R2, jb->h, jb->r, jb->M, z, l);
    double mx = l[0];
    for (int e = 1; e < jb->M; ++e)
      if (l[e] > mx) mx = l[e];
    double sum = 0.0;
    for (int e = 0; e < jb->M; ++e) sum += exp(l[e] - mx);
    jb->m[q] = mx;
    jb->Z[q] = sum;
    for (int e = 0; e < jb->M; ++e) jb->psum[e] += exp(l[e] - mx) / sum;
  }
  free(z);
  free(l);
  return NULL;
}

int oracle_train_stats(const uint16_t* X, const uint16_t* R1, const uint16_t* R2, int64_t N, int h,
                       int r, int M, const int64_t* rows, int64_t n_rows, double* m, double* Z,
                       double* psum, int nthreads) {
  if (N < 0 || h < 1 || r < 1 || M < 1 || n_rows < 0) return 1;
  if (!rows && n_rows > N) return 1;
  if (rows)
    for (int64_t q = 0; q < n_rows; ++q)
      if (rows[q] < 0 || rows[q] >= N) return 1;
  memset(psum, 0, sizeof(double) * (size_t)M);
  if (n_rows == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > n_rows) nthreads = (int)n_rows;
  pthread_t th[256];
  int inline_run[256];
  oracle_stats_job jobs[256];
  double* priv = (double*)calloc((size_t)nthreads * (size_t)M, sizeof(double));
  int64_t per = (n_rows + nthreads - 1) / nthreads;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    int64_t b = (int64_t)t * per, e = b + per;
    if (e > n_rows) e = n_rows;
    if (b >= e) break;
    jobs[t] = (oracle_stats_job){X, R1, R2, h, r, M, rows, b, e, m, Z, priv + (size_t)t * M};
    inline_run[t] = 0;
    if (pthread_create(&th[t], NULL, oracle_stats_worker, &jobs[t]) != 0) {
      oracle_stats_worker(&jobs[t]);
      inline_run[t] = 1;
    }
    used = t + 1;
  }
  for (int t = 0; t < used; ++t) {
    if (!inline_run[t]) pthread_join(th[t], NULL);
    for (int e = 0; e < M; ++e) psum[e] += priv[(size_t)t * M + e];
  }
  free(priv);
  return 0;
}

/* All M logits of the given tokens (n_rows x M), fp64. */
int oracle_logits(const uint16_t* X, const uint16_t* R1, const uint16_t* R2, int64_t N, int h,
                  int r, int M, const int64_t* rows, int64_t n_rows, double* out) {
  if (N < 0 || h < 1 || r < 1 || M < 1 || n_rows < 0) return 1;
  double* z = (double*)malloc(sizeof(double) * (size_t)r);
  for (int64_t q = 0; q < n_rows; ++q) {
    int64_t n = rows ? rows[q] : q;
    if (n < 0 || n >= N) {
      free(z);
      return 1;
    }
    oracle_token_logits(X + (size_t)n * h, R1, R2, h, r, M, z, out + (size_t)q * M);
  }
  free(z);
  return 0;
}

/* z = x . R1 of the given tokens (n_rows x r), fp64. */
int oracle_projection(const uint16_t* X, const uint16_t* R1, int64_t N, int h, int r,
                      const int64_t* rows, int64_t n_rows, double* out) {
  if (N < 0 || h < 1 || r < 1 || n_rows < 0) return 1;
  for (int64_t q = 0; q < n_rows; ++q) {
    int64_t n = rows ? rows[q] : q;
    if (n < 0 || n >= N) return 1;
    const uint16_t* x = X + (size_t)n * h;
    for (int i = 0; i < r; ++i) {
      double s = 0.0;
      for (int t = 0; t < h; ++t) s += oracle_bf16(x[t]) * oracle_bf16(R1[(size_t)t * r + i]);
      out[(size_t)q * r + i] = s;
    }
  }
  return 0;
}

/* Logit of single (token, expert) pairs, fp64: l = sum_i (sum_t x_t R1[t,i]) R2[i,e]. */
int oracle_logits_at(const uint16_t* X, const uint16_t* R1, const uint16_t* R2, int64_t N, int h,
                     int r, int M, int64_t n_pairs, const int64_t* rows, const int32_t* experts,
                     double* out) {
  double* z = (double*)malloc(sizeof(double) * (size_t)r);
  int64_t last = -1;
  for (int64_t p = 0; p < n_pairs; ++p) {
    int64_t n = rows[p];
    int e = experts[p];
    if (n < 0 || n >= N || e < 0 || e >= M) {
      free(z);
      return 1;
    }
    if (n != last) {
      const uint16_t* x = X + (size_t)n * h;
      for (int i = 0; i < r; ++i) {
        double s = 0.0;
        for (int t = 0; t < h; ++t) s += oracle_bf16(x[t]) * oracle_bf16(R1[(size_t)t * r + i]);
        z[i] = s;
      }
      last = n;
    }
    double s = 0.0;
    for (int i = 0; i < r; ++i) s += z[i] * oracle_bf16(R2[(size_t)i * M + e]);
    out[p] = s;
  }
  free(z);
  return 0;
}
