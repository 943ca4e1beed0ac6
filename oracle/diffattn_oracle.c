/*
 * diffattn_oracle.c -- float64 CPU oracle for the differential attention operator.
 *
 * TEST INFRASTRUCTURE. This file is the slow, plain reference that the CUDA path is
 * checked against. Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline / reference leg may build, load or call it. The product library never
 * links it, and it shares no code, header or constant with the CUDA sources.
 *
 * What it computes (one "differential unit" = one batch entry and one V1 head or one
 * V2 query-head pair), written straight from the definitions on the pages:
 *
 *   s_b[j] = q_b . k_b[j] / sqrt(d)                       b = 1, 2
 *   A_b    = softmax(s_b), max-subtracted                  "Differential Attention (V2)",
 *                                                          Build It, Step 1 (stable softmax)
 *   w[j]   = A_1[j] - lambda * A_2[j]                      same lesson, The Concept /
 *                                                          "The difference idea";
 *                                                          Build It, Step 3
 *   o[c]   = sum_j w[j] * v[j][c]                          same (DiffAttn = (A1 - lambda A2) V)
 *   V1 only: o <- o / sqrt(mean(o^2) + eps) * (1 - lambda_init)
 *                                                          same lesson, "V1 vs V2" and Key
 *                                                          Terms ("Per-head RMSNorm");
 *                                                          Hugging Face post on the DIFF
 *                                                          Transformer, "How?" (per-head
 *                                                          GroupNorm). eps, unit gain and the
 *                                                          (1 - lambda_init) factor are the
 *                                                          operator's stated configuration.
 *
 *   causal: key j is visible to query i iff j <= i ("Attention Variants: Sliding
 *   Window, Sparse, Differential", Build It, Step 1 causal_mask; Step 4 diff_attention).
 *   With Nk keys and Nq <= Nk queries (a chunk of new queries after Nk - Nq cached ones)
 *   query i sits at position i + Nk - Nq. A sliding window of W keys (same page, Build
 *   It, sliding-window mask) keeps keys j with pos - W < j <= pos.
 *
 *   lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init   ("Differential Attention (V2)",
 *            The Concept, "The difference idea"; Key Terms "lambda")
 *   lambda_init(depth) = 0.8 - 0.6 * exp(-0.3 * (depth - 1))  (skill-diff-attention-integrator,
 *            "Architecture diff")
 *
 * Both attention maps are materialised one query row at a time (every A_b[j] is formed
 * explicitly); there is no online softmax, tiling or fusion here. All arithmetic is
 * IEEE float64. Inputs arrive as float64 arrays holding exactly the values the GPU
 * consumed (bf16 and fp32 convert to float64 without rounding).
 *
 * Threads only split independent units (batch, head) across workers; every unit is
 * computed by the same sequential code, so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_NOMEM -2

/* lambda_init depth schedule (skill-diff-attention-integrator, "Architecture diff"). */
double oracle_lambda_init(int depth) { return 0.8 - 0.6 * exp(-0.3 * (double)(depth - 1)); }

/*
 * lambda re-parameterisation, one scalar per head (V1) or per pair (V2):
 *   lambda_h = exp(lq1_h . lk1_h) - exp(lq2_h . lk2_h) + lambda_init(depth)
 * The four vectors are [n_heads, dim] row-major.
 */
int oracle_lambda(const double* lq1, const double* lk1, const double* lq2, const double* lk2,
                  int n_heads, int dim, int depth, double* lambda_out) {
  if (n_heads < 0 || dim < 0 || !lambda_out) return ORACLE_ERR_ARG;
  double li = oracle_lambda_init(depth);
  for (int h = 0; h < n_heads; ++h) {
    double d1 = 0.0, d2 = 0.0;
    for (int c = 0; c < dim; ++c) {
      d1 += lq1[(long)h * dim + c] * lk1[(long)h * dim + c];
      d2 += lq2[(long)h * dim + c] * lk2[(long)h * dim + c];
    }
    lambda_out[h] = exp(d1) - exp(d2) + li;
  }
  return ORACLE_OK;
}

/* Row softmax with the maximum subtracted first ("Differential Attention (V2)",
 * Build It, Step 1). x has n >= 1 entries; overwritten with the probabilities. */
static void softmax_row(double* x, int n) {
  double m = x[0];
  for (int j = 1; j < n; ++j)
    if (x[j] > m) m = x[j];
  double s = 0.0;
  for (int j = 0; j < n; ++j) {
    x[j] = exp(x[j] - m);
    s += x[j];
  }
  for (int j = 0; j < n; ++j) x[j] /= s;
}

static double dot(const double* a, const double* b, int n) {
  double s = 0.0;
  for (int c = 0; c < n; ++c) s += a[c] * b[c];
  return s;
}

/*
 * One query row of differential attention over n_keys visible keys.
 *   q1, q2      : the two branch queries, d entries each
 *   k1, k2      : key rows j at k1 + j*ks, k2 + j*ks (d entries each)
 *   v           : value rows j at v + j*vs (dv entries each)
 *   a1, a2      : scratch of n_keys entries; receive the two attention-map rows
 *   o           : dv outputs (before any norm)
 * n_keys == 0 (no visible key) gives o = 0.
 */
static void diff_row(const double* q1, const double* q2, const double* k1, const double* k2,
                     long ks, const double* v, long vs, int n_keys, int d, int dv, double lam,
                     double* a1, double* a2, double* o) {
  for (int c = 0; c < dv; ++c) o[c] = 0.0;
  if (n_keys <= 0) return;
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int j = 0; j < n_keys; ++j) {
    a1[j] = dot(q1, k1 + (long)j * ks, d) * inv_sqrt_d;
    a2[j] = dot(q2, k2 + (long)j * ks, d) * inv_sqrt_d;
  }
  softmax_row(a1, n_keys);
  softmax_row(a2, n_keys);
  for (int j = 0; j < n_keys; ++j) {
    double w = a1[j] - lam * a2[j];
    const double* vj = v + (long)j * vs;
    for (int c = 0; c < dv; ++c) o[c] += w * vj[c];
  }
}

/* Per-head RMSNorm with unit gain, then the (1 - lambda_init) scale (V1 only). */
static void rmsnorm_scale(double* o, int n, double eps, double lambda_init) {
  double ss = 0.0;
  for (int c = 0; c < n; ++c) ss += o[c] * o[c];
  double r = sqrt(ss / (double)n + eps);
  for (int c = 0; c < n; ++c) o[c] = o[c] / r * (1.0 - lambda_init);
}

/* ------------------------------------------------------------------------------------ */
/* Work distribution: units are independent; thread t takes units t, t+T, t+2T, ...      */

typedef struct job job;
typedef void (*unit_fn)(const job*, long unit, double* a1, double* a2);

struct job {
  int variant; /* 1 = V1 prefill, 2 = V2 prefill, 3 = V2 decode, 4 = V1 decode */
  const double *q, *k, *v, *lam;
  const int* kv_len;
  const int* rows;
  int n_rows;
  int q_compact; /* 1: q holds only the sampled rows, [B, n_rows, ...] */
  int B, N, H, Hq, Hkv, d, causal, apply_norm;
  int Nk;     /* keys per batch entry (>= N, the queries); prefill only */
  int window; /* causal sliding window in keys; 0 = none */
  double eps, lambda_init;
  double* out;
  long n_units;
  int scratch_len;
  unit_fn fn;
};

typedef struct {
  const job* j;
  int tid, nthreads;
  int status;
} worker;

static void* worker_main(void* arg) {
  worker* w = (worker*)arg;
  const job* jb = w->j;
  double* a1 = (double*)malloc(sizeof(double) * (size_t)(jb->scratch_len > 0 ? jb->scratch_len : 1));
  double* a2 = (double*)malloc(sizeof(double) * (size_t)(jb->scratch_len > 0 ? jb->scratch_len : 1));
  if (!a1 || !a2) {
    free(a1);
    free(a2);
    w->status = ORACLE_ERR_NOMEM;
    return NULL;
  }
  for (long u = w->tid; u < jb->n_units; u += w->nthreads) jb->fn(jb, u, a1, a2);
  free(a1);
  free(a2);
  w->status = ORACLE_OK;
  return NULL;
}

static int run_job(const job* jb, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((long)nthreads > jb->n_units) nthreads = jb->n_units > 0 ? (int)jb->n_units : 1;
  pthread_t tids[256];
  worker ws[256];
  for (int t = 0; t < nthreads; ++t) {
    ws[t].j = jb;
    ws[t].tid = t;
    ws[t].nthreads = nthreads;
    ws[t].status = ORACLE_ERR_ARG;
  }
  if (nthreads == 1) {
    worker_main(&ws[0]);
    return ws[0].status;
  }
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    if (pthread_create(&tids[t], NULL, worker_main, &ws[t]) != 0) break;
    ++started;
  }
  for (int t = 0; t < started; ++t) pthread_join(tids[t], NULL);
  if (started < nthreads) {
    /* run the remaining workers on this thread */
    for (int t = started; t < nthreads; ++t) worker_main(&ws[t]);
  }
  for (int t = 0; t < nthreads; ++t)
    if (ws[t].status != ORACLE_OK) return ws[t].status;
  return ORACLE_OK;
}

/* ---- V1 prefill ---------------------------------------------------------------------
 * q, k : [B, N, H, 2, d]   (index 0 of the branch axis is branch 1)
 * v    : [B, N, H, 2d]
 * lam  : [H]
 * out  : [B, n_rows, H, 2d]; output row r is query position rows[r] (all N when rows==NULL)
 * q_compact = 1 (with rows): q holds only the sampled query rows, [B, n_rows, H, 2, d].
 * One unit = (b, h).
 */
static void v1_unit(const job* jb, long unit, double* a1, double* a2) {
  int b = (int)(unit / jb->H), h = (int)(unit % jb->H);
  int N = jb->N, H = jb->H, d = jb->d, dv = 2 * d;
  long tok_q = (long)H * 2 * d; /* element stride between tokens in q and k */
  long tok_v = (long)H * dv;
  int n_rows = jb->rows ? jb->n_rows : N;
  int nq = jb->q_compact ? n_rows : N; /* query rows stored per batch entry */
  const double* qb = jb->q + (long)b * nq * tok_q + (long)h * 2 * d;
  const double* kb = jb->k + (long)b * jb->Nk * tok_q + (long)h * 2 * d;
  const double* vb = jb->v + (long)b * jb->Nk * tok_v + (long)h * dv;
  for (int r = 0; r < n_rows; ++r) {
    int i = jb->rows ? jb->rows[r] : r;
    const double* q1 = qb + (long)(jb->q_compact ? r : i) * tok_q;
    const double* q2 = q1 + d;
    int hi = jb->causal ? i + (jb->Nk - N) : jb->Nk - 1; /* last visible key */
    int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;
    double* o = jb->out + (((long)b * n_rows + r) * H + h) * dv;
    diff_row(q1, q2, kb + (long)lo * tok_q, kb + (long)lo * tok_q + d, tok_q, vb + (long)lo * tok_v,
             tok_v, hi - lo + 1, d, dv, jb->lam[h], a1, a2, o);
    if (jb->apply_norm) rmsnorm_scale(o, dv, jb->eps, jb->lambda_init);
  }
}

/* Nq queries (the last Nq of Nk positions when causal), Nk keys, causal sliding window of
 * `window` keys (0 = none; only with causal). */
int oracle_prefill_v1_range(const double* q, const double* k, const double* v, const double* lam,
                            double lambda_init, int B, int Nq, int Nk, int H, int d, int causal,
                            int window, int apply_norm, double eps, const int* rows, int n_rows,
                            int q_compact, double* out, int nthreads) {
  if (!q || !k || !v || !lam || !out || B < 0 || Nq < 0 || Nk < Nq || H < 0 || d <= 0 || window < 0)
    return ORACLE_ERR_ARG;
  if (window > 0 && !causal) return ORACLE_ERR_ARG;
  if (rows) {
    for (int r = 0; r < n_rows; ++r)
      if (rows[r] < 0 || rows[r] >= Nq) return ORACLE_ERR_ARG;
  }
  job jb;
  memset(&jb, 0, sizeof(jb));
  jb.variant = 1;
  jb.q = q; jb.k = k; jb.v = v; jb.lam = lam;
  jb.rows = rows; jb.n_rows = n_rows; jb.q_compact = rows ? q_compact : 0;
  jb.B = B; jb.N = Nq; jb.Nk = Nk; jb.window = window; jb.H = H; jb.d = d; jb.causal = causal;
  jb.apply_norm = apply_norm;
  jb.eps = eps; jb.lambda_init = lambda_init; jb.out = out;
  jb.n_units = (long)B * H;
  jb.scratch_len = Nk;
  jb.fn = v1_unit;
  return run_job(&jb, nthreads);
}

int oracle_prefill_v1(const double* q, const double* k, const double* v, const double* lam,
                      double lambda_init, int B, int N, int H, int d, int causal, int apply_norm,
                      double eps, const int* rows, int n_rows, int q_compact, double* out,
                      int nthreads) {
  return oracle_prefill_v1_range(q, k, v, lam, lambda_init, B, N, N, H, d, causal, 0, apply_norm,
                                 eps, rows, n_rows, q_compact, out, nthreads);
}

/* ---- V2 prefill ---------------------------------------------------------------------
 * q    : [B, N, Hq, d]; query heads 2p and 2p+1 are branches 1 and 2 of pair p
 * k, v : [B, N, Hkv, d]; query head hq reads KV head hq / (Hq / Hkv)
 * lam  : [Hq/2]
 * out  : [B, n_rows, Hq/2, d]
 * q_compact = 1 (with rows): q holds only the sampled query rows, [B, n_rows, Hq, d].
 * One unit = (b, p).
 */
static void v2_unit(const job* jb, long unit, double* a1, double* a2) {
  int P = jb->Hq / 2;
  int b = (int)(unit / P), p = (int)(unit % P);
  int N = jb->N, d = jb->d;
  int group = jb->Hq / jb->Hkv;
  int h1 = 2 * p, h2 = 2 * p + 1;
  int g1 = h1 / group, g2 = h2 / group;
  long tok_q = (long)jb->Hq * d, tok_kv = (long)jb->Hkv * d;
  int n_rows = jb->rows ? jb->n_rows : N;
  int nq = jb->q_compact ? n_rows : N;
  const double* qb = jb->q + (long)b * nq * tok_q;
  const double* kb = jb->k + (long)b * jb->Nk * tok_kv;
  const double* vb = jb->v + (long)b * jb->Nk * tok_kv;
  for (int r = 0; r < n_rows; ++r) {
    int i = jb->rows ? jb->rows[r] : r;
    long qr = jb->q_compact ? r : i;
    const double* q1 = qb + qr * tok_q + (long)h1 * d;
    const double* q2 = qb + qr * tok_q + (long)h2 * d;
    int hi = jb->causal ? i + (jb->Nk - N) : jb->Nk - 1; /* last visible key */
    int lo = (jb->causal && jb->window > 0 && hi - jb->window + 1 > 0) ? hi - jb->window + 1 : 0;
    double* o = jb->out + (((long)b * n_rows + r) * P + p) * d;
    const double* k0 = kb + (long)lo * tok_kv;
    const double* v0 = vb + (long)lo * tok_kv;
    /* both branches of a pair read the same KV head when Hq/Hkv is even */
    diff_row(q1, q2, k0 + (long)g1 * d, k0 + (long)g2 * d, tok_kv, v0 + (long)g1 * d, tok_kv,
             hi - lo + 1, d, d, jb->lam[p], a1, a2, o);
  }
}

int oracle_prefill_v2_range(const double* q, const double* k, const double* v, const double* lam,
                            int B, int Nq, int Nk, int Hq, int Hkv, int d, int causal, int window,
                            const int* rows, int n_rows, int q_compact, double* out, int nthreads) {
  if (!q || !k || !v || !lam || !out || B < 0 || Nq < 0 || Nk < Nq || Hq <= 0 || Hkv <= 0 ||
      d <= 0 || window < 0)
    return ORACLE_ERR_ARG;
  if (window > 0 && !causal) return ORACLE_ERR_ARG;
  if (Hq % 2 != 0 || Hq % Hkv != 0 || (Hq / Hkv) % 2 != 0) return ORACLE_ERR_ARG;
  if (rows) {
    for (int r = 0; r < n_rows; ++r)
      if (rows[r] < 0 || rows[r] >= Nq) return ORACLE_ERR_ARG;
  }
  job jb;
  memset(&jb, 0, sizeof(jb));
  jb.variant = 2;
  jb.q = q; jb.k = k; jb.v = v; jb.lam = lam;
  jb.rows = rows; jb.n_rows = n_rows; jb.q_compact = rows ? q_compact : 0;
  jb.B = B; jb.N = Nq; jb.Nk = Nk; jb.window = window; jb.Hq = Hq; jb.Hkv = Hkv; jb.d = d;
  jb.causal = causal;
  jb.out = out;
  jb.n_units = (long)B * (Hq / 2);
  jb.scratch_len = Nk;
  jb.fn = v2_unit;
  return run_job(&jb, nthreads);
}

int oracle_prefill_v2(const double* q, const double* k, const double* v, const double* lam,
                      int B, int N, int Hq, int Hkv, int d, int causal, const int* rows,
                      int n_rows, int q_compact, double* out, int nthreads) {
  return oracle_prefill_v2_range(q, k, v, lam, B, N, N, Hq, Hkv, d, causal, 0, rows, n_rows,
                                 q_compact, out, nthreads);
}

/* ---- V2 decode ----------------------------------------------------------------------
 * One new query per batch entry attends every cached key 0 .. kv_len[b]-1.
 * q    : [B, Hq, d]
 * k, v : [B, L, Hkv, d] (L = cache capacity)
 * kv_len : [B] or NULL (= L)
 * lam  : [Hq/2]
 * out  : [B, Hq/2, d]
 * One unit = (b, p).
 */
static void dec_unit(const job* jb, long unit, double* a1, double* a2) {
  int P = jb->Hq / 2;
  int b = (int)(unit / P), p = (int)(unit % P);
  int L = jb->N, d = jb->d;
  int group = jb->Hq / jb->Hkv;
  int h1 = 2 * p, h2 = 2 * p + 1;
  int g1 = h1 / group, g2 = h2 / group;
  long tok_kv = (long)jb->Hkv * d;
  const double* kb = jb->k + (long)b * L * tok_kv;
  const double* vb = jb->v + (long)b * L * tok_kv;
  const double* q1 = jb->q + ((long)b * jb->Hq + h1) * d;
  const double* q2 = jb->q + ((long)b * jb->Hq + h2) * d;
  int n_keys = jb->kv_len ? jb->kv_len[b] : L;
  double* o = jb->out + ((long)b * P + p) * d;
  diff_row(q1, q2, kb + (long)g1 * d, kb + (long)g2 * d, tok_kv, vb + (long)g1 * d, tok_kv,
           n_keys, d, d, jb->lam[p], a1, a2, o);
}

int oracle_decode_v2(const double* q, const double* k, const double* v, const int* kv_len,
                     const double* lam, int B, int L, int Hq, int Hkv, int d, double* out,
                     int nthreads) {
  if (!q || !k || !v || !lam || !out || B < 0 || L < 0 || Hq <= 0 || Hkv <= 0 || d <= 0)
    return ORACLE_ERR_ARG;
  if (Hq % 2 != 0 || Hq % Hkv != 0 || (Hq / Hkv) % 2 != 0) return ORACLE_ERR_ARG;
  if (kv_len) {
    for (int b = 0; b < B; ++b)
      if (kv_len[b] < 0 || kv_len[b] > L) return ORACLE_ERR_ARG;
  }
  job jb;
  memset(&jb, 0, sizeof(jb));
  jb.variant = 3;
  jb.q = q; jb.k = k; jb.v = v; jb.lam = lam; jb.kv_len = kv_len;
  jb.B = B; jb.N = L; jb.Hq = Hq; jb.Hkv = Hkv; jb.d = d;
  jb.out = out;
  jb.n_units = (long)B * (Hq / 2);
  jb.scratch_len = L;
  jb.fn = dec_unit;
  return run_job(&jb, nthreads);
}

/* ---- V1 decode ----------------------------------------------------------------------
 * One new query per batch entry and head attends every cached key 0 .. kv_len[b]-1 of
 * that head; both branches read their own cached keys and the one cached value row.
 * q    : [B, H, 2, d]      (index 0 of the branch axis is branch 1)
 * k    : [B, L, H, 2, d]   (L = cache capacity)
 * v    : [B, L, H, 2d]
 * kv_len : [B] or NULL (= L)
 * lam  : [H]
 * out  : [B, H, 2d], per-head RMSNorm and (1 - lambda_init) scale when apply_norm
 * One unit = (b, h).
 */
static void dec1_unit(const job* jb, long unit, double* a1, double* a2) {
  int H = jb->H;
  int b = (int)(unit / H), h = (int)(unit % H);
  int L = jb->N, d = jb->d, dv = 2 * d;
  long tok_k = (long)H * 2 * d, tok_v = (long)H * dv;
  const double* kb = jb->k + (long)b * L * tok_k + (long)h * 2 * d;
  const double* vb = jb->v + (long)b * L * tok_v + (long)h * dv;
  const double* q1 = jb->q + ((long)b * H + h) * 2 * d;
  const double* q2 = q1 + d;
  int n_keys = jb->kv_len ? jb->kv_len[b] : L;
  double* o = jb->out + ((long)b * H + h) * dv;
  diff_row(q1, q2, kb, kb + d, tok_k, vb, tok_v, n_keys, d, dv, jb->lam[h], a1, a2, o);
  if (jb->apply_norm) rmsnorm_scale(o, dv, jb->eps, jb->lambda_init);
}

int oracle_decode_v1(const double* q, const double* k, const double* v, const int* kv_len,
                     const double* lam, double lambda_init, int B, int L, int H, int d,
                     int apply_norm, double eps, double* out, int nthreads) {
  if (!q || !k || !v || !lam || !out || B < 0 || L < 0 || H <= 0 || d <= 0) return ORACLE_ERR_ARG;
  if (kv_len) {
    for (int b = 0; b < B; ++b)
      if (kv_len[b] < 0 || kv_len[b] > L) return ORACLE_ERR_ARG;
  }
  job jb;
  memset(&jb, 0, sizeof(jb));
  jb.variant = 4;
  jb.q = q; jb.k = k; jb.v = v; jb.lam = lam; jb.kv_len = kv_len;
  jb.B = B; jb.N = L; jb.H = H; jb.d = d; jb.apply_norm = apply_norm;
  jb.eps = eps; jb.lambda_init = lambda_init; jb.out = out;
  jb.n_units = (long)B * H;
  jb.scratch_len = L;
  jb.fn = dec1_unit;
  return run_job(&jb, nthreads);
}

/* ---- attention-map rows (for the noise-floor measurements) ---------------------------
 * Writes the two softmax rows A_1, A_2 of a single V2 pair query row i (causal) so that
 * tests can measure the signal and noise mass the pages talk about.
 * q : [N, Hq, d], k : [N, Hkv, d] for one batch entry; a1, a2 : [i + 1].
 */
int oracle_map_row_v2(const double* q, const double* k, int N, int Hq, int Hkv, int d, int p,
                      int i, double* a1, double* a2) {
  if (!q || !k || !a1 || !a2 || i < 0 || i >= N || p < 0 || 2 * p + 1 >= Hq) return ORACLE_ERR_ARG;
  if (Hq % Hkv != 0) return ORACLE_ERR_ARG;
  int group = Hq / Hkv;
  int h1 = 2 * p, h2 = 2 * p + 1;
  long tok_q = (long)Hq * d, tok_kv = (long)Hkv * d;
  const double* q1 = q + (long)i * tok_q + (long)h1 * d;
  const double* q2 = q + (long)i * tok_q + (long)h2 * d;
  const double* k1 = k + (long)(h1 / group) * d;
  const double* k2 = k + (long)(h2 / group) * d;
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int j = 0; j <= i; ++j) {
    a1[j] = dot(q1, k1 + (long)j * tok_kv, d) * inv_sqrt_d;
    a2[j] = dot(q2, k2 + (long)j * tok_kv, d) * inv_sqrt_d;
  }
  softmax_row(a1, i + 1);
  softmax_row(a2, i + 1);
  return ORACLE_OK;
}
