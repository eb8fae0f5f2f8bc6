/*
 * kmip_oracle.c -- plain, slow, fp64 CPU oracle for k-Maximum-Inner-Product
 * (k-MIP) attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; the two agree only because both follow the same
 * definition.
 *
 * Definition followed (k-Maximum Inner Product Attention for Graph
 * Transformers and the Expressive Power of GraphGPS, Abstract): for every
 * query node the layer keeps the key nodes with the k largest inner products
 * ("a top-k operation" over the "most relevant key nodes per query") and
 * attends over that sparse set only.  Written out, for query i of graph g
 * and head h:
 *
 *   s_j   = sum_c Q[i,h,c] * K[j,h,c]            for every key j of graph g
 *   S     = the min(k, n_g) keys with the largest s_j
 *           (order: larger s first, equal s -> smaller j first)
 *   z_j   = scale * s_j,   lse = log sum_{j in S} exp(z_j)
 *   p_j   = exp(z_j - lse)
 *   out   = sum_{j in S} p_j V[j,h,:]
 *
 * and the backward pass through the selected scores (the pages time a
 * "training setting", Tables 10-12 and 16, without describing it; the
 * selection itself is piecewise constant and carries no gradient):
 *
 *   dP_j  = dO . V_j,   D = sum_j p_j dP_j,   dS_j = p_j (dP_j - D)
 *   dQ_i  = scale * sum_j dS_j K_j
 *   dK_j += scale * dS_j Q_i
 *   dV_j += p_j dO_i
 *
 * Readings where the pages are silent (each is listed with its reason in
 * the design notes): every key of the query's graph is a candidate,
 * including the query node itself; graphs are the contiguous node ranges
 * [offsets[g], offsets[g+1]); heads select independently; a graph with
 * n_g < k yields n_g keys and the index row is padded with -1; ties go to
 * the smaller node index; lse is a natural logarithm.
 *
 * Each query's scores are fully sorted (qsort), exactly as the definition
 * reads; no partial selection, blocking or reordering is used.
 *
 * Layouts: Q, K, V, dO, out, dQ, dK, dV are [N, H, d] row-major fp64;
 * idx is [N, H, k] int32; lse, gap, kth are [N, H] fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  double s;
  int64_t j;
} scored_t;

/* Larger score first; on equal scores the smaller node index first. */
static int cmp_scored(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  if (x->j < y->j) return -1;
  if (x->j > y->j) return 1;
  return 0;
}

typedef struct {
  const double *Q, *K, *V;
  const int64_t* offsets;
  int64_t G, N;
  int H, d, k;
  double scale;
  /* which (query, head) pairs: either all (pairs_q == NULL) or a list */
  const int64_t* pairs_q;
  const int32_t* pairs_h;
  int64_t npairs;
  /* outputs, indexed by pair number (list mode) or by (i, h) (all mode) */
  double* out;
  int32_t* idx;
  double* lse;
  double* gap;
  double* kth;
  /* work distribution */
  int64_t next;
  pthread_mutex_t lock;
} fwd_ctx;

/* Graph that node i belongs to: the g with offsets[g] <= i < offsets[g+1]. */
static int64_t graph_of(const int64_t* offsets, int64_t G, int64_t i) {
  int64_t lo = 0, hi = G; /* answer in [lo, hi) */
  while (hi - lo > 1) {
    int64_t mid = (lo + hi) / 2;
    if (offsets[mid] <= i) lo = mid; else hi = mid;
  }
  /* skip empty graphs that share the same start */
  while (lo + 1 < G && offsets[lo + 1] <= i) ++lo;
  return lo;
}

/* One (query i, head h): scores, full sort, softmax over the kept keys,
 * weighted sum of V rows.  Writes one row of each output at slot `row`. */
static void fwd_one(const fwd_ctx* c, int64_t i, int h, int64_t row, scored_t* buf) {
  const int d = c->d, H = c->H, k = c->k;
  int64_t g = graph_of(c->offsets, c->G, i);
  int64_t j0 = c->offsets[g], j1 = c->offsets[g + 1];
  int64_t n = j1 - j0;
  const double* q = c->Q + (i * H + h) * (int64_t)d;

  for (int64_t j = j0; j < j1; ++j) {
    const double* kr = c->K + (j * H + h) * (int64_t)d;
    double s = 0.0;
    for (int t = 0; t < d; ++t) s += q[t] * kr[t];
    buf[j - j0].s = s;
    buf[j - j0].j = j;
  }
  qsort(buf, (size_t)n, sizeof(scored_t), cmp_scored);

  int64_t keff = n < k ? n : k;
  int32_t* irow = c->idx + row * (int64_t)k;
  for (int t = 0; t < k; ++t) irow[t] = t < keff ? (int32_t)buf[t].j : -1;

  /* log-sum-exp of the scaled kept scores, max-shifted */
  double m = c->scale * buf[0].s;
  double sum = 0.0;
  for (int64_t t = 0; t < keff; ++t) sum += exp(c->scale * buf[t].s - m);
  double lse = m + log(sum);
  c->lse[row] = lse;

  double* o = c->out + row * (int64_t)d;
  for (int t = 0; t < d; ++t) o[t] = 0.0;
  for (int64_t t = 0; t < keff; ++t) {
    double p = exp(c->scale * buf[t].s - lse);
    const double* vr = c->V + (buf[t].j * H + h) * (int64_t)d;
    for (int u = 0; u < d; ++u) o[u] += p * vr[u];
  }

  c->kth[row] = buf[keff - 1].s;
  c->gap[row] = (n > k) ? buf[k - 1].s - buf[k].s : INFINITY;
}

static void* fwd_worker(void* arg) {
  fwd_ctx* c = (fwd_ctx*)arg;
  int64_t maxn = 0;
  for (int64_t g = 0; g < c->G; ++g) {
    int64_t n = c->offsets[g + 1] - c->offsets[g];
    if (n > maxn) maxn = n;
  }
  scored_t* buf = (scored_t*)malloc((size_t)(maxn > 0 ? maxn : 1) * sizeof(scored_t));
  if (!buf) return (void*)1;
  int64_t total = c->pairs_q ? c->npairs : c->N * c->H;
  for (;;) {
    pthread_mutex_lock(&c->lock);
    int64_t t = c->next;
    c->next += 16;
    pthread_mutex_unlock(&c->lock);
    if (t >= total) break;
    int64_t e = t + 16 < total ? t + 16 : total;
    for (; t < e; ++t) {
      if (c->pairs_q) fwd_one(c, c->pairs_q[t], c->pairs_h[t], t, buf);
      else fwd_one(c, t / c->H, (int)(t % c->H), t, buf);
    }
  }
  free(buf);
  return NULL;
}

static int check_offsets(const int64_t* offsets, int64_t G, int64_t N) {
  if (G < 1 || offsets[0] != 0 || offsets[G] != N) return 1;
  for (int64_t g = 0; g < G; ++g)
    if (offsets[g + 1] < offsets[g]) return 1;
  return 0;
}

static int run_fwd(fwd_ctx* c, int nthreads) {
  if (check_offsets(c->offsets, c->G, c->N)) return 1;
  if (c->k < 1 || c->d < 1 || c->H < 1) return 2;
  if (nthreads < 1) nthreads = 1;
  c->next = 0;
  pthread_mutex_init(&c->lock, NULL);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  int rc = 0;
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, fwd_worker, c);
  for (int t = 0; t < nthreads; ++t) {
    void* r = NULL;
    pthread_join(th[t], &r);
    if (r) rc = 3;
  }
  free(th);
  pthread_mutex_destroy(&c->lock);
  return rc;
}

/* Forward for every (query, head).  Returns 0 on success, 1 on malformed
 * offsets, 2 on bad sizes, 3 on allocation failure. */
int kmip_oracle_fwd(const double* Q, const double* K, const double* V,
                    const int64_t* offsets, int64_t G, int64_t N, int H, int d,
                    int k, double scale, double* out, int32_t* idx, double* lse,
                    double* gap, double* kth, int nthreads) {
  fwd_ctx c;
  memset(&c, 0, sizeof c);
  c.Q = Q; c.K = K; c.V = V; c.offsets = offsets; c.G = G; c.N = N;
  c.H = H; c.d = d; c.k = k; c.scale = scale;
  c.out = out; c.idx = idx; c.lse = lse; c.gap = gap; c.kth = kth;
  return run_fwd(&c, nthreads);
}

/* Forward for a list of (query, head) pairs; output row t belongs to pair t
 * (out [npairs, d], idx [npairs, k], lse/gap/kth [npairs]). */
int kmip_oracle_fwd_pairs(const double* Q, const double* K, const double* V,
                          const int64_t* offsets, int64_t G, int64_t N, int H,
                          int d, int k, double scale, const int64_t* pairs_q,
                          const int32_t* pairs_h, int64_t npairs, double* out,
                          int32_t* idx, double* lse, double* gap, double* kth,
                          int nthreads) {
  fwd_ctx c;
  memset(&c, 0, sizeof c);
  c.Q = Q; c.K = K; c.V = V; c.offsets = offsets; c.G = G; c.N = N;
  c.H = H; c.d = d; c.k = k; c.scale = scale;
  c.pairs_q = pairs_q; c.pairs_h = pairs_h; c.npairs = npairs;
  c.out = out; c.idx = idx; c.lse = lse; c.gap = gap; c.kth = kth;
  for (int64_t t = 0; t < npairs; ++t)
    if (pairs_q[t] < 0 || pairs_q[t] >= N || pairs_h[t] < 0 || pairs_h[t] >= H) return 2;
  return run_fwd(&c, nthreads);
}

/*
 * Given the selected sets idx [N, H, k] (-1 = padding), recompute the kept
 * scores in fp64 and apply the softmax and the weighted sum (out, lse), and,
 * when dO is non-NULL, the backward pass (dQ, dK, dV; dK and dV are
 * overwritten).  The selection is taken as given, so this checks the
 * attention over any set, e.g. one chosen on the GPU.  Serial, in the order
 * i = 0..N-1, h = 0..H-1, j in idx order.
 * Returns 0 on success, 2 on an index outside the query's graph.
 */
int kmip_oracle_given_idx(const double* Q, const double* K, const double* V,
                          const double* dO, const int32_t* idx,
                          const int64_t* offsets, int64_t G, int64_t N, int H,
                          int d, int k, double scale, double* out, double* lse,
                          double* dQ, double* dK, double* dV) {
  if (check_offsets(offsets, G, N)) return 1;
  double* s = (double*)malloc(sizeof(double) * (size_t)k);
  double* p = (double*)malloc(sizeof(double) * (size_t)k);
  double* dp = (double*)malloc(sizeof(double) * (size_t)k);
  if (!s || !p || !dp) { free(s); free(p); free(dp); return 3; }
  if (dO) {
    memset(dK, 0, sizeof(double) * (size_t)(N * H * d));
    memset(dV, 0, sizeof(double) * (size_t)(N * H * d));
  }
  int rc = 0;
  for (int64_t i = 0; i < N && !rc; ++i) {
    int64_t g = graph_of(offsets, G, i);
    for (int h = 0; h < H && !rc; ++h) {
      const int32_t* ir = idx + (i * H + h) * (int64_t)k;
      const double* q = Q + (i * H + h) * (int64_t)d;
      int n = 0;
      for (int t = 0; t < k; ++t) {
        if (ir[t] < 0) continue;
        if (ir[t] < offsets[g] || ir[t] >= offsets[g + 1]) { rc = 2; break; }
        const double* kr = K + ((int64_t)ir[t] * H + h) * (int64_t)d;
        double acc = 0.0;
        for (int u = 0; u < d; ++u) acc += q[u] * kr[u];
        s[t] = acc;
        ++n;
      }
      if (rc) break;
      double* o = out + (i * H + h) * (int64_t)d;
      for (int u = 0; u < d; ++u) o[u] = 0.0;
      if (n == 0) { lse[i * H + h] = -INFINITY; continue; }
      double m = -INFINITY;
      for (int t = 0; t < k; ++t)
        if (ir[t] >= 0 && scale * s[t] > m) m = scale * s[t];
      double sum = 0.0;
      for (int t = 0; t < k; ++t)
        if (ir[t] >= 0) sum += exp(scale * s[t] - m);
      double L = m + log(sum);
      lse[i * H + h] = L;
      for (int t = 0; t < k; ++t) {
        if (ir[t] < 0) continue;
        p[t] = exp(scale * s[t] - L);
        const double* vr = V + ((int64_t)ir[t] * H + h) * (int64_t)d;
        for (int u = 0; u < d; ++u) o[u] += p[t] * vr[u];
      }
      if (!dO) continue;
      const double* go = dO + (i * H + h) * (int64_t)d;
      double D = 0.0;
      for (int t = 0; t < k; ++t) {
        if (ir[t] < 0) continue;
        const double* vr = V + ((int64_t)ir[t] * H + h) * (int64_t)d;
        double acc = 0.0;
        for (int u = 0; u < d; ++u) acc += go[u] * vr[u];
        dp[t] = acc;
        D += p[t] * acc;
      }
      double* gq = dQ + (i * H + h) * (int64_t)d;
      for (int u = 0; u < d; ++u) gq[u] = 0.0;
      for (int t = 0; t < k; ++t) {
        if (ir[t] < 0) continue;
        double ds = p[t] * (dp[t] - D);
        int64_t base = ((int64_t)ir[t] * H + h) * (int64_t)d;
        for (int u = 0; u < d; ++u) {
          gq[u] += scale * ds * K[base + u];
          dK[base + u] += scale * ds * q[u];
          dV[base + u] += p[t] * go[u];
        }
      }
    }
  }
  free(s); free(p); free(dp);
  return rc;
}

/*
 * Full softmax attention over every key of the query's graph, for the
 * diagnostics that compare k-MIP attention with it (k-Maximum Inner Product
 * Attention for Graph Transformers ..., Figure 8: the L2 distance between
 * the two outputs, and the share of the full softmax weight that the k kept
 * keys carry).  For query i of graph g and head h:
 *
 *   lse_full = log sum_{j in g} exp(scale * s_j)     (max-shifted)
 *   out_full = sum_{j in g} exp(scale * s_j - lse_full) V[j,h,:]
 *
 * For a list of (query, head) pairs (pairs_q == NULL: every pair, rows in
 * (i, h) order).  Returns 0, or 1 on malformed offsets, 2 on a bad pair.
 */
typedef struct {
  const double *Q, *K, *V;
  const int64_t* offsets;
  int64_t G, N;
  int H, d;
  double scale;
  const int64_t* pairs_q;
  const int32_t* pairs_h;
  int64_t npairs;
  double* out;
  double* lse;
  int64_t next;
  pthread_mutex_t lock;
} full_ctx;

static void full_one(const full_ctx* c, int64_t i, int h, int64_t row, double* s) {
  const int d = c->d, H = c->H;
  int64_t g = graph_of(c->offsets, c->G, i);
  int64_t j0 = c->offsets[g], j1 = c->offsets[g + 1];
  const double* q = c->Q + (i * H + h) * (int64_t)d;
  double m = -INFINITY;
  for (int64_t j = j0; j < j1; ++j) {
    const double* kr = c->K + (j * H + h) * (int64_t)d;
    double acc = 0.0;
    for (int t = 0; t < d; ++t) acc += q[t] * kr[t];
    s[j - j0] = c->scale * acc;
    if (s[j - j0] > m) m = s[j - j0];
  }
  double sum = 0.0;
  for (int64_t j = j0; j < j1; ++j) sum += exp(s[j - j0] - m);
  double L = m + log(sum);
  c->lse[row] = L;
  double* o = c->out + row * (int64_t)d;
  for (int t = 0; t < d; ++t) o[t] = 0.0;
  for (int64_t j = j0; j < j1; ++j) {
    double p = exp(s[j - j0] - L);
    const double* vr = c->V + (j * H + h) * (int64_t)d;
    for (int t = 0; t < d; ++t) o[t] += p * vr[t];
  }
}

static void* full_worker(void* arg) {
  full_ctx* c = (full_ctx*)arg;
  int64_t maxn = 1;
  for (int64_t g = 0; g < c->G; ++g)
    if (c->offsets[g + 1] - c->offsets[g] > maxn) maxn = c->offsets[g + 1] - c->offsets[g];
  double* s = (double*)malloc(sizeof(double) * (size_t)maxn);
  if (!s) return (void*)1;
  int64_t total = c->pairs_q ? c->npairs : c->N * c->H;
  for (;;) {
    pthread_mutex_lock(&c->lock);
    int64_t t = c->next;
    c->next += 16;
    pthread_mutex_unlock(&c->lock);
    if (t >= total) break;
    int64_t e = t + 16 < total ? t + 16 : total;
    for (; t < e; ++t) {
      if (c->pairs_q) full_one(c, c->pairs_q[t], c->pairs_h[t], t, s);
      else full_one(c, t / c->H, (int)(t % c->H), t, s);
    }
  }
  free(s);
  return NULL;
}

int kmip_oracle_full(const double* Q, const double* K, const double* V,
                     const int64_t* offsets, int64_t G, int64_t N, int H, int d,
                     double scale, const int64_t* pairs_q, const int32_t* pairs_h,
                     int64_t npairs, double* out, double* lse, int nthreads) {
  if (check_offsets(offsets, G, N)) return 1;
  if (pairs_q)
    for (int64_t t = 0; t < npairs; ++t)
      if (pairs_q[t] < 0 || pairs_q[t] >= N || pairs_h[t] < 0 || pairs_h[t] >= H) return 2;
  full_ctx c;
  memset(&c, 0, sizeof c);
  c.Q = Q; c.K = K; c.V = V; c.offsets = offsets; c.G = G; c.N = N; c.H = H; c.d = d;
  c.scale = scale; c.pairs_q = pairs_q; c.pairs_h = pairs_h; c.npairs = npairs;
  c.out = out; c.lse = lse;
  if (nthreads < 1) nthreads = 1;
  pthread_mutex_init(&c.lock, NULL);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  int rc = 0;
  for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, full_worker, &c);
  for (int t = 0; t < nthreads; ++t) {
    void* r = NULL;
    pthread_join(th[t], &r);
    if (r) rc = 3;
  }
  free(th);
  pthread_mutex_destroy(&c.lock);
  return rc;
}
