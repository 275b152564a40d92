/*
 * fwpkm_oracle.c -- plain CPU oracle of the FwPKM retrieve + chunk-write loop.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file.  The product (the CUDA library) shares no
 * code with it and never calls it.
 *
 * Arithmetic is fp64 throughout.  The fast-weight state (V, K1, K2) is stored as
 * fp32 between chunks, exactly like the GPU state, so that both sides start every
 * chunk from representable values.  Every loop follows the method's definition in
 * the order the pages give it; there is no blocking, fusion or reordering.
 *
 * Sources (page title, section):
 *   [R]  "快速权重积键值记忆 Fast-weight Product Key Memory" (structured summary),
 *        section 方法步骤详情 (method steps 1-5) and 前置知识/积键值记忆 (PKM).
 *   [P]  "Fast-weight Product Key Memory" (paperlayer summary of arXiv 2601.00671v2),
 *        §2.2 PKM, §3 / §3.1 overview, §3.3 memorization, §3.4 addressing,
 *        §A.1 lookahead targets, §A.2 IDW scoring, §A.3 target normalisation,
 *        §A.4 loss reduction, §A.5 gating-weighted memorization, App. B pseudo code.
 *
 * Readings where the pages are silent (each one is a config field or flag):
 *   - IDW score: sigma = -log(eps_idw + ||q_j - K_j[a]||^2)  ([P] §A.2 names
 *     inverse-distance weighting on Euclidean distance only; softmax of this
 *     sigma is Shepard IDW with power 2).
 *   - per-half top-k size = final k; ties broken by lowest index.
 *   - "normalised weights" s' = softmax over the final k scores ([R] step 2).
 *   - lookahead target of token t is v_{t+1}; the last token of the sequence
 *     (of every pass) has no target ([P] §A.1).
 *   - z-score per token over d_v with population variance and eps_norm ([P] §A.3).
 *   - marginal slot usage pbar_j = chunk mean of the softmax of sigma over all n
 *     sub-keys ([P] §3.4 "marginal slot-usage distributions").
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_KEY_UPDATE 1
#define ORC_TARGET_NORM 2
#define ORC_LOOKAHEAD 4
#define ORC_GATE_WEIGHT 8

typedef struct {
  int n;      /* sub-keys per codebook; the memory has N = n*n slots */
  int h;      /* half query width; the query has d = 2h entries, half 1 first */
  int d_v;    /* value width */
  int k;      /* per-half top-k and final top-k */
  int chunk;  /* C: tokens per fast-weight update */
  double eps_idw;
  double eps_norm;
  double lr_key;
  unsigned flags;
} orc_cfg;

/* ---------------------------------------------------------------------------
 * Step 1 ([R] PKM; [P] §A.2): squared Euclidean distance of one half-query to
 * every sub-key of its codebook, in the direct form sum_e (q_e - K[a][e])^2.
 * ------------------------------------------------------------------------- */
void orc_subkey_dist(const orc_cfg* c, const double* qh, const float* K, double* D) {
  for (int a = 0; a < c->n; ++a) {
    double s = 0.0;
    for (int e = 0; e < c->h; ++e) {
      double diff = qh[e] - (double)K[(size_t)a * c->h + e];
      s += diff * diff;
    }
    D[a] = s;
  }
}

/* Step 2 ([R] PKM; [P] §2.2): the k nearest sub-keys of one half, ordered by
 * (distance ascending, index ascending).  Plain repeated selection. */
void orc_topk_half(const orc_cfg* c, const double* D, int32_t* A) {
  char* taken = (char*)calloc((size_t)c->n, 1);
  for (int r = 0; r < c->k; ++r) {
    int best = -1;
    for (int a = 0; a < c->n; ++a) {
      if (taken[a]) continue;
      if (best < 0 || D[a] < D[best]) best = a;  /* strict: keeps the lowest index on ties */
    }
    taken[best] = 1;
    A[r] = best;
  }
  free(taken);
}

/* IDW score of one sub-key ([P] §A.2 reading above). */
static double idw_score(const orc_cfg* c, double d2) { return -log(c->eps_idw + d2); }

/* Steps 3-4 ([R] PKM and step 2; [P] §2.2): restricted Cartesian search.
 * Given both halves' distance rows, return the final k slots I (rank order,
 * by score descending then slot ascending), their scores S and the softmax
 * weights w.  If forced != NULL the slot set and order are taken from it
 * instead (near-tie resynchronisation), and only S and w are computed. */
void orc_select(const orc_cfg* c, const double* D1, const double* D2, const int32_t* forced,
                int32_t* I, double* S, double* w) {
  const int k = c->k, n = c->n;
  if (forced) {
    for (int r = 0; r < k; ++r) {
      int32_t slot = forced[r];
      int a = slot / n, b = slot % n;
      I[r] = slot;
      S[r] = idw_score(c, D1[a]) + idw_score(c, D2[b]);
    }
  } else {
    int32_t* A1 = (int32_t*)malloc(sizeof(int32_t) * k);
    int32_t* A2 = (int32_t*)malloc(sizeof(int32_t) * k);
    orc_topk_half(c, D1, A1);
    orc_topk_half(c, D2, A2);
    /* all k*k candidate pairs (a, b) with score sigma1[a] + sigma2[b] */
    int kk = k * k;
    double* cs = (double*)malloc(sizeof(double) * kk);
    int32_t* cslot = (int32_t*)malloc(sizeof(int32_t) * kk);
    char* taken = (char*)calloc((size_t)kk, 1);
    for (int i = 0; i < k; ++i)
      for (int j = 0; j < k; ++j) {
        cs[i * k + j] = idw_score(c, D1[A1[i]]) + idw_score(c, D2[A2[j]]);
        cslot[i * k + j] = A1[i] * n + A2[j];
      }
    for (int r = 0; r < k; ++r) {
      int best = -1;
      for (int x = 0; x < kk; ++x) {
        if (taken[x]) continue;
        if (best < 0 || cs[x] > cs[best] || (cs[x] == cs[best] && cslot[x] < cslot[best])) best = x;
      }
      taken[best] = 1;
      I[r] = cslot[best];
      S[r] = cs[best];
    }
    free(A1); free(A2); free(cs); free(cslot); free(taken);
  }
  /* Step 4: softmax over the k final scores (the "normalised weights"). */
  double mx = S[0];
  for (int r = 1; r < k; ++r) if (S[r] > mx) mx = S[r];
  double z = 0.0;
  for (int r = 0; r < k; ++r) { w[r] = exp(S[r] - mx); z += w[r]; }
  for (int r = 0; r < k; ++r) w[r] /= z;
}

/* Steps 5-6 ([R] steps 2-3): vhat = sum_{rank order} w_r V[I_r];
 * o = g*vhat + (1-g)*v. */
void orc_read_values(const orc_cfg* c, const int32_t* I, const double* w, const float* V,
                     double* vhat) {
  for (int e = 0; e < c->d_v; ++e) vhat[e] = 0.0;
  for (int r = 0; r < c->k; ++r) {
    const float* row = V + (size_t)I[r] * c->d_v;
    for (int e = 0; e < c->d_v; ++e) vhat[e] += w[r] * (double)row[e];
  }
}

/* Target of a pair token ([P] §A.1 lookahead, §A.3 z-score normalisation). */
void orc_target(const orc_cfg* c, const double* u, double* tau) {
  const int dv = c->d_v;
  if (!(c->flags & ORC_TARGET_NORM)) {
    for (int e = 0; e < dv; ++e) tau[e] = u[e];
    return;
  }
  double mean = 0.0;
  for (int e = 0; e < dv; ++e) mean += u[e];
  mean /= dv;
  double var = 0.0;
  for (int e = 0; e < dv; ++e) var += (u[e] - mean) * (u[e] - mean);
  var /= dv;
  double inv = 1.0 / sqrt(var + c->eps_norm);
  for (int e = 0; e < dv; ++e) tau[e] = (u[e] - mean) * inv;
}

typedef struct {
  int32_t slot;
  int32_t t;
  int32_t r;
} orc_pair;

static int pair_cmp(const void* x, const void* y) {
  const orc_pair* a = (const orc_pair*)x;
  const orc_pair* b = (const orc_pair*)y;
  if (a->slot != b->slot) return a->slot < b->slot ? -1 : 1;
  if (a->t != b->t) return a->t < b->t ? -1 : 1;
  return 0;
}

/* ---------------------------------------------------------------------------
 * One chunk of one memory ([P] §3.1: reads use the state left by the previous
 * chunk; the fast weights are written after the chunk; App. B order: forward,
 * memorization, addressing).
 *
 *   len          tokens in this chunk (1..C)
 *   q [len][2h], v [len][d_v], g [len]   the chunk's inputs (fp64)
 *   v_next       value of the token after the chunk, or NULL if the chunk ends
 *                the sequence (its last token then has no lookahead target)
 *   K1, K2 [n][h], V [n*n][d_v]  fp32 state, updated in place
 *   o [len][d_v] output; I [len][k], w [len][k] (nullable) selected slots/weights
 *   forced [len][k] and force_mask [len] (both nullable): tokens whose mask is
 *   non-zero use the given slot list instead of the computed one.
 * ------------------------------------------------------------------------- */
/* Read phase of tokens [t0, t1) of a chunk ([R] steps 2-3): every token against the
 * frozen state.  Tokens are independent, so any split of the range gives the same values. */
typedef struct {
  const orc_cfg* c;
  int t0, t1;
  const double *q, *v, *g;
  const float *K1, *K2, *V;
  double *D1, *D2, *S, *w, *vhat, *o;
  int32_t* I;
  const int32_t *forced, *force_mask;
} orc_read_job;

static void* orc_read_range(void* arg) {
  const orc_read_job* j = (const orc_read_job*)arg;
  const orc_cfg* c = j->c;
  const int n = c->n, h = c->h, dv = c->d_v, k = c->k, d = 2 * h;
  for (int t = j->t0; t < j->t1; ++t) {
    orc_subkey_dist(c, j->q + (size_t)t * d, j->K1, j->D1 + (size_t)t * n);
    orc_subkey_dist(c, j->q + (size_t)t * d + h, j->K2, j->D2 + (size_t)t * n);
    const int32_t* f = (j->forced && j->force_mask && j->force_mask[t]) ? j->forced + (size_t)t * k : NULL;
    orc_select(c, j->D1 + (size_t)t * n, j->D2 + (size_t)t * n, f, j->I + (size_t)t * k, j->S + (size_t)t * k,
               j->w + (size_t)t * k);
    orc_read_values(c, j->I + (size_t)t * k, j->w + (size_t)t * k, j->V, j->vhat + (size_t)t * dv);
    for (int e = 0; e < dv; ++e)
      j->o[(size_t)t * dv + e] = j->g[t] * j->vhat[(size_t)t * dv + e] + (1.0 - j->g[t]) * j->v[(size_t)t * dv + e];
  }
  return NULL;
}

/* ---------------------------------------------------------------------------
 * Addressing step of one chunk of one memory ([R] step 5; [P] §3.4):
 * L_addr = -H(pbar_1) - H(pbar_2) with pbar_j the chunk mean of
 * P_j[t] = softmax_a(sigma_j[t][a]) over all n sub-keys, taken at the keys the chunk
 * was read with (D1, D2: the chunk's distance rows).  One gradient step of size lr_key
 * on K1, K2.
 * ------------------------------------------------------------------------- */
static void orc_key_step(const orc_cfg* c, int len, const double* q, const double* D1, const double* D2,
                         float* K1, float* K2) {
  const int n = c->n, h = c->h, d = 2 * h;
  double* P = (double*)malloc(sizeof(double) * (size_t)len * n);
  double* pbar = (double*)malloc(sizeof(double) * n);
  double* lp = (double*)malloc(sizeof(double) * n);
  double* gradK = (double*)malloc(sizeof(double) * (size_t)n * h);
  for (int j = 0; j < 2; ++j) {
    const double* Dj = j == 0 ? D1 : D2;
    float* Kj = j == 0 ? K1 : K2;
    for (int t = 0; t < len; ++t) {
      double z = 0.0;
      for (int a = 0; a < n; ++a) z += 1.0 / (c->eps_idw + Dj[(size_t)t * n + a]);
      for (int a = 0; a < n; ++a) P[(size_t)t * n + a] = (1.0 / (c->eps_idw + Dj[(size_t)t * n + a])) / z;
    }
    for (int a = 0; a < n; ++a) {
      double s = 0.0;
      for (int t = 0; t < len; ++t) s += P[(size_t)t * n + a];
      pbar[a] = s / len;
      lp[a] = log(pbar[a]);
    }
    for (size_t x = 0; x < (size_t)n * h; ++x) gradK[x] = 0.0;
    for (int t = 0; t < len; ++t) {
      double Lt = 0.0;
      for (int a = 0; a < n; ++a) Lt += P[(size_t)t * n + a] * lp[a];
      const double* qj = q + (size_t)t * d + (size_t)j * h;
      for (int b = 0; b < n; ++b) {
        /* dL_addr/dsigma_j[t][b] */
        double gam = P[(size_t)t * n + b] * (lp[b] - Lt) / len;
        /* dsigma/dK[b] = 2 (q - K[b]) / (eps + D) */
        double coef = gam * 2.0 / (c->eps_idw + Dj[(size_t)t * n + b]);
        for (int e = 0; e < h; ++e)
          gradK[(size_t)b * h + e] += coef * (qj[e] - (double)Kj[(size_t)b * h + e]);
      }
    }
    for (size_t x = 0; x < (size_t)n * h; ++x) Kj[x] = (float)((double)Kj[x] - c->lr_key * gradK[x]);
  }
  free(P); free(pbar); free(lp); free(gradK);
}

/* One chunk with its read phase split over `read_threads` threads (token ranges); the
 * write and the key step follow on the calling thread.  orc_chunk is the one-thread case. */
static void orc_chunk_threads(const orc_cfg* c, int len, const double* q, const double* v, const double* g,
                              const double* v_next, float* K1, float* K2, float* V, double* o, int32_t* I_out,
                              double* w_out, const int32_t* forced, const int32_t* force_mask, int read_threads) {
  const int n = c->n, h = c->h, dv = c->d_v, k = c->k, d = 2 * h;
  double* D1 = (double*)malloc(sizeof(double) * (size_t)len * n);
  double* D2 = (double*)malloc(sizeof(double) * (size_t)len * n);
  int32_t* I = (int32_t*)malloc(sizeof(int32_t) * (size_t)len * k);
  double* S = (double*)malloc(sizeof(double) * (size_t)len * k);
  double* w = (double*)malloc(sizeof(double) * (size_t)len * k);
  double* vhat = (double*)malloc(sizeof(double) * (size_t)len * dv);

  /* ---- read phase: every token of the chunk against the frozen state ---- */
  if (read_threads < 1) read_threads = 1;
  if (read_threads > len) read_threads = len;
  {
    orc_read_job* jobs = (orc_read_job*)malloc(sizeof(orc_read_job) * (size_t)read_threads);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)read_threads);
    for (int i = 0; i < read_threads; ++i) {
      orc_read_job jj = {c, (int)((long long)i * len / read_threads), (int)((long long)(i + 1) * len / read_threads),
                         q, v, g, K1, K2, V, D1, D2, S, w, vhat, o, I, forced, force_mask};
      jobs[i] = jj;
    }
    for (int i = 1; i < read_threads; ++i) pthread_create(&th[i], NULL, orc_read_range, &jobs[i]);
    orc_read_range(&jobs[0]);
    for (int i = 1; i < read_threads; ++i) pthread_join(th[i], NULL);
    free(jobs);
    free(th);
  }
  if (I_out) memcpy(I_out, I, sizeof(int32_t) * (size_t)len * k);
  if (w_out) memcpy(w_out, w, sizeof(double) * (size_t)len * k);

  /* ---- memorization ([R] step 4; [P] §3.3, §A.1-§A.5) ----
   * L_mem = 1/2 sum_t g_t ||tau_t - vhat_t||^2 summed (not averaged) over tokens
   * and features.  dL/dV_i = sum_{t: i in I_t} w_{t,i} g_t (vhat_t - tau_t).
   * Rows read by several tokens divide by their read count N_read,i; the step
   * size is 1 and nothing is clipped. */
  int npair_tok = 0;
  double* r = (double*)malloc(sizeof(double) * (size_t)len * dv);
  double* tau = (double*)malloc(sizeof(double) * dv);
  char* is_pair = (char*)calloc((size_t)len, 1);
  for (int t = 0; t < len; ++t) {
    const double* u;
    if (c->flags & ORC_LOOKAHEAD) {
      if (t + 1 < len) u = v + (size_t)(t + 1) * dv;
      else if (v_next) u = v_next;
      else continue; /* last token of the sequence: no lookahead target */
    } else {
      u = v + (size_t)t * dv;
    }
    is_pair[t] = 1;
    ++npair_tok;
    orc_target(c, u, tau);
    double gw = (c->flags & ORC_GATE_WEIGHT) ? g[t] : 1.0;
    for (int e = 0; e < dv; ++e) r[(size_t)t * dv + e] = gw * (vhat[(size_t)t * dv + e] - tau[e]);
  }
  orc_pair* pairs = (orc_pair*)malloc(sizeof(orc_pair) * (size_t)(npair_tok > 0 ? npair_tok : 1) * k);
  int np = 0;
  for (int t = 0; t < len; ++t) {
    if (!is_pair[t]) continue;
    for (int rr = 0; rr < k; ++rr) {
      pairs[np].slot = I[(size_t)t * k + rr];
      pairs[np].t = t;
      pairs[np].r = rr;
      ++np;
    }
  }
  qsort(pairs, (size_t)np, sizeof(orc_pair), pair_cmp); /* (slot, t) keys are unique */
  double* G = (double*)malloc(sizeof(double) * dv);
  for (int s0 = 0; s0 < np;) {
    int s1 = s0;
    while (s1 < np && pairs[s1].slot == pairs[s0].slot) ++s1;
    int32_t slot = pairs[s0].slot;
    int nread = s1 - s0;
    for (int e = 0; e < dv; ++e) G[e] = 0.0;
    for (int p = s0; p < s1; ++p) { /* token order */
      double wt = w[(size_t)pairs[p].t * k + pairs[p].r];
      for (int e = 0; e < dv; ++e) G[e] += wt * r[(size_t)pairs[p].t * dv + e];
    }
    float* row = V + (size_t)slot * dv;
    for (int e = 0; e < dv; ++e) row[e] = (float)((double)row[e] - G[e] / nread);
    s0 = s1;
  }

  if (c->flags & ORC_KEY_UPDATE) orc_key_step(c, len, q, D1, D2, K1, K2);

  free(D1); free(D2); free(I); free(S); free(w); free(vhat);
  free(r); free(tau); free(is_pair); free(pairs); free(G);
}

void orc_chunk(const orc_cfg* c, int len, const double* q, const double* v, const double* g,
               const double* v_next, float* K1, float* K2, float* V, double* o, int32_t* I_out,
               double* w_out, const int32_t* forced, const int32_t* force_mask) {
  orc_chunk_threads(c, len, q, v, g, v_next, K1, K2, V, o, I_out, w_out, forced, force_mask, 1);
}

/* ---------------------------------------------------------------------------
 * One chunk of H heads that share one value table ([P] §D.1 ablates the head count
 * with the slot count; §D.3: more heads raise the collision rate, i.e. heads read one
 * table).  Readings where the pages are silent:
 *   - head h has its own codebooks K1^h, K2^h and its own query q^h, and selects its own
 *     k slots I^h_t with its own softmax weights s'^h_t (steps 1-4 per head);
 *   - the memory's read is the mean of the heads' reads:
 *       vhat_t = (1/H) sum_h sum_{i in I^h_t} s'^h_{t,i} V_i
 *     (all H k weights sum to 1, as for one head reading H k slots), and
 *     o_t = g_t vhat_t + (1 - g_t) v_t;
 *   - the write is the gradient of L_mem = 1/2 sum_t g_t ||tau_t - vhat_t||^2 with
 *     respect to the shared rows, G_i = sum_t sum_h [i in I^h_t] (s'^h_{t,i} / H) r_t,
 *     divided by N_read,i = the number of the chunk's pair tokens that read row i
 *     through at least one head; V_i -= G_i / N_read,i;
 *   - each head's codebooks take their own addressing step (L_addr of that head).
 *   q [H][len][2h], v [len][d_v], g [len], v_next [d_v] or NULL (per sequence)
 *   K1, K2 [H][n][h] fp32 (updated), V [n*n][d_v] fp32 (shared, updated)
 *   o [len][d_v]; I_out [H][len][k], w_out [H][len][k] (nullable)
 *   forced [H][len][k] and force_mask [H][len] (both nullable): a head-token whose mask is
 *   non-zero uses the given slot list (near-tie resynchronisation).
 * ------------------------------------------------------------------------- */
typedef struct {
  int32_t slot;
  int32_t t;
  int32_t hd;
  int32_t r;
} orc_hpair;

static int hpair_cmp(const void* x, const void* y) {
  const orc_hpair* a = (const orc_hpair*)x;
  const orc_hpair* b = (const orc_hpair*)y;
  if (a->slot != b->slot) return a->slot < b->slot ? -1 : 1;
  if (a->t != b->t) return a->t < b->t ? -1 : 1;
  if (a->hd != b->hd) return a->hd < b->hd ? -1 : 1;
  return 0;
}

void orc_chunk_heads(const orc_cfg* c, int H, int len, const double* q, const double* v, const double* g,
                     const double* v_next, float* K1, float* K2, float* V, double* o, int32_t* I_out,
                     double* w_out, const int32_t* forced, const int32_t* force_mask) {
  const int n = c->n, h = c->h, dv = c->d_v, k = c->k, d = 2 * h;
  const size_t nk = (size_t)n * h;
  double* D1 = (double*)malloc(sizeof(double) * (size_t)H * len * n);
  double* D2 = (double*)malloc(sizeof(double) * (size_t)H * len * n);
  int32_t* I = (int32_t*)malloc(sizeof(int32_t) * (size_t)H * len * k);
  double* S = (double*)malloc(sizeof(double) * (size_t)H * len * k);
  double* w = (double*)malloc(sizeof(double) * (size_t)H * len * k);
  double* vh = (double*)malloc(sizeof(double) * dv);
  double* vhat = (double*)malloc(sizeof(double) * (size_t)len * dv);

  /* ---- read phase: every head of every token against the frozen state ---- */
  for (int t = 0; t < len; ++t) {
    for (int e = 0; e < dv; ++e) vhat[(size_t)t * dv + e] = 0.0;
    for (int hd = 0; hd < H; ++hd) {
      const size_t ht = (size_t)hd * len + t;
      const double* qt = q + ht * d;
      orc_subkey_dist(c, qt, K1 + (size_t)hd * nk, D1 + ht * n);
      orc_subkey_dist(c, qt + h, K2 + (size_t)hd * nk, D2 + ht * n);
      const int32_t* f = (forced && force_mask && force_mask[ht]) ? forced + ht * k : NULL;
      orc_select(c, D1 + ht * n, D2 + ht * n, f, I + ht * k, S + ht * k, w + ht * k);
      orc_read_values(c, I + ht * k, w + ht * k, V, vh);
      for (int e = 0; e < dv; ++e) vhat[(size_t)t * dv + e] += vh[e];
    }
    for (int e = 0; e < dv; ++e) {
      vhat[(size_t)t * dv + e] /= H;
      o[(size_t)t * dv + e] = g[t] * vhat[(size_t)t * dv + e] + (1.0 - g[t]) * v[(size_t)t * dv + e];
    }
  }
  if (I_out) memcpy(I_out, I, sizeof(int32_t) * (size_t)H * len * k);
  if (w_out) memcpy(w_out, w, sizeof(double) * (size_t)H * len * k);

  /* ---- memorization: the gradient of the gated loss on the shared rows ---- */
  double* r = (double*)malloc(sizeof(double) * (size_t)len * dv);
  double* tau = (double*)malloc(sizeof(double) * dv);
  char* is_pair = (char*)calloc((size_t)len, 1);
  int npair_tok = 0;
  for (int t = 0; t < len; ++t) {
    const double* u;
    if (c->flags & ORC_LOOKAHEAD) {
      if (t + 1 < len) u = v + (size_t)(t + 1) * dv;
      else if (v_next) u = v_next;
      else continue; /* last token of the sequence: no lookahead target */
    } else {
      u = v + (size_t)t * dv;
    }
    is_pair[t] = 1;
    ++npair_tok;
    orc_target(c, u, tau);
    double gw = (c->flags & ORC_GATE_WEIGHT) ? g[t] : 1.0;
    for (int e = 0; e < dv; ++e) r[(size_t)t * dv + e] = gw * (vhat[(size_t)t * dv + e] - tau[e]);
  }
  orc_hpair* pairs = (orc_hpair*)malloc(sizeof(orc_hpair) * (size_t)(npair_tok > 0 ? npair_tok : 1) * H * k);
  int np = 0;
  for (int t = 0; t < len; ++t) {
    if (!is_pair[t]) continue;
    for (int hd = 0; hd < H; ++hd)
      for (int rr = 0; rr < k; ++rr) {
        pairs[np].slot = I[((size_t)hd * len + t) * k + rr];
        pairs[np].t = t;
        pairs[np].hd = hd;
        pairs[np].r = rr;
        ++np;
      }
  }
  qsort(pairs, (size_t)np, sizeof(orc_hpair), hpair_cmp); /* (slot, t, head) keys are unique */
  double* G = (double*)malloc(sizeof(double) * dv);
  for (int s0 = 0; s0 < np;) {
    int s1 = s0;
    while (s1 < np && pairs[s1].slot == pairs[s0].slot) ++s1;
    const int32_t slot = pairs[s0].slot;
    int nread = 0;
    for (int e = 0; e < dv; ++e) G[e] = 0.0;
    for (int pp = s0; pp < s1; ++pp) { /* token order, then head order */
      if (pp == s0 || pairs[pp].t != pairs[pp - 1].t) ++nread;
      const double wt = w[((size_t)pairs[pp].hd * len + pairs[pp].t) * k + pairs[pp].r] / H;
      for (int e = 0; e < dv; ++e) G[e] += wt * r[(size_t)pairs[pp].t * dv + e];
    }
    float* row = V + (size_t)slot * dv;
    for (int e = 0; e < dv; ++e) row[e] = (float)((double)row[e] - G[e] / nread);
    s0 = s1;
  }

  /* ---- addressing: each head's own step ---- */
  if (c->flags & ORC_KEY_UPDATE)
    for (int hd = 0; hd < H; ++hd)
      orc_key_step(c, len, q + (size_t)hd * len * d, D1 + (size_t)hd * len * n, D2 + (size_t)hd * len * n,
                   K1 + (size_t)hd * nk, K2 + (size_t)hd * nk);

  free(D1); free(D2); free(I); free(S); free(w); free(vh); free(vhat);
  free(r); free(tau); free(is_pair); free(pairs); free(G);
}

/* ---------------------------------------------------------------------------
 * Whole sequence of one memory, n_iter passes over the same input
 * ([P] §3.1 chunk-sequential schedule; [R] 技术新颖性 iterative memorization).
 * The state carries across chunks and passes.  o, I, w hold the final pass.
 * ------------------------------------------------------------------------- */
static void orc_run_sequence_threads(const orc_cfg* c, int T, int n_iter, const double* q, const double* v,
                                     const double* g, float* K1, float* K2, float* V, double* o, int32_t* I,
                                     double* w, int read_threads) {
  const int d = 2 * c->h, dv = c->d_v, k = c->k;
  for (int pass = 0; pass < n_iter; ++pass) {
    for (int t0 = 0; t0 < T; t0 += c->chunk) {
      int len = T - t0 < c->chunk ? T - t0 : c->chunk;
      const double* v_next = (t0 + len < T) ? v + (size_t)(t0 + len) * dv : NULL;
      orc_chunk_threads(c, len, q + (size_t)t0 * d, v + (size_t)t0 * dv, g + t0, v_next, K1, K2, V,
                        o + (size_t)t0 * dv, I ? I + (size_t)t0 * k : NULL, w ? w + (size_t)t0 * k : NULL,
                        NULL, NULL, read_threads);
    }
  }
}

void orc_run_sequence(const orc_cfg* c, int T, int n_iter, const double* q, const double* v,
                      const double* g, float* K1, float* K2, float* V, double* o, int32_t* I,
                      double* w) {
  orc_run_sequence_threads(c, T, n_iter, q, v, g, K1, K2, V, o, I, w, 1);
}

/* Independent memories (sequence x head) in parallel threads: nothing is shared
 * between memories, so this is the same computation as one call per memory.  With more
 * threads than memories, each memory also splits the read phase of its chunks over
 * nthreads / M threads (token ranges).  I (nullable) receives the final pass's slots. */
typedef struct {
  const orc_cfg* c;
  int T, n_iter, M, nthreads, tid, read_threads;
  const double *q, *v, *g;
  float *K1, *K2, *V;
  double* o;
  int32_t* I;
} orc_job;

static void* orc_worker(void* arg) {
  orc_job* j = (orc_job*)arg;
  const orc_cfg* c = j->c;
  const size_t d = 2 * (size_t)c->h, dv = (size_t)c->d_v, n = (size_t)c->n, h = (size_t)c->h, k = (size_t)c->k;
  for (int m = j->tid; m < j->M; m += j->nthreads) {
    orc_run_sequence_threads(c, j->T, j->n_iter, j->q + (size_t)m * j->T * d, j->v + (size_t)m * j->T * dv,
                             j->g + (size_t)m * j->T, j->K1 + (size_t)m * n * h, j->K2 + (size_t)m * n * h,
                             j->V + (size_t)m * n * n * dv, j->o + (size_t)m * j->T * dv,
                             j->I ? j->I + (size_t)m * j->T * k : NULL, NULL, j->read_threads);
  }
  return NULL;
}

int orc_run_sequence_multi(const orc_cfg* c, int M, int T, int n_iter, const double* q,
                           const double* v, const double* g, float* K1, float* K2, float* V,
                           double* o, int32_t* I, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  const int read_threads = nthreads > M ? nthreads / M : 1;
  const int mem_threads = nthreads > M ? M : nthreads;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * mem_threads);
  orc_job* jobs = (orc_job*)malloc(sizeof(orc_job) * mem_threads);
  for (int i = 0; i < mem_threads; ++i) {
    orc_job jj = {c, T, n_iter, M, mem_threads, i, read_threads, q, v, g, K1, K2, V, o, I};
    jobs[i] = jj;
    pthread_create(&th[i], NULL, orc_worker, &jobs[i]);
  }
  for (int i = 0; i < mem_threads; ++i) pthread_join(th[i], NULL);
  free(th);
  free(jobs);
  return mem_threads * read_threads;
}
