/*
 * CPU oracle for the forward pass of one sparse Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product (the CUDA
 * path behind libmoe) never calls it, links it or shares code with it.
 *
 * Plain, slow and deliberately unoptimised: every quantity is computed from its
 * definition, one token at a time, accumulating in fp64 (double). Inputs are the
 * exact values the GPU receives (fp32, or bf16 bit patterns widened exactly).
 *
 * Sources (the reviewed pages; each function cites the passage it follows):
 *  [R&Q]  "A Replicate-and-Quantize Strategy for Plug-and-Play Load Balancing of
 *         Sparse Mixture-of-Experts LLMs" (pith.science/paper/HUR5XFER):
 *         Definition 1 (n_{i,j}, LIS = m * max_j n_{i,j} / (n k)); the note that
 *         the method applies to top-1, top-2 and shared-expert routing.
 *  [FloE] "FloE: On-the-Fly MoE Inference on Memory-constrained GPU"
 *         (pith.science/paper/WSOUZLYL): expert matrices W_gate, W_up, W_down
 *         with a SiLU gate ("What carries the argument", "Core claim").
 *  [Omni] "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale"
 *         (pith.science/paper/2602.05711): expert-centric scheduling (Fig. 3),
 *         Cartesian Product Router (Sec. 2.2, Eq. 8), exact top-K over the grid
 *         (App. A), atomic experts sigma(x w_in^T) w_out (Eq. 4), shared dense
 *         MLP branch.
 * Where the pages leave a step open the reading taken is stated at the step.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { O_F32 = 0, O_BF16 = 1 };
enum { O_SWIGLU = 0, O_RELU = 1 };
enum { O_SILU = 0, O_SIGMOID = 1 };

typedef struct {
  int32_t T, d, f, m, k;
  int32_t act;      /* O_SWIGLU or O_RELU */
  int32_t dtype;    /* O_F32 or O_BF16 */
  int32_t n_shared; /* always-on shared experts */
  int32_t f_shared;
  int32_t renorm;   /* 1: divide the k gate weights by their sum */
} oracle_cfg_t;

/* Exact value of element i of a fp32 or bf16 array. */
static double val(const void* p, int dtype, int64_t i) {
  if (dtype == O_F32) return (double)((const float*)p)[i];
  uint32_t b = (uint32_t)((const uint16_t*)p)[i] << 16;
  float f;
  memcpy(&f, &b, 4);
  return (double)f;
}

static double logistic(double z) { return 1.0 / (1.0 + exp(-z)); }

/* ------------------------------------------------------------------ routing */

/* Router logits (R&Q: token-choice routing over m experts; the router is a linear
 * map of the token). logit[t,e] = fl32( sum_i x[t,i] W_r[e,i] + bias[e] ), the sum
 * taken in fp64 and rounded once to fp32. bias may be NULL. */
int oracle_router_logits(int T, int d, int m, int dtype, const void* x, const void* w_r,
                         const float* bias, float* logits) {
  if (T < 0 || d <= 0 || m <= 0) return 1;
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < m; ++e) {
      double s = 0.0;
      for (int i = 0; i < d; ++i) s += val(x, dtype, (int64_t)t * d + i) * val(w_r, dtype, (int64_t)e * d + i);
      if (bias) s += (double)bias[e];
      logits[(int64_t)t * m + e] = (float)s;
    }
  return 0;
}

/* Top-k selection and gate weights for one token.
 * Selection: experts ordered by (logit descending, expert index ascending); the
 * first k are slots 0..k-1 in that order.
 * Weights: p = softmax over all m logits (fp64, max subtracted); w_s = p[idx_s],
 * or p[idx_s] / sum_s' p[idx_s'] when renormalised. */
static void topk_one(int m, int k, int renorm, const float* lg, int32_t* idx, double* w) {
  char* taken = (char*)calloc((size_t)m, 1);
  for (int s = 0; s < k; ++s) {
    int best = -1;
    for (int e = 0; e < m; ++e) {
      if (taken[e]) continue;
      if (best < 0 || lg[e] > lg[best]) best = e; /* strict '>' keeps the lower index on ties */
    }
    taken[best] = 1;
    idx[s] = best;
  }
  free(taken);
  double mx = -INFINITY;
  for (int e = 0; e < m; ++e)
    if ((double)lg[e] > mx) mx = (double)lg[e];
  double z = 0.0;
  for (int e = 0; e < m; ++e) z += exp((double)lg[e] - mx);
  double sel = 0.0;
  for (int s = 0; s < k; ++s) {
    w[s] = exp((double)lg[idx[s]] - mx) / z;
    sel += w[s];
  }
  if (renorm)
    for (int s = 0; s < k; ++s) w[s] /= sel;
}

int oracle_topk_softmax(int T, int m, int k, int renorm, const float* logits, int32_t* idx, double* w) {
  if (T < 0 || m <= 0 || k <= 0 || k > m) return 1;
  for (int t = 0; t < T; ++t)
    topk_one(m, k, renorm, logits + (int64_t)t * m, idx + (int64_t)t * k, w + (int64_t)t * k);
  return 0;
}

/* ------------------------------------------------------- histogram and LIS */

/* R&Q Definition 1: n_j = number of (token, slot) assignments routed to expert j
 * in this layer; LIS = m * max_j n_j / (n * k) with n = T tokens. offsets is the
 * exclusive prefix sum of the counts (segment starts, m+1 entries); argmax is the
 * lowest expert index attaining the maximum (the heavy hitter of R&Q Alg. 1).
 * Returns 2 if an expert id is outside [0, m). */
int oracle_histogram_lis(int T, int k, int m, const int32_t* idx, int32_t* counts, int32_t* offsets,
                         int32_t* max_count, int32_t* argmax, double* lis) {
  if (T <= 0 || k <= 0 || m <= 0) return 1;
  for (int e = 0; e < m; ++e) counts[e] = 0;
  for (int64_t q = 0; q < (int64_t)T * k; ++q) {
    if (idx[q] < 0 || idx[q] >= m) return 2;
    counts[idx[q]] += 1;
  }
  offsets[0] = 0;
  for (int e = 0; e < m; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int best = 0;
  for (int e = 1; e < m; ++e)
    if (counts[e] > counts[best]) best = e;
  *max_count = counts[best];
  *argmax = best;
  *lis = (double)((int64_t)m * counts[best]) / (double)((int64_t)T * k);
  return 0;
}

/* Expert-centric permutation (OmniMoE Fig. 3: tasks reordered so that each
 * active expert's tasks form one contiguous group). Task q = t*k + s. Walking the
 * tasks in increasing q, each takes the next free position of its expert's
 * segment: pos = offsets[e] + cursor[e]++. So segments are contiguous and hold
 * their tasks in increasing task id. perm[pos] = q, inv_perm[q] = pos. */
int oracle_permutation(int T, int k, int m, const int32_t* idx, const int32_t* offsets, int32_t* perm,
                       int32_t* inv_perm) {
  if (T <= 0 || k <= 0 || m <= 0) return 1;
  int32_t* cursor = (int32_t*)calloc((size_t)m, sizeof(int32_t));
  for (int64_t q = 0; q < (int64_t)T * k; ++q) {
    int e = idx[q];
    if (e < 0 || e >= m) {
      free(cursor);
      return 2;
    }
    int32_t pos = offsets[e] + cursor[e]++;
    perm[pos] = (int32_t)q;
    inv_perm[q] = pos;
  }
  free(cursor);
  return 0;
}

/* Replica dispatch (R&Q, "A Replicate-and-Quantize Strategy for Plug-and-Play
 * Load Balancing of Sparse Mixture-of-Experts LLMs", Sec. 2.5 / Algorithm 3: a
 * copy of the heavy-hitter is appended to the layer; the page gives no rule that
 * sends tokens to it, and its review suggests splitting the heavy-hitter's tokens
 * alternately between the original and the replica). The heavy-hitter h is the
 * expert with the most tasks, n_j of Definition 1 (lowest index on ties). Its
 * tasks are taken in increasing task id q = t*k + s, the order of its segment in
 * the expert-centric permutation: the 1st, 3rd, 5th, ... stay with h, the 2nd,
 * 4th, ... go to the replica, expert m. Every other task keeps its expert. */
int oracle_replica_split(int T, int k, int m, const int32_t* idx, int32_t* idx_out, int32_t* heavy) {
  if (T <= 0 || k <= 0 || m <= 0) return 1;
  int32_t* counts = (int32_t*)calloc((size_t)m, sizeof(int32_t));
  for (int64_t q = 0; q < (int64_t)T * k; ++q) {
    if (idx[q] < 0 || idx[q] >= m) {
      free(counts);
      return 2;
    }
    counts[idx[q]] += 1;
  }
  int h = 0;
  for (int e = 1; e < m; ++e)
    if (counts[e] > counts[h]) h = e;
  int64_t r = 0; /* tasks of h seen so far */
  for (int64_t q = 0; q < (int64_t)T * k; ++q) {
    if (idx[q] == h) {
      idx_out[q] = (r % 2 == 1) ? m : h;
      ++r;
    } else {
      idx_out[q] = idx[q];
    }
  }
  *heavy = h;
  free(counts);
  return 0;
}

/* ------------------------------------------------------------------ experts */

/* One expert applied to one token, fp64 throughout.
 * SwiGLU (FloE: W_gate, W_up, W_down with a SiLU gate; OmniMoE Sec. 2.1):
 *   g = x W_gate^T, u = x W_up^T, h = g * sigma(g) * u, y = h W_down^T.
 * ReLU (Switch-style two-matrix FFN): h = max(0, x W_1^T), y = h W_2^T, with
 *   W_1 passed as wg and W_2 as wd.
 * xr: the token as d doubles; wg, wu: [f, d]; wd: [d, f]; h: scratch of f doubles. */
static void expert_ffn(int d, int f, int act, int dtype, const double* xr, const void* wg, const void* wu,
                       const void* wd, double* h, double* y) {
  for (int j = 0; j < f; ++j) {
    double g = 0.0;
    for (int i = 0; i < d; ++i) g += xr[i] * val(wg, dtype, (int64_t)j * d + i);
    if (act == O_SWIGLU) {
      double u = 0.0;
      for (int i = 0; i < d; ++i) u += xr[i] * val(wu, dtype, (int64_t)j * d + i);
      h[j] = g * logistic(g) * u;
    } else {
      h[j] = g > 0.0 ? g : 0.0;
    }
  }
  for (int o = 0; o < d; ++o) {
    double s = 0.0;
    for (int j = 0; j < f; ++j) s += h[j] * val(wd, dtype, (int64_t)o * f + j);
    y[o] = s;
  }
}

int oracle_expert_ffn(int d, int f, int act, int dtype, const void* x_row, const void* wg, const void* wu,
                      const void* wd, double* y) {
  double* xr = (double*)malloc(sizeof(double) * (size_t)d);
  double* h = (double*)malloc(sizeof(double) * (size_t)f);
  for (int i = 0; i < d; ++i) xr[i] = val(x_row, dtype, i);
  expert_ffn(d, f, act, dtype, xr, wg, wu, wd, h, y);
  free(xr);
  free(h);
  return 0;
}

typedef struct {
  const oracle_cfg_t* c;
  const int32_t* tokens;
  int lo, hi;
  const void *x, *wg, *wu, *wd, *sg, *su, *sd;
  const int32_t* idx;
  const double* w;
  double* out;
} out_job_t;

/* Layer output for one token (combine step; the pages never write it out, the
 * standard reading is used): out_t = sum_s w[t,s] * FFN_{idx[t,s]}(x_t)
 *                                   + sum_sh FFN_sh(x_t)   (shared experts, weight 1:
 * R&Q's shared-expert routing; OmniMoE's always-active shared dense MLP). */
static void layer_output_token(const out_job_t* J, int t, double* xr, double* h, double* y, double* o) {
  const oracle_cfg_t* c = J->c;
  const int d = c->d, f = c->f, k = c->k;
  const int es = c->dtype == O_F32 ? 4 : 2;
  for (int i = 0; i < d; ++i) xr[i] = val(J->x, c->dtype, (int64_t)t * d + i);
  for (int i = 0; i < d; ++i) o[i] = 0.0;
  for (int s = 0; s < k; ++s) {
    int e = J->idx[(int64_t)t * k + s];
    const size_t mat = (size_t)f * d * es;
    expert_ffn(d, f, c->act, c->dtype, xr, (const char*)J->wg + e * mat,
               J->wu ? (const char*)J->wu + e * mat : 0, (const char*)J->wd + e * mat, h, y);
    double ws = J->w[(int64_t)t * k + s];
    for (int i = 0; i < d; ++i) o[i] += ws * y[i];
  }
  for (int sh = 0; sh < c->n_shared; ++sh) {
    const size_t mat = (size_t)c->f_shared * d * es;
    expert_ffn(d, c->f_shared, c->act, c->dtype, xr, (const char*)J->sg + sh * mat,
               J->su ? (const char*)J->su + sh * mat : 0, (const char*)J->sd + sh * mat, h, y);
    for (int i = 0; i < d; ++i) o[i] += y[i];
  }
}

static void* out_worker(void* p) {
  const out_job_t* J = (const out_job_t*)p;
  const oracle_cfg_t* c = J->c;
  int fmax = c->f > c->f_shared ? c->f : c->f_shared;
  double* xr = (double*)malloc(sizeof(double) * (size_t)c->d);
  double* h = (double*)malloc(sizeof(double) * (size_t)fmax);
  double* y = (double*)malloc(sizeof(double) * (size_t)c->d);
  for (int n = J->lo; n < J->hi; ++n) {
    int t = J->tokens ? J->tokens[n] : n;
    layer_output_token(J, t, xr, h, y, J->out + (int64_t)n * c->d);
  }
  free(xr);
  free(h);
  free(y);
  return 0;
}

static void run_jobs(out_job_t* base, int ntok, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > ntok) nthreads = ntok > 0 ? ntok : 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  int running[256];
  out_job_t jobs[256];
  int chunk = (ntok + nthreads - 1) / nthreads;
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = *base;
    jobs[i].lo = i * chunk;
    jobs[i].hi = (i + 1) * chunk < ntok ? (i + 1) * chunk : ntok;
    running[i] = 0;
    if (jobs[i].lo >= jobs[i].hi) continue;
    if (nthreads > 1 && pthread_create(&th[i], 0, out_worker, &jobs[i]) == 0)
      running[i] = 1;
    else
      out_worker(&jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i)
    if (running[i]) pthread_join(th[i], 0);
}

/* Layer output for a list of tokens (tokens == NULL: tokens 0..ntok-1), given the
 * routing (idx [T,k], w [T,k]). out: ntok x d doubles. */
int oracle_moe_output(const oracle_cfg_t* c, const int32_t* tokens, int ntok, const void* x, const void* w_gate,
                      const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                      const void* ws_down, const int32_t* idx, const double* w, double* out, int nthreads) {
  if (!c || c->d <= 0 || c->f <= 0 || c->k <= 0 || ntok < 0) return 1;
  if (c->act == O_SWIGLU && (!w_up || (c->n_shared && !ws_up))) return 1;
  for (int n = 0; n < ntok; ++n) {
    int t = tokens ? tokens[n] : n;
    if (t < 0 || t >= c->T) return 1;
    for (int s = 0; s < c->k; ++s)
      if (idx[(int64_t)t * c->k + s] < 0 || idx[(int64_t)t * c->k + s] >= c->m) return 2;
  }
  out_job_t J = {c, tokens, 0, 0, x, w_gate, c->act == O_SWIGLU ? w_up : 0, w_down,
                 ws_gate, c->act == O_SWIGLU ? ws_up : 0, ws_down, idx, w, out};
  run_jobs(&J, ntok, nthreads);
  return 0;
}

/* The whole layer forward for all T tokens, in the order the path takes it:
 * router logits -> top-k and gate weights -> counts, offsets and LIS -> the
 * expert-centric permutation -> expert FFNs -> weighted combine. logits_in (may
 * be NULL) replaces the router projection, as when the caller already holds the
 * fp32 logits. The permutation is produced for comparison; the output itself is
 * the per-token sum of its definition. */
int oracle_layer_forward(const oracle_cfg_t* c, const void* x, const void* w_r, const float* bias,
                         const float* logits_in, const void* w_gate, const void* w_up, const void* w_down,
                         const void* ws_gate, const void* ws_up, const void* ws_down, float* logits,
                         int32_t* idx, double* w, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv_perm, int32_t* max_count, int32_t* argmax, double* lis, double* out,
                         int nthreads) {
  int rc;
  if (logits_in)
    memcpy(logits, logits_in, sizeof(float) * (size_t)c->T * c->m);
  else if ((rc = oracle_router_logits(c->T, c->d, c->m, c->dtype, x, w_r, bias, logits)))
    return rc;
  if ((rc = oracle_topk_softmax(c->T, c->m, c->k, c->renorm, logits, idx, w))) return rc;
  if ((rc = oracle_histogram_lis(c->T, c->k, c->m, idx, counts, offsets, max_count, argmax, lis))) return rc;
  if ((rc = oracle_permutation(c->T, c->k, c->m, idx, offsets, perm, inv_perm))) return rc;
  return oracle_moe_output(c, 0, c->T, x, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, idx, w, out, nthreads);
}

/* Brute-force dense-masked evaluator (a second, differently structured check of
 * the same definition): every token is run through EVERY expert, and the
 * routing enters only as a mask, out_t = sum_e [e selected for t] * w_{t,e} *
 * FFN_e(x_t) + shared. Tiny inputs only (cost T*m expert evaluations). */
int oracle_dense_masked(const oracle_cfg_t* c, const void* x, const void* w_gate, const void* w_up,
                        const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down,
                        const int32_t* idx, const double* w, double* out) {
  const int d = c->d, f = c->f, m = c->m, k = c->k;
  const int es = c->dtype == O_F32 ? 4 : 2;
  int fmax = f > c->f_shared ? f : c->f_shared;
  double* xr = (double*)malloc(sizeof(double) * (size_t)d);
  double* h = (double*)malloc(sizeof(double) * (size_t)fmax);
  double* ye = (double*)malloc(sizeof(double) * (size_t)m * d);
  for (int t = 0; t < c->T; ++t) {
    for (int i = 0; i < d; ++i) xr[i] = val(x, c->dtype, (int64_t)t * d + i);
    for (int e = 0; e < m; ++e) {
      const size_t mat = (size_t)f * d * es;
      expert_ffn(d, f, c->act, c->dtype, xr, (const char*)w_gate + e * mat,
                 c->act == O_SWIGLU ? (const char*)w_up + e * mat : 0, (const char*)w_down + e * mat, h,
                 ye + (int64_t)e * d);
    }
    double* o = out + (int64_t)t * d;
    for (int i = 0; i < d; ++i) o[i] = 0.0;
    for (int e = 0; e < m; ++e) {
      double mask_w = 0.0;
      for (int s = 0; s < k; ++s)
        if (idx[(int64_t)t * k + s] == e) mask_w += w[(int64_t)t * k + s];
      for (int i = 0; i < d; ++i) o[i] += mask_w * ye[(int64_t)e * d + i];
    }
    for (int sh = 0; sh < c->n_shared; ++sh) {
      const size_t mat = (size_t)c->f_shared * d * es;
      expert_ffn(d, c->f_shared, c->act, c->dtype, xr, (const char*)ws_gate + sh * mat,
                 c->act == O_SWIGLU ? (const char*)ws_up + sh * mat : 0, (const char*)ws_down + sh * mat, h,
                 ye);
      for (int i = 0; i < d; ++i) o[i] += ye[i];
    }
  }
  free(xr);
  free(h);
  free(ye);
  return 0;
}

/* ------------------------------------------------------------ atomic experts */

/* Cartesian Product Router, row/column factors (OmniMoE Sec. 2.2, Eq. 8: the
 * joint expert probability factorises as p_r(i|x) p_c(j|x), so its log is the
 * sum of a row and a column log-probability).
 * lr[t,i] = fl32( z_i - logsumexp(z) ), z = x_t W_row^T in fp64; lc likewise. */
static void log_softmax_rows(int T, int d, int n, int dtype, const void* x, const void* w, float* out) {
  double* z = (double*)malloc(sizeof(double) * (size_t)n);
  for (int t = 0; t < T; ++t) {
    double mx = -INFINITY;
    for (int i = 0; i < n; ++i) {
      double s = 0.0;
      for (int q = 0; q < d; ++q) s += val(x, dtype, (int64_t)t * d + q) * val(w, dtype, (int64_t)i * d + q);
      z[i] = s;
      if (s > mx) mx = s;
    }
    double se = 0.0;
    for (int i = 0; i < n; ++i) se += exp(z[i] - mx);
    double lse = mx + log(se);
    for (int i = 0; i < n; ++i) out[(int64_t)t * n + i] = (float)(z[i] - lse);
  }
  free(z);
}

int oracle_atomic_logprobs(int T, int d, int Nr, int Nc, int dtype, const void* x, const void* w_row,
                           const void* w_col, float* lr, float* lc) {
  if (T <= 0 || d <= 0 || Nr <= 0 || Nc <= 0) return 1;
  log_softmax_rows(T, d, Nr, dtype, x, w_row, lr);
  log_softmax_rows(T, d, Nc, dtype, x, w_col, lc);
  return 0;
}

typedef struct {
  float s;
  int32_t id;
} scored_t;

/* (score descending, flat id ascending); -0.0 and +0.0 compare equal. */
static int cmp_scored(const void* a, const void* b) {
  const scored_t* p = (const scored_t*)a;
  const scored_t* q = (const scored_t*)b;
  if (p->s > q->s) return -1;
  if (p->s < q->s) return 1;
  return (p->id > q->id) - (p->id < q->id);
}

/* Exact global top-K over the implicit Nr x Nc grid (OmniMoE App. A: the
 * selection recovers the exact top-K indices over the grid). By brute force:
 * every expert (i, j), flat id i*Nc + j, gets S = fl32(lr_i + lc_j) (one fp32
 * addition); all Nr*Nc are sorted by (S desc, id asc) and the first K kept.
 * Gate weights: g = softmax of the K selected S, fp64 (the routing scores g_x of
 * OmniMoE Fig. 2; equal to the renormalised product p_r p_c of Eq. 8). */
int oracle_atomic_select(int T, int Nr, int Nc, int K, const float* lr, const float* lc, int32_t* idx,
                         double* g) {
  const int64_t N = (int64_t)Nr * Nc;
  if (T <= 0 || K <= 0 || K > N) return 1;
  scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)N);
  for (int t = 0; t < T; ++t) {
    for (int i = 0; i < Nr; ++i)
      for (int j = 0; j < Nc; ++j) {
        float s = lr[(int64_t)t * Nr + i] + lc[(int64_t)t * Nc + j];
        all[(int64_t)i * Nc + j].s = s;
        all[(int64_t)i * Nc + j].id = (int32_t)((int64_t)i * Nc + j);
      }
    qsort(all, (size_t)N, sizeof(scored_t), cmp_scored);
    double mx = (double)all[0].s, z = 0.0;
    for (int q = 0; q < K; ++q) z += exp((double)all[q].s - mx);
    for (int q = 0; q < K; ++q) {
      idx[(int64_t)t * K + q] = all[q].id;
      g[(int64_t)t * K + q] = exp((double)all[q].s - mx) / z;
    }
  }
  free(all);
  return 0;
}

/* Dynamic Expert Assembly with atomic experts (OmniMoE Eq. 4 and Fig. 2): each
 * selected expert e contributes g * act(x_t . w_in[e]) * w_out[e]; the
 * activation is unnamed on the page: SiLU (default) or the logistic sigmoid.
 * out: ntok x d doubles, tokens == NULL means 0..ntok-1. */
int oracle_atomic_output(int T, int d, int K, int act, int dtype, const void* x, const void* w_in,
                         const void* w_out, const int32_t* idx, const double* g, const int32_t* tokens, int ntok,
                         double* out) {
  if (T <= 0 || d <= 0 || K <= 0) return 1;
  for (int n = 0; n < ntok; ++n) {
    int t = tokens ? tokens[n] : n;
    if (t < 0 || t >= T) return 1;
    double* o = out + (int64_t)n * d;
    for (int i = 0; i < d; ++i) o[i] = 0.0;
    for (int s = 0; s < K; ++s) {
      int64_t e = idx[(int64_t)t * K + s];
      double z = 0.0;
      for (int i = 0; i < d; ++i) z += val(x, dtype, (int64_t)t * d + i) * val(w_in, dtype, e * d + i);
      double a = act == O_SILU ? z * logistic(z) : logistic(z);
      double c = g[(int64_t)t * K + s] * a;
      for (int i = 0; i < d; ++i) o[i] += c * val(w_out, dtype, e * d + i);
    }
  }
  return 0;
}
