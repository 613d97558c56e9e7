/*
 * fp64 CPU oracle for certified Top-k attention truncation.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * restatement of what the method computes; it exists so the CUDA path can be
 * checked against it.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py may load it.  It shares no code, header, table or
 * helper with the CUDA library in certified_top_sparse_b200/csrc.
 *
 * Source of the definitions: "A Mathematical Theory of Top-k Sparse Attention
 * via Total Variation Distance" (Tzachristas et al., arXiv 2512.07647),
 * abstract as printed on the fugumt.com page for 2512.07647v1:
 *   - P is the softmax of the logits of one query, P-hat its Top-k truncation
 *     renormalised on the kept keys;
 *   - TV(P, P-hat) equals the discarded softmax tail mass and equals
 *     1 - exp(-KL(P-hat || P));
 *   - the minimal k_eps is the smallest k with TV(P, P-hat) <= eps;
 *   - head-tail factorisation ||Attn - Attn_k||_2 = tau ||mu_tail - mu_head||_2
 *     with tau = TV, and the diameter bound ||Attn - Attn_k||_2 <= tau diam_{H,T};
 *   - refinements in terms of Var_P(V).
 * The logits are s_i = q.k_i / sqrt(d) (scaled dot-product attention).
 *
 * Readings where the page is silent:
 *   - ties in the logits are broken by the lower key index ranking first;
 *   - the ranking uses the exact fp64 dot product u_i = q.k_i (the scale
 *     1/sqrt(d) is positive, so the order is the same as for s_i, and ranking
 *     on u avoids ties that the division by sqrt(d) could create by rounding);
 *   - the tail mass is summed directly from the smallest key upward and the
 *     certificate test is tail/Z <= eps, "<=" as printed;
 *   - diam_{H,T} = max over head key i and tail key j of ||v_i - v_j||_2;
 *   - the Var_P(V) refinement used as an invariant is derived, not printed:
 *     err^2 <= tau/(1-tau) * Var_P(V) (law of total variance over the
 *     head/tail split).
 *
 * Every floating-point quantity is fp64; the inputs (fp32 or bf16 bytes) are
 * widened exactly.  Sums use Neumaier-compensated accumulation.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORA_F32 0
#define ORA_BF16 1

/* Column layout of the per-row statistics array (ORA_NSTAT doubles per row). */
enum {
  ST_TV = 0,        /* TV = discarded tail mass / Z                            */
  ST_TV_DEF,        /* TV by its definition: 1/2 sum_i |P_i - Phat_i|           */
  ST_KL,            /* KL(Phat || P) from explicit log-probabilities            */
  ST_ONE_M_EXPKL,   /* 1 - exp(-KL)                                            */
  ST_ERR,           /* tau * ||mu_tail - mu_head||_2                            */
  ST_ERR_DIRECT,    /* ||Attn - Attn_k||_2 with Attn from a plain dense pass    */
  ST_TV_KM1,        /* TV of the Top-(k-1) truncation (1 when k = 1)            */
  ST_GAP_U,         /* u_(k) - u_(k+1) (unscaled dot products); NaN when k = n  */
  ST_TIE_BOUND,     /* gamma_d (sum_j |q_j k_(k)j| + sum_j |q_j k_(k+1)j|)      */
  ST_VAR_P,         /* Var_P(V) = sum_i P_i ||v_i - Attn||^2                     */
  ST_DIAM,          /* diam_{H,T}; NaN unless requested; 0 when the tail is empty */
  ST_MAX_S,         /* max_i s_i                                                */
  ST_LOG_Z,         /* log sum_i exp(s_i - max s)                               */
  ST_HEAD_MASS,     /* H = sum_head P_i                                         */
  ST_GAP_BOUND,     /* single-gap bound 1/(1 + k/(n-k) exp(s_(k) - s_(k+1)))    */
  ST_MIN_HEAD_U,    /* u_(k) */
  ORA_NSTAT
};

int ora_nstat(void) { return ORA_NSTAT; }

/* ---- exact widening of the input element types ------------------------- */

static double widen(const void* base, int dtype, int64_t i) {
  if (dtype == ORA_F32) {
    return (double)((const float*)base)[i];
  }
  /* bf16 is the upper half of an IEEE binary32 word. */
  uint16_t h = ((const uint16_t*)base)[i];
  uint32_t bits = (uint32_t)h << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* ---- Neumaier compensated sum --------------------------------------------- */

typedef struct { double s, c; } csum;

static void cs_add(csum* a, double x) {
  double t = a->s + x;
  if (fabs(a->s) >= fabs(x)) a->c += (a->s - t) + x;
  else a->c += (x - t) + a->s;
  a->s = t;
}
static double cs_val(const csum* a) { return a->s + a->c; }

/* ---- ordering: logit descending, key index ascending ------------------- */

typedef struct { double u; int64_t i; } ukey;

static int cmp_desc(const void* pa, const void* pb) {
  const ukey* a = (const ukey*)pa;
  const ukey* b = (const ukey*)pb;
  if (a->u > b->u) return -1;
  if (a->u < b->u) return 1;
  return (a->i < b->i) ? -1 : (a->i > b->i);
}
static int cmp_i64(const void* pa, const void* pb) {
  int64_t a = *(const int64_t*)pa, b = *(const int64_t*)pb;
  return (a > b) - (a < b);
}

/* ---- one attention row ---------------------------------------------------- */

typedef struct {
  /* inputs */
  const void *q, *K, *V;
  int dtype;
  int64_t batch, n_heads, n_kv_heads, m, n, d;
  double eps;
  int want_diam;
  int select_only;  /* 1: stop after k, idx and the TV values (no value rows read) */
  /* outputs */
  double* out;
  double* attn;
  int32_t* k_out;
  int32_t* idx_out;
  double* stats;
  /* work split */
  int64_t row_begin, row_end;
  int status;
} job;

typedef struct {
  ukey* ord;        /* [n] keys in rank order                     */
  double* w;        /* [n] exp(s - max s) in rank order            */
  double* suffix;   /* [n+1] tail sums in rank order               */
  double* w_idx;    /* [n] exp(s - max s) by key index             */
  double* s_idx;    /* [n] s_i - max s by key index                */
  double* qv;       /* [d] */
  csum* acc;        /* [3d] head, tail and full output sums        */
  int64_t* head;    /* [n] kept key indices                        */
} scratch;

static int do_row(const job* J, int64_t row, scratch* S) {
  const int64_t n = J->n, d = J->d;
  const int64_t group = J->n_heads / J->n_kv_heads;
  /* row = ((b * n_heads) + h) * m + j */
  const int64_t bh = row / J->m;
  const int64_t h = bh % J->n_heads;
  const int64_t b = bh / J->n_heads;
  const int64_t kvh = h / group;
  const int64_t kv_base = (b * J->n_kv_heads + kvh) * n * d; /* element offset of K[b,kvh,0,0] */
  ukey* ord = S->ord;
  double* w = S->w;
  double* suffix = S->suffix;
  double* qv = S->qv;

  for (int64_t t = 0; t < d; ++t) qv[t] = widen(J->q, J->dtype, row * d + t);

  /* Step 1: logits.  u_i = q . k_i (fp64); s_i = u_i / sqrt(d). */
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int64_t i = 0; i < n; ++i) {
    double u = 0.0;
    for (int64_t t = 0; t < d; ++t) u += qv[t] * widen(J->K, J->dtype, kv_base + i * d + t);
    if (!isfinite(u)) return -5;
    ord[i].u = u;
    ord[i].i = i;
  }

  /* Step 2: order keys by logit (descending), ties by lower index first. */
  qsort(ord, (size_t)n, sizeof(ukey), cmp_desc);

  /* Step 3: softmax numerators relative to the largest logit, in rank order. */
  const double max_s = ord[0].u * inv_sqrt_d;
  for (int64_t r = 0; r < n; ++r) {
    const double s_rel = ord[r].u * inv_sqrt_d - max_s;
    w[r] = exp(s_rel);
    S->w_idx[ord[r].i] = w[r];
    S->s_idx[ord[r].i] = s_rel;
  }

  /* Step 4: tail sums, smallest key first.  suffix[k] = sum of w over ranks
     k..n-1, i.e. the mass discarded when the top k keys are kept; Z = suffix[0]. */
  {
    csum acc = {0.0, 0.0};
    suffix[n] = 0.0;
    for (int64_t r = n - 1; r >= 0; --r) {
      cs_add(&acc, w[r]);
      suffix[r] = cs_val(&acc);
    }
  }
  const double Z = suffix[0];

  /* Step 5: minimal k with TV = tail / Z <= eps. */
  int64_t k = n;
  for (int64_t kk = 1; kk <= n; ++kk) {
    if (suffix[kk] / Z <= J->eps) { k = kk; break; }
  }

  /* Head mass summed directly (largest first), tail mass, TV. */
  csum hs = {0.0, 0.0};
  for (int64_t r = 0; r < k; ++r) cs_add(&hs, w[r]);
  const double Hsum = cs_val(&hs);
  const double Tsum = suffix[k];
  const double tv = Tsum / Z;

  /* Kept key indices, ascending. */
  for (int64_t r = 0; r < k; ++r) S->head[r] = ord[r].i;
  qsort(S->head, (size_t)k, sizeof(int64_t), cmp_i64);
  int32_t* idx_row = J->idx_out + row * n;
  for (int64_t r = 0; r < k; ++r) idx_row[r] = (int32_t)S->head[r];
  J->k_out[row] = (int32_t)k;

  double* st = J->stats + row * ORA_NSTAT;
  if (J->select_only) {
    for (int c = 0; c < ORA_NSTAT; ++c) st[c] = NAN;
    st[ST_TV] = tv;
    st[ST_TV_KM1] = (k == 1) ? 1.0 : suffix[k - 1] / Z;
    st[ST_GAP_U] = (k < n) ? ord[k - 1].u - ord[k].u : NAN;
    st[ST_MAX_S] = max_s;
    st[ST_LOG_Z] = log(Z);
    st[ST_HEAD_MASS] = Hsum / Z;
    st[ST_MIN_HEAD_U] = ord[k - 1].u;
    return 0;
  }

  /* Step 6: in key index order, TV by its definition (1/2 sum |P - Phat|),
     KL(Phat || P) from explicit log-probabilities, and the head, tail and
     full weighted sums of the value rows. */
  const double logZ = log(Z);
  const double logH = log(Hsum);
  csum tvd = {0.0, 0.0}, kl = {0.0, 0.0};
  csum* ch = S->acc;
  csum* ct = S->acc + d;
  csum* ca = S->acc + 2 * d;
  for (int64_t t = 0; t < 3 * d; ++t) { S->acc[t].s = 0.0; S->acc[t].c = 0.0; }
  int64_t hp = 0;
  for (int64_t i = 0; i < n; ++i) {
    const int in_head = (hp < k && idx_row[hp] == i);
    if (in_head) ++hp;
    const double wi = S->w_idx[i];
    const double P = wi / Z;
    const double Phat = in_head ? wi / Hsum : 0.0;
    cs_add(&tvd, fabs(P - Phat));
    if (in_head) {
      const double logP = S->s_idx[i] - logZ;     /* log P_i    */
      const double logPhat = S->s_idx[i] - logH;  /* log Phat_i */
      cs_add(&kl, Phat * (logPhat - logP));
    }
    const int64_t vrow = kv_base + i * d;
    for (int64_t t = 0; t < d; ++t) {
      const double v = widen(J->V, J->dtype, vrow + t);
      cs_add(&ca[t], wi * v);
      if (in_head) cs_add(&ch[t], wi * v);
      else cs_add(&ct[t], wi * v);
    }
  }

  /* Step 7: mu_head = Attn_k (the output), mu_tail, Attn, the error. */
  double* out_row = J->out + row * d;
  double e2 = 0.0, ed2 = 0.0;
  for (int64_t t = 0; t < d; ++t) {
    const double mu_h = cs_val(&ch[t]) / Hsum;
    const double a = cs_val(&ca[t]) / Z;
    out_row[t] = mu_h;
    if (J->attn) J->attn[row * d + t] = a;
    if (k < n) {
      const double mu_t = cs_val(&ct[t]) / Tsum;
      e2 += (mu_t - mu_h) * (mu_t - mu_h);
    }
    ed2 += (a - mu_h) * (a - mu_h);
  }
  const double err = (k < n) ? tv * sqrt(e2) : 0.0;

  /* Var_P(V) = sum_i P_i ||v_i - Attn||^2 */
  csum var = {0.0, 0.0};
  for (int64_t i = 0; i < n; ++i) {
    double dd = 0.0;
    for (int64_t t = 0; t < d; ++t) {
      const double diff = widen(J->V, J->dtype, kv_base + i * d + t) - cs_val(&ca[t]) / Z;
      dd += diff * diff;
    }
    cs_add(&var, (S->w_idx[i] / Z) * dd);
  }

  /* diam_{H,T}: max over head i, tail j of ||v_i - v_j|| (optional, O(k(n-k)d)). */
  double diam = NAN;
  if (J->want_diam) {
    double best = 0.0;
    int64_t hp2 = 0;
    for (int64_t i = 0; i < n; ++i) {
      if (hp2 < k && idx_row[hp2] == i) { ++hp2; continue; }
      for (int64_t r = 0; r < k; ++r) {
        const int64_t hi = idx_row[r];
        double dd = 0.0;
        for (int64_t t = 0; t < d; ++t) {
          const double diff = widen(J->V, J->dtype, kv_base + hi * d + t) -
                              widen(J->V, J->dtype, kv_base + i * d + t);
          dd += diff * diff;
        }
        if (dd > best) best = dd;
      }
    }
    diam = sqrt(best);
  }

  /* Boundary diagnostics: gap between the last kept and first dropped logit,
     the fp32 dot-product rounding bound for those two keys, the single-gap
     bound and TV of the Top-(k-1) truncation. */
  double gap_u = NAN, tie_bound = NAN, gap_bound = 0.0;
  if (k < n) {
    gap_u = ord[k - 1].u - ord[k].u;
    const double unit = ldexp(1.0, -24);
    const double gamma_d = (double)d * unit / (1.0 - (double)d * unit);
    double a1 = 0.0, a2 = 0.0;
    for (int64_t t = 0; t < d; ++t) {
      a1 += fabs(qv[t] * widen(J->K, J->dtype, kv_base + ord[k - 1].i * d + t));
      a2 += fabs(qv[t] * widen(J->K, J->dtype, kv_base + ord[k].i * d + t));
    }
    tie_bound = gamma_d * (a1 + a2);
    gap_bound = 1.0 / (1.0 + ((double)k / (double)(n - k)) * exp(gap_u * inv_sqrt_d));
  }
  const double tv_km1 = (k == 1) ? 1.0 : suffix[k - 1] / Z;

  st[ST_TV] = tv;
  st[ST_TV_DEF] = 0.5 * cs_val(&tvd);
  st[ST_KL] = cs_val(&kl);
  st[ST_ONE_M_EXPKL] = -expm1(-cs_val(&kl));
  st[ST_ERR] = err;
  st[ST_ERR_DIRECT] = sqrt(ed2);
  st[ST_TV_KM1] = tv_km1;
  st[ST_GAP_U] = gap_u;
  st[ST_TIE_BOUND] = tie_bound;
  st[ST_VAR_P] = cs_val(&var);
  st[ST_DIAM] = (J->want_diam && k == n) ? 0.0 : diam;
  st[ST_MAX_S] = max_s;
  st[ST_LOG_Z] = logZ;
  st[ST_HEAD_MASS] = Hsum / Z;
  st[ST_GAP_BOUND] = gap_bound;
  st[ST_MIN_HEAD_U] = ord[k - 1].u;
  return 0;
}

static void* run_job(void* arg) {
  job* J = (job*)arg;
  const size_t n = (size_t)J->n, d = (size_t)J->d;
  scratch S;
  S.ord = (ukey*)malloc(sizeof(ukey) * n);
  S.w = (double*)malloc(sizeof(double) * n);
  S.suffix = (double*)malloc(sizeof(double) * (n + 1));
  S.w_idx = (double*)malloc(sizeof(double) * n);
  S.s_idx = (double*)malloc(sizeof(double) * n);
  S.qv = (double*)malloc(sizeof(double) * d);
  S.acc = (csum*)malloc(sizeof(csum) * 3 * d);
  S.head = (int64_t*)malloc(sizeof(int64_t) * n);
  if (!S.ord || !S.w || !S.suffix || !S.w_idx || !S.s_idx || !S.qv || !S.acc || !S.head) {
    J->status = -3;
  } else {
    for (int64_t row = J->row_begin; row < J->row_end && J->status == 0; ++row)
      J->status = do_row(J, row, &S);
  }
  free(S.ord); free(S.w); free(S.suffix); free(S.w_idx); free(S.s_idx);
  free(S.qv); free(S.acc); free(S.head);
  return NULL;
}

/*
 * Certified Top-k attention for every (batch, head, query) row, in fp64.
 *
 * q   : [batch, n_heads, m, d]        (dtype ORA_F32 or ORA_BF16 raw bytes)
 * K, V: [batch, n_kv_heads, n, d]
 * Query head h reads KV head h / (n_heads / n_kv_heads).
 * Outputs (rows = batch * n_heads * m):
 *   out     [rows, d]   Attn_k = mu_head
 *   attn    [rows, d]   dense Attn (may be NULL)
 *   k_out   [rows]
 *   idx_out [rows, n]   first k_out[row] entries: kept keys, ascending
 *   stats   [rows, ORA_NSTAT]
 * select_only = 1 stops each row after k, idx and the TV values (out, attn
 * and the value-dependent statistics are left as NaN / untouched).
 * Returns 0, -1 on bad arguments, -3 on allocation failure, -5 on a
 * non-finite logit.
 */
int ora_certified_topk_attn(const void* q, const void* K, const void* V, int dtype,
                            int64_t batch, int64_t n_heads, int64_t n_kv_heads, int64_t m,
                            int64_t n, int64_t d, double eps, int nthreads, int want_diam,
                            int select_only, double* out, double* attn, int32_t* k_out, int32_t* idx_out,
                            double* stats) {
  if (!q || !K || !V || !out || !k_out || !idx_out || !stats) return -1;
  if (dtype != ORA_F32 && dtype != ORA_BF16) return -1;
  if (batch < 1 || n_heads < 1 || n_kv_heads < 1 || m < 1 || n < 1 || d < 1) return -1;
  if (n_heads % n_kv_heads != 0) return -1;
  if (n > INT32_MAX) return -1;
  if (!(eps > 0.0 && eps < 1.0)) return -1;
  const int64_t rows = batch * n_heads * m;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > rows) nthreads = (int)rows;
  job* jobs = (job*)calloc((size_t)nthreads, sizeof(job));
  pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) { free(jobs); free(th); return -3; }
  for (int t = 0; t < nthreads; ++t) {
    job* J = &jobs[t];
    J->q = q; J->K = K; J->V = V; J->dtype = dtype;
    J->batch = batch; J->n_heads = n_heads; J->n_kv_heads = n_kv_heads; J->m = m;
    J->n = n; J->d = d; J->eps = eps; J->want_diam = want_diam; J->select_only = select_only;
    J->out = out; J->attn = attn; J->k_out = k_out; J->idx_out = idx_out; J->stats = stats;
    J->row_begin = rows * t / nthreads;
    J->row_end = rows * (t + 1) / nthreads;
    J->status = 0;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, run_job, &jobs[t]);
  run_job(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
  int status = 0;
  for (int t = 0; t < nthreads; ++t) if (jobs[t].status != 0) status = jobs[t].status;
  free(jobs); free(th);
  return status;
}

/*
 * Plain dense softmax attention in fp64 (no sorting, no truncation), used as
 * the reference output Attn(q, K, V).  Same layouts as above; out [rows, d].
 */
int ora_dense_attn(const void* q, const void* K, const void* V, int dtype, int64_t batch,
                   int64_t n_heads, int64_t n_kv_heads, int64_t m, int64_t n, int64_t d,
                   double* out) {
  if (!q || !K || !V || !out) return -1;
  if (n_heads % n_kv_heads != 0 || n < 1 || d < 1) return -1;
  const int64_t group = n_heads / n_kv_heads;
  const int64_t rows = batch * n_heads * m;
  double* s = (double*)malloc(sizeof(double) * (size_t)n);
  if (!s) return -3;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int64_t row = 0; row < rows; ++row) {
    const int64_t bh = row / m;
    const int64_t h = bh % n_heads, b = bh / n_heads;
    const int64_t kv_base = (b * n_kv_heads + h / group) * n * d;
    double mx = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
      double u = 0.0;
      for (int64_t t = 0; t < d; ++t)
        u += widen(q, dtype, row * d + t) * widen(K, dtype, kv_base + i * d + t);
      s[i] = u * inv_sqrt_d;
      if (s[i] > mx) mx = s[i];
    }
    csum z = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) { s[i] = exp(s[i] - mx); cs_add(&z, s[i]); }
    const double Z = cs_val(&z);
    for (int64_t t = 0; t < d; ++t) {
      csum a = {0.0, 0.0};
      for (int64_t i = 0; i < n; ++i) cs_add(&a, s[i] * widen(V, dtype, kv_base + i * d + t));
      out[row * d + t] = cs_val(&a) / Z;
    }
  }
  free(s);
  return 0;
}

/*
 * The truncation to a GIVEN kept set, in fp64: the same definitions as above
 * (abstract of "A Mathematical Theory of Top-k Sparse Attention via Total
 * Variation Distance") applied to an arbitrary set S instead of the top k.
 * Used to judge a kept set found elsewhere (for example by fp32 arithmetic
 * near a boundary): P-hat = P restricted to S and renormalised, TV = sum of P
 * over the keys outside S, out = mu_head = sum_S P_i v_i / sum_S P_i,
 * err = TV ||mu_tail - mu_head||_2 with the tail the complement of S,
 * KL(P-hat || P) from explicit log-probabilities, and the TV after dropping
 * the lowest-ranked key of S (rank: logit descending, lower index first).
 *
 * sets [rows, n]: the first counts[row] entries of each row are the distinct
 * key indices of S (any order), counts[row] >= 1.
 * res [rows, 4]: TV(S), KL, err, TV(S minus its lowest-ranked key).
 * out [rows, d].  Returns 0, -1 on bad arguments, -3 on allocation failure,
 * -5 on a non-finite logit.
 */
int ora_eval_kept_set(const void* q, const void* K, const void* V, int dtype, int64_t batch,
                      int64_t n_heads, int64_t n_kv_heads, int64_t m, int64_t n, int64_t d,
                      const int32_t* sets, const int32_t* counts, double* out, double* res) {
  if (!q || !K || !V || !sets || !counts || !out || !res) return -1;
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0 || n < 1 || d < 1 || m < 1 ||
      batch < 1)
    return -1;
  const int64_t group = n_heads / n_kv_heads;
  const int64_t rows = batch * n_heads * m;
  double* u = (double*)malloc(sizeof(double) * (size_t)n);
  double* w = (double*)malloc(sizeof(double) * (size_t)n);
  unsigned char* in_s = (unsigned char*)malloc((size_t)n);
  csum* acc = (csum*)malloc(sizeof(csum) * 2 * (size_t)d);
  if (!u || !w || !in_s || !acc) {
    free(u); free(w); free(in_s); free(acc);
    return -3;
  }
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  int status = 0;
  for (int64_t row = 0; row < rows && status == 0; ++row) {
    const int64_t bh = row / m;
    const int64_t h = bh % n_heads, b = bh / n_heads;
    const int64_t kv_base = (b * n_kv_heads + h / group) * n * d;
    const int64_t cnt = counts[row];
    if (cnt < 1 || cnt > n) { status = -1; break; }
    /* logits and the row maximum */
    double mx = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
      double x = 0.0;
      for (int64_t t = 0; t < d; ++t)
        x += widen(q, dtype, row * d + t) * widen(K, dtype, kv_base + i * d + t);
      if (!isfinite(x)) { status = -5; break; }
      u[i] = x;
      if (x > mx) mx = x;
    }
    if (status != 0) break;
    memset(in_s, 0, (size_t)n);
    int64_t low = -1;  /* lowest-ranked key of S */
    for (int64_t r = 0; r < cnt; ++r) {
      const int64_t i = sets[row * n + r];
      if (i < 0 || i >= n || in_s[i]) { status = -1; break; }
      in_s[i] = 1;
      if (low < 0 || u[i] < u[low] || (u[i] == u[low] && i > low)) low = i;
    }
    if (status != 0) break;
    /* masses: kept, dropped, total; sums in key index order */
    csum zs = {0.0, 0.0}, hs = {0.0, 0.0}, ts = {0.0, 0.0};
    for (int64_t t = 0; t < 2 * d; ++t) { acc[t].s = 0.0; acc[t].c = 0.0; }
    for (int64_t i = 0; i < n; ++i) {
      w[i] = exp((u[i] - mx) * inv_sqrt_d);
      cs_add(&zs, w[i]);
      cs_add(in_s[i] ? &hs : &ts, w[i]);
      csum* a = acc + (in_s[i] ? 0 : d);
      for (int64_t t = 0; t < d; ++t) cs_add(&a[t], w[i] * widen(V, dtype, kv_base + i * d + t));
    }
    const double Z = cs_val(&zs), Hm = cs_val(&hs), Tm = cs_val(&ts);
    const double logZ = log(Z), logH = log(Hm);
    csum kl = {0.0, 0.0};
    for (int64_t i = 0; i < n; ++i) {
      if (!in_s[i]) continue;
      const double s_rel = (u[i] - mx) * inv_sqrt_d;
      const double phat = w[i] / Hm;
      cs_add(&kl, phat * ((s_rel - logH) - (s_rel - logZ)));
    }
    double e2 = 0.0;
    for (int64_t t = 0; t < d; ++t) {
      const double mu_h = cs_val(&acc[t]) / Hm;
      out[row * d + t] = mu_h;
      if (Tm > 0.0) {
        const double mu_t = cs_val(&acc[d + t]) / Tm;
        e2 += (mu_t - mu_h) * (mu_t - mu_h);
      }
    }
    const double tv = Tm / Z;
    res[row * 4 + 0] = tv;
    res[row * 4 + 1] = cs_val(&kl);
    res[row * 4 + 2] = (Tm > 0.0) ? tv * sqrt(e2) : 0.0;
    res[row * 4 + 3] = (Tm + w[low]) / Z;
  }
  free(u); free(w); free(in_s); free(acc);
  return status;
}
