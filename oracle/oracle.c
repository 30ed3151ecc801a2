/*
 * Oracle for the draft-sample-and-verify step -- TEST INFRASTRUCTURE ONLY.
 * See oracle.h for what is computed, the readings taken, and the pins.
 * Plain C, double precision, one batch row at a time in the order the
 * method states; rows are independent, so they are spread over OpenMP
 * threads without changing any result.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int g_threads_used = 1;
int orc_threads_used(void) { return g_threads_used; }

/* ---------------------------------------------------------------------------
 * Philox4x32-10, Salmon et al. SC'11, section 4 ("Philox"): each round takes
 * the counter (c0,c1,c2,c3) and round key (k0,k1) to
 *   (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0));
 * the round key is bumped by the Weyl constants between rounds.  The paper's
 * multipliers and Weyl constants for N=4, W=32 are used.
 * ------------------------------------------------------------------------- */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += PHILOX_W0;
      k1 += PHILOX_W1;
    }
    uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
    uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    uint32_t n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

double orc_u01(uint32_t x) { return (double)(x >> 8) * (1.0 / 16777216.0); }

double orc_uniform(uint64_t seed, uint64_t cycle, uint32_t b, uint32_t pos, uint32_t tag) {
  uint32_t ctr[4], key[2], out[4];
  key[0] = (uint32_t)seed;
  key[1] = (uint32_t)(seed >> 32);
  ctr[0] = pos;
  ctr[1] = b;
  ctr[2] = (uint32_t)cycle;
  ctr[3] = (tag & 0xFFFFu) | ((uint32_t)((cycle >> 32) & 0xFFFFu) << 16);
  orc_philox4x32_10(ctr, key, out);
  return orc_u01(out[0]);
}

/* ------------------------------------------------------------------------- */

static double load_elem(const void *p, int32_t dtype, int64_t idx) {
  if (dtype == ORC_BF16) {
    uint16_t h = ((const uint16_t *)p)[idx];
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float *)p)[idx];
}

void orc_row_stats(const double *x, int32_t n, double T, double *m, double *Z) {
  double mx = -INFINITY;
  for (int32_t v = 0; v < n; ++v) {
    double l = x[v] / T;
    if (l > mx) mx = l;
  }
  double s = 0.0;
  for (int32_t v = 0; v < n; ++v) s += exp(x[v] / T - mx);
  *m = mx;
  *Z = s;
}

int32_t orc_icdf(const double *w, int32_t n, double u, int32_t *near) {
  double total = 0.0;
  for (int32_t v = 0; v < n; ++v) total += w[v];
  double target = u * total;
  double margin = 1e-6 * total;
  double c = 0.0;
  int32_t last_pos = -1;
  for (int32_t v = 0; v < n; ++v) {
    if (w[v] > 0.0) last_pos = v;
    double before = c;
    c += w[v];
    if (c > target) {
      if (near) *near = (target - before < margin) || (c - target < margin);
      return v;
    }
  }
  if (near) *near = 1;
  return last_pos;
}

/* Lowest index of the maximum; *near set when another index is within tol. */
static int32_t argmax_lowest(const double *x, int32_t n, int32_t *near, double rel_tol) {
  int32_t best = 0;
  for (int32_t v = 1; v < n; ++v)
    if (x[v] > x[best]) best = v;
  if (near) {
    double tol = rel_tol * fmax(1.0, fabs(x[best]));
    *near = 0;
    for (int32_t v = 0; v < n; ++v)
      if (v != best && x[best] - x[v] < tol) { *near = 1; break; }
  }
  return best;
}

/* probabilities of x/T: prob[v] = exp(x/T - m)/Z */
static void softmax_T(const double *x, int32_t n, double T, double *prob) {
  double m, Z;
  orc_row_stats(x, n, T, &m, &Z);
  for (int32_t v = 0; v < n; ++v) prob[v] = exp(x[v] / T - m) / Z;
}

int32_t orc_verify_probs(int32_t K, int32_t V, const double *p, const double *q,
                         const int32_t *d, const double *u_acc, const double *u_res,
                         int32_t *out, int32_t *tau, double *p_d,
                         int32_t *flag_accept, int32_t *flag_final) {
  if (flag_accept) *flag_accept = K;
  if (flag_final) *flag_final = 0;
  for (int32_t i = 0; i <= K; ++i) out[i] = -1;
  if (p_d)
    for (int32_t i = 0; i < K; ++i) p_d[i] = NAN;
  double *res = (double *)malloc(sizeof(double) * (size_t)V);
  int32_t stop = K;
  for (int32_t i = 0; i < K; ++i) {
    const double *pi = p + (size_t)i * V;
    const double *qi = q + (size_t)i * V;
    double pd = pi[d[i]], qd = qi[d[i]];
    if (p_d) p_d[i] = pd;
    double a = pd / qd;
    if (a > 1.0) a = 1.0;
    if (flag_accept && *flag_accept == K && fabs(u_acc[i] - a) < 1e-6) *flag_accept = i;
    if (u_acc[i] < a) {
      out[i] = d[i];
      continue;
    }
    /* first rejection: resample from the normalised residual max(p - q, 0) */
    double R = 0.0;
    for (int32_t v = 0; v < V; ++v) {
      double r = pi[v] - qi[v];
      res[v] = r > 0.0 ? r : 0.0;
#if defined(ORC_PLANT) && ORC_PLANT == 1
      res[v] = pi[v]; /* planted mistake: resample from p instead of the residual */
#endif
      R += res[v];
    }
    if (R == 0.0)
      for (int32_t v = 0; v < V; ++v) res[v] = pi[v];
    int32_t nearf = 0;
    out[i] = orc_icdf(res, V, u_res[i], &nearf);
    if (flag_final) *flag_final = nearf || (R < 1e-4);
    stop = i;
    break;
  }
  if (stop == K) {
    /* every draft accepted: bonus token from target row K */
    int32_t nearf = 0;
#if defined(ORC_PLANT) && ORC_PLANT == 3
    out[K] = orc_icdf(p + (size_t)(K - 1) * V, V, u_res[K], &nearf); /* planted: wrong row */
#else
    out[K] = orc_icdf(p + (size_t)K * V, V, u_res[K], &nearf);
#endif
    if (flag_final) *flag_final = nearf;
  }
  *tau = stop + 1;
  free(res);
  return stop;
}

/* ------------------------------------------------------------------------- */

static void biased_row(const orc_params *P, const void *base, const void *U, const void *W,
                       int32_t b, int32_t i, int32_t prev, double *z) {
  const int32_t K = P->K, V = P->V, r = P->r;
  const int64_t row = ((int64_t)b * K + i) * V;
  for (int32_t v = 0; v < V; ++v) z[v] = 0.0;
  /* bias[v] = sum_k U[prev,k] * W[k,v], accumulated in ascending k */
  for (int32_t k = 0; k < r; ++k) {
    double u = load_elem(U, P->dtype, (int64_t)prev * r + k);
    const int64_t wrow = (int64_t)k * V;
    for (int32_t v = 0; v < V; ++v) z[v] += u * load_elem(W, P->dtype, wrow + v);
  }
  for (int32_t v = 0; v < V; ++v) z[v] = load_elem(base, P->dtype, row + v) + z[v];
}

int orc_biased_row(const orc_params *P, const void *base, const void *U, const void *W,
                   int32_t b, int32_t i, int32_t prev, double *z) {
  if (!P || prev < 0 || prev >= P->V || b < 0 || b >= P->B || i < 0 || i >= P->K) return -1;
  biased_row(P, base, U, W, b, i, prev, z);
  return 0;
}

static int check_params(const orc_params *P, int32_t b_begin, int32_t b_end) {
  if (!P || P->B < 0 || P->K < 1 || P->V < 1 || P->r < 0) return -1;
  if (b_begin < 0 || b_end > P->B || b_begin > b_end) return -1;
  if (!P->greedy && !(P->temperature > 0.0)) return -1;
  if (P->verify_len)
    for (int32_t b = b_begin; b < b_end; ++b)
      if (P->verify_len[b] < 1 || P->verify_len[b] > P->K) return -4;
  return 0;
}

/* Verify length of row b: K_b, or K without a per-row array. */
static int32_t verify_len_of(const orc_params *P, int32_t b) {
  return P->verify_len ? P->verify_len[b] : P->K;
}

/* fp32 -> bf16 -> fp32, rounding to nearest with ties to even (finite x). */
static float round_bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  float y;
  memcpy(&y, &u, 4);
  return y;
}

/* RNN head state update (orc_params.Wh): s_new from s_old (NULL at i = 0). */
static void rnn_state(const orc_params *P, const void *U, int32_t prev, const float *s_old,
                      float *s_new) {
  const int32_t r = P->r;
  for (int32_t j = 0; j < r; ++j) {
    float acc = 0.0f;
#if !(defined(ORC_PLANT) && ORC_PLANT == 4) /* planted mistake: the state forgets the prefix */
    if (s_old)
      for (int32_t k = 0; k < r; ++k)
        acc = fmaf(s_old[k], (float)load_elem(P->Wh, P->dtype, (int64_t)j * r + k), acc);
#endif
    const float pre = (float)load_elem(U, P->dtype, (int64_t)prev * r + j) + acc;
    const float h = fminf(fmaxf(pre, -1.0f), 1.0f);
    s_new[j] = P->dtype == ORC_BF16 ? round_bf16(h) : h;
  }
}

/* z = base[b, i, :] + s . W for an explicit head state s[r] (double). */
static void biased_row_state(const orc_params *P, const void *base, const void *W, int32_t b,
                             int32_t i, const float *s, double *z) {
  const int32_t K = P->K, V = P->V, r = P->r;
  const int64_t row = ((int64_t)b * K + i) * V;
  for (int32_t v = 0; v < V; ++v) z[v] = 0.0;
  for (int32_t k = 0; k < r; ++k) {
    const double u = s[k];
    const int64_t wrow = (int64_t)k * V;
    for (int32_t v = 0; v < V; ++v) z[v] += u * load_elem(W, P->dtype, wrow + v);
  }
  for (int32_t v = 0; v < V; ++v) z[v] = load_elem(base, P->dtype, row + v) + z[v];
}

/* Draft one row: fills d[K], qd[K], zrows[K*V] (z values), flag. */
static int draft_row(const orc_params *P, const void *base, const void *U, const void *W,
                     int32_t b, int32_t prev0, int32_t *d, double *qd, double *zrows,
                     int32_t *flag_draft, double *scratch) {
  const int32_t K = P->K, V = P->V, Kb = verify_len_of(P, b);
  int32_t prev = prev0;
  float *st = NULL;  /* RNN head: the state of the last step and the next one */
  if (P->Wh) st = (float *)malloc(sizeof(float) * 2 * (size_t)(P->r > 0 ? P->r : 1));
  if (flag_draft) *flag_draft = K;
  for (int32_t i = Kb; i < K; ++i) {  /* positions past the verify length are not drafted */
    d[i] = -1;
    qd[i] = NAN;
  }
  for (int32_t i = 0; i < Kb; ++i) {
    double *z = zrows + (size_t)i * V;
    if (st) {
      float *s_new = st + (size_t)(i & 1) * P->r, *s_old = st + (size_t)((i + 1) & 1) * P->r;
      rnn_state(P, U, prev, i == 0 ? NULL : s_old, s_new);
      biased_row_state(P, base, W, b, i, s_new, z);
    } else {
      biased_row(P, base, U, W, b, i, prev, z);
    }
    int32_t near = 0, tok;
    if (P->greedy) {
      tok = argmax_lowest(z, V, &near, 1e-5);
      qd[i] = NAN;
    } else {
      double m, Z;
      orc_row_stats(z, V, P->temperature, &m, &Z);
      for (int32_t v = 0; v < V; ++v) scratch[v] = exp(z[v] / P->temperature - m);
      double u = orc_uniform(P->seed, P->cycle, (uint32_t)b, (uint32_t)i, ORC_TAG_DRAFT);
      tok = orc_icdf(scratch, V, u, &near);
      qd[i] = scratch[tok] / Z;
    }
    if (flag_draft && near && *flag_draft == K) *flag_draft = i;
    d[i] = tok;
#if defined(ORC_PLANT) && ORC_PLANT == 2
    prev = prev0; /* planted mistake: the Markov head always sees the last committed token */
#else
    prev = tok;
#endif
  }
  free(st);
  return 0;
}

/* Verify one row given z rows (draft logits, double) and tokens. */
static void verify_row(const orc_params *P, const void *target, const double *zrows,
                       const int32_t *d, int32_t b, int32_t *out, int32_t *tau, double *pd,
                       double *qd_out, int32_t *flag_accept, int32_t *flag_final) {
  const int32_t Kfull = P->K, V = P->V;
  const int32_t K = verify_len_of(P, b);  /* the row's verify length K_b; bonus from row K_b */
  const double T = P->temperature;
  for (int32_t j = 0; j <= Kfull; ++j) out[j] = -1;
  if (pd)
    for (int32_t j = 0; j < Kfull; ++j) pd[j] = NAN;
  if (qd_out)
    for (int32_t j = 0; j < Kfull; ++j) qd_out[j] = NAN;
  double *trow = (double *)malloc(sizeof(double) * (size_t)V * (K + 1));
  for (int32_t i = 0; i <= K; ++i)
    for (int32_t v = 0; v < V; ++v)
      trow[(size_t)i * V + v] = load_elem(target, P->dtype, ((int64_t)b * (Kfull + 1) + i) * V + v);
  if (P->greedy) {
    /* accept while argmax(target_i) == d_i; emit the target arg-max at the stop */
    int32_t i;
    for (int32_t j = 0; j <= K; ++j) out[j] = -1;
    for (i = 0; i < K; ++i) {
      int32_t am = argmax_lowest(trow + (size_t)i * V, V, NULL, 0.0);
      if (pd) pd[i] = NAN;
      if (am == d[i]) {
        out[i] = d[i];
        continue;
      }
      out[i] = am;
      break;
    }
    if (i == K) out[K] = argmax_lowest(trow + (size_t)K * V, V, NULL, 0.0);
    *tau = i + 1;
    if (flag_accept) *flag_accept = Kfull;
    if (flag_final) *flag_final = 0;
    free(trow);
    return;
  }
  double *p = (double *)malloc(sizeof(double) * (size_t)V * (K + 1));
  double *q = (double *)malloc(sizeof(double) * (size_t)V * K);
  for (int32_t i = 0; i <= K; ++i) softmax_T(trow + (size_t)i * V, V, T, p + (size_t)i * V);
  for (int32_t i = 0; i < K; ++i) softmax_T(zrows + (size_t)i * V, V, T, q + (size_t)i * V);
  double *u_acc = (double *)malloc(sizeof(double) * (size_t)K);
  double *u_res = (double *)malloc(sizeof(double) * (size_t)(K + 1));
  for (int32_t i = 0; i < K; ++i)
    u_acc[i] = orc_uniform(P->seed, P->cycle, (uint32_t)b, (uint32_t)i, ORC_TAG_ACCEPT);
  for (int32_t i = 0; i <= K; ++i)
    u_res[i] = orc_uniform(P->seed, P->cycle, (uint32_t)b, (uint32_t)i, ORC_TAG_RESAMPLE);
  orc_verify_probs(K, V, p, q, d, u_acc, u_res, out, tau, pd, flag_accept, flag_final);
  if (flag_accept && *flag_accept == K) *flag_accept = Kfull;  /* "no flag" is K */
  if (qd_out)
    for (int32_t i = 0; i < K; ++i) qd_out[i] = q[(size_t)i * V + d[i]];
  free(u_acc);
  free(u_res);
  free(p);
  free(q);
  free(trow);
}

#define ROWP(ptr, n) ((ptr) ? (ptr) + (size_t)(bb) * (n) : NULL)

int orc_cycle(const orc_params *P, const void *base, const void *target, const void *U,
              const void *W, const int32_t *last_token, int32_t b_begin, int32_t b_end,
              orc_outputs *o) {
  if (check_params(P, b_begin, b_end) || !base || !target || !last_token || !o) return -1;
  if (P->r > 0 && (!U || !W)) return -1;
  const int32_t K = P->K, V = P->V;
  for (int32_t b = b_begin; b < b_end; ++b)
    if (last_token[b] < 0 || last_token[b] >= V) return -2;
  int bad = 0;
  int threads = 1;
#pragma omp parallel reduction(| : bad)
  {
#ifdef _OPENMP
#pragma omp single
    threads = omp_get_num_threads();
#endif
    double *z = (double *)malloc(sizeof(double) * (size_t)K * V);
    double *scratch = (double *)malloc(sizeof(double) * (size_t)V);
    int32_t *d = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    double *qd = (double *)malloc(sizeof(double) * (size_t)K);
    int32_t *outb = (int32_t *)malloc(sizeof(int32_t) * (size_t)(K + 1));
#pragma omp for schedule(dynamic, 1)
    for (int32_t b = b_begin; b < b_end; ++b) {
      const int32_t bb = b - b_begin;
      int32_t fd = K, fa = K, ff = 0, tau = 0;
      draft_row(P, base, U, W, b, last_token[b], d, qd, z, &fd, scratch);
      verify_row(P, target, z, d, b, outb, &tau, ROWP(o->p_draft, K), NULL, &fa, &ff);
      if (o->draft) memcpy(o->draft + (size_t)bb * K, d, sizeof(int32_t) * K);
      if (o->q_draft) memcpy(o->q_draft + (size_t)bb * K, qd, sizeof(double) * K);
      if (o->out) memcpy(o->out + (size_t)bb * (K + 1), outb, sizeof(int32_t) * (K + 1));
      if (o->tau) o->tau[bb] = tau;
      if (o->flag_draft) o->flag_draft[bb] = fd;
      if (o->flag_accept) o->flag_accept[bb] = fa;
      if (o->flag_final) o->flag_final[bb] = ff;
      if (tau < 1 || tau > K + 1) bad = 1;
    }
    free(z); free(scratch); free(d); free(qd); free(outb);
  }
  g_threads_used = threads;
  return bad ? -3 : 0;
}

int orc_draft(const orc_params *P, const void *base, const void *U, const void *W,
              const int32_t *last_token, int32_t b_begin, int32_t b_end, orc_outputs *o) {
  if (check_params(P, b_begin, b_end) || !base || !last_token || !o) return -1;
  if (P->r > 0 && (!U || !W)) return -1;
  const int32_t K = P->K, V = P->V;
  for (int32_t b = b_begin; b < b_end; ++b)
    if (last_token[b] < 0 || last_token[b] >= V) return -2;
  int threads = 1;
#pragma omp parallel
  {
#ifdef _OPENMP
#pragma omp single
    threads = omp_get_num_threads();
#endif
    double *z = (double *)malloc(sizeof(double) * (size_t)K * V);
    double *scratch = (double *)malloc(sizeof(double) * (size_t)V);
    int32_t *d = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
    double *qd = (double *)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
    for (int32_t b = b_begin; b < b_end; ++b) {
      const int32_t bb = b - b_begin;
      int32_t fd = K;
      draft_row(P, base, U, W, b, last_token[b], d, qd, z, &fd, scratch);
      if (o->draft) memcpy(o->draft + (size_t)bb * K, d, sizeof(int32_t) * K);
      if (o->q_draft) memcpy(o->q_draft + (size_t)bb * K, qd, sizeof(double) * K);
      if (o->flag_draft) o->flag_draft[bb] = fd;
      if (o->biased) memcpy(o->biased + (size_t)bb * K * V, z, sizeof(double) * (size_t)K * V);
    }
    free(z); free(scratch); free(d); free(qd);
  }
  g_threads_used = threads;
  return 0;
}

int orc_verify(const orc_params *P, const void *target, const void *draft_logits,
               const int32_t *draft, int32_t b_begin, int32_t b_end, orc_outputs *o) {
  if (check_params(P, b_begin, b_end) || !target || !draft_logits || !draft || !o) return -1;
  const int32_t K = P->K, V = P->V;
  for (int32_t b = b_begin; b < b_end; ++b)
    for (int32_t i = 0; i < verify_len_of(P, b); ++i)
      if (draft[(size_t)b * K + i] < 0 || draft[(size_t)b * K + i] >= V) return -2;
  int threads = 1;
#pragma omp parallel
  {
#ifdef _OPENMP
#pragma omp single
    threads = omp_get_num_threads();
#endif
    double *z = (double *)malloc(sizeof(double) * (size_t)K * V);
    int32_t *outb = (int32_t *)malloc(sizeof(int32_t) * (size_t)(K + 1));
#pragma omp for schedule(dynamic, 1)
    for (int32_t b = b_begin; b < b_end; ++b) {
      const int32_t bb = b - b_begin;
      int32_t fa = K, ff = 0, tau = 0;
      for (int32_t i = 0; i < K; ++i)
        for (int32_t v = 0; v < V; ++v)
          z[(size_t)i * V + v] =
              load_elem(draft_logits, P->draft_dtype, ((int64_t)b * K + i) * V + v);
      verify_row(P, target, z, draft + (size_t)b * K, b, outb, &tau, ROWP(o->p_draft, K),
                 ROWP(o->q_draft, K), &fa, &ff);
      if (o->out) memcpy(o->out + (size_t)bb * (K + 1), outb, sizeof(int32_t) * (K + 1));
      if (o->tau) o->tau[bb] = tau;
      if (o->flag_accept) o->flag_accept[bb] = fa;
      if (o->flag_final) o->flag_final[bb] = ff;
      if (o->flag_draft) o->flag_draft[bb] = K;
    }
    free(z); free(outb);
  }
  g_threads_used = threads;
  return 0;
}
