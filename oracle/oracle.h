/*
 * Oracle for the draft-sample-and-verify step of block-parallel speculative
 * decoding (DSpark parallel core + sequential Markov head, verified by
 * speculative rejection sampling).
 *
 * TEST INFRASTRUCTURE ONLY.  This plain, slow, double-precision CPU code is
 * the yardstick the CUDA path is checked against.  Only the test suite, the
 * smoke check and the CPU-baseline leg of the benchmark may load it; the
 * product path never does.  It shares no source with the CUDA library.
 *
 * What it computes (citations name the page and its section):
 *  - aigest.pl "DeepSeek prezentuje DSpark", section "Innowacje w tworzeniu
 *    tokenów": a heavy parallel core gives base logits for every block
 *    position; a light sequential head adds a prefix-dependent bias before
 *    each token is sampled.  The default head is a Markov head that sees only
 *    the immediately preceding token, factorised at low rank (rank 256).
 *    Reading: bias_i = U[prev] . W, prev = last committed token at i = 0,
 *    else the previous draft token.
 *  - same page, section "Jak działa spekulatywne dekodowanie DSpark?":
 *    rejection sampling keeps the longest valid prefix and adds one extra
 *    token, and preserves the target distribution exactly.  Reading: the
 *    textbook rule -- accept d_i with probability min(1, p_i(d_i)/q_i(d_i)),
 *    stop at the first rejection and resample there from the normalised
 *    residual max(p - q, 0); if all K drafts are accepted, draw a bonus token
 *    from target row K.
 *  - telemetr.me DFlash post: mean accepted length counts the bonus token;
 *    aigest.pl: L = (T_draft + T_verify) / tau.  Reading: tau = accepted + 1.
 *
 * Random numbers: counter-based Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
 * "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11), implemented here
 * from the paper's definition.  key = (lo32(seed), hi32(seed)); counter =
 * (position, batch row, lo32(cycle), tag | (bits 32..47 of cycle) << 16);
 * word 0 of the output is mapped to [0,1) as (x >> 8) * 2^-24.
 * Tags: 0 = draft draw, 1 = accept test, 2 = residual / bonus draw.
 *
 * Near-threshold accounting: the GPU decides in fp32, the oracle in fp64.  A
 * decision whose uniform lies within 1e-6 of its threshold (relative to the
 * distribution's total for inverse-CDF draws), a greedy draft arg-max whose
 * runner-up is within 1e-5 * max(1, |z|), or a residual draw whose residual
 * mass is below 1e-4 (fp32 cancellation exceeds the margin there) is flagged;
 * flagged decisions are counted, not compared.
 *
 * Parity pins: every function here is checked by the CPU test suite against
 * brute-force enumeration, closed forms, library routines and hand-worked
 * examples.  Philox has no published known-answer vector in this container;
 * it is pinned by uniformity tests, by the GPU library's own independent
 * Philox4_32_10 (curand) and by bit-exact agreement with the CUDA kernels.
 */
#ifndef SPEC_ORACLE_H
#define SPEC_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };
enum { ORC_TAG_DRAFT = 0, ORC_TAG_ACCEPT = 1, ORC_TAG_RESAMPLE = 2 };

typedef struct {
  int32_t B, K, V, r;
  int32_t dtype;        /* ORC_F32 or ORC_BF16: base, target, U, W */
  int32_t draft_dtype;  /* verify-only: dtype of the given draft logits */
  double temperature;   /* > 0 unless greedy */
  int32_t greedy;
  uint64_t seed;
  uint64_t cycle;
  /* [B] per-row verify length K_b in 1..K, or NULL (every row K).  aigest.pl
   * "Optymalizacja weryfikacji i wydajności": a scheduler fixes the verify
   * length of each request.  Reading: row b drafts and verifies positions
   * 0..K_b-1 only and takes its bonus from target row K_b (the rule above
   * with K_b in place of K); draft[b, i] = -1 and q_draft NaN for i >= K_b. */
  const int32_t *verify_len;
  /* [r, r] (dtype) recurrent weights of the RNN sequential head, or NULL for
   * the Markov head.  aigest.pl "DeepSeek prezentuje DSpark", section
   * "Innowacje w tworzeniu tokenów": an optional RNN head tracks the whole
   * block prefix instead of the previous token only.  The pages give no
   * formula.  Reading (an Elman recurrence in the Markov head's factors):
   *   s_{-1} = 0,  s_i[j] = clamp(U[prev_i, j] + sum_k Wh[j, k] s_{i-1}[k], -1, 1),
   *   bias_i = s_i . W,
   * prev_i as for the Markov head.  The state is the bias's low-rank operand,
   * so it is kept in the head's dtype: in fp32 the sum runs as fmaf in
   * ascending k from 0, the U term is added after it, the clamp is exact, and
   * for bf16 the result is rounded to bf16 (nearest, ties to even).  Every
   * step of this is exactly reproducible, so both sides hold the same state
   * bit for bit. */
  const void *Wh;
} orc_params;

/* Per-row outputs for rows [b_begin, b_end); arrays are indexed by b - b_begin.
 * Any pointer may be NULL. */
typedef struct {
  int32_t *draft;       /* [n, K]   draft tokens d_i                              */
  int32_t *out;         /* [n, K+1] emitted tokens, -1 after tau                  */
  int32_t *tau;         /* [n]      emitted count, 1..K+1                         */
  double *p_draft;      /* [n, K]   p_i(d_i) where tested, NaN elsewhere / greedy */
  double *q_draft;      /* [n, K]   q_i(d_i), NaN in greedy mode                  */
  int32_t *flag_draft;  /* [n] first position whose draft draw is near-threshold, else K */
  int32_t *flag_accept; /* [n] first position whose accept test is near-threshold, else K */
  int32_t *flag_final;  /* [n] 1 if the correction / bonus draw is near-threshold */
  double *biased;       /* [n, K, V] z = base + U[prev].W (draft-only call)     */
} orc_outputs;

/* Philox4x32-10 block function: out = Philox(ctr, key). */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
/* (x >> 8) * 2^-24 */
double orc_u01(uint32_t x);
/* The uniform drawn for (seed, cycle, batch row, position, tag). */
double orc_uniform(uint64_t seed, uint64_t cycle, uint32_t b, uint32_t pos, uint32_t tag);

/* First index v with inclusive prefix C[v] > u * sum(w); if none, the last index
 * with w > 0; -1 if all weights are zero.  *near is set when u*sum lies within
 * 1e-6*sum of an edge of the chosen index's CDF interval. */
int32_t orc_icdf(const double *w, int32_t n, double u, int32_t *near);

/* Row statistics of x/T over n entries: m = max, Z = sum exp(x/T - m). */
void orc_row_stats(const double *x, int32_t n, double T, double *m, double *Z);

/* Verify one block given probabilities and explicit uniforms (the algorithm
 * with its random draws passed in).  p: [K+1][V] target probabilities,
 * q: [K][V] draft probabilities, d: [K] draft tokens, u_acc: [K] accept
 * uniforms, u_res: [K+1] residual/bonus uniforms (index = stop row).
 * Writes out[K+1], *tau, p_d[K] (NaN where untested); returns the stop row.
 * flag_accept / flag_final as in orc_outputs (may be NULL). */
int32_t orc_verify_probs(int32_t K, int32_t V, const double *p, const double *q,
                         const int32_t *d, const double *u_acc, const double *u_res,
                         int32_t *out, int32_t *tau, double *p_d,
                         int32_t *flag_accept, int32_t *flag_final);

/* The full cycle: sequential Markov-biased drafting, then verification. */
int orc_cycle(const orc_params *P, const void *base, const void *target, const void *U,
              const void *W, const int32_t *last_token, int32_t b_begin, int32_t b_end,
              orc_outputs *o);

/* Drafting only (fills draft, q_draft, flag_draft, biased). */
int orc_draft(const orc_params *P, const void *base, const void *U, const void *W,
              const int32_t *last_token, int32_t b_begin, int32_t b_end, orc_outputs *o);

/* Verification only, given final draft logits [B,K,V] (dtype draft_dtype) and
 * draft tokens [B,K] (fills out, tau, p_draft, q_draft, flag_accept, flag_final). */
int orc_verify(const orc_params *P, const void *target, const void *draft_logits,
               const int32_t *draft, int32_t b_begin, int32_t b_end, orc_outputs *o);

/* One biased draft row: z = base[b,i,:] + U[prev,:] . W (double). */
int orc_biased_row(const orc_params *P, const void *base, const void *U, const void *W,
                   int32_t b, int32_t i, int32_t prev, double *z);

/* Threads the last orc_cycle / orc_draft / orc_verify call used. */
int orc_threads_used(void);

#ifdef __cplusplus
}
#endif
#endif
