/*
 * specdec -- the draft-sample-and-verify step of block-parallel speculative
 * decoding on NVIDIA B200 (sm_100a), as a C-ABI library (libspecdec.so).
 *
 * The step (pages: aigest.pl "DeepSeek prezentuje DSpark"; telemetr.me DFlash
 * post; mkdocs.reaper.mx DeepSeek-V4.1-Flash "06-extensions", DSpark table):
 *   a parallel drafter gives base logits for K block positions in one pass;
 *   a sequential Markov head adds bias_i = U[prev] . W (rank r) before each
 *   draft token is sampled, prev being the last committed token for i = 0 and
 *   the previous draft token after that ("Innowacje w tworzeniu tokenów");
 *   the target's K+1 logit rows then verify the block by rejection sampling:
 *   the longest accepted prefix plus one extra token, with the target
 *   distribution preserved exactly ("Jak działa spekulatywne dekodowanie").
 *   Accept d_i iff u < min(1, p_i(d_i)/q_i(d_i)); at the first rejection emit
 *   a draw from max(p_i - q_i, 0) normalised (p_i if that is all zero); if all
 *   K pass, emit a bonus draw from target row K.  Greedy mode drafts arg-max
 *   tokens and accepts while arg-max(target_i) equals d_i.  tau = accepted + 1
 *   is the quantity in L = (T_draft + T_verify) / tau.
 *   p = softmax(target / T), q = softmax((base + bias) / T).
 *
 * Random numbers: Philox4x32-10 (Salmon et al., SC'11), key = seed,
 * counter = (position, row_offset + batch row, lo32(cycle), tag | bits 32..47 of cycle << 16),
 * word 0 mapped to [0,1) as (x >> 8) * 2^-24; tag 0 = draft draw, 1 = accept
 * test, 2 = residual or bonus draw.  Sampling is by inverse CDF in ascending
 * token order: the first token whose inclusive prefix mass exceeds u * total.
 * Ties in arg-max go to the lowest index.
 *
 * Layouts (row-major, V contiguous, caller-owned device memory):
 *   base        [B, K, V]    dtype        draft base logits
 *   target      [B, K+1, V]  dtype        target logits, row K = bonus row
 *   U           [V, r]       dtype        Markov factor, row = previous token
 *   W           [r, V]       dtype        Markov factor
 *   last_token  [B]          int32        last committed token
 *   draft       [B, K]       int32        draft tokens d_i
 *   out         [B, K+1]     int32        emitted tokens; entries >= tau are -1
 *   tau         [B]          int32        1 .. K+1
 *   p_draft     [B, K]       float        p_i(d_i) where the accept test ran, NaN after
 *   q_draft     [B, K]       float        q_i(d_i)
 *   biased_out  [B, K, V]    float        z = base + bias (optional)
 * dtype is SPEC_BF16 (bf16 logits and factors; bias products on tcgen05
 * tensor cores, fp32 accumulate) or SPEC_F32 (fp32 throughout).  All
 * arithmetic after loading is fp32.  In greedy mode p_draft / q_draft are
 * filled with NaN.
 *
 * Calls are asynchronous on `stream`.  Errors found on the host (bad sizes,
 * NULL pointers, a workspace too small) are returned before anything is
 * launched.  Errors found on the device (a token id out of range, a wait that
 * ran past spin_limit polls) are recorded in the workspace and returned by
 * spec_sync_status().  Every device-side wait is bounded; a kernel that gives
 * up records SPEC_ERR_TIMEOUT and returns, leaving the outputs undefined.
 * One workspace serves one stream at a time; calls that share a workspace
 * must be ordered on one stream.
 */
#ifndef SPECDEC_H
#define SPECDEC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *spec_stream_t; /* same type as cudaStream_t */

typedef enum {
  SPEC_OK = 0,
  SPEC_ERR_INVALID_ARG = -1,   /* NULL pointer, size out of range, bad temperature */
  SPEC_ERR_UNSUPPORTED = -2,   /* shape the kernels do not handle (message says which) */
  SPEC_ERR_CUDA = -3,          /* a CUDA runtime call failed */
  SPEC_ERR_TIMEOUT = -4,       /* a device-side wait exceeded spin_limit polls */
  SPEC_ERR_WORKSPACE = -5,     /* workspace NULL, too small or misaligned */
  SPEC_ERR_TOKEN_RANGE = -6    /* a token id (last_token / draft) outside [0, V) */
} spec_status;

typedef enum { SPEC_F32 = 0, SPEC_BF16 = 1 } spec_dtype;

/* Flags */
#define SPEC_FLAG_FMA_BIAS 1u  /* compute the Markov bias with fp32 FMAs instead of tensor cores */
#define SPEC_FLAG_TRACE 2u     /* spec_cycle / spec_markov_bias_sample: record a device timeline.
                                  CTA 0 writes %globaltimer (ns) into the workspace at byte offset
                                  256 as uint64 [K+2][32]: row i < K = draft step i (slots: 0 start,
                                  1 rows gathered, 2 epilogue done, 3 partials published, 4 target
                                  rows streamed, 5 barrier passed, 6 partials combined, 7 owner
                                  draws done, 8 tokens known; 9..31 finer diagnostics: tensor-core
                                  issue, wait totals, per-chunk times), row K = final step, row
                                  K+1 = prologue.  Only the first batch group is recorded. */

typedef struct {
  int32_t B;             /* batch rows, >= 1 */
  int32_t K;             /* draft block length, 1 .. 1024 */
  int32_t V;             /* vocabulary, >= 1; bf16 needs V % 8 == 0, f32 V % 4 == 0 */
  int32_t r;             /* Markov rank: 0 (no head) or 1..256; bf16 tensor-core path needs r % 64 == 0 */
  int32_t dtype;         /* spec_dtype of base, target, U, W */
  int32_t draft_dtype;   /* spec_verify_block: spec_dtype of draft_logits */
  float temperature;     /* > 0 unless greedy */
  int32_t greedy;        /* 0 = stochastic, 1 = greedy */
  uint64_t seed;         /* Philox key */
  uint64_t cycle;        /* Philox counter words 2..3 (advance it every cycle) */
  uint64_t spin_limit;   /* polls before a device wait gives up; 0 = default (about 2 s) */
  uint32_t flags;        /* SPEC_FLAG_* */
  uint32_t row_offset;   /* global index of batch row 0: row b draws from Philox counter word
                            row_offset + b, so a batch split into shards (calls or GPUs) with
                            their starting rows draws exactly what one call over it draws;
                            row_offset + B must not exceed 2^31 */
} spec_params;

/* Bytes of device workspace the calls need for these parameters on the
 * current device (0 if the parameters are invalid).  Alignment: 256 bytes. */
size_t spec_workspace_size(const spec_params *p);

/* Zero a workspace (asynchronously on `stream`).  Required once before first
 * use, and again after any call whose spec_sync_status was not SPEC_OK. */
spec_status spec_workspace_init(void *workspace, size_t bytes, spec_stream_t stream);

/* Markov-head bias for one draft step (section "Innowacje w tworzeniu
 * tokenów"): bias[b, v] = sum_k U[prev[b], k] * W[k, v], fp32 accumulate.
 * prev [B] int32 (device), bias [B, V] float (device). */
spec_status spec_markov_bias(const spec_params *p, const void *U, const void *W,
                             const int32_t *prev, float *bias, void *workspace,
                             spec_stream_t stream);

/* Sequential drafting: for i = 0..K-1, z = base_i + U[prev] . W, d_i drawn
 * from softmax(z / T) (arg-max in greedy mode), prev = d_i.  One persistent
 * launch carries all K steps.  q_draft and biased_out may be NULL. */
spec_status spec_markov_bias_sample(const spec_params *p, const void *base, const void *U,
                                    const void *W, const int32_t *last_token, int32_t *draft,
                                    float *q_draft, float *biased_out, void *workspace,
                                    spec_stream_t stream);

/* Verification of given drafts against the target rows (section "Jak działa
 * spekulatywne dekodowanie"): draft_logits [B, K, V] are the final (biased)
 * draft logits in draft_dtype, draft [B, K] the tokens drawn from them.
 * One persistent launch with early exit (B <= 4096 and V up to 2048 tokens
 * per SM): positions are decided a few at a time, and the draft and target
 * rows of a position past a row's first rejection are never read.  So
 * q_draft[b, i] is written for the positions whose accept test ran (NaN
 * after), like p_draft.  Larger shapes take a multi-launch path that reads
 * every row and writes q_draft for all K positions.  p_draft and q_draft may
 * be NULL. */
spec_status spec_verify_block(const spec_params *p, const void *target, const void *draft_logits,
                              const int32_t *draft, int32_t *out, int32_t *tau, float *p_draft,
                              float *q_draft, void *workspace, spec_stream_t stream);

/* spec_verify_block with a verify length per request (the scheduler's K_b,
 * section "Optymalizacja weryfikacji i wydajności"): verify_len [B] int32
 * (device), K_b in 1..K.  Row b verifies positions 0..K_b-1 and draws its
 * bonus from target row K_b, so tau_b <= K_b + 1; rows past K_b are never
 * read.  A K_b outside 1..K is clamped and reported as SPEC_ERR_INVALID_ARG by
 * spec_sync_status.  Shapes the one-launch path does not take return
 * SPEC_ERR_UNSUPPORTED. */
spec_status spec_verify_block_kb(const spec_params *p, const void *target,
                                 const void *draft_logits, const int32_t *draft,
                                 const int32_t *verify_len, int32_t *out, int32_t *tau,
                                 float *p_draft, float *q_draft, void *workspace,
                                 spec_stream_t stream);

/* One whole cycle: drafting and verification fused in one persistent launch
 * (target rows are read only up to each row's first rejection).  draft,
 * p_draft and q_draft may be NULL. */
spec_status spec_cycle(const spec_params *p, const void *base, const void *target, const void *U,
                       const void *W, const int32_t *last_token, int32_t *draft, int32_t *out,
                       int32_t *tau, float *p_draft, float *q_draft, void *workspace,
                       spec_stream_t stream);

/* One cycle with a verify length per request (aigest.pl "DeepSeek prezentuje
 * DSpark", section "Optymalizacja weryfikacji i wydajności": a scheduler fixes
 * how many draft tokens of each request are verified, and its early stop keeps
 * the method lossless).  verify_len [B] int32 (device): K_b in 1..K.  Row b
 * drafts and verifies positions 0..K_b-1 and draws its bonus from target row
 * K_b, so tau_b <= K_b + 1 and the draws are the full block's first K_b draws
 * (the same random counters); draft[b, i] = -1 and q_draft[b, i] = NaN for
 * i >= K_b, and target rows past K_b are never read.  A K_b outside 1..K is
 * clamped and reported as SPEC_ERR_INVALID_ARG by spec_sync_status.  Tensor-core
 * path only (bf16, rank a multiple of 64 up to 256); other shapes return
 * SPEC_ERR_UNSUPPORTED.  spec_cycle is this call with every K_b = K. */
spec_status spec_cycle_kb(const spec_params *p, const void *base, const void *target,
                          const void *U, const void *W, const int32_t *last_token,
                          const int32_t *verify_len, int32_t *draft, int32_t *out, int32_t *tau,
                          float *p_draft, float *q_draft, void *workspace, spec_stream_t stream);

/* A decode loop: n_cycles cycles in one persistent launch (aigest.pl "DeepSeek
 * prezentuje DSpark", section "Jak działa spekulatywne dekodowanie DSpark?":
 * decoding repeats draft-and-verify cycles, each costing T_draft + T_verify
 * for its tau tokens).  The token a row emits last in cycle c (its correction
 * or its bonus token) is the committed token cycle c + 1 starts from, and
 * cycle c draws with Philox cycle counter p->cycle + c; cycle c is otherwise
 * spec_cycle_kb on slice c of the inputs.  Its verify lengths come from
 * verify_len, or from confidence scores (section "Optymalizacja weryfikacji i
 * wydajności": a score per draft position estimating the chance that its
 * token survives verification given accepted predecessors): K_b is the number
 * of leading positions whose prefix survival, the fp32 product of the scores
 * of positions 0..i taken in position order, is >= conf_threshold, and at
 * least 1 (a NaN score ends the prefix); or K with neither.
 *   base        [C, B, K, V]    dtype   (C = n_cycles; slice c feeds cycle c)
 *   target      [C, B, K+1, V]  dtype
 *   conf        [C, B, K]       float   or NULL
 *   verify_len  [C, B]          int32   or NULL (not both with conf)
 *   U, W, last_token            as for spec_cycle (last_token: cycle 0's)
 *   draft, p_draft, q_draft [C, B, K]; out [C, B, K+1]; tau [C, B]
 *   next_token  [B]             int32   the last token each row emitted in the
 *               last cycle (the next call's last_token); required when
 *               n_cycles > 1 (it carries the tokens between cycles), and it
 *               may be the same buffer as last_token.
 * n_cycles is 1..65536.  Tensor-core path only (bf16, rank a multiple of 64 up
 * to 256); other shapes return SPEC_ERR_UNSUPPORTED.  Device-side errors are
 * reported as for spec_cycle_kb. */
spec_status spec_decode_loop(const spec_params *p, int32_t n_cycles, const void *base,
                             const void *target, const float *conf, float conf_threshold,
                             const int32_t *verify_len, const void *U, const void *W,
                             const int32_t *last_token, int32_t *draft, int32_t *out, int32_t *tau,
                             float *p_draft, float *q_draft, int32_t *next_token, void *workspace,
                             spec_stream_t stream);

/* One cycle with the RNN sequential head in place of the Markov head
 * (aigest.pl "DeepSeek prezentuje DSpark", section "Innowacje w tworzeniu
 * tokenów": an optional RNN head tracks the whole block prefix).  The pages
 * give no formula; the reading implemented is an Elman recurrence in the
 * Markov head's factors:
 *   s_{-1} = 0,  s_i = bf16(clamp(U[prev_i] + Wh s_{i-1}, -1, 1)),  bias_i = s_i . W,
 * prev_i as for the Markov head.  (Wh s_{i-1})[j] is the fp32 fmaf chain over
 * k = 0..r-1 of s_{i-1}[k] * Wh[j, k] starting from 0, U[prev_i, j] is added
 * after it, and the result is clamped and rounded to bf16 (nearest, ties to
 * even), so the state is the same bit for bit on any implementation that
 * follows these steps.  Wh [r, r] bf16 (device), row j holding the weights of
 * output j.  The recurrence of step i + 1 is computed during step i across
 * the CTAs, so only its state update stays on the sequential path.  Otherwise
 * as spec_cycle.  Tensor-core path only (bf16, rank a multiple of 64 up to
 * 256); other shapes return SPEC_ERR_UNSUPPORTED. */
spec_status spec_cycle_rnn(const spec_params *p, const void *base, const void *target,
                           const void *U, const void *W, const void *Wh,
                           const int32_t *last_token, int32_t *draft, int32_t *out, int32_t *tau,
                           float *p_draft, float *q_draft, void *workspace, spec_stream_t stream);

/* spec_cycle without a workspace argument, for callers that cannot allocate
 * device memory when they run a cycle (code whose allocations all belong to a
 * framework pool, a host thread that must not call cudaMalloc because it
 * synchronises the device, a plugin that only receives input and output
 * buffers).  The pages have no counterpart: this is a deployment convenience.
 * Scratch lives in a fixed 8 MiB device array inside the library, present on
 * every GPU that loads it until the process exits; nothing is allocated per
 * call.  Shapes whose spec_workspace_size exceeds 8 MiB are rejected with
 * SPEC_ERR_WORKSPACE (and a message on stderr).  The first call on a device
 * looks up the array's device address (again after the device's context was
 * replaced, e.g. by cudaDeviceReset); make that first call before any stream
 * capture.  All calls share the array: calls that overlap on the GPU race, so
 * order them on one stream.  status_out (device int32, may be NULL) receives
 * the device-side status of the call, stream-ordered after it. */
spec_status spec_cycle_noalloc(const spec_params *p, const void *base, const void *target,
                               const void *U, const void *W, const int32_t *last_token,
                               int32_t *draft, int32_t *out, int32_t *tau, float *p_draft,
                               float *q_draft, int32_t *status_out, spec_stream_t stream);

/* Verify-length scheduler (host logic; no device work, no stream, callable
 * without a GPU).  mkdocs.reaper.mx DeepSeek-V4.1-Flash "06-extensions", DSpark
 * table: the scheduler chooses each request's verify length from the prefix
 * survival probabilities of the confidence head and the engine's throughput
 * curve measured beforehand, to maximise expected throughput under the current
 * load; aigest.pl "DeepSeek prezentuje DSpark", "Optymalizacja weryfikacji i
 * wydajności": that curve is SPS(B), profiled once at start-up.  Reading: with
 * S_{b,i} = prod_{j<=i} clamp(conf[b][j], 0, 1) (a NaN score counts as 0),
 * choose k_b in 1..K maximising
 *   E * SPS(M),  E = sum_b (1 + sum_{i<k_b} S_{b,i}),  M = sum_b (k_b + 1)
 * (expected tokens per step times steps per second for a target pass over M
 * rows); among equal maxima the smallest total length, among allocations of
 * that total the one taking the larger S first, ties to the lower row b.
 *   conf        [B, K] float, host    confidence scores per draft position
 *   sps         [n_sps] double, host  steps per second of a target pass over m
 *                                     rows, m = 0 .. n_sps-1; 0 past the table
 *   verify_len  [B] int32, host       output k_b, ready for spec_cycle_kb
 *   expected    [2] double, host      output (E, E * SPS(M)); may be NULL
 * Errors: SPEC_ERR_INVALID_ARG for a NULL pointer, B or K < 1, B*K > 2^26,
 * n_sps < 1, or an SPS entry that is negative, NaN or infinite (nothing is
 * written then).  Cost O(BK log BK) on the calling thread. */
spec_status spec_schedule_verify_len(const float *conf, int32_t B, int32_t K,
                                     const double *sps, int32_t n_sps, int32_t *verify_len,
                                     double *expected);

/* Keep [ptr, ptr + bytes) resident in L2 for kernels later launched on
 * `stream` (a persisting access-policy window on the stream; the persisting
 * L2 carve-out of the calling process's context is raised to fit, up to the
 * device maximum).  Meant for the Markov factor W, which every draft step
 * re-reads.  bytes = 0 removes the window and releases persisting lines.  The
 * carve-out belongs to this process's context and ends with it. */
spec_status spec_l2_persist(const void *ptr, size_t bytes, spec_stream_t stream);

/* Synchronise `stream` and return the device-side status recorded in the
 * workspace by the calls issued on it (SPEC_OK if none failed). */
spec_status spec_sync_status(const void *workspace, spec_stream_t stream);

/* Human-readable name of a status code. */
const char *spec_status_string(spec_status s);

/* Number of kernel launches the last call on this thread issued. */
int32_t spec_last_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif
