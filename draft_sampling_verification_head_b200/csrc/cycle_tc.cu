// Fused persistent draft-sample-and-verify kernel, tensor-core path (bf16
// logits and Markov factors, rank a multiple of 64 up to 256).
//
// Method (aigest.pl "DeepSeek prezentuje DSpark"; mkdocs.reaper.mx
// DeepSeek-V4.1-Flash "06-extensions", DSpark table):
//   "Innowacje w tworzeniu tokenów": the parallel core's base logits plus a
//   prefix-dependent Markov bias U[prev] . W added before each of the K draft
//   tokens is sampled -- K sequential steps, step i needing d_{i-1};
//   "Jak działa spekulatywne dekodowanie DSpark?": the longest accepted prefix
//   plus one extra token, target distribution preserved exactly.
//
// Design (one launch, one CTA per SM, cooperative so all CTAs are resident):
//  * The vocabulary is cut into 128-token chunks; CTA c owns nc consecutive
//    chunks for the whole launch.  Batch rows are processed in groups of N
//    (16/32/64/128), the tcgen05 N dimension.  Warps: 8 compute warps, a W TMA
//    producer, the MMA issuer and two target warps.
//  * The bias of a step is, per chunk, D[v, n] = W^T[v, :] . U[prev_n]^T, one
//    tcgen05.mma kind::f16 chain (M = 128 tokens, N rows, K = r).  W^T of the
//    CTA's first NT chunks is copied into tensor memory once per launch and
//    used as the A operand there for every step; the other chunks' W^T
//    streams from L2 through a TMA ring (128-byte swizzle).  The gathered U
//    rows are the swizzled K-major B operand.  Accumulators are double
//    buffered: a chunk's MMA overlaps the previous chunk's epilogue.
//  * Epilogue: the accumulator tile (lane = token, column = batch row) is
//    transposed through shared memory so that each lane holds consecutive
//    tokens of one row; the lane adds that row's base logits (read from L2,
//    where they were prefetched one step ahead) and takes exact statistics
//    (max, sum exp2) of each 32-token bucket.  Nothing needs a second round:
//    every statistic is exact.
//  * Target statistics (max, sum or arg-max of each target row over the
//    CTA's slice), for rows still verifying and, at a row's last verified
//    position, its bonus row: the first positions by the compute warps at the
//    start of each job, the rest by the two target warps, which copy row
//    slices into shared-memory rings and run up to two positions ahead of
//    the draft chain.
//  * Row n's reducer (CTA n mod G) combines the per-CTA partials in ascending
//    token order, finds the CTA and then the bucket holding the inverse-CDF
//    target, forms that bucket's 32 logits from the bf16 inputs with the whole
//    CTA, scans them, runs the accept test and publishes a 64-byte record.
//    Greedy steps take the arg-max instead.
//  * Verification runs on the fly (a row's target rows are not read past its
//    first rejection).  A last step recomputes the bias at each row's stop
//    position and draws the residual max(p - q, 0), or the bonus from target
//    row K, the same way.
//  * Every wait is bounded (spin limit); a CTA that gives up records
//    SPEC_ERR_TIMEOUT in the workspace, the others notice and all exit.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace specdec {

namespace {

constexpr int kCH = 128;             // tokens per chunk (UMMA M)
constexpr int kComputeThreads = 256;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kTargetWarp0 = 10;     // warps 10 and 11: target row statistics
constexpr int kThreads = 384;
constexpr int kTSMax = 16;           // row-slice slots per target warp, at most
template <int N>
constexpr int kNSof = N >= 128 ? 4 : 6;  // W ring stages (fewer beside a 128-row operand)
constexpr int kKS = 4;               // MMA K-steps (16 rank rows each) per stage
constexpr int kWChunk = kCH * 16 * 2;         // 4 KB: one K-step of one chunk
constexpr int kWStage = kKS * kWChunk;        // 16 KB: 64 rank rows of one chunk
constexpr int kMaxNT = 3;            // chunks whose W^T stays in tensor memory
constexpr int kMaxG = 160;           // CTAs a launch may use; partial-row stride
constexpr unsigned FULL = 0xffffffffu;
// Low 16 bits of a tensor-memory cell of the A operand hold the even rank index.
constexpr bool kPackEvenLow = true;

struct RecT;

struct ArgsTC {
  CUtensorMap tmW;
  const __nv_bfloat16* base;
  const __nv_bfloat16* target;
  const __nv_bfloat16* U;
  const __nv_bfloat16* W;
  const int32_t* last_token;
  const int32_t* vlen;   // [C][B] per-row verify length K_b (1..K), or null
  const float* conf;     // [C][B][K] confidence scores (used without vlen), or null
  int32_t* next_token;   // [B] each row's last emitted token (carried between cycles), or null
  const __nv_bfloat16* Wh;  // [r][r] RNN head recurrence (row j: weights of s_{i-1}), or null (Markov)
  float* P;              // [2][N][r] RNN head: Wh s_{i-1} of the group's rows, by step parity
  __nv_bfloat16* shist;  // [K][N][r] RNN head: the state of every step (final-step bias)
  int32_t* draft;
  int32_t* out;
  int32_t* tau;
  float* p_draft;
  float* q_draft;
  WsHeader* hdr;
  float4* dpart;     // [2][K+1][N][kMaxG]: draft (max, sum, max, 0) or (max, idx, max, 0); final (R, P)
  float2* tpart;     // [2][K+1][N][kMaxG]: target (max, sum) or (max, idx)
  int32_t* tokens;   // [2][K][N]
  RecT* rec;         // [2][K+1][N] row records (slot K: the final draw)
  uint64_t* rtag;    // [2][K+1][N] record tags: (tag << 32) | accept << 31 | token
  float2* gbk;       // [G][nbk][N] bucket statistics of every CTA (current step)
  uint64_t* trace;   // [K+2][kTracePhases] device timeline of CTA 0, or null
  int B, K, V, r, G, nc, nchunks, greedy, ngroups, NT;
  float k;           // log2(e) / T (1 in greedy mode)
  float conf_thr;    // prefix survival a verified position needs (with conf)
  int ncyc;          // cycles C run by this launch, one after another
  uint64_t seed, cycle, spin;
  uint32_t row0;     // global index of batch row 0 (Philox counter word 1)
  int nbk;           // buckets per CTA (4 per chunk)
  int nts;           // row-slice slots per target warp (what shared memory holds)
  int npro;          // leading positions whose target statistics the compute warps
                     // take at the start of each job (the rest: the target warps)
};

// One record per batch row and step, written by the row's reducer.
struct alignas(16) RecT {
  float M, S;        // draft distribution of the step: max of z, sum exp2((z - M) k)
  float Mt, St;      // target row i statistics
  float MtK, StK;    // target row K statistics (last draft step, rows still verifying)
  float trem;        // inverse-CDF target inside the owner CTA's slice (inf: last mass)
  int32_t owner;     // CTA that owns the draw
  int32_t token;     // draft token of the step (drawn, or the arg-max); final: emitted token
  int32_t acc;       // accept outcome
  int32_t flags;     // bit 1: the final draw uses p (empty residual)
  int32_t tam;       // greedy: target arg-max of row i
  int32_t tamK;      // greedy: target arg-max of row K
  int32_t pad[3];
};
static_assert(sizeof(RecT) == 64, "records are four 16-byte words");

template <int N>
struct CtlT {
  uint64_t wfull[kNSof<N>], wempty[kNSof<N>], dfull[2], dfree[2];
  uint64_t bready, tready, mmadone;
  uint64_t tfull[2][kTSMax];  // target row slices landed (one ring per target warp)
  uint32_t tgo_cnt;        // target jobs released to the target warps (all jobs so far)
  uint32_t tdone_cnt[2];   // target jobs finished by each target warp (all jobs so far)
  uint32_t tmem_slot;
  int32_t abort_local;
  int32_t prev[N];
  int32_t alive[N];
  int32_t stoprow[N];
  int32_t tok[N];
  int32_t acc[N];        // accept outcome of the step, from the record tags
  int32_t kb[N];         // verify length of each row of the group
  float zM[N], zS[N];    // draft statistics of the stop row
  float fMt[N], fSt[N];  // target statistics of the final row (stop row or row K)
  alignas(16) float4 fcst[N];  // final step: target max, 1 / target sum, draft max, 1 / draft sum
  float qa[4][N], qb[4][N];    // per-quadrant partials: draft / final residual
  RecT rrec[N];          // records of the rows this CTA reduces, before publication
  float zpart[8][32];    // per-warp partial Markov biases of a draw's 32 tokens
  int32_t dbk;           // the draw's bucket (entry of the row's bucket array)
  float dtin;            // inverse-CDF target inside that bucket
};

SPEC_DEV void store_rec(RecT* dst, const RecT& r) {
  const float4* s4 = reinterpret_cast<const float4*>(&r);
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) d4[j] = s4[j];
}
SPEC_DEV RecT load_rec(const RecT* src) {
  RecT r;
  float4* d4 = reinterpret_cast<float4*>(&r);
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int j = 0; j < 4; ++j) d4[j] = __ldcg(s4 + j);
  return r;
}

SPEC_DEV void named_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
SPEC_DEV void quartet_sync(int q) { asm volatile("bar.sync %0, 128;" ::"r"(2 + q) : "memory"); }

// D[tmem] (+)= A[tmem] * B[smem], kind::f16 (bf16 inputs, fp32 accumulate)
SPEC_DEV void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

SPEC_DEV void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
      "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]),
      "r"(r[30]), "r"(r[31])
      : "memory");
}

// tcgen05.ld of NCOL consecutive columns (NCOL a multiple of 8), waited.
template <int NCOL>
SPEC_DEV void tmem_ld_cols(uint32_t taddr, float (&v)[NCOL]) {
  if constexpr (NCOL % 16 == 0) {
#pragma unroll
    for (int c = 0; c < NCOL / 16; ++c) tmem_ld16(taddr + c * 16, v + c * 16);
  } else {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr));
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
  }
  tmem_ld_wait();
}

// Transpose of a warp's tile through its shared buffer: on entry lane t holds
// columns 0..NCOL-1 of token t; on exit lane l holds tokens
// (l % L) * NCOL .. + NCOL - 1 of column l / L (L = 32 / NCOL).  Rows of the
// buffer are 16-byte-chunk swizzled and, for NCOL < 32, permuted so that both
// the stores and the loads are free of bank conflicts.
template <int NCOL>
SPEC_DEV int tr_row(int t) {
  return t ^ ((t / NCOL) & (32 / NCOL - 1));
}
template <int NCOL>
SPEC_DEV void transpose_in(float* buf, const float (&d)[NCOL], int lane) {
  constexpr int CPR = NCOL / 4;  // 16-byte chunks per row
  const int p = tr_row<NCOL>(lane);
  float4* row = reinterpret_cast<float4*>(buf + p * NCOL);
#pragma unroll
  for (int c = 0; c < CPR; ++c)
    row[c ^ (p & (CPR - 1))] = make_float4(d[4 * c], d[4 * c + 1], d[4 * c + 2], d[4 * c + 3]);
}
template <int NCOL>
SPEC_DEV void transpose_out(const float* buf, float (&z)[NCOL], int lane) {
  constexpr int CPR = NCOL / 4;
  constexpr int L = 32 / NCOL;
  const int col = lane / L, tg = lane % L;
#pragma unroll
  for (int e = 0; e < NCOL; ++e) {
    const int p = tr_row<NCOL>(tg * NCOL + e);
    z[e] = buf[p * NCOL + (((col >> 2) ^ (p & (CPR - 1))) << 2) + (col & 3)];
  }
}

// Eight bf16 values of a 16-byte word, in ascending address order.
SPEC_DEV void bf16x8(const uint4& w, float* x) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(u[j] << 16);
    x[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
  }
}

// Counters in shared memory shared by the warps of one CTA (release/acquire
// at CTA scope: what the writer stored before is visible to the reader after).
SPEC_DEV uint32_t ld_acquire_cta_smem(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
SPEC_DEV void st_release_cta_smem(uint32_t* p, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
SPEC_DEV void add_release_cta_smem(uint32_t* p, uint32_t v) {
  asm volatile("red.release.cta.shared::cta.add.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// Pairs of fp32 values in one 64-bit register for the packed fp32 pipe
// (sm_100: add / fma .f32x2, each lane rounded exactly like the scalar op).
SPEC_DEV uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
SPEC_DEV void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
SPEC_DEV uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
SPEC_DEV uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Target statistics of a row slice, the same arithmetic wherever they are
// taken.  One 16-byte piece (8 logits of tokens tok0 .. tok0 + 7) into a lane's
// running arg-max (greedy) or (max, sum of exp2((x - max) k)), the sum
// rescaled once per piece.
template <bool kGreedy>
SPEC_DEV void piece_stats(const uint4& w, int tok0, float k, float& m, float& s, int32_t& mi) {
  float x[8];
  bf16x8(w, x);
  if constexpr (kGreedy) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (x[e] > m) {
        m = x[e];
        mi = tok0 + e;
      }
  } else {
    // the piece's max in packed bf16 (exact), then one conversion
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
    const __nv_bfloat162 mx = __hmax2(__hmax2(h2[0], h2[1]), __hmax2(h2[2], h2[3]));
    const float mn = fmaxf(m, fmaxf(__low2float(mx), __high2float(mx)));
    // without branches: while every value so far is -inf, mk = 0 and every
    // exp2 below is exp2(-inf) = 0 (s stays 0)
    const float mk = mn > -INFINITY ? mn * k : 0.f;
    const uint64_t kk = f2pack(k, k), nmk = f2pack(-mk, -mk);
    float y[8];
#pragma unroll
    for (int e = 0; e < 8; e += 2) f2unpack(f2fma(f2pack(x[e], x[e + 1]), kk, nmk), y[e], y[e + 1]);
    float sv[4];
#pragma unroll
    for (int e = 0; e < 4; e += 2)
      f2unpack(f2add(f2pack(fexp2(y[e]), fexp2(y[e + 1])), f2pack(fexp2(y[e + 4]), fexp2(y[e + 5]))),
               sv[e], sv[e + 1]);
    const float s8 = (sv[0] + sv[1]) + (sv[2] + sv[3]);
    s = fmaf(s, fexp2(fmaf(m, k, -mk)), s8);
    m = mn;
  }
}
// The lanes' statistics combined over the warp (every lane gets the result).
template <bool kGreedy>
SPEC_DEV void warp_stats(float& m, float& s, int32_t& mi, float k) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    if constexpr (kGreedy) {
      const int32_t i2 = __shfl_xor_sync(0xffffffffu, mi, off);
      amax_combine(m, mi, m2, i2);
    } else {
      const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
      ms_combine(m, s, m2, s2, k);
    }
  }
}

// Verify length K_b of row gb (cycle-major row index c * B + b): the given
// length clamped to 1..K; or, from confidence scores, the number of leading
// positions whose prefix survival (fp32 product of the scores of positions
// 0..i, in position order) is at least the threshold, at least 1; else K.
SPEC_DEV int row_verify_len(const ArgsTC& a, int64_t gb) {
  const int K = a.K;
  if (a.vlen) return min(max(__ldg(a.vlen + gb), 1), K);
  if (!a.conf) return K;
  const float* c = a.conf + gb * K;
  float s = 1.f;
  int kb = 0;
  for (int i = 0; i < K; ++i) {
    s = __fmul_rn(s, __ldg(c + i));
    if (!(s >= a.conf_thr)) break;  // a NaN score ends the prefix too
    kb = i + 1;
  }
  return max(kb, 1);
}

template <typename T>
SPEC_DEV float ld_elem(const T* p, int64_t i);
template <>
SPEC_DEV float ld_elem<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

// ---------------------------------------------------------------------------
template <int N>
__global__ void __launch_bounds__(kThreads, 1) k_cycle_tc(const __grid_constant__ ArgsTC a) {
  constexpr int NCOL = N / 2;           // columns (batch rows) per compute warp
  constexpr int NS = NCOL > 32 ? NCOL / 32 : 1;  // column slabs a warp takes in turn
  constexpr int SC = NCOL / NS;         // columns per slab (at most 32)
  constexpr int L = 32 / SC;            // lanes per row after the transpose
  constexpr int NV = SC / 8;            // 16-byte words per lane and logit row
  constexpr int kNS = kNSof<N>;         // W ring stages
  using T = __nv_bfloat16;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int nkb = a.r / 64;             // 64-rank blocks = W ring stages per chunk
  uint8_t* sW = smem;                                       // kNS x 16 KB
  uint8_t* sU = sW + (size_t)kNS * kWStage;                 // nkb x N x 128 B
  float* sT = reinterpret_cast<float*>(sU + (size_t)nkb * N * 128);  // 8 x 32 x SC floats
  const size_t rslot = (size_t)a.nc * kCH * sizeof(__nv_bfloat16);  // one row slice of the CTA
  uint8_t* sR = reinterpret_cast<uint8_t*>(sT + 8 * 32 * SC);        // 2 x nts row slices
  const int kTS = a.nts;
  CtlT<N>* ctl = reinterpret_cast<CtlT<N>*>(sR + 2 * kTS * rslot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  const int G = a.G, K = a.K, V = a.V;
  const int chunk0 = cta * a.nc;
  const int ncc = min(a.nc, a.nchunks - chunk0);  // chunks owned by this CTA
  const int ntc = min(a.NT, ncc);                 // of which in tensor memory
  const int has_final = a.greedy ? 0 : 1;
  const int nrounds = K + has_final;              // MMA rounds per group
  // jobs: (cycle, group) pairs in cycle-major order; rows of job t are
  // c * B + g * N + n in the inputs and outputs (c = t / ngroups, g = t % ngroups)
  const int njobs = a.ngroups * a.ncyc;
  WsHeader* hdr = a.hdr;
  const T* base = a.base;
  const T* target = a.target;
  const T* Ug = a.U;
  const T* Wg = a.W;
  const float k = a.k;
  const uint32_t DB = (uint32_t)a.NT * 128;       // first accumulator column

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&ctl->wfull[i], 1);
      mbar_init(&ctl->wempty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->dfull[b], 1);
      mbar_init(&ctl->dfree[b], kComputeThreads / 32);
    }
    mbar_init(&ctl->bready, 1);
    mbar_init(&ctl->tready, 1);
    mbar_init(&ctl->mmadone, 1);
    for (int w = 0; w < 2; ++w)
      for (int i = 0; i < kTSMax; ++i) mbar_init(&ctl->tfull[w][i], 1);
    ctl->tgo_cnt = 0;
    ctl->tdone_cnt[0] = ctl->tdone_cnt[1] = 0;
    ctl->abort_local = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ctl->tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = ctl->tmem_slot;

  // =========================================================================
  // W producer: first the NT resident chunks (read once, by the compute warps,
  // into tensor memory), then per MMA round the streamed chunks, in the MMA's
  // order.  Stage = 64 rank rows of one chunk, two 64-token boxes per K-step.
  // =========================================================================
  if (warp == kProducerWarp) {
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_last();
      const uint64_t pol_once = policy_evict_last();  // the draws re-read W columns from L2
      tma_prefetch_desc(&a.tmW);
      uint32_t Lw = 0;
      bool ok = true;
      auto load_stage = [&](int c, int s, uint64_t pol) {
        const uint32_t slot = Lw % kNS;
        if (Lw >= kNS &&
            !mbar_wait_bounded(&ctl->wempty[slot], ((Lw / kNS) - 1) & 1, a.spin, &hdr->abort)) {
          record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, 100 + c);
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(&ctl->wfull[slot], (uint32_t)kWStage);
        const int v0 = (chunk0 + c) * kCH;
        for (int j = 0; j < kKS; ++j) {
          uint8_t* dst = sW + (size_t)slot * kWStage + (size_t)j * kWChunk;
          const int kr = (s * kKS + j) * 16;
          tma_load_2d(dst, &a.tmW, &ctl->wfull[slot], v0, kr, pol);
          tma_load_2d(dst + kWChunk / 2, &a.tmW, &ctl->wfull[slot], v0 + 64, kr, pol);
        }
        ++Lw;
      };
      for (int c = 0; c < ntc && ok; ++c)
        for (int s = 0; s < nkb && ok; ++s) load_stage(c, s, pol_once);
      for (int t = 0; t < njobs && ok; ++t)
        for (int rd = 0; rd < nrounds && ok; ++rd)
          for (int c = ntc; c < ncc && ok; ++c)
            for (int s = 0; s < nkb && ok; ++s) load_stage(c, s, pol_stream);
      // nothing in flight at exit: the latest load into every slot has landed
      for (uint32_t L2 = (Lw > kNS ? Lw - kNS : 0); L2 < Lw; ++L2)
        mbar_drain(&ctl->wfull[L2 % kNS], (L2 / kNS) & 1);
    }
  }
  // =========================================================================
  // MMA issuer
  // =========================================================================
  else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc_ss = idesc_bf16_f32(128, N, /*a_mn_major=*/true, /*b_mn_major=*/false);
      const uint32_t idesc_ts = idesc_bf16_f32(128, N, /*a_mn_major=*/false, /*b_mn_major=*/false);
      uint32_t Lw = (uint32_t)(ntc * nkb), cc = 0, rd_ctr = 0;
      bool ok = mbar_wait_bounded(&ctl->tready, 0, a.spin, &hdr->abort);
      if (!ok) record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_BREADY, cta, -1);
      tc_fence_after();
      for (int t = 0; t < njobs && ok; ++t) {
        for (int rd = 0; rd < nrounds && ok; ++rd, ++rd_ctr) {
          if (!mbar_wait_bounded(&ctl->bready, rd_ctr & 1, a.spin, &hdr->abort)) {
            record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_BREADY, cta, rd);
            ok = false;
            break;
          }
          tc_fence_after();
          if (a.trace && cta == 0 && t == 0) a.trace[(size_t)min(rd, K) * kTracePhases + 9] = globaltimer_ns();
          for (int c = 0; c < ncc && ok; ++c, ++cc) {
            const uint32_t b = cc & 1;
            if (cc >= 2 &&
                !mbar_wait_bounded(&ctl->dfree[b], ((cc >> 1) - 1) & 1, a.spin, &hdr->abort)) {
              record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_TFREE, cta, rd);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t dcol = taddr + DB + b * (uint32_t)N;
            if (c < ntc) {  // A = W^T resident in tensor memory
              for (int ks = 0; ks < nkb * 4; ++ks) {
                const uint64_t bd = smem_desc_sw128(
                    smem_u32(sU + (size_t)(ks >> 2) * N * 128) + (ks & 3) * 32, 16, 1024);
                umma_bf16_ts(dcol, taddr + (uint32_t)(c * 128 + ks * 8), bd, idesc_ts, ks != 0);
              }
            } else {        // A = W^T streamed through the ring
              for (int s = 0; s < nkb && ok; ++s) {
                const uint32_t slot = Lw % kNS;
                if (!mbar_wait_bounded(&ctl->wfull[slot], (Lw / kNS) & 1, a.spin, &hdr->abort)) {
                  record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, rd);
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_u32(sW + (size_t)slot * kWStage);
#pragma unroll
                for (int j = 0; j < kKS; ++j) {
                  const int ks = s * kKS + j;
                  const uint64_t bd = smem_desc_sw128(
                      smem_u32(sU + (size_t)(ks >> 2) * N * 128) + (ks & 3) * 32, 16, 1024);
                  const uint64_t ad = smem_desc_sw128(a_base + j * kWChunk, kWChunk / 2, 1024);
                  umma_bf16(dcol, ad, bd, idesc_ss, ks != 0);
                }
                umma_commit(&ctl->wempty[slot]);
                ++Lw;
              }
              if (!ok) break;
            }
            umma_commit(&ctl->dfull[b]);
          }
          if (a.trace && cta == 0 && t == 0) a.trace[(size_t)min(rd, K) * kTracePhases + 10] = globaltimer_ns();
        }
      }
      umma_commit(&ctl->mmadone);
      mbar_drain(&ctl->mmadone, 0);
    }
  }
  // =========================================================================
  // Target warps: statistics of target row j (rows still verifying; at a
  // row's last verified position also its bonus row K_b) over this CTA's
  // slice, one job per position from npro on, released by the compute warps
  // up to two positions ahead of the draft chain.  Each warp fetches its
  // rows' slices with bulk copies into a private ring and reduces them from
  // shared memory.
  // =========================================================================
  else if (warp >= kTargetWarp0) {
    const int tw = warp - kTargetWarp0;
    uint8_t* ring = sR + (size_t)tw * kTS * rslot;
    const int vlo = chunk0 * kCH, vhi = min(V, (chunk0 + ncc) * kCH);
    const uint32_t bytes = (uint32_t)((vhi - vlo) * sizeof(T));
    const int npieces = (vhi - vlo) / 8;
    const uint64_t pol = policy_evict_first();
    uint32_t tu = 0, tcn = 0, J = 0;  // copies issued, copies consumed, target jobs taken
    bool ok = true;
    for (int t = 0; t < njobs && ok; ++t) {
      const int g = t % a.ngroups, par = t & 1;
      const int64_t gb0 = (int64_t)(t / a.ngroups) * a.B + (int64_t)g * N;  // row 0 of the job
      const int nb_g = min(N, a.B - g * N);
      // positions below npro were taken by the compute warps at the job's start
      for (int j = a.npro; j < K && ok; ++j, ++J) {
        {  // wait until the compute warps release this position (bounded)
          uint64_t it = 0;
          while (ld_acquire_cta_smem(&ctl->tgo_cnt) <= J) {
            if (++it >= a.spin || ((it & 63) == 0 && ld_volatile_u32(&hdr->abort))) {
              if (lane == 0 && it >= a.spin) record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_BREADY, cta, 3000 + j);
              ok = false;
              break;
            }
            __nanosleep(64);
          }
          if (!ok) break;
        }
        if (a.trace && cta == 0 && t == 0 && tw == 0 && lane == 0)
          a.trace[(size_t)j * kTracePhases + 4] = globaltimer_ns();  // target job taken
          // this lane's row n = 2 l + tw (+ 64 h) and its verify length K_b
        for (int h = 0; h < (N + 63) / 64 && ok; ++h) {
          const int nl = 2 * lane + tw + 64 * h;
          const bool inrow = nl < nb_g && nl < N;
          const int kbl = inrow ? row_verify_len(a, gb0 + nl) : 0;
          const bool verifying =
              inrow && j < kbl && (j == 0 || *reinterpret_cast<volatile int32_t*>(&ctl->alive[nl]) != 0);
          if (verifying && j + 1 < kbl) {  // the next job's target rows of this row into L2
            const int64_t bb = gb0 + nl;
            prefetch_l2_bulk(target + (bb * (K + 1) + j + 1) * V + vlo, bytes);
            if (j + 2 == kbl) prefetch_l2_bulk(target + (bb * (K + 1) + kbl) * V + vlo, bytes);
          }
          // rows still verifying at position j (a snapshot: a row that stops
          // meanwhile only costs an unused slice); items: (row, target row j)
          // and, at a row's last verified position, (row, target row K_b)
          const uint32_t rows = __ballot_sync(FULL, verifying);
          const uint32_t lastm = __ballot_sync(FULL, verifying && j == kbl - 1);
          uint32_t imask = rows, cmask = rows;
          int isub = 0, csub = 0;
          auto next_item = [&](uint32_t& m, int& sub, int& n, int& trow) {
            if (!m) return false;
            const int l = __ffs(m) - 1;
            n = 2 * l + tw + 64 * h;
            trow = sub == 0 ? j : j + 1;
            if (((lastm >> l) & 1u) && sub == 0) {
              sub = 1;
            } else {
              sub = 0;
              m &= m - 1;
            }
            return true;
          };
          auto issue = [&]() {  // lane 0: one copy into the slot freed last
            int n, trow;
            if (!next_item(imask, isub, n, trow)) return;
            const uint32_t slot = tu % kTS;
            if (lane == 0) {
              mbar_arrive_expect_tx(&ctl->tfull[tw][slot], bytes);
              bulk_load(ring + slot * rslot,
                        target + ((gb0 + n) * (K + 1) + trow) * V + vlo, bytes,
                        &ctl->tfull[tw][slot], pol);
            }
            ++tu;
          };
          while (tu - tcn < (uint32_t)kTS && imask) issue();
          int n, trow;
          while (next_item(cmask, csub, n, trow)) {
            const uint32_t slot = tcn % kTS;
            if (!mbar_wait_bounded(&ctl->tfull[tw][slot], (tcn / kTS) & 1, a.spin, &hdr->abort)) {
              if (lane == 0) record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, 4000 + j);
              ok = false;
              break;
            }
            const uint4* sl = reinterpret_cast<const uint4*>(ring + slot * rslot);
            float m = -INFINITY, sm = 0.f;
            int32_t mi = 0x7fffffff;
            // one pass: the lane's pieces p = lane + 32 u are read four at a
            // time (their shared-memory latencies overlap); stochastic rows
            // keep a running (max, sum) rescaled once per piece
            auto pass = [&](auto greedy_tag) {  // one code path per mode
              constexpr bool kGreedy = decltype(greedy_tag)::value;
              for (int p0 = lane; p0 < npieces; p0 += 128) {
                uint4 w4[4];
  #pragma unroll
                for (int u = 0; u < 4; ++u)
                  w4[u] = p0 + 32 * u < npieces ? sl[p0 + 32 * u] : make_uint4(0, 0, 0, 0);
  #pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const int p = p0 + 32 * u;
                  if (p >= npieces) break;
                  piece_stats<kGreedy>(w4[u], vlo + 8 * p, k, m, sm, mi);
                }
              }
            };
            if (a.greedy)
              pass(std::true_type{});
            else
              pass(std::false_type{});
            __syncwarp();
            ++tcn;
            issue();  // the slot is free: the next slice is in flight while this one reduces
            if (a.greedy)
              warp_stats<true>(m, sm, mi, k);
            else
              warp_stats<false>(m, sm, mi, k);
            if (lane == 0)
              a.tpart[(((int64_t)par * (K + 1) + trow) * N + n) * kMaxG + cta] =
                  a.greedy ? make_float2(m, __int_as_float(mi)) : make_float2(m, sm);
          }
        }  // halves
        if (!ok) break;
        __threadfence();  // the partials are visible device-wide before the job is reported
        __syncwarp();
        if (lane == 0) add_release_cta_smem(&ctl->tdone_cnt[tw], 1u);
        if (a.trace && cta == 0 && t == 0 && tw == 0 && lane == 0)
          a.trace[(size_t)j * kTracePhases + 31] = globaltimer_ns();  // target job published
      }
    }
    // nothing in flight at exit
    while (tcn < tu) {
      mbar_drain(&ctl->tfull[tw][tcn % kTS], (tcn / kTS) & 1);
      ++tcn;
    }
  }
  // =========================================================================
  // Compute warps
  // =========================================================================
  else {
    const int q4 = warp & 3;               // tensor-memory lane quadrant (32 tokens of a chunk)
    const int n0 = (warp >> 2) * NCOL;     // first column (batch row) of this warp
    const int jj = lane / L, tg = lane % L;
    // the batch row this lane holds after the transpose of slab s
    auto slab_row = [&](int s) { return n0 + s * SC + jj; };
    float* tbuf = sT + warp * 32 * SC;
    uint32_t cc = 0, nbar = 0;
    const uint32_t ev0 = ld_volatile_u32(&hdr->events);  // record tags of this launch start here
    bool failed = false;
    // the current job: index, cycle of the launch, first row (cycle-major), Philox cycle
    int jt = 0, jcy = 0;
    int64_t jb0 = 0;
    uint64_t jcyc = a.cycle;
    // the committed token row b's block starts from: the given last token in
    // the first cycle, then the last token the row emitted in the cycle before
    auto first_token = [&](int b) -> int32_t {
      return jcy == 0 ? __ldg(a.last_token + b) : __ldcg(a.next_token + b);
    };
    // the row's last emitted token of this cycle: carried to the next cycle
    auto emit_last = [&](int b, int32_t tok) {
      if (a.next_token) a.next_token[b] = tok;
    };
    auto soft_fail = [&](int code, int site, int x, int y) {
      record_error(hdr, code, site, x, y);
      ctl->abort_local = 1;
    };
    auto grid_arrive = [&]() {
      named_sync();
      if (tid == 0) {
        // the barrier above orders the CTA's writes before this release
        red_release_add_u32(&hdr->bar, 1u);
        ++nbar;
      }
    };
    auto grid_wait = [&]() {
      if (tid == 0) {
        if (!grid_wait_count(hdr, &hdr->bar, nbar * (uint32_t)G, a.spin, SITE_GRID_BARRIER))
          ctl->abort_local = 1;
      }
      named_sync();
      return ctl->abort_local == 0;
    };
    const float NaNf = __int_as_float(0x7fc00000);
    const int vslice_lo = chunk0 * kCH;
    const int vslice_hi = min(V, (chunk0 + ncc) * kCH);
    const uint32_t slice_bytes = (uint32_t)((vslice_hi - vslice_lo) * sizeof(T));
    uint64_t* trace = (a.trace != nullptr && cta == 0 && tid == 0) ? a.trace : nullptr;
    auto mark = [&](int g, int step, int phase) {
      if (trace && g == 0 && jt == 0) trace[(size_t)step * kTracePhases + phase] = globaltimer_ns();
    };

    mark(0, K + 1, 2);
    // ---- W^T of the resident chunks into tensor memory (once per launch).
    // Stage L (chunk L / nkb, rank block L % nkb) is read by the quartet of
    // warps L & 1: warp q4 takes tokens 32 q4 .. 32 q4 + 31 and packs two
    // consecutive ranks per 32-bit cell.
    {
      const int quartet = warp >> 2;
      const int m = q4 * 32 + lane;  // token of the chunk = tensor-memory lane
      const int hf = m >> 6, t = m & 63;
      for (int Ls = quartet; Ls < ntc * nkb; Ls += 2) {
        const uint32_t slot = (uint32_t)Ls % kNS;
        if (!mbar_wait_bounded(&ctl->wfull[slot], ((uint32_t)Ls / kNS) & 1, a.spin, &hdr->abort))
          soft_fail(SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, -2);
        const int c = Ls / nkb, s = Ls % nkb;
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < kKS; ++j) {
          const uint8_t* blk = sW + (size_t)slot * kWStage + (size_t)j * kWChunk + hf * (kWChunk / 2);
#pragma unroll
          for (int rp = 0; rp < 8; ++rp) {
            const int r0 = 2 * rp, r1 = 2 * rp + 1;
            const uint32_t lo = *reinterpret_cast<const uint16_t*>(
                blk + r0 * 128 + (((t >> 3) ^ (r0 & 7)) << 4) + (t & 7) * 2);
            const uint32_t hi = *reinterpret_cast<const uint16_t*>(
                blk + r1 * 128 + (((t >> 3) ^ (r1 & 7)) << 4) + (t & 7) * 2);
            pk[j * 8 + rp] = kPackEvenLow ? (lo | (hi << 16)) : (hi | (lo << 16));
          }
        }
        tmem_st32(taddr + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(c * 128 + s * 32), pk);
        quartet_sync(quartet);  // every warp of the quartet has read the stage
        if (q4 == 0 && lane == 0) mbar_arrive(&ctl->wempty[slot]);
      }
      tmem_st_wait();
      tc_fence_before();
      named_sync();
      if (tid == 0) mbar_arrive(&ctl->tready);
      if (ctl->abort_local) failed = true;
    }

    // ---- Gather U[prev] rows (ctl->prev) into the B operand.
    // B operand of step i: the Markov head's U[prev] rows, or the RNN head's
    // state s_i = bf16(clamp(U[prev] + Wh s_{i-1}, -1, 1)) (Wh s_{i-1} from P,
    // computed during the step before); at the final step (step == K) the RNN
    // head takes each stopped row's saved state of its stop row instead.
    auto gather_u = [&](int nb_g, int step) {
      const int cpr = a.r / 8;  // 16-byte chunks per row
      constexpr int kItAll = N * 32 / kComputeThreads;  // r <= 256: at most 32 chunks per row
      constexpr int kIt = kItAll < 8 ? kItAll : 8;      // words in flight per thread
      for (int t0 = 0; t0 < kItAll; t0 += kIt) {
      uint4 val[kIt];
#pragma unroll
      for (int t = 0; t < kIt; ++t) {  // all loads first, from clamped (valid) rows
        const int idx = tid + (t0 + t) * kComputeThreads;
        const int n = min(idx / cpr, N - 1), c = idx % cpr;
        if (a.Wh && step == K) {
          const int j = ctl->alive[n] ? 0 : min(ctl->stoprow[n], K - 1);  // rows past the group: any saved row
          val[t] = __ldcg(reinterpret_cast<const uint4*>(a.shist + ((size_t)j * N + n) * a.r) + c);
        } else {
          val[t] = __ldg(reinterpret_cast<const uint4*>(Ug + (size_t)ctl->prev[n] * a.r) + c);
        }
      }
      if (a.Wh && step < K) {
#pragma unroll
        for (int t = 0; t < kIt; ++t) {
          const int idx = tid + (t0 + t) * kComputeThreads;
          const int n = min(idx / cpr, N - 1), c = idx % cpr;
          float pw[8];
          if (step > 0) {
            const float4* pp = reinterpret_cast<const float4*>(a.P + ((size_t)(step & 1) * N + n) * a.r + c * 8);
            const float4 p0 = __ldcg(pp), p1 = __ldcg(pp + 1);
            pw[0] = p0.x; pw[1] = p0.y; pw[2] = p0.z; pw[3] = p0.w;
            pw[4] = p1.x; pw[5] = p1.y; pw[6] = p1.z; pw[7] = p1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) pw[e] = 0.f;
          }
          float x[8];
          bf16x8(val[t], x);
          uint32_t h[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo_ = fminf(fmaxf(__fadd_rn(x[2 * e], pw[2 * e]), -1.f), 1.f);
            const float hi_ = fminf(fmaxf(__fadd_rn(x[2 * e + 1], pw[2 * e + 1]), -1.f), 1.f);
            const __nv_bfloat162 bb = __floats2bfloat162_rn(lo_, hi_);
            h[e] = *reinterpret_cast<const uint32_t*>(&bb);
          }
          val[t] = make_uint4(h[0], h[1], h[2], h[3]);
          // the state of this step, for a final-step bias at this row
          if (cta == 0 && idx < N * cpr && idx / cpr < nb_g)
            *(reinterpret_cast<uint4*>(a.shist + ((size_t)step * N + idx / cpr) * a.r) + c) = val[t];
        }
      }
#pragma unroll
      for (int t = 0; t < kIt; ++t) {
        const int idx = tid + (t0 + t) * kComputeThreads;
        const int n = idx / cpr, c = idx % cpr;
        if (idx >= N * cpr) continue;
        const int ka = c >> 3, j = c & 7;
        *reinterpret_cast<uint4*>(sU + (size_t)ka * N * 128 + n * 128 + ((j ^ (n & 7)) << 4)) =
            n < nb_g ? val[t] : make_uint4(0, 0, 0, 0);
      }
      }  // batches
      fence_proxy_async_smem();
      named_sync();
      if (tid == 0) mbar_arrive(&ctl->bready);
    };

    // Accumulator tile of the next chunk for this thread (lane = token, NCOL
    // columns), handed back to the MMA once loaded; then transposed.
    // (Slab s of the warp's columns; the accumulator is waited for at slab 0
    // and handed back after the last slab.)
    auto acc_tile = [&](float (&z)[SC], int s) {
      const uint32_t b = cc & 1;
      if (s == 0) {
        if (!mbar_wait_bounded(&ctl->dfull[b], (cc >> 1) & 1, a.spin, &hdr->abort))
          soft_fail(SPEC_ERR_TIMEOUT, SITE_MBAR_MMA, cta, (int)cc);
        tc_fence_after();
      }
      float d[SC];
      tmem_ld_cols<SC>(taddr + ((uint32_t)(q4 * 32) << 16) + DB + b * (uint32_t)N + (uint32_t)(n0 + s * SC), d);
      if (s == NS - 1) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->dfree[b]);
        ++cc;
      }
      transpose_in<SC>(tbuf, d, lane);
      __syncwarp();
      transpose_out<SC>(tbuf, z, lane);
      __syncwarp();
    };

    // Scan of one 32-token bucket (whole warp): weights per lane, target
    // tin within the bucket; returns the winning lane.
    auto bucket_scan = [&](float wv, float tin) {
      float incl = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned cross = __ballot_sync(FULL, incl > tin);
      if (cross) return __ffs(cross) - 1;
      const unsigned pos = __ballot_sync(FULL, wv > 0.f);
      return pos ? 31 - __clz(pos) : 0;
    };

    // ---- the draw of one row (stochastic steps and the final step), by the
    // whole CTA of the row's reducer, from the record ctl->rrec[j]:
    // 1. warp 0 walks the owner CTA's published bucket statistics in ascending
    //    token order to the bucket holding the inverse-CDF target;
    // 2. the bucket's 32 logits are formed here: z = base + U[prev].W with
    //    the rank split over the 8 warps (the same bf16 inputs as the tensor
    //    cores, fp32 accumulation);
    // 3. warp 0 scans the bucket (kind 0: q_i, then the accept test against
    //    p_i; kind 2: the residual or the bonus row) and writes the outputs.
    auto draw_row = [&](int kind, int g, int par, int i, int n, int j) {
      if (kind == 0 && i >= ctl->kb[n]) return;  // past the row's verify length: no draft
      RecT& rr = ctl->rrec[j];
      const int b = g * N + n;
      const int64_t gb = jb0 + n;
      const int o = rr.owner;
      const float M = rr.M;
      const bool use_p = (rr.flags & 2) != 0;
      const bool alive = ctl->alive[n] != 0;
      const int row = kind == 0 ? i : (alive ? ctl->kb[n] : ctl->stoprow[n]);
      if (warp == 0) {
        const int nbk_o = min(a.nc, a.nchunks - o * a.nc) * 4;
        const float tin = rr.trem;
        float carry = 0.f, tin_in = INFINITY;
        int pick = -1, lastb = -1;
        for (int b0 = 0; b0 < nbk_o && pick < 0; b0 += 32) {  // 32 buckets per pass
          const int bk = b0 + lane;
          float w = 0.f;
          if (bk < nbk_o) {
            const float2 pv = __ldcg(a.gbk + ((size_t)o * a.nbk + bk) * N + n);
            w = kind == 0 ? (pv.y > 0.f ? pv.y * fexp2((pv.x - M) * k) : 0.f)
                          : (use_p ? pv.y : pv.x);
          }
          float incl = w;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += y;
          }
          const unsigned cross = __ballot_sync(FULL, carry + incl > tin);
          const unsigned pos = __ballot_sync(FULL, w > 0.f);
          if (pos) lastb = b0 + 31 - __clz(pos);
          if (cross) {
            const int l = __ffs(cross) - 1;
            pick = b0 + l;
            tin_in = tin - (carry + __shfl_sync(FULL, incl - w, l));
          }
          carry += __shfl_sync(FULL, incl, 31);
        }
        if (pick < 0) {
          pick = lastb < 0 ? 0 : lastb;
          tin_in = INFINITY;
        }
        if (lane == 0) {
          ctl->dbk = pick;
          ctl->dtin = tin_in;
        }
      }
      named_sync();
      if (j == 0 && kind == 0) mark(g, i, 14);
      const int bk = ctl->dbk;
      const int v0 = (o * a.nc + (bk >> 2)) * kCH + (bk & 3) * 32;
      const int v = v0 + lane, vc = min(v, V - 1);
      float tv = 0.f, bv = 0.f;
      if (warp == 0) {  // the row's logits at the bucket's tokens, in flight meanwhile
        if (kind == 0) {
          bv = ld_elem(base, (gb * K + i) * V + vc);
          tv = ld_elem(target, (gb * (K + 1) + i) * V + vc);
        } else {
          tv = ld_elem(target, (gb * (K + 1) + row) * V + vc);
          if (!alive) bv = ld_elem(base, (gb * K + row) * V + vc);
        }
      }
      {  // warp w: rank rows [w*ks, w*ks + ks)
        const int ks = (a.r + 7) / 8, k0 = warp * ks, k1 = min(a.r, k0 + ks);
        // the bias operand of the row: U[prev] (Markov head) or the RNN state in sU
        float uval = 0.f;
        if (k0 + lane < k1) {
          const int kk = k0 + lane, c = kk >> 3;
          uval = a.Wh ? __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                            sU + (size_t)(c >> 3) * N * 128 + n * 128 + (((c & 7) ^ (n & 7)) << 4) +
                            (kk & 7) * 2))
                      : ld_elem(Ug, (int64_t)ctl->prev[n] * a.r + kk);
        }
        // lane l: the 8 tokens v0 + 8 (l & 3) .. + 7 of rank rows k0 + (l >> 2) + 8 j,
        // one 16-byte load per rank row (V % 8 == 0: a group of 8 is all in or all out)
        const int g8 = lane & 3, rs = lane >> 2;
        const int vg = v0 + 8 * g8;
        uint4 wq[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int kk = k0 + rs + 8 * j;
          wq[j] = (vg < V && kk < k1)
                      ? __ldg(reinterpret_cast<const uint4*>(Wg + (int64_t)kk * V + vg))
                      : make_uint4(0, 0, 0, 0);
        }
        float acc8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc8[e] = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float u = __shfl_sync(FULL, uval, rs + 8 * j);
          float xw[8];
          bf16x8(wq[j], xw);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc8[e] = fmaf(u, xw[e], acc8[e]);
        }
        // the 8 lanes of a token group (equal l & 3) hold its rank rows
#pragma unroll
        for (int off = 4; off < 32; off <<= 1)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc8[e] += __shfl_xor_sync(FULL, acc8[e], off);
        if (rs == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) ctl->zpart[warp][8 * g8 + e] = acc8[e];
        }
      }
      named_sync();
      if (j == 0 && kind == 0) mark(g, i, 15);
      if (warp == 0) {
        float bias = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) bias += ctl->zpart[w][lane];
        const bool valid = v < V;
        if (kind == 0) {
          const float z = bias + bv, S = rr.S;
          const float e = valid ? fexp2((z - M) * k) : 0.f;
          const int wl = bucket_scan(e, ctl->dtin);
          const int d = v0 + wl;
          const float zd = __shfl_sync(FULL, z, wl), td = __shfl_sync(FULL, tv, wl);
          const float qd = fexp2((zd - M) * k) / S;
          int accept = 1;
          float pd = __int_as_float(0x7fc00000);
          if (alive) {
            pd = fexp2((td - rr.Mt) * k) / rr.St;
            const float ratio = fexp2(((td - rr.Mt) - (zd - M)) * k) * (S / rr.St);
            const float uacc =
                philox_uniform(a.seed, jcyc, a.row0 + (uint32_t)b, (uint32_t)i, TAG_ACCEPT);
            accept = uacc < fminf(ratio, 1.0f) ? 1 : 0;
          }
          if (lane == 0) {
            prefetch_l2_bulk(Ug + (size_t)d * a.r, (uint32_t)(a.r * sizeof(T)));  // the next gather
            rr.token = d;
            rr.acc = accept;
            a.tokens[((int64_t)par * K + i) * N + n] = d;
            if (a.draft) a.draft[gb * K + i] = d;
            if (a.q_draft) a.q_draft[gb * K + i] = qd;
            if (alive) {
              if (a.p_draft) a.p_draft[gb * K + i] = pd;
              if (accept) a.out[gb * (K + 1) + i] = d;
            }
          }
        } else {  // the same expressions as the final epilogue's bucket masses
          const float4 c = ctl->fcst[n];
          const float p = fexp2((tv - c.x) * k) * c.y;
          const float q = c.w != 0.f ? fexp2((bias + bv - c.z) * k) * c.w : 0.f;
          const float w = valid ? ((alive || use_p) ? p : fmaxf(p - q, 0.f)) : 0.f;
          const int wl = bucket_scan(w, ctl->dtin);
          if (lane == 0) {
            rr.token = v0 + wl;
            a.out[gb * (K + 1) + row] = v0 + wl;
            emit_last(b, v0 + wl);
          }
        }
      }
      named_sync();
    };

    // ---- row reducers.  Row n of a group is combined by one warp of CTA
    // n % G; lanes hold E consecutive per-CTA partials each, so a warp prefix
    // sum walks the CTAs in ascending token order.
    //  kind 0: draft step i -- stochastic: total, owner CTA, the target inside
    //          it, plus target row i statistics (and row K's at the last step)
    //          for rows still verifying, then the draw; greedy: the arg-max
    //          tokens and the accept outcome;
    //  kind 2: final residual / bonus masses -- owner of the last draw.
    constexpr int E = (kMaxG + 31) / 32;
    auto reduce_rows = [&](int kind, int g, int par, int i, int nb_g) {
      int mine = 0, local = 0;
      const int slot = kind == 0 ? i : K;  // partial and record slot
      for (int n = cta; n < nb_g; n += G, ++local) {
        ++mine;
        if ((local & 7) != warp) continue;  // warp-uniform
        const int b = g * N + n;
        const int64_t gb = jb0 + n;
        const int c0 = lane * E;
        const int kbn = ctl->kb[n];
        // verifying at this step; and this step is the row's last verified position
        const bool live = ctl->alive[n] != 0 && (kind != 0 || i < kbn);
        const bool last = kind == 0 && i == kbn - 1;
        RecT rc;
        rc.M = 0.f; rc.S = 1.f; rc.Mt = 0.f; rc.St = 1.f; rc.MtK = 0.f; rc.StK = 1.f;
        rc.trem = INFINITY; rc.owner = 0; rc.token = 0; rc.acc = 1; rc.flags = 0;
        rc.tam = 0; rc.tamK = 0; rc.pad[0] = rc.pad[1] = rc.pad[2] = 0;
        const float4* pp = a.dpart + ((((int64_t)par * (K + 1) + slot) * N + n) * kMaxG + c0);
        float4 v[E];
#pragma unroll
        for (int t = 0; t < E; ++t) v[t] = __ldcg(pp + t);
        // arg-max or (max, sum) over the CTAs' partials of one target row
        auto target_row = [&](int trow, float& Mo, float& So, int32_t& Io) {
          const float2* tp = a.tpart + ((((int64_t)par * (K + 1) + trow) * N + n) * kMaxG + c0);
          float2 tv[E];
#pragma unroll
          for (int t = 0; t < E; ++t) tv[t] = __ldcg(tp + t);
          if (a.greedy) {
            float av = -INFINITY;
            int32_t ai = 0x7fffffff;
#pragma unroll
            for (int t = 0; t < E; ++t)
              if (c0 + t < G) amax_combine(av, ai, tv[t].x, __float_as_int(tv[t].y));
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
              const float a2 = __shfl_xor_sync(FULL, av, off);
              const int32_t i2 = __shfl_xor_sync(FULL, ai, off);
              amax_combine(av, ai, a2, i2);
            }
            Io = ai;
          } else {
            float Mt = -INFINITY;
#pragma unroll
            for (int t = 0; t < E; ++t)
              if (c0 + t < G) Mt = fmaxf(Mt, tv[t].x);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) Mt = fmaxf(Mt, __shfl_xor_sync(FULL, Mt, off));
            float st = 0.f;
#pragma unroll
            for (int t = 0; t < E; ++t)
              if (c0 + t < G && tv[t].y > 0.f) st += tv[t].y * fexp2((tv[t].x - Mt) * k);
            Mo = Mt;
            So = warp_sum(st);
          }
        };
        if (kind == 0 && a.greedy) {
          float av = -INFINITY;
          int32_t ai = 0x7fffffff;
#pragma unroll
          for (int t = 0; t < E; ++t)
            if (c0 + t < G) amax_combine(av, ai, v[t].x, __float_as_int(v[t].y));
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) {
            const float a2 = __shfl_xor_sync(FULL, av, off);
            const int32_t i2 = __shfl_xor_sync(FULL, ai, off);
            amax_combine(av, ai, a2, i2);
          }
          rc.token = ai;
          if (lane == 0 && i + 1 < K)  // the next gather reads this row of U
            prefetch_l2_bulk(Ug + (size_t)ai * a.r, (uint32_t)(a.r * sizeof(T)));
        } else {
          float w[E];
          float M = -INFINITY;
          bool use_p = false;
          if (kind == 0) {
#pragma unroll
            for (int t = 0; t < E; ++t)
              if (c0 + t < G) M = fmaxf(M, v[t].x);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
#pragma unroll
            for (int t = 0; t < E; ++t)
              w[t] = (c0 + t < G && v[t].y > 0.f) ? v[t].y * fexp2((v[t].x - M) * k) : 0.f;
          } else {
            float rt = 0.f;
#pragma unroll
            for (int t = 0; t < E; ++t)
              if (c0 + t < G) rt += v[t].x;
            rt = warp_sum(rt);
            use_p = !(rt > 0.f);
#pragma unroll
            for (int t = 0; t < E; ++t) w[t] = c0 + t < G ? (use_p ? v[t].y : v[t].x) : 0.f;
          }
          float loc = 0.f;
#pragma unroll
          for (int t = 0; t < E; ++t) loc += w[t];
          float incl = loc;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += y;
          }
          const float total = __shfl_sync(FULL, incl, 31);
          const int row = kind == 0 ? i : (live ? kbn : ctl->stoprow[n]);
          const float u = philox_uniform(a.seed, jcyc, a.row0 + (uint32_t)b, (uint32_t)row,
                                         kind == 0 ? TAG_DRAFT : TAG_RESAMPLE);
          const float tgt = u * total;
          float cum = incl - loc, before = 0.f;
          int found = 0x7fffffff, lastpos = -1;
#pragma unroll
          for (int t = 0; t < E; ++t) {
            if (w[t] > 0.f) lastpos = c0 + t;
            if (found == 0x7fffffff && w[t] > 0.f && cum + w[t] > tgt) {
              found = c0 + t;
              before = cum;
            }
            cum += w[t];
          }
          int own = found;
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) own = min(own, __shfl_xor_sync(FULL, own, off));
          int lp = lastpos;
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) lp = max(lp, __shfl_xor_sync(FULL, lp, off));
          const bool fb = own == 0x7fffffff;
          const float bown = __shfl_sync(FULL, before, fb ? 0 : own / E);
          rc.owner = fb ? max(lp, 0) : own;
          rc.trem = fb ? INFINITY : tgt - bown;
          rc.M = M;
          rc.S = total;
          if (kind == 2 && use_p) rc.flags |= 2;
        }
        if (kind == 0 && live) {
          target_row(i, rc.Mt, rc.St, rc.tam);
          if (last) target_row(kbn, rc.MtK, rc.StK, rc.tamK);  // the bonus row K_b
          if (a.greedy) {
            rc.acc = rc.tam == rc.token ? 1 : 0;
            if (lane == 0) {  // greedy step of a row still verifying
              a.out[gb * (K + 1) + i] = rc.acc ? rc.token : rc.tam;
              if (last && rc.acc) a.out[gb * (K + 1) + kbn] = rc.tamK;
              if (!rc.acc) emit_last(b, rc.tam);
              else if (last) emit_last(b, rc.tamK);
            }
          }
        }
        if (kind == 0 && a.greedy && lane == 0 && a.draft && i < kbn)
          a.draft[gb * K + i] = rc.token;
        if (lane == 0) ctl->rrec[local] = rc;
      }
      named_sync();
      if (kind == 0) mark(g, i, 13);
      // stochastic draws, one row at a time by the whole CTA
      if ((kind == 0 && !a.greedy) || kind == 2)
        for (int j = 0; j < mine; ++j) draw_row(kind, g, par, i, cta + j * G, j);
      if (tid < mine) {  // the record, then its tag (release: the record is visible first)
        const int n = cta + tid * G;
        const RecT& rc = ctl->rrec[tid];
        const size_t at = ((size_t)par * (K + 1) + slot) * N + n;
        store_rec(a.rec + at, rc);
        const uint32_t tag = ev0 + (uint32_t)(jt * (K + 1) + slot + 1);
        st_release_u64(a.rtag + at, ((uint64_t)tag << 32) | ((uint64_t)(rc.acc & 1) << 31) |
                                        (uint64_t)(uint32_t)(rc.token & 0x7fffffff));
      }
      return mine;
    };
    // Wait until every row's record of this slot carries this step's tag;
    // thread n < nb_g polls row n.  Returns false if the launch is aborted.
    auto records_hop = [&](int job, int par, int slot, int nb_g) {
      if (tid < nb_g) {
        const uint64_t* t = a.rtag + ((size_t)par * (K + 1) + slot) * N + tid;
        const uint32_t want = ev0 + (uint32_t)(job * (K + 1) + slot + 1);
        bool ok = false;
        for (uint64_t it = 0; it < a.spin; ++it) {
          const uint64_t wv = ld_acquire_u64(t);
          if ((uint32_t)(wv >> 32) == want) {
            ok = true;
            ctl->tok[tid] = (int32_t)(wv & 0x7fffffffu);
            ctl->acc[tid] = (int32_t)((wv >> 31) & 1u);
            break;
          }
          if ((it & 15) == 15 && ld_volatile_u32(&hdr->abort)) break;
          __nanosleep(32);
        }
        if (!ok) {
          if (!ld_volatile_u32(&hdr->abort))
            record_error(hdr, SPEC_ERR_TIMEOUT, SITE_REC_WAIT, cta, 6000 + slot);
          ctl->abort_local = 1;
        }
      }
      named_sync();
      return ctl->abort_local == 0;
    };
    // Quadrant partials of one quantity (lanes with tg == 0 hold the row's
    // value over this warp's tokens) into the CTA partial per row.
    auto put_quadrant = [&](float (*qa)[N], float (*qb)[N], float x, float y, int row) {
      if (tg == 0) {
        qa[q4][row] = x;
        qb[q4][row] = y;
      }
    };

    for (int t = 0; t < njobs && !failed; ++t) {
      const int g = t % a.ngroups, par = t & 1;
      const int nb_g = min(N, a.B - g * N);
      jt = t;
      jcy = t / a.ngroups;
      jb0 = (int64_t)jcy * a.B + (int64_t)g * N;
      jcyc = a.cycle + (uint64_t)jcy;
      for (int n = tid; n < N; n += kComputeThreads) {
        ctl->alive[n] = n < nb_g ? 1 : 0;
        ctl->stoprow[n] = K;
        int kbn = K;
        if (n < nb_g) {
          if (a.vlen) {
            const int32_t raw = __ldg(a.vlen + jb0 + n);
            if (raw < 1 || raw > K) record_error(hdr, SPEC_ERR_INVALID_ARG, SITE_TOKEN_RANGE, g * N + n, raw);
          }
          kbn = row_verify_len(a, jb0 + n);
        }
        ctl->kb[n] = kbn;
      }
      if (cta == 0) {
        for (int idx = tid; idx < nb_g * K; idx += kComputeThreads) {
          const int64_t o = jb0 * K + idx;
          const int pos = idx % K;
          const bool past = pos >= row_verify_len(a, jb0 + idx / K);
          if (a.p_draft) a.p_draft[o] = NaNf;
          if (a.q_draft && (a.greedy || past)) a.q_draft[o] = NaNf;
          if (a.draft && past) a.draft[o] = -1;
        }
      }
      named_sync();
      mark(g, K + 1, 0);
      // Target statistics of positions 0 .. npro-1 (every row verifies them,
      // and their target jobs would gate the first steps): the compute warps
      // take them here, before the first step, with the target warps' own
      // arithmetic.  Items (row n, target row): (n, j) for j < min(npro, K_b),
      // and (n, K_b) when K_b <= npro (the bonus row of a row whose last
      // verified position is among them).  A warp takes four items at a time,
      // read straight from global memory.
      if (a.npro > 0) {
        // Items in a dense order: q < P nb_g is (row q % nb_g, position q / nb_g),
        // then q - P nb_g the bonus row of that row (used when K_b <= P).  A warp
        // takes four consecutive items at a time and reads them together.
        auto take = [&](auto greedy_tag) {
          constexpr bool kG = decltype(greedy_tag)::value;
          constexpr int W = kComputeThreads / 32;
          const int P = a.npro, slots = nb_g * (P + 1);
          const int npieces = (vslice_hi - vslice_lo) / 8;
          for (int q0 = warp * 4; q0 < slots; q0 += 4 * W) {
            int nI[4], tI[4];
            bool vI[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = q0 + e;
              nI[e] = 0;
              tI[e] = 0;
              vI[e] = false;
              if (q < P * nb_g) {
                nI[e] = q % nb_g;
                tI[e] = q / nb_g;
                vI[e] = tI[e] < ctl->kb[nI[e]];
              } else if (q < slots) {
                nI[e] = q - P * nb_g;
                tI[e] = ctl->kb[nI[e]];
                vI[e] = tI[e] <= P;
              }
            }
            if (!(vI[0] || vI[1] || vI[2] || vI[3])) continue;  // warp-uniform
            float m[4], sm[4];
            int32_t mi[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              m[e] = -INFINITY;
              sm[e] = 0.f;
              mi[e] = 0x7fffffff;
            }
            for (int p0 = lane; p0 < npieces; p0 += 128) {
              uint4 w[4][4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    target + ((jb0 + nI[e]) * (K + 1) + tI[e]) * V + vslice_lo);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  w[e][u] = (vI[e] && p0 + 32 * u < npieces) ? __ldcg(src + p0 + 32 * u)
                                                             : make_uint4(0, 0, 0, 0);
              }
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int pp = p0 + 32 * u;
                if (pp >= npieces) break;
#pragma unroll
                for (int e = 0; e < 4; ++e)  // unused items reduce zeros (discarded)
                  piece_stats<kG>(w[e][u], vslice_lo + 8 * pp, k, m[e], sm[e], mi[e]);
              }
            }
            // the four items' warp reductions interleaved
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float m2 = __shfl_xor_sync(FULL, m[e], off);
                if constexpr (kG) {
                  const int32_t i2 = __shfl_xor_sync(FULL, mi[e], off);
                  amax_combine(m[e], mi[e], m2, i2);
                } else {
                  const float s2 = __shfl_xor_sync(FULL, sm[e], off);
                  ms_combine(m[e], sm[e], m2, s2, k);
                }
              }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (lane == 0 && vI[e])
                a.tpart[(((int64_t)par * (K + 1) + tI[e]) * N + nI[e]) * kMaxG + cta] =
                    kG ? make_float2(m[e], __int_as_float(mi[e])) : make_float2(m[e], sm[e]);
            }
          }
        };
        if (a.greedy)
          take(std::true_type{});
        else
          take(std::false_type{});
      }
      // step 0's base logits and the target warps' first row of this CTA's
      // slice into L2 (after the loads above, which need the memory first)
      if (tid < nb_g) {
        const int64_t b = jb0 + tid;
        prefetch_l2_bulk(base + b * K * V + vslice_lo, slice_bytes);
        if (a.npro < K) prefetch_l2_bulk(target + (b * (K + 1) + a.npro) * V + vslice_lo, slice_bytes);
      }
      named_sync();
      // the target warps may take positions npro, npro + 1 of this job
      if (tid == 0)
        st_release_cta_smem(&ctl->tgo_cnt, (uint32_t)(t * (K - a.npro) + min(2, K - a.npro)));
      mark(g, K + 1, 1);

      for (int i = 0; i < K; ++i) {
        // ---------------- gather the Markov rows for this step
        mark(g, i, 0);
        for (int n = tid; n < N; n += kComputeThreads) {
          int p = 0;
          if (n < nb_g) {
            p = (i == 0) ? first_token(g * N + n) : ctl->tok[n];
            if (p < 0 || p >= V) {
              record_error(hdr, SPEC_ERR_TOKEN_RANGE, SITE_TOKEN_RANGE, g * N + n, p);
              p = 0;
            }
          }
          ctl->prev[n] = p;
        }
        named_sync();
        gather_u(nb_g, i);
        // the next step's base logits into L2 while this step runs
        if (tid < nb_g && i + 1 < K)
          prefetch_l2_bulk(base + ((jb0 + tid) * K + i + 1) * V + vslice_lo, slice_bytes);
        if (a.Wh && i + 1 < K) {
          // RNN head: this CTA's share of Wh s_i for the next step (fp32 fmaf in
          // ascending k), visible to every CTA after this step's grid barrier
          const int cpr = a.r / 8;
          for (int o = cta * kComputeThreads + tid; o < nb_g * a.r; o += G * kComputeThreads) {
            const int n = o / a.r, j = o % a.r;
            const uint4* wr = reinterpret_cast<const uint4*>(a.Wh + (size_t)j * a.r);
            float acc = 0.f;
            for (int c = 0; c < cpr; ++c) {
              const uint4 sw = *reinterpret_cast<const uint4*>(sU + (size_t)(c >> 3) * N * 128 + n * 128 +
                                                              (((c & 7) ^ (n & 7)) << 4));
              float xs[8], xw[8];
              bf16x8(sw, xs);
              bf16x8(__ldg(wr + c), xw);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc = fmaf(xs[e], xw[e], acc);
            }
            a.P[((size_t)((i + 1) & 1) * N + n) * a.r + j] = acc;
          }
        }
        mark(g, i, 1);

        // ---------------- epilogue: z = bias + base, exact bucket statistics
        {
          // per slab: stochastic (max, sum); greedy arg-max (value, index)
          float pm[NS], ps[NS];
          int32_t pi[NS];
#pragma unroll
          for (int sl = 0; sl < NS; ++sl) {
            pm[sl] = -INFINITY;
            ps[sl] = 0.f;
            pi[sl] = 0x7fffffff;
          }
          uint4 nb[NV];
          auto issue = [&](int cl, int sl) {  // base logits of chunk cl, slab sl, this lane's row
            const int nr = slab_row(sl);
            const bool ok = nr < nb_g;
            const T* bsrc = base + ((jb0 + (ok ? nr : 0)) * K + i) * V;
            const int vv0 = (chunk0 + cl) * kCH + q4 * 32 + tg * SC;
#pragma unroll
            for (int u = 0; u < NV; ++u)
              nb[u] = (ok && vv0 + 8 * u < V) ? __ldcs(reinterpret_cast<const uint4*>(bsrc + vv0 + 8 * u))
                                              : make_uint4(0, 0, 0, 0);
          };
          issue(0, 0);
          for (int cl = 0; cl < ncc; ++cl) {
#pragma unroll
            for (int sl = 0; sl < NS; ++sl) {
              const int nr = slab_row(sl);
              const bool rowok = nr < nb_g;
              uint4 cb[NV];
#pragma unroll
              for (int u = 0; u < NV; ++u) cb[u] = nb[u];
              // the next tile's base logits in flight meanwhile
              if (sl + 1 < NS) issue(cl, sl + 1);
              else if (cl + 1 < ncc) issue(cl + 1, 0);
              float z[SC];
              acc_tile(z, sl);
              const int vv0 = (chunk0 + cl) * kCH + q4 * 32 + tg * SC;
              const bool full = rowok && vv0 + SC <= V;  // every token of this lane is valid
              float x[8];
              if (full) {  // the common case without per-token checks (pairs: packed adds)
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                  bf16x8(cb[u], x);
#pragma unroll
                  for (int e = 0; e < 8; e += 2)
                    f2unpack(f2add(f2pack(z[8 * u + e], z[8 * u + e + 1]), f2pack(x[e], x[e + 1])),
                             z[8 * u + e], z[8 * u + e + 1]);
                }
              } else {
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                  bf16x8(cb[u], x);
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const int ee = 8 * u + e;
                    z[ee] = (rowok && vv0 + ee < V) ? z[ee] + x[e] : -INFINITY;
                  }
                }
              }
              float m = -INFINITY;
              int32_t mi = 0x7fffffff;
              if (a.greedy) {
                // four interleaved arg-max chains (lowest index on ties), then combined
                float mv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                int32_t mx[4] = {0x7fffffff, 0x7fffffff, 0x7fffffff, 0x7fffffff};
#pragma unroll
                for (int ee = 0; ee < SC; ++ee)
                  if (z[ee] > mv[ee & 3]) {
                    mv[ee & 3] = z[ee];
                    mx[ee & 3] = vv0 + ee;
                  }
                m = mv[0];
                mi = mx[0];
#pragma unroll
                for (int c4 = 1; c4 < 4; ++c4) amax_combine(m, mi, mv[c4], mx[c4]);
#pragma unroll
                for (int o = 1; o < L; o <<= 1) {
                  const float m2 = __shfl_xor_sync(FULL, m, o);
                  const int32_t i2 = __shfl_xor_sync(FULL, mi, o);
                  amax_combine(m, mi, m2, i2);
                }
                amax_combine(pm[sl], pi[sl], m, mi);
              } else {
                // four interleaved chains for the max and for the sum (short dependencies)
                float mv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int ee = 0; ee < SC; ++ee) mv[ee & 3] = fmaxf(mv[ee & 3], z[ee]);
                m = fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3]));
                float sum = 0.f;
                if (m > -INFINITY) {
                  // four chains (element ee into chain ee % 4), kept as two packed pairs
                  const float mk = m * k;
                  const uint64_t kk = f2pack(k, k), nmk = f2pack(-mk, -mk);
                  uint64_t s01 = f2pack(0.f, 0.f), s23 = f2pack(0.f, 0.f);
#pragma unroll
                  for (int ee = 0; ee < SC; ee += 4) {
                    float y0, y1, y2, y3;
                    f2unpack(f2fma(f2pack(z[ee], z[ee + 1]), kk, nmk), y0, y1);
                    f2unpack(f2fma(f2pack(z[ee + 2], z[ee + 3]), kk, nmk), y2, y3);
                    s01 = f2add(s01, f2pack(fexp2(y0), fexp2(y1)));
                    s23 = f2add(s23, f2pack(fexp2(y2), fexp2(y3)));
                  }
                  float sv[4];
                  f2unpack(s01, sv[0], sv[1]);
                  f2unpack(s23, sv[2], sv[3]);
                  sum = (sv[0] + sv[1]) + (sv[2] + sv[3]);
                }
#pragma unroll
                for (int o = 1; o < L; o <<= 1) {
                  const float m2 = __shfl_xor_sync(FULL, m, o), s2 = __shfl_xor_sync(FULL, sum, o);
                  ms_combine(m, sum, m2, s2, k);
                }
                if (tg == 0 && rowok)
                  a.gbk[((size_t)cta * a.nbk + cl * 4 + q4) * N + nr] = make_float2(m, sum);
                ms_combine(pm[sl], ps[sl], m, sum, k);
              }
            }
            if (trace && g == 0 && cl < 8) trace[(size_t)i * kTracePhases + 16 + cl] = globaltimer_ns();
          }
#pragma unroll
          for (int sl = 0; sl < NS; ++sl) {
            if (a.greedy)
              put_quadrant(ctl->qa, ctl->qb, pm[sl], __int_as_float(pi[sl]), slab_row(sl));
            else
              put_quadrant(ctl->qa, ctl->qb, pm[sl], ps[sl], slab_row(sl));
          }
        }
        named_sync();
        mark(g, i, 2);
        // ---------------- CTA partials per batch row (quadrants in token order)
        if (tid < N) {
          const int n = tid;
          float m = ctl->qa[0][n], sm = ctl->qb[0][n];
          if (a.greedy) {
            int32_t mi = __float_as_int(sm);
            for (int q = 1; q < 4; ++q) amax_combine(m, mi, ctl->qa[q][n], __float_as_int(ctl->qb[q][n]));
            sm = __int_as_float(mi);
          } else {
            for (int q = 1; q < 4; ++q) ms_combine(m, sm, ctl->qa[q][n], ctl->qb[q][n], k);
          }
          a.dpart[(((int64_t)par * (K + 1) + i) * N + n) * kMaxG + cta] = make_float4(m, sm, m, 0.f);
        }
        // this CTA's target partials of row i (and row K) are out; the target
        // warps may take the next row
        // (positions below npro were taken at the job's start); the target
        // warps may then run up to two positions ahead
        if (tid == 0) {
          const int KT = K - a.npro;  // target-warp positions per job
          if (i >= a.npro) {
            // each target warp has finished this position (a warp may be ahead)
            const uint32_t need = (uint32_t)(t * KT + (i - a.npro) + 1);
            uint64_t it = 0;
            while (ld_acquire_cta_smem(&ctl->tdone_cnt[0]) < need ||
                   ld_acquire_cta_smem(&ctl->tdone_cnt[1]) < need) {
              if (++it >= a.spin || ((it & 63) == 0 && ld_volatile_u32(&hdr->abort))) {
                if (it >= a.spin) record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_BREADY, cta, 5000 + i);
                ctl->abort_local = 1;
                break;
              }
              __nanosleep(32);
            }
          }
          const uint32_t rel = (uint32_t)(t * KT + min(KT, max(2, i + 3 - a.npro)));
          if (KT > 0 && rel > ctl->tgo_cnt) st_release_cta_smem(&ctl->tgo_cnt, rel);
        }
        grid_arrive();
        mark(g, i, 3);
        if (!grid_wait()) {
          failed = true;
          break;
        }
        mark(g, i, 5);
        // ---------------- row reducers draw the token of their rows
        const int mine = reduce_rows(0, g, par, i, nb_g);
        mark(g, i, 12);
        if (a.trace && g == 0 && tid == 0 && mine)
          atomicMax(reinterpret_cast<unsigned long long*>(a.trace) + (size_t)i * kTracePhases + 7,
                    (unsigned long long)globaltimer_ns());
        if (!records_hop(t, par, i, nb_g)) {
          failed = true;
          break;
        }
        // accept outcomes from the tags; a row that stops (or the bonus at the
        // last step) reads its full record for the final step's statistics
        for (int n = tid; n < nb_g; n += kComputeThreads) {
          const bool lastn = i == ctl->kb[n] - 1;
          if (ctl->alive[n] && i < ctl->kb[n] && (!ctl->acc[n] || lastn)) {
            const RecT r = load_rec(a.rec + ((int64_t)par * (K + 1) + i) * N + n);
            if (!ctl->acc[n]) {
              ctl->alive[n] = 0;
              ctl->stoprow[n] = i;
              ctl->zM[n] = r.M;    // draft statistics of the stop row
              ctl->zS[n] = r.S;
              ctl->fMt[n] = r.Mt;  // target statistics of the stop row
              ctl->fSt[n] = r.St;
            } else {
              ctl->fMt[n] = r.MtK;  // every draft accepted: the bonus comes from row K_b
              ctl->fSt[n] = r.StK;
            }
          }
        }
        named_sync();
        mark(g, i, 6);
        if (ctl->abort_local) {  // read after the last named barrier of the step
          failed = true;
          break;
        }
      }  // draft steps
      if (failed) break;

      if (has_final) {
        // ---------------- final step: residual at the stop row, or the bonus.
        mark(g, K, 0);
        for (int n = tid; n < N; n += kComputeThreads) {
          int p = 0;
          if (n < nb_g && !ctl->alive[n]) {
            const int j = ctl->stoprow[n];
            p = j == 0 ? first_token(g * N + n)
                       : __ldcg(a.tokens + ((int64_t)par * K + (j - 1)) * N + n);
            if (p < 0 || p >= V) p = 0;
          }
          ctl->prev[n] = p;
          if (n < nb_g)
            ctl->fcst[n] = make_float4(ctl->fMt[n], 1.f / ctl->fSt[n], ctl->zM[n],
                                       ctl->alive[n] ? 0.f : 1.f / ctl->zS[n]);
        }
        named_sync();
        gather_u(nb_g, K);
        if (tid < nb_g) {  // the final rows of this CTA's slice into L2
          const int64_t b = jb0 + tid;
          const bool alive = ctl->alive[tid] != 0;
          const int row = alive ? ctl->kb[tid] : ctl->stoprow[tid];
          prefetch_l2_bulk(target + (b * (K + 1) + row) * V + vslice_lo, slice_bytes);
          if (!alive) prefetch_l2_bulk(base + (b * K + row) * V + vslice_lo, slice_bytes);
        }
        mark(g, K, 1);
        {
          float Rs[NS], Ps[NS];
#pragma unroll
          for (int sl = 0; sl < NS; ++sl) Rs[sl] = Ps[sl] = 0.f;
          uint4 nt[NV], nb[NV];
          // the stop row's (or bonus row's) target logits and, for stopped rows,
          // the draft base of that row: chunk cl, slab sl, this lane's row
          auto issue = [&](int cl, int sl) {
            const int nr = slab_row(sl);
            const bool rowok = nr < nb_g;
            const bool ralive = rowok && ctl->alive[nr] != 0;
            const int frow = ralive ? ctl->kb[nr] : (rowok ? ctl->stoprow[nr] : 0);
            const int64_t brow = jb0 + (rowok ? nr : 0);
            const T* tsrc = target + (brow * (K + 1) + frow) * V;
            const T* bsrc = base + (brow * K + min(frow, K - 1)) * V;
            const int vv0 = (chunk0 + cl) * kCH + q4 * 32 + tg * SC;
#pragma unroll
            for (int u = 0; u < NV; ++u) {
              const int vv = vv0 + 8 * u;
              const bool ok = rowok && vv < V;
              nt[u] = ok ? __ldcs(reinterpret_cast<const uint4*>(tsrc + vv)) : make_uint4(0, 0, 0, 0);
              nb[u] = (ok && !ralive) ? __ldcs(reinterpret_cast<const uint4*>(bsrc + vv))
                                      : make_uint4(0, 0, 0, 0);
            }
          };
          issue(0, 0);
          for (int cl = 0; cl < ncc; ++cl) {
#pragma unroll
            for (int sl = 0; sl < NS; ++sl) {
              const int nr = slab_row(sl);
              const bool rowok = nr < nb_g;
              const float4 c = rowok ? ctl->fcst[nr] : make_float4(0.f, 0.f, 0.f, 0.f);
              uint4 ct[NV], cb[NV];
#pragma unroll
              for (int u = 0; u < NV; ++u) {
                ct[u] = nt[u];
                cb[u] = nb[u];
              }
              if (sl + 1 < NS) issue(cl, sl + 1);  // the next tile's logits in flight meanwhile
              else if (cl + 1 < ncc) issue(cl + 1, 0);
              float z[SC];
              acc_tile(z, sl);  // the bias at the stop row (alive rows: unused)
              const int vv0 = (chunk0 + cl) * kCH + q4 * 32 + tg * SC;
              const bool any = rowok && vv0 < V;
              float r = 0.f, p = 0.f;
              float xt[8], xb[8];
              // residual mass and target mass; a row that accepted every draft
              // has 1 / draft sum = 0: r = p (the checks are hoisted out of the
              // common cases; the expressions are the same in every branch)
              if (any && vv0 + SC <= V && c.w != 0.f) {
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                  bf16x8(ct[u], xt);
                  bf16x8(cb[u], xb);
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const float pe = fexp2((xt[e] - c.x) * k) * c.y;
                    const float qe = fexp2((z[8 * u + e] + xb[e] - c.z) * k) * c.w;
                    r += fmaxf(pe - qe, 0.f);
                    p += pe;
                  }
                }
              } else if (any && vv0 + SC <= V) {
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                  bf16x8(ct[u], xt);
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const float pe = fexp2((xt[e] - c.x) * k) * c.y;
                    r += pe;  // fmaxf(pe - 0, 0) = pe
                    p += pe;
                  }
                }
              } else {
#pragma unroll
                for (int u = 0; u < NV; ++u) {
                  bf16x8(ct[u], xt);
                  bf16x8(cb[u], xb);
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const bool ok = any && vv0 + 8 * u + e < V;
                    const float pe = fexp2((xt[e] - c.x) * k) * c.y;
                    const float qe = c.w != 0.f ? fexp2((z[8 * u + e] + xb[e] - c.z) * k) * c.w : 0.f;
                    r += ok ? fmaxf(pe - qe, 0.f) : 0.f;
                    p += ok ? pe : 0.f;
                  }
                }
              }
#pragma unroll
              for (int o = 1; o < L; o <<= 1) {
                r += __shfl_xor_sync(FULL, r, o);
                p += __shfl_xor_sync(FULL, p, o);
              }
              if (tg == 0 && rowok)
                a.gbk[((size_t)cta * a.nbk + cl * 4 + q4) * N + nr] = make_float2(r, p);
              Rs[sl] += r;
              Ps[sl] += p;
            }
            if (trace && g == 0 && cl < 8) trace[(size_t)K * kTracePhases + 16 + cl] = globaltimer_ns();
          }
#pragma unroll
          for (int sl = 0; sl < NS; ++sl) put_quadrant(ctl->qa, ctl->qb, Rs[sl], Ps[sl], slab_row(sl));
        }
        named_sync();
        mark(g, K, 2);
        if (tid < N) {
          const int n = tid;
          const float R = (ctl->qa[0][n] + ctl->qa[1][n]) + (ctl->qa[2][n] + ctl->qa[3][n]);
          const float P = (ctl->qb[0][n] + ctl->qb[1][n]) + (ctl->qb[2][n] + ctl->qb[3][n]);
          a.dpart[(((int64_t)par * (K + 1) + K) * N + n) * kMaxG + cta] = make_float4(R, P, 0.f, 0.f);
        }
        grid_arrive();
        mark(g, K, 3);
        if (!grid_wait()) {
          failed = true;
          break;
        }
        mark(g, K, 4);
        // the reducers draw each row's residual / bonus token and write it
        reduce_rows(2, g, par, K, nb_g);
        // the next job overwrites the bucket statistics, and the next cycle
        // starts from the tokens drawn here: every draw is done first
        if (t + 1 < njobs && !records_hop(t, par, K, nb_g)) {
          failed = true;
          break;
        }
        mark(g, K, 5);
      }
      // tau and the -1 padding after it
      if (cta == 0) {
        for (int n = tid; n < nb_g; n += kComputeThreads) {
          const int64_t b = jb0 + n;
          const int j = ctl->alive[n] ? ctl->kb[n] : ctl->stoprow[n];
          a.tau[b] = j + 1;
          for (int i2 = j + 1; i2 <= K; ++i2) a.out[b * (K + 1) + i2] = -1;
        }
      }
      named_sync();
      mark(g, K, 6);
      if (ctl->abort_local) failed = true;
    }  // jobs
    (void)soft_fail;
  }

  // =========================================================================
  // exit: all roles meet, tensor memory is released, the last CTA resets the
  // launch counters so the next launch on this workspace starts from zero.
  // =========================================================================
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(taddr, 512);
  }
  if (tid == 0) {
    __threadfence();
    const uint32_t prior = atomicAdd(&hdr->exit_count, 1u);
    if (prior == (uint32_t)G - 1) {
      __threadfence();
      hdr->bar = 0;
      hdr->rec = 0;
      hdr->abort = 0;
      hdr->events += (uint32_t)(njobs * (K + 1));  // tags of the next launch differ
      __threadfence();
      atomicExch(&hdr->exit_count, 0u);
    }
  }
}

constexpr size_t kSmemBudget = 227 * 1024;

// Shared memory without the target rings, and the ring slots that fit beside it.
template <int N>
size_t smem_fixed_tc(int r) {
  constexpr int NCOL = N / 2;
  constexpr int SC = NCOL > 32 ? 32 : NCOL;
  size_t s = 1024;  // alignment slack
  s += (size_t)kNSof<N> * kWStage;
  s += (size_t)(r / 64) * N * 128;
  s += (size_t)8 * 32 * SC * sizeof(float);
  s += sizeof(CtlT<N>);
  return s;
}
template <int N>
int ring_slots_tc(int r, int nc) {
  const size_t fixed = smem_fixed_tc<N>(r);
  const size_t rslot = (size_t)nc * kCH * sizeof(__nv_bfloat16);
  if (fixed + 2 * rslot > kSmemBudget) return 0;
  return (int)std::min<size_t>(kTSMax, (kSmemBudget - fixed) / (2 * rslot));
}
template <int N>
size_t smem_bytes_tc(int r, int nc) {
  return smem_fixed_tc<N>(r) + (size_t)2 * ring_slots_tc<N>(r, nc) * nc * kCH * sizeof(__nv_bfloat16);
}

template <int N>
cudaError_t launch_tc(const ArgsTC& args, int G, size_t smem, cudaStream_t st) {
  auto fn = k_cycle_tc<N>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  void* params[] = {const_cast<ArgsTC*>(&args)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(fn), dim3(G), dim3(kThreads),
                                     params, smem, st);
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }
size_t dpart_bytes(int K, int N) { return a256(sizeof(float4) * 2 * (size_t)(K + 1) * N * kMaxG); }
size_t tpart_bytes(int K, int N) { return a256(sizeof(float2) * 2 * (size_t)(K + 1) * N * kMaxG); }
size_t tok_bytes(int K, int N) { return a256(sizeof(int32_t) * 2 * (size_t)K * N); }
size_t rec_bytes(int K, int N) { return a256(sizeof(RecT) * 2 * (size_t)(K + 1) * N); }
size_t rtag_bytes(int K, int N) { return a256(sizeof(uint64_t) * 2 * (size_t)(K + 1) * N); }
size_t gbk_bytes(const CycleGeom& g) { return a256(sizeof(float2) * (size_t)g.G * g.nc * 4 * g.N); }
size_t rnn_p_bytes(int N, int r) { return a256(sizeof(float) * 2 * (size_t)N * r); }
size_t rnn_hist_bytes(int K, int N, int r) { return a256(sizeof(__nv_bfloat16) * (size_t)K * N * r); }

}  // namespace

bool cycle_tc_geometry(int B, int K, int V, int r, int dtype, uint32_t flags, int num_sms,
                       CycleGeom* g, const char** why) {
  if (dtype != SPEC_BF16 || r <= 0 || r % 64 != 0 || r > 256 || (flags & SPEC_FLAG_FMA_BIAS)) {
    *why = "not the tensor-core path";
    return false;
  }
  const int nchunks = (V + kCH - 1) / kCH;
  const int nc = (nchunks + num_sms - 1) / num_sms;
  g->nchunks = nchunks;
  g->nc = nc;
  g->G = (nchunks + nc - 1) / nc;
  if (g->G > kMaxG) {
    *why = "more CTAs than the kernel's partial buffers allow";
    return false;
  }
  g->N = B > 64 ? 128 : (B > 32 ? 64 : (B > 16 ? 32 : 16));
  g->tc = true;
  g->smem = g->N == 128 ? smem_bytes_tc<128>(r, nc)
          : g->N == 64 ? smem_bytes_tc<64>(r, nc)
                        : (g->N == 32 ? smem_bytes_tc<32>(r, nc) : smem_bytes_tc<16>(r, nc));
  const int nts = g->N == 128 ? ring_slots_tc<128>(r, nc)
                : g->N == 64 ? ring_slots_tc<64>(r, nc)
                             : (g->N == 32 ? ring_slots_tc<32>(r, nc) : ring_slots_tc<16>(r, nc));
  if (nts < 2 || g->smem > kSmemBudget) {
    *why = "shared memory budget exceeded";
    return false;
  }
  (void)K;
  return true;
}

size_t cycle_tc_ws_bytes(int K, int r, const CycleGeom& g) {
  return cycle_trace_bytes(K) + dpart_bytes(K, g.N) + tpart_bytes(K, g.N) + tok_bytes(K, g.N) +
         rec_bytes(K, g.N) + rtag_bytes(K, g.N) + gbk_bytes(g) + rnn_p_bytes(g.N, r) +
         rnn_hist_bytes(K, g.N, r);
}

cudaError_t launch_cycle_tc(const CycleLaunch& L, const CycleGeom& g, WsHeader* hdr, uint8_t* body,
                            const CUtensorMap* tmW, cudaStream_t st) {
  ArgsTC a;
  memset(&a, 0, sizeof(a));
  a.tmW = *tmW;
  a.base = reinterpret_cast<const __nv_bfloat16*>(L.base);
  a.target = reinterpret_cast<const __nv_bfloat16*>(L.target);
  a.U = reinterpret_cast<const __nv_bfloat16*>(L.U);
  a.W = reinterpret_cast<const __nv_bfloat16*>(L.W);
  a.last_token = L.last_token;
  a.vlen = L.vlen;
  a.conf = L.conf;
  a.next_token = L.next_token;
  a.Wh = reinterpret_cast<const __nv_bfloat16*>(L.Wh);
  a.draft = L.draft;
  a.out = L.out;
  a.tau = L.tau;
  a.p_draft = L.p_draft;
  a.q_draft = L.q_draft;
  a.hdr = hdr;
  a.trace = L.trace ? reinterpret_cast<uint64_t*>(body) : nullptr;
  body += cycle_trace_bytes(L.K);
  a.dpart = reinterpret_cast<float4*>(body);
  body += dpart_bytes(L.K, g.N);
  a.tpart = reinterpret_cast<float2*>(body);
  body += tpart_bytes(L.K, g.N);
  a.tokens = reinterpret_cast<int32_t*>(body);
  body += tok_bytes(L.K, g.N);
  a.rec = reinterpret_cast<RecT*>(body);
  body += rec_bytes(L.K, g.N);
  a.rtag = reinterpret_cast<uint64_t*>(body);
  body += rtag_bytes(L.K, g.N);
  a.gbk = reinterpret_cast<float2*>(body);
  body += gbk_bytes(g);
  a.P = reinterpret_cast<float*>(body);
  body += rnn_p_bytes(g.N, L.r);
  a.shist = reinterpret_cast<__nv_bfloat16*>(body);
  a.nbk = g.nc * 4;
  // target statistics of the first positions taken by the compute warps at a
  // job's start: two; three for long blocks of 128-row groups, whose first
  // target jobs (128 row slices each) otherwise gate several steps
  a.npro = std::min(g.N == 128 && L.K >= 16 ? 3 : 2, L.K);
  a.nts = g.N == 128 ? ring_slots_tc<128>(L.r, g.nc)
        : g.N == 64 ? ring_slots_tc<64>(L.r, g.nc)
                    : (g.N == 32 ? ring_slots_tc<32>(L.r, g.nc) : ring_slots_tc<16>(L.r, g.nc));
  a.B = L.B;
  a.K = L.K;
  a.V = L.V;
  a.r = L.r;
  a.G = g.G;
  a.nc = g.nc;
  a.nchunks = g.nchunks;
  a.greedy = L.greedy;
  a.ngroups = (L.B + g.N - 1) / g.N;
  a.NT = std::min(std::min(kMaxNT, g.nc), (512 - 2 * g.N) / 128);  // TMEM: accumulators first
  a.k = L.greedy ? 1.0f : 1.4426950408889634f / L.temperature;
  a.conf_thr = L.conf_thr;
  a.ncyc = std::max(L.ncyc, 1);
  a.seed = L.seed;
  a.row0 = L.row0;
  a.cycle = L.cycle;
  a.spin = L.spin;
  switch (g.N) {
    case 16: return launch_tc<16>(a, g.G, g.smem, st);
    case 32: return launch_tc<32>(a, g.G, g.smem, st);
    case 64: return launch_tc<64>(a, g.G, g.smem, st);
    default: return launch_tc<128>(a, g.G, g.smem, st);
  }
}

}  // namespace specdec
