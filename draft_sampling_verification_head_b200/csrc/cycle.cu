// Fused persistent draft-sample-and-verify kernel.
//
// Method (aigest.pl "DeepSeek prezentuje DSpark"; mkdocs.reaper.mx
// DeepSeek-V4.1-Flash "06-extensions", DSpark table):
//   "Innowacje w tworzeniu tokenów": base logits from the parallel core plus a
//   prefix-dependent Markov bias U[prev] . W added before each of the K draft
//   tokens is sampled -- K sequential steps, step i needing d_{i-1};
//   "Jak działa spekulatywne dekodowanie DSpark?": the longest accepted prefix
//   plus one extra token, target distribution preserved exactly.
//
// Design (one launch, one CTA per SM, cooperative so all CTAs are resident):
//  * The vocabulary is cut into 128-token chunks; CTA c owns nc consecutive
//    chunks for the whole launch.  Batch rows are processed in groups of N
//    (16/32/64) = the tcgen05 N dimension.  Warps: 8 compute warps, a W TMA
//    producer, the MMA issuer and a base-tile producer.
//  * Per draft step, per chunk: D[v, b] = W^T[v, :] . U[prev_b]^T + base[b, v]
//    is one tcgen05.mma chain into tensor memory (M = 128 tokens, N batch rows,
//    K = r, then N more K-rows that add the base tile against an identity):
//    W^T streams through a TMA ring (128-byte swizzle, L2 evict-last), the
//    gathered U rows form the swizzled K-major B operand, the base tile
//    arrives by TMA.  Meanwhile the compute warps take the target row's
//    statistics over the CTA's slice.
//  * The epilogue reduces softmax statistics of z / T per 32-token bucket with
//    a transposing butterfly (one exp2 per element; from step 1 on as plain
//    sums against the previous step's max), publishes them per bucket and per
//    CTA, and meets the other CTAs at a grid barrier.
//  * Row n's reducer (CTA n mod G) combines the per-CTA partials in ascending
//    token order, finds the CTA and then the bucket holding the inverse-CDF
//    target, forms that bucket's 32 logits from the bf16 inputs with the whole
//    CTA, scans them, runs the accept test with p_i(d_i) / q_i(d_i) and writes
//    the outputs and a 48-byte record; a counter hands the records to every
//    CTA.  Greedy steps take the arg-max instead.
//  * Verification runs on the fly (early exit: a row's target rows are never
//    read past its first rejection).  A last step recomputes the bias at each
//    row's stop position, gathers the stop rows' logits and draws the residual
//    max(p - q, 0) (or the bonus from target row K) the same way.
//  * Every wait is bounded (spin limit); a CTA that gives up records
//    SPEC_ERR_TIMEOUT in the workspace, the others notice and all exit.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace specdec {

namespace {

constexpr int kCH = 128;            // tokens per chunk (UMMA M)
constexpr int kComputeThreads = 256;
constexpr int kThreads = 352;       // 8 compute warps + W producer + MMA + base producer
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kBaseWarp = 10;
constexpr int kNS = 6;              // W ring stages
constexpr int kNBS = 4;             // base tile ring stages
constexpr int kIL = 1;              // chunks whose MMA chains are interleaved
constexpr int kMaxNC = 32;
// One W ring stage = kKS MMA K-steps (16 rank rows each) of up to kIL
// chunks: per chunk and K-step two 64-token halves of [16 rows][128 B],
// 128-byte swizzled.
constexpr int kKS = 4 / kIL;                     // K-steps per stage
constexpr int kWChunk = kCH * 16 * 2;            // 4 KB per chunk and K-step
constexpr int kWStage = kIL * kKS * kWChunk;     // 16 KB
constexpr int kMaxG = 160;          // CTAs a launch may use (>= SM count); partial-row stride
constexpr unsigned FULL = 0xffffffffu;

struct Args {
  CUtensorMap tmW;
  CUtensorMap tmBase;
  const void* base;
  const void* target;
  const void* U;
  const void* W;
  const int32_t* last_token;
  int32_t* draft;
  int32_t* out;
  int32_t* tau;
  float* p_draft;
  float* q_draft;
  float* biased_out;
  WsHeader* hdr;
  float4* dpart;     // [2][K+1][N][kMaxG]: (m, s, true max, 0) or (max, idx, max, 0)
  float2* tpart;     // [2][K+1][N][kMaxG]: (m, s) or (max, idx)
  int32_t* tokens;   // [2][K][N]
  struct Rec* rec;   // [2][K+2][N] row records
  float2* gbk;       // [G][nbk][N] this step's bucket statistics of every CTA
  uint64_t* trace;   // [K+2][kTracePhases] device timeline of CTA 0, or null
  int B, K, V, r, G, nc, nchunks, mode, greedy, ngroups;
  float k;           // log2(e) / T (1 in greedy mode)
  uint64_t seed, cycle, spin;
  uint32_t row0;  // global index of batch row 0 (Philox counter word 1)
  int nbk;        // buckets per CTA (4 per chunk)
};

// One record per batch row and reduction, written by the row's reducer.
struct alignas(16) Rec {
  float M, S;       // scale (reference) and total of the draw's distribution
  float Mx;         // true max of z this step (the next step's reference)
  float Mt, St;     // target row statistics
  float trem;       // inverse-CDF target inside the owner CTA's slice (inf: last mass)
  int32_t owner;    // CTA that owns the draw
  int32_t token;    // draft token of the step (drawn, or the arg-max)
  int32_t acc;      // accept outcome
  int32_t flags;    // bit 0: redo the step exactly; bit 1: final draw uses p
  int32_t tam;      // greedy: target arg-max
  int32_t pad;
};
static_assert(sizeof(Rec) == 48, "records are three 16-byte words");

template <int N>
struct Ctl {
  uint64_t wfull[kNS], wempty[kNS], bfull[kNBS], bempty[kNBS], dfull[kMaxNC];
  uint64_t bready, tfree, mmadone;
  uint64_t ring_free;  // the final step no longer needs the base ring slots
  uint32_t tmem_slot;
  int32_t abort_local;
  int32_t prev[N];
  int32_t alive[N];
  int32_t stoprow[N];
  int32_t tok[N];
  float M[N], S[N];     // global draft stats of the current step
  float zM[N], zS[N];   // draft stats of the stop row
  float Mt[N], St[N];   // target stats of row i during a step
  float fMt[N], fSt[N]; // target stats of the final row (stop row or row K)
  alignas(16) float ref[N];  // per-row reference of the fast path (previous step's max)
  float cmax[4][N];     // true max per row and tensor-memory quadrant
  float psum[4][N];     // fast path: this CTA's sum per row and tensor-memory quadrant
  alignas(16) float4 fcst[N];  // final step per row: target max, 1 / target sum, draft max, 1 / draft sum
  int32_t redo;
  Rec rrec[N];          // records of the rows this CTA reduces, before publication
  float zpart[8][32];   // per-warp partial Markov biases of a draw's 32 tokens
  int32_t dbk;          // the draw's bucket inside the owner CTA
  float dtin;           // inverse-CDF target inside that bucket
};



SPEC_DEV void store_rec(Rec* dst, const Rec& r) {
  const float4* s4 = reinterpret_cast<const float4*>(&r);
  float4* d4 = reinterpret_cast<float4*>(dst);
  d4[0] = s4[0];
  d4[1] = s4[1];
  d4[2] = s4[2];
}
SPEC_DEV Rec load_rec(const Rec* src) {
  Rec r;
  float4* d4 = reinterpret_cast<float4*>(&r);
  const float4* s4 = reinterpret_cast<const float4*>(src);
  d4[0] = __ldcg(s4);
  d4[1] = __ldcg(s4 + 1);
  d4[2] = __ldcg(s4 + 2);
  return r;
}

// Shared region of the MMA's U operand: tensor cores, bf16 rows in 64-wide
// k-blocks; otherwise fp32 rows.
template <typename T, bool TC, int N>
__host__ __device__ inline size_t u_region_bytes(int r) {
  return TC ? (size_t)(r / 64) * N * 128 : (size_t)N * r * 4;
}

// Shared region for the CTA's per-bucket statistics of one step.
__host__ __device__ inline size_t bucket_region_bytes(int nc, int N) {
  return (size_t)nc * 4 * N * sizeof(float2);
}

SPEC_DEV void named_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Eight consecutive logits as raw 16-byte loads (streaming, L1 bypass).
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 a;
};
template <>
struct Raw8<float> {
  float4 a, b;
};
SPEC_DEV Raw8<__nv_bfloat16> raw_load(const __nv_bfloat16* p) {
  return Raw8<__nv_bfloat16>{__ldcs(reinterpret_cast<const uint4*>(p))};
}
SPEC_DEV Raw8<float> raw_load(const float* p) {
  return Raw8<float>{__ldcs(reinterpret_cast<const float4*>(p)),
                     __ldcs(reinterpret_cast<const float4*>(p) + 1)};
}
SPEC_DEV void raw_expand(const Raw8<__nv_bfloat16>& r, float* x) {
  const uint32_t w[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(w[j] << 16);
    x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}
SPEC_DEV void raw_expand(const Raw8<float>& r, float* x) {
  x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
  x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
}

template <typename T>
SPEC_DEV float to_f(T x);
template <>
SPEC_DEV float to_f<float>(float x) {
  return x;
}
template <>
SPEC_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// ---- transposing butterflies: NCOL column values per lane -> lane L holds
// column (L >> (5 - log2 NCOL)) reduced over all 32 lanes in element 0.
template <int NCOL>
SPEC_DEV void bfly_ms(float (&m)[NCOL], float (&s)[NCOL], float k, int lane) {
#pragma unroll
  for (int h = NCOL / 2, off = 16; h >= 1; h >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float sm = up ? m[j] : m[j + h], ss = up ? s[j] : s[j + h];
      float km = up ? m[j + h] : m[j], ks = up ? s[j + h] : s[j];
      const float rm = __shfl_xor_sync(FULL, sm, off), rs = __shfl_xor_sync(FULL, ss, off);
      ms_combine(km, ks, rm, rs, k);
      m[j] = km;
      s[j] = ks;
    }
  }
#pragma unroll
  for (int off = 16 / NCOL; off >= 1; off >>= 1) {
    const float rm = __shfl_xor_sync(FULL, m[0], off), rs = __shfl_xor_sync(FULL, s[0], off);
    ms_combine(m[0], s[0], rm, rs, k);
  }
}

template <int NCOL>
SPEC_DEV void bfly_amax(float (&m)[NCOL], int32_t (&ix)[NCOL], int lane) {
#pragma unroll
  for (int h = NCOL / 2, off = 16; h >= 1; h >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float sm = up ? m[j] : m[j + h];
      const int32_t si = up ? ix[j] : ix[j + h];
      float km = up ? m[j + h] : m[j];
      int32_t ki = up ? ix[j + h] : ix[j];
      const float rm = __shfl_xor_sync(FULL, sm, off);
      const int32_t ri = __shfl_xor_sync(FULL, si, off);
      amax_combine(km, ki, rm, ri);
      m[j] = km;
      ix[j] = ki;
    }
  }
#pragma unroll
  for (int off = 16 / NCOL; off >= 1; off >>= 1) {
    const float rm = __shfl_xor_sync(FULL, m[0], off);
    const int32_t ri = __shfl_xor_sync(FULL, ix[0], off);
    amax_combine(m[0], ix[0], rm, ri);
  }
}

template <int NCOL>
SPEC_DEV void bfly_sum2(float (&a)[NCOL], float (&c)[NCOL], int lane) {
#pragma unroll
  for (int h = NCOL / 2, off = 16; h >= 1; h >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float sa = up ? a[j] : a[j + h], sc = up ? c[j] : c[j + h];
      const float ka = up ? a[j + h] : a[j], kc = up ? c[j + h] : c[j];
      a[j] = ka + __shfl_xor_sync(FULL, sa, off);
      c[j] = kc + __shfl_xor_sync(FULL, sc, off);
    }
  }
#pragma unroll
  for (int off = 16 / NCOL; off >= 1; off >>= 1) {
    a[0] += __shfl_xor_sync(FULL, a[0], off);
    c[0] += __shfl_xor_sync(FULL, c[0], off);
  }
}

template <int NCOL>
SPEC_DEV void bfly_sum1(float (&a)[NCOL], int lane) {
#pragma unroll
  for (int h = NCOL / 2, off = 16; h >= 1; h >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float sa = up ? a[j] : a[j + h];
      const float ka = up ? a[j + h] : a[j];
      a[j] = ka + __shfl_xor_sync(FULL, sa, off);
    }
  }
#pragma unroll
  for (int off = 16 / NCOL; off >= 1; off >>= 1) a[0] += __shfl_xor_sync(FULL, a[0], off);
}

template <int NCOL>
SPEC_DEV void bfly_max1(float (&a)[NCOL], int lane) {
#pragma unroll
  for (int h = NCOL / 2, off = 16; h >= 1; h >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const float sa = up ? a[j] : a[j + h];
      const float ka = up ? a[j + h] : a[j];
      a[j] = fmaxf(ka, __shfl_xor_sync(FULL, sa, off));
    }
  }
#pragma unroll
  for (int off = 16 / NCOL; off >= 1; off >>= 1) a[0] = fmaxf(a[0], __shfl_xor_sync(FULL, a[0], off));
}

// tcgen05.ld of NCOL consecutive columns (NCOL multiple of 8)
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
template <int NCOL>
SPEC_DEV void tmem_st_cols(uint32_t taddr, const float (&v)[NCOL]) {
  if constexpr (NCOL % 16 == 0) {
#pragma unroll
    for (int c = 0; c < NCOL / 16; ++c) tmem_st16(taddr + c * 16, v + c * 16);
  } else {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
        : "memory");
  }
  tmem_st_wait();
}

template <typename T>
SPEC_DEV float ld_elem(const T* p, int64_t i) {
  return to_f<T>(p[i]);
}

// ---------------------------------------------------------------------------
template <typename T, bool TC, int N>
__global__ void __launch_bounds__(kThreads, 1) k_cycle(const __grid_constant__ Args a) {
  constexpr int NCOL = N / 2;        // columns per compute warp
  constexpr int TPB = kComputeThreads / N;  // threads per batch row in the combine phases
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int nkb = a.r / 64;
  uint8_t* sW = smem;                                               // TC: kNS x 16 KB
  uint8_t* sU = sW + (TC ? (size_t)kNS * kWStage : 0);              // TC: nkb x N x 128 B
  float* sUf = reinterpret_cast<float*>(sU);                        // FMA: N x r floats
  const size_t u_bytes = u_region_bytes<T, TC, N>(a.r);
  // TC: N x N identity (B operand, K-major, 128-byte swizzle) that makes the
  // MMA add each base tile to the bias
  uint8_t* sI = sU + ((u_bytes + 1023) & ~size_t(1023));
  T* sBase = reinterpret_cast<T*>(sI + (TC ? (size_t)N * 128 : 0));  // kNBS x N x 128 tokens
  const size_t base_bytes = (size_t)kNBS * N * kCH * sizeof(T);
  float2* sBucket = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(sBase) + base_bytes);
  Ctl<N>* ctl = reinterpret_cast<Ctl<N>*>(reinterpret_cast<uint8_t*>(sBucket) +
                                          bucket_region_bytes(a.nc, N));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  const int G = a.G, K = a.K, V = a.V;
  const int chunk0 = cta * a.nc;
  const int ncc = min(a.nc, a.nchunks - chunk0);  // chunks owned by this CTA
  const int has_final = (a.mode == MODE_CYCLE && !a.greedy) ? 1 : 0;
  const int nsteps = K + has_final;  // MMA steps per group
  WsHeader* hdr = a.hdr;
  const T* base = reinterpret_cast<const T*>(a.base);
  const T* target = reinterpret_cast<const T*>(a.target);
  const T* Ug = reinterpret_cast<const T*>(a.U);
  const T* Wg = reinterpret_cast<const T*>(a.W);
  const float k = a.k;
  const uint32_t ncols = [&] {
    uint32_t c = 32;
    while (c < (uint32_t)(a.nc * N)) c <<= 1;
    return c;
  }();

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&ctl->wfull[i], 1);
      mbar_init(&ctl->wempty[i], 1);
    }
    for (int i = 0; i < kNBS; ++i) {
      mbar_init(&ctl->bfull[i], 1);
      mbar_init(&ctl->bempty[i], TC ? 1 : kComputeThreads / 32);  // TC: freed by the MMA
    }
    for (int i = 0; i < kMaxNC; ++i) mbar_init(&ctl->dfull[i], 1);
    mbar_init(&ctl->ring_free, 1);
    mbar_init(&ctl->bready, 1);
    mbar_init(&ctl->tfree, 1);
    mbar_init(&ctl->mmadone, 1);
    ctl->abort_local = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&ctl->tmem_slot, ncols);
    tmem_relinquish();
  }
  if (TC) {  // identity I[n][k] = (n == k), k < 64, rows of 128 bytes, 16-byte chunks swizzled
    for (int idx = tid; idx < N * 64; idx += kThreads) {
      const int n = idx >> 6, kk = idx & 63;
      reinterpret_cast<__nv_bfloat16*>(sI + n * 128 + (((kk >> 3) ^ (n & 7)) << 4))[kk & 7] =
          __float2bfloat16(n == kk ? 1.f : 0.f);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = ctl->tmem_slot;

  // =========================================================================
  // TMA producers, each in its own consumption order: the W ring (tensor-core
  // path) on one warp, the base logit tiles on another, so neither stream
  // waits behind the other.
  // =========================================================================
  if (warp == kProducerWarp) {
    if (TC && lane == 0) {
      const uint64_t polW = policy_evict_last();
      tma_prefetch_desc(&a.tmW);
      uint32_t Lw = 0;
      bool ok = true;
      for (int g = 0; g < a.ngroups && ok; ++g) {
        for (int s = 0; s < nsteps && ok; ++s) {
          // stages in the MMA's order: K-step by K-step over kIL chunks at a time
          for (int c0 = 0; c0 < ncc && ok; c0 += kIL) {
            const int nil = min(kIL, ncc - c0);
            for (int ks0 = 0; ks0 < nkb * 4; ks0 += kKS) {
              const uint32_t slot = Lw % kNS;
              if (Lw >= kNS &&
                  !mbar_wait_bounded(&ctl->wempty[slot], ((Lw / kNS) - 1) & 1, a.spin,
                                     &hdr->abort)) {
                record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, 100 + s);
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&ctl->wfull[slot], (uint32_t)(nil * kKS * kWChunk));
              for (int j = 0; j < kKS; ++j)
                for (int c = 0; c < nil; ++c) {
                  const int v0 = (chunk0 + c0 + c) * kCH;
                  uint8_t* dst = sW + (size_t)slot * kWStage + (size_t)(j * kIL + c) * kWChunk;
                  tma_load_2d(dst, &a.tmW, &ctl->wfull[slot], v0, (ks0 + j) * 16, polW);
                  tma_load_2d(dst + kWChunk / 2, &a.tmW, &ctl->wfull[slot], v0 + 64,
                              (ks0 + j) * 16, polW);
                }
              ++Lw;
            }
          }
        }
      }
      // drain: the most recent load on every slot must have landed
      for (uint32_t L = (Lw > kNS ? Lw - kNS : 0); L < Lw; ++L)
        mbar_drain(&ctl->wfull[L % kNS], (L / kNS) & 1);
    }
  } else if (warp == kBaseWarp) {
    // Draft steps: one base tile [N rows x 128 tokens] per chunk and step, by
    // lane 0 through the tensor map.  (The final step's stop-row tiles are
    // gathered into the same slots by the compute warps.)
    const uint64_t polB = policy_evict_first();
    if (lane == 0) tma_prefetch_desc(&a.tmBase);
    uint32_t Lb = 0;
    int ok = 1;
    auto wait0 = [&](uint64_t* bar, uint32_t parity, int where) {  // lane 0 waits, all learn
      int r = 1;
      if (lane == 0 && !mbar_wait_bounded(bar, parity, a.spin, &hdr->abort)) {
        record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_BASE, cta, where);
        r = 0;
      }
      return __shfl_sync(FULL, r, 0);
    };
    for (int g = 0; g < a.ngroups && ok; ++g) {
      // the previous group's final step gathers its stop rows into these
      // slots: start this group's tiles once it has finished with them
      if (g > 0 && has_final) ok = wait0(&ctl->ring_free, (uint32_t)(g - 1) & 1, 2000 + g);
      for (int s = 0; s < K && ok; ++s) {
        for (int cl = 0; cl < ncc && ok; ++cl) {
          const uint32_t slot = Lb % kNBS;
          if (Lb >= kNBS) ok = wait0(&ctl->bempty[slot], ((Lb / kNBS) - 1) & 1, s);
          if (!ok) break;
          if (lane == 0) {
            mbar_arrive_expect_tx(&ctl->bfull[slot], (uint32_t)(N * kCH * sizeof(T)));
            if (TC) {  // [N][64] per half: tokens 0..63, then 64..127
              tma_load_3d(sBase + (size_t)slot * N * kCH, &a.tmBase, &ctl->bfull[slot],
                          (chunk0 + cl) * kCH, s, g * N, polB);
              tma_load_3d(sBase + (size_t)slot * N * kCH + N * 64, &a.tmBase,
                          &ctl->bfull[slot], (chunk0 + cl) * kCH + 64, s, g * N, polB);
            } else {
              tma_load_3d(sBase + (size_t)slot * N * kCH, &a.tmBase, &ctl->bfull[slot],
                          (chunk0 + cl) * kCH, s, g * N, polB);
            }
          }
          ++Lb;
        }
      }
    }
    // nothing in flight at exit: the latest copy into every slot has landed
    if (lane == 0) {
      for (uint32_t L = (Lb > kNBS ? Lb - kNBS : 0); L < Lb; ++L)
        mbar_drain(&ctl->bfull[L % kNBS], (L / kNBS) & 1);
    }
  }
  // =========================================================================
  // MMA issuer (tensor-core path)
  // =========================================================================
  else if (warp == kMmaWarp) {
    if (TC && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, N, /*a_mn_major=*/true, /*b_mn_major=*/false);
      uint32_t Lw = 0, Lb = 0, step_ctr = 0;
      bool ok = true;
      for (int g = 0; g < a.ngroups && ok; ++g) {
        for (int s = 0; s < nsteps && ok; ++s, ++step_ctr) {
          if (!mbar_wait_bounded(&ctl->bready, step_ctr & 1, a.spin, &hdr->abort)) {
            record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_BREADY, cta, s);
            ok = false;
            break;
          }
          if (step_ctr > 0 &&
              !mbar_wait_bounded(&ctl->tfree, (step_ctr - 1) & 1, a.spin, &hdr->abort)) {
            record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_TFREE, cta, s);
            ok = false;
            break;
          }
          tc_fence_after();
          if (a.trace && cta == 0 && g == 0) a.trace[(size_t)min(s, K) * kTracePhases + 9] = globaltimer_ns();
          // kIL chunks at a time, their MMAs alternating: each chunk's K-steps
          // accumulate into its own columns, so consecutive MMAs are independent
          for (int c0 = 0; c0 < ncc && ok; c0 += kIL) {
            const int nil = min(kIL, ncc - c0);
            for (int ks0 = 0; ks0 < nkb * 4; ks0 += kKS) {
              const uint32_t slot = Lw % kNS;
              if (!mbar_wait_bounded(&ctl->wfull[slot], (Lw / kNS) & 1, a.spin, &hdr->abort)) {
                record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, s);
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t a_base = smem_u32(sW + (size_t)slot * kWStage);
#pragma unroll
              for (int j = 0; j < kKS; ++j) {
                const int ks = ks0 + j;
                const uint64_t bd = smem_desc_sw128(
                    smem_u32(sU + (size_t)(ks >> 2) * N * 128) + (ks & 3) * 32, 16, 1024);
#pragma unroll
                for (int c = 0; c < kIL; ++c) {
                  if (c >= nil) break;
                  const uint64_t ad =
                      smem_desc_sw128(a_base + (j * kIL + c) * kWChunk, kWChunk / 2, 1024);
                  umma_bf16(taddr + (uint32_t)((c0 + c) * N), ad, bd, idesc, ks != 0);
                }
              }
              umma_commit(&ctl->wempty[slot]);
              ++Lw;
            }
            if (!ok) break;
            // z = bias + base: D += base^T (M = tokens, K = batch rows, MN-major)
            // x I (K-major), exact in fp32 since every product is base x 1 or x 0
            if (ok && s < K) {
              uint32_t a_base[kIL];
              for (int c = 0; c < nil; ++c) {
                const uint32_t bslot = (Lb + c) % kNBS;
                if (!mbar_wait_bounded(&ctl->bfull[bslot], ((Lb + c) / kNBS) & 1, a.spin,
                                       &hdr->abort)) {
                  record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_BASE, cta, s);
                  ok = false;
                  break;
                }
                a_base[c] = smem_u32(sBase + (size_t)bslot * N * kCH);
              }
              if (!ok) break;
              tc_fence_after();
              const uint32_t b_base = smem_u32(sI);
#pragma unroll
              for (int kk = 0; kk < N / 16; ++kk) {
                const uint64_t bd = smem_desc_sw128(b_base + kk * 32, 16, 1024);
#pragma unroll
                for (int c = 0; c < kIL; ++c) {
                  if (c >= nil) break;
                  const uint64_t ad = smem_desc_sw128(a_base[c] + kk * 2048, N * 128, 1024);
                  umma_bf16(taddr + (uint32_t)((c0 + c) * N), ad, bd, idesc, 1u);
                }
              }
              for (int c = 0; c < nil; ++c) umma_commit(&ctl->bempty[(Lb + c) % kNBS]);
              Lb += nil;
            }
            if (!ok) break;
            for (int c = 0; c < nil; ++c) {
              umma_commit(&ctl->dfull[c0 + c]);
              if (a.trace && cta == 0 && g == 0 && c0 + c < 8)
                a.trace[(size_t)min(s, K) * kTracePhases + 24 + c0 + c] = globaltimer_ns();
            }
          }
          if (a.trace && cta == 0 && g == 0) a.trace[(size_t)min(s, K) * kTracePhases + 10] = globaltimer_ns();
        }
      }
      umma_commit(&ctl->mmadone);
      mbar_drain(&ctl->mmadone, 0);
    }
  }
  // =========================================================================
  // Compute warps
  // =========================================================================
  else {
    const int q4 = warp & 3;         // tensor-memory lane quadrant
    const int n0 = (warp >> 2) * NCOL;  // first column (batch row) of this warp
    uint32_t step_ctr = 0, Lb = 0;
    uint32_t nbar = 0, rec_expected = 0;
    // Failures are folded into the CTA-wide flag ctl->abort_local; it is only
    // read right after a named barrier, so every compute thread takes the same
    // branch (a waiter that gives up keeps executing until that point).
    bool failed = false;
    auto soft_fail = [&](int code, int site, int x, int y) {
      record_error(hdr, code, site, x, y);
      ctl->abort_local = 1;
    };
    auto grid_barrier = [&]() {  // all compute threads call it
      named_sync();
      if (tid == 0) {
        // the barrier above orders the CTA's writes before this release
        red_release_add_u32(&hdr->bar, 1u);
        ++nbar;
        if (!grid_wait_count(hdr, &hdr->bar, nbar * (uint32_t)G, a.spin, SITE_GRID_BARRIER))
          ctl->abort_local = 1;
      }
      named_sync();
      return ctl->abort_local == 0;
    };
    // split-phase: arrive now, wait later
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
    // device timeline (trace flag): CTA 0, first group, one row of marks per step
    uint64_t* trace = (a.trace != nullptr && cta == 0 && tid == 0) ? a.trace : nullptr;
    auto mark = [&](int g, int step, int phase) {
      if (trace && g == 0) trace[(size_t)step * kTracePhases + phase] = globaltimer_ns();
    };

    // Target row statistics over this CTA's slice for the rows still alive.
    // Each warp takes RB rows at a time and issues every 16-byte load of the
    // batch before using any, so the loads overlap.
    auto target_row_stats = [&](int g, int par, int row, int nb_g) {
      constexpr int RB = 2;
      constexpr int VPL = 4;
      for (int nb = warp; nb < nb_g; nb += 8 * RB) {
        int rn[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          const int n = nb + 8 * r;
          rn[r] = (n < nb_g && ctl->alive[n]) ? n : -1;
        }
        float m[RB], s[RB], av[RB];
        int32_t ai[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          m[r] = -INFINITY;
          s[r] = 0.f;
          av[r] = -INFINITY;
          ai[r] = 0x7fffffff;
        }
        for (int vb = vslice_lo; vb < vslice_hi; vb += VPL * 256) {
          Raw8<T> x[RB][VPL];
#pragma unroll
          for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int u = 0; u < VPL; ++u) {
              const int v = vb + u * 256 + lane * 8;
              const int vv = v < vslice_hi ? v : vslice_lo;
              const int nn = rn[r] >= 0 ? rn[r] : 0;
              x[r][u] = raw_load(target + ((int64_t)(g * N + nn) * (K + 1) + row) * V + vv);
            }
#pragma unroll
          for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int u = 0; u < VPL; ++u) {
              const int v = vb + u * 256 + lane * 8;
              if (rn[r] < 0 || v >= vslice_hi) continue;
              float e[8];
              raw_expand(x[r][u], e);
              float lm = e[0];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                if (e[j] > av[r]) {
                  av[r] = e[j];
                  ai[r] = v + j;
                }
                lm = fmaxf(lm, e[j]);
              }
              if (!a.greedy) {
                if (lm > m[r]) {
                  s[r] *= fexp2((m[r] - lm) * k);
                  m[r] = lm;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) s[r] += fexp2((e[j] - m[r]) * k);
              }
            }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          if (rn[r] < 0) continue;  // warp-uniform
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) {
            const float m2 = __shfl_xor_sync(FULL, m[r], off), s2 = __shfl_xor_sync(FULL, s[r], off);
            const float a2 = __shfl_xor_sync(FULL, av[r], off);
            const int32_t i2 = __shfl_xor_sync(FULL, ai[r], off);
            ms_combine(m[r], s[r], m2, s2, k);
            amax_combine(av[r], ai[r], a2, i2);
          }
          if (lane == 0) {
            a.tpart[(((int64_t)par * (K + 1) + row) * N + rn[r]) * kMaxG + cta] =
                a.greedy ? make_float2(av[r], __int_as_float(ai[r])) : make_float2(m[r], s[r]);
            // step 0: the CTA's target max is its reference for the draft sums
            if (row == 0 && !a.greedy) ctl->ref[rn[r]] = m[r];
          }
        }
      }
    };

    // ---- CTA partial per batch row is formed by TPB threads per row
    const int grp_n = tid / TPB, grp_sub = tid % TPB;

    // Gather U[prev] rows (ctl->prev) into the B operand.
    auto gather_u = [&](int nb_g) {
      if (TC) {
        const int cpr = a.r / 8;  // 16-byte chunks per row
        constexpr int kIt = N * 32 / kComputeThreads;  // r <= 256: at most 32 chunks per row
        uint4 val[kIt];
#pragma unroll
        for (int t = 0; t < kIt; ++t) {  // all loads first, from clamped (valid) rows
          const int idx = tid + t * kComputeThreads;
          const int n = min(idx / cpr, N - 1), c = idx % cpr;
          val[t] = __ldg(reinterpret_cast<const uint4*>(Ug + (size_t)ctl->prev[n] * a.r) + c);
        }
#pragma unroll
        for (int t = 0; t < kIt; ++t) {
          const int idx = tid + t * kComputeThreads;
          const int n = idx / cpr, c = idx % cpr;
          if (idx >= N * cpr) continue;
          const int ka = c >> 3, j = c & 7;
          *reinterpret_cast<uint4*>(sU + (size_t)ka * N * 128 + n * 128 + ((j ^ (n & 7)) << 4)) =
              n < nb_g ? val[t] : make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      } else {
        for (int idx = tid; idx < N * a.r; idx += kComputeThreads) {
          const int n = idx / a.r, kk = idx % a.r;
          sUf[idx] = n < nb_g ? ld_elem(Ug, (int64_t)ctl->prev[n] * a.r + kk) : 0.f;
        }
      }
      named_sync();
      if (TC && tid == 0) mbar_arrive(&ctl->bready);
    };

    // Bias tile of chunk cl for this thread: (token v, NCOL columns).
    auto bias_tile = [&](int cl, float (&d)[NCOL]) {
      const uint32_t tcol = taddr + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(cl * N + n0);
      if (TC) {
        if (!mbar_wait_bounded(&ctl->dfull[cl], step_ctr & 1, a.spin, &hdr->abort))
          soft_fail(SPEC_ERR_TIMEOUT, SITE_MBAR_MMA, cta, (int)step_ctr);
        tc_fence_after();
        tmem_ld_cols<NCOL>(tcol, d);
      } else {
        const int v = (chunk0 + cl) * kCH + q4 * 32 + lane;
#pragma unroll
        for (int j = 0; j < NCOL; ++j) d[j] = 0.f;
        if (v < V) {
          for (int kk = 0; kk < a.r; ++kk) {
            const float w = ld_elem(Wg, (int64_t)kk * V + v);
#pragma unroll
            for (int j = 0; j < NCOL; ++j) d[j] = fmaf(sUf[(n0 + j) * a.r + kk], w, d[j]);
          }
        }
        tmem_st_cols<NCOL>(tcol, d);
      }
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

    // Final step: chunk cl's target tile (every row's stop row, or row K) and
    // base tile (rows that stopped) into base-ring slots 2(cl&1), 2(cl&1)+1,
    // as 16-byte asynchronous copies by all compute threads, one commit group
    // per chunk.  Rows past the batch, stopped rows' base and tokens past V are
    // left stale and only read under guards.
    auto final_tiles_issue = [&](int g, int cl, int nb_g) {
      constexpr int EPP = 16 / (int)sizeof(T);  // elements per 16-byte piece
      constexpr int PPR = kCH / EPP;            // pieces per 128-token row
      T* tt = sBase + (size_t)((cl & 1) * 2) * N * kCH;
      T* bt = tt + (size_t)N * kCH;
      const int v0 = (chunk0 + cl) * kCH;
      const int npc = min(kCH, V - v0) / EPP;
      for (int idx = tid; idx < 2 * N * PPR; idx += kComputeThreads) {
        const int t = idx / (N * PPR), n = (idx / PPR) % N, pc = idx % PPR;
        if (n >= nb_g || pc >= npc) continue;
        const bool alive = ctl->alive[n] != 0;
        if (t == 1 && alive) continue;
        const int row = alive ? K : ctl->stoprow[n];
        const int64_t b = (int64_t)g * N + n;
        const T* src = t == 0 ? target + (b * (K + 1) + row) * V + v0 + pc * EPP
                              : base + (b * K + row) * V + v0 + pc * EPP;
        cp_async16((t == 0 ? tt : bt) + (size_t)n * kCH + pc * EPP, src);
      }
      cp_async_commit();
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
      Rec& rr = ctl->rrec[j];
      if (kind == 0 && (rr.flags & 1)) return;  // the step is redone exactly
      const bool tr = kind == 0 && j == 0;
      const int b = g * N + n;
      const int o = rr.owner;
      const float M = rr.M;
      const bool use_p = (rr.flags & 2) != 0;
      const bool alive = ctl->alive[n] != 0;
      const int row = kind == 0 ? i : (alive ? K : ctl->stoprow[n]);
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
            w = kind == 0 ? (pv.y > 0.f ? pv.y * fexp2((pv.x - M) * k) : 0.f) : (use_p ? pv.y : pv.x);
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
      if (tr) mark(g, i, 14);
      const int bk = ctl->dbk;
      const int v0 = (o * a.nc + (bk >> 2)) * kCH + (bk & 3) * 32;
      const int v = v0 + lane, vc = min(v, V - 1);
      float tv = 0.f, bv = 0.f;
      if (warp == 0) {  // the row's logits at the bucket's tokens, in flight meanwhile
        if (kind == 0) {
          bv = ld_elem(base, ((int64_t)b * K + i) * V + vc);
          if (a.mode == MODE_CYCLE) tv = ld_elem(target, ((int64_t)b * (K + 1) + i) * V + vc);
        } else {
          tv = ld_elem(target, ((int64_t)b * (K + 1) + row) * V + vc);
          if (!alive) bv = ld_elem(base, ((int64_t)b * K + row) * V + vc);
        }
      }
      {  // warp w: rank rows [w*ks, w*ks + ks)
        const int ks = (a.r + 7) / 8, k0 = warp * ks, k1 = min(a.r, k0 + ks);
        const int prev = ctl->prev[n];
        const float uval = k0 + lane < k1 ? ld_elem(Ug, (int64_t)prev * a.r + k0 + lane) : 0.f;
        float wv[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) wv[t] = k0 + t < k1 ? ld_elem(Wg, (int64_t)(k0 + t) * V + vc) : 0.f;
        float part = 0.f;
#pragma unroll
        for (int t = 0; t < 32; ++t) part = fmaf(__shfl_sync(FULL, uval, t), wv[t], part);
        ctl->zpart[warp][lane] = part;
      }
      named_sync();
      if (tr) mark(g, i, 15);
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
          const bool test = a.mode == MODE_CYCLE && alive;
          int accept = 1;
          float pd = __int_as_float(0x7fc00000);
          if (test) {
            pd = fexp2((td - rr.Mt) * k) / rr.St;
            const float ratio = fexp2(((td - rr.Mt) - (zd - M)) * k) * (S / rr.St);
            const float uacc =
                philox_uniform(a.seed, a.cycle, a.row0 + (uint32_t)b, (uint32_t)i, TAG_ACCEPT);
            accept = uacc < fminf(ratio, 1.0f) ? 1 : 0;
          }
          if (lane == 0) {
            rr.token = d;
            rr.acc = accept;
            a.tokens[((int64_t)par * K + i) * N + n] = d;
            if (a.draft) a.draft[(int64_t)b * K + i] = d;
            if (a.q_draft) a.q_draft[(int64_t)b * K + i] = qd;
            if (test) {
              if (a.p_draft) a.p_draft[(int64_t)b * K + i] = pd;
              if (accept) a.out[(int64_t)b * (K + 1) + i] = d;
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
            a.out[(int64_t)b * (K + 1) + row] = v0 + wl;
          }
        }
      }
      named_sync();
    };

    // ---- row reducers.  Row n of a group is combined by one warp of CTA
    // n % G; lanes hold E consecutive per-CTA partials each, so a warp prefix
    // sum walks the CTAs in ascending token order.  The reducer finds the CTA
    // holding the row's inverse-CDF target, draws the token (draw_row) and
    // publishes a record.
    //  kind 0: draft step i -- stochastic: scale, total, owner, residual target,
    //          true max; greedy: the arg-max token; plus target row i
    //          statistics (or arg-max and the accept outcome) for live rows;
    //  kind 1: target row K statistics (or arg-max) for rows that accepted all;
    //  kind 2: final residual / bonus masses -- owner of the last draw.
    constexpr int E = (kMaxG + 31) / 32;
    auto reduce_rows = [&](int kind, int g, int par, int i, int nb_g, bool fast) {
      int mine = 0, local = 0;
      for (int n = cta; n < nb_g; n += G, ++local) {
        ++mine;
        if ((local & 7) != warp) continue;  // warp-uniform
        const int b = g * N + n;
        const int c0 = lane * E;
        Rec rc;
        rc.M = 0.f; rc.S = 1.f; rc.Mx = 0.f; rc.Mt = 0.f; rc.St = 1.f; rc.trem = INFINITY;
        rc.owner = 0; rc.token = 0; rc.acc = 1; rc.flags = 0; rc.tam = 0; rc.pad = 0;
        if (kind == 0 || kind == 2) {
          const int slot = kind == 0 ? i : K;
          const float4* pp = a.dpart + ((((int64_t)par * (K + 1) + slot) * N + n) * kMaxG + c0);
          float4 v[E];
#pragma unroll
          for (int t = 0; t < E; ++t) v[t] = __ldcg(pp + t);
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
          } else {
            float w[E];
            float M = -INFINITY, mx = -INFINITY;
            bool use_p = false;
            if (kind == 0) {
#pragma unroll
              for (int t = 0; t < E; ++t)
                if (c0 + t < G) {
                  M = fmaxf(M, v[t].x);
                  mx = fmaxf(mx, v[t].z);
                }
#pragma unroll
              for (int off = 16; off >= 1; off >>= 1) {
                M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
                mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, off));
              }
#pragma unroll
              for (int t = 0; t < E; ++t)
                w[t] = (c0 + t < G && v[t].y > 0.f) ? v[t].y * fexp2((v[t].x - M) * k) : 0.f;
            } else {
              float rt = 0.f, pt = 0.f;
#pragma unroll
              for (int t = 0; t < E; ++t)
                if (c0 + t < G) {
                  rt += v[t].x;
                  pt += v[t].y;
                }
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
            const int row = kind == 0 ? i : (ctl->alive[n] ? K : ctl->stoprow[n]);
            const float u = philox_uniform(a.seed, a.cycle, a.row0 + (uint32_t)b, (uint32_t)row,
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
            rc.Mx = mx;
            if (kind == 0 && fast && (fabsf(mx - M) * k > 64.f || !(total > 0.f))) rc.flags |= 1;
            if (kind == 2 && use_p) rc.flags |= 2;
          }
        }
        const bool live = ctl->alive[n] != 0;
        if ((kind == 0 && a.mode == MODE_CYCLE && live) || (kind == 1 && live)) {
          const int row = kind == 0 ? i : K;
          const float2* tp = a.tpart + ((((int64_t)par * (K + 1) + row) * N + n) * kMaxG + c0);
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
            rc.tam = ai;
            if (kind == 0) rc.acc = ai == rc.token ? 1 : 0;
            if (kind == 0 && lane == 0)  // greedy step of a row still verifying
              a.out[(int64_t)b * (K + 1) + i] = rc.acc ? rc.token : rc.tam;
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
            rc.Mt = Mt;
            rc.St = warp_sum(st);
          }
        }
        if (kind == 0 && a.greedy && lane == 0 && a.draft) a.draft[(int64_t)b * K + i] = rc.token;
        if (lane == 0) ctl->rrec[local] = rc;
      }
      named_sync();
      if (kind == 0) mark(g, i, 13);
      // stochastic draws, one row at a time by the whole CTA
      if ((kind == 0 && !a.greedy) || kind == 2)
        for (int j = 0; j < mine; ++j) draw_row(kind, g, par, i, cta + j * G, j);
      const int slot = kind == 0 ? i : (kind == 1 ? K : K + 1);
      if (tid < mine)
        store_rec(a.rec + ((int64_t)par * (K + 2) + slot) * N + (cta + tid * G), ctl->rrec[tid]);
      return mine;
    };
    // publish this CTA's records and wait until every row's record exists
    auto records_hop = [&](int mine, int nb_g) {
      named_sync();
      if (tid == 0) {
        if (mine) red_release_add_u32(&hdr->rec, (uint32_t)mine);
        rec_expected += (uint32_t)nb_g;
        if (!grid_wait_count(hdr, &hdr->rec, rec_expected, a.spin, SITE_REC_WAIT))
          ctl->abort_local = 1;
      }
      named_sync();
      return ctl->abort_local == 0;
    };

    for (int g = 0; g < a.ngroups && !failed; ++g) {
      const int par = g & 1;
      const int nb_g = min(N, a.B - g * N);
      for (int n = tid; n < N; n += kComputeThreads) {
        ctl->alive[n] = n < nb_g ? 1 : 0;
        ctl->stoprow[n] = K;
        ctl->ref[n] = 0.f;
      }
      if (cta == 0 && a.mode == MODE_CYCLE) {
        for (int idx = tid; idx < nb_g * K; idx += kComputeThreads) {
          const int64_t o = (int64_t)(g * N) * K + idx;
          if (a.p_draft) a.p_draft[o] = NaNf;
          if (a.q_draft && a.greedy) a.q_draft[o] = NaNf;
        }
      }
      if (cta == 0 && a.mode == MODE_DRAFT && a.greedy && a.q_draft) {
        for (int idx = tid; idx < nb_g * K; idx += kComputeThreads)
          a.q_draft[(int64_t)(g * N) * K + idx] = NaNf;
      }
      named_sync();
      mark(g, K + 1, 0);
      mark(g, K + 1, 1);

      for (int i = 0; i < K; ++i) {
        // ---------------- gather the Markov rows for this step
        mark(g, i, 0);
        for (int n = tid; n < N; n += kComputeThreads) {
          int p = 0;
          if (n < nb_g) {
            p = (i == 0) ? __ldg(a.last_token + g * N + n) : ctl->tok[n];
            if (p < 0 || p >= V) {
              record_error(hdr, SPEC_ERR_TOKEN_RANGE, SITE_TOKEN_RANGE, g * N + n, p);
              p = 0;
            }
          }
          ctl->prev[n] = p;
        }
        named_sync();
        gather_u(nb_g);
        // pull the next target row of every live batch row into L2 for the next
        // step, and take this step's target row statistics while the tensor
        // cores run the bias (the epilogue would only wait for them)
        if (a.mode == MODE_CYCLE && tid < nb_g && ctl->alive[tid])
          prefetch_l2_bulk(target + ((int64_t)(g * N + tid) * (K + 1) + i + 1) * V + vslice_lo,
                           (uint32_t)((vslice_hi - vslice_lo) * sizeof(T)));
        mark(g, i, 1);
        if (a.mode == MODE_CYCLE) target_row_stats(g, par, i, nb_g);
        if (i == 0) named_sync();  // step 0's references, written above

        // The bucket statistics are plain sums against a per-row reference:
        // the previous step's true max (all CTAs alike), or at step 0 of a
        // cycle this CTA's max of target row 0 (partials carry their own
        // reference, so CTAs may differ).  Drafting alone starts exactly.
        bool fast = !a.greedy && (i > 0 || a.mode == MODE_CYCLE);
        for (int attempt = 0; attempt < 2; ++attempt) {
          // ---------------- epilogue: z = base + bias, bucket statistics
          uint64_t t_wait = 0;
          float psum = 0.f;
          float rmax[NCOL];
#pragma unroll
          for (int j = 0; j < NCOL; ++j) rmax[j] = -INFINITY;
          for (int cl = 0; cl < ncc; ++cl) {
            float d[NCOL];
            const int vl = q4 * 32 + lane;
            const int v = (chunk0 + cl) * kCH + vl;
            const bool valid = v < V;
            const uint32_t tcol = taddr + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(cl * N + n0);
            if (attempt == 0) {
              const uint64_t t_w0 = trace ? globaltimer_ns() : 0;
              bias_tile(cl, d);  // TC: already z = bias + base, added by the MMA
              if (trace) t_wait += globaltimer_ns() - t_w0;
              if (!TC) {
                const uint32_t bslot = Lb % kNBS;
                if (!mbar_wait_bounded(&ctl->bfull[bslot], (Lb / kNBS) & 1, a.spin, &hdr->abort))
                  soft_fail(SPEC_ERR_TIMEOUT, SITE_MBAR_BASE, cta, i);
                const T* bt = sBase + (size_t)bslot * N * kCH;
#pragma unroll
                for (int j = 0; j < NCOL; ++j) d[j] += to_f<T>(bt[(n0 + j) * kCH + vl]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->bempty[bslot]);
                ++Lb;
              }
#pragma unroll
              for (int j = 0; j < NCOL; ++j) d[j] = valid ? d[j] : -INFINITY;
              if (a.biased_out && valid) {
#pragma unroll
                for (int j = 0; j < NCOL; ++j) {
                  const int b = g * N + n0 + j;
                  if (n0 + j < nb_g) a.biased_out[((int64_t)b * K + i) * V + v] = d[j];
                }
              }
              // fp32 path: z replaces the bias in tensor memory for a redo
              if (!TC && !a.greedy) tmem_st_cols<NCOL>(tcol, d);  // TC: z is in tensor memory
            } else {
              tmem_ld_cols<NCOL>(tcol, d);  // z of this step, kept in tensor memory
#pragma unroll
              for (int j = 0; j < NCOL; ++j) d[j] = valid ? d[j] : -INFINITY;
            }
            float2* bk = sBucket + ((size_t)cl * 4 + q4) * N;
            constexpr int REP = 32 / NCOL;
            if (a.greedy) {
              int32_t ix[NCOL];
#pragma unroll
              for (int j = 0; j < NCOL; ++j) ix[j] = valid ? v : 0x7fffffff;
              bfly_amax<NCOL>(d, ix, lane);
              if ((lane & (REP - 1)) == 0) bk[n0 + lane / REP] = make_float2(d[0], __int_as_float(ix[0]));
            } else if (fast) {
              const float4* r4 = reinterpret_cast<const float4*>(ctl->ref + n0);
#pragma unroll
              for (int j4 = 0; j4 < NCOL / 4; ++j4) {
                const float4 rr = r4[j4];
                const float rv[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  const int j = 4 * j4 + t;
                  rmax[j] = fmaxf(rmax[j], d[j]);
                  d[j] = valid ? fexp2((d[j] - rv[t]) * k) : 0.f;
                }
              }
              bfly_sum1<NCOL>(d, lane);
              psum += d[0];  // this lane's column, summed over the CTA's chunks
              if ((lane & (REP - 1)) == 0) {
                const float2 st = make_float2(ctl->ref[n0 + lane / REP], d[0]);
                bk[n0 + lane / REP] = st;
                a.gbk[((size_t)cta * a.nbk + cl * 4 + q4) * N + n0 + lane / REP] = st;
              }
            } else {
              float s[NCOL];
#pragma unroll
              for (int j = 0; j < NCOL; ++j) s[j] = valid ? 1.f : 0.f;
              bfly_ms<NCOL>(d, s, k, lane);
              if ((lane & (REP - 1)) == 0) {
                bk[n0 + lane / REP] = make_float2(d[0], s[0]);
                a.gbk[((size_t)cta * a.nbk + cl * 4 + q4) * N + n0 + lane / REP] = make_float2(d[0], s[0]);
              }
            }
            if (trace && g == 0 && cl < 8 && attempt == 0)
              trace[(size_t)i * kTracePhases + 16 + cl] = globaltimer_ns();
          }
          if (fast) {  // true max of z per row over this warp's tokens, and its sum
            bfly_max1<NCOL>(rmax, lane);
            if ((lane & (32 / NCOL - 1)) == 0) {
              ctl->cmax[q4][n0 + lane / (32 / NCOL)] = rmax[0];
              ctl->psum[q4][n0 + lane / (32 / NCOL)] = psum;
            }
          }
          tc_fence_before();  // z stores above are read by other warps after the barrier
          named_sync();
          tc_fence_after();
          mark(g, i, 2);
          if (a.trace && g == 0 && tid == 0 && attempt == 0)
            atomicMax(reinterpret_cast<unsigned long long*>(a.trace) + (size_t)i * kTracePhases + 8,
                      (unsigned long long)globaltimer_ns());
          if (trace && g == 0) {
            trace[(size_t)i * kTracePhases + 11] = t_wait;
          }
          // ---------------- CTA partial per batch row
          if (fast) {  // common reference: the four quadrants' running sums
            if (tid < N) {
              const int n = tid;
              const float sum = (ctl->psum[0][n] + ctl->psum[1][n]) + (ctl->psum[2][n] + ctl->psum[3][n]);
              const float tmax = fmaxf(fmaxf(ctl->cmax[0][n], ctl->cmax[1][n]),
                                       fmaxf(ctl->cmax[2][n], ctl->cmax[3][n]));
              a.dpart[(((int64_t)par * (K + 1) + i) * N + n) * kMaxG + cta] =
                  make_float4(ctl->ref[n], sum, tmax, 0.f);
            }
          } else {  // (max, sum) pairs or arg-max over the buckets, TPB threads per row
            const int n = grp_n;
            float m = -INFINITY, s = 0.f;
            int32_t ai = 0x7fffffff;
            for (int bk = grp_sub; bk < ncc * 4; bk += TPB) {
              const float2 p = sBucket[(size_t)bk * N + n];
              if (a.greedy)
                amax_combine(m, ai, p.x, __float_as_int(p.y));
              else
                ms_combine(m, s, p.x, p.y, k);
            }
#pragma unroll
            for (int off = TPB / 2; off >= 1; off >>= 1) {
              const float m2 = __shfl_xor_sync(FULL, m, off), s2 = __shfl_xor_sync(FULL, s, off);
              const int32_t i2 = __shfl_xor_sync(FULL, ai, off);
              if (a.greedy)
                amax_combine(m, ai, m2, i2);
              else
                ms_combine(m, s, m2, s2, k);
            }
            if (grp_sub == 0)
              a.dpart[(((int64_t)par * (K + 1) + i) * N + n) * kMaxG + cta] =
                  a.greedy ? make_float4(m, __int_as_float(ai), m, 0.f) : make_float4(m, s, m, 0.f);
          }
          grid_arrive();
          mark(g, i, 3);
          mark(g, i, 4);
          if (!grid_wait()) {
            failed = true;
            break;
          }
          mark(g, i, 5);
          // ---------------- row reducers draw the token of their rows and
          // publish one record per row
          if (tid == 0) ctl->redo = 0;
          const int mine = reduce_rows(0, g, par, i, nb_g, fast);
          mark(g, i, 12);
          // timeline: the last reducer and the last epilogue over all CTAs
          if (a.trace && g == 0 && tid == 0) {
            if (mine) atomicMax(reinterpret_cast<unsigned long long*>(a.trace) + (size_t)i * kTracePhases + 7,
                                (unsigned long long)globaltimer_ns());
          }
          if (!records_hop(mine, nb_g)) {
            failed = true;
            break;
          }
          for (int n = tid; n < nb_g; n += kComputeThreads) {
            const Rec r = load_rec(a.rec + ((int64_t)par * (K + 2) + i) * N + n);
            if (!a.greedy) {
              ctl->M[n] = r.M;
              ctl->S[n] = r.S;
              ctl->ref[n] = r.Mx;
              ctl->Mt[n] = r.Mt;
              ctl->St[n] = r.St;
              if (r.flags & 1) ctl->redo = 1;
            }
          }
          named_sync();
          mark(g, i, 6);
          if (!ctl->redo) break;  // read after the barrier: the same in every thread
          fast = false;           // exact statistics, re-read from tensor memory
        }
        if (failed) break;
        // tensor memory is free for the next step's MMA
        tc_fence_before();
        named_sync();
        if (TC && tid == 0) mbar_arrive(&ctl->tfree);
        // the step's tokens and accept outcomes, from the records
        for (int n = tid; n < nb_g; n += kComputeThreads) {
          const Rec r = load_rec(a.rec + ((int64_t)par * (K + 2) + i) * N + n);
          ctl->tok[n] = r.token;
          if (a.mode == MODE_CYCLE && ctl->alive[n] && !r.acc) {
            ctl->alive[n] = 0;
            ctl->stoprow[n] = i;
            ctl->zM[n] = r.M;    // draft statistics of the stop row
            ctl->zS[n] = r.S;
            ctl->fMt[n] = r.Mt;  // target statistics of the stop row
            ctl->fSt[n] = r.St;
          }
        }
        named_sync();
        ++step_ctr;
        if (ctl->abort_local) {  // read after the last named barrier of the step
          failed = true;
          break;
        }
      }  // draft steps
      if (failed) break;
      // alive / stoprow are final: pull this CTA's slice of each row's final
      // target row (and stop-row base row) into L2, and start copying the first
      // two chunks' tiles, while the final step's first exchange runs.  The
      // base ring is idle here: every draft tile of the group has been read,
      // and the base producer waits for ring_free before the next group.
      if (has_final) {
        if (tid < nb_g) {
          const bool alive = ctl->alive[tid] != 0;
          const int row = alive ? K : ctl->stoprow[tid];
          const uint32_t sl = (uint32_t)((vslice_hi - vslice_lo) * sizeof(T));
          prefetch_l2_bulk(target + ((int64_t)(g * N + tid) * (K + 1) + row) * V + vslice_lo, sl);
          if (!alive) prefetch_l2_bulk(base + ((int64_t)(g * N + tid) * K + row) * V + vslice_lo, sl);
        }
        final_tiles_issue(g, 0, nb_g);
        if (ncc > 1) final_tiles_issue(g, 1, nb_g);
      }

      if (a.mode == MODE_CYCLE) {
        if (!a.greedy) {
          // ---------------- final step: residual at the stop row, or the bonus.
          // U rows at each row's stop position first, so the bias MMA runs
          // while row K's target statistics and their exchange complete.
          for (int n = tid; n < N; n += kComputeThreads) {
            int p = 0;
            if (n < nb_g && !ctl->alive[n]) {
              const int j = ctl->stoprow[n];
              p = j == 0 ? __ldg(a.last_token + g * N + n)
                         : __ldcg(a.tokens + ((int64_t)par * K + (j - 1)) * N + n);
              if (p < 0 || p >= V) p = 0;
            }
            ctl->prev[n] = p;
          }
          named_sync();
          gather_u(nb_g);
        }
        mark(g, K, 0);
        target_row_stats(g, par, K, nb_g);  // row K of the rows that accepted every draft
        if (!grid_barrier()) {
          failed = true;
          break;
        }
        mark(g, K, 1);
        {
          const int mine = reduce_rows(1, g, par, K, nb_g, false);
          if (!records_hop(mine, nb_g)) {
            failed = true;
            break;
          }
          for (int n = tid; n < nb_g; n += kComputeThreads) {
            if (!ctl->alive[n]) continue;
            const Rec r = load_rec(a.rec + ((int64_t)par * (K + 2) + K) * N + n);
            if (a.greedy) {
              if (cta == 0) a.out[(int64_t)(g * N + n) * (K + 1) + K] = r.tam;
            } else {
              ctl->fMt[n] = r.Mt;
              ctl->fSt[n] = r.St;
            }
          }
          named_sync();
        }
        if (!a.greedy) {
          for (int n = tid; n < nb_g; n += kComputeThreads)  // final-row constants
            ctl->fcst[n] = make_float4(ctl->fMt[n], 1.f / ctl->fSt[n], ctl->zM[n],
                                       ctl->alive[n] ? 0.f : 1.f / ctl->zS[n]);
          named_sync();
          mark(g, K, 2);
          uint64_t t_fmma = 0, t_ftile = 0;
          for (int cl = 0; cl < ncc; ++cl) {
            float d[NCOL];
            const uint64_t t_m0 = trace ? globaltimer_ns() : 0;
            bias_tile(cl, d);
            if (trace) t_fmma += globaltimer_ns() - t_m0;
            const int v = (chunk0 + cl) * kCH + q4 * 32 + lane;
            const bool valid = v < V;
            // gathered stop-row tiles of this chunk (entries past the copied
            // rows / tokens are stale and only read under the guards below)
            float tv[NCOL], bvv[NCOL];
            {
              const uint64_t t_t0 = trace ? globaltimer_ns() : 0;
              if (cl + 1 < ncc)
                cp_async_wait<1>();  // this thread's copies of chunk cl have landed
              else
                cp_async_wait<0>();
              named_sync();          // ... and every other thread's
              if (trace) t_ftile += globaltimer_ns() - t_t0;
              const T* tt = sBase + (size_t)((cl & 1) * 2) * N * kCH;
              const T* bt = tt + (size_t)N * kCH;
              const int vl = q4 * 32 + lane;
#pragma unroll
              for (int j = 0; j < NCOL; ++j) {
                tv[j] = to_f<T>(tt[(n0 + j) * kCH + vl]);
                bvv[j] = to_f<T>(bt[(n0 + j) * kCH + vl]);
              }
              named_sync();  // slots of chunk cl read by everyone: refill them
              if (cl + 2 < ncc) final_tiles_issue(g, cl + 2, nb_g);
            }
            // residual mass r (into tv) and target mass p (into bvv), in place;
            // a row that accepted everything has 1 / draft sum = 0: r = p
#pragma unroll
            for (int j = 0; j < NCOL; ++j) {
              const int n = n0 + j;
              const float4 c = ctl->fcst[n];
              const bool ok = valid && n < nb_g;
              const float p = fexp2((tv[j] - c.x) * k) * c.y;
              const float q = c.w != 0.f ? fexp2((d[j] + bvv[j] - c.z) * k) * c.w : 0.f;
              tv[j] = ok ? fmaxf(p - q, 0.f) : 0.f;
              bvv[j] = ok ? p : 0.f;
            }
            bfly_sum2<NCOL>(tv, bvv, lane);
            float2* bk = sBucket + ((size_t)cl * 4 + q4) * N;
            if ((lane & (32 / NCOL - 1)) == 0) {
              bk[n0 + lane / (32 / NCOL)] = make_float2(tv[0], bvv[0]);
              a.gbk[((size_t)cta * a.nbk + cl * 4 + q4) * N + n0 + lane / (32 / NCOL)] =
                  make_float2(tv[0], bvv[0]);
            }
            if (trace && g == 0 && cl < 8) trace[(size_t)K * kTracePhases + 16 + cl] = globaltimer_ns();
          }
          if (tid == 0) mbar_arrive(&ctl->ring_free);  // last tile read: slots free
          if (trace && g == 0) {
            trace[(size_t)K * kTracePhases + 11] = t_fmma;
            trace[(size_t)K * kTracePhases + 12] = t_ftile;
          }
          named_sync();
          {
            const int n = grp_n;
            float R = 0.f, P = 0.f;
            for (int bk = grp_sub; bk < ncc * 4; bk += TPB) {
              const float2 p = sBucket[(size_t)bk * N + n];
              R += p.x;
              P += p.y;
            }
#pragma unroll
            for (int off = TPB / 2; off >= 1; off >>= 1) {
              R += __shfl_xor_sync(FULL, R, off);
              P += __shfl_xor_sync(FULL, P, off);
            }
            if (grp_sub == 0)
              a.dpart[(((int64_t)par * (K + 1) + K) * N + n) * kMaxG + cta] = make_float4(R, P, 0.f, 0.f);
          }
          mark(g, K, 3);
          if (!grid_barrier()) {
            failed = true;
            break;
          }
          mark(g, K, 4);
          // the reducers draw each row's residual / bonus token and write it
          const int mine = reduce_rows(2, g, par, K, nb_g, false);
          if (!records_hop(mine, nb_g)) {
            failed = true;
            break;
          }
          mark(g, K, 5);
          tc_fence_before();
          named_sync();
          if (TC && tid == 0) mbar_arrive(&ctl->tfree);
          ++step_ctr;
        }
        // tau and the -1 padding after it
        if (cta == 0) {
          for (int n = tid; n < nb_g; n += kComputeThreads) {
            const int b = g * N + n;
            const int j = ctl->alive[n] ? K : ctl->stoprow[n];
            a.tau[b] = j + 1;
            for (int i2 = j + 1; i2 <= K; ++i2) a.out[(int64_t)b * (K + 1) + i2] = -1;
          }
        }
        named_sync();
        mark(g, K, 6);
      }
    }  // groups
    cp_async_wait<0>();  // no copy into shared memory outlives the CTA (failure paths)
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
    tmem_dealloc(taddr, ncols);
  }
  if (tid == 0) {
    __threadfence();
    const uint32_t prior = atomicAdd(&hdr->exit_count, 1u);
    if (prior == (uint32_t)G - 1) {
      __threadfence();
      hdr->bar = 0;
      hdr->rec = 0;
      hdr->abort = 0;
      __threadfence();
      atomicExch(&hdr->exit_count, 0u);
    }
  }
}

template <typename T, bool TC, int N>
size_t smem_bytes(int r, int nc) {
  const int nkb = r / 64;
  size_t s = 1024;  // alignment slack
  if (TC) s += (size_t)kNS * kWStage;
  const size_t u = u_region_bytes<T, TC, N>(r);
  (void)nkb;
  s += (u + 1023) & ~size_t(1023);
  if (TC) s += (size_t)N * 128;  // identity operand
  s += (size_t)kNBS * N * kCH * sizeof(T);
  s += bucket_region_bytes(nc, N);
  s += sizeof(Ctl<N>);
  return s;
}

template <typename T, bool TC, int N>
cudaError_t launch_t(const Args& args, int G, size_t smem, cudaStream_t st) {
  auto fn = k_cycle<T, TC, N>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  void* params[] = {const_cast<Args*>(&args)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(fn), dim3(G), dim3(kThreads),
                                     params, smem, st);
}

template <typename T, bool TC>
size_t smem_for(int N, int r, int nc) {
  switch (N) {
    case 16: return smem_bytes<T, TC, 16>(r, nc);
    case 32: return smem_bytes<T, TC, 32>(r, nc);
    default: return smem_bytes<T, TC, 64>(r, nc);
  }
}

}  // namespace

bool cycle_geometry(int B, int K, int V, int r, int dtype, uint32_t flags, int num_sms,
                    CycleGeom* g, const char** why) {
  const int nchunks = (V + kCH - 1) / kCH;
  const int nc = (nchunks + num_sms - 1) / num_sms;
  if (nc > kMaxNC) {
    *why = "vocabulary too large for one pass (more than 32 chunks of 128 tokens per SM)";
    return false;
  }
  int N = 64;
  while (N > 16 && ((N > 16 && B <= N / 2) || nc * N > 512)) N >>= 1;
  if (nc * N > 512) {
    *why = "tensor memory cannot hold the step's bias tiles";
    return false;
  }
  const bool tc = dtype == SPEC_BF16 && r > 0 && r % 64 == 0 && r <= 256 &&
                  !(flags & SPEC_FLAG_FMA_BIAS);
  if (!tc && r > 256) {
    *why = "rank above 256 is not supported";
    return false;
  }
  g->nchunks = nchunks;
  g->nc = nc;
  g->G = (nchunks + nc - 1) / nc;
  if (g->G > kMaxG) {
    *why = "more CTAs than the kernel's partial buffers allow";
    return false;
  }
  g->N = N;
  g->tc = tc;
  g->smem = dtype == SPEC_BF16 ? (tc ? smem_for<__nv_bfloat16, true>(N, r, nc)
                                     : smem_for<__nv_bfloat16, false>(N, r, nc))
                               : smem_for<float, false>(N, r, nc);
  if (g->smem > 227 * 1024) {
    *why = "shared memory budget exceeded";
    return false;
  }
  (void)K;
  return true;
}

namespace {
size_t a256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

// Workspace body: trace | dpart | tpart | tokens | records | bucket statistics,
// each 256-byte aligned.
size_t cycle_trace_bytes(int K) { return a256(sizeof(uint64_t) * (size_t)(K + 2) * kTracePhases); }
namespace {
size_t dpart_bytes(int K, int N) { return a256(sizeof(float4) * 2 * (size_t)(K + 1) * N * kMaxG); }
size_t tpart_bytes(int K, int N) { return a256(sizeof(float2) * 2 * (size_t)(K + 1) * N * kMaxG); }
size_t tok_bytes(int K, int N) { return a256(sizeof(int32_t) * 2 * (size_t)K * N); }
size_t rec_bytes(int K, int N) { return a256(sizeof(Rec) * 2 * (size_t)(K + 2) * N); }
size_t gbk_bytes(const CycleGeom& g) { return a256(sizeof(float2) * (size_t)g.G * g.nc * 4 * g.N); }
}  // namespace
size_t cycle_ws_bytes(int K, const CycleGeom& g) {
  return cycle_trace_bytes(K) + dpart_bytes(K, g.N) + tpart_bytes(K, g.N) + tok_bytes(K, g.N) +
         rec_bytes(K, g.N) + gbk_bytes(g);
}

cudaError_t launch_cycle(const CycleLaunch& L, const CycleGeom& g, WsHeader* hdr, uint8_t* body,
                         const CUtensorMap* tmW, const CUtensorMap* tmBase, cudaStream_t st) {
  Args a;
  memset(&a, 0, sizeof(a));
  if (tmW) a.tmW = *tmW;
  a.tmBase = *tmBase;
  a.base = L.base;
  a.target = L.target;
  a.U = L.U;
  a.W = L.W;
  a.last_token = L.last_token;
  a.draft = L.draft;
  a.out = L.out;
  a.tau = L.tau;
  a.p_draft = L.p_draft;
  a.q_draft = L.q_draft;
  a.biased_out = L.biased_out;
  a.hdr = hdr;
  a.trace = L.trace ? reinterpret_cast<uint64_t*>(body) : nullptr;
  body += cycle_trace_bytes(L.K);
  a.dpart = reinterpret_cast<float4*>(body);
  body += dpart_bytes(L.K, g.N);
  a.tpart = reinterpret_cast<float2*>(body);
  body += tpart_bytes(L.K, g.N);
  a.tokens = reinterpret_cast<int32_t*>(body);
  body += tok_bytes(L.K, g.N);
  a.rec = reinterpret_cast<Rec*>(body);
  body += rec_bytes(L.K, g.N);
  a.gbk = reinterpret_cast<float2*>(body);
  a.nbk = g.nc * 4;
  a.B = L.B;
  a.K = L.K;
  a.V = L.V;
  a.r = L.r;
  a.G = g.G;
  a.nc = g.nc;
  a.nchunks = g.nchunks;
  a.mode = L.mode;
  a.greedy = L.greedy;
  a.ngroups = (L.B + g.N - 1) / g.N;
  a.k = L.greedy ? 1.0f : 1.4426950408889634f / L.temperature;
  a.seed = L.seed;
  a.row0 = L.row0;
  a.cycle = L.cycle;
  a.spin = L.spin;
  if (L.dtype == SPEC_BF16) {
    if (g.tc) {
      switch (g.N) {
        case 16: return launch_t<__nv_bfloat16, true, 16>(a, g.G, g.smem, st);
        case 32: return launch_t<__nv_bfloat16, true, 32>(a, g.G, g.smem, st);
        default: return launch_t<__nv_bfloat16, true, 64>(a, g.G, g.smem, st);
      }
    }
    switch (g.N) {
      case 16: return launch_t<__nv_bfloat16, false, 16>(a, g.G, g.smem, st);
      case 32: return launch_t<__nv_bfloat16, false, 32>(a, g.G, g.smem, st);
      default: return launch_t<__nv_bfloat16, false, 64>(a, g.G, g.smem, st);
    }
  }
  switch (g.N) {
    case 16: return launch_t<float, false, 16>(a, g.G, g.smem, st);
    case 32: return launch_t<float, false, 32>(a, g.G, g.smem, st);
    default: return launch_t<float, false, 64>(a, g.G, g.smem, st);
  }
}

}  // namespace specdec
