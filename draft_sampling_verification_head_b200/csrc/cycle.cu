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
//    (16/32/64) = the tcgen05 N dimension.
//  * Per draft step, per chunk: the bias tile D[v, b] = W^T[v, :] . U[prev_b]^T
//    is one tcgen05.mma chain (M = 128 tokens, N batch rows, K = r) into tensor
//    memory; W^T streams through an 8-stage TMA ring (128-byte swizzle, L2
//    evict-last), the gathered U rows form the swizzled K-major B operand, and
//    the base logit tile arrives by TMA.  D stays in tensor memory for the whole
//    step (nc * N <= 512 columns), so the owner of a sample can re-read it.
//  * The epilogue adds the base tile and reduces softmax statistics of
//    z / T per 32-token bucket with a transposing butterfly (one exp2 per
//    element), then per CTA; the (m, s) partials are exchanged through global
//    memory behind a grid barrier.  Every CTA combines all partials in the same
//    fixed order, so all agree on Z, on the prefix masses and on which CTA owns
//    the inverse-CDF draw; the owner walks its buckets and scans one bucket with
//    a warp prefix sum.  Greedy steps take the arg-max instead (no owner step).
//  * Cycle mode verifies on the fly: while waiting at each grid barrier the
//    CTAs stream the next target row for the rows still alive (early exit: a
//    row is never read past its first rejection), and the owner of d_i decides
//    the accept test with p_i(d_i) / q_i(d_i).  A last step recomputes the bias
//    of each row's stop position and draws the residual max(p - q, 0) (or the
//    bonus from target row K) with the same two-level inverse CDF.
//  * Every wait is bounded (spin limit); a CTA that gives up records
//    SPEC_ERR_TIMEOUT in the workspace, the others notice and all exit.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace specdec {

namespace {

constexpr int kCH = 128;            // tokens per chunk (UMMA M)
constexpr int kComputeThreads = 256;
constexpr int kThreads = 320;       // 8 compute warps + TMA warp + MMA warp
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kNS = 8;              // W ring stages
constexpr int kNBS = 2;             // base tile ring stages
constexpr int kMaxNC = 32;
constexpr int kWStage = kCH * 64 * 2;  // 16 KB: 128 tokens x 64 rank, bf16
constexpr int kMaxG = 160;          // CTAs a launch may use (>= SM count); partial-row stride
constexpr int kOwnBatch = 8;        // owned rows scanned together by one warp
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
  float2* dpart;     // [2][K+1][N][kMaxG]
  float2* tpart;     // [2][K+1][N][kMaxG]
  int32_t* tokens;   // [2][K][N]
  int32_t* accf;     // [2][K][N]
  StopInfo* stopinfo;// [2][N]
  uint64_t* trace;   // [K+2][kTracePhases] device timeline of CTA 0, or null
  int B, K, V, r, G, nc, nchunks, mode, greedy, ngroups;
  float k;           // log2(e) / T (1 in greedy mode)
  uint64_t seed, cycle, spin;
};

template <int N>
struct Ctl {
  uint64_t wfull[kNS], wempty[kNS], bfull[kNBS], bempty[kNBS], dfull[kMaxNC];
  uint64_t bready, tfree, mmadone;
  uint32_t tmem_slot;
  int32_t abort_local;
  int32_t n_owned;
  int32_t owned[N];
  int32_t obucket[N];
  float obtarget[N];
  int32_t prev[N];
  int32_t alive[N];
  int32_t stoprow[N];
  int32_t tok[N];
  float M[N], S[N];     // global draft stats of the current step
  float zM[N], zS[N];   // draft stats of the stop row
  float Mt[N], St[N];   // target stats (row i during a step, stop row / row K at the end)
  int16_t wlist[8][N];  // owned rows per compute warp
  int32_t wcount[8];
};

SPEC_DEV void named_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

SPEC_DEV uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

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
  const size_t u_bytes = TC ? (size_t)nkb * N * 128 : (size_t)N * a.r * 4;
  T* sBase = reinterpret_cast<T*>(sU + ((u_bytes + 1023) & ~size_t(1023)));  // kNBS x N x 128
  const size_t base_bytes = (size_t)kNBS * N * kCH * sizeof(T);
  float2* sBucket = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(sBase) + base_bytes);
  Ctl<N>* ctl = reinterpret_cast<Ctl<N>*>(reinterpret_cast<uint8_t*>(sBucket) +
                                          (size_t)a.nc * 4 * N * sizeof(float2));

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
      mbar_init(&ctl->bempty[i], kComputeThreads / 32);
    }
    for (int i = 0; i < kMaxNC; ++i) mbar_init(&ctl->dfull[i], 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = ctl->tmem_slot;

  // =========================================================================
  // TMA producer: W ring (tensor-core path) and base tiles, in consumption order
  // =========================================================================
  if (warp == kProducerWarp) {
    if (lane == 0) {
      const uint64_t polW = policy_evict_last(), polB = policy_evict_first();
      if (TC) tma_prefetch_desc(&a.tmW);
      tma_prefetch_desc(&a.tmBase);
      uint32_t Lw = 0, Lb = 0;
      bool ok = true;
      for (int g = 0; g < a.ngroups && ok; ++g) {
        for (int s = 0; s < nsteps && ok; ++s) {
          for (int cl = 0; cl < ncc && ok; ++cl) {
            const int v0 = (chunk0 + cl) * kCH;
            if (TC) {
              for (int kb = 0; kb < nkb; ++kb) {
                const uint32_t slot = Lw % kNS;
                if (Lw >= kNS &&
                    !mbar_wait_bounded(&ctl->wempty[slot], ((Lw / kNS) - 1) & 1, a.spin,
                                       &hdr->abort)) {
                  record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, 100 + s);
                  ok = false;
                  break;
                }
                mbar_arrive_expect_tx(&ctl->wfull[slot], kWStage);
                tma_load_2d(sW + (size_t)slot * kWStage, &a.tmW, &ctl->wfull[slot], v0, kb * 64,
                            polW);
                tma_load_2d(sW + (size_t)slot * kWStage + kWStage / 2, &a.tmW,
                            &ctl->wfull[slot], v0 + 64, kb * 64, polW);
                ++Lw;
              }
            }
            if (ok && s < K) {
              const uint32_t slot = Lb % kNBS;
              if (Lb >= kNBS &&
                  !mbar_wait_bounded(&ctl->bempty[slot], ((Lb / kNBS) - 1) & 1, a.spin,
                                     &hdr->abort)) {
                record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_BASE, cta, s);
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&ctl->bfull[slot], (uint32_t)(N * kCH * sizeof(T)));
              tma_load_3d(sBase + (size_t)slot * N * kCH, &a.tmBase, &ctl->bfull[slot], v0, s,
                          g * N, polB);
              ++Lb;
            }
          }
        }
      }
      // drain: the most recent load on every slot must have landed
      for (uint32_t L = (Lw > kNS ? Lw - kNS : 0); L < Lw; ++L)
        mbar_drain(&ctl->wfull[L % kNS], (L / kNS) & 1);
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
      uint32_t Lw = 0, step_ctr = 0;
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
          for (int cl = 0; cl < ncc && ok; ++cl) {
            const uint32_t dcol = taddr + (uint32_t)(cl * N);
            for (int kb = 0; kb < nkb; ++kb) {
              const uint32_t slot = Lw % kNS;
              if (!mbar_wait_bounded(&ctl->wfull[slot], (Lw / kNS) & 1, a.spin, &hdr->abort)) {
                record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, s);
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t a_base = smem_u32(sW + (size_t)slot * kWStage);
              const uint32_t b_base = smem_u32(sU + (size_t)kb * N * 128);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc_sw128(a_base + kk * 2048, 8192, 1024);
                const uint64_t bd = smem_desc_sw128(b_base + kk * 32, 16, 1024);
                umma_bf16(dcol, ad, bd, idesc, (kb | kk) != 0);
              }
              umma_commit(&ctl->wempty[slot]);
              ++Lw;
            }
            if (ok) umma_commit(&ctl->dfull[cl]);
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
    uint32_t nbar = 0, tok_expected = 0;
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
        __threadfence();
        red_release_add_u32(&hdr->bar, 1u);
        ++nbar;
        if (!grid_wait_count(hdr, &hdr->bar, nbar * (uint32_t)G, a.spin, SITE_GRID_BARRIER) ||
            ld_volatile_u32(&hdr->abort))
          ctl->abort_local = 1;
        __threadfence();
      }
      named_sync();
      return ctl->abort_local == 0;
    };
    // split-phase: arrive now, wait later
    auto grid_arrive = [&]() {
      named_sync();
      if (tid == 0) {
        __threadfence();
        red_release_add_u32(&hdr->bar, 1u);
        ++nbar;
      }
    };
    auto grid_wait = [&]() {
      if (tid == 0) {
        if (!grid_wait_count(hdr, &hdr->bar, nbar * (uint32_t)G, a.spin, SITE_GRID_BARRIER) ||
            ld_volatile_u32(&hdr->abort))
          ctl->abort_local = 1;
        __threadfence();
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
                  s[r] *= exp2f((m[r] - lm) * k);
                  m[r] = lm;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) s[r] += exp2f((e[j] - m[r]) * k);
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
          if (lane == 0)
            a.tpart[(((int64_t)par * (K + 1) + row) * N + rn[r]) * kMaxG + cta] =
                a.greedy ? make_float2(av[r], __int_as_float(ai[r])) : make_float2(m[r], s[r]);
        }
      }
    };

    // ---- combine of the G per-CTA partials of one batch row: TPB threads per
    // row, each holding a contiguous slice of the partials in registers (all
    // loads in flight together).  Identical arithmetic in every CTA.
    constexpr int MAXC = kMaxG / TPB;  // partials per thread (even: 16-byte loads)
    static_assert(MAXC % 2 == 0, "partial slices are read as float4");
    const int grp_n = tid / TPB, grp_sub = tid % TPB;
    const int c_lo = grp_sub * MAXC;
    const int c_hi = min(G, c_lo + MAXC);
    // Unconditional 16-byte loads over the padded row (entries past G or of
    // rows not in use are replaced afterwards), so all are in flight together.
    auto load_slice = [&](const float2* pp, bool on, float2 (&reg)[MAXC], float2 dflt) {
      const float4* p4 = reinterpret_cast<const float4*>(pp + c_lo);
#pragma unroll
      for (int j = 0; j < MAXC / 2; ++j) {
        const float4 q = __ldcg(p4 + j);
        reg[2 * j] = make_float2(q.x, q.y);
        reg[2 * j + 1] = make_float2(q.z, q.w);
      }
#pragma unroll
      for (int j = 0; j < MAXC; ++j)
        if (!(on && c_lo + j < c_hi)) reg[j] = dflt;
    };
    // (m, s) partials -> global M, S (valid in every thread of the group)
    auto group_ms = [&](const float2 (&reg)[MAXC], float& M, float& S) {
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < MAXC; ++j) m = fmaxf(m, reg[j].x);
#pragma unroll
      for (int off = TPB / 2; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
      float loc = 0.f;
#pragma unroll
      for (int j = 0; j < MAXC; ++j)
        if (reg[j].y > 0.f) loc += reg[j].y * exp2f((reg[j].x - m) * k);
      float sum = loc;
#pragma unroll
      for (int off = TPB / 2; off >= 1; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
      M = m;
      S = sum;
    };
    auto group_amax = [&](const float2 (&reg)[MAXC], float& av, int32_t& ai) {
      av = -INFINITY;
      ai = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < MAXC; ++j) amax_combine(av, ai, reg[j].x, __float_as_int(reg[j].y));
#pragma unroll
      for (int off = TPB / 2; off >= 1; off >>= 1) {
        const float a2 = __shfl_xor_sync(FULL, av, off);
        const int32_t i2 = __shfl_xor_sync(FULL, ai, off);
        amax_combine(av, ai, a2, i2);
      }
    };
    // Inverse-CDF owner among the G CTAs for weights w_c (given by wfun(j)),
    // scanned in ascending c; returns true in the one thread whose slice holds
    // the owner, with the owner index and the mass before it.
    // weight of a partial: wmode 0 -> s * exp2((m - M) k) (softmax partials),
    // 1 -> .x (residual mass), 2 -> .y (target mass)
    auto pweight = [&](const float2& p, int wmode, float M) {
      if (wmode == 0) return p.y > 0.f ? p.y * exp2f((p.x - M) * k) : 0.f;
      return wmode == 1 ? p.x : p.y;
    };
    auto group_owner = [&](const float2 (&reg)[MAXC], int wmode, float M, float tgt, int& own,
                           float& before, bool& fallback) {
      float loc = 0.f;
#pragma unroll
      for (int j = 0; j < MAXC; ++j) loc += pweight(reg[j], wmode, M);
      float incl = loc;
#pragma unroll
      for (int o = 1; o < TPB; o <<= 1) {
        const float y = __shfl_up_sync(FULL, incl, o, TPB);
        if (grp_sub >= o) incl += y;
      }
      float cum = incl - loc;
      int found = 0x7fffffff, lastpos = -1;
      before = 0.f;
#pragma unroll
      for (int j = 0; j < MAXC; ++j) {
        if (c_lo + j >= c_hi) continue;
        const float wj = pweight(reg[j], wmode, M);
        if (wj > 0.f) lastpos = c_lo + j;
        if (found == 0x7fffffff && cum + wj > tgt) {
          found = c_lo + j;
          before = cum;
        }
        cum += wj;
      }
      int o2 = found;
#pragma unroll
      for (int off = TPB / 2; off >= 1; off >>= 1) o2 = min(o2, __shfl_xor_sync(FULL, o2, off));
      int lp = lastpos;
#pragma unroll
      for (int off = TPB / 2; off >= 1; off >>= 1) lp = max(lp, __shfl_xor_sync(FULL, lp, off));
      fallback = o2 == 0x7fffffff;
      own = fallback ? lp : o2;
      return fallback ? (lastpos == own && own >= 0) : (found == own);
    };

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

    // Owner scan of one 32-token bucket (whole warp): weights per lane, target
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

    // Bucket walk for every owned row (one thread each), then per-warp work
    // lists: a row goes to one of the two warps of its bucket's quadrant.
    // `mass(n, cl, q)` gives the bucket weight in the owner's scale.
    // fin = false: softmax buckets (m, s) in the scale of ctl->M[n];
    // fin = true: residual / target mass buckets, chosen by ctl->S[n] != 0.
    auto bucket_mass = [&](int n, int cl, int q, bool fin) {
      const float2 p = sBucket[((size_t)cl * 4 + q) * N + n];
      if (!fin) return p.y > 0.f ? p.y * exp2f((p.x - ctl->M[n]) * k) : 0.f;
      return ctl->S[n] != 0.f ? p.y : p.x;
    };
    auto walk_and_assign = [&](bool fin) {
      const int n_owned = ctl->n_owned;
      const int nbk = ncc * 4;  // buckets in ascending token order
      for (int o = warp; o < n_owned; o += 8) {  // one warp per owned row
        const int n = ctl->owned[o];
        const float tin = ctl->obtarget[o];
        float carry = 0.f;
        int pick = -1, lastb = -1;
        float tin_in = INFINITY;
        for (int b0 = 0; b0 < nbk && pick < 0; b0 += 32) {  // 32 buckets per pass
          const int bk = b0 + lane;
          const float w = bk < nbk ? bucket_mass(n, bk >> 2, bk & 3, fin) : 0.f;
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
        if (lane == 0) {
          if (pick < 0) {
            pick = lastb < 0 ? 0 : lastb;
            tin_in = INFINITY;
          }
          ctl->obucket[o] = pick;
          ctl->obtarget[o] = tin_in;
        }
      }
      named_sync();
      if (tid < 4) {
        int c0 = 0, c1 = 0, alt = 0;
        for (int o = 0; o < n_owned; ++o) {
          if ((ctl->obucket[o] & 3) != tid) continue;
          if (alt) ctl->wlist[tid + 4][c1++] = (int16_t)o;
          else ctl->wlist[tid][c0++] = (int16_t)o;
          alt ^= 1;
        }
        ctl->wcount[tid] = c0;
        ctl->wcount[tid + 4] = c1;
      }
      named_sync();
    };

    for (int g = 0; g < a.ngroups && !failed; ++g) {
      const int par = g & 1;
      const int nb_g = min(N, a.B - g * N);
      for (int n = tid; n < N; n += kComputeThreads) {
        ctl->alive[n] = n < nb_g ? 1 : 0;
        ctl->stoprow[n] = K;
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
      if (a.mode == MODE_CYCLE) target_row_stats(g, par, 0, nb_g);
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
        // pull the next target row of every live batch row into L2 now; the
        // background pass reads it while this step's barrier completes
        if (a.mode == MODE_CYCLE && tid < nb_g && ctl->alive[tid])
          prefetch_l2_bulk(target + ((int64_t)(g * N + tid) * (K + 1) + i + 1) * V + vslice_lo,
                           (uint32_t)((vslice_hi - vslice_lo) * sizeof(T)));
        mark(g, i, 1);

        // ---------------- epilogue: z = base + bias, bucket statistics
        uint64_t t_wait = 0;
        for (int cl = 0; cl < ncc; ++cl) {
          float d[NCOL];
          const uint64_t t_w0 = trace ? globaltimer_ns() : 0;
          bias_tile(cl, d);
          if (trace) t_wait += globaltimer_ns() - t_w0;
          const uint32_t bslot = Lb % kNBS;
          if (!mbar_wait_bounded(&ctl->bfull[bslot], (Lb / kNBS) & 1, a.spin, &hdr->abort))
            soft_fail(SPEC_ERR_TIMEOUT, SITE_MBAR_BASE, cta, i);
          const T* bt = sBase + (size_t)bslot * N * kCH;
          const int vl = q4 * 32 + lane;
          const int v = (chunk0 + cl) * kCH + vl;
          const bool valid = v < V;
#pragma unroll
          for (int j = 0; j < NCOL; ++j)
            d[j] = valid ? d[j] + to_f<T>(bt[(n0 + j) * kCH + vl]) : -INFINITY;
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->bempty[bslot]);
          ++Lb;
          // z replaces the bias in tensor memory: the owner scan reads it back
          if (!a.greedy)
            tmem_st_cols<NCOL>(taddr + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(cl * N + n0), d);
          if (a.biased_out && valid) {
#pragma unroll
            for (int j = 0; j < NCOL; ++j) {
              const int b = g * N + n0 + j;
              if (n0 + j < nb_g) a.biased_out[((int64_t)b * K + i) * V + v] = d[j];
            }
          }
          float2* bk = sBucket + ((size_t)cl * 4 + q4) * N;
          if (a.greedy) {
            int32_t ix[NCOL];
#pragma unroll
            for (int j = 0; j < NCOL; ++j) ix[j] = valid ? v : 0x7fffffff;
            bfly_amax<NCOL>(d, ix, lane);
            if ((lane & (32 / NCOL - 1)) == 0)
              bk[n0 + lane / (32 / NCOL)] = make_float2(d[0], __int_as_float(ix[0]));
          } else {
            float s[NCOL];
#pragma unroll
            for (int j = 0; j < NCOL; ++j) s[j] = valid ? 1.f : 0.f;
            bfly_ms<NCOL>(d, s, k, lane);
            if ((lane & (32 / NCOL - 1)) == 0) bk[n0 + lane / (32 / NCOL)] = make_float2(d[0], s[0]);
          }
        }
        tc_fence_before();  // z stores above are read by other warps after the barrier
        named_sync();
        tc_fence_after();
        mark(g, i, 2);
        if (trace && g == 0) trace[(size_t)i * kTracePhases + 11] = t_wait;
        // ---------------- CTA partial per batch row (TPB threads per row)
        {
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
                a.greedy ? make_float2(m, __int_as_float(ai)) : make_float2(m, s);
        }
        grid_arrive();
        mark(g, i, 3);
        // background while the barrier completes: next target row, rows alive so far
        if (a.mode == MODE_CYCLE) target_row_stats(g, par, i + 1, nb_g);
        mark(g, i, 4);
        if (!grid_wait()) {
          failed = true;
          break;
        }
        mark(g, i, 5);

        // ---------------- combine partials: every CTA, same order
        if (tid == 0) ctl->n_owned = 0;
        named_sync();
        {
          const int n = grp_n;
          const bool row_on = n < nb_g;
          float2 reg[MAXC];
          load_slice(a.dpart + (((int64_t)par * (K + 1) + i) * N + n) * kMaxG, row_on, reg,
                     a.greedy ? make_float2(-INFINITY, __int_as_float(0x7fffffff))
                              : make_float2(-INFINITY, 0.f));
          if (a.greedy) {
            float av;
            int32_t ai;
            group_amax(reg, av, ai);
            if (grp_sub == 0 && row_on) ctl->tok[n] = ai;
            if (a.mode == MODE_CYCLE) {
              const bool al = row_on && ctl->alive[n];
              load_slice(a.tpart + (((int64_t)par * (K + 1) + i) * N + n) * kMaxG, al, reg,
                         make_float2(-INFINITY, __int_as_float(0x7fffffff)));
              float tv;
              int32_t tam;
              group_amax(reg, tv, tam);
              if (grp_sub == 0 && al) {
                const int b = g * N + n;
                const bool acc = tam == ai;
                if (cta == 0) a.out[(int64_t)b * (K + 1) + i] = acc ? ai : tam;
                if (!acc) {
                  ctl->alive[n] = 0;
                  ctl->stoprow[n] = i;
                }
              }
            }
          } else {
            float M, S;
            group_ms(reg, M, S);
            mark(g, i, 12);
            const int b = g * N + n;
            const float u = philox_uniform(a.seed, a.cycle, (uint32_t)b, (uint32_t)i, TAG_DRAFT);
            const float tgt = u * S;
            int own;
            float before;
            bool fb;
            const bool holder = group_owner(reg, 0, M, tgt, own, before, fb);
            mark(g, i, 13);
            if (row_on) {
              if (grp_sub == 0) {
                ctl->M[n] = M;
                ctl->S[n] = S;
              }
              if (holder && own == cta) {
                const int slot = atomicAdd(&ctl->n_owned, 1);
                ctl->owned[slot] = n;
                ctl->obtarget[slot] = fb ? INFINITY : tgt - before;
              }
            }
            if (a.mode == MODE_CYCLE) {
              // target statistics of row i for the rows still alive (used by owners)
              const bool al = row_on && ctl->alive[n];
              load_slice(a.tpart + (((int64_t)par * (K + 1) + i) * N + n) * kMaxG, al, reg,
                         make_float2(-INFINITY, 0.f));
              float Mt, St;
              group_ms(reg, Mt, St);
              if (grp_sub == 0 && al) {
                ctl->Mt[n] = Mt;
                ctl->St[n] = St;
              }
              mark(g, i, 14);
            }
          }
        }
        named_sync();
        mark(g, i, 6);

        if (a.greedy) {
          if (cta == 0)
            for (int n = tid; n < nb_g; n += kComputeThreads)
              if (a.draft) a.draft[(int64_t)(g * N + n) * K + i] = ctl->tok[n];
          tc_fence_before();
          named_sync();
          if (TC && tid == 0) mbar_arrive(&ctl->tfree);
        } else {
          // ---------------- owners: bucket walk, then batched bucket scans
          walk_and_assign(false);
          mark(g, i, 15);
          const int cnt = ctl->wcount[warp];
          for (int bs = 0; bs < cnt; bs += kOwnBatch) {
            int oo[kOwnBatch];
            float dv[kOwnBatch], td[kOwnBatch], zd[kOwnBatch], qd[kOwnBatch];
            int dtok[kOwnBatch];
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) {
              oo[j] = bs + j < cnt ? ctl->wlist[warp][bs + j] : -1;
              dtok[j] = 0;
            }
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) {
              dv[j] = 0.f;
              if (oo[j] < 0) continue;
              const int cl = ctl->obucket[oo[j]] >> 2, n = ctl->owned[oo[j]];
              tmem_ld1(taddr + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(cl * N + n), &dv[j]);
            }
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) {
              if (oo[j] < 0) continue;
              const int cl = ctl->obucket[oo[j]] >> 2, n = ctl->owned[oo[j]];
              const float M = ctl->M[n], S = ctl->S[n];
              const int v = (chunk0 + cl) * kCH + q4 * 32 + lane;
              const bool valid = v < V;
              const float z = valid ? dv[j] : -INFINITY;  // z = base + bias, kept in tensor memory
              const float e = valid ? exp2f((z - M) * k) : 0.f;
              const int wl = bucket_scan(e, ctl->obtarget[oo[j]]);
              dtok[j] = (chunk0 + cl) * kCH + q4 * 32 + wl;
              zd[j] = __shfl_sync(FULL, z, wl);
              qd[j] = exp2f((zd[j] - M) * k) / S;
            }
            const bool cyc = a.mode == MODE_CYCLE;
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) {
              const int oj = oo[j] < 0 ? 0 : oo[j];
              const int n = min(ctl->owned[oj], nb_g - 1);
              const int dt = oo[j] < 0 ? 0 : min(max(dtok[j], 0), V - 1);
              td[j] = cyc ? ld_elem(target, ((int64_t)(g * N + n) * (K + 1) + i) * V + dt) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) {
              if (oo[j] < 0) continue;
              const int n = ctl->owned[oo[j]];
              const int b = g * N + n;
              const float M = ctl->M[n], S = ctl->S[n];
              const bool alive = cyc && ctl->alive[n];
              int accept = 1;
              float pd = NaNf;
              if (alive) {
                const float Mt = ctl->Mt[n], St = ctl->St[n];
                pd = exp2f((td[j] - Mt) * k) / St;
                const float ratio = exp2f(((td[j] - Mt) - (zd[j] - M)) * k) * (S / St);
                const float uacc = philox_uniform(a.seed, a.cycle, (uint32_t)b, (uint32_t)i, TAG_ACCEPT);
                accept = uacc < fminf(ratio, 1.0f) ? 1 : 0;
              }
              if (lane == 0) {
                a.tokens[((int64_t)par * K + i) * N + n] = dtok[j];
                a.accf[((int64_t)par * K + i) * N + n] = accept;
                if (a.draft) a.draft[(int64_t)b * K + i] = dtok[j];
                if (a.q_draft) a.q_draft[(int64_t)b * K + i] = qd[j];
                if (alive) {
                  if (a.p_draft) a.p_draft[(int64_t)b * K + i] = pd;
                  if (accept)
                    a.out[(int64_t)b * (K + 1) + i] = dtok[j];
                  else
                    a.stopinfo[(int64_t)par * N + n] = StopInfo{i, ctl->Mt[n], ctl->St[n], M, S};
                }
              }
            }
          }
          mark(g, i, 7);
          tc_fence_before();
          named_sync();
          if (TC && tid == 0) mbar_arrive(&ctl->tfree);
          if (tid == 0) {
            __threadfence();
            const int n_owned = ctl->n_owned;
            if (n_owned) red_release_add_u32(&hdr->tok, (uint32_t)n_owned);
            tok_expected += (uint32_t)nb_g;
            if (!grid_wait_count(hdr, &hdr->tok, tok_expected, a.spin, SITE_TOKEN_WAIT) ||
                ld_volatile_u32(&hdr->abort))
              ctl->abort_local = 1;
            __threadfence();
          }
          named_sync();
          mark(g, i, 8);
          if (ctl->abort_local) {
            failed = true;
            break;
          }
          for (int n = tid; n < nb_g; n += kComputeThreads) {
            ctl->tok[n] = __ldcg(a.tokens + ((int64_t)par * K + i) * N + n);
            if (a.mode == MODE_CYCLE && ctl->alive[n] &&
                !__ldcg(a.accf + ((int64_t)par * K + i) * N + n)) {
              const uint32_t sl = (uint32_t)((vslice_hi - vslice_lo) * sizeof(T));
              prefetch_l2_bulk(target + ((int64_t)(g * N + n) * (K + 1) + i) * V + vslice_lo, sl);
              prefetch_l2_bulk(base + ((int64_t)(g * N + n) * K + i) * V + vslice_lo, sl);
              ctl->alive[n] = 0;
              ctl->stoprow[n] = i;
              ctl->zM[n] = ctl->M[n];
              ctl->zS[n] = ctl->S[n];
              ctl->Mt[n] = __ldcg(&a.stopinfo[(int64_t)par * N + n].mt);
              ctl->St[n] = __ldcg(&a.stopinfo[(int64_t)par * N + n].st);
            }
          }
          named_sync();
        }
        ++step_ctr;
        if (ctl->abort_local) {  // read after the last named barrier of the step
          failed = true;
          break;
        }
      }  // draft steps
      if (failed) break;

      if (a.mode == MODE_CYCLE) {
        // row-K target partials (written after the last barrier) become visible
        mark(g, K, 0);
        if (!grid_barrier()) {
          failed = true;
          break;
        }
        mark(g, K, 1);
        {
          // target statistics of row K for the rows that accepted every draft
          const int n = grp_n;
          const bool al = n < nb_g && ctl->alive[n];
          float2 reg[MAXC];
          load_slice(a.tpart + (((int64_t)par * (K + 1) + K) * N + n) * kMaxG, al, reg,
                     a.greedy ? make_float2(-INFINITY, __int_as_float(0x7fffffff))
                              : make_float2(-INFINITY, 0.f));
          if (a.greedy) {
            float tv;
            int32_t tam;
            group_amax(reg, tv, tam);
            if (grp_sub == 0 && al && cta == 0) a.out[(int64_t)(g * N + n) * (K + 1) + K] = tam;
          } else {
            float Mt, St;
            group_ms(reg, Mt, St);
            if (grp_sub == 0 && al) {
              ctl->Mt[n] = Mt;
              ctl->St[n] = St;
            }
          }
        }
        named_sync();
        if (!a.greedy) {
          // ---------------- final step: residual at the stop row, or the bonus
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
          mark(g, K, 2);
          for (int cl = 0; cl < ncc; ++cl) {
            float d[NCOL];
            bias_tile(cl, d);
            const int v = (chunk0 + cl) * kCH + q4 * 32 + lane;
            const bool valid = v < V;
            float tv[NCOL], bvv[NCOL];
#pragma unroll
            for (int j = 0; j < NCOL; ++j) {  // loads from clamped valid addresses
              const int n = min(n0 + j, nb_g - 1);
              const int b = g * N + n;
              const int row = ctl->alive[n] ? K : ctl->stoprow[n];
              const int vv = valid ? v : V - 1;
              tv[j] = ld_elem(target, ((int64_t)b * (K + 1) + row) * V + vv);
              bvv[j] = ld_elem(base, ((int64_t)b * K + min(row, K - 1)) * V + vv);
            }
            // residual mass r (into tv) and target mass p (into bvv), in place
#pragma unroll
            for (int j = 0; j < NCOL; ++j) {
              const int n = n0 + j;
              float r = 0.f, p = 0.f;
              if (valid && n < nb_g) {
                p = exp2f((tv[j] - ctl->Mt[n]) * k) / ctl->St[n];
                r = p;
                if (!ctl->alive[n])
                  r = fmaxf(p - exp2f((d[j] + bvv[j] - ctl->zM[n]) * k) / ctl->zS[n], 0.f);
              }
              tv[j] = r;
              bvv[j] = p;
            }
            bfly_sum2<NCOL>(tv, bvv, lane);
            float2* bk = sBucket + ((size_t)cl * 4 + q4) * N;
            if ((lane & (32 / NCOL - 1)) == 0) bk[n0 + lane / (32 / NCOL)] = make_float2(tv[0], bvv[0]);
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
              a.dpart[(((int64_t)par * (K + 1) + K) * N + n) * kMaxG + cta] = make_float2(R, P);
          }
          mark(g, K, 3);
          if (!grid_barrier()) {
            failed = true;
            break;
          }
          mark(g, K, 4);
          if (tid == 0) ctl->n_owned = 0;
          named_sync();
          {
            const int n = grp_n;
            const bool row_on = n < nb_g;
            float2 reg[MAXC];
            load_slice(a.dpart + (((int64_t)par * (K + 1) + K) * N + n) * kMaxG, row_on, reg,
                       make_float2(0.f, 0.f));
            float lr = 0.f, lp = 0.f;
#pragma unroll
            for (int j = 0; j < MAXC; ++j) {
              lr += reg[j].x;
              lp += reg[j].y;
            }
            float Rt = lr, Pt = lp;
#pragma unroll
            for (int off = TPB / 2; off >= 1; off >>= 1) {
              Rt += __shfl_xor_sync(FULL, Rt, off);
              Pt += __shfl_xor_sync(FULL, Pt, off);
            }
            const bool use_p = !(Rt > 0.f);
            const int b = g * N + n;
            const int row = (row_on && ctl->alive[n]) ? K : (row_on ? ctl->stoprow[n] : 0);
            const float u = philox_uniform(a.seed, a.cycle, (uint32_t)b, (uint32_t)row, TAG_RESAMPLE);
            const float tgt = u * (use_p ? Pt : Rt);
            int own;
            float before;
            bool fb;
            const bool holder = group_owner(reg, use_p ? 2 : 1, 0.f, tgt, own, before, fb);
            if (row_on) {
              if (grp_sub == 0) ctl->S[n] = use_p ? 1.f : 0.f;  // which mass the scan uses
              if (holder && own == cta) {
                const int slot = atomicAdd(&ctl->n_owned, 1);
                ctl->owned[slot] = n;
                ctl->obtarget[slot] = fb ? INFINITY : tgt - before;
              }
            }
          }
          named_sync();
          walk_and_assign(true);
          const int cnt = ctl->wcount[warp];
          for (int bs = 0; bs < cnt; bs += kOwnBatch) {
            int oo[kOwnBatch];
            float dv[kOwnBatch], tvv[kOwnBatch], bvv[kOwnBatch];
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) oo[j] = bs + j < cnt ? ctl->wlist[warp][bs + j] : -1;
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) {
              dv[j] = 0.f;
              if (oo[j] < 0) continue;
              const int cl = ctl->obucket[oo[j]] >> 2, n = ctl->owned[oo[j]];
              tmem_ld1(taddr + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(cl * N + n), &dv[j]);
            }
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) {  // loads from clamped valid addresses
              const int oj = oo[j] < 0 ? 0 : oo[j];
              const int cl = ctl->obucket[oj] >> 2, n = min(ctl->owned[oj], nb_g - 1);
              const int b = g * N + n;
              const int row = ctl->alive[n] ? K : ctl->stoprow[n];
              const int v = min((chunk0 + cl) * kCH + q4 * 32 + lane, V - 1);
              tvv[j] = ld_elem(target, ((int64_t)b * (K + 1) + row) * V + v);
              bvv[j] = ld_elem(base, ((int64_t)b * K + min(row, K - 1)) * V + v);
            }
#pragma unroll
            for (int j = 0; j < kOwnBatch; ++j) {
              if (oo[j] < 0) continue;
              const int cl = ctl->obucket[oo[j]] >> 2, n = ctl->owned[oo[j]];
              const int b = g * N + n;
              const bool use_p = ctl->S[n] != 0.f;
              const bool bonus = ctl->alive[n] != 0;
              const int row = bonus ? K : ctl->stoprow[n];
              const int v = (chunk0 + cl) * kCH + q4 * 32 + lane;
              float w = 0.f;
              if (v < V) {
                const float p = exp2f((tvv[j] - ctl->Mt[n]) * k) / ctl->St[n];
                w = p;
                if (!bonus && !use_p)
                  w = fmaxf(p - exp2f((dv[j] + bvv[j] - ctl->zM[n]) * k) / ctl->zS[n], 0.f);
              }
              const int wl = bucket_scan(w, ctl->obtarget[oo[j]]);
              if (lane == 0) a.out[(int64_t)b * (K + 1) + row] = (chunk0 + cl) * kCH + q4 * 32 + wl;
            }
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
      hdr->tok = 0;
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
  const size_t u = TC ? (size_t)nkb * N * 128 : (size_t)N * r * 4;
  s += (u + 1023) & ~size_t(1023);
  s += (size_t)kNBS * N * kCH * sizeof(T);
  s += (size_t)nc * 4 * N * sizeof(float2);
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

// Workspace body: trace | dpart | tpart | tokens | accf | stopinfo, each 256-byte aligned.
size_t cycle_trace_bytes(int K) { return a256(sizeof(uint64_t) * (size_t)(K + 2) * kTracePhases); }
size_t cycle_ws_bytes(int K, const CycleGeom& g) {
  const size_t part = sizeof(float2) * 2 * (size_t)(K + 1) * g.N * kMaxG;
  const size_t tok = sizeof(int32_t) * 2 * (size_t)K * g.N;
  return cycle_trace_bytes(K) + 2 * a256(part) + 2 * a256(tok) +
         a256(sizeof(StopInfo) * 2 * g.N);
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
  const size_t part = a256(sizeof(float2) * 2 * (size_t)(L.K + 1) * g.N * kMaxG);
  const size_t tok = a256(sizeof(int32_t) * 2 * (size_t)L.K * g.N);
  a.trace = L.trace ? reinterpret_cast<uint64_t*>(body) : nullptr;
  body += cycle_trace_bytes(L.K);
  a.dpart = reinterpret_cast<float2*>(body);
  a.tpart = reinterpret_cast<float2*>(body + part);
  a.tokens = reinterpret_cast<int32_t*>(body + 2 * part);
  a.accf = reinterpret_cast<int32_t*>(body + 2 * part + tok);
  a.stopinfo = reinterpret_cast<StopInfo*>(body + 2 * part + 2 * tok);
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
