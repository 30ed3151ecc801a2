// Stand-alone verification of a drafted block against the target's K+1 rows
// (aigest.pl "DeepSeek prezentuje DSpark", section "Jak działa spekulatywne
// dekodowanie DSpark?": keep the longest accepted prefix and add one token,
// preserving the target distribution exactly).  Reading: accept d_i iff
// u < min(1, p_i(d_i)/q_i(d_i)); at the first rejection draw from
// max(p_i - q_i, 0) (p_i if that is all zero); after K acceptances draw the
// bonus from target row K.  Greedy: accept while arg-max(target_i) == d_i.
//
// Kernels (all HBM-bound, 128-bit loads):
//   k_row_stats       per (row, segment): softmax partials (m, s) and arg-max
//   k_accept          per batch row: the accept chain, tau, stop row
//   k_residual_part   per (row, segment): residual / bonus mass
//   k_residual_pick   per batch row: two-level inverse CDF over the residual
#include "common.cuh"
#include "kernels.cuh"

namespace specdec {

namespace {

constexpr int kThreads = 256;

template <typename T>
struct Vec8 {
  float x[8];
};

// Load 8 consecutive elements starting at an 8-aligned index of a row whose
// base is 16-byte aligned.
SPEC_DEV void load8(const __nv_bfloat16* p, float* x) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(w[j] << 16);
    x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}
SPEC_DEV void load8(const float* p, float* x) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

struct BlockScratch {
  float m[kThreads / 32];
  float s[kThreads / 32];
  float av[kThreads / 32];
  int32_t ai[kThreads / 32];
};

// Reduce (m, s) and (max, argmax) over the block; result valid in thread 0.
SPEC_DEV void block_reduce_stats(float& m, float& s, float& av, int32_t& ai, float k,
                                 BlockScratch& sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float a2 = __shfl_xor_sync(0xffffffffu, av, o);
    const int32_t i2 = __shfl_xor_sync(0xffffffffu, ai, o);
    ms_combine(m, s, m2, s2, k);
    amax_combine(av, ai, a2, i2);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sh.m[w] = m;
    sh.s[w] = s;
    sh.av[w] = av;
    sh.ai[w] = ai;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int j = 1; j < kThreads / 32; ++j) {
      ms_combine(m, s, sh.m[j], sh.s[j], k);
      amax_combine(av, ai, sh.av[j], sh.ai[j]);
    }
  }
  __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_row_stats(const T* __restrict__ rows, int64_t nrows,
                                                        int V, int seg_len, int nseg, float k,
                                                        int greedy, RowPartial* __restrict__ out) {
  __shared__ BlockScratch sh;
  const int64_t total = nrows * nseg;
  for (int64_t job = blockIdx.x; job < total; job += gridDim.x) {
    const int64_t row = job / nseg;
    const int seg = (int)(job % nseg);
    const int lo = seg * seg_len, hi = min(V, lo + seg_len);
    const T* x = rows + row * (int64_t)V;
    float m = -INFINITY, s = 0.f, av = -INFINITY;
    int32_t ai = 0x7fffffff;
    // vector body: 8 elements per thread per step
    const int vlo = lo, vhi = lo + ((hi - lo) & ~7);
    for (int v = vlo + threadIdx.x * 8; v < vhi; v += kThreads * 8) {
      float e[8];
      load8(x + v, e);
      float lm = e[0];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (e[j] > av) {
          av = e[j];
          ai = v + j;
        }
        lm = fmaxf(lm, e[j]);
      }
      if (!greedy) {
        if (lm > m) {
          s *= exp2f((m - lm) * k);
          m = lm;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) s += exp2f((e[j] - m) * k);
      }
    }
    for (int v = vhi + threadIdx.x; v < hi; v += kThreads) {
      const float e = load_f(x, v);
      if (e > av) {
        av = e;
        ai = v;
      }
      if (!greedy) {
        if (e > m) {
          s *= exp2f((m - e) * k);
          m = e;
        }
        s += exp2f((e - m) * k);
      }
    }
    block_reduce_stats(m, s, av, ai, k, sh);
    if (threadIdx.x == 0) out[job] = RowPartial{m, s, av, ai};
  }
}

// Combine the nseg partials of one row.
SPEC_DEV RowPartial combine_row(const RowPartial* p, int nseg, float k) {
  RowPartial r = p[0];
  for (int j = 1; j < nseg; ++j) {
    ms_combine(r.m, r.s, p[j].m, p[j].s, k);
    amax_combine(r.amax, r.aidx, p[j].amax, p[j].aidx);
  }
  return r;
}

template <typename T, typename TD>
__global__ void k_accept(const T* __restrict__ target, const TD* __restrict__ draft_logits,
                         const int32_t* __restrict__ draft, const RowPartial* __restrict__ tstats,
                         const RowPartial* __restrict__ dstats, int B, int K, int V, int nseg,
                         float k, int greedy, uint64_t seed, uint64_t cycle, uint32_t row0,
                         int32_t* __restrict__ out, int32_t* __restrict__ tau,
                         float* __restrict__ p_draft, float* __restrict__ q_draft,
                         StopInfo* __restrict__ stop, WsHeader* hdr) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const float nanv = __int_as_float(0x7fc00000);
  int j = K;
  for (int i = 0; i <= K; ++i) out[(int64_t)b * (K + 1) + i] = -1;
  if (p_draft)
    for (int i = 0; i < K; ++i) p_draft[(int64_t)b * K + i] = nanv;
  if (q_draft && greedy)
    for (int i = 0; i < K; ++i) q_draft[(int64_t)b * K + i] = nanv;
  StopInfo si{K, 0.f, 1.f, 0.f, 1.f};
  for (int i = 0; i < K; ++i) {
    int d = draft[(int64_t)b * K + i];
    if (d < 0 || d >= V) {
      record_error(hdr, SPEC_ERR_TOKEN_RANGE, SITE_TOKEN_RANGE, b, d);
      d = 0;
    }
    const RowPartial tp = combine_row(tstats + ((int64_t)b * (K + 1) + i) * nseg, nseg, k);
    if (greedy) {
      if (tp.aidx == d) {
        out[(int64_t)b * (K + 1) + i] = d;
        continue;
      }
      out[(int64_t)b * (K + 1) + i] = tp.aidx;
      j = i;
      break;
    }
    const RowPartial dp = combine_row(dstats + ((int64_t)b * K + i) * nseg, nseg, k);
    const float td = load_f(target, ((int64_t)b * (K + 1) + i) * V + d);
    const float zd = load_f(draft_logits, ((int64_t)b * K + i) * V + d);
    const float pd = exp2f((td - tp.m) * k) / tp.s;
    const float qd = exp2f((zd - dp.m) * k) / dp.s;
    if (p_draft) p_draft[(int64_t)b * K + i] = pd;
    // ratio p/q from one exponent of small magnitude
    float a = exp2f(((td - tp.m) - (zd - dp.m)) * k) * (dp.s / tp.s);
    a = fminf(a, 1.0f);
    const float u = philox_uniform(seed, cycle, row0 + (uint32_t)b, (uint32_t)i, TAG_ACCEPT);
    if (u < a) {
      out[(int64_t)b * (K + 1) + i] = d;
      continue;
    }
    j = i;
    si = StopInfo{i, tp.m, tp.s, dp.m, dp.s};
    break;
  }
  if (!greedy && q_draft) {
    for (int i = 0; i < K; ++i) {
      int d = draft[(int64_t)b * K + i];
      d = (d < 0 || d >= V) ? 0 : d;
      const RowPartial dp = combine_row(dstats + ((int64_t)b * K + i) * nseg, nseg, k);
      const float zd = load_f(draft_logits, ((int64_t)b * K + i) * V + d);
      q_draft[(int64_t)b * K + i] = exp2f((zd - dp.m) * k) / dp.s;
    }
  }
  if (j == K) {
    const RowPartial tp = combine_row(tstats + ((int64_t)b * (K + 1) + K) * nseg, nseg, k);
    if (greedy) out[(int64_t)b * (K + 1) + K] = tp.aidx;
    si = StopInfo{K, tp.m, tp.s, 0.f, 1.f};
  }
  tau[b] = j + 1;
  stop[b] = si;
}

template <typename T, typename TD>
__global__ void __launch_bounds__(kThreads) k_residual_part(
    const T* __restrict__ target, const TD* __restrict__ draft_logits,
    const StopInfo* __restrict__ stop, int B, int K, int V, int seg_len, int nseg, float k,
    float2* __restrict__ part) {
  __shared__ float red[2][kThreads / 32];
  const int64_t total = (int64_t)B * nseg;
  for (int64_t job = blockIdx.x; job < total; job += gridDim.x) {
    const int b = (int)(job / nseg), seg = (int)(job % nseg);
    const StopInfo si = stop[b];
    const int lo = seg * seg_len, hi = min(V, lo + seg_len);
    const T* t = target + ((int64_t)b * (K + 1) + si.j) * V;
    const TD* z = si.j < K ? draft_logits + ((int64_t)b * K + si.j) * V : nullptr;
    const float inv_st = 1.0f / si.st, inv_sz = 1.0f / si.sz;
    float R = 0.f, P = 0.f;
    for (int v = lo + threadIdx.x; v < hi; v += kThreads) {
      const float p = exp2f((load_f(t, v) - si.mt) * k) * inv_st;
      float r = p;
      if (z) r = fmaxf(p - exp2f((load_f(z, v) - si.mz) * k) * inv_sz, 0.f);
      R += r;
      P += p;
    }
    R = warp_sum(R);
    P = warp_sum(P);
    if ((threadIdx.x & 31) == 0) {
      red[0][threadIdx.x >> 5] = R;
      red[1][threadIdx.x >> 5] = P;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float a = 0.f, c = 0.f;
      for (int w = 0; w < kThreads / 32; ++w) {
        a += red[0][w];
        c += red[1][w];
      }
      part[job] = make_float2(a, c);
    }
    __syncthreads();
  }
}

template <typename T, typename TD>
__global__ void __launch_bounds__(kThreads) k_residual_pick(
    const T* __restrict__ target, const TD* __restrict__ draft_logits,
    const StopInfo* __restrict__ stop, const float2* __restrict__ part, int B, int K, int V,
    int seg_len, int nseg, float k, uint64_t seed, uint64_t cycle, uint32_t row0,
    int32_t* __restrict__ out) {
  __shared__ float sh_target;
  __shared__ int sh_seg, sh_use_p;
  __shared__ float wsum[kThreads / 32];
  __shared__ int wbest[kThreads / 32], wlast[kThreads / 32];
  const int b = blockIdx.x;
  if (b >= B) return;
  const StopInfo si = stop[b];
  if (threadIdx.x == 0) {
    const float2* pp = part + (int64_t)b * nseg;
    float R = 0.f, P = 0.f;
    for (int s = 0; s < nseg; ++s) {
      R += pp[s].x;
      P += pp[s].y;
    }
    const int use_p = !(R > 0.f);
    const float tot = use_p ? P : R;
    const float u = philox_uniform(seed, cycle, row0 + (uint32_t)b, (uint32_t)si.j, TAG_RESAMPLE);
    const float tgt = u * tot;
    float c = 0.f;
    int seg = -1, lastpos = 0;
    for (int s = 0; s < nseg; ++s) {
      const float w = use_p ? pp[s].y : pp[s].x;
      if (w > 0.f) lastpos = s;
      if (c + w > tgt) {
        seg = s;
        break;
      }
      c += w;
    }
    if (seg < 0) {  // rounding pushed the target past the last edge
      seg = lastpos;
      c = 0.f;
      for (int s = 0; s < lastpos; ++s) c += use_p ? pp[s].y : pp[s].x;
    }
    sh_seg = seg;
    sh_use_p = use_p;
    sh_target = tgt - c;
  }
  __syncthreads();
  const int seg = sh_seg, use_p = sh_use_p;
  const float tgt = sh_target;
  const int lo = seg * seg_len, hi = min(V, lo + seg_len);
  const T* t = target + ((int64_t)b * (K + 1) + si.j) * V;
  const TD* z = (si.j < K && !use_p) ? draft_logits + ((int64_t)b * K + si.j) * V : nullptr;
  const float inv_st = 1.0f / si.st, inv_sz = 1.0f / si.sz;
  // each thread owns a contiguous sub-range of the segment
  const int per = (hi - lo + kThreads - 1) / kThreads;
  const int mlo = lo + threadIdx.x * per, mhi = min(hi, mlo + per);
  auto weight = [&](int v) {
    const float p = exp2f((load_f(t, v) - si.mt) * k) * inv_st;
    if (!z) return p;
    return fmaxf(p - exp2f((load_f(z, v) - si.mz) * k) * inv_sz, 0.f);
  };
  float local = 0.f;
  for (int v = mlo; v < mhi; ++v) local += weight(v);
  // exclusive block scan of the per-thread sums, in thread (= token) order
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  float before = 0.f;
  for (int j = 0; j < w; ++j) before += wsum[j];
  float c = before + incl - local;
  int best = 0x7fffffff, last = -1;
  for (int v = mlo; v < mhi; ++v) {
    const float wv = weight(v);
    if (wv > 0.f) last = v;
    c += wv;
    if (c > tgt) {
      best = v;
      break;
    }
  }
  // block-wide: smallest crossing index, else the last index with mass
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
    last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
  }
  __syncthreads();
  if (lane == 0) {
    wbest[w] = best;
    wlast[w] = last;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int bb = 0x7fffffff, ll = -1;
    for (int j = 0; j < kThreads / 32; ++j) {
      bb = min(bb, wbest[j]);
      ll = max(ll, wlast[j]);
    }
    out[(int64_t)b * (K + 1) + si.j] = bb != 0x7fffffff ? bb : (ll >= 0 ? ll : lo);
  }
}

}  // namespace

int verify_seg_len(int V) { return V <= 16384 ? V : 8192; }

template <typename T, typename TD>
cudaError_t launch_verify(const T* target, const TD* draft_logits, const int32_t* draft,
                          int32_t* out, int32_t* tau, float* p_draft, float* q_draft, int B,
                          int K, int V, float temperature, int greedy, uint64_t seed,
                          uint64_t cycle, uint32_t row0, uint8_t* ws_body, WsHeader* hdr,
                          int num_sms,
                          cudaStream_t st, int* launches) {
  const int seg_len = verify_seg_len(V);
  const int nseg = (V + seg_len - 1) / seg_len;
  const float k = greedy ? 1.0f : 1.4426950408889634f / temperature;
  // every region starts on a 256-byte boundary
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t o_t = 0;
  const size_t o_d = a256(o_t + sizeof(RowPartial) * (size_t)B * (K + 1) * nseg);
  const size_t o_s = a256(o_d + sizeof(RowPartial) * (size_t)B * K * nseg);
  const size_t o_p = a256(o_s + sizeof(StopInfo) * (size_t)B);
  RowPartial* tstats = reinterpret_cast<RowPartial*>(ws_body + o_t);
  RowPartial* dstats = reinterpret_cast<RowPartial*>(ws_body + o_d);
  StopInfo* stop = reinterpret_cast<StopInfo*>(ws_body + o_s);
  float2* part = reinterpret_cast<float2*>(ws_body + o_p);
  const int cap = num_sms * 8;
  auto grid_for = [&](int64_t jobs) { return (int)std::min<int64_t>(jobs, cap); };
  k_row_stats<T><<<grid_for((int64_t)B * (K + 1) * nseg), kThreads, 0, st>>>(
      target, (int64_t)B * (K + 1), V, seg_len, nseg, k, greedy, tstats);
  ++*launches;
  if (!greedy) {
    k_row_stats<TD><<<grid_for((int64_t)B * K * nseg), kThreads, 0, st>>>(
        draft_logits, (int64_t)B * K, V, seg_len, nseg, k, 0, dstats);
    ++*launches;
  }
  k_accept<T, TD><<<(B + 127) / 128, 128, 0, st>>>(target, draft_logits, draft, tstats, dstats, B,
                                                   K, V, nseg, k, greedy, seed, cycle, row0, out, tau,
                                                   p_draft, q_draft, stop, hdr);
  ++*launches;
  if (!greedy) {
    k_residual_part<T, TD><<<grid_for((int64_t)B * nseg), kThreads, 0, st>>>(
        target, draft_logits, stop, B, K, V, seg_len, nseg, k, part);
    k_residual_pick<T, TD><<<B, kThreads, 0, st>>>(target, draft_logits, stop, part, B, K, V,
                                                   seg_len, nseg, k, seed, cycle, row0, out);
    *launches += 2;
  }
  return cudaGetLastError();
}

size_t verify_ws_bytes(int B, int K, int V) {
  const int seg_len = verify_seg_len(V);
  const int64_t nseg = (V + seg_len - 1) / seg_len;
  auto a256 = [](size_t x) { return (x + 255) & ~size_t(255); };
  return a256(sizeof(RowPartial) * (size_t)B * (K + 1) * nseg) +
         a256(sizeof(RowPartial) * (size_t)B * K * nseg) + a256(sizeof(StopInfo) * (size_t)B) +
         a256(sizeof(float2) * (size_t)B * nseg);
}

#define INST(T, TD)                                                                           \
  template cudaError_t launch_verify<T, TD>(const T*, const TD*, const int32_t*, int32_t*,    \
                                            int32_t*, float*, float*, int, int, int, float,   \
                                            int, uint64_t, uint64_t, uint32_t, uint8_t*,      \
                                            WsHeader*, int, cudaStream_t, int*);
INST(float, float)
INST(__nv_bfloat16, __nv_bfloat16)
INST(__nv_bfloat16, float)
INST(float, __nv_bfloat16)
#undef INST

}  // namespace specdec
