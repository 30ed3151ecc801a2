// Verification of a drafted block in one persistent launch with early exit
// (aigest.pl "DeepSeek prezentuje DSpark", section "Jak działa spekulatywne
// dekodowanie DSpark?": keep the longest accepted prefix and add one token,
// with the target distribution preserved exactly).  Reading: accept d_i iff
// u < min(1, p_i(d_i) / q_i(d_i)); at the first rejection draw from
// max(p_i - q_i, 0) normalised (p_i if that is all zero); after K_b
// acceptances draw the bonus token from target row K_b.  Greedy: accept while
// arg-max(target_i) == d_i, emit the target arg-max at the first mismatch
// (row K_b's after K_b matches).
//
// Every CTA owns one slice of the vocabulary (a multiple of 32 tokens) for
// every row.  Positions are decided in waves of kWave: in a wave each CTA
// reads, for every row still verifying, its slice of the target and draft
// rows of the wave's positions (and the bonus row when the wave reaches K_b),
// and writes per-slice softmax statistics; after a grid barrier the row's
// reducer CTA (row b % G) combines them, runs the accept tests in position
// order and publishes the row's state with a tag.  A row that stopped at j
// gets one more pass in the next wave: the residual max(p_j - q_j, 0) in
// 32-token buckets per slice; the reducer then draws the token by a
// two-level inverse CDF (slice totals, the owner slice's buckets, 32 logits).
// Rows past their stop are never read again; draft and target rows beyond a
// row's stop are never read at all.
#include "common.cuh"
#include "kernels.cuh"

namespace specdec {

namespace {

constexpr int kVThreads = 512;
constexpr int kVWarps = kVThreads / 32;
constexpr int kWave = 4;             // positions decided per grid round
constexpr int kMaxRowsV = 4096;      // rows whose state one CTA keeps in shared memory
constexpr int kMaxGV = 160;          // CTAs a launch may use
constexpr int kEV = (kMaxGV + 31) / 32;
constexpr int kMaxPiecesV = 8;       // 8-element pieces per lane and slice (bonus pass)
constexpr unsigned FULLV = 0xffffffffu;
constexpr int kVTraceWaves = 64, kVTraceSlots = 8;

enum : int32_t { ROW_VERIFYING = 0, ROW_STOPPED = 1, ROW_DONE = 2 };

// A row's state after a wave, published by its reducer.
struct alignas(16) RecV {
  int32_t kind;   // ROW_VERIFYING, ROW_STOPPED (residual pending at j) or ROW_DONE
  int32_t j;      // stop row
  int32_t pad[2];
  float4 st;      // stop row statistics: target (max, sum), draft (max, sum)
};

struct ArgsV {
  const void* target;
  const void* draft_logits;
  const int32_t* draft;
  const int32_t* vlen;  // [B] verify length K_b (1..K), or null (K)
  int32_t* out;
  int32_t* tau;
  float* p_draft;
  float* q_draft;
  WsHeader* hdr;
  float4* part;   // [B][kWave][G] target (max, sum), draft (max, sum); greedy (max, idx)
  float2* bpart;  // [B][G] bonus row: slice (max, sum); greedy (max, idx)
  float2* fin;    // [B][G] residual: slice (R, P)
  float2* gbk;    // [B][G][nbk] 32-token buckets: residual (r, p); bonus (0, p / slice max)
  RecV* rec;      // [B]
  uint64_t* rtag; // [B] (tag << 32) | kind
  uint64_t* trace;  // [kVTraceWaves][kVTraceSlots] device timeline (CTA 0 and maxima), or null
  int B, K, V, G, seg, nbk, greedy;
  int S;          // slots of each warp's ring
  int slotb;      // bytes of one slot: the target slice, then (at doff) the draft slice
  int doff;
  float k;        // log2(e) / T (1 in greedy mode)
  uint64_t seed, cycle, spin;
  uint32_t row0;
};

// Eight logits kept as loaded (bf16: one 16-byte word; fp32: two), widened on use.
template <typename T>
struct Raw8 {
  uint4 w[sizeof(T) / 2];
};
template <typename T>
SPEC_DEV void ldraw(const T* p, Raw8<T>& r, bool stream) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int h = 0; h < (int)(sizeof(T) / 2); ++h) r.w[h] = stream ? __ldcs(q + h) : __ldg(q + h);
}
template <typename T>
SPEC_DEV float elem(const Raw8<T>& r, int e);
template <>
SPEC_DEV float elem<__nv_bfloat16>(const Raw8<__nv_bfloat16>& r, int e) {
  const uint32_t x = e < 4 ? (e < 2 ? r.w[0].x : r.w[0].y) : (e < 6 ? r.w[0].z : r.w[0].w);
  return __uint_as_float((e & 1) ? (x & 0xFFFF0000u) : (x << 16));
}
template <>
SPEC_DEV float elem<float>(const Raw8<float>& r, int e) {
  const uint4 h = r.w[e >> 2];
  const uint32_t x = (e & 3) == 0 ? h.x : ((e & 3) == 1 ? h.y : ((e & 3) == 2 ? h.z : h.w));
  return __uint_as_float(x);
}

// Eight logits from shared memory (a slice staged by a bulk copy).
template <typename T>
SPEC_DEV Raw8<T> load_raw8(const T* p) {
  Raw8<T> r;
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int h = 0; h < (int)(sizeof(T) / 2); ++h) r.w[h] = q[h];
  return r;
}

// Max of the 8 logits of a piece (bf16: packed pair maxima, exact).
SPEC_DEV float piece_max(const Raw8<__nv_bfloat16>& r) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.w[0]);
  const __nv_bfloat162 m = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
  return fmaxf(__low2float(m), __high2float(m));
}
SPEC_DEV float piece_max(const Raw8<float>& r) {
  float m = -INFINITY;
#pragma unroll
  for (int e = 0; e < 8; ++e) m = fmaxf(m, elem(r, e));
  return m;
}
// sum over the piece of exp2(x k - mk) (= exp2((x - m) k) with mk = m k),
// two partial sums
template <typename T>
SPEC_DEV float piece_sumexp(const Raw8<T>& r, float mk, float k) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    s0 += fexp2(fmaf(elem(r, e), k, -mk));
    s1 += fexp2(fmaf(elem(r, e + 1), k, -mk));
  }
  return s0 + s1;
}
// A piece of eight -inf logits: fills the pieces a lane does not hold, so
// that the per-lane statistics need no per-piece checks.
template <typename T>
SPEC_DEV Raw8<T> neg_inf_raw8() {
  Raw8<T> r;
  const uint32_t v = sizeof(T) == 2 ? 0xFF80FF80u : 0xFF800000u;
#pragma unroll
  for (int h = 0; h < (int)(sizeof(T) / 2); ++h) r.w[h] = make_uint4(v, v, v, v);
  return r;
}
// (max, sum exp2((x - max) k)) of the kLanePieces pieces held by this lane
// (pieces it does not hold are -inf), folded into (m, s)
constexpr int kLanePieces = 4;
template <typename T>
SPEC_DEV void lane_ms(const Raw8<T>* x, float k, float& m, float& s) {
  float mm = -INFINITY;
#pragma unroll
  for (int u = 0; u < kLanePieces; ++u) mm = fmaxf(mm, piece_max(x[u]));
  if (mm > -INFINITY) {
    const float mk = mm * k;
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < kLanePieces; ++u) ss += piece_sumexp(x[u], mk, k);
    ms_combine(m, s, mm, ss, k);
  }
}

SPEC_DEV uint64_t policy_evict_normal_v() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Verify length K_b of row b (K without a per-row array), clamped to 1..K.
SPEC_DEV int vrow_len(const ArgsV& a, int b) {
  return a.vlen ? min(max(__ldg(a.vlen + b), 1), a.K) : a.K;
}

// Warp combine of (max, sum) pairs held one per lane.
SPEC_DEV void warp_ms(float& m, float& s, float k) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float m2 = __shfl_xor_sync(FULLV, m, o);
    const float s2 = __shfl_xor_sync(FULLV, s, o);
    ms_combine(m, s, m2, s2, k);
  }
}
SPEC_DEV void warp_amax(float& v, int32_t& i) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float v2 = __shfl_xor_sync(FULLV, v, o);
    const int32_t i2 = __shfl_xor_sync(FULLV, i, o);
    amax_combine(v, i, v2, i2);
  }
}

// First lane whose inclusive prefix of w exceeds tin, else the last lane with
// positive weight (0 if none).
SPEC_DEV int scan32(float w, float tin, int lane) {
  float incl = w;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(FULLV, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned cross = __ballot_sync(FULLV, incl > tin);
  if (cross) return __ffs(cross) - 1;
  const unsigned pos = __ballot_sync(FULLV, w > 0.f);
  return pos ? 31 - __clz(pos) : 0;
}

template <typename T, typename TD>
__global__ void __launch_bounds__(kVThreads, 1) k_verify_ee(const __grid_constant__ ArgsV a) {
  extern __shared__ __align__(16) uint8_t smem_v[];
  const int B = a.B, K = a.K, V = a.V, G = a.G;
  float4* sst = reinterpret_cast<float4*>(smem_v);                   // [B] stop-row statistics
  int16_t* skb = reinterpret_cast<int16_t*>(sst + B);                // [B] verify length
  int16_t* sj = skb + B;                                             // [B] stop row
  int16_t* sready = sj + B;  // [B] a draw of this CTA pending: its data is visible after this grid barrier
  int8_t* skind = reinterpret_cast<int8_t*>(sready + B);             // [B] row state
  int8_t* sdk = skind + B;                                           // [B] pending draw: residual or bonus
  const int S = a.S;
  uint64_t* wbar_all = reinterpret_cast<uint64_t*>(smem_v + ((size_t)B * 24 + 15) / 16 * 16);
  int32_t* wq_all = reinterpret_cast<int32_t*>(wbar_all + kVWarps * S);  // [warp][S] item
  int32_t* wrow_all = wq_all + kVWarps * S;                               // [warp][S] logit row
  uint8_t* ring_all = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(wrow_all + kVWarps * S) + 127) & ~uintptr_t(127));
  __shared__ float4 cst[kWave];          // decide: combined statistics per position
  __shared__ float2 ctd[kWave];          // decide: (target, draft) logit at the draft token
  __shared__ int32_t cdt[kWave];         // decide: draft token
  __shared__ float2 cbonus;              // greedy decide: bonus (max, idx)
  __shared__ int32_t abort_local, n_active, item_ctr;

  const T* target = reinterpret_cast<const T*>(a.target);
  const TD* dl = reinterpret_cast<const TD*>(a.draft_logits);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  uint64_t* wbar = wbar_all + warp * S;
  int32_t* wq = wq_all + warp * S;
  int32_t* wrow = wrow_all + warp * S;
  uint8_t* ring = ring_all + (size_t)warp * S * a.slotb;
  const uint32_t slotb = (uint32_t)a.slotb, doff = (uint32_t)a.doff;
  const uint64_t pol = policy_evict_normal_v();
  uint32_t issued = 0, consumed = 0;  // this warp's ring: copies issued / consumed
  bool failed_copy = false;
  const int lo = cta * a.seg, hi = min(V, lo + a.seg);
  const int np = (hi - lo) / 8;            // 8-element pieces of this CTA's slice
  const uint32_t tbytes = (uint32_t)((hi - lo) * sizeof(T)), dbytes = (uint32_t)((hi - lo) * sizeof(TD));
  const float k = a.k;
  const float NaNf = __int_as_float(0x7fc00000);
  WsHeader* hdr = a.hdr;
  const uint32_t ev0 = ld_volatile_u32(&hdr->events);
  uint32_t nbar = 0;
  bool failed = false;
  // timeline: slot 0 read start, 1 arrive, 2 barrier passed, 3 decided, 4 hop
  // done (CTA 0); 5 latest arrive, 6 latest publication (all CTAs)
  auto mark = [&](int wv, int slot) {
    if (a.trace && tid == 0 && wv < kVTraceWaves) {
      const uint64_t t = globaltimer_ns();
      if (slot >= 5)
        atomicMax(reinterpret_cast<unsigned long long*>(a.trace) + wv * kVTraceSlots + slot,
                  (unsigned long long)t);
      else if (cta == 0)
        a.trace[wv * kVTraceSlots + slot] = t;
    }
  };

  for (int b = tid; b < B; b += kVThreads) {
    skb[b] = (int16_t)vrow_len(a, b);
    sj[b] = 0;
    skind[b] = ROW_VERIFYING;
    sready[b] = 0;
    sdk[b] = 0;
    sst[b] = make_float4(0.f, 1.f, 0.f, 1.f);
  }
  if (tid == 0) abort_local = 0;
  if (tid < kVWarps * S) mbar_init(&wbar_all[tid], 1);
  if (tid == 0) fence_mbar_init();
  if (cta == 0) {  // outputs past each row's stop keep these values
    for (int idx = tid; idx < B * (K + 1); idx += kVThreads) a.out[idx] = -1;
    for (int idx = tid; idx < B * K; idx += kVThreads) {
      if (a.p_draft) a.p_draft[idx] = NaNf;
      if (a.q_draft) a.q_draft[idx] = NaNf;
    }
    if (a.vlen)
      for (int b = tid; b < B; b += kVThreads) {
        const int32_t raw = __ldg(a.vlen + b);
        if (raw < 1 || raw > K) record_error(hdr, SPEC_ERR_INVALID_ARG, SITE_TOKEN_RANGE, b, raw);
      }
  }
  __syncthreads();

  // ---- grid barrier (release / acquire on the launch counter, bounded)
  auto grid_arrive = [&]() {
    __syncthreads();
    if (tid == 0) {
      red_release_add_u32(&hdr->bar, 1u);
    }
    ++nbar;
  };
  auto grid_wait = [&]() {
    if (tid == 0 &&
        !grid_wait_count(hdr, &hdr->bar, nbar * (uint32_t)G, a.spin, SITE_GRID_BARRIER))
      abort_local = 1;
    __syncthreads();
    return abort_local == 0;
  };

  // ---- one draw by one warp: residual at the stop row (kind ROW_STOPPED) or
  // the bonus from row K_b; writes out[b][row]
  auto draw = [&](int b, int kind) {
    const int c0 = lane * kEV;
    const bool bonus = kind != ROW_STOPPED;
    const int row = bonus ? skb[b] : sj[b];
    const float4 st = sst[b];
    float w[kEV], mloc[kEV];
    float M = -INFINITY;
    bool use_p = false;
    if (bonus) {
#pragma unroll
      for (int t = 0; t < kEV; ++t) {
        const float2 v = c0 + t < G ? __ldcg(a.bpart + (size_t)b * G + c0 + t) : make_float2(-INFINITY, 0.f);
        mloc[t] = v.x;
        w[t] = v.y;
        M = fmaxf(M, v.x);
      }
      M = warp_max(M);
#pragma unroll
      for (int t = 0; t < kEV; ++t) w[t] = w[t] > 0.f ? w[t] * fexp2((mloc[t] - M) * k) : 0.f;
    } else {
      float R = 0.f;
      float2 v[kEV];
#pragma unroll
      for (int t = 0; t < kEV; ++t) {
        v[t] = c0 + t < G ? __ldcg(a.fin + (size_t)b * G + c0 + t) : make_float2(0.f, 0.f);
        R += v[t].x;
      }
      use_p = !(warp_sum(R) > 0.f);
#pragma unroll
      for (int t = 0; t < kEV; ++t) w[t] = use_p ? v[t].y : v[t].x;
    }
    float loc = 0.f;
#pragma unroll
    for (int t = 0; t < kEV; ++t) loc += w[t];
    float incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(FULLV, incl, o);
      if (lane >= o) incl += y;
    }
    const float total = __shfl_sync(FULLV, incl, 31);
    const float u = philox_uniform(a.seed, a.cycle, a.row0 + (uint32_t)b, (uint32_t)row, TAG_RESAMPLE);
    const float tgt = u * total;
    float cum = incl - loc, before = 0.f;
    int found = 0x7fffffff, lastpos = -1;
#pragma unroll
    for (int t = 0; t < kEV; ++t) {
      if (w[t] > 0.f) lastpos = c0 + t;
      if (found == 0x7fffffff && w[t] > 0.f && cum + w[t] > tgt) {
        found = c0 + t;
        before = cum;
      }
      cum += w[t];
    }
    int own = found;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) own = min(own, __shfl_xor_sync(FULLV, own, o));
    int lp = lastpos;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) lp = max(lp, __shfl_xor_sync(FULLV, lp, o));
    const bool fb = own == 0x7fffffff;
    const float bown = __shfl_sync(FULLV, before, fb ? 0 : own / kEV);
    const int o = fb ? max(lp, 0) : own;
    float tin = fb ? INFINITY : tgt - bown;
    // bonus buckets hold masses relative to the owner slice's own max
    float mo = 0.f;
    if (bonus) {
      const float mown = __ldcg(a.bpart + (size_t)b * G + o).x;
      mo = mown;
      const float sc = fexp2((mown - M) * k);
      tin = sc > 0.f ? tin / sc : INFINITY;
    }
    // the owner slice's buckets, ascending
    const float2* bk = a.gbk + ((size_t)b * G + o) * a.nbk;
    float carry = 0.f, tin_in = INFINITY;
    int pick = -1, lastb = -1;
    for (int b0 = 0; b0 < a.nbk && pick < 0; b0 += 32) {
      const int q = b0 + lane;
      float wb = 0.f;
      if (q < a.nbk) {
        const float2 pv = __ldcg(bk + q);
        wb = bonus ? pv.y : (use_p ? pv.y : pv.x);
      }
      float in2 = wb;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(FULLV, in2, off);
        if (lane >= off) in2 += y;
      }
      const unsigned cross = __ballot_sync(FULLV, carry + in2 > tin);
      const unsigned pos = __ballot_sync(FULLV, wb > 0.f);
      if (pos) lastb = b0 + 31 - __clz(pos);
      if (cross) {
        const int l = __ffs(cross) - 1;
        pick = b0 + l;
        tin_in = tin - (carry + __shfl_sync(FULLV, in2 - wb, l));
      }
      carry += __shfl_sync(FULLV, in2, 31);
    }
    if (pick < 0) {
      pick = lastb < 0 ? 0 : lastb;
      tin_in = INFINITY;
    }
    // the bucket's 32 logits, with the same expressions as the bucket pass
    const int v0 = o * a.seg + pick * 32;
    const int v = v0 + lane;
    const bool valid = v < V;
    const int vc = min(v, V - 1);
    const float tv = load_f(target, ((int64_t)b * (K + 1) + row) * V + vc);
    float wt;
    if (bonus) {
      wt = valid ? fexp2((tv - mo) * k) : 0.f;
    } else {
      const float p = fexp2((tv - st.x) * k) * (1.0f / st.y);
      float r = p;
      if (!use_p) {
        const float zv = load_f(dl, ((int64_t)b * K + row) * V + vc);
        r = fmaxf(p - fexp2((zv - st.z) * k) * (1.0f / st.w), 0.f);
      }
      wt = valid ? r : 0.f;
    }
    const int wl = scan32(wt, tin_in, lane);
    if (lane == 0) a.out[(int64_t)b * (K + 1) + row] = v0 + wl;
  };
  // this CTA's pending draws whose data became visible at grid barrier
  // `upto` or earlier, one row per warp
  auto run_draws = [&](int upto) {
    __syncthreads();
    for (int m = warp; cta + m * G < B; m += kVWarps) {
      const int b = cta + m * G;
      const int r = sready[b];
      if (r > 0 && r <= upto) {
        draw(b, sdk[b]);
        __syncwarp();
        if (lane == 0) sready[b] = 0;
      }
    }
    __syncthreads();
  };
  // queue a draw of row b (this CTA is its reducer)
  auto queue_draw = [&](int b, int kind, int ready) {
    sdk[b] = (int8_t)kind;
    sready[b] = (int16_t)ready;
  };

  int w = 0;
  for (;; ++w) {
    const int i0 = w * kWave;
    // ------------------------------------------------------------- read phase
    // items: first this CTA's rows with a draw whose data is visible; then
    // (row b, slot s): s < kWave: position i0 + s of a verifying row;
    // s == kWave: its bonus row (when the wave reaches K_b) or, for a row
    // that stopped in the previous wave, the residual at its stop row.  The
    // slices of the wave are prefetched into L2 first; warps take items from
    // a shared counter.
    mark(w, 0);
    // ------------------------------------------------------------- read phase
    // items: first this CTA's rows with a draw whose data is visible; then
    // (row b, slot s): s < kWave: position i0 + s of a verifying row;
    // s == kWave: its bonus row (when the wave reaches K_b) or, for a row
    // that stopped in the previous wave, the residual at its stop row.  Warps
    // take items from a shared counter and keep up to S of them in flight:
    // bulk copies of the CTA's slices into the warp's ring in shared memory.
    const int nown = cta < B ? (B - cta + G - 1) / G : 0;
    const int nitems = nown + B * (kWave + 1);
    if (tid == 0) item_ctr = 0;
    __syncthreads();
    {
      bool more = true;
      for (;;) {
        while (more && issued - consumed < (uint32_t)S) {
          int id = 0;
          if (lane == 0) id = atomicAdd(&item_ctr, 1);
          id = __shfl_sync(FULLV, id, 0);
          if (id >= nitems) {
            more = false;
            break;
          }
          if (id < nown) {  // a draw
            const int b = cta + id * G;
            const int r = sready[b];
            if (r > 0 && r <= (int)nbar) {
              draw(b, sdk[b]);
              __syncwarp();
              if (lane == 0) sready[b] = 0;
            }
            continue;
          }
          id -= nown;
          const int b = id / (kWave + 1), sl = id % (kWave + 1);
          const int kind = skind[b], kb = skb[b];
          int ik = -1, trow = 0;  // item kind: 0 statistics, 1 bonus, 2 residual
          if (kind == ROW_VERIFYING) {
            if (sl < kWave && i0 + sl < kb) {
              ik = 0;
              trow = i0 + sl;
            } else if (sl == kWave && kb <= i0 + kWave) {
              ik = 1;
              trow = kb;
            }
          } else if (kind == ROW_STOPPED && sl == kWave) {
            ik = 2;
            trow = sj[b];
          }
          if (ik < 0) continue;
          const uint32_t slot = issued % (uint32_t)S;
          const bool with_d = ik == 2 || (ik == 0 && !a.greedy);
          if (lane == 0) {
            uint8_t* dst = ring + slot * slotb;
            mbar_arrive_expect_tx(&wbar[slot], tbytes + (with_d ? dbytes : 0u));
            bulk_load(dst, target + ((int64_t)b * (K + 1) + trow) * V + lo, tbytes, &wbar[slot],
                      pol);
            if (with_d)
              bulk_load(dst + doff, dl + ((int64_t)b * K + trow) * V + lo, dbytes, &wbar[slot], pol);
            wq[slot] = (b << 4) | (ik << 2);
            wrow[slot] = trow;
          }
          ++issued;
          __syncwarp();
        }
        if (issued == consumed) break;
        const uint32_t slot = consumed % (uint32_t)S;
        const bool landed = mbar_wait_bounded(&wbar[slot], (consumed / (uint32_t)S) & 1, a.spin,
                                              &hdr->abort);
        if (!__all_sync(FULLV, landed)) {
          if (lane == 0 && !ld_volatile_u32(&hdr->abort))
            record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, cta, w);
          failed_copy = true;
          break;
        }
        const int qv = wq[slot];
        const int b = qv >> 4, ik = (qv >> 2) & 3;
        const uint8_t* src = ring + slot * slotb;
        const T* xt = reinterpret_cast<const T*>(src);
        const TD* xd = reinterpret_cast<const TD*>(src + doff);
        const int npu = (np + 31) / 32;  // pieces per lane
        if (ik == 0) {  // statistics of target row i (and draft row i)
          const int sl = wrow[slot] - i0;
          float4 r;
          if (a.greedy) {
            float m = -INFINITY;
            int32_t mi = 0x7fffffff;
            for (int u = 0; u < npu; ++u) {
              const int pc = 32 * u + lane;
              if (pc < np) {
                const Raw8<T> x = load_raw8(xt + 8 * pc);
                const float pm = piece_max(x);
                if (pm > m) {  // the first element equal to the piece max
                  int e0 = 7;
#pragma unroll
                  for (int e = 7; e >= 0; --e)
                    if (elem(x, e) == pm) e0 = e;
                  m = pm;
                  mi = lo + 8 * pc + e0;
                }
              }
            }
            warp_amax(m, mi);
            r = make_float4(m, __int_as_float(mi), 0.f, 0.f);
          } else {
            float mt = -INFINITY, st_ = 0.f, md = -INFINITY, sd_ = 0.f;
            for (int u0 = 0; u0 < npu; u0 += kLanePieces) {
              Raw8<T> x[kLanePieces];
              Raw8<TD> y[kLanePieces];
#pragma unroll
              for (int u = 0; u < kLanePieces; ++u) {
                const int pc = 32 * (u0 + u) + lane;
                const bool in = u0 + u < npu && pc < np;
                x[u] = in ? load_raw8(xt + 8 * pc) : neg_inf_raw8<T>();
                y[u] = in ? load_raw8(xd + 8 * pc) : neg_inf_raw8<TD>();
              }
              lane_ms(x, k, mt, st_);
              lane_ms(y, k, md, sd_);
            }
            warp_ms(mt, st_, k);
            warp_ms(md, sd_, k);
            r = make_float4(mt, st_, md, sd_);
          }
          if (lane == 0) a.part[((size_t)b * kWave + sl) * G + cta] = r;
        } else if (ik == 1) {  // bonus row K_b: slice max, then 32-token buckets relative to it
          float m = -INFINITY;
          int32_t mi = 0x7fffffff;
          for (int u = 0; u < npu; ++u) {
            const int pc = 32 * u + lane;
            if (pc < np) {
              const Raw8<T> x = load_raw8(xt + 8 * pc);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                if (a.greedy) {
                  if (elem(x, e) > m) {
                    m = elem(x, e);
                    mi = lo + 8 * pc + e;
                  }
                } else {
                  m = fmaxf(m, elem(x, e));
                }
              }
            }
          }
          if (a.greedy) {
            warp_amax(m, mi);
            if (lane == 0) a.bpart[(size_t)b * G + cta] = make_float2(m, __int_as_float(mi));
          } else {
            m = warp_max(m);
            float ssum = 0.f;
            for (int u = 0; u < npu; ++u) {
              const int pc = 32 * u + lane;
              float bw = 0.f;
              if (pc < np) {
                const Raw8<T> x = load_raw8(xt + 8 * pc);
#pragma unroll
                for (int e = 0; e < 8; ++e) bw += fexp2((elem(x, e) - m) * k);
              }
              // the 4 pieces of a bucket sit in 4 neighbouring lanes, in token order
              bw += __shfl_xor_sync(FULLV, bw, 1);
              bw += __shfl_xor_sync(FULLV, bw, 2);
              const int q = pc >> 2;
              if ((lane & 3) == 0 && q < a.nbk) {
                a.gbk[((size_t)b * G + cta) * a.nbk + q] = make_float2(0.f, bw);
                ssum += bw;
              }
            }
            ssum = warp_sum(ssum);
            if (lane == 0) a.bpart[(size_t)b * G + cta] = make_float2(m, ssum);
          }
        } else {  // residual buckets at the stop row
          const float4 st = sst[b];
          const float it = 1.0f / st.y, id_ = 1.0f / st.w;
          float R = 0.f, P = 0.f;
          for (int u = 0; u < npu; ++u) {
            const int pc = 32 * u + lane;
            float br = 0.f, bp = 0.f;
            if (pc < np) {
              const Raw8<T> x = load_raw8(xt + 8 * pc);
              const Raw8<TD> y = load_raw8(xd + 8 * pc);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float p = fexp2((elem(x, e) - st.x) * k) * it;
                const float q = fexp2((elem(y, e) - st.z) * k) * id_;
                br += fmaxf(p - q, 0.f);
                bp += p;
              }
            }
            br += __shfl_xor_sync(FULLV, br, 1);
            bp += __shfl_xor_sync(FULLV, bp, 1);
            br += __shfl_xor_sync(FULLV, br, 2);
            bp += __shfl_xor_sync(FULLV, bp, 2);
            const int q = pc >> 2;
            if ((lane & 3) == 0 && q < a.nbk) {
              a.gbk[((size_t)b * G + cta) * a.nbk + q] = make_float2(br, bp);
              R += br;
              P += bp;
            }
          }
          R = warp_sum(R);
          P = warp_sum(P);
          if (lane == 0) a.fin[(size_t)b * G + cta] = make_float2(R, P);
        }
        __syncwarp();  // every lane has read the slot: it may be refilled
        ++consumed;
      }
    }
    if (__syncthreads_or(failed_copy ? 1 : 0)) {
      failed = true;
      break;
    }
    mark(w, 1);
    mark(w, 5);
    grid_arrive();
    if (!grid_wait()) {
      failed = true;
      break;
    }
    mark(w, 2);
    // rows that stopped in the previous wave have their residual data now
    for (int b = tid; b < B; b += kVThreads)
      if (skind[b] == ROW_STOPPED) {
        if (b % G == cta) queue_draw(b, ROW_STOPPED, (int)nbar);
        skind[b] = ROW_DONE;
      }
    __syncthreads();
    // ------------------------------------------------------------- decide phase
    for (int b = cta; b < B; b += G) {
      if (skind[b] != ROW_VERIFYING) continue;
      const int kb = skb[b];
      const int npos = min(kWave, kb - i0);
      const bool has_bonus = kb <= i0 + kWave;
      const int c0 = lane * kEV;
      if (warp < 2 * npos && (warp % 2 == 0 || !a.greedy)) {
        const int p = warp >> 1;
        const bool isd = warp & 1;
        float m = -INFINITY, s_ = 0.f;
        int32_t mi = 0x7fffffff;
#pragma unroll
        for (int t = 0; t < kEV; ++t) {
          if (c0 + t < G) {
            const float4 v = __ldcg(a.part + ((size_t)b * kWave + p) * G + c0 + t);
            if (a.greedy) amax_combine(m, mi, v.x, __float_as_int(v.y));
            else if (isd) ms_combine(m, s_, v.z, v.w, k);
            else ms_combine(m, s_, v.x, v.y, k);
          }
        }
        if (a.greedy) {
          warp_amax(m, mi);
          if (lane == 0) cst[p] = make_float4(m, __int_as_float(mi), 0.f, 0.f);
        } else {
          warp_ms(m, s_, k);
          if (lane == 0) {
            if (isd) {
              cst[p].z = m;
              cst[p].w = s_;
            } else {
              cst[p].x = m;
              cst[p].y = s_;
            }
          }
        }
      } else if (warp == kVWarps - 1 && lane < npos) {  // the draft tokens and their logits
        const int i = i0 + lane;
        int d = __ldg(a.draft + (int64_t)b * K + i);
        if (d < 0 || d >= V) {
          record_error(hdr, SPEC_ERR_TOKEN_RANGE, SITE_TOKEN_RANGE, b, d);
          d = 0;
        }
        cdt[lane] = d;
        ctd[lane] = make_float2(load_f(target, ((int64_t)b * (K + 1) + i) * V + d),
                                a.greedy ? 0.f : load_f(dl, ((int64_t)b * K + i) * V + d));
      } else if (warp == kVWarps - 2 && a.greedy && has_bonus) {
        float m = -INFINITY;
        int32_t mi = 0x7fffffff;
#pragma unroll
        for (int t = 0; t < kEV; ++t)
          if (c0 + t < G) {
            const float2 v = __ldcg(a.bpart + (size_t)b * G + c0 + t);
            amax_combine(m, mi, v.x, __float_as_int(v.y));
          }
        warp_amax(m, mi);
        if (lane == 0) cbonus = make_float2(m, __int_as_float(mi));
      }
      __syncthreads();
      if (warp == 0) {
        // every position of the wave in its own lane; the first rejection stops the row
        bool acc = false;
        float pd = 0.f, qd = 0.f;
        int d = 0, amax = 0;
        if (lane < npos) {
          const int i = i0 + lane;
          d = cdt[lane];
          const float4 c = cst[lane];
          const float2 x = ctd[lane];
          if (a.greedy) {
            amax = __float_as_int(c.y);
            acc = amax == d;
          } else {
            pd = fexp2((x.x - c.x) * k) / c.y;
            qd = fexp2((x.y - c.z) * k) / c.w;
            const float ratio = fexp2(((x.x - c.x) - (x.y - c.z)) * k) * (c.w / c.y);
            const float uacc =
                philox_uniform(a.seed, a.cycle, a.row0 + (uint32_t)b, (uint32_t)i, TAG_ACCEPT);
            acc = uacc < fminf(ratio, 1.0f);
          }
        }
        const unsigned rej = __ballot_sync(FULLV, lane < npos && !acc);
        const int first = rej ? __ffs(rej) - 1 : npos;  // position of the wave that stopped
        if (lane < npos && lane <= first) {
          const int i = i0 + lane;
          if (!a.greedy) {
            if (a.p_draft) a.p_draft[(int64_t)b * K + i] = pd;
            if (a.q_draft) a.q_draft[(int64_t)b * K + i] = qd;
          }
          if (lane < first) a.out[(int64_t)b * (K + 1) + i] = d;
          else if (a.greedy) a.out[(int64_t)b * (K + 1) + i] = amax;
        }
        if (lane == 0) {
          int kind = ROW_VERIFYING, j = 0;
          float4 sts = make_float4(0.f, 1.f, 0.f, 1.f);
          if (first < npos) {
            a.tau[b] = i0 + first + 1;
            kind = a.greedy ? ROW_DONE : ROW_STOPPED;
            j = i0 + first;
            if (!a.greedy) sts = cst[first];
          } else if (has_bonus) {  // every draft up to K_b accepted
            a.tau[b] = kb + 1;
            if (a.greedy)
              a.out[(int64_t)b * (K + 1) + kb] = __float_as_int(cbonus.y);
            else
              queue_draw(b, ROW_DONE, (int)nbar);  // bonus buckets were written in this wave
            kind = ROW_DONE;
          }
          RecV r;
          r.kind = kind;
          r.j = j;
          r.pad[0] = r.pad[1] = 0;
          r.st = sts;
          a.rec[b] = r;
          st_release_u64(a.rtag + b, ((uint64_t)(ev0 + (uint32_t)w + 1u) << 32) | (uint32_t)kind);
        }
      }
      __syncthreads();
    }
    mark(w, 3);
    mark(w, 6);
    // ------------------------------------------------------------- records hop
    if (tid == 0) n_active = 0;
    __syncthreads();
    int active = 0;
    for (int b = tid; b < B; b += kVThreads) {
      if (skind[b] != ROW_VERIFYING) continue;
      const uint32_t want = ev0 + (uint32_t)w + 1u;
      bool ok = false;
      uint64_t wv = 0;
      for (uint64_t it = 0; it < a.spin; ++it) {
        wv = ld_acquire_u64(a.rtag + b);
        if ((uint32_t)(wv >> 32) == want) {
          ok = true;
          break;
        }
        if ((it & 15) == 15 && ld_volatile_u32(&hdr->abort)) break;
        __nanosleep(32);
      }
      if (!ok) {
        if (!ld_volatile_u32(&hdr->abort)) record_error(hdr, SPEC_ERR_TIMEOUT, SITE_REC_WAIT, cta, b);
        abort_local = 1;
        break;
      }
      const int kind = (int)(uint32_t)(wv & 0xffffffffu);
      if (kind == ROW_STOPPED) {
        sj[b] = (int16_t)__ldcg(&a.rec[b].j);
        sst[b] = __ldcg(&a.rec[b].st);
      }
      skind[b] = (int8_t)kind;
      active += kind != ROW_DONE;
    }
    if (active) atomicAdd(&n_active, active);
    __syncthreads();
    if (abort_local) {
      failed = true;
      break;
    }
    mark(w, 4);
    if (n_active == 0) break;  // (rows stopped in this wave count: their residual pass is next)
  }
  if (!failed) run_draws(1 << 30);
  // nothing in flight at exit
  for (; consumed < issued; ++consumed) mbar_drain(&wbar[consumed % (uint32_t)S], (consumed / (uint32_t)S) & 1);

  // exit: the last CTA resets the launch counters; tags of the next launch differ
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t prior = atomicAdd(&hdr->exit_count, 1u);
    if (prior == (uint32_t)G - 1) {
      __threadfence();
      hdr->bar = 0;
      hdr->rec = 0;
      hdr->abort = 0;
      hdr->events += (uint32_t)((K + kWave - 1) / kWave + 2);  // bound on the waves of a launch
      __threadfence();
      atomicExch(&hdr->exit_count, 0u);
    }
  }
}

size_t a256v(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

constexpr int kMaxSlotsV = 4;
constexpr size_t kSmemBudgetV = 227 * 1024 - 1024;  // dynamic shared memory beside the static part

bool verify_ee_geometry(int B, int V, int num_sms, int tsize, int dsize, int greedy,
                        VerifyGeom* g) {
  if (B < 1 || B > kMaxRowsV || num_sms < 1) return false;
  const int gmax = std::min(num_sms, kMaxGV);
  int s = (V + gmax - 1) / gmax;
  s = (s + 31) / 32 * 32;
  g->seg = s;
  g->G = (V + s - 1) / s;
  const size_t tb = ((size_t)s * tsize + 127) / 128 * 128;
  const size_t db = greedy ? 0 : ((size_t)s * dsize + 127) / 128 * 128;
  g->doff = (int)tb;
  g->slotb = (int)(tb + db);
  const size_t state = ((size_t)B * 24 + 15) / 16 * 16;
  for (int S = kMaxSlotsV; S >= 1; --S) {
    const size_t need = state + (size_t)kVWarps * S * (8 + 4 + 4) + 128 + (size_t)kVWarps * S * g->slotb;
    if (need <= kSmemBudgetV) {
      g->S = S;
      g->smem = need;
      return true;
    }
  }
  return false;
}

size_t verify_ee_ws_bytes(int B, int V, int num_sms) {
  if (B < 1 || B > kMaxRowsV || num_sms < 1) return 0;
  const int gmax = std::min(num_sms, kMaxGV);
  int seg = (V + gmax - 1) / gmax;
  seg = (seg + 31) / 32 * 32;
  const int G = (V + seg - 1) / seg;
  const size_t nbk = (size_t)seg / 32;
  return a256v(sizeof(uint64_t) * kVTraceWaves * kVTraceSlots) +
         a256v(sizeof(float4) * (size_t)B * kWave * G) + a256v(sizeof(float2) * (size_t)B * G) * 2 +
         a256v(sizeof(float2) * (size_t)B * G * nbk) + a256v(sizeof(RecV) * (size_t)B) +
         a256v(sizeof(uint64_t) * (size_t)B);
}

template <typename T, typename TD>
cudaError_t launch_verify_ee(const T* target, const TD* draft_logits, const int32_t* draft,
                             const int32_t* vlen, int32_t* out, int32_t* tau, float* p_draft,
                             float* q_draft, int B, int K, int V, float temperature, int greedy,
                             uint64_t seed, uint64_t cycle, uint32_t row0, uint64_t spin,
                             bool trace, uint8_t* body, WsHeader* hdr, int num_sms,
                             cudaStream_t st) {
  ArgsV a;
  memset(&a, 0, sizeof(a));
  VerifyGeom vg;
  if (!verify_ee_geometry(B, V, num_sms, (int)sizeof(T), (int)sizeof(TD), greedy, &vg))
    return cudaErrorInvalidValue;
  const int G = vg.G, seg = vg.seg;
  a.S = vg.S;
  a.slotb = vg.slotb;
  a.doff = vg.doff;
  a.target = target;
  a.draft_logits = draft_logits;
  a.draft = draft;
  a.vlen = vlen;
  a.out = out;
  a.tau = tau;
  a.p_draft = p_draft;
  a.q_draft = q_draft;
  a.hdr = hdr;
  a.B = B;
  a.K = K;
  a.V = V;
  a.G = G;
  a.seg = seg;
  a.nbk = seg / 32;
  a.greedy = greedy;
  a.k = greedy ? 1.0f : 1.4426950408889634f / temperature;
  a.seed = seed;
  a.cycle = cycle;
  a.spin = spin;
  a.row0 = row0;
  a.trace = trace ? reinterpret_cast<uint64_t*>(body) : nullptr;
  body += a256v(sizeof(uint64_t) * kVTraceWaves * kVTraceSlots);
  a.part = reinterpret_cast<float4*>(body);
  body += a256v(sizeof(float4) * (size_t)B * kWave * G);
  a.bpart = reinterpret_cast<float2*>(body);
  body += a256v(sizeof(float2) * (size_t)B * G);
  a.fin = reinterpret_cast<float2*>(body);
  body += a256v(sizeof(float2) * (size_t)B * G);
  a.gbk = reinterpret_cast<float2*>(body);
  body += a256v(sizeof(float2) * (size_t)B * G * a.nbk);
  a.rec = reinterpret_cast<RecV*>(body);
  body += a256v(sizeof(RecV) * (size_t)B);
  a.rtag = reinterpret_cast<uint64_t*>(body);
  const size_t smem = vg.smem;
  auto fn = k_verify_ee<T, TD>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  void* params[] = {&a};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(fn), dim3(G), dim3(kVThreads),
                                     params, smem, st);
}

#define INST(T, TD)                                                                          \
  template cudaError_t launch_verify_ee<T, TD>(const T*, const TD*, const int32_t*,          \
                                               const int32_t*, int32_t*, int32_t*, float*,   \
                                               float*, int, int, int, float, int, uint64_t,  \
                                               uint64_t, uint32_t, uint64_t, bool, uint8_t*, \
                                               WsHeader*, int, cudaStream_t);
INST(float, float)
INST(__nv_bfloat16, __nv_bfloat16)
INST(__nv_bfloat16, float)
INST(float, __nv_bfloat16)
#undef INST

}  // namespace specdec
