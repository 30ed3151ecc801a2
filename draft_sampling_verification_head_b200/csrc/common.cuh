// Device-side building blocks shared by the specdec kernels (sm_100a only):
// Philox4x32-10, bf16 loads, PTX wrappers for mbarriers, TMA, tcgen05 and
// bounded waits, and the workspace header.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "specdec.h"

#define SPEC_DEV __device__ __forceinline__

namespace specdec {

// ----------------------------------------------------------------------------
// Workspace header: first 256 bytes of every workspace.  Counters are reset by
// the last CTA of each persistent launch, so every launch starts from zero.
// ----------------------------------------------------------------------------
struct WsHeader {
  int32_t status;       // sticky first error (spec_status), 0 = ok
  int32_t err_where;    // diagnostic: code site of the first error
  int32_t err_a;        // diagnostic values
  int32_t err_b;
  uint32_t bar;         // grid-barrier arrivals in the current launch
  uint32_t spare;       // unused
  uint32_t exit_count;  // CTAs that finished the current launch
  uint32_t abort;       // nonzero once a CTA of the current launch gave up
  uint32_t rec;         // row records published in the current launch
  uint32_t pad[54];
  uint32_t events;      // tensor-core cycle: step events of all earlier launches on this
                        // workspace (record tags); kept last so a reset of the rest keeps it
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

enum ErrSite : int32_t {
  SITE_NONE = 0,
  SITE_GRID_BARRIER = 1,
  SITE_UNUSED_2 = 2,
  SITE_MBAR_FULL = 3,
  SITE_MBAR_MMA = 4,
  SITE_MBAR_BASE = 5,
  SITE_TOKEN_RANGE = 6,
  SITE_MBAR_BREADY = 7,
  SITE_MBAR_TFREE = 8,
  SITE_REC_WAIT = 9,
};

SPEC_DEV void record_error(WsHeader* h, int32_t code, int32_t site, int32_t a, int32_t b) {
  if (atomicCAS(&h->status, 0, code) == 0) {
    h->err_where = site;
    h->err_a = a;
    h->err_b = b;
  }
  atomicExch(&h->abort, 1u);
}

SPEC_DEV uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
SPEC_DEV void red_release_add_u32(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
SPEC_DEV uint64_t ld_acquire_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
SPEC_DEV void st_release_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
SPEC_DEV uint32_t ld_volatile_u32(const uint32_t* p) {
  return *reinterpret_cast<const volatile uint32_t*>(p);
}

// ----------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of
// (c0,c1,c2,c3) -> (hi(M1 c2)^c1^k0, lo(M1 c2), hi(M0 c0)^c3^k1, lo(M0 c0))
// with the key bumped by the Weyl constants between rounds.
// ----------------------------------------------------------------------------
struct Philox4 {
  uint32_t x, y, z, w;
};

SPEC_DEV Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                               uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += W0;
      k1 += W1;
    }
    const uint32_t hi0 = __umulhi(M0, c0), lo0 = M0 * c0;
    const uint32_t hi1 = __umulhi(M1, c2), lo1 = M1 * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return Philox4{c0, c1, c2, c3};
}

enum : uint32_t { TAG_DRAFT = 0, TAG_ACCEPT = 1, TAG_RESAMPLE = 2 };

// (x >> 8) * 2^-24: exact in fp32, in [0, 1)
SPEC_DEV float u01(uint32_t x) { return (float)(x >> 8) * (1.0f / 16777216.0f); }

SPEC_DEV float philox_uniform(uint64_t seed, uint64_t cycle, uint32_t b, uint32_t pos,
                              uint32_t tag) {
  const uint32_t c3 = (tag & 0xFFFFu) | ((uint32_t)((cycle >> 32) & 0xFFFFu) << 16);
  Philox4 r = philox4x32_10(pos, b, (uint32_t)cycle, c3, (uint32_t)seed, (uint32_t)(seed >> 32));
  return u01(r.x);
}

// ----------------------------------------------------------------------------
// Element loads
// ----------------------------------------------------------------------------
SPEC_DEV float bf16_bits_to_float(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

template <typename T>
SPEC_DEV float load_f(const T* p, int64_t i);
template <>
SPEC_DEV float load_f<float>(const float* p, int64_t i) {
  return __ldg(p + i);
}
template <>
SPEC_DEV float load_f<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return bf16_bits_to_float(__ldg(reinterpret_cast<const unsigned short*>(p) + i));
}

// ----------------------------------------------------------------------------
// Shared-memory address helpers, mbarriers (bounded waits)
// ----------------------------------------------------------------------------
SPEC_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

SPEC_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
SPEC_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
SPEC_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
SPEC_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// One poll; the thread may be suspended in hardware for up to ~1 us while the
// phase is incomplete, so waiting warps do not take issue slots.
SPEC_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000u)
      : "memory");
  return ok != 0;
}
// Wait for phase `parity` of an mbarrier; gives up after `limit` polls or as
// soon as the launch has been aborted.  Returns false on give-up.
SPEC_DEV bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit,
                                const uint32_t* abort_flag) {
  for (uint64_t it = 0; it < limit; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 63 && ld_volatile_u32(abort_flag)) return false;
  }
  return false;
}

// Polls used when draining copies / MMAs that were already issued: those
// always complete, so the drain does not use the caller's (possibly tiny) limit.
constexpr uint64_t kDrainPolls = 1ull << 22;
SPEC_DEV bool mbar_drain(uint64_t* bar, uint32_t parity) {
  for (uint64_t it = 0; it < kDrainPolls; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Bulk prefetch of [p, p + bytes) into L2 (16-byte aligned, size a multiple of 16).
SPEC_DEV void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

SPEC_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor): each CTA loads its own tiles.
// ----------------------------------------------------------------------------
SPEC_DEV void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
SPEC_DEV uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
SPEC_DEV uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
SPEC_DEV void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x, int32_t y,
                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// 16-byte asynchronous copy global -> shared (bypassing L1), grouped by
// commit_group / wait_group.  Both addresses 16-byte aligned.
SPEC_DEV void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
SPEC_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int PENDING>
SPEC_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(PENDING) : "memory");
}

// Untiled bulk copy global -> this CTA's shared memory, completion counted in
// bytes on the mbarrier.  Both addresses 16-byte aligned, bytes a multiple of 16.
SPEC_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                        uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
SPEC_DEV void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x, int32_t y,
                          int32_t z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, tensor memory)
// ----------------------------------------------------------------------------
SPEC_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
SPEC_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
SPEC_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
SPEC_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
SPEC_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, fp32 accumulate)
SPEC_DEV void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on an mbarrier once all previously issued tcgen05 ops of this thread complete.
SPEC_DEV void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread
SPEC_DEV void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}
SPEC_DEV void tmem_ld1(uint32_t taddr, float* v) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  *v = __uint_as_float(r);
}
SPEC_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
SPEC_DEV void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
SPEC_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (sm_100 "version 1" format):
// start>>4 in bits 0-13, LBO>>4 in 16-29, SBO>>4 in 32-45, version 1 in 46-47,
// layout type in 61-63 (2 = 128-byte swizzle).
SPEC_DEV uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor for kind::f16: D fp32, A and B bf16, A MN-major
// (bit 15), B K-major, N>>3 in bits 17-22, M>>4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, bool a_mn_major,
                                                      bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// ----------------------------------------------------------------------------
// Grid-wide synchronisation on the workspace header (bounded).
// ----------------------------------------------------------------------------
// Arrive (release) and wait (acquire) until `target` arrivals; one thread per CTA.
SPEC_DEV bool grid_wait_count(WsHeader* h, const uint32_t* counter, uint32_t target,
                              uint64_t limit, int32_t site) {
  for (uint64_t it = 0; it < limit; ++it) {
    // both loads in flight together: the abort flag first (relaxed), then the
    // counter (acquire, which orders only what follows it)
    const uint32_t ab = ld_volatile_u32(&h->abort);
    const uint32_t c = ld_acquire_u32(counter);
    if (ab) return false;
    if (c >= target) return true;
    __nanosleep(32);
  }
  record_error(h, SPEC_ERR_TIMEOUT, site, (int32_t)target, (int32_t)ld_volatile_u32(counter));
  return false;
}

// Device clock in nanoseconds (timelines of the trace flag).
SPEC_DEV uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

SPEC_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
SPEC_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32, a few ulp of
// relative error); results below 2^-126 flush to zero.  Every exponential of the
// fused cycle goes through this one function, so a quantity computed in two
// places (a bucket total and the scan inside the bucket) agrees bit for bit.
SPEC_DEV float fexp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Softmax statistics are kept as (m, s): m = max of the raw logits x,
// s = sum exp2((x - m) * k) with k = log2(e) / T.  Differences x - m are taken
// before scaling so that the dominant terms carry no rounding from the scale.
// Combine two such pairs.
// Branch-free: one exp2, of the smaller max relative to the larger.
SPEC_DEV void ms_combine(float& m, float& s, float m2, float s2, float k) {
  const bool first = m >= m2;
  const float mb = first ? m : m2, ml = first ? m2 : m;
  const float sb = first ? s : s2, sl = first ? s2 : s;
  const float e = (ml == -INFINITY) ? 0.f : fexp2((ml - mb) * k);
  m = mb;
  s = fmaf(sl, e, sb);
}

// Arg-max pair with lowest-index tie-break.
SPEC_DEV void amax_combine(float& v, int32_t& i, float v2, int32_t i2) {
  if (v2 > v || (v2 == v && i2 < i)) {
    v = v2;
    i = i2;
  }
}

}  // namespace specdec
