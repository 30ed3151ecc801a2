// C-ABI entry points (include/specdec.h): argument validation on the host,
// workspace layout, tensor maps and launches.  No allocation happens here.
#include <curand_kernel.h>

#include <climits>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "specdec_debug.h"

namespace specdec {

namespace {

thread_local int32_t g_last_launches = 0;

constexpr uint64_t kDefaultSpin = 4000000ull;  // polls of ~0.5 us back-off: about 2 s
constexpr int32_t kMaxLoopCycles = 1 << 16;     // record tags of one launch stay below 2^31

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by all calls; returns SPEC_OK or the error.
spec_status check_params(const spec_params* p) {
  if (!p) return SPEC_ERR_INVALID_ARG;
  if (p->B < 1 || p->K < 1 || p->K > 1024 || p->V < 1 || p->r < 0 || p->r > 256)
    return SPEC_ERR_INVALID_ARG;
  if (p->dtype != SPEC_F32 && p->dtype != SPEC_BF16) return SPEC_ERR_INVALID_ARG;
  if ((uint64_t)p->row_offset + (uint64_t)p->B > (uint64_t(1) << 31)) return SPEC_ERR_INVALID_ARG;
  if (!p->greedy && !(p->temperature > 0.f)) return SPEC_ERR_INVALID_ARG;
  if (p->V % 8 != 0) return SPEC_ERR_UNSUPPORTED;  // rows must start on 16-byte boundaries
  return SPEC_OK;
}

uint64_t spin_of(const spec_params* p) { return p->spin_limit ? p->spin_limit : kDefaultSpin; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

WsHeader* header_of(void* ws) { return reinterpret_cast<WsHeader*>(ws); }
uint8_t* body_of(void* ws) { return reinterpret_cast<uint8_t*>(ws) + sizeof(WsHeader); }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

// W [r, V] bf16: boxes of 64 tokens x box_k rank rows, 128-byte swizzle.
bool make_tmap_W(CUtensorMap* m, const void* W, int r, int V, int box_k) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)V, (cuuint64_t)r};
  const cuuint64_t strides[1] = {(cuuint64_t)V * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_k};
  const cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Base logits [B, K, V] as a 3-D map.  Tensor-core path: boxes of 64 tokens x
// 1 step x N rows with the 128-byte swizzle, the operand layout the bias MMA
// adds them with; otherwise 128 tokens x 1 x N rows, unswizzled.
bool make_tmap_base(CUtensorMap* m, const void* base, int dtype, int B, int K, int V, int N,
                    bool tc) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  const size_t es = dtype == SPEC_BF16 ? 2 : 4;
  const cuuint64_t dims[3] = {(cuuint64_t)V, (cuuint64_t)K, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)V * es, (cuuint64_t)K * V * es};
  const cuuint32_t box[3] = {tc ? 64u : 128u, 1, (cuuint32_t)N};
  const cuuint32_t estr[3] = {1, 1, 1};
  return f(m, dtype == SPEC_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
           3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           tc ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- debug kernels: Philox stream and the CUDA library's own Philox4_32_10 ----
namespace {
__global__ void k_debug_philox(const uint32_t* ctr, const uint32_t* key, uint32_t* out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const Philox4 r = philox4x32_10(ctr[4 * i], ctr[4 * i + 1], ctr[4 * i + 2], ctr[4 * i + 3],
                                  key[2 * i], key[2 * i + 1]);
  out[4 * i] = r.x;
  out[4 * i + 1] = r.y;
  out[4 * i + 2] = r.z;
  out[4 * i + 3] = r.w;
}
// curand's generator with the same counter: key = seed, counter words 2..3 =
// subsequence, words 0..1 = offset / 4.
__global__ void k_debug_curand(const uint32_t* ctr, const uint32_t* key, uint32_t* out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  curandStatePhilox4_32_10_t st;
  const unsigned long long seed = (unsigned long long)key[2 * i] |
                                  ((unsigned long long)key[2 * i + 1] << 32);
  const unsigned long long sub = (unsigned long long)ctr[4 * i + 2] |
                                 ((unsigned long long)ctr[4 * i + 3] << 32);
  const unsigned long long off = ((unsigned long long)ctr[4 * i] |
                                  ((unsigned long long)ctr[4 * i + 1] << 32)) * 4ull;
  curand_init(seed, sub, off, &st);
  const uint4 r = curand4(&st);
  out[4 * i] = r.x;
  out[4 * i + 1] = r.y;
  out[4 * i + 2] = r.z;
  out[4 * i + 3] = r.w;
}
}  // namespace

cudaError_t launch_debug_philox(const uint32_t* ctr, const uint32_t* key, uint32_t* out, int n,
                                cudaStream_t st) {
  k_debug_philox<<<(n + 255) / 256, 256, 0, st>>>(ctr, key, out, n);
  return cudaGetLastError();
}
cudaError_t launch_debug_curand_philox(const uint32_t* ctr, const uint32_t* key, uint32_t* out,
                                       int n, cudaStream_t st) {
  k_debug_curand<<<(n + 255) / 256, 256, 0, st>>>(ctr, key, out, n);
  return cudaGetLastError();
}

template <typename T, typename TD>
cudaError_t verify_dispatch(const spec_params* p, const void* target,
                                   const void* draft_logits, const int32_t* draft,
                                   const int32_t* vlen, int32_t* out, int32_t* tau, float* p_draft,
                                   float* q_draft, bool fused, uint8_t* body, WsHeader* h, int sms,
                                   cudaStream_t st, int* launches) {
  const int gr = p->greedy ? 1 : 0;
  if (fused) {
    *launches = 1;
    return launch_verify_ee((const T*)target, (const TD*)draft_logits, draft, vlen, out, tau,
                            p_draft, q_draft, p->B, p->K, p->V, p->temperature, gr, p->seed,
                            p->cycle, p->row_offset, spin_of(p), (p->flags & SPEC_FLAG_TRACE) != 0,
                            body, h, sms, st);
  }
  return launch_verify((const T*)target, (const TD*)draft_logits, draft, out, tau, p_draft,
                       q_draft, p->B, p->K, p->V, p->temperature, gr, p->seed, p->cycle,
                       p->row_offset, body, h, sms, st, launches);
}

}  // namespace specdec

using namespace specdec;

extern "C" {

const char* spec_status_string(spec_status s) {
  switch (s) {
    case SPEC_OK: return "SPEC_OK";
    case SPEC_ERR_INVALID_ARG: return "SPEC_ERR_INVALID_ARG";
    case SPEC_ERR_UNSUPPORTED: return "SPEC_ERR_UNSUPPORTED";
    case SPEC_ERR_CUDA: return "SPEC_ERR_CUDA";
    case SPEC_ERR_TIMEOUT: return "SPEC_ERR_TIMEOUT";
    case SPEC_ERR_WORKSPACE: return "SPEC_ERR_WORKSPACE";
    case SPEC_ERR_TOKEN_RANGE: return "SPEC_ERR_TOKEN_RANGE";
  }
  return "SPEC_ERR_UNKNOWN";
}

int32_t spec_last_launch_count(void) { return g_last_launches; }

size_t spec_workspace_size(const spec_params* p) {
  if (check_params(p) != SPEC_OK) return 0;
  const int sms = num_sms();
  if (sms <= 0) return 0;
  size_t need = std::max(verify_ws_bytes(p->B, p->K, p->V), verify_ee_ws_bytes(p->B, p->V, sms));
  CycleGeom g;
  const char* why = nullptr;
  if (cycle_geometry(p->B, p->K, p->V, p->r, p->dtype, p->flags, sms, &g, &why))
    need = std::max(need, cycle_ws_bytes(p->K, g));
  if (cycle_tc_geometry(p->B, p->K, p->V, p->r, p->dtype, p->flags, sms, &g, &why))
    need = std::max(need, cycle_tc_ws_bytes(p->K, p->r, g));
  return round256(sizeof(WsHeader) + need);
}

spec_status spec_workspace_init(void* ws, size_t bytes, spec_stream_t stream) {
  if (!ws || bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return SPEC_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, bytes, (cudaStream_t)stream) == cudaSuccess ? SPEC_OK
                                                                             : SPEC_ERR_CUDA;
}

spec_status spec_sync_status(const void* ws, spec_stream_t stream) {
  if (!ws) return SPEC_ERR_WORKSPACE;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SPEC_ERR_CUDA;
  int32_t st = 0;
  if (cudaMemcpy(&st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return SPEC_ERR_CUDA;
  return (spec_status)st;
}

spec_status spec_markov_bias(const spec_params* p, const void* U, const void* W,
                             const int32_t* prev, float* bias, void* ws, spec_stream_t stream) {
  g_last_launches = 0;
  spec_status s = check_params(p);
  if (s != SPEC_OK) return s;
  if (p->r < 1 || !U || !W || !prev || !bias) return SPEC_ERR_INVALID_ARG;
  if (!aligned16(U) || !aligned16(W)) return SPEC_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SPEC_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  const bool tc = p->dtype == SPEC_BF16 && p->r % 64 == 0 && !(p->flags & SPEC_FLAG_FMA_BIAS);
  cudaError_t e;
  if (tc) {
    CUtensorMap tm;
    if (!make_tmap_W(&tm, W, p->r, p->V, 64)) return SPEC_ERR_CUDA;
    e = launch_bias_tc(tm, reinterpret_cast<const __nv_bfloat16*>(U), prev, bias, p->B, p->V,
                       p->r, header_of(ws), spin_of(p), st);
  } else if (p->dtype == SPEC_BF16) {
    e = launch_bias_fma(reinterpret_cast<const __nv_bfloat16*>(U),
                        reinterpret_cast<const __nv_bfloat16*>(W), prev, bias, p->B, p->V, p->r,
                        header_of(ws), st);
  } else {
    e = launch_bias_fma(reinterpret_cast<const float*>(U), reinterpret_cast<const float*>(W), prev,
                        bias, p->B, p->V, p->r, header_of(ws), st);
  }
  g_last_launches = 1;
  return e == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

// The fused cycle on the tensor-core path (geometry already decided).
// Extra inputs of the tensor-core cycle: cycles per launch, confidence scores
// with their threshold, the carried last tokens, the RNN head's recurrence
// (one plain cycle of the Markov head: all unset).
struct LoopInputs {
  int ncyc = 1;
  const float* conf = nullptr;
  float conf_thr = 0.f;
  int32_t* next_token = nullptr;
  const void* Wh = nullptr;
};

static spec_status run_cycle_tc(const spec_params* p, const CycleGeom& g, const void* base,
                                const void* target, const void* U, const void* W,
                                const int32_t* last_token, const int32_t* vlen, int32_t* draft,
                                int32_t* out, int32_t* tau, float* p_draft, float* q_draft,
                                void* ws, spec_stream_t stream,
                                const LoopInputs& loop = LoopInputs()) {
  CUtensorMap tmW;
  if (!make_tmap_W(&tmW, W, p->r, p->V, kCycleWBoxK)) return SPEC_ERR_CUDA;
  CycleLaunch L;
  memset(&L, 0, sizeof(L));
  L.base = base;
  L.target = target;
  L.U = U;
  L.W = W;
  L.last_token = last_token;
  L.vlen = vlen;
  L.conf = loop.conf;
  L.conf_thr = loop.conf_thr;
  L.next_token = loop.next_token;
  L.ncyc = loop.ncyc;
  L.Wh = loop.Wh;
  L.draft = draft;
  L.out = out;
  L.tau = tau;
  L.p_draft = p_draft;
  L.q_draft = q_draft;
  L.B = p->B;
  L.K = p->K;
  L.V = p->V;
  L.r = p->r;
  L.dtype = p->dtype;
  L.mode = MODE_CYCLE;
  L.greedy = p->greedy ? 1 : 0;
  L.temperature = p->temperature;
  L.seed = p->seed;
  L.cycle = p->cycle;
  L.row0 = p->row_offset;
  L.spin = spin_of(p);
  L.trace = (p->flags & SPEC_FLAG_TRACE) != 0;
  cudaError_t e = launch_cycle_tc(L, g, header_of(ws), body_of(ws), &tmW, (cudaStream_t)stream);
  g_last_launches = 1;
  if (e != cudaSuccess) {
    fprintf(stderr, "specdec: launch failed: %s\n", cudaGetErrorString(e));
    return SPEC_ERR_CUDA;
  }
  return SPEC_OK;
}

static spec_status run_cycle(const spec_params* p, int mode, const void* base, const void* target,
                             const void* U, const void* W, const int32_t* last_token,
                             const int32_t* vlen, int32_t* draft, int32_t* out, int32_t* tau,
                             float* p_draft, float* q_draft, float* biased_out, void* ws,
                             spec_stream_t stream) {
  g_last_launches = 0;
  spec_status s = check_params(p);
  if (s != SPEC_OK) return s;
  if (!base || !last_token || (p->r > 0 && (!U || !W))) return SPEC_ERR_INVALID_ARG;
  if (mode == MODE_CYCLE && (!target || !out || !tau)) return SPEC_ERR_INVALID_ARG;
  if (mode == MODE_DRAFT && !draft) return SPEC_ERR_INVALID_ARG;
  if (!aligned16(base) || (target && !aligned16(target)) || (U && !aligned16(U)) ||
      (W && !aligned16(W)))
    return SPEC_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SPEC_ERR_WORKSPACE;
  const int sms = num_sms();
  if (sms <= 0) return SPEC_ERR_CUDA;
  CycleGeom g;
  const char* why = nullptr;
  if (mode == MODE_CYCLE && cycle_tc_geometry(p->B, p->K, p->V, p->r, p->dtype, p->flags, sms, &g, &why))
    return run_cycle_tc(p, g, base, target, U, W, last_token, vlen, draft, out, tau, p_draft,
                        q_draft, ws, stream);
  if (vlen) {
    fprintf(stderr, "specdec: per-row verify lengths need the tensor-core cycle (bf16, rank a "
                    "multiple of 64 up to 256): %s\n", why);
    return SPEC_ERR_UNSUPPORTED;
  }
  if (!cycle_geometry(p->B, p->K, p->V, p->r, p->dtype, p->flags, sms, &g, &why)) {
    fprintf(stderr, "specdec: unsupported shape: %s\n", why);
    return SPEC_ERR_UNSUPPORTED;
  }
  CUtensorMap tmW, tmBase;
  memset(&tmW, 0, sizeof(tmW));
  if (g.tc && !make_tmap_W(&tmW, W, p->r, p->V, kCycleWBoxK)) return SPEC_ERR_CUDA;
  if (!make_tmap_base(&tmBase, base, p->dtype, p->B, p->K, p->V, g.N, g.tc)) return SPEC_ERR_CUDA;
  CycleLaunch L;
  memset(&L, 0, sizeof(L));
  L.base = base;
  L.target = target;
  L.U = U;
  L.W = W;
  L.last_token = last_token;
  L.draft = draft;
  L.out = out;
  L.tau = tau;
  L.p_draft = p_draft;
  L.q_draft = q_draft;
  L.biased_out = biased_out;
  L.B = p->B;
  L.K = p->K;
  L.V = p->V;
  L.r = p->r;
  L.dtype = p->dtype;
  L.mode = mode;
  L.greedy = p->greedy ? 1 : 0;
  L.temperature = p->temperature;
  L.seed = p->seed;
  L.cycle = p->cycle;
  L.row0 = p->row_offset;
  L.spin = spin_of(p);
  L.trace = (p->flags & SPEC_FLAG_TRACE) != 0;
  cudaError_t e = launch_cycle(L, g, header_of(ws), body_of(ws), g.tc ? &tmW : nullptr, &tmBase,
                               (cudaStream_t)stream);
  g_last_launches = 1;
  if (e != cudaSuccess) {
    fprintf(stderr, "specdec: launch failed: %s\n", cudaGetErrorString(e));
    return SPEC_ERR_CUDA;
  }
  return SPEC_OK;
}

spec_status spec_markov_bias_sample(const spec_params* p, const void* base, const void* U,
                                    const void* W, const int32_t* last_token, int32_t* draft,
                                    float* q_draft, float* biased_out, void* ws,
                                    spec_stream_t stream) {
  return run_cycle(p, MODE_DRAFT, base, nullptr, U, W, last_token, nullptr, draft, nullptr,
                   nullptr, nullptr, q_draft, biased_out, ws, stream);
}

spec_status spec_cycle(const spec_params* p, const void* base, const void* target, const void* U,
                       const void* W, const int32_t* last_token, int32_t* draft, int32_t* out,
                       int32_t* tau, float* p_draft, float* q_draft, void* ws,
                       spec_stream_t stream) {
  return run_cycle(p, MODE_CYCLE, base, target, U, W, last_token, nullptr, draft, out, tau,
                   p_draft, q_draft, nullptr, ws, stream);
}

spec_status spec_cycle_kb(const spec_params* p, const void* base, const void* target, const void* U,
                          const void* W, const int32_t* last_token, const int32_t* verify_len,
                          int32_t* draft, int32_t* out, int32_t* tau, float* p_draft,
                          float* q_draft, void* ws, spec_stream_t stream) {
  if (!verify_len) return SPEC_ERR_INVALID_ARG;
  return run_cycle(p, MODE_CYCLE, base, target, U, W, last_token, verify_len, draft, out, tau,
                   p_draft, q_draft, nullptr, ws, stream);
}

spec_status spec_decode_loop(const spec_params* p, int32_t n_cycles, const void* base,
                             const void* target, const float* conf, float conf_threshold,
                             const int32_t* verify_len, const void* U, const void* W,
                             const int32_t* last_token, int32_t* draft, int32_t* out, int32_t* tau,
                             float* p_draft, float* q_draft, int32_t* next_token, void* ws,
                             spec_stream_t stream) {
  g_last_launches = 0;
  spec_status s = check_params(p);
  if (s != SPEC_OK) return s;
  if (n_cycles < 1 || n_cycles > kMaxLoopCycles || (conf && verify_len)) return SPEC_ERR_INVALID_ARG;
  if (n_cycles > 1 && !next_token) return SPEC_ERR_INVALID_ARG;
  if ((int64_t)n_cycles * p->B > INT32_MAX) return SPEC_ERR_INVALID_ARG;
  if (!base || !target || !last_token || !out || !tau || !U || !W || p->r < 1)
    return SPEC_ERR_INVALID_ARG;
  if (!aligned16(base) || !aligned16(target) || !aligned16(U) || !aligned16(W))
    return SPEC_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SPEC_ERR_WORKSPACE;
  const int sms = num_sms();
  if (sms <= 0) return SPEC_ERR_CUDA;
  CycleGeom g;
  const char* why = nullptr;
  if (!cycle_tc_geometry(p->B, p->K, p->V, p->r, p->dtype, p->flags, sms, &g, &why)) {
    fprintf(stderr, "specdec: the decode loop needs the tensor-core cycle (bf16, rank a multiple "
                    "of 64 up to 256): %s\n", why);
    return SPEC_ERR_UNSUPPORTED;
  }
  LoopInputs loop;
  loop.ncyc = n_cycles;
  loop.conf = conf;
  loop.conf_thr = conf_threshold;
  loop.next_token = next_token;
  return run_cycle_tc(p, g, base, target, U, W, last_token, verify_len, draft, out, tau, p_draft,
                      q_draft, ws, stream, loop);
}

static spec_status run_verify(const spec_params* p, const void* target, const void* draft_logits,
                              const int32_t* draft, const int32_t* vlen, int32_t* out,
                              int32_t* tau, float* p_draft, float* q_draft, void* ws,
                              spec_stream_t stream) {
  g_last_launches = 0;
  spec_status s = check_params(p);
  if (s != SPEC_OK) return s;
  if (p->draft_dtype != SPEC_F32 && p->draft_dtype != SPEC_BF16) return SPEC_ERR_INVALID_ARG;
  if (!target || !draft_logits || !draft || !out || !tau) return SPEC_ERR_INVALID_ARG;
  if (!aligned16(target) || !aligned16(draft_logits)) return SPEC_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SPEC_ERR_WORKSPACE;
  const int sms = num_sms();
  if (sms <= 0) return SPEC_ERR_CUDA;
  VerifyGeom vg;
  const bool fused = verify_ee_geometry(p->B, p->V, sms, p->dtype == SPEC_BF16 ? 2 : 4,
                                        p->draft_dtype == SPEC_BF16 ? 2 : 4, p->greedy ? 1 : 0, &vg);
  if (vlen && !fused) {
    fprintf(stderr, "specdec: per-row verify lengths need the one-launch verification (B <= 4096 "
                    "and a vocabulary slice per SM that fits its shared-memory ring)\n");
    return SPEC_ERR_UNSUPPORTED;
  }
  int launches = 0;
  cudaError_t e;
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader* h = header_of(ws);
  uint8_t* body = body_of(ws);
  if (p->dtype == SPEC_BF16 && p->draft_dtype == SPEC_BF16)
    e = verify_dispatch<__nv_bfloat16, __nv_bfloat16>(p, target, draft_logits, draft, vlen, out, tau,
                                                      p_draft, q_draft, fused, body, h, sms, st,
                                                      &launches);
  else if (p->dtype == SPEC_BF16)
    e = verify_dispatch<__nv_bfloat16, float>(p, target, draft_logits, draft, vlen, out, tau,
                                              p_draft, q_draft, fused, body, h, sms, st, &launches);
  else if (p->draft_dtype == SPEC_BF16)
    e = verify_dispatch<float, __nv_bfloat16>(p, target, draft_logits, draft, vlen, out, tau,
                                              p_draft, q_draft, fused, body, h, sms, st, &launches);
  else
    e = verify_dispatch<float, float>(p, target, draft_logits, draft, vlen, out, tau, p_draft,
                                      q_draft, fused, body, h, sms, st, &launches);
  g_last_launches = launches;
  if (e != cudaSuccess) {
    fprintf(stderr, "specdec: launch failed: %s\n", cudaGetErrorString(e));
    return SPEC_ERR_CUDA;
  }
  return SPEC_OK;
}

spec_status spec_cycle_rnn(const spec_params* p, const void* base, const void* target,
                           const void* U, const void* W, const void* Wh, const int32_t* last_token,
                           int32_t* draft, int32_t* out, int32_t* tau, float* p_draft,
                           float* q_draft, void* ws, spec_stream_t stream) {
  g_last_launches = 0;
  spec_status s = check_params(p);
  if (s != SPEC_OK) return s;
  if (!base || !target || !last_token || !out || !tau || !U || !W || !Wh || p->r < 1)
    return SPEC_ERR_INVALID_ARG;
  if (!aligned16(base) || !aligned16(target) || !aligned16(U) || !aligned16(W) || !aligned16(Wh))
    return SPEC_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SPEC_ERR_WORKSPACE;
  const int sms = num_sms();
  if (sms <= 0) return SPEC_ERR_CUDA;
  CycleGeom g;
  const char* why = nullptr;
  if (!cycle_tc_geometry(p->B, p->K, p->V, p->r, p->dtype, p->flags, sms, &g, &why)) {
    fprintf(stderr, "specdec: the RNN head needs the tensor-core cycle (bf16, rank a multiple "
                    "of 64 up to 256): %s\n", why);
    return SPEC_ERR_UNSUPPORTED;
  }
  LoopInputs loop;
  loop.Wh = Wh;
  return run_cycle_tc(p, g, base, target, U, W, last_token, nullptr, draft, out, tau, p_draft,
                      q_draft, ws, stream, loop);
}

spec_status spec_verify_block(const spec_params* p, const void* target, const void* draft_logits,
                              const int32_t* draft, int32_t* out, int32_t* tau, float* p_draft,
                              float* q_draft, void* ws, spec_stream_t stream) {
  return run_verify(p, target, draft_logits, draft, nullptr, out, tau, p_draft, q_draft, ws,
                    stream);
}

spec_status spec_verify_block_kb(const spec_params* p, const void* target,
                                 const void* draft_logits, const int32_t* draft,
                                 const int32_t* verify_len, int32_t* out, int32_t* tau,
                                 float* p_draft, float* q_draft, void* ws, spec_stream_t stream) {
  if (!verify_len) return SPEC_ERR_INVALID_ARG;
  return run_verify(p, target, draft_logits, draft, verify_len, out, tau, p_draft, q_draft, ws,
                    stream);
}

spec_status spec_l2_persist(const void* ptr, size_t bytes, spec_stream_t stream) {
  cudaStream_t st = (cudaStream_t)stream;
  cudaStreamAttrValue v;
  memset(&v, 0, sizeof(v));
  if (bytes == 0 || ptr == nullptr) {
    v.accessPolicyWindow.num_bytes = 0;
    if (cudaStreamSetAttribute(st, cudaStreamAttributeAccessPolicyWindow, &v) != cudaSuccess)
      return SPEC_ERR_CUDA;
    return cudaCtxResetPersistingL2Cache() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
  }
  int dev = 0, max_persist = 0, max_window = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&max_persist, cudaDevAttrMaxPersistingL2CacheSize, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&max_window, cudaDevAttrMaxAccessPolicyWindowSize, dev) != cudaSuccess)
    return SPEC_ERR_CUDA;
  if (max_persist <= 0 || max_window <= 0) return SPEC_ERR_UNSUPPORTED;
  const size_t window = std::min(bytes, (size_t)max_window);
  const size_t carve = std::min(window, (size_t)max_persist);
  if (cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, carve) != cudaSuccess) return SPEC_ERR_CUDA;
  v.accessPolicyWindow.base_ptr = const_cast<void*>(ptr);
  v.accessPolicyWindow.num_bytes = window;
  v.accessPolicyWindow.hitRatio = (float)carve / (float)window;
  v.accessPolicyWindow.hitProp = cudaAccessPropertyPersisting;
  v.accessPolicyWindow.missProp = cudaAccessPropertyStreaming;
  return cudaStreamSetAttribute(st, cudaStreamAttributeAccessPolicyWindow, &v) == cudaSuccess
             ? SPEC_OK
             : SPEC_ERR_CUDA;
}

spec_status spec_debug_philox(const uint32_t* ctr, const uint32_t* key, uint32_t* out, int32_t n,
                              spec_stream_t stream) {
  if (!ctr || !key || !out || n < 0) return SPEC_ERR_INVALID_ARG;
  if (n == 0) return SPEC_OK;
  return launch_debug_philox(ctr, key, out, n, (cudaStream_t)stream) == cudaSuccess
             ? SPEC_OK
             : SPEC_ERR_CUDA;
}

spec_status spec_debug_curand_philox(const uint32_t* ctr, const uint32_t* key, uint32_t* out,
                                     int32_t n, spec_stream_t stream) {
  if (!ctr || !key || !out || n < 0) return SPEC_ERR_INVALID_ARG;
  if (n == 0) return SPEC_OK;
  return launch_debug_curand_philox(ctr, key, out, n, (cudaStream_t)stream) == cudaSuccess
             ? SPEC_OK
             : SPEC_ERR_CUDA;
}

}  // extern "C"
