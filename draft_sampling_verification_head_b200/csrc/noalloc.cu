// spec_cycle_noalloc: the fused cycle without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run a
// cycle: code inside a framework that owns every allocation (a custom
// allocator or a memory pool that must not be bypassed), a host thread that is
// not allowed to call cudaMalloc because it would synchronise the device, or a
// plugin that only receives input and output buffers.  For them this entry
// point keeps the cycle's scratch in a fixed, file-scope device array that is
// part of the loaded library: nothing is allocated per call.
//
// The array costs kNoAllocScratchBytes of device memory on every GPU that
// loads the library, until the process exits.  Every call uses the same array,
// so calls must not overlap on the GPU: two calls in flight at once (on two
// streams, or on two host threads without ordering) race on it.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "specdec.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context the address belongs to

// Unique id of the calling thread's current context (0 if unavailable): the
// array's address is valid for one context, and a device reset or a new
// primary context loads the module again, possibly elsewhere.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
        q2 == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrentFn>(f1);
      get_id = reinterpret_cast<GetIdFn>(f2);
    }
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
      get_id(ctx, &id) == CUDA_SUCCESS)
    return id;
  return 0;
}

// Device address of the array for the current device, looked up with that
// device current the first time the device is used in a context (and again
// if the context changed, e.g. after cudaDeviceReset).  In host code the
// array's name is only a host-side stand-in, never a device address.
void* scratch_for_current_device(spec_status* err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = SPEC_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long ctx = current_context_id();
  if (!g_scratch_addr[dev] || (ctx != 0 && ctx != g_scratch_ctx[dev])) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      *err = SPEC_ERR_CUDA;
      return nullptr;
    }
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" spec_status spec_cycle_noalloc(const spec_params* p, const void* base,
                                          const void* target, const void* U, const void* W,
                                          const int32_t* last_token, int32_t* draft, int32_t* out,
                                          int32_t* tau, float* p_draft, float* q_draft,
                                          int32_t* status_out, spec_stream_t stream) {
  if (!p) return SPEC_ERR_INVALID_ARG;
  const size_t need = spec_workspace_size(p);
  if (need == 0) return SPEC_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) {
    fprintf(stderr,
            "spec_cycle_noalloc: these sizes need %zu bytes of scratch, the built-in buffer "
            "holds %zu; use spec_cycle with a workspace instead\n",
            need, kNoAllocScratchBytes);
    return SPEC_ERR_WORKSPACE;
  }
  spec_status err = SPEC_OK;
  void* ws = scratch_for_current_device(&err);
  if (!ws) return err;
  cudaStream_t st = (cudaStream_t)stream;
  // the previous call leaves its status and counters behind: start from zero.
  // The header's last word (the count of earlier step events, which keeps the
  // record tags of consecutive calls apart) is kept; the rest of the scratch
  // needs no clearing: a launch writes every entry before reading it.
  if (cudaMemsetAsync(ws, 0, sizeof(specdec::WsHeader) - sizeof(uint32_t), st) != cudaSuccess)
    return SPEC_ERR_CUDA;
  const spec_status s = spec_cycle(p, base, target, U, W, last_token, draft, out, tau, p_draft,
                                   q_draft, ws, stream);
  if (s != SPEC_OK) return s;
  if (status_out &&
      cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return SPEC_ERR_CUDA;
  return SPEC_OK;
}
