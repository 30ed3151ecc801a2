// Internal interfaces between the C-ABI layer and the kernels.
#pragma once

#include "common.cuh"

namespace specdec {

struct RowPartial {
  float m;      // max of raw logits over the segment
  float s;      // sum exp2((x - m) * k)
  float amax;   // arg-max value
  int32_t aidx; // arg-max index (lowest on ties)
};

struct StopInfo {
  int32_t j;   // stop row (K = all drafts accepted, bonus from row K)
  float mt;    // target row j softmax stats
  float st;
  float mz;    // draft row j softmax stats
  float sz;
};

// ---- Markov bias, one step -------------------------------------------------
size_t bias_tc_smem_bytes(int r, int N);
cudaError_t launch_bias_tc(const CUtensorMap& tmW, const __nv_bfloat16* U, const int32_t* prev,
                           float* bias, int B, int V, int r, WsHeader* hdr, uint64_t spin,
                           cudaStream_t st);
template <typename T>
cudaError_t launch_bias_fma(const T* U, const T* W, const int32_t* prev, float* bias, int B, int V,
                            int r, WsHeader* hdr, cudaStream_t st);

// ---- Stand-alone verification ----------------------------------------------
int verify_seg_len(int V);
size_t verify_ws_bytes(int B, int K, int V);
template <typename T, typename TD>
cudaError_t launch_verify(const T* target, const TD* draft_logits, const int32_t* draft,
                          int32_t* out, int32_t* tau, float* p_draft, float* q_draft, int B,
                          int K, int V, float temperature, int greedy, uint64_t seed,
                          uint64_t cycle, uint32_t row0, uint8_t* ws_body, WsHeader* hdr, int num_sms,
                          cudaStream_t st, int* launches);

// One persistent launch with early exit (rows up to 4096, slices whose ring
// fits shared memory); geometry false otherwise.
struct VerifyGeom {
  int G, seg;          // CTAs, tokens per CTA slice
  int S, slotb, doff;  // ring slots per warp, slot bytes, draft offset in a slot
  size_t smem;         // dynamic shared memory
};
bool verify_ee_geometry(int B, int V, int num_sms, int tsize, int dsize, int greedy,
                        VerifyGeom* g);
size_t verify_ee_ws_bytes(int B, int V, int num_sms);
template <typename T, typename TD>
cudaError_t launch_verify_ee(const T* target, const TD* draft_logits, const int32_t* draft,
                             const int32_t* vlen, int32_t* out, int32_t* tau, float* p_draft,
                             float* q_draft, int B, int K, int V, float temperature, int greedy,
                             uint64_t seed, uint64_t cycle, uint32_t row0, uint64_t spin,
                             bool trace, uint8_t* body, WsHeader* hdr, int num_sms,
                             cudaStream_t st);

// ---- Fused persistent draft (+ verify) ---------------------------------------
enum CycleMode : int32_t { MODE_CYCLE = 0, MODE_DRAFT = 1 };

struct CycleGeom {
  int G;        // CTAs (one per SM at most)
  int nc;       // 128-token chunks per CTA
  int nchunks;  // ceil(V / 128)
  int N;        // batch rows per group (MMA N): 16, 32 or 64
  bool tc;      // tensor-core bias
  size_t smem;  // dynamic shared memory bytes
};

// Decide the launch geometry; returns false (with a reason) if unsupported.
bool cycle_geometry(int B, int K, int V, int r, int dtype, uint32_t flags, int num_sms,
                    CycleGeom* g, const char** why);
size_t cycle_ws_bytes(int K, const CycleGeom& g);
constexpr int kTracePhases = 32;  // timeline slots per step
size_t cycle_trace_bytes(int K);

struct CycleLaunch {
  const void* base;
  const void* target;
  const void* U;
  const void* W;
  const int32_t* last_token;
  const int32_t* vlen;  // [C][B] per-row verify length K_b, or null (tensor-core cycle only)
  const float* conf;    // [C][B][K] confidence scores, or null (tensor-core cycle only)
  float conf_thr;       // prefix survival threshold for conf
  int32_t* next_token;  // [B] last emitted token per row, carried between cycles, or null
  int ncyc;             // cycles per launch (0 or 1: one)
  const void* Wh;       // [r][r] RNN head recurrence, or null (Markov head; tensor-core cycle only)
  int32_t* draft;
  int32_t* out;
  int32_t* tau;
  float* p_draft;
  float* q_draft;
  float* biased_out;
  int B, K, V, r, dtype, mode, greedy;
  float temperature;
  uint64_t seed, cycle, spin;
  uint32_t row0;  // global index of batch row 0 (Philox counter word 1)
  bool trace;
};

cudaError_t launch_cycle(const CycleLaunch& L, const CycleGeom& g, WsHeader* hdr, uint8_t* body,
                         const CUtensorMap* tmW, const CUtensorMap* tmBase, cudaStream_t st);

// Tensor-core path of the fused cycle (bf16, rank a multiple of 64 up to 256):
// W^T partly resident in tensor memory, double-buffered accumulators, exact
// bucket statistics.  Geometry returns false for other shapes.
bool cycle_tc_geometry(int B, int K, int V, int r, int dtype, uint32_t flags, int num_sms,
                       CycleGeom* g, const char** why);
size_t cycle_tc_ws_bytes(int K, int r, const CycleGeom& g);
cudaError_t launch_cycle_tc(const CycleLaunch& L, const CycleGeom& g, WsHeader* hdr, uint8_t* body,
                            const CUtensorMap* tmW, cudaStream_t st);

// ---- Tensor maps --------------------------------------------------------------
bool make_tmap_W(CUtensorMap* m, const void* W, int r, int V, int box_k);
constexpr int kCycleWBoxK = 16;  // rank rows per W box of the fused cycle (one MMA K-step)
bool make_tmap_base(CUtensorMap* m, const void* base, int dtype, int B, int K, int V, int N,
                    bool tc);

// ---- Debug ------------------------------------------------------------------------
cudaError_t launch_debug_philox(const uint32_t* ctr, const uint32_t* key, uint32_t* out, int n,
                                cudaStream_t st);
cudaError_t launch_debug_curand_philox(const uint32_t* ctr, const uint32_t* key, uint32_t* out,
                                       int n, cudaStream_t st);

}  // namespace specdec
