// Markov-head bias for one draft step (aigest.pl "DeepSeek prezentuje DSpark",
// section "Innowacje w tworzeniu tokenów": the sequential Markov head adds a
// bias that depends only on the preceding token, factorised at low rank):
//   bias[b, v] = sum_k U[prev[b], k] * W[k, v].
//
// Tensor-core form (bf16, r % 64 == 0): each CTA owns one 128-token chunk of
// the vocabulary and computes the transposed tile D[v, b] = W^T[v, :] . U_g^T
// with tcgen05.mma (M = 128 tokens, N = 16..64 batch rows, K = r), A = W^T
// staged by TMA with 128-byte swizzle (MN-major), B = the gathered U rows
// (K-major, swizzled by the gathering threads), D in tensor memory.
// FMA form (fp32 or forced): plain fp32 fused multiply-adds.
#include "common.cuh"
#include "kernels.cuh"

namespace specdec {

namespace {

constexpr int kChunk = 128;       // tokens per CTA (UMMA M)
constexpr int kKBlock = 64;       // rank elements per TMA box / smem stage (128 bytes of bf16)
constexpr int kStageBytes = kChunk * kKBlock * 2;  // 16 KB: two 64x64 boxes

__global__ void __launch_bounds__(160) k_bias_tc(const __grid_constant__ CUtensorMap tmW,
                                                 const __nv_bfloat16* __restrict__ U,
                                                 const int32_t* __restrict__ prev,
                                                 float* __restrict__ bias, int B, int V, int r,
                                                 int N, WsHeader* hdr, uint64_t spin) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int nkb = r / kKBlock;
  uint8_t* sW = smem;                                  // nkb stages of 16 KB
  uint8_t* sU = sW + (size_t)nkb * kStageBytes;        // nkb atoms of N x 128 B
  uint64_t* bars = reinterpret_cast<uint64_t*>(sU + (size_t)nkb * N * 128);
  uint64_t* full = bars;             // [nkb]
  uint64_t* mma_bar = bars + 4;      // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int v0 = blockIdx.x * kChunk;
  const uint32_t ncols = N <= 32 ? 32u : 64u;

  if (tid == 0) {
    for (int i = 0; i < nkb; ++i) mbar_init(&full[i], 1);
    mbar_init(mma_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = *tmem_slot;

  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmW);
    const uint64_t pol = policy_evict_last();
    for (int kb = 0; kb < nkb; ++kb) {
      mbar_arrive_expect_tx(&full[kb], kStageBytes);
      tma_load_2d(sW + (size_t)kb * kStageBytes, &tmW, &full[kb], v0, kb * kKBlock, pol);
      tma_load_2d(sW + (size_t)kb * kStageBytes + kStageBytes / 2, &tmW, &full[kb], v0 + 64,
                  kb * kKBlock, pol);
    }
  }

  const uint32_t idesc = idesc_bf16_f32(128, N, /*a_mn_major=*/true, /*b_mn_major=*/false);
  const int ngroups = (B + N - 1) / N;
  bool ok = true;
  for (int g = 0; g < ngroups; ++g) {
    // gather U[prev[b]] rows into the K-major, 128-byte-swizzled B operand
    if (warp < 4) {
      const int chunks_per_row = r / 8;  // 16-byte chunks
      for (int idx = tid; idx < N * chunks_per_row; idx += 128) {
        const int n = idx / chunks_per_row, c = idx % chunks_per_row;
        const int b = g * N + n;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (b < B) {
          int p = __ldg(prev + b);
          if (p < 0 || p >= V) {
            record_error(hdr, SPEC_ERR_TOKEN_RANGE, SITE_TOKEN_RANGE, b, p);
            p = 0;
          }
          val = __ldg(reinterpret_cast<const uint4*>(U + (size_t)p * r) + c);
        }
        const int ka = c >> 3, j = c & 7;
        uint8_t* dst = sU + (size_t)ka * N * 128 + n * 128 + ((j ^ (n & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = val;
      }
      fence_proxy_async_smem();
    }
    __syncthreads();
    if (warp == 4 && lane == 0) {
      tc_fence_after();
      for (int kb = 0; kb < nkb && ok; ++kb) {
        if (!mbar_wait_bounded(&full[kb], 0, spin, &hdr->abort)) {
          record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_FULL, kb, g);
          ok = false;
          break;
        }
        const uint32_t a_base = smem_u32(sW + (size_t)kb * kStageBytes);
        const uint32_t b_base = smem_u32(sU + (size_t)kb * N * 128);
#pragma unroll
        for (int kk = 0; kk < kKBlock / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(a_base + kk * 2048, 8192, 1024);
          const uint64_t bd = smem_desc_sw128(b_base + kk * 32, 16, 1024);
          umma_bf16(taddr, ad, bd, idesc, (kb | kk) != 0);
        }
      }
      umma_commit(mma_bar);  // arrives even after a give-up, once issued ops finish
    }
    if (warp < 4) {
      if (!mbar_wait_bounded(mma_bar, g & 1, spin, &hdr->abort)) {
        record_error(hdr, SPEC_ERR_TIMEOUT, SITE_MBAR_MMA, g, 0);
        ok = false;
      }
      tc_fence_after();
      const int v = v0 + warp * 32 + lane;
      for (int c16 = 0; c16 < N / 16; ++c16) {
        float vals[16];
        tmem_ld16(taddr + ((uint32_t)(warp * 32) << 16) + c16 * 16, vals);
        tmem_ld_wait();
        if (ok && v < V) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int b = g * N + c16 * 16 + j;
            if (b < B) bias[(size_t)b * V + v] = vals[j];
          }
        }
      }
      tc_fence_before();
    }
    // the same decision in every thread
    if (__syncthreads_or(!ok || ld_volatile_u32(&hdr->abort))) break;
  }
  // drain: every TMA load issued above must land before the CTA exits
  if (warp == 4 && lane == 0) {
    for (int kb = 0; kb < nkb; ++kb) mbar_drain(&full[kb], 0);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(taddr, ncols);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_bias_fma(const T* __restrict__ U, const T* __restrict__ W,
                                                  const int32_t* __restrict__ prev,
                                                  float* __restrict__ bias, int B, int V, int r,
                                                  WsHeader* hdr) {
  extern __shared__ float sUf[];  // [16][r]
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  for (int g = 0; g < B; g += 16) {
    const int nb = min(16, B - g);
    __syncthreads();
    for (int idx = threadIdx.x; idx < nb * r; idx += blockDim.x) {
      const int n = idx / r, k = idx % r;
      int p = __ldg(prev + g + n);
      if (p < 0 || p >= V) {
        if (k == 0) record_error(hdr, SPEC_ERR_TOKEN_RANGE, SITE_TOKEN_RANGE, g + n, p);
        p = 0;
      }
      sUf[n * r + k] = load_f(U, (int64_t)p * r + k);
    }
    __syncthreads();
    if (v < V) {
      float acc[16];
#pragma unroll
      for (int n = 0; n < 16; ++n) acc[n] = 0.f;
      for (int k = 0; k < r; ++k) {
        const float w = load_f(W, (int64_t)k * V + v);
#pragma unroll
        for (int n = 0; n < 16; ++n) acc[n] = fmaf(sUf[n * r + k], w, acc[n]);
      }
      for (int n = 0; n < nb; ++n) bias[(size_t)(g + n) * V + v] = acc[n];
    }
  }
}

}  // namespace

size_t bias_tc_smem_bytes(int r, int N) {
  return 1024 + (size_t)(r / kKBlock) * kStageBytes + (size_t)(r / kKBlock) * N * 128 + 64;
}

cudaError_t launch_bias_tc(const CUtensorMap& tmW, const __nv_bfloat16* U, const int32_t* prev,
                           float* bias, int B, int V, int r, WsHeader* hdr, uint64_t spin,
                           cudaStream_t st) {
  const int N = B <= 16 ? 16 : (B <= 32 ? 32 : 64);
  const size_t smem = bias_tc_smem_bytes(r, N);
  cudaError_t e = cudaFuncSetAttribute(k_bias_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = (V + kChunk - 1) / kChunk;
  k_bias_tc<<<grid, 160, smem, st>>>(tmW, U, prev, bias, B, V, r, N, hdr, spin);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_bias_fma(const T* U, const T* W, const int32_t* prev, float* bias, int B, int V,
                            int r, WsHeader* hdr, cudaStream_t st) {
  const size_t smem = (size_t)16 * r * sizeof(float);
  const int grid = (V + 255) / 256;
  k_bias_fma<T><<<grid, 256, smem, st>>>(U, W, prev, bias, B, V, r, hdr);
  return cudaGetLastError();
}
template cudaError_t launch_bias_fma<float>(const float*, const float*, const int32_t*, float*,
                                            int, int, int, WsHeader*, cudaStream_t);
template cudaError_t launch_bias_fma<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                    const int32_t*, float*, int, int, int,
                                                    WsHeader*, cudaStream_t);

}  // namespace specdec
