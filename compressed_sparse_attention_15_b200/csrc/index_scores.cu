// A2: indexer scores.
//
// "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1, Indexer: the
// scorer uses dot-product attention with per-head importance weights. Score
// of compressed entry j for query q (sequence b = q / q_per_seq):
//     s[q,j] = sum_h wi[q,h] * max(0, qi[q,h,:] . ki[b,j,:]),   j < n_cmp[q].
//
// This file holds the generic fp32-FFMA kernel (any Hi <= 128, Di <= 256,
// fp32, bf16, or FP8 E4M3 codes with per-row scales: qi = sq * e4m3(codes),
// ki = sk * e4m3(codes)). The tensor-core kernel for the Flash shape (Hi = 64,
// Di = 128, bf16 or E4M3) lives in index_tc.cu; launch_index_scores picks one.
#include <cuda_fp8.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace csa {

cudaError_t launch_index_scores_tc(const ScoreArgs &a, cudaStream_t stream, bool *taken);

namespace {

constexpr int kTileJ = 64;  // entries per block

// Element value: fp32 / bf16 as is; a uint8 is an FP8 E4M3 code (the
// hardware conversion), its row scale applied by the caller.
template <typename T>
__device__ __forceinline__ float elem(T x) {
  if constexpr (std::is_same<T, uint8_t>::value) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(x, __NV_E4M3);
    return __half2float(__half(h));
  } else {
    return to_f(x);
  }
}

// Block: 256 threads = 4 head groups x 64 entries. Thread (g, e) sums heads
// h = g, g+4, ... for entry j0 + e; the four partial sums are then added.
template <typename T>
__global__ void __launch_bounds__(256) index_scores_generic_kernel(ScoreArgs a) {
  extern __shared__ float sm[];
  const int Hi = a.Hi, Di = a.Di;
  float *sq = sm;                         // [Hi][Di]
  float *sk = sq + Hi * Di;               // [64][Di + 1] (padded against bank conflicts)
  float *sw = sk + kTileJ * (Di + 1);     // [Hi]
  float *part = sw + Hi;                  // [4][64]
  pdl_wait();
  pdl_release();
  const int q = blockIdx.x;
  const int n = clamp_count(a.n_cmp[q], a.N_max, threadIdx.x == 0 ? a.status : nullptr);
  const int j0 = blockIdx.y * kTileJ;
  if (j0 >= n) return;
  const int b = q / a.q_per_seq;
  const T *qi = static_cast<const T *>(a.qi) + (size_t)q * Hi * Di;
  const T *ki = static_cast<const T *>(a.ki) + ((size_t)b * a.N_max + j0) * Di;
  constexpr bool kFp8 = std::is_same<T, uint8_t>::value;
  for (int i = threadIdx.x; i < Hi * Di; i += blockDim.x)
    sq[i] = kFp8 ? elem(qi[i]) * a.sq[(size_t)q * Hi + i / Di] : elem(qi[i]);
  for (int i = threadIdx.x; i < Hi; i += blockDim.x) sw[i] = a.wi[(size_t)q * Hi + i];
  const int rows = min(kTileJ, n - j0);
  for (int i = threadIdx.x; i < kTileJ * Di; i += blockDim.x) {
    const int r = i / Di, d = i - r * Di;
    float v = 0.f;
    if (r < rows) v = kFp8 ? elem(ki[(size_t)r * Di + d]) * a.sk[(size_t)b * a.N_max + j0 + r] : elem(ki[(size_t)r * Di + d]);
    sk[r * (Di + 1) + d] = v;
  }
  __syncthreads();
  const int e = threadIdx.x & 63, g = threadIdx.x >> 6;
  float acc = 0.f;
  for (int h = g; h < Hi; h += 4) {
    float dot = 0.f;
    const float *qh = sq + h * Di;
    const float *kr = sk + e * (Di + 1);
    for (int d = 0; d < Di; ++d) dot = fmaf(qh[d], kr[d], dot);
    acc = fmaf(sw[h], fmaxf(dot, 0.f), acc);
  }
  part[g * kTileJ + e] = acc;
  __syncthreads();
  if (threadIdx.x < kTileJ && e < rows)
    a.scores[(size_t)q * a.N_max + j0 + e] = (part[e] + part[kTileJ + e]) + (part[2 * kTileJ + e] + part[3 * kTileJ + e]);
}

}  // namespace

cudaError_t launch_index_scores(const ScoreArgs &a, cudaStream_t stream) {
  bool taken = false;
  cudaError_t err = launch_index_scores_tc(a, stream, &taken);
  if (taken) return err;
  const size_t smem = ((size_t)a.Hi * a.Di + (size_t)kTileJ * (a.Di + 1) + a.Hi + 4 * kTileJ) * sizeof(float);
  dim3 grid(a.Q, (a.N_max + kTileJ - 1) / kTileJ);
  static DeviceOnce attr;  // set for the largest size the ABI admits
  once_per_device(attr, [] {
    const int max_smem = (128 * 256 + kTileJ * 257 + 128 + 4 * kTileJ) * 4;
    cudaFuncSetAttribute(index_scores_generic_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    cudaFuncSetAttribute(index_scores_generic_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    cudaFuncSetAttribute(index_scores_generic_kernel<uint8_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  });
  if (a.dtype == CSA_DTYPE_E4M3)
    return launch_pdl(index_scores_generic_kernel<uint8_t>, grid, dim3(256), smem, stream, a);
  if (a.dtype == CSA_DTYPE_F32) return launch_pdl(index_scores_generic_kernel<float>, grid, dim3(256), smem, stream, a);
  return launch_pdl(index_scores_generic_kernel<bf16>, grid, dim3(256), smem, stream, a);
}

}  // namespace csa
