// Row f2: the indexer's own compressor, and the rotation / FP8 encoding of
// indexer rows.
//
// "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the indexer
// "has its own dedicated KV compressor with Hadamard rotation"; the model's
// quantization_config ("deepseek-ai/DeepSeek-V4-Flash-0731", table "Config
// changes") is FP8 E4M3 with dynamic scales. For entry j of the indexer's raw
// KV (the A1 window geometry, head dim D a power of two):
//     c = RMSNorm(pool_j(kv, gate, ape)) * norm_w          (as csa_compress)
//     k = c H_D / sqrt(D)                                    (Sylvester-Hadamard)
// and, when FP8 output is asked for, per row: scale = amax|k| / 448 (1 for a
// zero row), code = E4M3(k / scale), rounded to nearest even, saturating.
// The queries take the same rotation (csa_hadamard_rows), so scores are those
// of the unrotated rows in exact arithmetic.
//
// One warp per row: lane l holds elements [l EPL, l EPL + EPL) (EPL = D / 32);
// the transform is EPL-wide butterflies in registers, then five shuffle
// stages across lanes. fp32 arithmetic throughout.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRmsEps = 1e-6f;
constexpr int kWarps = 8;  // rows per 256-thread block

// In-warp orthonormal Hadamard transform of one row, y = x H / sqrt(32 EPL).
template <int EPL>
__device__ __forceinline__ void fwht_warp(float (&v)[EPL], int lane, float inv_sqrt_n) {
#pragma unroll
  for (int h = 1; h < EPL; h <<= 1)
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if ((i & h) == 0) {
        const float x = v[i], y = v[i + h];
        v[i] = x + y;
        v[i + h] = x - y;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1)
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = (lane & m) ? o - v[i] : v[i] + o;
    }
#pragma unroll
  for (int i = 0; i < EPL; ++i) v[i] *= inv_sqrt_n;
}

template <typename T>
__device__ __forceinline__ float ld_elem(const T *p) {
  return to_f(*p);
}

// Write one row held EPL values per lane: in the element type T, or as E4M3
// codes + a per-row scale (codes != nullptr).
template <typename T, int EPL>
__device__ __forceinline__ void store_row(float (&v)[EPL], int lane, T *out, uint8_t *codes, float *scale) {
  if (codes) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = amax > 0.f ? amax / 448.f : 1.f;
#pragma unroll
    for (int i = 0; i < EPL; i += 2) {
      const __nv_fp8x2_storage_t two =
          __nv_cvt_float2_to_fp8x2(make_float2(v[i] / sc, v[i + 1] / sc), __NV_SATFINITE, __NV_E4M3);
      *reinterpret_cast<__nv_fp8x2_storage_t *>(codes + lane * EPL + i) = two;
    }
    if (lane == 0) *scale = sc;
  } else {
#pragma unroll
    for (int i = 0; i < EPL; ++i) out[lane * EPL + i] = from_f<T>(v[i]);
  }
}

// One warp per (sequence, entry): pool + RMSNorm + rotation (+ FP8).
template <typename T, int EPL>
__global__ void __launch_bounds__(32 * kWarps) index_compress_kernel(CompressArgs a, uint8_t *codes, float *scales,
                                                                     long long scale_ss, float inv_sqrt_n) {
  pdl_wait();
  pdl_release();
  const int lane = threadIdx.x & 31;
  const long long e = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (e >= (long long)a.B * a.N) return;
  const int b = (int)(e / a.N), j = (int)(e - (long long)b * a.N);
  const T *kv = static_cast<const T *>(a.kv) + b * a.kv_ss + (long long)j * a.stride * a.D + lane * EPL;
  const T *gate = static_cast<const T *>(a.gate) + b * a.gate_ss + (long long)j * a.stride * a.D + lane * EPL;
  const float *ape = a.ape + lane * EPL;
  float m[EPL], l[EPL], acc[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
    acc[i] = 0.f;
  }
  // running softmax over the window positions, per dimension
  for (int p = 0; p < a.win; ++p) {
    float kf[EPL], x[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      kf[i] = ld_elem(kv + (long long)p * a.D + i);
      x[i] = (ld_elem(gate + (long long)p * a.D + i) + ape[(size_t)p * a.D + i]) * kLog2e;
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const float mx = fmaxf(m[i], x[i]);
      const float ex = exp2f(fminf(m[i], x[i]) - mx);
      const bool up = x[i] > m[i];
      const float s_old = up ? ex : 1.f, s_new = up ? 1.f : ex;
      l[i] = l[i] * s_old + s_new;
      acc[i] = acc[i] * s_old + kf[i] * s_new;
      m[i] = mx;
    }
  }
  float v[EPL], ss = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    v[i] = acc[i] / l[i];
    ss += v[i] * v[i];
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)a.D + kRmsEps);
#pragma unroll
  for (int i = 0; i < EPL; ++i) v[i] *= r * a.norm_w[lane * EPL + i];
  fwht_warp<EPL>(v, lane, inv_sqrt_n);
  const long long row = b * a.out_ss + (long long)j * a.D;
  store_row<T, EPL>(v, lane, static_cast<T *>(a.out) + row, codes ? codes + row : nullptr,
                    scales ? scales + b * scale_ss + j : nullptr);
}

// One warp per row of x [rows, D]: rotation (+ FP8).
template <typename T, int EPL>
__global__ void __launch_bounds__(32 * kWarps) hadamard_rows_kernel(const T *x, T *out, uint8_t *codes, float *scales,
                                                                    long long rows, float inv_sqrt_n) {
  pdl_wait();
  pdl_release();
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  constexpr int D = 32 * EPL;
  float v[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) v[i] = ld_elem(x + r * D + lane * EPL + i);
  fwht_warp<EPL>(v, lane, inv_sqrt_n);
  store_row<T, EPL>(v, lane, out ? out + r * D : nullptr, codes ? codes + r * D : nullptr, scales ? scales + r : nullptr);
}

template <typename T, int EPL>
cudaError_t launch_prep(const CompressArgs *ca, const void *x, void *out, uint8_t *codes, float *scales,
                        long long rows, long long scale_ss, cudaStream_t stream) {
  const float inv_sqrt_n = (float)(1.0 / sqrt(32.0 * EPL));
  const unsigned blocks = (unsigned)((rows + kWarps - 1) / kWarps);
  if (ca)
    return launch_pdl(index_compress_kernel<T, EPL>, dim3(blocks), dim3(32 * kWarps), 0, stream, *ca, codes, scales,
                      scale_ss, inv_sqrt_n);
  return launch_pdl(hadamard_rows_kernel<T, EPL>, dim3(blocks), dim3(32 * kWarps), 0, stream,
                    static_cast<const T *>(x), static_cast<T *>(out), codes, scales, rows, inv_sqrt_n);
}

template <typename T>
cudaError_t dispatch_d(int D, const CompressArgs *ca, const void *x, void *out, uint8_t *codes, float *scales,
                       long long rows, long long scale_ss, cudaStream_t stream) {
  switch (D) {
    case 64: return launch_prep<T, 2>(ca, x, out, codes, scales, rows, scale_ss, stream);
    case 128: return launch_prep<T, 4>(ca, x, out, codes, scales, rows, scale_ss, stream);
    case 256: return launch_prep<T, 8>(ca, x, out, codes, scales, rows, scale_ss, stream);
    case 512: return launch_prep<T, 16>(ca, x, out, codes, scales, rows, scale_ss, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_index_compress(const CompressArgs &a, uint8_t *codes, float *scales, long long scale_ss,
                                  cudaStream_t stream) {
  const long long rows = (long long)a.B * a.N;
  if (rows == 0) return cudaSuccess;
  return a.dtype == CSA_DTYPE_F32 ? dispatch_d<float>(a.D, &a, nullptr, nullptr, codes, scales, rows, scale_ss, stream)
                                  : dispatch_d<bf16>(a.D, &a, nullptr, nullptr, codes, scales, rows, scale_ss, stream);
}

cudaError_t launch_hadamard_rows(const void *x, void *out, uint8_t *codes, float *scales, long long rows, int D,
                                 int dtype, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  return dtype == CSA_DTYPE_F32 ? dispatch_d<float>(D, nullptr, x, out, codes, scales, rows, 0, stream)
                                : dispatch_d<bf16>(D, nullptr, x, out, codes, scales, rows, 0, stream);
}

}  // namespace csa
