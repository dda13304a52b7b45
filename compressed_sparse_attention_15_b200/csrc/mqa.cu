// A4 / A5: MQA over compressed rows + sliding window + attention sink.
//
// "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1 (sliding window
// of the nearest 128 tokens; learnable per-head attention sink) and section 2
// (keys and values share one head_dim = 512 representation). For query q of
// sequence b and head h, over the row set
//     R = {kv_cmp[b, idx[q, r]] : idx >= 0}  (CSA)  or  {kv_cmp[b, j] : j < n_cmp[q]}  (HCA)
//       U {kv_win[b, t] : max(0, e - W + 1) <= t <= e},  e = win_end[q],
// logits scale * q_h . row (K = V) plus the unscaled sink logit with a zero
// value; out_h = softmax-weighted sum of the rows.
//
// This file holds the generic fp32-FFMA kernel (any H <= 128, D <= 1024,
// fp32 or bf16): one block per (query, group of HG heads) walks the whole
// row list in chunks of 32 rows with an online softmax. The tensor-core
// split-K kernel for the Flash shape (H = 64, D = 512, bf16) is in mqa_tc.cu.
#include "common.cuh"
#include "kernels.h"

namespace csa {

cudaError_t launch_mqa_tc(const MqaArgs &a, cudaStream_t stream, bool *taken);
size_t mqa_tc_partial_bytes(int Q, int H, int D, int rows_max);

namespace {

constexpr int kRC = 32;       // rows per chunk
constexpr int kThreads = 256;
constexpr int kMaxDPT = 4;    // dims per thread: D <= 1024

template <typename T, int HG>
__global__ void __launch_bounds__(kThreads) mqa_generic_kernel(MqaArgs a) {
  extern __shared__ float sm[];
  const int D = a.D, H = a.H;
  float *qs = sm;                   // [HG][D]
  float *rows = qs + HG * D;        // [kRC][D]
  float *S = rows + kRC * D;        // [HG][kRC]
  __shared__ const T *rowptr[kRC];
  __shared__ float m_s[HG], l_s[HG], alpha_s[HG];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qq = blockIdx.x, h0 = blockIdx.y * HG;
  pdl_wait();
  pdl_release();
  const int b = qq / a.q_per_seq;
  uint32_t *st = tid == 0 ? a.status : nullptr;
  const int nsel = a.idx ? a.k : clamp_count(a.n_cmp[qq], a.N_max, st);
  int e = a.win_end[qq];
  if (e < 0 || e >= a.T_raw) {
    raise_status(st, CSA_STATUS_BAD_WINDOW);
    e = e < 0 ? 0 : a.T_raw - 1;
  }
  const int wlo = max(0, e - a.win_len + 1);
  const int R = nsel + (e - wlo + 1);
  const T *kv_cmp = static_cast<const T *>(a.kv_cmp) + (size_t)b * a.N_max * D;
  const T *kv_win = static_cast<const T *>(a.kv_win) + (size_t)b * a.T_raw * D;
  const T *qp = static_cast<const T *>(a.q) + ((size_t)qq * H + h0) * D;
  for (int i = tid; i < HG * D; i += kThreads) qs[i] = to_f(qp[i]);
  if (tid < HG) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }
  float o[HG][kMaxDPT];
#pragma unroll
  for (int h = 0; h < HG; ++h)
#pragma unroll
    for (int i = 0; i < kMaxDPT; ++i) o[h][i] = 0.f;

  for (int r0 = 0; r0 < R; r0 += kRC) {
    __syncthreads();
    if (tid < kRC) {
      const int r = r0 + tid;
      const T *p = nullptr;
      if (r < nsel) {
        int j = a.idx ? a.idx[(size_t)qq * a.k + r] : r;
        if (j < -1 || j >= a.N_max) { raise_status(a.status, CSA_STATUS_BAD_INDEX); j = -1; }
        if (j >= 0) p = kv_cmp + (size_t)j * D;
      } else if (r < R) {
        p = kv_win + (size_t)(wlo + r - nsel) * D;
      }
      rowptr[tid] = p;
    }
    __syncthreads();
    for (int i = tid; i < kRC * D; i += kThreads) {
      const int rr = i / D, d = i - rr * D;
      const T *p = rowptr[rr];
      rows[i] = p ? to_f(p[d]) : 0.f;
    }
    __syncthreads();
    for (int rr = warp; rr < kRC; rr += kThreads / 32) {
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        float dot = 0.f;
        for (int d = lane; d < D; d += 32) dot = fmaf(qs[h * D + d], rows[rr * D + d], dot);
        dot = warp_sum(dot);
        if (lane == 0) S[h * kRC + rr] = rowptr[rr] ? dot * a.scale : -INFINITY;
      }
    }
    __syncthreads();
    if (warp < HG) {
      const int h = warp;
      const float x = S[h * kRC + lane];
      const float m_old = m_s[h];
      const float m_new = fmaxf(m_old, warp_max(x));
      float p = 0.f, alpha = 1.f;
      if (m_new != -INFINITY) {
        p = expf(x - m_new);
        alpha = expf(m_old - m_new);
      }
      S[h * kRC + lane] = p;
      const float sum = warp_sum(p);
      if (lane == 0) {
        l_s[h] = l_s[h] * alpha + sum;
        m_s[h] = m_new;
        alpha_s[h] = alpha;
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kMaxDPT; ++i) {
      const int d = tid + kThreads * i;
      if (d < D) {
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          float acc = o[h][i] * alpha_s[h];
          for (int rr = 0; rr < kRC; ++rr) acc = fmaf(S[h * kRC + rr], rows[rr * D + d], acc);
          o[h][i] = acc;
        }
      }
    }
  }
  __syncthreads();
  T *out = static_cast<T *>(a.out) + ((size_t)qq * H + h0) * D;
#pragma unroll
  for (int h = 0; h < HG; ++h) {
    const float m = m_s[h], l = l_s[h], sink = a.sink[h0 + h];
    const float M = fmaxf(m, sink);
    const float wm = m == -INFINITY ? 0.f : expf(m - M);
    const float f = wm / (l * wm + expf(sink - M));
#pragma unroll
    for (int i = 0; i < kMaxDPT; ++i) {
      const int d = tid + kThreads * i;
      if (d < D) out[(size_t)h * D + d] = from_f<T>(o[h][i] * f);
    }
  }
}

template <typename T, int HG>
cudaError_t launch_generic(const MqaArgs &a, cudaStream_t stream) {
  const size_t smem = ((size_t)(HG + kRC) * a.D + HG * kRC) * sizeof(float);
  static DeviceOnce attr;  // set for the largest D the ABI admits
  once_per_device(attr, [] {
    cudaFuncSetAttribute(mqa_generic_kernel<T, HG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(((size_t)(HG + kRC) * 1024 + HG * kRC) * sizeof(float)));
  });
  dim3 grid(a.Q, a.H / HG);
  return launch_pdl(mqa_generic_kernel<T, HG>, grid, dim3(kThreads), smem, stream, a);
}

template <typename T>
cudaError_t launch_generic_t(const MqaArgs &a, cudaStream_t stream) {
  if (a.H % 8 == 0) return launch_generic<T, 8>(a, stream);
  if (a.H % 4 == 0) return launch_generic<T, 4>(a, stream);
  if (a.H % 2 == 0) return launch_generic<T, 2>(a, stream);
  return launch_generic<T, 1>(a, stream);
}

}  // namespace

size_t mqa_partial_bytes(int Q, int H, int D, int rows_max) { return mqa_tc_partial_bytes(Q, H, D, rows_max); }

cudaError_t launch_mqa(const MqaArgs &a, cudaStream_t stream) {
  bool taken = false;
  cudaError_t err = launch_mqa_tc(a, stream, &taken);
  if (taken) return err;
  return a.dtype == CSA_DTYPE_F32 ? launch_generic_t<float>(a, stream) : launch_generic_t<bf16>(a, stream);
}

}  // namespace csa
