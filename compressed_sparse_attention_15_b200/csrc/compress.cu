// A1: gated-pooling KV compressor + RMSNorm.
//
// "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the compressor
// folds each window of raw per-token KV into one entry by a learned gated
// pooling with absolute position embeddings inside the window, then applies
// an RMSNorm. For entry j over tokens t = j*stride + i and dimension d:
//     a[i,d] = softmax_i(gate[t,d] + ape[i,d]),  c[d] = sum_i a[i,d] kv[t,d],
//     out = c / sqrt(mean(c^2) + 1e-6) * norm_w.
//
// The softmax is evaluated in one streaming pass per dimension with a running
// maximum (one exponential per window element): for each new logit x,
//     m' = max(m, x), e = exp(min(m, x) - m'),
//     (l, acc) <- x > m ? (l*e + 1, acc*e + v) : (l + e, acc + e*v).
// This is the standard online-softmax recurrence; it equals the two-pass
// definition up to rounding.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRmsEps = 1e-6f;

// Generic kernel: one warp per entry, lanes stride over D. Any dtype, any D,
// any window. fp32 path and fallback for unaligned bf16 tensors.
template <typename T>
__global__ void __launch_bounds__(256) compress_generic_kernel(CompressArgs a) {
  extern __shared__ float c_smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, wpb = blockDim.x >> 5;
  float *c = c_smem + (size_t)warp * a.D;
  const long long total = (long long)a.B * a.N;
  const T *kv = static_cast<const T *>(a.kv);
  const T *gate = static_cast<const T *>(a.gate);
  T *out = static_cast<T *>(a.out);
  for (long long e = (long long)blockIdx.x * wpb + warp; e < total; e += (long long)gridDim.x * wpb) {
    const int b = (int)(e / a.N), j = (int)(e % a.N);
    const T *kvj = kv + b * a.kv_ss + (long long)j * a.stride * a.D;
    const T *gj = gate + b * a.gate_ss + (long long)j * a.stride * a.D;
    float ss = 0.f;
    for (int d = lane; d < a.D; d += 32) {
      float m = -INFINITY, l = 0.f, acc = 0.f;
      for (int i = 0; i < a.win; ++i) {
        const float x = to_f(gj[(long long)i * a.D + d]) + a.ape[(size_t)i * a.D + d];
        const float v = to_f(kvj[(long long)i * a.D + d]);
        const float mx = fmaxf(m, x);
        const float ex = expf(fminf(m, x) - mx);
        const bool up = x > m;
        const float s_old = up ? ex : 1.f, s_new = up ? 1.f : ex;
        l = l * s_old + s_new;
        acc = acc * s_old + v * s_new;
        m = mx;
      }
      const float cd = acc / l;
      c[d] = cd;
      ss += cd * cd;
    }
    ss = warp_sum(ss);
    const float r = 1.0f / sqrtf(ss / (float)a.D + kRmsEps);
    __syncwarp();
    T *o = out + b * a.out_ss + (long long)j * a.D;
    for (int d = lane; d < a.D; d += 32) o[d] = from_f<T>(c[d] * r * a.norm_w[d]);
    __syncwarp();
  }
}

// Vectorised bf16 kernel (D <= 512, D % 8 == 0). One warp owns a whole output
// row: lane L holds the 16-byte vectors L, L+32, ... (VPL of them, 8 dims
// each), so the RMSNorm is a warp reduction and all loads/stores are 16-byte
// and coalesced. Each warp walks a contiguous run of entries of one
// sequence. When win == 2*stride
// (the overlapping CSA windows) the second half of a window is kept in
// registers and reused as the first half of the next window, so every raw
// token is read from memory once.
struct alignas(16) V8 {
  __nv_bfloat162 h[4];
};

__device__ __forceinline__ void unpack(const V8 &v, float f[8]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 t = __bfloat1622float2(v.h[k]);
    f[2 * k] = t.x;
    f[2 * k + 1] = t.y;
  }
}

template <int VPL>
struct RowState {
  float m[VPL][8], l[VPL][8], acc[VPL][8];
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int v = 0; v < VPL; ++v)
#pragma unroll
      for (int k = 0; k < 8; ++k) { m[v][k] = -INFINITY; l[v][k] = 0.f; acc[v][k] = 0.f; }
  }
  // Fold one token (its 8-dim vectors) seen at window position i.
  __device__ __forceinline__ void fold(const V8 (&kv)[VPL], const V8 (&g)[VPL], const float *ape_i,
                                       int lane, int nvec) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int vec = lane + 32 * v;
      if (vec < nvec) {
        float kf[8], gf[8];
        unpack(kv[v], kf);
        unpack(g[v], gf);
        const float4 a0 = __ldg(reinterpret_cast<const float4 *>(ape_i + vec * 8));
        const float4 a1 = __ldg(reinterpret_cast<const float4 *>(ape_i + vec * 8 + 4));
        const float ap[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float x = (gf[k] + ap[k]) * kLog2e;  // base-2 logit
          const float mx = fmaxf(m[v][k], x);
          const float ex = exp2f(fminf(m[v][k], x) - mx);
          const bool up = x > m[v][k];
          const float s_old = up ? ex : 1.f, s_new = up ? 1.f : ex;
          l[v][k] = l[v][k] * s_old + s_new;
          acc[v][k] = acc[v][k] * s_old + kf[k] * s_new;
          m[v][k] = mx;
        }
      }
    }
  }
};

template <int VPL>
__device__ __forceinline__ void load_tok(V8 (&dst)[VPL], const bf16 *row, int lane, int nvec) {
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int vec = lane + 32 * v;
    if (vec < nvec) {
      const uint4 r = __ldg(reinterpret_cast<const uint4 *>(row) + vec);
      dst[v] = *reinterpret_cast<const V8 *>(&r);
    }
  }
}

template <int VPL>
__device__ __forceinline__ void finish_row(RowState<VPL> &st, const float *norm_w, bf16 *orow, int lane,
                                           int nvec, int D) {
  float ss = 0.f;
#pragma unroll
  for (int v = 0; v < VPL; ++v)
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float c = (lane + 32 * v < nvec) ? st.acc[v][k] / st.l[v][k] : 0.f;
      st.acc[v][k] = c;
      ss += c * c;
    }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)D + kRmsEps);
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int vec = lane + 32 * v;
    if (vec < nvec) {
      const float4 w0 = __ldg(reinterpret_cast<const float4 *>(norm_w + vec * 8));
      const float4 w1 = __ldg(reinterpret_cast<const float4 *>(norm_w + vec * 8 + 4));
      const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      V8 o;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        o.h[k] = __floats2bfloat162_rn(st.acc[v][2 * k] * r * w[2 * k], st.acc[v][2 * k + 1] * r * w[2 * k + 1]);
      reinterpret_cast<uint4 *>(orow)[vec] = *reinterpret_cast<const uint4 *>(&o);
    }
  }
}

// Each warp: entries [e0, e1) of the flattened (sequence, entry) space,
// restarting the carry at sequence boundaries.
template <int VPL, int CARRY_S>
__global__ void __launch_bounds__(256) compress_bf16_kernel(CompressArgs a, long long per_warp) {
  const int lane = threadIdx.x & 31;
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long total = (long long)a.B * a.N;
  long long e = gw * per_warp;
  const long long e1 = min(total, e + per_warp);
  if (e >= e1) return;
  const int nvec = a.D / 8;
  const bf16 *kv = static_cast<const bf16 *>(a.kv);
  const bf16 *gate = static_cast<const bf16 *>(a.gate);
  bf16 *out = static_cast<bf16 *>(a.out);
  RowState<VPL> st;
  if (CARRY_S > 0) {
    constexpr int S = CARRY_S > 0 ? CARRY_S : 1;  // win == 2 * S == 2 * stride
    V8 ck[S][VPL], cg[S][VPL];
    int cur_b = -1;
    int j = 0;
    for (; e < e1; ++e) {
      const int b = (int)(e / a.N);
      j = (int)(e - (long long)b * a.N);
      const bf16 *kvb = kv + b * a.kv_ss;
      const bf16 *gb = gate + b * a.gate_ss;
      if (b != cur_b) {  // (re)load the first half of the window
#pragma unroll
        for (int i = 0; i < S; ++i) {
          load_tok<VPL>(ck[i], kvb + ((long long)j * S + i) * a.D, lane, nvec);
          load_tok<VPL>(cg[i], gb + ((long long)j * S + i) * a.D, lane, nvec);
        }
        cur_b = b;
      }
      V8 nk[S][VPL], ng[S][VPL];
#pragma unroll
      for (int i = 0; i < S; ++i) {
        load_tok<VPL>(nk[i], kvb + ((long long)j * S + S + i) * a.D, lane, nvec);
        load_tok<VPL>(ng[i], gb + ((long long)j * S + S + i) * a.D, lane, nvec);
      }
      st.reset();
#pragma unroll
      for (int i = 0; i < S; ++i) st.fold(ck[i], cg[i], a.ape + (size_t)i * a.D, lane, nvec);
#pragma unroll
      for (int i = 0; i < S; ++i) st.fold(nk[i], ng[i], a.ape + (size_t)(S + i) * a.D, lane, nvec);
      finish_row<VPL>(st, a.norm_w, out + b * a.out_ss + (long long)j * a.D, lane, nvec, a.D);
#pragma unroll
      for (int i = 0; i < S; ++i)
#pragma unroll
        for (int v = 0; v < VPL; ++v) { ck[i][v] = nk[i][v]; cg[i][v] = ng[i][v]; }
    }
  } else {
    for (; e < e1; ++e) {
      const int b = (int)(e / a.N);
      const int j = (int)(e - (long long)b * a.N);
      const bf16 *kvj = kv + b * a.kv_ss + (long long)j * a.stride * a.D;
      const bf16 *gj = gate + b * a.gate_ss + (long long)j * a.stride * a.D;
      st.reset();
      int i = 0;
      for (; i + 4 <= a.win; i += 4) {  // four tokens in flight per step
        V8 tk[4][VPL], tg[4][VPL];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          load_tok<VPL>(tk[u], kvj + (long long)(i + u) * a.D, lane, nvec);
          load_tok<VPL>(tg[u], gj + (long long)(i + u) * a.D, lane, nvec);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) st.fold(tk[u], tg[u], a.ape + (size_t)(i + u) * a.D, lane, nvec);
      }
      for (; i < a.win; ++i) {
        V8 tk[VPL], tg[VPL];
        load_tok<VPL>(tk, kvj + (long long)i * a.D, lane, nvec);
        load_tok<VPL>(tg, gj + (long long)i * a.D, lane, nvec);
        st.fold(tk, tg, a.ape + (size_t)i * a.D, lane, nvec);
      }
      finish_row<VPL>(st, a.norm_w, out + b * a.out_ss + (long long)j * a.D, lane, nvec, a.D);
    }
  }
}

int g_num_sms = 0;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_num_sms = n > 0 ? n : 148;
  }
  return g_num_sms;
}

template <int VPL, int CARRY_S>
cudaError_t launch_bf16(const CompressArgs &a, cudaStream_t stream) {
  const long long total = (long long)a.B * a.N;
  // About 16 resident warps per SM, each walking a contiguous run.
  long long warps = (long long)num_sms() * 16;
  if (warps > total) warps = total;
  const long long per_warp = (total + warps - 1) / warps;
  warps = (total + per_warp - 1) / per_warp;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  compress_bf16_kernel<VPL, CARRY_S><<<(unsigned)blocks, threads, 0, stream>>>(a, per_warp);
  note_launches(1);
  return cudaGetLastError();
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

cudaError_t launch_compress(const CompressArgs &a, cudaStream_t stream) {
  if (a.N <= 0) return cudaSuccess;
  const bool vec_ok = a.dtype == CSA_DTYPE_BF16 && a.D % 8 == 0 && a.D <= 512 && aligned16(a.kv) &&
                      aligned16(a.gate) && aligned16(a.out) && aligned16(a.ape) && aligned16(a.norm_w) &&
                      a.kv_ss % 8 == 0 && a.gate_ss % 8 == 0 && a.out_ss % 8 == 0;
  if (vec_ok) {
    const int nvec = a.D / 8;
    const bool carry4 = a.win == 8 && a.stride == 4;  // the CSA geometry
    if (nvec <= 32) return carry4 ? launch_bf16<1, 4>(a, stream) : launch_bf16<1, 0>(a, stream);
    return carry4 ? launch_bf16<2, 4>(a, stream) : launch_bf16<2, 0>(a, stream);
  }
  const int threads = 256, wpb = threads / 32;
  const size_t smem = (size_t)wpb * a.D * sizeof(float);
  const long long total = (long long)a.B * a.N;
  long long blocks = (total + wpb - 1) / wpb;
  if (blocks > 65535LL * 16) blocks = 65535LL * 16;
  static bool attr_set = false;  // the attribute is a per-function fact: set it once
  if (!attr_set) {
    cudaFuncSetAttribute(compress_generic_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * 4096 * 4);
    cudaFuncSetAttribute(compress_generic_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * 4096 * 4);
    attr_set = true;
  }
  if (a.dtype == CSA_DTYPE_F32)
    compress_generic_kernel<float><<<(unsigned)blocks, threads, smem, stream>>>(a);
  else
    compress_generic_kernel<bf16><<<(unsigned)blocks, threads, smem, stream>>>(a);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace csa
