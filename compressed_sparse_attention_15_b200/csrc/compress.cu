// A1: gated-pooling KV compressor + RMSNorm.
//
// "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the compressor
// folds each window of raw per-token KV into one entry by a learned gated
// pooling with absolute position embeddings inside the window, then applies
// an RMSNorm. For entry j over tokens t = j*stride + i and dimension d:
//     a[i,d] = softmax_i(gate[t,d] + ape[i,d]),  c[d] = sum_i a[i,d] kv[t,d],
//     out = c / sqrt(mean(c^2) + 1e-6) * norm_w.
//
// Three kernels, all fp32 arithmetic:
//  * compress_window_kernel (bf16, D % 8 == 0): one CTA (or, for windows of
//    32+ tokens, a cluster of up to 8 CTAs splitting the positions) per
//    entry; the positions are split over G thread groups, each thread owns
//    one 16-byte vector (8 dims) and keeps a running (max, sum, weighted sum)
//    over its positions; the G partial states are merged through shared
//    memory; a cluster's blocks then each finish D / C of the dims from all
//    blocks' states through distributed shared memory. Used when there
//    are few entries (the per-step append) or long windows (HCA).
//  * compress_stream_kernel (bf16, CSA geometry win = 2 * stride): streams
//    many entries; WPR warps own a row (8 dims per lane), each 8-token window
//    is reduced with an exact two-pass softmax in registers (max, then exp2),
//    the half-window shared with the next entry is carried in registers, and
//    the RMSNorm sum is exchanged between the row's warps.
//  * compress_generic_kernel: any dtype / D / window (the fp32 path).
// The running-state merge is the usual log-sum-exp rescaling; it equals the
// two-pass definition up to rounding.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRmsEps = 1e-6f;

// RoPE of the pair (x0, x1) = dims (d, d + 1), d even, of entry j of sequence
// b when d lies in the rope dims (the last a.rope_dims). The angle is formed
// and reduced in double: positions reach 2^20 and beyond, where a float angle
// would keep no fractional bits.
__device__ __forceinline__ void rope_pair(const CompressArgs &a, int b, int j, int d, float &x0, float &x1) {
  const int d0 = a.D - a.rope_dims;
  if (a.rope_dims == 0 || d < d0) return;
  const double p = (double)((a.pos0 ? a.pos0[b] : 0) + (long long)j * a.stride + a.win - 1);
  const double ang = p * pow(a.rope_theta, -(double)(d - d0) / a.rope_dims);  // pair (d - d0) / 2
  double sn, cs;
  sincos(ang, &sn, &cs);
  const float c = (float)cs, s = (float)sn;
  const float y0 = x0 * c - x1 * s, y1 = x0 * s + x1 * c;
  x0 = y0;
  x1 = y1;
}

// RoPE of 8 consecutive dims [d, d + 8) held by one thread (d a multiple of 8).
__device__ __forceinline__ void rope8(const CompressArgs &a, int b, int j, int d, float (&c)[8]) {
  if (a.rope_dims == 0 || d + 8 <= a.D - a.rope_dims) return;
#pragma unroll
  for (int m = 0; m < 8; m += 2) rope_pair(a, b, j, d + m, c[m], c[m + 1]);
}

// ------------------------------------------------------------------ generic

template <typename T>
__global__ void __launch_bounds__(256) compress_generic_kernel(CompressArgs a) {
  extern __shared__ float c_smem[];
  pdl_wait();
  pdl_release();
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
    for (int d = lane; d < a.D; d += 32) {
      float x = c[d] * r * a.norm_w[d];
      if (a.rope_dims) {  // the pair partner comes from shared memory
        const int dp = d ^ 1;
        float y = c[dp] * r * a.norm_w[dp];
        if (d & 1) {
          rope_pair(a, b, j, dp, y, x);
        } else {
          rope_pair(a, b, j, d, x, y);
        }
      }
      o[d] = from_f<T>(x);
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------------ bf16 helpers

__device__ __forceinline__ void unpack8(const uint4 &v, float f[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 t = __bfloat1622float2(h[k]);
    f[2 * k] = t.x;
    f[2 * k + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float f[8]) {
  uint4 v;
  uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
    w[k] = *reinterpret_cast<uint32_t *>(&t);
  }
  return v;
}

// ------------------------------------------------------------------ window-parallel

// Block = G groups x nvec threads (nvec = D / 8, a multiple of 32); thread
// (g, v) handles dims [8v, 8v + 8) at window positions i = i0 + g, i0 + g + G,
// ... < i1. One cluster of C blocks per (sequence, entry): block c of the
// cluster takes positions [c P, c P + P), P = ceil(win / C); the C partial
// states are merged by block 0 through distributed shared memory.
// kRope: rotate the rope dims of each written entry (a.rope_dims > 0); its
// own instantiation, so the plain kernel carries none of the rotation's code
// or registers.
template <bool kRope>
__global__ void __launch_bounds__(512) compress_window_kernel(CompressArgs a, int G) {
  extern __shared__ float ws[];  // [G][3][8][nvec] partial states, then [32] sums, then [3][8][nvec] block state
  if (!a.late_wait) pdl_wait();
  pdl_release();
  // late_wait: complete only after the kernel this one follows
  auto finish = [&] {
    if (a.late_wait && threadIdx.x == 0) pdl_wait();
  };
  const int nvec = a.D / 8;
  const int v = threadIdx.x % nvec, g = threadIdx.x / nvec;
  const uint32_t C = cluster_size(), crank = cluster_rank();
  const int P = (a.win + (int)C - 1) / (int)C;
  const int pos0 = (int)crank * P, pos1 = min(a.win, pos0 + P);
  const long long e = blockIdx.x / C;
  const int b = (int)(e / a.N), j = (int)(e - (long long)b * a.N);
  const bf16 *kvj = static_cast<const bf16 *>(a.kv) + b * a.kv_ss + (long long)j * a.stride * a.D;
  const bf16 *gj = static_cast<const bf16 *>(a.gate) + b * a.gate_ss + (long long)j * a.stride * a.D;
  float m[8], l[8], acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    m[k] = -INFINITY;
    l[k] = 0.f;
    acc[k] = 0.f;
  }
  // positions pos0 + g, pos0 + g + G, ... with four rows of loads in flight per step
  for (int i0 = pos0 + g; i0 < pos1; i0 += 4 * G) {
    uint4 kvv[4], gv[4];
    float4 ap0[4], ap1[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * G;
      if (i < pos1) {
        kvv[u] = __ldg(reinterpret_cast<const uint4 *>(kvj + (long long)i * a.D) + v);
        gv[u] = __ldg(reinterpret_cast<const uint4 *>(gj + (long long)i * a.D) + v);
        ap0[u] = __ldg(reinterpret_cast<const float4 *>(a.ape + (size_t)i * a.D + 8 * v));
        ap1[u] = __ldg(reinterpret_cast<const float4 *>(a.ape + (size_t)i * a.D + 8 * v + 4));
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * G;
      if (i < pos1) {
        float kf[8], gf[8];
        unpack8(kvv[u], kf);
        unpack8(gv[u], gf);
        const float4 a0 = ap0[u], a1 = ap1[u];
        const float ap[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float x = (gf[k] + ap[k]) * kLog2e;
          const float mx = fmaxf(m[k], x);
          const float ex = exp2f(fminf(m[k], x) - mx);
          const bool up = x > m[k];
          const float s_old = up ? ex : 1.f, s_new = up ? 1.f : ex;
          l[k] = l[k] * s_old + s_new;
          acc[k] = acc[k] * s_old + kf[k] * s_new;
          m[k] = mx;
        }
      }
    }
  }
  // publish the G partial states
  float *sm = ws;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    sm[((g * 3 + 0) * 8 + k) * nvec + v] = m[k];
    sm[((g * 3 + 1) * 8 + k) * nvec + v] = l[k];
    sm[((g * 3 + 2) * 8 + k) * nvec + v] = acc[k];
  }
  __syncthreads();
  float *red = ws + (size_t)G * 3 * 8 * nvec;  // [32]
  float *blk = red + 32;                        // [3][8][nvec]: this block's merged state, or [D] results
  const int t = threadIdx.x;
  // Merge the G states, one dimension per thread: dim 8 vv + kk at
  // i = kk * nvec + vv (consecutive threads read consecutive words).
  float ssl = 0.f;
  for (int i = t; i < a.D; i += blockDim.x) {
    float M = -INFINITY;
    for (int h = 0; h < G; ++h) M = fmaxf(M, sm[(h * 3 + 0) * 8 * nvec + i]);
    float L = 0.f, A = 0.f;
    for (int h = 0; h < G; ++h) {
      const float mh = sm[(h * 3 + 0) * 8 * nvec + i];
      const float w = mh == -INFINITY ? 0.f : exp2f(mh - M);
      L += sm[(h * 3 + 1) * 8 * nvec + i] * w;
      A += sm[(h * 3 + 2) * 8 * nvec + i] * w;
    }
    if (C > 1) {
      blk[0 * 8 * nvec + i] = M;
      blk[1 * 8 * nvec + i] = L;
      blk[2 * 8 * nvec + i] = A;
    } else {
      const float cd = A / L;
      blk[i] = cd;
      ssl += cd * cd;
    }
  }
  if (C > 1) {
    // Block c of the cluster finishes dims [c D / C, (c + 1) D / C): merge
    // the C block states of each, then the RMSNorm with the cluster's total
    // sum of squares (every remote load of a thread issued before use).
    cluster_sync();  // every block's state is published
    const int per = a.D / (int)C;
    const bool mine = t < per;
    const int d = (int)crank * per + t;
    const int di = (d & 7) * nvec + (d >> 3);  // dim 8v + k lives at [.][k][v]
    float cd = 0.f;
    if (mine) {
      float mr[8], lr[8], ar[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < (int)C) {
          mr[r] = ld_peer_f(&blk[di], r);
          lr[r] = ld_peer_f(&blk[8 * nvec + di], r);
          ar[r] = ld_peer_f(&blk[16 * nvec + di], r);
        }
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < (int)C) M = fmaxf(M, mr[r]);
      float L = 0.f, A = 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < (int)C) {
          const float w = mr[r] == -INFINITY ? 0.f : exp2f(mr[r] - M);
          L += lr[r] * w;
          A += ar[r] * w;
        }
      cd = A / L;
    }
    const float ss = warp_sum(mine ? cd * cd : 0.f);
    if ((t & 31) == 0) red[t >> 5] = ss;  // at most 16 warps
    __syncthreads();
    if (t == 0) {
      float tot = 0.f;
      for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) tot += red[w];
      red[16] = tot;  // this block's share, read by the peers
    }
    cluster_sync();  // every block's share is published
    if (mine) {
      float sr[8], tot = 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < (int)C) sr[r] = ld_peer_f(&red[16], r);
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < (int)C) tot += sr[r];
      const float rn = 1.0f / sqrtf(tot / (float)a.D + kRmsEps);
      bf16 *o = static_cast<bf16 *>(a.out) + b * a.out_ss + (long long)j * a.D;
      float x = cd * rn * a.norm_w[d];
      if constexpr (kRope) {  // the pair partner is the neighbouring thread's dim
        float y = __shfl_xor_sync(0xffffffffu, x, 1);
        if (d & 1)
          rope_pair(a, b, j, d - 1, y, x);
        else
          rope_pair(a, b, j, d, x, y);
      }
      o[d] = __float2bfloat16_rn(x);
    }
    cluster_sync();  // no block leaves while a peer may still read its share
    finish();
    return;
  }
  const float ss = warp_sum(ssl);
  if ((t & 31) == 0) red[t >> 5] = ss;  // at most 16 warps
  __syncthreads();
  if (t < nvec) {
    float tot = 0.f;
    for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) tot += red[w];
    const float rn = 1.0f / sqrtf(tot / (float)a.D + kRmsEps);
    const float4 w0 = __ldg(reinterpret_cast<const float4 *>(a.norm_w + 8 * t));
    const float4 w1 = __ldg(reinterpret_cast<const float4 *>(a.norm_w + 8 * t + 4));
    const float nw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float c[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) c[k] = blk[k * nvec + t] * rn * nw[k];
    bf16 *o = static_cast<bf16 *>(a.out) + b * a.out_ss + (long long)j * a.D;
    if constexpr (kRope) rope8(a, b, j, 8 * t, c);
    reinterpret_cast<uint4 *>(o)[t] = pack8(c);
  }
  finish();
}

// ------------------------------------------------------------------ streaming (CSA)

// WPR warps own one row (8 dims per lane, D = 256 * WPR); each group of WPR
// warps walks a contiguous run of the flattened (sequence, entry) space.
// S = stride, window = 2 S; ape (pre-scaled by log2 e) lives in shared memory.
template <int WPR, int S, bool kRope>
__global__ void __launch_bounds__(256) compress_stream_kernel(CompressArgs a, long long per_group) {
  // (kRope as for compress_window_kernel)
  constexpr int W = 2 * S;
  extern __shared__ float ape_s[];  // [W][D] * log2 e
  __shared__ float grp_sum[8];
  const int D = a.D;
  pdl_wait();
  pdl_release();
  for (int i = threadIdx.x; i < W * D; i += blockDim.x) ape_s[i] = a.ape[i] * kLog2e;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = warp / WPR, sub = warp % WPR;
  const int v = sub * 32 + lane;  // this lane's 16-byte vector of the row
  const long long gid = (long long)blockIdx.x * (8 / WPR) + grp;
  const long long total = (long long)a.B * a.N;
  long long e = gid * per_group;
  const long long e1 = min(total, e + per_group);
  const bf16 *kv = static_cast<const bf16 *>(a.kv);
  const bf16 *gate = static_cast<const bf16 *>(a.gate);
  bf16 *out = static_cast<bf16 *>(a.out);
  const float4 n0 = __ldg(reinterpret_cast<const float4 *>(a.norm_w + 8 * v));
  const float4 n1 = __ldg(reinterpret_cast<const float4 *>(a.norm_w + 8 * v + 4));
  const float nw[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
  uint4 ck[S], cg[S];  // the carried half window (packed bf16)
  int cur_b = -1, cur_j = -2;
  for (; e < e1; ++e) {
    const int b = (int)(e / a.N);
    const int j = (int)(e - (long long)b * a.N);
    const bf16 *kvb = kv + b * a.kv_ss;
    const bf16 *gb = gate + b * a.gate_ss;
    if (b != cur_b || j != cur_j + 1) {
#pragma unroll
      for (int i = 0; i < S; ++i) {
        ck[i] = __ldg(reinterpret_cast<const uint4 *>(kvb + ((long long)j * S + i) * D) + v);
        cg[i] = __ldg(reinterpret_cast<const uint4 *>(gb + ((long long)j * S + i) * D) + v);
      }
    }
    cur_b = b;
    cur_j = j;
    uint4 nk[S], ng[S];
#pragma unroll
    for (int i = 0; i < S; ++i) {
      nk[i] = __ldg(reinterpret_cast<const uint4 *>(kvb + ((long long)j * S + S + i) * D) + v);
      ng[i] = __ldg(reinterpret_cast<const uint4 *>(gb + ((long long)j * S + S + i) * D) + v);
    }
    // pass 1: base-2 logits and their per-dim maximum over the window
    float x[W][8];
    float mx[8];
#pragma unroll
    for (int i = 0; i < W; ++i) {
      float gf[8];
      unpack8(i < S ? cg[i] : ng[i - S], gf);
      const float4 a0 = *reinterpret_cast<const float4 *>(ape_s + i * D + 8 * v);
      const float4 a1 = *reinterpret_cast<const float4 *>(ape_s + i * D + 8 * v + 4);
      const float ap[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        x[i][k] = fmaf(gf[k], kLog2e, ap[k]);
        mx[k] = i == 0 ? x[i][k] : fmaxf(mx[k], x[i][k]);
      }
    }
    // pass 2: weights, their sum and the weighted sum of kv
    float l[8], acc[8];
#pragma unroll
    for (int i = 0; i < W; ++i) {
      float kf[8];
      unpack8(i < S ? ck[i] : nk[i - S], kf);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float p = exp2f(x[i][k] - mx[k]);
        l[k] = i == 0 ? p : l[k] + p;
        acc[k] = i == 0 ? p * kf[k] : fmaf(p, kf[k], acc[k]);
      }
    }
    float c[8], ss = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      c[k] = acc[k] / l[k];
      ss = fmaf(c[k], c[k], ss);
    }
    ss = warp_sum(ss);
    if (WPR > 1) {
      // exchange the partial sums of the row's warps (one named barrier per group)
      if (lane == 0) grp_sum[warp] = ss;
      asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(32 * WPR) : "memory");
      ss = 0.f;
#pragma unroll
      for (int w = 0; w < WPR; ++w) ss += grp_sum[grp * WPR + w];
      asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(32 * WPR) : "memory");
    }
    const float r = 1.0f / sqrtf(ss / (float)D + kRmsEps);
#pragma unroll
    for (int k = 0; k < 8; ++k) c[k] = c[k] * r * nw[k];
    if constexpr (kRope) rope8(a, b, j, 8 * v, c);
    reinterpret_cast<uint4 *>(out + b * a.out_ss + (long long)j * D)[v] = pack8(c);
#pragma unroll
    for (int i = 0; i < S; ++i) {
      ck[i] = nk[i];
      cg[i] = ng[i];
    }
  }
}

int num_sms() { return device_sm_count(); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

template <int WPR, int S>
cudaError_t launch_stream(const CompressArgs &a, cudaStream_t stream) {
  const long long total = (long long)a.B * a.N;
  const int groups_per_block = 8 / WPR;  // 256 threads
  long long groups = (long long)num_sms() * groups_per_block * 2;
  if (groups > total) groups = total;
  const long long per = (total + groups - 1) / groups;
  groups = (total + per - 1) / per;
  const long long blocks = (groups + groups_per_block - 1) / groups_per_block;
  const size_t smem = (size_t)2 * S * a.D * sizeof(float);
  return launch_pdl(a.rope_dims ? compress_stream_kernel<WPR, S, true> : compress_stream_kernel<WPR, S, false>,
                    dim3((unsigned)blocks), dim3(256), smem, stream, a, per);
}

}  // namespace

cudaError_t launch_compress(const CompressArgs &a, cudaStream_t stream) {
  if (a.N <= 0) return cudaSuccess;
  const long long total = (long long)a.B * a.N;
  const bool vec_ok = a.dtype == CSA_DTYPE_BF16 && a.D % 8 == 0 && a.D >= 64 && a.D <= 1024 && aligned16(a.kv) &&
                      aligned16(a.gate) && aligned16(a.out) && aligned16(a.ape) && aligned16(a.norm_w) &&
                      a.kv_ss % 8 == 0 && a.gate_ss % 8 == 0 && a.out_ss % 8 == 0;
  if (vec_ok) {
    const bool csa4 = a.win == 8 && a.stride == 4;
    if (csa4 && total > 4LL * num_sms() && (a.D == 512 || a.D == 256))
      return a.D == 512 ? launch_stream<2, 4>(a, stream) : launch_stream<1, 4>(a, stream);
    if ((a.D / 8) % 32 == 0) {
      const int nvec = a.D / 8;
      // Long windows and few entries: a cluster of C blocks per entry, at
      // least 16 positions each, about two blocks per SM in all. C is a power
      // of two (it divides D) and at most 4: a block fills an SM, and
      // clusters of 8 such blocks do not all fit in the GPCs at once.
      int C = 1;
      if (a.win >= 32) {
        const long long fill = (2LL * num_sms() + total - 1) / total;
        while (2 * C <= 4 && 2 * C <= a.win / 16 && 2 * C <= fill) C *= 2;
      }
      const int P = (a.win + C - 1) / C;
      int G = P < 16 ? P : 16;
      while (G > 1 && G * nvec > 512) G >>= 1;
      const size_t smem = ((size_t)(G + 1) * 3 * 8 * nvec + 32) * sizeof(float);
      static DeviceOnce attr;
      once_per_device(attr, [] {
        for (auto kern : {compress_window_kernel<false>, compress_window_kernel<true>})
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(((size_t)4 * 8 * 512 + 32) * sizeof(float)));
      });
      return launch_pdl_cluster(a.rope_dims ? compress_window_kernel<true> : compress_window_kernel<false>,
                                dim3((unsigned)(total * C)), dim3(G * nvec), smem, stream, (unsigned)C, a, G);
    }
  }
  const int threads = 256, wpb = threads / 32;
  const size_t smem = (size_t)wpb * a.D * sizeof(float);
  long long blocks = (total + wpb - 1) / wpb;
  if (blocks > 65535LL * 16) blocks = 65535LL * 16;
  static DeviceOnce attr;
  once_per_device(attr, [] {
    cudaFuncSetAttribute(compress_generic_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * 4096 * 4);
    cudaFuncSetAttribute(compress_generic_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * 4096 * 4);
  });
  if (a.dtype == CSA_DTYPE_F32)
    return launch_pdl(compress_generic_kernel<float>, dim3((unsigned)blocks), dim3(threads), smem, stream, a);
  return launch_pdl(compress_generic_kernel<bf16>, dim3((unsigned)blocks), dim3(threads), smem, stream, a);
}

}  // namespace csa
