// A3: exact top-k selection of indexer scores.
//
// "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the indexer
// "selects top-k compressed positions" (model card: index_topk = 512). The
// selected set is the min(k, n) entries of largest score, ties resolved
// towards the smaller index; it is written in ascending index order and
// padded with -1.
//
// Method: radix select (MSD, 8-bit digits) on an order-preserving 32-bit key
// of the fp32 score finds the k-th largest key tau and how many entries equal
// to tau are still needed (kk). A final ordered pass keeps every entry with
// key > tau and the first kk entries (by index) with key == tau; an
// exclusive prefix count over the block gives each kept entry its output
// slot, so the output is in ascending index order and deterministic.
// One 1024-thread block per query.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

struct TopkShared {
  uint32_t hist[256];
  uint32_t warp_gt[kWarps], warp_eq[kWarps];
  uint32_t prefix, kk;
};

__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a) {
  __shared__ TopkShared sh;
  const int q = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = clamp_count(a.n_cmp[q], a.N_max, threadIdx.x == 0 ? a.status : nullptr);
  const float *s = a.scores + (size_t)q * a.N_max;
  int32_t *out = a.out_idx + (size_t)q * a.k;
  const int k = a.k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  if (threadIdx.x == 0) { sh.prefix = 0; sh.kk = (uint32_t)k; }
  uint32_t mask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (threadIdx.x < 256) sh.hist[threadIdx.x] = 0;
    __syncthreads();
    const uint32_t prefix = sh.prefix;
    for (int j = threadIdx.x; j < n; j += kThreads) {
      const uint32_t u = score_key(s[j]);
      if ((u & mask) == prefix) atomicAdd(&sh.hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane L owns bins 8L .. 8L+7; find the bin holding the kk-th largest.
      const uint32_t kk = sh.kk;
      uint32_t t = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) t += sh.hist[lane * 8 + i];
      uint32_t incl = t;  // inclusive suffix sum over lanes >= lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += y;
      }
      const uint32_t above = incl - t;
      if (above < kk && kk <= incl) {
        uint32_t c = above;
        for (int bin = lane * 8 + 7; bin >= lane * 8; --bin) {
          const uint32_t h = sh.hist[bin];
          if (c + h >= kk) {
            sh.kk = kk - c;
            sh.prefix = prefix | ((uint32_t)bin << shift);
            break;
          }
          c += h;
        }
      }
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t tau = sh.prefix, kk = sh.kk;
  // Ordered compaction: warp w scans the contiguous range [lo, hi).
  const int per_warp = (((n + kWarps - 1) / kWarps) + 31) & ~31;
  const int lo = min(n, warp * per_warp), hi = min(n, lo + per_warp);
  uint32_t g = 0, e = 0;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? score_key(s[j]) : 0u;
    g += __popc(__ballot_sync(0xffffffffu, j < hi && u > tau));
    e += __popc(__ballot_sync(0xffffffffu, j < hi && u == tau));
  }
  if (lane == 0) { sh.warp_gt[warp] = g; sh.warp_eq[warp] = e; }
  __syncthreads();
  uint32_t G = 0, E = 0;
  for (int w = 0; w < warp; ++w) { G += sh.warp_gt[w]; E += sh.warp_eq[w]; }
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? score_key(s[j]) : 0u;
    const bool is_gt = j < hi && u > tau, is_eq = j < hi && u == tau;
    const uint32_t mg = __ballot_sync(0xffffffffu, is_gt), me = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t Gl = G + __popc(mg & lt), El = E + __popc(me & lt);
    if (is_gt) out[Gl + min(El, kk)] = j;
    else if (is_eq && El < kk) out[Gl + El] = j;
    G += __popc(mg);
    E += __popc(me);
  }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream) {
  topk_kernel<<<a.Q, kThreads, 0, stream>>>(a);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace csa
