// A3: exact top-k selection of indexer scores.
//
// "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the indexer
// "selects top-k compressed positions" (model card: index_topk = 512). The
// selected set is the min(k, n) entries of largest score, ties resolved
// towards the smaller index; it is written in ascending index order and
// padded with -1.
//
// Method: radix select (MSD, 11-bit digits over the occupied key range) on
// an order-preserving 32-bit key of each fp32 score finds the k-th largest
// key tau and how many entries equal to tau are still needed (kk). A final
// ordered pass keeps every entry with key > tau and the first kk entries (by
// index) with key == tau; per-warp ballots and an exclusive prefix over the
// block give each kept entry its output slot, so the output is ascending and
// deterministic.
//
// Launch shapes. Few queries (a decode batch): the list of one query is cut
// into C contiguous slices, one CTA of a thread-block cluster each (C <= 8,
// about SMs / Q); the slices' histograms are summed through distributed
// shared memory at every radix pass, and each CTA emits its own slice at the
// offset given by the counts of the slices before it. Many queries: one
// 1024-thread CTA per query with the keys cached in shared memory (up to
// 48K entries). Longer lists with many queries take two stages: the exact
// top-k of 4K-32K-entry segments in parallel, then the same selection over
// the concatenated segment winners. Without scratch space a single CTA per
// query does it all (re-reading the scores per pass beyond 48K entries).
#include "cluster_select.cuh"
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kSmemKeys = 48 * 1024;

using sel::kFew;

struct TopkShared {
  uint32_t hist[kBins];
  uint32_t scan[kWarps];
  uint32_t warp_gt[kWarps], warp_eq[kWarps];
  uint32_t prefix, kk, kmin, krange, bcnt, ncand;
  uint32_t cand[kFew];
};

template <bool kCached>
__device__ __forceinline__ uint32_t key_at(const uint32_t *keys, const float *s, int j) {
  return kCached ? keys[j] : score_key(s[j]);
}

// Select the k largest of n keys (ties -> smaller position) and call
// emit(slot, position, key) for each, slots 0..k-1 in ascending position.
// The radix digits are taken over (key - min key), from the highest set bit
// of the key range down, so the first digit already splits the keys that
// actually occur (scores of one query usually share sign and exponent).
template <bool kCached, class Emit>
__device__ void select_and_emit(TopkShared &sh, const uint32_t *keys, const float *s, int n, int k, Emit emit) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // key range
  uint32_t lo_k = 0xffffffffu, hi_k = 0u;
  for (int j = threadIdx.x; j < n; j += kThreads) {
    const uint32_t u = key_at<kCached>(keys, s, j);
    lo_k = min(lo_k, u);
    hi_k = max(hi_k, u);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo_k = min(lo_k, __shfl_xor_sync(0xffffffffu, lo_k, o));
    hi_k = max(hi_k, __shfl_xor_sync(0xffffffffu, hi_k, o));
  }
  if (lane == 0) {
    sh.warp_gt[warp] = lo_k;
    sh.warp_eq[warp] = hi_k;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = sh.warp_gt[lane], b = sh.warp_eq[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
      b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
    }
    if (lane == 0) {
      sh.kmin = a;
      sh.prefix = 0;
      sh.kk = (uint32_t)k;
    }
    if (lane == 1) sh.krange = b - a;
  }
  __syncthreads();
  const uint32_t kmin = sh.kmin, range = sh.krange;
  const int nbits = range == 0 ? 0 : 32 - __clz(range);
  uint32_t mask = 0;  // bits of (key - kmin) fixed so far
  for (int top = nbits; top > 0;) {
    const int width = top >= 11 ? 11 : top;
    const int shift = top - width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = threadIdx.x; i < kBins; i += kThreads) sh.hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = sh.prefix;
    for (int j = threadIdx.x; j < n; j += kThreads) {
      const uint32_t u = key_at<kCached>(keys, s, j) - kmin;
      if ((u & mask) == prefix) atomicAdd(&sh.hist[(u >> shift) & dmask], 1u);
    }
    __syncthreads();
    // Thread t owns bins B-1-2t and B-2-2t (descending), so an exclusive
    // prefix over threads counts the candidates in higher bins.
    const int b_hi = kBins - 1 - 2 * threadIdx.x, b_lo = b_hi - 1;
    const uint32_t c_hi = sh.hist[b_hi], c_lo = sh.hist[b_lo];
    const uint32_t above = sel::block_excl_scan<kWarps>(c_hi + c_lo, sh.scan, lane, warp);
    const uint32_t kk = sh.kk;
    if (above < kk && kk <= above + c_hi + c_lo) {
      const bool in_hi = kk <= above + c_hi;
      const uint32_t bin = in_hi ? b_hi : b_lo;
      sh.kk = kk - (in_hi ? above : above + c_hi);
      sh.prefix = prefix | (bin << shift);
      sh.bcnt = in_hi ? c_hi : c_lo;
      sh.ncand = 0;
    }
    mask |= dmask << shift;
    top = shift;
    __syncthreads();
    if (top > 0 && sh.bcnt <= kFew) {
      // Few keys share the boundary bin: collect them and let one warp find
      // the exact kk-th largest instead of further passes over every key.
      const uint32_t pre = sh.prefix;
      for (int j = threadIdx.x; j < n; j += kThreads) {
        const uint32_t u = key_at<kCached>(keys, s, j) - kmin;
        if ((u & mask) == pre) sh.cand[atomicAdd(&sh.ncand, 1u)] = u;
      }
      __syncthreads();
      if (warp == 0) {
        const int nc = (int)sh.ncand;
        uint32_t t, ngt;
        sel::warp_select(lane < nc ? sh.cand[lane] : 0u, nc, sh.kk, t, ngt);
        if (lane == 0) {
          sh.prefix = t;
          sh.kk -= ngt;
        }
      }
      __syncthreads();
      break;
    }
  }
  const uint32_t tau = sh.prefix + kmin, kk = sh.kk;
  // Ordered compaction: warp w scans the contiguous range [lo, hi).
  const int per_warp = (((n + kWarps - 1) / kWarps) + 31) & ~31;
  const int lo = min(n, warp * per_warp), hi = min(n, lo + per_warp);
  uint32_t g = 0, e = 0;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? key_at<kCached>(keys, s, j) : 0u;
    g += __popc(__ballot_sync(0xffffffffu, j < hi && u > tau));
    e += __popc(__ballot_sync(0xffffffffu, j < hi && u == tau));
  }
  if (lane == 0) {
    sh.warp_gt[warp] = g;
    sh.warp_eq[warp] = e;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scans over the warps: each warp's first output slot
    const uint32_t x0 = sh.warp_gt[lane], y0 = sh.warp_eq[lane];
    uint32_t x = x0, y = y0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t xs = __shfl_up_sync(0xffffffffu, x, o), ys = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) {
        x += xs;
        y += ys;
      }
    }
    sh.warp_gt[lane] = x - x0;
    sh.warp_eq[lane] = y - y0;
  }
  __syncthreads();
  uint32_t G = sh.warp_gt[warp], E = sh.warp_eq[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? key_at<kCached>(keys, s, j) : 0u;
    const bool is_gt = j < hi && u > tau, is_eq = j < hi && u == tau;
    const uint32_t mg = __ballot_sync(0xffffffffu, is_gt), me = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t Gl = G + __popc(mg & lt), El = E + __popc(me & lt);
    if (is_gt) emit(Gl + min(El, kk), j, u);
    else if (is_eq && El < kk) emit(Gl + El, j, u);
    G += __popc(mg);
    E += __popc(me);
  }
}

__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a, int use_cache) {
  extern __shared__ uint32_t keys[];
  __shared__ TopkShared sh;
  pdl_wait();
  pdl_release();
  const int q = blockIdx.x;
  const int n = clamp_count(a.n_cmp[q], a.N_max, threadIdx.x == 0 ? a.status : nullptr);
  const float *s = a.scores + (size_t)q * a.N_max;
  int32_t *out = a.out_idx + (size_t)q * a.k;
  const int k = a.k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  auto emit = [out](uint32_t slot, int j, uint32_t) { out[slot] = j; };
  if (use_cache && n <= kSmemKeys) {
    uint32_t lo = 0xffffffffu, hi = 0u;
    sel::cache_keys<kThreads>(keys, s, n, lo, hi);
    __syncthreads();
    select_and_emit<true>(sh, keys, s, n, k, emit);
  } else {
    select_and_emit<false>(sh, keys, s, n, k, emit);
  }
}

// One query per cluster; CTA c of C selects over the slice
// [c * S, c * S + S) of the list, S = ceil(n / C) rounded up to 32.
__global__ void __launch_bounds__(kThreads) topk_cluster_kernel(TopkArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ alignas(16) uint32_t hist[2 * kBins];
  __shared__ sel::Shared cs;
  pdl_wait();
  pdl_release();
  const uint32_t C = cluster_size(), c = cluster_rank();
  const int q = blockIdx.y;
  const int n = clamp_count(a.n_cmp[q], a.N_max, (threadIdx.x == 0 && c == 0) ? a.status : nullptr);
  const int k = a.k;
  int32_t *out = a.out_idx + (size_t)q * k;
  if (n <= k) {  // the same for every CTA of the cluster: no CTA touches a peer
    if (c == 0)
      for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  const int S = ((n + (int)C - 1) / (int)C + 31) & ~31;
  const int j0 = (int)c * S;
  const int len = max(0, min(S, n - j0));
  uint32_t lo = 0xffffffffu, hi = 0u;
  sel::cache_keys<kThreads>(keys, a.scores + (size_t)q * a.N_max + j0, len, lo, hi);
  sel::cluster_select<kThreads, 4, 8>(cs, hist, keys, len, j0, k, C, c, lo, hi,
                                      [&](uint32_t slot, int j) { out[slot] = j; });
  cluster_wait();  // no peer reads this CTA's shared memory any more
}

// Two-stage selection for long lists. Stage 1: segment g of query q (`seg`
// entries) keeps its own top-k (an entry of the global top-k set is always in
// its segment's top-k set under the same order) as (key, index) candidates,
// ascending. Stage 2: the concatenated candidates of a query are ascending in
// index, so selecting by position with the same tie rule gives the global set.
// Segments start at 4K entries and double until the winners of all segments
// fit the stage-2 shared-memory cache.
bool plan_two_stage(int N_max, int k, int *seg, int *nseg) {
  // While a row's keys fit in shared memory the single-pass kernel reads the
  // scores once and is faster than two launches.
  if (N_max <= kSmemKeys) return false;
  for (int s = 4096; s <= 32768; s *= 2) {
    const int n = (N_max + s - 1) / s;
    if ((long long)n * k <= kSmemKeys / 2 && n <= kThreads && N_max > 2 * s) {
      *seg = s;
      *nseg = n;
      return true;
    }
  }
  return false;
}

__global__ void __launch_bounds__(kThreads) topk_stage1_kernel(TopkArgs a, uint32_t *cand_key, int32_t *cand_idx,
                                                               int32_t *cand_cnt, int nseg, int kSeg) {
  extern __shared__ uint32_t keys[];
  __shared__ TopkShared sh;
  pdl_wait();
  pdl_release();
  const int g = blockIdx.x, q = blockIdx.y;
  const int n = clamp_count(a.n_cmp[q], a.N_max, (threadIdx.x == 0 && g == 0) ? a.status : nullptr);
  const int j0 = g * kSeg;
  const int len = max(0, min(kSeg, n - j0));
  const float *s = a.scores + (size_t)q * a.N_max + j0;
  const size_t cbase = ((size_t)q * nseg + g) * a.k;
  uint32_t *ck = cand_key + cbase;
  int32_t *ci = cand_idx + cbase;
  if (threadIdx.x == 0) cand_cnt[(size_t)q * nseg + g] = min(len, a.k);
  if (len <= a.k) {
    for (int i = threadIdx.x; i < len; i += kThreads) {
      ck[i] = score_key(s[i]);
      ci[i] = j0 + i;
    }
    return;
  }
  uint32_t lo = 0xffffffffu, hi = 0u;
  sel::cache_keys<kThreads>(keys, s, len, lo, hi);
  __syncthreads();
  select_and_emit<true>(sh, keys, s, len, a.k, [ck, ci, j0](uint32_t slot, int j, uint32_t u) {
    ck[slot] = u;
    ci[slot] = j0 + j;
  });
}

__global__ void __launch_bounds__(kThreads) topk_stage2_kernel(TopkArgs a, const uint32_t *cand_key,
                                                               const int32_t *cand_idx, const int32_t *cand_cnt,
                                                               int nseg) {
  extern __shared__ uint32_t keys[];  // [kSmemKeys / 2] keys then [kSmemKeys / 2] indices
  __shared__ TopkShared sh;
  pdl_wait();
  pdl_release();
  __shared__ int offs[kThreads + 1];
  int32_t *idxs = reinterpret_cast<int32_t *>(keys + kSmemKeys / 2);
  const int q = blockIdx.x;
  const int n = clamp_count(a.n_cmp[q], a.N_max, nullptr);
  int32_t *out = a.out_idx + (size_t)q * a.k;
  if (n <= a.k) {
    for (int i = threadIdx.x; i < a.k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  if (threadIdx.x == 0) {
    int o = 0;
    for (int g = 0; g < nseg; ++g) {
      offs[g] = o;
      o += cand_cnt[(size_t)q * nseg + g];
    }
    offs[nseg] = o;
  }
  __syncthreads();
  const int total = offs[nseg];
  for (int g = 0; g < nseg; ++g) {
    const int c = offs[g + 1] - offs[g];
    const size_t cbase = ((size_t)q * nseg + g) * a.k;
    for (int i = threadIdx.x; i < c; i += kThreads) {
      keys[offs[g] + i] = cand_key[cbase + i];
      idxs[offs[g] + i] = cand_idx[cbase + i];
    }
  }
  __syncthreads();
  select_and_emit<true>(sh, keys, nullptr, total, a.k,
                        [out, idxs](uint32_t slot, int j, uint32_t) { out[slot] = idxs[j]; });
}

}  // namespace

// Cluster size for one query's list: about SMs / Q CTAs, at most 8, at
// least 2K entries per CTA, the slice's keys within the shared-memory cache.
int plan_cluster(int Q, int N_max, int k) {
  if (Q < 1 || N_max <= k || N_max < 4096) return 0;
  int C = device_sm_count() / Q;
  C = C > 8 ? 8 : C;
  const int by_len = (N_max + 2047) / 2048;
  C = C > by_len ? by_len : C;
  if (C < 2 || (N_max + C - 1) / C > kSmemKeys - 32 || Q > 65535) return 0;
  return C;
}

size_t topk_scratch_bytes(int Q, int N_max, int k) {
  int seg, nseg;
  if (!plan_two_stage(N_max, k, &seg, &nseg)) return 0;
  return (size_t)Q * nseg * (k * 8 + 4) + 256;
}

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream, void *scratch, size_t scratch_bytes) {
  static DeviceOnce attr;
  once_per_device(attr, [] {
    cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemKeys * 4);
    cudaFuncSetAttribute(topk_stage1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 32768 * 4);
    cudaFuncSetAttribute(topk_stage2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemKeys * 4);
    cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemKeys * 4);
  });
  if (const int C = plan_cluster(a.Q, a.N_max, a.k)) {
    const int S = ((a.N_max + C - 1) / C + 31) & ~31;
    return launch_pdl_cluster(topk_cluster_kernel, dim3(C, a.Q), dim3(kThreads), (size_t)S * 4, stream, (unsigned)C,
                              a);
  }
  int seg = 0, nseg = 0;
  const size_t need = topk_scratch_bytes(a.Q, a.N_max, a.k);
  if (need > 0 && scratch && scratch_bytes >= need && a.Q <= 65535 && plan_two_stage(a.N_max, a.k, &seg, &nseg)) {
    uint32_t *ck = static_cast<uint32_t *>(scratch);
    int32_t *ci = reinterpret_cast<int32_t *>(ck + (size_t)a.Q * nseg * a.k);
    int32_t *cc = ci + (size_t)a.Q * nseg * a.k;
    cudaError_t e = launch_pdl(topk_stage1_kernel, dim3(nseg, a.Q), dim3(kThreads), (size_t)seg * 4, stream, a, ck, ci,
                               cc, nseg, seg);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_stage2_kernel, dim3(a.Q), dim3(kThreads), (size_t)kSmemKeys * 4, stream, a,
                      (const uint32_t *)ck, (const int32_t *)ci, (const int32_t *)cc, nseg);
  }
  const int cache = a.N_max > a.k;  // a query can only need the keys when n > k
  const int keys = a.N_max < kSmemKeys ? a.N_max : kSmemKeys;
  const size_t smem = cache ? (size_t)keys * 4 : 0;
  return launch_pdl(topk_kernel, dim3(a.Q), dim3(kThreads), smem, stream, a, (int)(cache && a.N_max <= kSmemKeys));
}

}  // namespace csa
