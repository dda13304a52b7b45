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
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kSmemKeys = 48 * 1024;

constexpr int kFew = 32;  // a boundary bin this small is finished by one warp

struct TopkShared {
  uint32_t hist[kBins];
  uint32_t scan[kWarps];
  uint32_t warp_gt[kWarps], warp_eq[kWarps];
  uint32_t prefix, kk, kmin, krange, bcnt, ncand;
  uint32_t cand[kFew];
};

// The kk-th largest (1 <= kk <= n) of n <= 32 keys held one per lane (lanes
// >= n hold nothing), and how many of the keys exceed it. Every lane of the
// warp gets both.
__device__ __forceinline__ void warp_select(uint32_t c, int n, uint32_t kk, uint32_t &tau, uint32_t &n_gt) {
  const int lane = threadIdx.x & 31;
  uint32_t gt = 0, ge = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t cj = __shfl_sync(0xffffffffu, c, j);
    if (j < n) {
      gt += cj > c;
      ge += cj >= c;
    }
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, lane < n && gt < kk && kk <= ge);
  const int src = __ffs(hit) - 1;
  tau = __shfl_sync(0xffffffffu, c, src);
  n_gt = __shfl_sync(0xffffffffu, gt, src);
}

// Exclusive prefix sum over the block (thread order) of one value per thread.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *scan, int lane, int warp) {
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scan[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = scan[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    scan[lane] = t;
  }
  __syncthreads();
  const uint32_t r = x - v + (warp > 0 ? scan[warp - 1] : 0u);
  __syncthreads();
  return r;
}

// keys[j] = score_key(s[j]) for j < len, with 8 loads per thread in flight
// (a plain strided loop waits out one load latency per iteration). Returns
// this thread's min and max key in lo / hi.
__device__ __forceinline__ void cache_keys(uint32_t *keys, const float *s, int len, uint32_t &lo, uint32_t &hi) {
  constexpr int U = 8;
  for (int j0 = threadIdx.x; j0 < len; j0 += kThreads * U) {
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * kThreads;
      x[u] = j < len ? s[j] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * kThreads;
      if (j < len) {
        const uint32_t k = score_key(x[u]);
        keys[j] = k;
        lo = min(lo, k);
        hi = max(hi, k);
      }
    }
  }
}

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
    const uint32_t above = block_excl_scan(c_hi + c_lo, sh.scan, lane, warp);
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
        warp_select(lane < nc ? sh.cand[lane] : 0u, nc, sh.kk, t, ngt);
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
  uint32_t G = 0, E = 0;
  for (int w = 0; w < warp; ++w) {
    G += sh.warp_gt[w];
    E += sh.warp_eq[w];
  }
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
    cache_keys(keys, s, n, lo, hi);
    __syncthreads();
    select_and_emit<true>(sh, keys, s, n, k, emit);
  } else {
    select_and_emit<false>(sh, keys, s, n, k, emit);
  }
}

struct ClusterShared {
  alignas(16) uint32_t hist[2][kBins];  // pass p uses hist[p & 1]; peers read it after the pass's cluster barrier
  uint32_t scan[kWarps];
  uint32_t warp_gt[kWarps], warp_eq[kWarps];
  uint32_t lmin, lmax, cnt_gt, cnt_eq;  // this slice's key range and kept counts (read by peers)
  uint32_t prefix, kk, kmin, krange, base_gt, base_eq, bcnt, ncand;
  uint32_t cand[kFew];  // this slice's keys in the boundary bin (when the bin holds <= kFew in all)
};

// One query per cluster; CTA c of C selects over the slice
// [c * S, c * S + S) of the list, S = ceil(n / C) rounded up to 32.
__global__ void __launch_bounds__(kThreads) topk_cluster_kernel(TopkArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ ClusterShared cs;
  pdl_wait();
  pdl_release();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
  const float *s = a.scores + (size_t)q * a.N_max + j0;

  // Keys of the slice into shared memory, with the slice's key range.
  uint32_t lo_k = 0xffffffffu, hi_k = 0u;
  cache_keys(keys, s, len, lo_k, hi_k);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo_k = min(lo_k, __shfl_xor_sync(0xffffffffu, lo_k, o));
    hi_k = max(hi_k, __shfl_xor_sync(0xffffffffu, hi_k, o));
  }
  if (lane == 0) {
    cs.warp_gt[warp] = lo_k;
    cs.warp_eq[warp] = hi_k;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t x = cs.warp_gt[lane], y = cs.warp_eq[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
      y = max(y, __shfl_xor_sync(0xffffffffu, y, o));
    }
    if (lane == 0) {
      cs.lmin = x;
      cs.lmax = y;
    }
  }
  cluster_sync();  // every slice's range is published
  if (warp == 0) {
    uint32_t x = 0xffffffffu, y = 0u;
    if ((uint32_t)lane < C) {
      x = ld_peer(&cs.lmin, lane);
      y = ld_peer(&cs.lmax, lane);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
      y = max(y, __shfl_xor_sync(0xffffffffu, y, o));
    }
    if (lane == 0) {
      cs.kmin = x;
      cs.krange = y - x;
      cs.prefix = 0;
      cs.kk = (uint32_t)k;
    }
  }
  __syncthreads();
  const uint32_t kmin = cs.kmin, range = cs.krange;
  const int nbits = range == 0 ? 0 : 32 - __clz(range);
  uint32_t mask = 0;
  int pass = 0;
  for (int top = nbits; top > 0; ++pass) {
    const int width = top >= 11 ? 11 : top;
    const int shift = top - width;
    const uint32_t dmask = (1u << width) - 1u;
    uint32_t *hist = cs.hist[pass & 1];
    for (int i = threadIdx.x; i < kBins; i += kThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = cs.prefix;
    for (int j = threadIdx.x; j < len; j += kThreads) {
      const uint32_t u = keys[j] - kmin;
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    cluster_sync();  // every slice's histogram of this pass is complete
    // Threads 0..511 sum bins 4t'..4t'+3 (t' = 511 - t, descending order) of
    // every slice with one 16-byte remote load per slice.
    uint32_t cb[4] = {0u, 0u, 0u, 0u};
    if (threadIdx.x < kBins / 4) {
      const int b0 = kBins - 4 - 4 * threadIdx.x;
      uint4 pv[8];
#pragma unroll
      for (uint32_t r = 0; r < 8; ++r)
        if (r < C) pv[r] = ld_peer_u4(&hist[b0], r);
#pragma unroll
      for (uint32_t r = 0; r < 8; ++r)
        if (r < C) {
          cb[0] += pv[r].w;  // bin b0 + 3 (highest first)
          cb[1] += pv[r].z;
          cb[2] += pv[r].y;
          cb[3] += pv[r].x;
        }
    }
    const uint32_t tot = cb[0] + cb[1] + cb[2] + cb[3];
    const uint32_t above = block_excl_scan(tot, cs.scan, lane, warp);
    const uint32_t kk = cs.kk;
    if (threadIdx.x < kBins / 4 && above < kk && kk <= above + tot) {
      uint32_t acc = above, bc = cb[0];
      int i = 0;
#pragma unroll
      for (int q = 0; q < 3; ++q)
        if (i == q && kk > acc + bc) {
          acc += bc;
          i = q + 1;
          bc = cb[q + 1];
        }
      const uint32_t bin = (uint32_t)(kBins - 1 - 4 * threadIdx.x - i);
      cs.kk = kk - acc;
      cs.prefix = prefix | (bin << shift);
      cs.bcnt = bc;
      cs.ncand = 0;
    }
    mask |= dmask << shift;
    top = shift;
    __syncthreads();
    if (top > 0 && cs.bcnt <= kFew) {
      // Few keys share the boundary bin across the cluster: every slice
      // publishes its share, every CTA gathers all of them and one warp finds
      // the exact kk-th largest (the same in every CTA).
      const uint32_t pre = cs.prefix;
      for (int j = threadIdx.x; j < len; j += kThreads) {
        const uint32_t u = keys[j] - kmin;
        if ((u & mask) == pre) cs.cand[atomicAdd(&cs.ncand, 1u)] = u;
      }
      cluster_sync();  // every slice's candidates are published
      if (warp == 0) {
        const uint32_t cnt = (uint32_t)lane < C ? ld_peer(&cs.ncand, lane) : 0u;
        uint32_t inc = cnt;  // inclusive scan of the slices' counts
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += y;
        }
        const uint32_t excl = inc - cnt;
        const int nc = (int)__shfl_sync(0xffffffffu, inc, 31);
        // candidate number `lane` belongs to the last slice starting at or before it
        uint32_t owner = 0, base = 0;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const uint32_t e_r = __shfl_sync(0xffffffffu, excl, r), c_r = __shfl_sync(0xffffffffu, cnt, r);
          if ((uint32_t)r < C && c_r > 0 && e_r <= (uint32_t)lane) {
            owner = (uint32_t)r;
            base = e_r;
          }
        }
        const uint32_t c = lane < nc ? ld_peer(&cs.cand[lane - base], owner) : 0u;
        uint32_t t, ngt;
        warp_select(c, nc, cs.kk, t, ngt);
        if (lane == 0) {
          cs.prefix = t;
          cs.kk -= ngt;
        }
      }
      __syncthreads();
      break;
    }
  }
  const uint32_t tau = cs.prefix + kmin, kk = cs.kk;

  // Ordered compaction: count, exchange the slice totals, then emit.
  const int per_warp = (((len + kWarps - 1) / kWarps) + 31) & ~31;
  const int lo = min(len, warp * per_warp), hi = min(len, lo + per_warp);
  uint32_t g = 0, e = 0;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? keys[j] : 0u;
    g += __popc(__ballot_sync(0xffffffffu, j < hi && u > tau));
    e += __popc(__ballot_sync(0xffffffffu, j < hi && u == tau));
  }
  if (lane == 0) {
    cs.warp_gt[warp] = g;
    cs.warp_eq[warp] = e;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t x = cs.warp_gt[lane], y = cs.warp_eq[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      x += __shfl_xor_sync(0xffffffffu, x, o);
      y += __shfl_xor_sync(0xffffffffu, y, o);
    }
    if (lane == 0) {
      cs.cnt_gt = x;
      cs.cnt_eq = y;
    }
  }
  cluster_sync();  // every slice's counts are published
  if (warp == 0) {
    uint32_t x = 0, y = 0;
    if ((uint32_t)lane < c) {
      x = ld_peer(&cs.cnt_gt, lane);
      y = ld_peer(&cs.cnt_eq, lane);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      x += __shfl_xor_sync(0xffffffffu, x, o);
      y += __shfl_xor_sync(0xffffffffu, y, o);
    }
    if (lane == 0) {
      cs.base_gt = x;
      cs.base_eq = y;
    }
  }
  cluster_arrive();  // this CTA reads no peer after this point
  __syncthreads();
  uint32_t G = cs.base_gt, E = cs.base_eq;
  for (int w = 0; w < warp; ++w) {
    G += cs.warp_gt[w];
    E += cs.warp_eq[w];
  }
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? keys[j] : 0u;
    const bool is_gt = j < hi && u > tau, is_eq = j < hi && u == tau;
    const uint32_t mg = __ballot_sync(0xffffffffu, is_gt), me = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t Gl = G + __popc(mg & lt), El = E + __popc(me & lt);
    if (is_gt) out[Gl + min(El, kk)] = j0 + j;
    else if (is_eq && El < kk) out[Gl + El] = j0 + j;
    G += __popc(mg);
    E += __popc(me);
  }
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
  cache_keys(keys, s, len, lo, hi);
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
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int C = sms / Q;
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
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemKeys * 4);
    cudaFuncSetAttribute(topk_stage1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 32768 * 4);
    cudaFuncSetAttribute(topk_stage2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemKeys * 4);
    cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemKeys * 4);
    attr_set = true;
  }
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
