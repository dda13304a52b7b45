// Exact top-k of one query's list by a thread-block cluster (A3), shared by
// the top-k kernel and the MQA kernel that selects its own rows.
//
// Selection rule ("DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1:
// the indexer "selects top-k compressed positions"): the k entries of largest
// score, ties resolved towards the smaller index, emitted in ascending index
// order. Scores arrive as order-preserving 32-bit keys.
//
// CTA c of a cluster of C holds the contiguous slice [j0, j0 + len) of the
// list in shared memory. Radix select over the cluster's key range with
// 11-bit digits: every pass builds the slice's histogram, the slices'
// histograms are summed through distributed shared memory, and every CTA
// finds the same boundary bin. Once the boundary bin holds at most 32 keys
// over the cluster, they are gathered and one warp finishes the selection.
// The keys above the threshold, and the first kk keys equal to it, are then
// emitted at slots given by ascending index across the cluster (each slice's
// counts are exchanged once).
#pragma once

#include "common.cuh"

namespace csa {
namespace sel {

constexpr int kBins = 2048;
constexpr int kFew = 32;  // a boundary bin this small is finished by one warp

struct Shared {
  uint32_t scan[32];
  uint32_t warp_gt[32], warp_eq[32];
  uint32_t lmin, lmax, cnt_gt, cnt_eq;  // this slice's key range and kept counts (read by peers)
  uint32_t prefix, kk, kmin, krange, base_gt, base_eq, bcnt, ncand;
  uint32_t cand[kFew];  // this slice's keys in the boundary bin (read by peers)
};

// Exclusive prefix sum over the block (thread order) of one value per thread;
// NW warps.
template <int NW>
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
    uint32_t t = lane < NW ? scan[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < NW) scan[lane] = t;
  }
  __syncthreads();
  const uint32_t r = x - v + (warp > 0 ? scan[warp - 1] : 0u);
  __syncthreads();
  return r;
}

// The kk-th largest (1 <= kk <= n) of n <= 32 keys held one per lane, and how
// many of them exceed it; every lane of the warp gets both.
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

// keys[j] = score_key(s[j]) for j < len, NT threads with 8 loads each in
// flight (a plain strided loop waits out one load latency per iteration).
// Folds this thread's keys into lo / hi.
template <int NT>
__device__ __forceinline__ void cache_keys(uint32_t *keys, const float *s, int len, uint32_t &lo, uint32_t &hi) {
  constexpr int U = 8;
  for (int j0 = threadIdx.x; j0 < len; j0 += NT * U) {
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * NT;
      x[u] = j < len ? s[j] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * NT;
      if (j < len) {
        const uint32_t k = score_key(x[u]);
        keys[j] = k;
        lo = min(lo, k);
        hi = max(hi, k);
      }
    }
  }
}

// Select the k largest of the cluster's keys (n > k in all) and call
// emit(slot, j0 + j) for this slice's kept entries. NT threads per CTA, all
// taking part, each passing the min / max (lo_k / hi_k) of the keys it
// cached; BPT histogram bins per thread in the merge (kBins / BPT <= NT); at
// most MAXC CTAs per cluster. hist2: 2 x kBins words, 16-byte aligned. On
// return this CTA has arrived on the cluster barrier after its last access
// to a peer (emit may store to peers before that); the caller waits on it
// before it reuses keys, hist2 or cs, or exits.
template <int NT, int BPT, int MAXC, class Emit>
__device__ void cluster_select(Shared &cs, uint32_t *hist2, const uint32_t *keys, int len, int j0, int k, uint32_t C,
                               uint32_t c, uint32_t lo_k, uint32_t hi_k, Emit emit) {
  constexpr int NW = NT / 32;
  constexpr int kActive = kBins / BPT;
  static_assert(kActive <= NT && BPT % 4 == 0 && NW <= 32 && MAXC <= 32, "launch shape");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the slice's key range, then the cluster's
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
    uint32_t x = lane < NW ? cs.warp_gt[lane] : 0xffffffffu, y = lane < NW ? cs.warp_eq[lane] : 0u;
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
    uint32_t *hist = hist2 + (pass & 1) * kBins;  // peers read it after this pass's cluster barrier
    for (int i = threadIdx.x; i < kBins; i += NT) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = cs.prefix;
    for (int j = threadIdx.x; j < len; j += NT) {
      const uint32_t u = keys[j] - kmin;
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    cluster_sync();  // every slice's histogram of this pass is complete
    // Thread t < kActive sums bins [kBins - BPT (t + 1), kBins - BPT t) of
    // every slice (16-byte remote loads), highest bin first.
    uint32_t cb[BPT];
#pragma unroll
    for (int i = 0; i < BPT; ++i) cb[i] = 0u;
    if (threadIdx.x < kActive) {
      const int b0 = kBins - BPT * (threadIdx.x + 1);
#pragma unroll
      for (int v = 0; v < BPT / 4; ++v) {
        uint4 pv[MAXC];
#pragma unroll
        for (uint32_t r = 0; r < MAXC; ++r)
          if (r < C) pv[r] = ld_peer_u4(&hist[b0 + 4 * v], r);
#pragma unroll
        for (uint32_t r = 0; r < MAXC; ++r)
          if (r < C) {  // cb[i]: bin b0 + BPT - 1 - i
            cb[BPT - 1 - 4 * v] += pv[r].x;
            cb[BPT - 2 - 4 * v] += pv[r].y;
            cb[BPT - 3 - 4 * v] += pv[r].z;
            cb[BPT - 4 - 4 * v] += pv[r].w;
          }
      }
    }
    uint32_t tot = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) tot += cb[i];
    const uint32_t above = block_excl_scan<NW>(tot, cs.scan, lane, warp);
    const uint32_t kk = cs.kk;
    if (threadIdx.x < kActive && above < kk && kk <= above + tot) {
      uint32_t acc = above, bc = cb[0];
      int i = 0;
#pragma unroll
      for (int q = 0; q < BPT - 1; ++q)
        if (i == q && kk > acc + bc) {
          acc += bc;
          i = q + 1;
          bc = cb[q + 1];
        }
      const uint32_t bin = (uint32_t)(kBins - 1 - BPT * threadIdx.x - i);
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
      for (int j = threadIdx.x; j < len; j += NT) {
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
        for (int r = 0; r < MAXC; ++r) {
          const uint32_t e_r = __shfl_sync(0xffffffffu, excl, r), c_r = __shfl_sync(0xffffffffu, cnt, r);
          if ((uint32_t)r < C && c_r > 0 && e_r <= (uint32_t)lane) {
            owner = (uint32_t)r;
            base = e_r;
          }
        }
        const uint32_t cv = lane < nc ? ld_peer(&cs.cand[lane - base], owner) : 0u;
        uint32_t t, ngt;
        warp_select(cv, nc, cs.kk, t, ngt);
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
  const int per_warp = (((len + NW - 1) / NW) + 31) & ~31;
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
  if (warp == 0) {  // each warp's offset within the slice, and the slice's totals
    const uint32_t x0 = lane < NW ? cs.warp_gt[lane] : 0u, y0 = lane < NW ? cs.warp_eq[lane] : 0u;
    uint32_t x = x0, y = y0;  // inclusive scans over the warps
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t xs = __shfl_up_sync(0xffffffffu, x, o), ys = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) {
        x += xs;
        y += ys;
      }
    }
    if (lane < NW) {
      cs.warp_gt[lane] = x - x0;
      cs.warp_eq[lane] = y - y0;
    }
    if (lane == 31) {
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
  __syncthreads();
  uint32_t G = cs.base_gt + cs.warp_gt[warp], E = cs.base_eq + cs.warp_eq[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? keys[j] : 0u;
    const bool is_gt = j < hi && u > tau, is_eq = j < hi && u == tau;
    const uint32_t mg = __ballot_sync(0xffffffffu, is_gt), me = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t Gl = G + __popc(mg & lt), El = E + __popc(me & lt);
    if (is_gt) emit(Gl + min(El, kk), j0 + j);
    else if (is_eq && El < kk) emit(Gl + El, j0 + j);
    G += __popc(mg);
    E += __popc(me);
  }
  cluster_arrive();  // this CTA's remote loads and stores are done
}

}  // namespace sel
}  // namespace csa
