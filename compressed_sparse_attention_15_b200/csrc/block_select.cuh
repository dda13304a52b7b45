// Exact top-k of one list by one thread block of any size (A3), used by the
// fused decode-step kernel.
//
// Selection rule ("DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1:
// the indexer "selects top-k compressed positions"): the k entries of largest
// score, ties resolved towards the smaller position, emitted in ascending
// position order. Scores arrive as order-preserving 32-bit keys (score_key).
//
// Method: radix select over (key - min key) with 11-bit digits from the
// highest set bit of the key range down; each pass histograms the keys that
// share the prefix fixed so far, and an exclusive scan over the bins (highest
// first) finds the bin holding the kk-th largest key. Once that bin holds at
// most 32 keys one warp finishes the selection. A final ordered pass keeps
// every key above the threshold and the first kk keys equal to it (by
// position), each warp scanning a contiguous range, so the output slots are
// ascending in position and deterministic.
#pragma once

#include "cluster_select.cuh"
#include "common.cuh"

namespace csa {
namespace bsel {

constexpr int kBins = sel::kBins;  // 2048
constexpr int kFew = sel::kFew;    // 32

// Named barrier over the NT participating threads (threads 0 .. NT-1 of the
// block; other warps of the block may be busy elsewhere).
template <int NT>
__device__ __forceinline__ void nbar(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(NT) : "memory");
}

struct Shared {
  uint32_t scan[32];
  uint32_t warp_gt[32], warp_eq[32];
  uint32_t prefix, kk, kmin, krange, bcnt, ncand;
  uint32_t cand[kFew];
};

// Exclusive prefix sum over threads 0 .. NT-1 (thread order) of one value per
// thread, synchronising on named barrier `bar`.
template <int NT>
__device__ __forceinline__ uint32_t excl_scan(uint32_t v, uint32_t *scan, int lane, int warp, int bar) {
  constexpr int NW = NT / 32;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scan[warp] = x;
  nbar<NT>(bar);
  if (warp == 0) {
    uint32_t t = lane < NW ? scan[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < NW) scan[lane] = t;
  }
  nbar<NT>(bar);
  const uint32_t r = x - v + (warp > 0 ? scan[warp - 1] : 0u);
  nbar<NT>(bar);
  return r;
}

// Select the k largest of the n keys key_at(0 .. n-1) (n > k >= 1) and call
// emit(slot, position) for each, slots 0 .. k-1 in ascending position.
// Threads 0 .. NT-1 of the block take part and synchronise on named barrier
// `bar`; hist: NH x kBins words of shared memory, NH private histogram copies
// (warp w counts into copy w % NH: fewer threads contend for one counter).
template <int NT, int NH, class KeyAt, class Emit>
__device__ void select(Shared &sh, uint32_t *hist, int n, int k, int bar, KeyAt key_at, Emit emit) {
  constexpr int NW = NT / 32;
  constexpr int BPT = (kBins + NT - 1) / NT;  // bins per thread in the scan
  static_assert(NT % 32 == 0 && NW <= 32, "block shape");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // key range
  uint32_t lo_k = 0xffffffffu, hi_k = 0u;
  for (int j = threadIdx.x; j < n; j += NT) {
    const uint32_t u = key_at(j);
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
  nbar<NT>(bar);
  if (warp == 0) {
    uint32_t a = lane < NW ? sh.warp_gt[lane] : 0xffffffffu, b = lane < NW ? sh.warp_eq[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
      b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
    }
    if (lane == 0) {
      sh.kmin = a;
      sh.krange = b - a;
      sh.prefix = 0;
      sh.kk = (uint32_t)k;
    }
  }
  nbar<NT>(bar);
  const uint32_t kmin = sh.kmin, range = sh.krange;
  const int nbits = range == 0 ? 0 : 32 - __clz(range);
  uint32_t mask = 0;  // bits of (key - kmin) fixed so far
  for (int top = nbits; top > 0;) {
    const int width = top >= 11 ? 11 : top;
    const int shift = top - width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = threadIdx.x; i < NH * kBins; i += NT) hist[i] = 0;
    nbar<NT>(bar);
    const uint32_t prefix = sh.prefix;
    uint32_t *my_hist = hist + (warp % NH) * kBins;
    for (int j = threadIdx.x; j < n; j += NT) {
      const uint32_t u = key_at(j) - kmin;
      if ((u & mask) == prefix) atomicAdd(&my_hist[(u >> shift) & dmask], 1u);
    }
    nbar<NT>(bar);
    // Thread t owns bins kBins-1-BPT t .. kBins-BPT(t+1) (descending), so an
    // exclusive scan over threads counts the keys in higher bins.
    uint32_t cb[BPT];
    uint32_t tot = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int bin = kBins - 1 - BPT * threadIdx.x - i;
      uint32_t c = 0;
      if (bin >= 0) {
#pragma unroll
        for (int r = 0; r < NH; ++r) c += hist[r * kBins + bin];
      }
      cb[i] = c;
      tot += c;
    }
    const uint32_t above = excl_scan<NT>(tot, sh.scan, lane, warp, bar);
    const uint32_t kk = sh.kk;
    if (above < kk && kk <= above + tot) {
      uint32_t acc = above;
      int i = 0;
#pragma unroll
      for (int q = 0; q < BPT - 1; ++q)
        if (i == q && kk > acc + cb[q]) {
          acc += cb[q];
          i = q + 1;
        }
      uint32_t bc = cb[0];
#pragma unroll
      for (int q = 1; q < BPT; ++q)
        if (i == q) bc = cb[q];
      const uint32_t bin = (uint32_t)(kBins - 1 - BPT * threadIdx.x - i);
      sh.kk = kk - acc;
      sh.prefix = prefix | (bin << shift);
      sh.bcnt = bc;
      sh.ncand = 0;
    }
    mask |= dmask << shift;
    top = shift;
    nbar<NT>(bar);
    if (top > 0 && sh.bcnt <= kFew) {
      // Few keys share the boundary bin: collect them and let one warp find
      // the exact kk-th largest instead of further passes over every key.
      const uint32_t pre = sh.prefix;
      for (int j = threadIdx.x; j < n; j += NT) {
        const uint32_t u = key_at(j) - kmin;
        if ((u & mask) == pre) sh.cand[atomicAdd(&sh.ncand, 1u)] = u;
      }
      nbar<NT>(bar);
      if (warp == 0) {
        const int nc = (int)sh.ncand;
        uint32_t t, ngt;
        sel::warp_select(lane < nc ? sh.cand[lane] : 0u, nc, sh.kk, t, ngt);
        if (lane == 0) {
          sh.prefix = t;
          sh.kk -= ngt;
        }
      }
      nbar<NT>(bar);
      break;
    }
  }
  const uint32_t tau = sh.prefix + kmin, kk = sh.kk;
  // Ordered compaction: warp w scans the contiguous range [lo, hi).
  const int per_warp = (((n + NW - 1) / NW) + 31) & ~31;
  const int lo = min(n, warp * per_warp), hi = min(n, lo + per_warp);
  uint32_t g = 0, e = 0;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? key_at(j) : 0u;
    g += __popc(__ballot_sync(0xffffffffu, j < hi && u > tau));
    e += __popc(__ballot_sync(0xffffffffu, j < hi && u == tau));
  }
  if (lane == 0) {
    sh.warp_gt[warp] = g;
    sh.warp_eq[warp] = e;
  }
  nbar<NT>(bar);
  if (warp == 0) {  // exclusive scans over the warps: each warp's first output slot
    const uint32_t x0 = lane < NW ? sh.warp_gt[lane] : 0u, y0 = lane < NW ? sh.warp_eq[lane] : 0u;
    uint32_t x = x0, y = y0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t xs = __shfl_up_sync(0xffffffffu, x, o), ys = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) {
        x += xs;
        y += ys;
      }
    }
    if (lane < NW) {
      sh.warp_gt[lane] = x - x0;
      sh.warp_eq[lane] = y - y0;
    }
  }
  nbar<NT>(bar);
  uint32_t G = sh.warp_gt[warp], E = sh.warp_eq[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < hi ? key_at(j) : 0u;
    const bool is_gt = j < hi && u > tau, is_eq = j < hi && u == tau;
    const uint32_t mg = __ballot_sync(0xffffffffu, is_gt), me = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t Gl = G + __popc(mg & lt), El = E + __popc(me & lt);
    if (is_gt) emit(Gl + min(El, kk), j);
    else if (is_eq && El < kk) emit(Gl + El, j);
    G += __popc(mg);
    E += __popc(me);
  }
  nbar<NT>(bar);  // the shared state may be reused at once
}

}  // namespace bsel
}  // namespace csa
