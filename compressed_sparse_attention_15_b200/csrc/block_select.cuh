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

// Select the k largest of the n keys keys[0 .. n-1] (shared memory; n > k >=
// 1) and call emit(slot, position) for each, slots 0 .. k-1 in ascending
// position. Threads 0 .. NT-1 of the block take part and synchronise on
// named barrier `bar`; hist: NH x kBins words of shared memory, NH private
// histogram copies (warp w counts into copy w % NH). Every pass over the keys
// keeps U independent loads in flight per thread: the passes are bound by
// shared-memory latency, not throughput, at this block size.
template <int NT, int NH, class Emit>
__device__ void select(Shared &sh, uint32_t *hist, const uint32_t *keys, int n, int k, int bar, Emit emit) {
  constexpr int NW = NT / 32;
  constexpr int U = 4;
  constexpr int BPT = (kBins + NT - 1) / NT;  // bins per thread in the scan
  static_assert(NT % 32 == 0 && NW <= 32, "block shape");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // key range (the first histogram is zeroed meanwhile)
  for (int i = threadIdx.x; i < NH * kBins; i += NT) hist[i] = 0;
  uint32_t lo_k = 0xffffffffu, hi_k = 0u;
  for (int j0 = threadIdx.x; j0 < n; j0 += U * NT) {
    uint32_t u[U];
#pragma unroll
    for (int i = 0; i < U; ++i) u[i] = j0 + i * NT < n ? keys[j0 + i * NT] : keys[j0];
#pragma unroll
    for (int i = 0; i < U; ++i) {
      lo_k = min(lo_k, u[i]);
      hi_k = max(hi_k, u[i]);
    }
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
  uint32_t kmin, range;
  {  // every warp reduces the warp results itself (no second barrier)
    uint32_t a = lane < NW ? sh.warp_gt[lane] : 0xffffffffu, b = lane < NW ? sh.warp_eq[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
      b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
    }
    kmin = a;
    range = b - a;
  }
  const int nbits = range == 0 ? 0 : 32 - __clz(range);
  uint32_t mask = 0, prefix = 0, kk = (uint32_t)k;
  uint32_t *my_hist = hist + (warp % NH) * kBins;
  for (int top = nbits; top > 0;) {
    const int width = top >= 11 ? 11 : top;
    const int shift = top - width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int j0 = threadIdx.x; j0 < n; j0 += U * NT) {
      uint32_t u[U];
#pragma unroll
      for (int i = 0; i < U; ++i) u[i] = j0 + i * NT < n ? keys[j0 + i * NT] - kmin : ~0u;
#pragma unroll
      for (int i = 0; i < U; ++i)
        if (j0 + i * NT < n && (u[i] & mask) == prefix) atomicAdd(&my_hist[(u[i] >> shift) & dmask], 1u);
    }
    nbar<NT>(bar);
    // Thread t owns bins kBins-1-BPT t .. kBins-BPT(t+1) (descending), so an
    // exclusive scan over threads counts the keys in higher bins.
    uint32_t cb[BPT];
    uint32_t tot = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int b = kBins - 1 - BPT * threadIdx.x - i;
      uint32_t c = 0;
      if (b >= 0) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          c += hist[r * kBins + b];
          hist[r * kBins + b] = 0;  // zeroed for the next pass (read by this thread only)
        }
      }
      cb[i] = c;
      tot += c;
    }
    const uint32_t above = excl_scan<NT>(tot, sh.scan, lane, warp, bar);
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
    prefix = sh.prefix;
    kk = sh.kk;
    if (top > 0 && sh.bcnt <= kFew) {
      // Few keys share the boundary bin: collect them and let one warp find
      // the exact kk-th largest instead of further passes over every key.
      for (int j0 = threadIdx.x; j0 < n; j0 += U * NT) {
        uint32_t u[U];
#pragma unroll
        for (int i = 0; i < U; ++i) u[i] = j0 + i * NT < n ? keys[j0 + i * NT] - kmin : ~0u;
#pragma unroll
        for (int i = 0; i < U; ++i)
          if (j0 + i * NT < n && (u[i] & mask) == prefix) sh.cand[atomicAdd(&sh.ncand, 1u)] = u[i];
      }
      nbar<NT>(bar);
      if (warp == 0) {
        const int nc = (int)sh.ncand;
        uint32_t t, ngt;
        sel::warp_select(lane < nc ? sh.cand[lane] : 0u, nc, kk, t, ngt);
        if (lane == 0) {
          sh.prefix = t;
          sh.kk = kk - ngt;
        }
      }
      nbar<NT>(bar);
      prefix = sh.prefix;
      kk = sh.kk;
      break;
    }
  }
  const uint32_t tau = prefix + kmin;
  // Ordered compaction: warp w scans the contiguous range [lo, hi), U groups
  // of 32 keys per round.
  const int per_warp = (((n + NW - 1) / NW) + 32 * U - 1) & ~(32 * U - 1);
  const int lo = min(n, warp * per_warp), hi = min(n, lo + per_warp);
  uint32_t g = 0, e = 0;
  for (int base = lo; base < hi; base += 32 * U) {
    uint32_t u[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int j = base + 32 * i + lane;
      u[i] = j < hi ? keys[j] : 0u;
    }
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const bool in = base + 32 * i + lane < hi;
      g += __popc(__ballot_sync(0xffffffffu, in && u[i] > tau));
      e += __popc(__ballot_sync(0xffffffffu, in && u[i] == tau));
    }
  }
  if (lane == 0) {
    sh.warp_gt[warp] = g;
    sh.warp_eq[warp] = e;
  }
  nbar<NT>(bar);
  uint32_t G, E;
  {  // each warp's first output slot: exclusive scans over the warps (every warp for itself)
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
    G = __shfl_sync(0xffffffffu, x - x0, warp);
    E = __shfl_sync(0xffffffffu, y - y0, warp);
  }
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32 * U) {
    uint32_t u[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int j = base + 32 * i + lane;
      u[i] = j < hi ? keys[j] : 0u;
    }
#pragma unroll
    for (int i = 0; i < U; ++i) {
      const int j = base + 32 * i + lane;
      const bool is_gt = j < hi && u[i] > tau, is_eq = j < hi && u[i] == tau;
      const uint32_t mg = __ballot_sync(0xffffffffu, is_gt), me = __ballot_sync(0xffffffffu, is_eq);
      const uint32_t Gl = G + __popc(mg & lt), El = E + __popc(me & lt);
      if (is_gt) emit(Gl + min(El, kk), j);
      else if (is_eq && El < kk) emit(Gl + El, j);
      G += __popc(mg);
      E += __popc(me);
    }
  }
  nbar<NT>(bar);  // the shared state may be reused at once
}

}  // namespace bsel
}  // namespace csa
