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
// Launch shapes. Lists of up to 16K entries: one 1024-thread CTA per query
// holding every key in registers (topk_block_kernel, few block barriers).
// Longer lists with few queries (a decode batch): the list of one query is cut
// into C contiguous slices, one CTA of a thread-block cluster each (C <= 8,
// about SMs / Q). Slices of up to 40K keys first try the sample-and-filter
// scheme over the cluster (four cluster barriers: key range, summed sample
// histograms, candidate counts, candidates gathered into CTA 0, which selects
// among them); otherwise the slices' histograms are summed through distributed
// shared memory at every radix pass, and each CTA emits its own slice at the
// offset given by the counts of the slices before it. Many queries with
// lists of up to 40K entries: one 1024-thread CTA per query, keys cached in
// shared memory, the same sample-and-filter scheme (topk_filter_kernel); up
// to 48K entries: the exact passes over the cached keys. Longer lists with many queries take two stages: the exact
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

// ---------------------------------------------------------------- one CTA
// One 1024-thread CTA per query with every key in registers: warp w holds the
// 32 R positions [32 R w, 32 R (w + 1)), lane l those of them congruent to l
// mod 32 (n <= 1024 R; coalesced loads). Selection on one SM is bound by
// instruction issue, so most keys are dropped early: a sample of the keys
// (one per thread) gives a lower threshold with enough keys above it (the
// sample's rank is the expected count plus four standard deviations), those
// keys go to shared memory in position order, and the exact radix select
// runs over them only. When the candidates are too few or too many for the
// buffer, the radix select runs over all keys instead. Either way the
// selection is exact.

struct BlockShared {
  uint32_t hist[2][kBins];
  uint32_t wtot[2][kWarps];
  uint32_t wmin[kWarps], wmax[kWarps];
  uint32_t wg[kWarps], we[kWarps];
  uint32_t dec[2][3];  // per pass parity: boundary bin, keys above it, keys in it
  uint32_t cand[kFew];
  uint32_t ncand;
  uint32_t sel_t, sel_ngt;  // the few-candidates finish, computed by warp 0
};
constexpr int kCandCap = 4096;  // candidate buffer (dynamic shared memory: keys, then positions)
constexpr int kFilterKeys = 40 * 1024;  // longest list of topk_filter_kernel (keys + candidates in shared memory)

// Exclusive prefix over the warps of a per-warp value (every lane passes its
// warp's value). One barrier; every thread gets its warp's offset and the
// total.
__device__ __forceinline__ void warp_offsets(uint32_t *slot, uint32_t v, int lane, int warp, uint32_t &off,
                                             uint32_t &total) {
  if (lane == 0) slot[warp] = v;
  __syncthreads();
  uint32_t inc = slot[lane];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  const uint32_t p = __shfl_sync(0xffffffffu, inc, warp > 0 ? warp - 1 : 0);
  off = warp > 0 ? p : 0u;
  total = __shfl_sync(0xffffffffu, inc, 31);
}

// One radix pass's histogram scan: the bins of `h` hold the matching keys;
// finds the bin where the count from the top reaches `want` (computed by
// want_of(total) once the total is known) and returns (bin, keys above it,
// keys in it), `want` and `total` in every thread; the bin is meaningful
// only for 1 <= want <= total. Three barriers (the caller's histogram is
// complete at the first).
template <class WantOf>
__device__ __forceinline__ void boundary_bin(BlockShared &sh, const uint32_t *h, int pass, int lane, int warp,
                                             WantOf want_of, uint32_t &bin, uint32_t &above_out, uint32_t &cb,
                                             uint32_t &want, uint32_t &total) {
  __syncthreads();
  // warp w scans bins [kBins - 64 (w + 1), kBins - 64 w) from the top: lane
  // l holds bins hb = kBins - 1 - 64 w - 2 l and hb - 1
  const int hb = kBins - 1 - 64 * warp - 2 * lane;
  const uint32_t c_hi = h[hb], c_lo = h[hb - 1], c = c_hi + c_lo;
  uint32_t inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) sh.wtot[pass & 1][warp] = inc;
  __syncthreads();
  uint32_t winc = sh.wtot[pass & 1][lane];  // every warp combines the 32 warp totals itself
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, winc, o);
    if (lane >= o) winc += y;
  }
  total = __shfl_sync(0xffffffffu, winc, 31);
  want = want_of(total);
  const uint32_t w_above = __shfl_sync(0xffffffffu, winc, warp > 0 ? warp - 1 : 0);
  const uint32_t above = (warp > 0 ? w_above : 0u) + inc - c;  // matching keys in the bins above this lane's two
  if (above < want && want <= above + c) {  // exactly one lane of the block (when 1 <= want <= total)
    const bool in_hi = want <= above + c_hi;
    uint32_t *d = sh.dec[pass & 1];
    d[0] = in_hi ? (uint32_t)hb : (uint32_t)(hb - 1);
    d[1] = in_hi ? above : above + c_hi;
    d[2] = in_hi ? c_hi : c_lo;
  }
  __syncthreads();
  bin = sh.dec[pass & 1][0];
  above_out = sh.dec[pass & 1][1];
  cb = sh.dec[pass & 1][2];
}

// Exact radix select over the keys kv[r] (r < nv) of every thread, in units u
// = kv - base, `range` the largest u: returns in every thread the threshold
// tau_u and kk, the number of keys equal to it that are kept (the other k -
// kk kept keys exceed it). Both histograms are clear on entry and sh.ncand is
// 0; MSD digits of 11 bits from the top set bit of the range.
template <int RR>
__device__ __forceinline__ void radix_select(BlockShared &sh, const uint32_t (&kv)[RR], int nv, uint32_t base,
                                             uint32_t range, uint32_t k, int lane, int warp, uint32_t &tau_u,
                                             uint32_t &kk_out) {
  uint32_t prefix = 0u, mask = 0u, kk = k;
  tau_u = 0u;  // range 0: every key equals base
  int top = range == 0u ? 0 : 32 - __clz(range);
  for (int pass = 0; top > 0; ++pass) {
    const int width = top >= 11 ? 11 : top;
    const int shift = top - width;
    const uint32_t dmask = (1u << width) - 1u;
    uint32_t *h = sh.hist[pass & 1];
#pragma unroll
    for (int r = 0; r < RR; ++r) {
      const uint32_t u = kv[r] - base;
      if (r < nv && (u & mask) == prefix) atomicAdd(&h[(u >> shift) & dmask], 1u);
    }
    uint32_t bin, above, cb, want, total;
    boundary_bin(sh, h, pass, lane, warp, [kk](uint32_t) { return kk; }, bin, above, cb, want, total);
    kk -= above;
    prefix |= bin << shift;
    mask |= dmask << shift;
    top = shift;
    // no thread reads this histogram any more: cleared for pass + 2
    for (int i = threadIdx.x; i < kBins; i += kThreads) h[i] = 0u;
    if (top == 0) {  // every bit fixed: the prefix is the threshold
      tau_u = prefix;
      break;
    }
    if (kk == cb && prefix != 0u) {  // every key of the boundary bin is kept: u >= prefix
      tau_u = prefix - 1u;
      kk = 0u;
      break;
    }
    if (cb <= (uint32_t)kFew) {
      // Few keys in the boundary bin: gather them; warp 0 finds the kk-th
      // largest among them.
#pragma unroll
      for (int r = 0; r < RR; ++r) {
        const uint32_t u = kv[r] - base;
        if (r < nv && (u & mask) == prefix) sh.cand[atomicAdd(&sh.ncand, 1u)] = u;
      }
      __syncthreads();
      if (warp == 0) {
        const int nc = (int)sh.ncand;
        uint32_t t, ngt;
        sel::warp_select(lane < nc ? sh.cand[lane] : 0u, nc, kk, t, ngt);
        if (lane == 0) {
          sh.sel_t = t;
          sh.sel_ngt = ngt;
        }
      }
      __syncthreads();
      tau_u = sh.sel_t;
      kk -= sh.sel_ngt;
      break;
    }
  }
  kk_out = kk;
}

// The exact top k of C candidates (k <= C <= kCandCap) gathered in shared
// memory in position order: cbuf[i] the key in units above the floor (the
// largest unit is urange), cbuf[kCandCap + i] the position. Writes the k
// positions to out in ascending order (ties: the first positions). Every
// thread of the block takes part; both histograms are clear and sh.ncand is 0.
__device__ __forceinline__ void select_candidates(BlockShared &sh, const uint32_t *cbuf, int C, uint32_t urange,
                                                  uint32_t k, int32_t *out, int lane, int warp) {
  // thread t: candidates 4t .. 4t + 3
  const int c0 = 4 * (int)threadIdx.x;
  const int ncv = max(0, min(4, C - c0));
  uint32_t cv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) cv[i] = i < ncv ? cbuf[c0 + i] : 0u;
  uint32_t tau, kk;
  radix_select<4>(sh, cv, ncv, 0u, urange, k, lane, warp, tau, kk);
  // ordered compaction over the candidates
  uint32_t g = 0u, e = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    g += (i < ncv && cv[i] > tau) ? 1u : 0u;
    e += (i < ncv && cv[i] == tau) ? 1u : 0u;
  }
  uint32_t gi = g, ei = e;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t yg = __shfl_up_sync(0xffffffffu, gi, o), ye = __shfl_up_sync(0xffffffffu, ei, o);
    if (lane >= o) {
      gi += yg;
      ei += ye;
    }
  }
  uint32_t og, oe, tg, te;
  warp_offsets(sh.wg, __shfl_sync(0xffffffffu, gi, 31), lane, warp, og, tg);
  warp_offsets(sh.we, __shfl_sync(0xffffffffu, ei, 31), lane, warp, oe, te);
  uint32_t G = og + gi - g, E = oe + ei - e;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i < ncv && cv[i] > tau) {
      out[G + min(E, kk)] = (int32_t)cbuf[kCandCap + c0 + i];
      ++G;
    } else if (i < ncv && cv[i] == tau) {
      if (E < kk) out[G + E] = (int32_t)cbuf[kCandCap + c0 + i];
      ++E;
    }
  }
}

template <int R>
__global__ void __launch_bounds__(kThreads) topk_block_kernel(TopkArgs a) {
  __shared__ alignas(16) BlockShared sh;
  extern __shared__ uint32_t cbuf[];  // R >= 8: [kCandCap] candidate keys, then [kCandCap] positions
  pdl_wait();
  pdl_release();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const int q = blockIdx.x;
  const int n = clamp_count(a.n_cmp[q], a.N_max, threadIdx.x == 0 ? a.status : nullptr);
  const int k = a.k;
  int32_t *out = a.out_idx + (size_t)q * k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  const float *s = a.scores + (size_t)q * a.N_max;
  // key r of this thread: position base + 32 r, valid for r < nvr
  const int base = 32 * R * warp + lane;
  const int nvr = base < n ? min(R, (n - base + 31) / 32) : 0;
  uint32_t key[R];  // the raw bits first: every load in flight before the first is used
#pragma unroll
  for (int r = 0; r < R; ++r) key[r] = r < nvr ? __float_as_uint(__ldcg(s + base + 32 * r)) : 0u;
  uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    key[r] = score_key(__uint_as_float(key[r]));
    if (r < nvr) {
      lo = min(lo, key[r]);
      hi = max(hi, key[r]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    sh.wmin[warp] = lo;
    sh.wmax[warp] = hi;
  }
  for (int i = threadIdx.x; i < 2 * kBins; i += kThreads) (&sh.hist[0][0])[i] = 0u;
  if (threadIdx.x == 0) sh.ncand = 0u;
  __syncthreads();
  lo = sh.wmin[lane];
  hi = sh.wmax[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const uint32_t kmin = lo, range = hi - lo;

  if constexpr (R >= 8) {
    // The sample: key warp % R of every thread (1,024 keys, 32 runs of 32).
    const int rs = warp % R;
    uint32_t su = 0u;
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (r == rs) su = key[r] - kmin;
    const int top = range == 0u ? 0 : 32 - __clz(range);
    const int shift1 = top > 11 ? top - 11 : 0;
    if (rs < nvr) atomicAdd(&sh.hist[0][su >> shift1], 1u);
    // rank m among the S samples: the expected number of samples in the
    // top k, plus four standard deviations and 8
    auto rank_of = [&](uint32_t S) {
      const float mu = (float)k * (float)S / (float)n;
      return (uint32_t)ceilf(mu + 4.f * sqrtf(mu) + 8.f);
    };
    uint32_t bin, above, cb, m, S;
    boundary_bin(sh, sh.hist[0], 0, lane, warp, rank_of, bin, above, cb, m, S);
    for (int i = threadIdx.x; i < kBins; i += kThreads) sh.hist[0][i] = 0u;  // cleared for the selection
    if (range != 0u && m < S) {
      // candidates: keys at or above the lower edge of the sample's boundary bin
      const uint32_t ulow = bin << shift1;
      uint32_t c = 0u;
#pragma unroll
      for (int r = 0; r < R; ++r) c += __popc(__ballot_sync(0xffffffffu, r < nvr && key[r] - kmin >= ulow));
      uint32_t off, C;
      warp_offsets(sh.wg, c, lane, warp, off, C);
      if (C >= (uint32_t)k && C <= (uint32_t)kCandCap) {
        // in position order: warp by warp, key slot by key slot, lane by lane
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const bool sel = r < nvr && key[r] - kmin >= ulow;
          const uint32_t mm = __ballot_sync(0xffffffffu, sel);
          if (sel) {
            const uint32_t slot = off + __popc(mm & lt);
            cbuf[slot] = key[r] - kmin - ulow;
            cbuf[kCandCap + slot] = (uint32_t)(base + 32 * r);
          }
          off += __popc(mm);
        }
        __syncthreads();
        select_candidates(sh, cbuf, (int)C, range - ulow, (uint32_t)k, out, lane, warp);
        return;
      }
    }
    __syncthreads();  // the sample's histogram is clear before the selection over every key
  }

  // Selection over every key, then the ordered compaction: warp w's kept
  // keys go to the slots after those of warps 0 .. w - 1, in position order
  // within the warp (ballots); ties take the first kk positions.
  uint32_t tau_u, kk;
  radix_select<R>(sh, key, nvr, kmin, range, (uint32_t)k, lane, warp, tau_u, kk);
  const uint32_t tau = tau_u + kmin;
  uint32_t g = 0u, e = 0u;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const bool v = r < nvr;
    g += __popc(__ballot_sync(0xffffffffu, v && key[r] > tau));
    e += __popc(__ballot_sync(0xffffffffu, v && key[r] == tau));
  }
  uint32_t G, E, tg, te;
  warp_offsets(sh.wg, g, lane, warp, G, tg);
  warp_offsets(sh.we, e, lane, warp, E, te);
  if (g + e == 0u) return;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int j = base + 32 * r;
    const bool is_gt = r < nvr && key[r] > tau, is_eq = r < nvr && key[r] == tau;
    const uint32_t mg = __ballot_sync(0xffffffffu, is_gt), me = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t Gl = G + __popc(mg & lt), El = E + __popc(me & lt);
    if (is_gt) out[Gl + min(El, kk)] = j;
    else if (is_eq && El < kk) out[Gl + El] = j;
    G += __popc(mg);
    E += __popc(me);
  }
}

// Lists of 16K to 40K entries when every query has its own CTA (many
// queries: a prefill chunk): the block kernel's sample-and-filter scheme over
// keys cached in shared memory instead of registers (R = ceil(n / 1024) per
// thread, positions base + 32 r, so each warp owns a contiguous run). If the
// sample's floor admits fewer than k or more than kCandCap keys, the exact
// multi-pass select runs over the cached keys instead.
__global__ void __launch_bounds__(kThreads) topk_filter_kernel(TopkArgs a) {
  extern __shared__ uint32_t kc[];  // [N_max rounded to 4] keys, then [kCandCap] keys, [kCandCap] positions
  __shared__ alignas(16) BlockShared sh;
  __shared__ TopkShared ts;
  pdl_wait();
  pdl_release();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  const int q = blockIdx.x;
  const int n = clamp_count(a.n_cmp[q], a.N_max, threadIdx.x == 0 ? a.status : nullptr);
  const int k = a.k;
  int32_t *out = a.out_idx + (size_t)q * k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }
  const float *s = a.scores + (size_t)q * a.N_max;
  uint32_t *cbuf = kc + ((a.N_max + 3) & ~3);
  uint32_t lo = 0xffffffffu, hi = 0u;
  sel::cache_keys<kThreads>(kc, s, n, lo, hi);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    sh.wmin[warp] = lo;
    sh.wmax[warp] = hi;
  }
  for (int i = threadIdx.x; i < 2 * kBins; i += kThreads) (&sh.hist[0][0])[i] = 0u;
  if (threadIdx.x == 0) sh.ncand = 0u;
  __syncthreads();  // (also: every key is cached)
  lo = sh.wmin[lane];
  hi = sh.wmax[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const uint32_t kmin = lo, range = hi - lo;
  const int R = (n + kThreads - 1) / kThreads;
  const int base = 32 * R * warp + lane;
  const int nvr = base < n ? min(R, (n - base + 31) / 32) : 0;
  {
    // The sample: key warp % R of every thread (up to 1,024 keys).
    const int rs = warp % R;
    const int top = range == 0u ? 0 : 32 - __clz(range);
    const int shift1 = top > 11 ? top - 11 : 0;
    if (rs < nvr) atomicAdd(&sh.hist[0][(kc[base + 32 * rs] - kmin) >> shift1], 1u);
    auto rank_of = [&](uint32_t S) {  // as in the block kernel
      const float mu = (float)k * (float)S / (float)n;
      return (uint32_t)ceilf(mu + 4.f * sqrtf(mu) + 8.f);
    };
    uint32_t bin, above, cb, m, S;
    boundary_bin(sh, sh.hist[0], 0, lane, warp, rank_of, bin, above, cb, m, S);
    for (int i = threadIdx.x; i < kBins; i += kThreads) sh.hist[0][i] = 0u;  // cleared for the selection
    if (range != 0u && m < S) {
      const uint32_t ulow = bin << shift1;
      uint32_t c = 0u;
      for (int r = 0; r < R; ++r) c += __popc(__ballot_sync(0xffffffffu, r < nvr && kc[base + 32 * r] - kmin >= ulow));
      uint32_t off, C;
      warp_offsets(sh.wg, c, lane, warp, off, C);
      if (C >= (uint32_t)k && C <= (uint32_t)kCandCap) {
        for (int r = 0; r < R; ++r) {  // in position order, as in the block kernel
          const uint32_t u = r < nvr ? kc[base + 32 * r] - kmin : 0u;
          const bool sel = r < nvr && u >= ulow;
          const uint32_t mm = __ballot_sync(0xffffffffu, sel);
          if (sel) {
            const uint32_t slot = off + __popc(mm & lt);
            cbuf[slot] = u - ulow;
            cbuf[kCandCap + slot] = (uint32_t)(base + 32 * r);
          }
          off += __popc(mm);
        }
        __syncthreads();
        select_candidates(sh, cbuf, (int)C, range - ulow, (uint32_t)k, out, lane, warp);
        return;
      }
    }
  }
  __syncthreads();
  select_and_emit<true>(ts, kc, s, n, k, [out](uint32_t slot, int j, uint32_t) { out[slot] = j; });
}

// One query per cluster; CTA c of C selects over the slice
// [c * S, c * S + S) of the list, S = ceil(n / C) rounded up to 32, cached
// in shared memory. With `filt` (the slice and a candidate buffer fit in
// shared memory) the block kernel's sample-and-filter scheme runs over the
// cluster first (cluster_filter); when the sampled floor admits fewer than
// k or more than kCandCap keys, every CTA takes the exact cluster radix
// select instead.
__device__ bool cluster_filter(BlockShared &sh, sel::Shared &cs, uint32_t *hist, const uint32_t *keys, uint32_t *cbuf,
                               int len, int j0, int S, int n, int k, uint32_t C, uint32_t c, uint32_t lo, uint32_t hi,
                               int32_t *out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  // (1) the cluster's key range
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    sh.wmin[warp] = lo;
    sh.wmax[warp] = hi;
  }
  for (int i = threadIdx.x; i < kBins; i += kThreads) hist[i] = 0u;  // this slice's sample histogram
  for (int i = threadIdx.x; i < 2 * kBins; i += kThreads) (&sh.hist[0][0])[i] = 0u;
  if (threadIdx.x == 0) sh.ncand = 0u;
  __syncthreads();
  if (warp == 0) {
    lo = sh.wmin[lane];
    hi = sh.wmax[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      cs.lmin = lo;
      cs.lmax = hi;
    }
  }
  cluster_sync();  // every slice's range is published
  if (warp == 0) {
    lo = (uint32_t)lane < C ? ld_peer(&cs.lmin, lane) : 0xffffffffu;
    hi = (uint32_t)lane < C ? ld_peer(&cs.lmax, lane) : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      cs.kmin = lo;
      cs.krange = hi - lo;
    }
  }
  __syncthreads();
  const uint32_t kmin = cs.kmin, range = cs.krange;
  // (2) the sample: one key per thread, spread over the slice; the slices'
  // histograms are summed into sh.hist[0]
  const int top = range == 0u ? 0 : 32 - __clz(range);
  const int shift1 = top > 11 ? top - 11 : 0;
  {
    const int js = (int)(((long long)threadIdx.x * S) / kThreads);
    if (js < len) atomicAdd(&hist[(keys[js] - kmin) >> shift1], 1u);
  }
  cluster_sync();  // every slice's sample histogram is complete
  for (int b = 4 * (int)threadIdx.x; b < kBins; b += 4 * kThreads) {
    uint4 t = make_uint4(0u, 0u, 0u, 0u);
    for (uint32_t r = 0; r < C; ++r) {
      const uint4 v = ld_peer_u4(&hist[b], r);
      t.x += v.x;
      t.y += v.y;
      t.z += v.z;
      t.w += v.w;
    }
    *reinterpret_cast<uint4 *>(&sh.hist[0][b]) = t;
  }
  auto rank_of = [&](uint32_t Sn) {  // as in the block kernel
    const float mu = (float)k * (float)Sn / (float)n;
    return (uint32_t)ceilf(mu + 4.f * sqrtf(mu) + 8.f);
  };
  uint32_t bin, above, cb, m, Sn;
  boundary_bin(sh, sh.hist[0], 0, lane, warp, rank_of, bin, above, cb, m, Sn);
  for (int i = threadIdx.x; i < kBins; i += kThreads) sh.hist[0][i] = 0u;  // cleared for the selection
  const bool floor_ok = range != 0u && m < Sn;
  const uint32_t ulow = bin << shift1;
  // (3) this slice's candidates (keys at or above the floor), counted in
  // position order: warp w scans a contiguous run of the slice
  const int per_warp = (((len + kWarps - 1) / kWarps) + 31) & ~31;
  const int wlo = min(len, warp * per_warp), whi = min(len, wlo + per_warp);
  uint32_t cnt = 0u;
  for (int base = wlo; base < whi; base += 32) {
    const int j = base + lane;
    cnt += __popc(__ballot_sync(0xffffffffu, floor_ok && j < whi && keys[j] - kmin >= ulow));
  }
  uint32_t off, Cl;
  warp_offsets(sh.wg, cnt, lane, warp, off, Cl);
  if (threadIdx.x == 0) cs.cnt_gt = Cl;
  cluster_sync();  // every slice's count is published; no peer reads a sample histogram any more
  if (warp == 0) {
    const uint32_t x = (uint32_t)lane < C ? ld_peer(&cs.cnt_gt, lane) : 0u;
    uint32_t inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    const uint32_t excl = __shfl_sync(0xffffffffu, inc - x, (int)c), total = __shfl_sync(0xffffffffu, inc, 31);
    if (lane == 0) {
      cs.base_gt = excl;
      cs.bcnt = total;
    }
  }
  __syncthreads();
  const uint32_t Ctot = cs.bcnt, cbase = cs.base_gt;
  if (!(floor_ok && Ctot >= (uint32_t)k && Ctot <= (uint32_t)kCandCap)) return false;  // the same in every CTA
  // (4) the candidates go to CTA 0 in position order; it selects among them
  uint32_t slot0 = cbase + off;
  for (int base = wlo; base < whi; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < whi ? keys[j] - kmin : 0u;
    const bool selb = j < whi && u >= ulow;
    const uint32_t mm = __ballot_sync(0xffffffffu, selb);
    if (selb) {
      const uint32_t slot = slot0 + __popc(mm & lt);
      st_peer(&cbuf[slot], 0u, u - ulow);
      st_peer(&cbuf[kCandCap + slot], 0u, (uint32_t)(j0 + j));
    }
    slot0 += __popc(mm);
  }
  cluster_sync();  // every candidate is in CTA 0; no CTA touches a peer after this
  if (c == 0) select_candidates(sh, cbuf, (int)Ctot, range - ulow, (uint32_t)k, out, lane, warp);
  return true;
}

__global__ void __launch_bounds__(kThreads) topk_cluster_kernel(TopkArgs a, int filt) {
  extern __shared__ uint32_t keys[];  // [S] slice keys (then, with filt, [2 kCandCap] candidates)
  __shared__ alignas(16) uint32_t hist[2 * kBins];
  __shared__ sel::Shared cs;
  __shared__ alignas(16) BlockShared sh;
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
  if (filt) {
    uint32_t *cbuf = keys + (((a.N_max + (int)C - 1) / (int)C + 31) & ~31);  // past the largest slice
    if (cluster_filter(sh, cs, hist, keys, cbuf, len, j0, S, n, k, C, c, lo, hi, out)) return;
  }
  sel::cluster_select<kThreads, 4, 8>(cs, hist, keys, len, j0, k, C, c, lo, hi,
                                      [&](uint32_t slot, int j) { out[slot] = j; });
  cluster_wait();  // no peer reads this CTA's shared memory any more
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
    for (auto kern : {topk_block_kernel<8>, topk_block_kernel<16>})
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * kCandCap * (int)sizeof(uint32_t));
    cudaFuncSetAttribute(topk_filter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (kFilterKeys + 2 * kCandCap) * (int)sizeof(uint32_t));
  });
  // Lists of up to 16 K entries: one CTA per query, keys in registers.
  if (a.N_max <= 16 * kThreads) {
    const int R = (a.N_max + kThreads - 1) / kThreads;
    auto kern = R <= 4 ? topk_block_kernel<4> : R <= 8 ? topk_block_kernel<8> : topk_block_kernel<16>;
    return launch_pdl(kern, dim3(a.Q), dim3(kThreads), R <= 4 ? 0 : 2 * kCandCap * sizeof(uint32_t), stream, a);
  }
  if (const int C = plan_cluster(a.Q, a.N_max, a.k)) {
    const int S = ((a.N_max + C - 1) / C + 31) & ~31;
    // the sample-and-filter front when the slice and the candidate buffer fit
    const int filt = S <= kFilterKeys ? 1 : 0;
    const size_t smem = (size_t)S * 4 + (filt ? 2 * kCandCap * sizeof(uint32_t) : 0);
    return launch_pdl_cluster(topk_cluster_kernel, dim3(C, a.Q), dim3(kThreads), smem, stream, (unsigned)C, a, filt);
  }
  // Up to 40 K entries with a CTA per query: sample, filter, select over
  // the keys cached in shared memory.
  if (a.N_max <= kFilterKeys) {
    const size_t smem = (((size_t)a.N_max + 3) & ~(size_t)3) * 4 + 2 * kCandCap * sizeof(uint32_t);
    return launch_pdl(topk_filter_kernel, dim3(a.Q), dim3(kThreads), smem, stream, a);
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
