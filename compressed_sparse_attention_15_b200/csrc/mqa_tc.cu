// A4 / A5 on the tensor cores for the Flash attention shape: 64 query heads,
// one shared KV head, head_dim 512, K = V, bf16 in, fp32 accumulation; the
// V4-Pro shape (128 heads) runs as two 64-head groups per query, one block
// row each, reading the same KV rows (the second read mostly from L2)
// ("DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: sliding window
// + compressed rows + per-head attention sink; section 2: keys and values
// share one 512-dim representation).
//
// Transposed formulation:
//   S^T[r, h]  = sum_d KV[r, d] Q[h, d]      M = 64 rows,  N = 64 heads, K-major A and B
//   O^T[d, h] += sum_r KV[r, d] P^T[r, h]    M = 128 dims, N = 64 heads, A = the same KV
//                                            tile read MN-major, B = P^T (MN-major)
// A 64-row x 512-dim KV tile is loaded once into shared memory (128-byte
// swizzled, 64-dim boxes) and feeds both products. Two tile buffers, two S^T
// TMEM buffers and two P^T buffers make a software pipeline: while the
// softmax warps turn S^T(t) into P(t), the tensor core computes S^T(t+1) and
// the loaders fill the other buffer. The MMA thread issues S^T and P.V each
// as soon as its inputs are ready.
// An M = 64 accumulator occupies TMEM lanes 0-15 of each 32-lane quarter, so
// each softmax warp owns 16 rows; read with the 16x256b shape, every thread
// holds 2 rows x 16 heads. The per-head tile maximum is a 3-step shuffle
// reduction plus a 4-warp exchange; the running per-head maximum only moves
// (and O^T is rescaled in TMEM, after the previous P.V has completed) when a
// tile's maximum exceeds it by more than 2^8, so P <= 256 in bf16.
//
// Loads: contiguous runs of 64 rows (HCA entries, window rows) are single TMA
// boxes of 64 rows; top-k rows are gathered with 16-byte cp.async copies by
// the loader warps (TMA gathers issue too slowly for 1 KB rows). The
// compressed segment is padded to a multiple of 4 rows (unused, masked).
//
// Work split: query q's row list is cut into `splits` (<= 16) runs of whole
// tiles, one CTA each. Normally the CTAs of a query form one thread-block
// cluster (the largest size for which every query's cluster is resident at
// once); when that caps the splits well below SMs / Q, they are plain blocks
// and mqa_combine_kernel merges their partials.
// With one split the CTA folds in the sink and writes the output; otherwise
// every CTA writes its unnormalised (m, l, O) to the workspace and, in a
// cluster, after a cluster barrier merges 1/splits of the output from all of
// them (L2 reads; distributed-shared-memory reads of the same data measured
// several times slower).
// Roles (416 threads): warps 0-7 load (four per tile buffer), warp 8 issues
// the MMAs and owns TMEM, warps 9-12 run the softmax and the epilogue. All
// mbarrier waits are bounded; the softmax warps take every decision to stop
// together (a barrier reduction), so no named barrier is left half-joined.
#include "cluster_select.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace csa {

namespace {

constexpr int kH = 64, kD = 512;
constexpr int kRows = 64;                           // rows per tile
constexpr uint32_t kBoxBytes = kRows * 128;         // 64 rows x 64 dims: 8 KB
constexpr uint32_t kTileBytes = 8 * kBoxBytes;      // 64 rows x 512 dims: 64 KB
constexpr uint32_t kQBoxBytes = kH * 128;           // 64 heads x 64 dims: 8 KB
constexpr uint32_t kQBytes = 8 * kQBoxBytes;        // 64 KB
constexpr uint32_t kPBytes = kRows * kH * 2;        // 8 KB
constexpr int kLoadWarps = 8;                       // four per tile buffer
constexpr int kWarpsPerBuf = kLoadWarps / 2;
constexpr int kRowsPerWarp = kRows / kWarpsPerBuf;  // 16 rows of a tile per loader warp
constexpr int kMmaWarp = kLoadWarps;
constexpr int kSoftWarp0 = kLoadWarps + 1;          // 4 softmax warps: one per TMEM lane quarter
constexpr int kThreads = 32 * (kSoftWarp0 + 4);
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxSplits = 16;                      // splits of one query form one cluster (<= 16 CTAs)
constexpr uint32_t kColO = 0;                       // O^T chunk m at columns 64m (M = 128 layout)
constexpr uint32_t kColS = 256;                     // S^T buffer j at 256 + 64j (M = 64 layout)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kSelMax = 1024;                       // largest k selected inside the kernel
constexpr int kSelKeys = 2 * kTileBytes / 4;        // slice keys that fit in the tile buffers
// Rounds of tiles whose rows the loaders bring into L2 ahead of their load:
// with two tile buffers a tile's load can only start once the buffer is
// free, so the L2 prefetches are what keeps more of the stream in flight.
constexpr int kAhead = 1;

struct Small {
  uint64_t q_full, kv_full[2], kv_empty[2], s_full[2], p_full[2], pv_done[4], o_done;
  float red[4][kH];
  alignas(16) float mref[kH];
  float alpha[kH];
  float lsum[kH];
  uint32_t tmem_base;
  int abort;
  int rescale;
  int need[4];  // per tile (mod 4): some logit exceeded the running maximum by more than 2^8
  const bf16 *rowp[kLoadWarps][kRowsPerWarp];  // gathered tiles: source of each of a loader warp's rows (null: zero-fill)
  sel::Shared cs;                    // in-kernel top-k: cluster exchange
  int32_t sel[kSelMax];              // in-kernel top-k: the selected entry of each list position of this split
};

constexpr size_t kSmemBytes = 1024 + 2 * kTileBytes + kQBytes + 2 * kPBytes + sizeof(Small);
static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
static_assert(2 * kPBytes == 2 * sel::kBins * 4, "the P buffers hold the two selection histograms");

// Row list of one query: the window rows [0, nwin) (kv_win rows wlo ..
// wlo + nwin - 1, padded with unused rows to whole tiles: w64), then the
// compressed rows [w64, w64 + nsel) in list order (selected entries, or the
// visible entries of a dense list; nsel4 = nsel padded to a multiple of 4).
// Window tiles are contiguous runs and need nothing the selection produces.
struct RowList {
  int nsel, nsel4, wlo, nwin, w64, R;
};

__device__ __forceinline__ RowList row_list(const MqaArgs &a, int qq, uint32_t *status) {
  RowList L;
  L.nsel = (a.idx || a.scores) ? a.k : clamp_count(a.n_cmp[qq], a.N_max, status);
  int e = a.win_end[qq];
  if (e < 0 || e >= a.T_raw) {
    raise_status(status, CSA_STATUS_BAD_WINDOW);
    e = e < 0 ? 0 : a.T_raw - 1;
  }
  L.wlo = max(0, e - a.win_len + 1);
  L.nwin = e - L.wlo + 1;
  L.w64 = (L.nwin + kRows - 1) / kRows * kRows;
  L.nsel4 = (L.nsel + 3) & ~3;
  L.R = L.w64 + L.nsel;
  return L;
}

// The tiles [t0, t1) of split `split`: runs of tiles_per_split tiles; with
// the window on top (a selection's window tiles computed before the kernel
// waits on its predecessor, its compressed tiles after) split 0 takes the
// window tiles on top of its run and the runs cover the compressed tiles.
__device__ __forceinline__ void split_tiles(const RowList &L, int split, int tiles_per_split, bool window_on_top,
                                            int &t0, int &t1) {
  const int tiles_all = (L.R + kRows - 1) / kRows, wt = L.w64 / kRows;
  if (window_on_top) {
    t0 = split == 0 ? 0 : wt + split * tiles_per_split;
    t1 = min(tiles_all, wt + (split + 1) * tiles_per_split);
  } else {
    t0 = split * tiles_per_split;
    t1 = min(tiles_all, t0 + tiles_per_split);
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// L2 prefetch of `bytes` contiguous bytes at p (16-byte aligned, a multiple
// of 16).
__device__ __forceinline__ void bulk_prefetch_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// 2^x on the SFU (relative error about 2^-22; flushes subnormal results to
// zero, which only ever meets weights far below the bf16 resolution of P).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Named barrier over n threads that also ORs `pred` across them: every
// participant gets the same answer.
__device__ __forceinline__ bool bar_any(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, %2, %3, p; selp.u32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// out[h][d..d+3] = sum_r coef[r][h] * O_r[h][d..d+3] for the 4-dim groups
// [g0, g1) of one query (O_r: the split partials, [64][512] fp32 each). Each
// thread takes kB groups per round, all kB * splits loads issued first.
template <int kB, int kS>
__device__ __forceinline__ void merge_groups(const float *po, const float *coef, bf16 *out, int splits, int g0,
                                             int g1) {
  for (int base = g0 + threadIdx.x; base < g1; base += kThreads * kB) {
    float4 v[kB][kS];
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int gi = base + i * kThreads;
      const int h = gi / (kD / 4), d = 4 * (gi % (kD / 4));
#pragma unroll
      for (int r = 0; r < kS; ++r)
        if (r < splits && gi < g1) v[i][r] = __ldcg(reinterpret_cast<const float4 *>(po + ((size_t)r * kH + h) * kD + d));
    }
#pragma unroll
    for (int i = 0; i < kB; ++i) {
      const int gi = base + i * kThreads;
      if (gi >= g1) break;
      const int h = gi / (kD / 4), d = 4 * (gi % (kD / 4));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < kS; ++r)
        if (r < splits) {
          const float c = coef[r * kH + h];
          acc.x = fmaf(c, v[i][r].x, acc.x);
          acc.y = fmaf(c, v[i][r].y, acc.y);
          acc.z = fmaf(c, v[i][r].z, acc.z);
          acc.w = fmaf(c, v[i][r].w, acc.w);
        }
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
      *reinterpret_cast<uint2 *>(out + h * kD + d) =
          make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
    }
  }
}

// tcgen05.ld of 16 TMEM lanes x 64 columns (16x256b shape, 8 repeats): for
// column group c, thread t gets r[4c + e] = (lane t/4, column 8c + 2(t%4) + e)
// and r[4c + 2 + e] = (lane t/4 + 8, same column), e = 0, 1.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Top-k of query qq's indexer scores by the cluster of its splits, all
// threads taking part (the selection csa_topk makes). List position r of the
// selection (row w64 + r of the row list) lands in sel[r] of the split whose
// tiles hold it, and in idx_out
// (written by head group 0); each selected row is prefetched into L2 as it is
// found. The slice's keys use the tile buffers and the histograms the P
// buffers, neither in use yet.
__device__ void select_rows(const MqaArgs &a, Small *sm, uint8_t *kv, uint8_t *ps, int qq, int hg, int b,
                            int tiles_per_split, int w64) {
  const uint32_t C = cluster_size(), c = cluster_rank();
  const int n = clamp_count(a.n_cmp[qq], a.N_max, (threadIdx.x == 0 && c == 0) ? a.status : nullptr);
  const int k = a.k;
  int32_t *out = hg == 0 ? a.idx_out + (size_t)qq * k : nullptr;
  if (n <= k) {  // the same in every block of the cluster: no block touches a peer
    for (int i = threadIdx.x; i < k; i += kThreads) {
      const int j = i < n ? i : -1;
      sm->sel[i] = j;
      if (out && c == 0) out[i] = j;
    }
  } else {
    const int S = ((n + (int)C - 1) / (int)C + 31) & ~31;
    const int j0 = (int)c * S, len = max(0, min(S, n - j0));
    uint32_t *keys = reinterpret_cast<uint32_t *>(kv);
    uint32_t lo = 0xffffffffu, hi = 0u;
    sel::cache_keys<kThreads>(keys, a.scores + (size_t)qq * a.N_max + j0, len, lo, hi);
    const bf16 *rows = static_cast<const bf16 *>(a.kv_cmp) + (size_t)b * a.N_max * kD;
    const int rows_per_split = kRows * tiles_per_split;
    sel::cluster_select<kThreads, 8, kMaxSplits>(
        sm->cs, reinterpret_cast<uint32_t *>(ps), keys, len, j0, k, C, c, lo, hi, [&](uint32_t slot, int j) {
          st_peer(&sm->sel[slot], (slot + (uint32_t)w64) / (uint32_t)rows_per_split, (uint32_t)j);
          if (out) out[slot] = j;
          bulk_prefetch_l2(rows + (size_t)j * kD, kD * 2);
        });
    cluster_wait();  // every selected position is in its split's sel; no peer reads this block any more
  }
  // the keys were written through the generic proxy; the tile buffers are
  // next written by TMA and cp.async
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
}

// kFused: the selection is made here from a.scores (select_rows) instead of
// read from a.idx; a separate instantiation, so the plain kernel carries none
// of its code.
template <bool kFused>
__global__ void __launch_bounds__(kThreads, 1)
    mqa_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_cmp_t,
                  const __grid_constant__ CUtensorMap tm_win_t, MqaArgs a, int splits, int tiles_per_split,
                  float scale_log2, float *part_o, float *part_ml, int cluster_merge) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *kv = smem;                              // [2 tiles][8 boxes][64 rows][128 B]
  uint8_t *qs = smem + 2 * kTileBytes;             // [8 boxes][64 heads][128 B]
  uint8_t *ps = qs + kQBytes;                      // [2][64 rows][128 B]  (P^T, MN-major)
  Small *sm = reinterpret_cast<Small *>(ps + 2 * kPBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx.y = qv: one group of 64 heads of query qq (H = 64 G)
  const int G = a.H / kH;
  const int split = blockIdx.x, qv = blockIdx.y, qq = qv / G, hg = qv - qq * G;
  const int b = qq / a.q_per_seq;

  if (threadIdx.x == 0) {
    tc::mbar_init(&sm->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sm->kv_full[i], 32 * kWarpsPerBuf);
      tc::mbar_init(&sm->kv_empty[i], 1);
      tc::mbar_init(&sm->s_full[i], 1);
      tc::mbar_init(&sm->p_full[i], 4 * 32);
    }
    for (int i = 0; i < 4; ++i) tc::mbar_init(&sm->pv_done[i], 1);
    tc::mbar_init(&sm->o_done, 1);
    sm->abort = 0;
    sm->rescale = 0;
    for (int i = 0; i < 4; ++i) sm->need[i] = 0;
    tc::fence_barrier_init();
  }
  if (threadIdx.x < kH) {
    sm->mref[threadIdx.x] = -INFINITY;
    sm->alpha[threadIdx.x] = 1.f;
  }
  if (warp == kMmaWarp) tc::tmem_alloc(&sm->tmem_base, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = sm->tmem_base;
  volatile int *abort = &sm->abort;
  // early: the queries and the window tiles do not depend on the previous
  // kernel; every role waits for it before its first compressed tile, and
  // before any global write. Otherwise everything waits here.
  const bool early = !kFused && a.early;
  if (!early) pdl_wait();  // inputs (indices, queries, caches) may come from the previous kernel
  const uint64_t lim = tc::wait_limit_of(a.status);
  pdl_release();

  const RowList L = row_list(a, qq, threadIdx.x == 0 ? a.status : nullptr);
  constexpr bool fused = kFused;
  const bool sparse = fused || a.idx != nullptr;
  // (a selection's compressed tiles all wait: split 0 takes the window tiles
  // on top of its run; a dense list's tiles are split evenly)
  int t0, t1;
  split_tiles(L, split, tiles_per_split, early && sparse, t0, t1);
  const int ntiles = max(0, t1 - t0);
  // Whether this CTA's tile li needs the previous kernel done (early mode):
  // a compressed tile of a selection, or of a dense list holding a row that
  // kernel writes.
  auto tile_dep = [&](int li) -> bool {
    const int r0 = (t0 + li) * kRows;
    if (r0 < L.w64) return false;
    if (sparse || a.dep_row0 < 0) return true;
    const int p0 = r0 - L.w64, p1 = min(p0 + kRows, L.nsel);
    return p0 < p1 && p0 < a.dep_row0 + a.dep_rows && a.dep_row0 < p1;
  };
  if (warp == kMmaWarp && lane == 0 && ntiles > 0) {
    tc::prefetch_tmap(&tm_q);
    tc::mbar_arrive_expect_tx(&sm->q_full, kQBytes);
    for (int bx = 0; bx < kD / 64; ++bx) tc::tma_load_2d(qs + bx * kQBoxBytes, &tm_q, bx * 64, qv * kH, &sm->q_full);
  }
  if constexpr (kFused) select_rows(a, sm, kv, ps, qq, hg, b, tiles_per_split, L.w64);
  // entry of the selection at list position p < nsel
  auto sel_at = [&](int p) -> int { return fused ? sm->sel[p] : a.idx[(size_t)qq * a.k + p]; };

  if (warp < kLoadWarps) {
    // ------------------------------------------------------------ loaders
    // Warps 4g .. 4g + 3 fill tile buffer g (tiles g, g + 2, ...), 16 rows
    // of each tile each (part = warp % 4: rows 16 part .. 16 part + 15). A
    // contiguous run is 8 TMA boxes issued by lane 0 of warp 4g. A gathered
    // tile is 16-byte cp.async copies, 32 per lane, each warp instruction
    // moving 512 contiguous bytes of one row; every lane waits for its own
    // copies, fences them for the tensor core and arrives, so kv_full
    // expects 128 arrivals either way. Each warp also prefetches its rows of
    // its next kAhead tiles into L2 while the buffer is busy.
    const int g = warp / kWarpsPerBuf, part = warp % kWarpsPerBuf;
    const uint32_t buf_base = tc::smem_u32(kv) + g * kTileBytes;
    bool waited = !early;
    if (warp == 0 && lane == 0) {
      tc::prefetch_tmap(&tm_cmp_t);
      tc::prefetch_tmap(&tm_win_t);
    }
    // Source row of row-list row r (null: padding or an unused slot).
    auto src_row = [&](int r) -> const bf16 * {
      if (r < L.w64)
        return r < L.nwin ? static_cast<const bf16 *>(a.kv_win) + ((size_t)b * a.T_raw + L.wlo + r) * kD : nullptr;
      const int p = r - L.w64;
      if (p < L.nsel) {
        int j = sparse ? sel_at(p) : p;
        if (j < -1 || j >= a.N_max) {
          raise_status(a.status, CSA_STATUS_BAD_INDEX);
          j = -1;
        }
        return j >= 0 ? static_cast<const bf16 *>(a.kv_cmp) + ((size_t)b * a.N_max + j) * kD : nullptr;
      }
      return nullptr;
    };
    // A tile is one contiguous run when it lies in the window part, or in the
    // compressed part of a dense (HCA) row list.
    auto is_run = [&](int r0, bool &win_run) {
      win_run = r0 < L.w64;
      return win_run || (!sparse && r0 - L.w64 + kRows <= L.nsel4);
    };
    // Bring this warp's rows of tile li into L2 ahead of their load, which can
    // only start once the tile buffer is free: the load then waits on L2.
    // (A run's rows are contiguous in memory: one bulk prefetch of this
    // warp's 16 rows streams them from HBM in order, where the tile's TMA
    // boxes each read 128 bytes of every row.)
    auto prefetch_l2 = [&](int li) {
      if (li >= ntiles) return;
      const int r0 = (t0 + li) * kRows;
      bool win_run;
      if (is_run(r0, win_run)) {
        if (lane == 0) {
          // first row of this warp's part, and how many rows of the sequence's buffer remain from it
          const int first = win_run ? L.wlo + r0 + kRowsPerWarp * part : r0 - L.w64 + kRowsPerWarp * part;
          const int avail = (win_run ? a.T_raw : a.N_max) - first;
          const int rows = avail < kRowsPerWarp ? avail : kRowsPerWarp;
          if (rows > 0) {
            const bf16 *base = win_run ? static_cast<const bf16 *>(a.kv_win) + ((size_t)b * a.T_raw + first) * kD
                                       : static_cast<const bf16 *>(a.kv_cmp) + ((size_t)b * a.N_max + first) * kD;
            bulk_prefetch_l2(base, (uint32_t)rows * kD * 2);
          }
        }
      } else if (lane < kRowsPerWarp && (!early || waited)) {  // (a gathered tile's rows need the selection)
        if (const bf16 *p = src_row(r0 + kRowsPerWarp * part + lane)) bulk_prefetch_l2(p, kD * 2);
      }
    };
    int last = -1;
    for (int li = g; li < ntiles; li += 2) {
      const int r0 = (t0 + li) * kRows;
      if (!waited && tile_dep(li)) {  // the first tile that needs the previous kernel done
        pdl_wait();
        waited = true;
      }
      bool win_run;
      const bool run = is_run(r0, win_run);
      __syncwarp();  // the previous tile's copies have read rowp[warp]
      if (!run && lane < kRowsPerWarp) sm->rowp[warp][lane] = src_row(r0 + kRowsPerWarp * part + lane);
      if (li == g) {  // the first tile streams in order too; later tiles are prefetched kAhead rounds ahead
        if (run) prefetch_l2(li);
        for (int r = 1; r <= kAhead; ++r) prefetch_l2(li + 2 * r);
      }
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm->kv_empty[g], ((li >> 1) & 1) ^ 1, abort, a.status, lim))) break;
      if (run) {
        if (part == 0 && lane == 0) {
          tc::mbar_arrive_expect_tx(&sm->kv_full[g], kTileBytes);
          const int row = win_run ? b * a.T_raw + L.wlo + r0 : b * a.N_max + (r0 - L.w64);
          for (int bx = 0; bx < 8; ++bx)
            tc::tma_load_2d(kv + g * kTileBytes + bx * kBoxBytes, win_run ? &tm_win_t : &tm_cmp_t, 64 * bx, row,
                            &sm->kv_full[g]);
        } else {
          tc::mbar_arrive(&sm->kv_full[g]);
        }
      } else {
        __syncwarp();  // rowp[warp] written by every lane
#pragma unroll 8
        for (int i = 0; i < 2 * kRowsPerWarp; ++i) {
          const int rw = i >> 1, c16 = lane + 32 * (i & 1);  // 16-byte piece c16 of this warp's row rw
          const int row = kRowsPerWarp * part + rw;           // row within the tile
          const bf16 *src = sm->rowp[warp][rw];
          const uint32_t dst = buf_base + (c16 >> 3) * kBoxBytes + row * 128 + (((c16 & 7) ^ (row & 7)) << 4);
          cp_async16(dst, src ? src + c16 * 8 : static_cast<const bf16 *>(a.kv_win), src != nullptr);
        }
      }
      if (li > g) prefetch_l2(li + 2 * kAhead);
      if (!run) {
        cp_async_wait_all();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc::mbar_arrive(&sm->kv_full[g]);
      }
      last = li;
    }
    // Drain: a TMA tile still in flight must land before the CTA exits.
    if (part == 0 && lane == 0 && last >= 0) tc::mbar_drain(&sm->kv_full[g], (last >> 1) & 1);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const bool q_issued = ntiles > 0;  // the Q load was issued above
      constexpr uint32_t idesc_s = tc::idesc_bf16(64, 64, 0, 0);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(128, 64, 1, 1);
      const uint32_t kv_base = tc::smem_u32(kv), q_base = tc::smem_u32(qs), p_base = tc::smem_u32(ps);
      bool ok = ntiles == 0 || tc::mbar_wait(&sm->q_full, 0, abort, a.status, lim);
      const uint64_t ad_kv = tc::sw128_desc(kv_base, 16, 1024), bd_q = tc::sw128_desc(q_base, 16, 1024);
      const uint64_t ad_v = tc::sw128_desc(kv_base, kBoxBytes, 1024), bd_p = tc::sw128_desc(p_base, kPBytes, 1024);
      // Two streams of work, issued as soon as each is ready: S^T(ns) once
      // tile ns has landed (and the softmax is done with S^T(ns - 2)), and
      // P.V(np) once P(np) is written. Neither waits behind the other, so the
      // P.V that frees a tile buffer is never held up by the next tile's load.
      int ns = 0, np = 0;
      uint32_t idle = 0;
      uint64_t t_idle = 0;
      while (ok && np < ntiles) {
        bool progressed = false;
        if (np < ns && tc::mbar_test_wait(&sm->p_full[np & 1], (np >> 1) & 1)) {
          // O^T += V^T(np) P^T(np)
          const int pb = np & 1;
          tc::fence_after_sync();
          const uint64_t ad0 = ad_v + (uint64_t)((pb * kTileBytes) >> 4), bd0 = bd_p + (uint64_t)((pb * kPBytes) >> 4);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
#pragma unroll
            for (int j = 0; j < kRows / 16; ++j)
              tc::mma_bf16(tmem + kColO + 64 * m, ad0 + (uint64_t)((2 * m * kBoxBytes + j * 2048) >> 4),
                           bd0 + (uint64_t)((j * 2048) >> 4), idesc_pv, np > 0 || j > 0);
          }
          tc::commit(&sm->kv_empty[pb]);
          tc::commit(&sm->pv_done[np & 3]);
          ++np;
          progressed = true;
        }
        // S^T(ns) overwrites the S^T buffer of tile ns - 2: P.V(ns - 2) must
        // have been issued, i.e. its softmax has finished reading it.
        if (ns < ntiles && ns <= np + 1 && tc::mbar_test_wait(&sm->kv_full[ns & 1], (ns >> 1) & 1)) {
          const int buf = ns & 1;
          tc::fence_after_sync();
          const uint64_t ad0 = ad_kv + (uint64_t)((buf * kTileBytes) >> 4);
#pragma unroll
          for (int j = 0; j < kD / 16; ++j)
            tc::mma_bf16(tmem + kColS + 64 * buf, ad0 + (uint64_t)(((j >> 2) * kBoxBytes + (j & 3) * 32) >> 4),
                         bd_q + (uint64_t)(((j >> 2) * kQBoxBytes + (j & 3) * 32) >> 4), idesc_s, j > 0);
          tc::commit(&sm->s_full[buf]);
          ++ns;
          progressed = true;
        }
        if (progressed) {
          idle = 0;
          t_idle = 0;
          continue;
        }
        if (*abort) {
          ok = false;
        } else {
          __nanosleep(32);  // neither product is ready: leave the issue slots to the other warps
        }
        if (ok && (++idle & 63) == 0) {
          const uint64_t now = tc::globaltimer_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (now - t_idle > lim) {
            raise_status(a.status, CSA_STATUS_WAIT_TIMEOUT);
            *abort = 1;
            ok = false;
          }
        }
      }
      tc::commit(&sm->o_done);
      tc::mbar_drain(&sm->o_done, 0);
      if (q_issued) tc::mbar_drain(&sm->q_full, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    // A warp owns the 16 S^T rows of its TMEM quarter (M = 64 layout) and
    // reads them with the 16x256b shape: lane t holds rows rq = t/4 and
    // rq + 8 for heads 8c + 2cq + {0, 1} (c = 0..7, cq = t%4).
    const int rq = lane >> 2, cq = lane & 3;
    const int rowA = quarter * 16 + rq, rowB = rowA + 8;  // tile rows of this thread
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool leader = warp == kSoftWarp0;
    float l[16];  // running sums of heads 8c + 2cq + e at l[2c + e]
#pragma unroll
    for (int i = 0; i < 16; ++i) l[i] = 0.f;
    bool ok = true, waited = !early;
    // a row-list row holds a key: a window row below nwin, a compressed row
    // with a valid entry
    auto valid_row = [&](int r) -> bool {
      if (r < L.w64) return r < L.nwin;
      const int p = r - L.w64;
      if (p >= L.nsel) return false;
      if (!sparse) return true;
      const int j = sel_at(p);
      return j >= 0 && j < a.N_max;
    };
    for (int li = 0; li < ntiles; ++li) {
      const int buf = li & 1;
      if (!waited && tile_dep(li)) {  // the first tile that needs the previous kernel done
        pdl_wait();
        waited = true;
      }
      const int rA = (t0 + li) * kRows + rowA, rB = rA + 8;
      const bool validA = valid_row(rA), validB = valid_row(rB);
      const bool got = __all_sync(0xffffffffu, tc::mbar_wait(&sm->s_full[buf], (li >> 1) & 1, abort, a.status, lim));
      tc::fence_after_sync();
      uint32_t v[32];
      tmem_ld_16x256b_x8(tmem + lane_off + kColS + 64 * buf, v);
      tc::tmem_ld_wait();
      // logits in log2 units; invalid rows are -inf
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          v[4 * c + e] = __float_as_uint(validA ? __uint_as_float(v[4 * c + e]) * scale_log2 : -INFINITY);
          v[4 * c + 2 + e] = __float_as_uint(validB ? __uint_as_float(v[4 * c + 2 + e]) * scale_log2 : -INFINITY);
        }
      // Fast path: the running per-head maximum moves only when some logit
      // of the tile exceeds it by more than 2^8 (always on the first tile).
      bool over = false;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float2 mr = *reinterpret_cast<const float2 *>(&sm->mref[8 * c + 2 * cq]);
        over |= __uint_as_float(v[4 * c]) > mr.x + kRescaleLog2 || __uint_as_float(v[4 * c + 1]) > mr.y + kRescaleLog2 ||
                __uint_as_float(v[4 * c + 2]) > mr.x + kRescaleLog2 || __uint_as_float(v[4 * c + 3]) > mr.y + kRescaleLog2;
      }
      if (leader && lane == 0) sm->need[(li + 2) & 3] = 0;  // slot of tile li + 2, last read at tile li - 2
      if (__any_sync(0xffffffffu, over) && lane == 0) atomicOr(&sm->need[li & 3], 1);
      if (bar_any(1, 128, !(got && ok))) {  // S^T(li) missing, or the previous P.V never completed
        ok = false;
        break;
      }
      bool rescale = false;
      if (sm->need[li & 3] != 0) {
        // per-head tile maximum: over the thread's two rows, then over the 8
        // lanes of the same cq, then over the 4 warps
        float mx[16];
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
          for (int e = 0; e < 2; ++e) mx[2 * c + e] = fmaxf(__uint_as_float(v[4 * c + e]), __uint_as_float(v[4 * c + 2 + e]));
#pragma unroll
        for (int o = 4; o < 32; o <<= 1)
#pragma unroll
          for (int i = 0; i < 16; ++i) mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], o));
        if (rq == 0) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
#pragma unroll
            for (int e = 0; e < 2; ++e) sm->red[quarter][8 * c + 2 * cq + e] = mx[2 * c + e];
        }
        named_sync(1, 128);
        if (leader) {
          bool any = false;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int h = 2 * lane + i;
            const float tm = fmaxf(fmaxf(sm->red[0][h], sm->red[1][h]), fmaxf(sm->red[2][h], sm->red[3][h]));
            const float mo = sm->mref[h];
            float al = 1.f;
            if (mo == -INFINITY || tm > mo + kRescaleLog2) {
              const float mn = fmaxf(mo, tm);
              al = mo == -INFINITY ? 0.f : exp2f(mo - mn);
              sm->mref[h] = mn;
              any |= mo != -INFINITY;
            }
            sm->alpha[h] = al;
          }
          any = __any_sync(0xffffffffu, any);
          if (lane == 0) sm->rescale = any ? 1 : 0;
        }
        named_sync(1, 128);
        rescale = sm->rescale != 0;
        if (rescale) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float2 al = *reinterpret_cast<const float2 *>(&sm->alpha[8 * c + 2 * cq]);
            l[2 * c] *= al.x;
            l[2 * c + 1] *= al.y;
          }
        }
      }
      // P = 2^(x - mref), rounded to bf16, summed per head, packed in pairs of heads and
      // stored into rows rowA / rowB of P^T (128-byte rows, 16-byte chunks
      // swizzled by row & 7; rowA and rowB share row & 7).
      {
        const uint32_t pbase = tc::smem_u32(ps) + buf * kPBytes + 4 * cq;
        const uint32_t swz = rowA & 7;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float2 mr = *reinterpret_cast<const float2 *>(&sm->mref[8 * c + 2 * cq]);
          // (an invalid row is -inf, and so may mref be while no valid row has been seen)
          const float pa0 = validA ? ex2_approx(__uint_as_float(v[4 * c]) - mr.x) : 0.f;
          const float pa1 = validA ? ex2_approx(__uint_as_float(v[4 * c + 1]) - mr.y) : 0.f;
          const float pb0 = validB ? ex2_approx(__uint_as_float(v[4 * c + 2]) - mr.x) : 0.f;
          const float pb1 = validB ? ex2_approx(__uint_as_float(v[4 * c + 3]) - mr.y) : 0.f;
          __nv_bfloat162 ta = __floats2bfloat162_rn(pa0, pa1), tb = __floats2bfloat162_rn(pb0, pb1);
          // the sums take the same bf16 weights as P.V, so that a dominant
          // row's weight (up to 2^8 between rescales) cancels exactly
          const float2 fa = __bfloat1622float2(ta), fb = __bfloat1622float2(tb);
          l[2 * c] += fa.x + fb.x;
          l[2 * c + 1] += fa.y + fb.y;
          const uint32_t off = (uint32_t)((c ^ swz) << 4);
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(pbase + rowA * 128 + off), "r"(*reinterpret_cast<uint32_t *>(&ta))
                       : "memory");
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(pbase + rowB * 128 + off), "r"(*reinterpret_cast<uint32_t *>(&tb))
                       : "memory");
        }
      }
      if (li > 0 && rescale) {
        // O^T is rescaled in TMEM: P.V of the previous tile must be complete
        // first. (Only then: S^T(li) completing implied every earlier P.V
        // but that one, and a P(li) that needs no rescale does not wait. One
        // barrier per tile slot mod 4, so a skipped phase is never mistaken
        // for another: slot (li - 1) mod 4 next completes for tile li + 3.)
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&sm->pv_done[(li - 1) & 3], ((li - 1) >> 2) & 1, abort, a.status, lim));
        tc::fence_after_sync();
        if (ok) {
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              uint32_t v[32];
              const uint32_t ta = tmem + lane_off + kColO + 64 * m + 32 * half;
              tc::tmem_ld32(ta, v);
              tc::tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * sm->alpha[32 * half + c]);
              tmem_st32(ta, v);
            }
          }
          tmem_st_wait();
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc::fence_before_sync();
      tc::mbar_arrive(&sm->p_full[buf]);
    }
    // ---- epilogue: per-head sums, then O (partials, or the final output)
    if (!waited) pdl_wait();  // (no global write before the previous kernel is done)
    ok = __all_sync(0xffffffffu, ok && (ntiles == 0 || tc::mbar_wait(&sm->o_done, 0, abort, a.status, lim)));
    tc::fence_after_sync();
#pragma unroll
    for (int o = 4; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < 16; ++i) l[i] += __shfl_xor_sync(0xffffffffu, l[i], o);
    if (rq == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int e = 0; e < 2; ++e) sm->red[quarter][8 * c + 2 * cq + e] = l[2 * c + e];
    }
    ok = !bar_any(1, 128, !ok);  // every softmax warp takes the same branch below
    if (leader) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int h = 2 * lane + i;
        sm->lsum[h] = (sm->red[0][h] + sm->red[1][h]) + (sm->red[2][h] + sm->red[3][h]);
      }
    }
    named_sync(1, 128);
    const int orow = quarter * 32 + lane;  // O^T row (dims) within a 128-dim chunk
    if (splits > 1) {
      // This split's unnormalised O (fp32, [64 heads][512 dims]) and its
      // (mref, lsum) go to the workspace, for the cluster merge below.
      const size_t pidx = (size_t)qv * splits + split;
      if (leader) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int h = 2 * lane + i;
          part_ml[(pidx * 2) * kH + h] = sm->mref[h];
          part_ml[(pidx * 2 + 1) * kH + h] = sm->lsum[h];
        }
      }
      float *po = part_o + pidx * (size_t)kH * kD;
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + orow;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          if (ok && ntiles > 0) {
            tc::tmem_ld32(tmem + lane_off + kColO + 64 * m + 32 * half, v);
            tc::tmem_ld_wait();
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = 0u;
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) po[(size_t)(32 * half + c) * kD + d] = __uint_as_float(v[c]);
        }
      }
    } else if (ok) {
      // One split: fold in the sink (logit sink[h], value 0) and normalise.
      if (leader) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int h = 2 * lane + i;
          const float mr = sm->mref[h], sk = a.sink[hg * kH + h] * kLog2e;
          const float M = fmaxf(mr, sk);
          const float wm = mr == -INFINITY ? 0.f : exp2f(mr - M);
          sm->alpha[h] = wm / (sm->lsum[h] * wm + exp2f(sk - M));
        }
      }
      named_sync(1, 128);
      bf16 *out = static_cast<bf16 *>(a.out) + (size_t)qv * kH * kD;
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + orow;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          tc::tmem_ld32(tmem + lane_off + kColO + 64 * m + 32 * half, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c)
            out[(size_t)(32 * half + c) * kD + d] = __float2bfloat16_rn(__uint_as_float(v[c]) * sm->alpha[32 * half + c]);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  if (splits > 1 && cluster_merge) {
    // The splits of query qq are the blocks of one cluster (rank = split):
    // the cluster barrier orders every split's partials (global memory) before
    // the merge. Every block merges 1/splits of the outputs with the sink:
    //   M = max(max_s m_s, sink), L = sum_s l_s 2^(m_s - M) + 2^(sink - M),
    //   out = sum_s O_s 2^(m_s - M) / L   (m and sink in log2 units).
    cluster_sync();
    float *coef = reinterpret_cast<float *>(ps);  // [splits][64]: 2^(m_s - M) / L
    const float *pml = part_ml + (size_t)qv * splits * 2 * kH;
    if (threadIdx.x < kH) {
      const int h = threadIdx.x;
      float mr[kMaxSplits], lr[kMaxSplits];
#pragma unroll
      for (int r = 0; r < kMaxSplits; ++r)
        if (r < splits) {
          mr[r] = pml[(2 * r) * kH + h];
          lr[r] = pml[(2 * r + 1) * kH + h];
        }
      const float sk = a.sink[hg * kH + h] * kLog2e;
      float M = sk;
#pragma unroll
      for (int r = 0; r < kMaxSplits; ++r)
        if (r < splits) M = fmaxf(M, mr[r]);
      float Lsum = exp2f(sk - M), w[kMaxSplits];
#pragma unroll
      for (int r = 0; r < kMaxSplits; ++r)
        if (r < splits) {
          w[r] = mr[r] == -INFINITY ? 0.f : exp2f(mr[r] - M);
          Lsum += lr[r] * w[r];
        }
      const float inv = 1.f / Lsum;
#pragma unroll
      for (int r = 0; r < kMaxSplits; ++r)
        if (r < splits) coef[r * kH + h] = w[r] * inv;
    }
    __syncthreads();
    const float *po = part_o + (size_t)qv * splits * kH * kD;
    bf16 *out = static_cast<bf16 *>(a.out) + (size_t)qv * kH * kD;
    constexpr int kGroups = kH * kD / 4;  // 4-dim groups of the output
    const int g0 = split * kGroups / splits, g1 = (split + 1) * kGroups / splits;
    // Batches of groups with every partial load in flight before the sums
    // (a group at a time waits out one L2 latency per group).
    if (splits <= 4)
      merge_groups<4, 4>(po, coef, out, splits, g0, g1);
    else if (splits <= 8)
      merge_groups<2, 8>(po, coef, out, splits, g0, g1);
    else
      merge_groups<1, kMaxSplits>(po, coef, out, splits, g0, g1);
  }
}

// Merge of the split partials when the splits of a query are not one
// cluster (more splits than cluster residency allows): one block per
// (query, head); thread t owns dims 4t..4t+3 and issues the loads of all
// splits at once. Same formula as the in-kernel merge.
__global__ void __launch_bounds__(128) mqa_combine_kernel(const float *part_o, const float *part_ml,
                                                          const float *sink, bf16 *out, int splits, int G) {
  extern __shared__ float w[];  // [splits] weights, then [2][splits] (m, l)
  const int qq = blockIdx.x, h = blockIdx.y;  // qq: a group of 64 heads of query qq / G
  pdl_wait();
  pdl_release();
  float *ml = w + splits;
  for (int i = threadIdx.x; i < 2 * splits; i += blockDim.x) {
    const int which = i / splits, sp = i - which * splits;
    ml[i] = part_ml[(((size_t)qq * splits + sp) * 2 + which) * kH + h];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const float sk = sink[(qq % G) * kH + h] * kLog2e;
    float M = sk;
    for (int sp = 0; sp < splits; ++sp) M = fmaxf(M, ml[sp]);
    float Lsum = exp2f(sk - M);
    for (int sp = 0; sp < splits; ++sp) {
      const float ww = ml[sp] == -INFINITY ? 0.f : exp2f(ml[sp] - M);
      w[sp] = ww;
      Lsum += ml[splits + sp] * ww;
    }
    const float inv = 1.f / Lsum;
    for (int sp = 0; sp < splits; ++sp) w[sp] *= inv;
  }
  __syncthreads();
  const int d = 4 * threadIdx.x;
  const float *src = part_o + ((size_t)qq * splits * kH + h) * kD + d;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int sp = 0; sp < splits; ++sp) {
    const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + (size_t)sp * kH * kD));
    const float ww = w[sp];
    acc.x = fmaf(ww, v.x, acc.x);
    acc.y = fmaf(ww, v.y, acc.y);
    acc.z = fmaf(ww, v.z, acc.z);
    acc.w = fmaf(ww, v.w, acc.w);
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
  *reinterpret_cast<uint2 *>(out + ((size_t)qq * kH + h) * kD + d) =
      make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
}

int num_sms_cached() { return device_sm_count(); }

void set_kernel_attributes() {
  static DeviceOnce attr;
  once_per_device(attr, [] {
    for (auto kern : {mqa_tc_kernel<false>, mqa_tc_kernel<true>}) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    }
  });
}

// How many clusters of `size` CTAs of this kernel the GPU holds at once
// (one CTA per SM, and a cluster must fit in one GPC).
int max_active_clusters(int size) {
  static std::atomic<int> cache[kMaxDevices][kMaxSplits + 1];  // per device: 0 unknown, -1 none
  if (size < 1 || size > kMaxSplits) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  int c = cache[dev][size].load(std::memory_order_relaxed);
  if (c == 0) {
    set_kernel_attributes();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(size, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = size;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    // (both instantiations: one block per SM, the same shared memory)
    if (cudaOccupancyMaxActiveClusters(&n, mqa_tc_kernel<false>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    c = n > 0 ? n : -1;
    cache[dev][size].store(c, std::memory_order_relaxed);
  }
  return c > 0 ? c : 0;
}

// Split query rows into runs of whole tiles. Preferred: the largest
// cluster size (up to SMs / Q and 16) for which all Q clusters are resident
// at once, merged inside the kernel. When cluster residency caps the splits
// well below SMs / Q (1.25x or more), the splits are plain blocks instead and
// a combine kernel merges them.
void plan_splits(int Q, int rows_max, int *splits, int *tiles_per_split, bool *cluster_merge) {
  const int tiles = (rows_max + kRows - 1) / kRows;
  int hi = num_sms_cached() / (Q > 0 ? Q : 1);
  hi = hi > kMaxSplits ? kMaxSplits : hi;
  hi = hi > tiles ? tiles : hi;
  int cl = 1, cl_tps = tiles > 0 ? tiles : 1;
  for (int s = hi; s >= 2; --s) {
    const int tps = (tiles + s - 1) / s;
    const int sp = (tiles + tps - 1) / tps;
    if (sp >= 2 && max_active_clusters(sp) >= Q) {
      cl = sp;
      cl_tps = tps;
      break;
    }
  }
  int fr = 1, fr_tps = tiles > 0 ? tiles : 1;
  if (hi >= 2) {
    fr_tps = (tiles + hi - 1) / hi;
    fr = (tiles + fr_tps - 1) / fr_tps;
  }
  if (fr >= 2 && 4 * fr >= 5 * cl) {
    *splits = fr;
    *tiles_per_split = fr_tps;
    *cluster_merge = false;
  } else {
    *splits = cl;
    *tiles_per_split = cl_tps;
    *cluster_merge = cl > 1;
  }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool tc_shape(const MqaArgs &a) {
  return a.dtype == CSA_DTYPE_BF16 && (a.H == kH || a.H == 2 * kH) && a.D == kD &&
         (long long)a.Q * (a.H / kH) <= 65535 && aligned16(a.q) &&
         aligned16(a.kv_cmp) && aligned16(a.kv_win) && aligned16(a.out);
}

// Rows of the longest row list: the window padded to whole tiles, then the
// compressed rows (window_on_top: the compressed rows alone, which the split
// plan covers; split 0 takes the window tiles on top).
int rows_max_of(const MqaArgs &a, bool window_on_top) {
  const int nsel = (a.idx || a.scores) ? a.k : a.N_max;
  return window_on_top ? nsel : (a.win_len + kRows - 1) / kRows * kRows + nsel;
}

}  // namespace

// Upper bound on the split partials for any row list of at most rows_max
// rows (+3 rows of padding): Q x min(tiles, SMs / Q, 16) x 64 x (512 + 2) fp32.
size_t mqa_tc_partial_bytes(int Q, int H, int D, int rows_max) {
  if ((H != kH && H != 2 * kH) || D != kD || Q < 1) return 0;
  Q *= H / kH;  // one row list per group of 64 heads
  const int tiles = (rows_max + kRows + kRows - 1) / kRows;  // (+ the window's padding to whole tiles)
  int s = num_sms_cached() / Q;
  s = s > kMaxSplits ? kMaxSplits : s;
  s = s < 1 ? 1 : (s > tiles ? tiles : s);
  if (s <= 1) return 0;
  return (size_t)Q * s * kH * (kD + 2) * sizeof(float);
}

namespace {

cudaError_t launch_tc(const MqaArgs &a, cudaStream_t stream, bool *taken) {
  *taken = false;
  if (!tc_shape(a)) return cudaSuccess;
  int splits, tps;
  bool cluster_merge;
  const int G = a.H / kH, QV = a.Q * G;  // blocks per split: one per group of 64 heads of a query
  const bool window_on_top = a.early && !a.scores && a.idx;  // see split_tiles
  plan_splits(QV, rows_max_of(a, window_on_top), &splits, &tps, &cluster_merge);
  // In-kernel selection: the splits of a query must be one cluster, and each
  // block's slice of the scores must fit in its tile buffers.
  if (a.scores && (!cluster_merge || a.k > kSelMax || (((a.N_max + splits - 1) / splits + 31) & ~31) > kSelKeys ||
                   !a.idx_out || !a.n_cmp))
    return cudaSuccess;
  CUtensorMap tm_q, tm_cmp_t, tm_win_t;
  const uint64_t cmp_rows = (uint64_t)a.B * a.N_max, win_rows = (uint64_t)a.B * a.T_raw;
  if (!make_tmap_bf16_2d(&tm_q, a.q, kD, (uint64_t)a.Q * a.H, kD * 2, 64, kH) ||
      !make_tmap_bf16_2d(&tm_cmp_t, a.kv_cmp, kD, cmp_rows, kD * 2, 64, kRows) ||
      !make_tmap_bf16_2d(&tm_win_t, a.kv_win, kD, win_rows, kD * 2, 64, kRows))
    return cudaSuccess;
  const size_t need = splits > 1 ? (size_t)QV * splits * kH * (kD + 2) * sizeof(float) : 0;
  if (need > a.partial_bytes) return cudaSuccess;  // cannot happen with the documented workspace size
  float *part_o = static_cast<float *>(a.partials);
  float *part_ml = part_o + (size_t)QV * splits * kH * kD;
  set_kernel_attributes();
  *taken = true;
  cudaError_t e = launch_pdl_cluster(a.scores ? mqa_tc_kernel<true> : mqa_tc_kernel<false>, dim3(splits, QV), dim3(kThreads), kSmemBytes, stream,
                                     cluster_merge ? (unsigned)splits : 1u, tm_q, tm_cmp_t, tm_win_t, a, splits, tps,
                                     a.scale * kLog2e, part_o, part_ml, (int)cluster_merge);
  if (e != cudaSuccess || splits <= 1 || cluster_merge) return e;
  return launch_pdl(mqa_combine_kernel, dim3(QV, kH), dim3(kD / 4), splits * 3 * sizeof(float), stream,
                    (const float *)part_o, (const float *)part_ml, a.sink, static_cast<bf16 *>(a.out), splits, G);
}

}  // namespace

cudaError_t launch_mqa_tc(const MqaArgs &a, cudaStream_t stream, bool *taken) {
  MqaArgs b = a;
  b.scores = nullptr;
  return launch_tc(b, stream, taken);
}

cudaError_t launch_topk_mqa_tc(const MqaArgs &a, cudaStream_t stream, bool *taken) {
  *taken = false;
  if (!a.scores) return cudaSuccess;
  MqaArgs b = a;
  b.idx = nullptr;
  return launch_tc(b, stream, taken);
}

}  // namespace csa
