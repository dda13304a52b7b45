// A4 / A5 on the tensor cores for the Flash attention shape: 64 query heads,
// one shared KV head, head_dim 512, K = V, bf16 in, fp32 accumulation
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
// TMA loads tile t+2. The MMA thread issues S(t+1) before PV(t).
// An M = 64 accumulator occupies TMEM lanes 0-15 of each 32-lane quarter, so
// each softmax warp owns 16 rows; a row's 64 head logits stay in one thread.
// The per-head tile maximum is a warp transpose-reduction plus a 4-warp
// exchange; the running per-head maximum only moves (and O^T is rescaled in
// TMEM, after the previous P.V has completed) when a tile's maximum exceeds
// it by more than 2^8, so P <= 256 in bf16.
//
// Loads: contiguous runs of 64 rows (HCA entries, window rows) are single TMA
// boxes of 64 rows; top-k rows use TMA tile::gather4 (4 rows per instruction;
// the compressed segment is padded to a multiple of 4 rows so no group mixes
// the compressed cache and the raw window buffer).
//
// Work split: query q's row list is cut into `splits` runs of whole tiles, one
// CTA each. With one split the CTA folds in the sink and writes the output;
// otherwise it writes (m, l, O) partials merged by mqa_combine_kernel.
// Roles (192 threads): warp 0 loads, warp 1 issues the MMAs and owns TMEM,
// warps 2-5 run the softmax and the epilogue. All waits are bounded.
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
constexpr int kThreads = 192;
constexpr int kMmaWarp = 1;
constexpr int kSoftWarp0 = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;                       // O^T chunk m at columns 64m (M = 128 layout)
constexpr uint32_t kColS = 256;                     // S^T buffer j at 256 + 64j (M = 64 layout)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;

struct Small {
  uint64_t q_full, kv_full[2], kv_empty[2], s_full[2], p_full[2], pv_done, o_done;
  float red[4][kH];
  alignas(16) float mref[kH];
  float alpha[kH];
  float lsum[kH];
  uint32_t tmem_base;
  int abort;
  int rescale;
  int need[4];  // per tile (mod 4): some logit exceeded the running maximum by more than 2^8
};

constexpr size_t kSmemBytes = 1024 + 2 * kTileBytes + kQBytes + 2 * kPBytes + sizeof(Small);

// Row list of one query: compressed rows [0, nsel) (padded with unused rows
// up to nsel4, a multiple of 4), then the window rows [nsel4, R).
struct RowList {
  int nsel, nsel4, wlo, R;
};

__device__ __forceinline__ RowList row_list(const MqaArgs &a, int qq, uint32_t *status) {
  RowList L;
  L.nsel = a.idx ? a.k : clamp_count(a.n_cmp[qq], a.N_max, status);
  int e = a.win_end[qq];
  if (e < 0 || e >= a.T_raw) {
    raise_status(status, CSA_STATUS_BAD_WINDOW);
    e = e < 0 ? 0 : a.T_raw - 1;
  }
  L.wlo = max(0, e - a.win_len + 1);
  L.nsel4 = (L.nsel + 3) & ~3;
  L.R = L.nsel4 + (e - L.wlo + 1);
  return L;
}

// TMA row coordinate of list position r: in the compressed cache viewed as
// [B * N_max, 512] when r < nsel4, else in the window buffer viewed as
// [B * T_raw, 512]. Unused and padding positions get a valid row of the same
// tensor (their logits are masked).
__device__ __forceinline__ int row_coord(const MqaArgs &a, const RowList &L, int qq, int b, int r) {
  if (r < L.nsel4) {
    int j = -1;
    if (r < L.nsel) {
      j = a.idx ? a.idx[(size_t)qq * a.k + r] : r;
      if (j < -1 || j >= a.N_max) {
        raise_status(a.status, CSA_STATUS_BAD_INDEX);
        j = -1;
      }
    }
    return b * a.N_max + (j >= 0 ? j : 0);
  }
  return b * a.T_raw + (r < L.R ? L.wlo + (r - L.nsel4) : L.wlo);
}

__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *map, int col, const int (&rc)[4],
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(tc::smem_u32(bar)), "r"(col), "r"(rc[0]), "r"(rc[1]),
        "r"(rc[2]), "r"(rc[3])
      : "memory");
}

// 2^x on the SFU (relative error about 2^-22; flushes subnormal results to
// zero, which only ever meets weights far below the bf16 resolution of P).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// Warp transpose-reduction of 64 per-lane values: afterwards lane l holds the
// reduction over the 32 lanes of heads 2l and 2l+1 in v[0], v[1].
template <bool kMax>
__device__ __forceinline__ void transpose_reduce64(float (&v)[64], int lane) {
#pragma unroll
  for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
    const bool hi = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float send = hi ? v[i] : v[i + n];
      const float keep = hi ? v[i + n] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    mqa_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_cmp_g,
                  const __grid_constant__ CUtensorMap tm_win_g, const __grid_constant__ CUtensorMap tm_cmp_t,
                  const __grid_constant__ CUtensorMap tm_win_t, MqaArgs a, int splits, int tiles_per_split,
                  float scale_log2, float *part_o, float *part_ml) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *kv = smem;                              // [2 tiles][8 boxes][64 rows][128 B]
  uint8_t *qs = smem + 2 * kTileBytes;             // [8 boxes][64 heads][128 B]
  uint8_t *ps = qs + kQBytes;                      // [2][64 rows][128 B]  (P^T, MN-major)
  Small *sm = reinterpret_cast<Small *>(ps + 2 * kPBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, qq = blockIdx.y;
  const int b = qq / a.q_per_seq;

  if (threadIdx.x == 0) {
    tc::mbar_init(&sm->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sm->kv_full[i], 1);
      tc::mbar_init(&sm->kv_empty[i], 1);
      tc::mbar_init(&sm->s_full[i], 1);
      tc::mbar_init(&sm->p_full[i], 4 * 32);
    }
    tc::mbar_init(&sm->pv_done, 1);
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
  pdl_wait();  // inputs (indices, queries, caches) may come from the previous kernel
  pdl_release();

  const RowList L = row_list(a, qq, threadIdx.x == 0 ? a.status : nullptr);
  const int tiles_all = (L.R + kRows - 1) / kRows;
  const int t0 = split * tiles_per_split;
  const int t1 = min(tiles_all, t0 + tiles_per_split);
  const int ntiles = max(0, t1 - t0);

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    const uint32_t kv_base = tc::smem_u32(kv);
    if (lane == 0) {
      tc::prefetch_tmap(&tm_cmp_g);
      tc::prefetch_tmap(&tm_win_g);
      tc::prefetch_tmap(&tm_cmp_t);
      tc::prefetch_tmap(&tm_win_t);
    }
    int issued = 0;
    for (int li = 0; li < ntiles && !*abort; ++li) {
      const int buf = li & 1;
      const int r0 = (t0 + li) * kRows;
      // A tile is one contiguous run when it lies in the window part, or in
      // the compressed part of a dense (HCA) row list.
      const bool win_run = r0 >= L.nsel4;
      const bool cmp_run = !a.idx && r0 + kRows <= L.nsel4;
      int rc[4];
      const CUtensorMap *gmap = &tm_cmp_g;
      if (!win_run && !cmp_run && lane < 16) {
        const int r = r0 + 4 * lane;
#pragma unroll
        for (int i = 0; i < 4; ++i) rc[i] = row_coord(a, L, qq, b, r + i);
        gmap = r < L.nsel4 ? &tm_cmp_g : &tm_win_g;
      }
      const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&sm->kv_empty[buf], ((li >> 1) & 1) ^ 1, abort, a.status));
      if (!ok) break;
      const uint32_t dst = kv_base + buf * kTileBytes;
      if (lane == 0) tc::mbar_arrive_expect_tx(&sm->kv_full[buf], kTileBytes);
      __syncwarp();
      if (win_run || cmp_run) {
        if (lane < 8) {
          const int row = win_run ? b * a.T_raw + L.wlo + (r0 - L.nsel4) : b * a.N_max + r0;
          tc::tma_load_2d(kv + buf * kTileBytes + lane * kBoxBytes, win_run ? &tm_win_t : &tm_cmp_t, 64 * lane, row,
                          &sm->kv_full[buf]);
        }
      } else if (lane < 16) {
#pragma unroll
        for (int bx = 0; bx < 8; ++bx) tma_gather4(dst + bx * kBoxBytes + lane * 512, gmap, 64 * bx, rc, &sm->kv_full[buf]);
      }
      issued = li + 1;
    }
    // Drain: the copies of the last two tiles must have landed before exit.
    if (lane == 0)
      for (int li = max(0, issued - 2); li < issued; ++li) tc::mbar_drain(&sm->kv_full[li & 1], (li >> 1) & 1);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool q_issued = false;
      if (ntiles > 0) {
        tc::prefetch_tmap(&tm_q);
        tc::mbar_arrive_expect_tx(&sm->q_full, kQBytes);
        for (int bx = 0; bx < kD / 64; ++bx)
          tc::tma_load_2d(qs + bx * kQBoxBytes, &tm_q, bx * 64, qq * kH, &sm->q_full);
        q_issued = true;
      }
      constexpr uint32_t idesc_s = tc::idesc_bf16(64, 64, 0, 0);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(128, 64, 1, 1);
      const uint32_t kv_base = tc::smem_u32(kv), q_base = tc::smem_u32(qs), p_base = tc::smem_u32(ps);
      bool ok = ntiles == 0 || tc::mbar_wait(&sm->q_full, 0, abort, a.status);
      auto pv = [&](int t) {  // O^T += V^T(t) P^T(t)
        const int pb = t & 1;
        if (!tc::mbar_wait(&sm->p_full[pb], (t >> 1) & 1, abort, a.status)) return false;
        tc::fence_after_sync();
        const uint64_t ad0 = tc::sw128_desc(kv_base + pb * kTileBytes, kBoxBytes, 1024);
        const uint64_t bd0 = tc::sw128_desc(p_base + pb * kPBytes, kPBytes, 1024);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
#pragma unroll
          for (int j = 0; j < kRows / 16; ++j)
            tc::mma_bf16(tmem + kColO + 64 * m, ad0 + (uint64_t)((2 * m * kBoxBytes + j * 2048) >> 4),
                         bd0 + (uint64_t)((j * 2048) >> 4), idesc_pv, t > 0 || j > 0);
        }
        tc::commit(&sm->kv_empty[pb]);
        tc::commit(&sm->pv_done);
        return true;
      };
      for (int li = 0; ok && li < ntiles; ++li) {
        const int buf = li & 1;
        ok = tc::mbar_wait(&sm->kv_full[buf], (li >> 1) & 1, abort, a.status);
        if (!ok) break;
        tc::fence_after_sync();
        // descriptors differ only in the start-address field (16-byte units)
        const uint64_t ad0 = tc::sw128_desc(kv_base + buf * kTileBytes, 16, 1024);
        const uint64_t bd0 = tc::sw128_desc(q_base, 16, 1024);
#pragma unroll
        for (int j = 0; j < kD / 16; ++j)
          tc::mma_bf16(tmem + kColS + 64 * buf, ad0 + (uint64_t)(((j >> 2) * kBoxBytes + (j & 3) * 32) >> 4),
                       bd0 + (uint64_t)(((j >> 2) * kQBoxBytes + (j & 3) * 32) >> 4), idesc_s, j > 0);
        tc::commit(&sm->s_full[buf]);
        if (li > 0) ok = pv(li - 1);
      }
      if (ok && ntiles > 0) pv(ntiles - 1);
      tc::commit(&sm->o_done);
      tc::mbar_drain(&sm->o_done, 0);
      if (q_issued) tc::mbar_drain(&sm->q_full, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 16 + lane;                 // S^T row (lanes 0-15 of the quarter)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool leader = warp == kSoftWarp0;
    float l[kH];
#pragma unroll
    for (int h = 0; h < kH; ++h) l[h] = 0.f;
    bool ok = true;
    int idx_next = 0;
    {
      const int r = t0 * kRows + row;
      if (ntiles > 0 && lane < 16 && a.idx && r < L.nsel) idx_next = a.idx[(size_t)qq * a.k + r];
    }
    for (int li = 0; li < ntiles; ++li) {
      const int buf = li & 1;
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&sm->s_full[buf], (li >> 1) & 1, abort, a.status));
      if (!ok) break;
      tc::fence_after_sync();
      const int r = (t0 + li) * kRows + row;
      bool valid = lane < 16;
      if (valid) valid = r < L.nsel4 ? (r < L.nsel && (!a.idx || (idx_next >= 0 && idx_next < a.N_max))) : r < L.R;
      if (li + 1 < ntiles && lane < 16) {  // the next tile's index, loaded while this tile is processed
        const int rn = r + kRows;
        idx_next = (a.idx && rn < L.nsel) ? a.idx[(size_t)qq * a.k + rn] : 0;
      }
      const uint32_t sbase = tmem + lane_off + kColS + 64 * buf;
      uint32_t v0[32], v1[32];
      tc::tmem_ld32(sbase, v0);
      tc::tmem_ld32(sbase + 32, v1);
      tc::tmem_ld_wait();
      // Fast path: the running per-head maximum moves only when some logit
      // of the tile exceeds it by more than 2^8 (always on the first tile).
      bool over = false;
      if (valid) {
#pragma unroll
        for (int h = 0; h < kH; h += 4) {
          const float4 mr = *reinterpret_cast<const float4 *>(&sm->mref[h]);
          const float mm[4] = {mr.x, mr.y, mr.z, mr.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float x = __uint_as_float(h + i < 32 ? v0[h + i] : v1[h + i - 32]) * scale_log2;
            over |= x > mm[i] + kRescaleLog2;
          }
        }
      }
      if (leader && lane == 0) sm->need[(li + 2) & 3] = 0;  // slot of tile li + 2, last read at tile li - 2
      if (__any_sync(0xffffffffu, over) && lane == 0) atomicOr(&sm->need[li & 3], 1);
      named_sync(1, 128);
      bool rescale = false;
      if (sm->need[li & 3] != 0) {
        {
          float red[kH];
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            red[h] = valid ? __uint_as_float(v0[h]) * scale_log2 : -INFINITY;
            red[h + 32] = valid ? __uint_as_float(v1[h]) * scale_log2 : -INFINITY;
          }
          transpose_reduce64<true>(red, lane);
          sm->red[quarter][2 * lane] = red[0];
          sm->red[quarter][2 * lane + 1] = red[1];
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
          for (int h = 0; h < kH; ++h) l[h] *= sm->alpha[h];
        }
        tc::tmem_ld32(sbase, v0);  // the logits again (registers were released for the reduction)
        tc::tmem_ld32(sbase + 32, v1);
        tc::tmem_ld_wait();
      }
      // P = 2^(x - mref), summed per head, packed to bf16 into P^T row `row`.
      uint32_t pk[32];
#pragma unroll
      for (int h = 0; h < kH; h += 4) {
        const float4 mr = *reinterpret_cast<const float4 *>(&sm->mref[h]);
        const float mm[4] = {mr.x, mr.y, mr.z, mr.w};
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float x = fmaf(__uint_as_float(h + i < 32 ? v0[h + i] : v1[h + i - 32]), scale_log2, -mm[i]);
          p[i] = valid ? ex2_approx(x) : 0.f;
          l[h + i] += p[i];
        }
        __nv_bfloat162 t0 = __floats2bfloat162_rn(p[0], p[1]), t1 = __floats2bfloat162_rn(p[2], p[3]);
        pk[h >> 1] = *reinterpret_cast<uint32_t *>(&t0);
        pk[(h >> 1) + 1] = *reinterpret_cast<uint32_t *>(&t1);
      }
      if (lane < 16) {
        const uint32_t prow = tc::smem_u32(ps) + buf * kPBytes + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t addr = prow + ((c ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * c]), "r"(pk[4 * c + 1]),
                       "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                       : "memory");
        }
      }
      if (li > 0) {
        // P.V of the previous tile must be complete before O^T may be
        // touched; consumed every tile so the barrier phases stay in step.
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&sm->pv_done, (li - 1) & 1, abort, a.status));
        if (!ok) break;
        tc::fence_after_sync();
        if (rescale) {
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
    ok = __all_sync(0xffffffffu, ok && (ntiles == 0 || tc::mbar_wait(&sm->o_done, 0, abort, a.status)));
    tc::fence_after_sync();
    transpose_reduce64<false>(l, lane);
    sm->red[quarter][2 * lane] = l[0];
    sm->red[quarter][2 * lane + 1] = l[1];
    named_sync(1, 128);
    if (leader) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int h = 2 * lane + i;
        sm->lsum[h] = (sm->red[0][h] + sm->red[1][h]) + (sm->red[2][h] + sm->red[3][h]);
      }
    }
    named_sync(1, 128);
    const int orow = quarter * 32 + lane;  // O^T row (dims) within a 128-dim chunk
    const size_t pidx = (size_t)qq * splits + split;
    if (ok && splits > 1) {
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
          if (ntiles > 0) {
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
          const float mr = sm->mref[h], sk = a.sink[h] * kLog2e;
          const float M = fmaxf(mr, sk);
          const float wm = mr == -INFINITY ? 0.f : exp2f(mr - M);
          sm->alpha[h] = wm / (sm->lsum[h] * wm + exp2f(sk - M));
        }
      }
      named_sync(1, 128);
      bf16 *out = static_cast<bf16 *>(a.out) + (size_t)qq * kH * kD;
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
}

// Merge the split partials of each query with the sink:
//   M = max(max_s m_s, sink), L = sum_s l_s 2^(m_s - M) + 2^(sink - M),
//   out = sum_s O_s 2^(m_s - M) / L   (m and sink in log2 units).
// One block per (query, head); thread t owns dims 4t..4t+3 and issues the
// loads of all splits at once.
__global__ void __launch_bounds__(128) mqa_combine_kernel(const float *part_o, const float *part_ml,
                                                          const float *sink, bf16 *out, int splits) {
  extern __shared__ float w[];  // [splits] weights, then [2][splits] (m, l)
  const int qq = blockIdx.x, h = blockIdx.y;
  pdl_wait();
  pdl_release();
  float *ml = w + splits;
  for (int i = threadIdx.x; i < 2 * splits; i += blockDim.x) {
    const int which = i / splits, s = i - which * splits;
    ml[i] = part_ml[(((size_t)qq * splits + s) * 2 + which) * kH + h];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const float sk = sink[h] * kLog2e;
    float M = sk;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, ml[s]);
    float Lsum = exp2f(sk - M);
    for (int s = 0; s < splits; ++s) {
      const float ww = ml[s] == -INFINITY ? 0.f : exp2f(ml[s] - M);
      w[s] = ww;
      Lsum += ml[splits + s] * ww;
    }
    const float inv = 1.f / Lsum;
    for (int s = 0; s < splits; ++s) w[s] *= inv;
  }
  __syncthreads();
  const int d = 4 * threadIdx.x;
  const float *src = part_o + ((size_t)qq * splits * kH + h) * kD + d;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int s = 0; s < splits; ++s) {
    const float4 v = *reinterpret_cast<const float4 *>(src + (size_t)s * kH * kD);
    const float ww = w[s];
    acc.x = fmaf(ww, v.x, acc.x);
    acc.y = fmaf(ww, v.y, acc.y);
    acc.z = fmaf(ww, v.z, acc.z);
    acc.w = fmaf(ww, v.w, acc.w);
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 pk = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
  *reinterpret_cast<uint2 *>(out + ((size_t)qq * kH + h) * kD + d) = pk;
}

int num_sms_cached() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

void plan_splits(int Q, int rows_max, int *splits, int *tiles_per_split) {
  const int tiles = (rows_max + kRows - 1) / kRows;
  int s = num_sms_cached() / (Q > 0 ? Q : 1);
  s = s < 1 ? 1 : (s > tiles ? tiles : s);
  const int tps = (tiles + s - 1) / s;
  *tiles_per_split = tps;
  *splits = (tiles + tps - 1) / tps;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool tc_shape(const MqaArgs &a) {
  return a.dtype == CSA_DTYPE_BF16 && a.H == kH && a.D == kD && a.Q <= 65535 && aligned16(a.q) &&
         aligned16(a.kv_cmp) && aligned16(a.kv_win) && aligned16(a.out);
}

int rows_max_of(const MqaArgs &a) { return (((a.idx ? a.k : a.N_max) + 3) & ~3) + a.win_len; }

}  // namespace

size_t mqa_tc_partial_bytes(int Q, int H, int D, int rows_max) {
  if (H != kH || D != kD || Q < 1) return 0;
  // Upper bound on the split count the launcher can pick for any row list of
  // at most rows_max rows (+3 rows of padding): min(tiles, SMs / Q).
  const int tiles = (rows_max + 3 + kRows - 1) / kRows;
  int s = num_sms_cached() / Q;
  s = s < 1 ? 1 : (s > tiles ? tiles : s);
  if (s <= 1) return 0;
  return (size_t)Q * s * kH * (kD + 2) * sizeof(float);
}

cudaError_t launch_mqa_tc(const MqaArgs &a, cudaStream_t stream, bool *taken) {
  *taken = false;
  if (!tc_shape(a)) return cudaSuccess;
  int splits, tps;
  plan_splits(a.Q, rows_max_of(a), &splits, &tps);
  const size_t need = splits > 1 ? (size_t)a.Q * splits * kH * (kD + 2) * sizeof(float) : 0;
  if (need > a.partial_bytes) return cudaSuccess;  // cannot happen with the documented workspace size
  CUtensorMap tm_q, tm_cmp_g, tm_win_g, tm_cmp_t, tm_win_t;
  const uint64_t cmp_rows = (uint64_t)a.B * a.N_max, win_rows = (uint64_t)a.B * a.T_raw;
  if (!make_tmap_bf16_2d(&tm_q, a.q, kD, (uint64_t)a.Q * kH, kD * 2, 64, kH) ||
      !make_tmap_bf16_2d(&tm_cmp_g, a.kv_cmp, kD, cmp_rows, kD * 2, 64, 1) ||
      !make_tmap_bf16_2d(&tm_win_g, a.kv_win, kD, win_rows, kD * 2, 64, 1) ||
      !make_tmap_bf16_2d(&tm_cmp_t, a.kv_cmp, kD, cmp_rows, kD * 2, 64, kRows) ||
      !make_tmap_bf16_2d(&tm_win_t, a.kv_win, kD, win_rows, kD * 2, 64, kRows))
    return cudaSuccess;
  float *part_o = static_cast<float *>(a.partials);
  float *part_ml = part_o + (size_t)a.Q * splits * kH * kD;
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(mqa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    attr_set = true;
  }
  dim3 grid(splits, a.Q);
  *taken = true;
  cudaError_t e = launch_pdl(mqa_tc_kernel, grid, dim3(kThreads), kSmemBytes, stream, tm_q, tm_cmp_g, tm_win_g, tm_cmp_t,
                             tm_win_t, a, splits, tps, a.scale * kLog2e, part_o, part_ml);
  if (e != cudaSuccess || splits <= 1) return e;
  return launch_pdl(mqa_combine_kernel, dim3(a.Q, kH), dim3(kD / 4), splits * 3 * sizeof(float), stream,
                    (const float *)part_o, (const float *)part_ml, a.sink, static_cast<bf16 *>(a.out), splits);
}

}  // namespace csa
