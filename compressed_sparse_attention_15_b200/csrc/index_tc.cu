// A2 on the tensor cores for the Flash indexer shape (64 heads x 128 dims):
// s[q,j] = sum_h wi[q,h] * max(0, qi[q,h] . ki[b,j])
// ("DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1, Indexer;
// index_n_heads = 64, index_head_dim = 128 in the model card's config.json).
// Two element formats: bf16 (kind::f16 MMAs, K = 16), and FP8 E4M3 codes
// with per-row scales (kind::f8f6f4 MMAs, K = 32; quantization_config fmt
// e4m3 of "deepseek-ai/DeepSeek-V4-Flash-0731"): with qi = sq * codes and
// ki = sk * codes, s[q,j] = sk[j] * sum_h (wi[q,h] sq[q,h]) max(0, acc[h]),
// acc being the code-by-code product (all scales positive).
//
// Layout of the contraction: the compressed keys are the MMA's M dimension
// (128 entries per tile), the 64 heads its N, the 128 dims its K. One tile is
// 8 tcgen05.mma (M128 N64 K16) into a 128-lane x 64-column fp32 TMEM
// accumulator, so each epilogue thread owns one entry's 64 head products and
// the weighted ReLU sum over heads is thread-local.
//
// Pipeline (persistent, one CTA per SM; 192 threads, 320 for E4M3, 576 for
// query groups):
//   warp 0      TMA producer: 32 KB key tiles (128 bf16 / 256 FP8 entries)
//               into a 5-stage ring, and the query's head block (16 / 8 KB)
//               into one of two query slots;
//   warp 1      MMA issuer (one thread) and TMEM owner (2 accumulators);
//   warps 2..   epilogue, one per TMEM lane quarter and 128-entry row block
//               (4 warps; 8 for the two blocks of an E4M3 tile, 16 for the
//               4 queries of a group): tcgen05.ld, ReLU, weighted sum,
//               coalesced store.
// Each CTA walks a contiguous range of the flat (query, tile) space. Every
// wait is bounded; a timeout raises CSA_STATUS_WAIT_TIMEOUT, all roles stop,
// in-flight copies and MMAs are drained (bounded) and TMEM is freed.
//
// Prefill (several queries per sequence, bf16): kG = 4 queries of one
// sequence share each key tile. Their 4 x 64 heads are the MMA's N (256):
// one tile load and one M128 N256 product per 4 queries instead of four of
// each, so the kernel becomes tensor-bound instead of tile-bound. The four
// head blocks take 64 KB, so there is one query slot (a new group's block
// loads once the last group's MMAs are done) and four key stages.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace csa {

namespace {

constexpr int kHi = 64, kDi = 128;


// Per element format: a stage is 32 KB of keys in two TMA boxes of 128 rows x
// 128 bytes (the swizzle span): bf16 tiles are 128 entries split along the
// dims (64 + 64), E4M3 tiles are 256 entries split along the rows (128 +
// 128, one MMA row block each), so both formats pay the per-tile costs
// (barriers, MMA issue, epilogue hand-off) once per 32 KB.
template <bool kFp8, int kG>
struct Fmt {
  static_assert(kG == 1 || (kG == 4 && !kFp8), "query groups: bf16 only");
  static constexpr int kElem = kFp8 ? 1 : 2;
  static constexpr int kStages = kG == 1 ? 5 : 4;
  static constexpr int kQSlots = kG == 1 ? 2 : 1;
  static constexpr int kSub = kFp8 ? 2 : 1;                // 128-row MMA blocks per tile
  static constexpr int kTileRows = 128 * kSub;
  static constexpr int kKBoxes = kFp8 ? 1 : 2;             // 128-byte K boxes per row (query block too)
  static constexpr int kKSteps = kFp8 ? 4 : 8;             // MMAs per row block (32 bytes of K each)
  static constexpr uint32_t kBoxBytes = 128 * 128;         // 16 KB
  static constexpr uint32_t kTileBytes = 2 * kBoxBytes;    // 32 KB
  static constexpr uint32_t kQBytes = kG * kHi * kDi * kElem;  // one query group's head blocks
  static constexpr uint32_t kQBox = kQBytes / kKBoxes;      // 8 KB (32 KB for 4 queries)
  static constexpr uint32_t kAccCols = 64 * kSub * kG;     // TMEM columns of one accumulator
  static constexpr uint32_t kTmemCols = 2 * kAccCols;
  static constexpr uint32_t kIdesc = kFp8 ? tc::idesc_e4m3(128, 64) : tc::idesc_bf16(128, 64 * kG, 0, 0);
  // Epilogue warps: one per TMEM lane quarter and row block, so that each
  // warp reduces one 128-entry block of a tile (E4M3 tiles hold two); for
  // query groups one per lane quarter and query of the group.
  static constexpr int kEpiWarps = 4 * kSub * (kG > 1 ? kG : 1);
  static constexpr int kThreads = 32 * (2 + kEpiWarps);
  // per epilogue warp: its group's head weights and visible counts
  static constexpr uint32_t kWBytes = kG == 1 ? 0 : kEpiWarps * (kG * kHi * 4 + kG * 4);
};

template <int kStages>
struct Bars {
  uint64_t full[kStages], empty[kStages], qfull[2], qempty[2], accfull[2], accempty[2], mma_done;
  uint32_t tmem_base;
  int abort;
};

template <bool kFp8, int kG>
constexpr size_t smem_bytes() {
  using F = Fmt<kFp8, kG>;
  return 1024 + F::kStages * F::kTileBytes + F::kQSlots * F::kQBytes + F::kWBytes + sizeof(Bars<F::kStages>);
}
static_assert(smem_bytes<false, 1>() <= 227 * 1024 && smem_bytes<true, 1>() <= 227 * 1024 &&
                  smem_bytes<false, 4>() <= 227 * 1024,
              "shared memory per block");

struct Tile {
  int q, j0;
};

// Tile t of the flat (query group, 128-entry tile) space (q: the group). Every tile of a query's
// row is loaded and multiplied; entries at or past the query's visible count
// are only masked in the epilogue, so that no role waits on that count
// before its first copy or MMA.
__device__ __forceinline__ Tile tile_of(long long t, int tiles_per_q, int tile_rows) {
  Tile r;
  r.q = (int)(t / tiles_per_q);
  r.j0 = (int)(t - (long long)r.q * tiles_per_q) * tile_rows;
  return r;
}

template <bool kFp8, int kG>
__global__ void __launch_bounds__(Fmt<kFp8, kG>::kThreads, 1)
    index_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_ki, const __grid_constant__ CUtensorMap tm_qi,
                           ScoreArgs a, int tiles_per_q, long long total, long long per_cta) {
  using F = Fmt<kFp8, kG>;
  constexpr int kStages = F::kStages;
  constexpr uint32_t kTileBytes = F::kTileBytes, kQBytes = F::kQBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stage_buf = smem;
  uint8_t *q_buf = smem + kStages * kTileBytes;
  float *w_buf = reinterpret_cast<float *>(q_buf + F::kQSlots * kQBytes);  // kG > 1: [epilogue warp][kG x 64 + kG]
  Bars<kStages> *bars = reinterpret_cast<Bars<kStages> *>(q_buf + F::kQSlots * kQBytes + F::kWBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long t_begin = (long long)blockIdx.x * per_cta;
  const long long t_end = min(total, t_begin + per_cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->qfull[s], 1);
      tc::mbar_init(&bars->qempty[s], 1);
      tc::mbar_init(&bars->accfull[s], 1);
      tc::mbar_init(&bars->accempty[s], F::kEpiWarps * 32);
    }
    tc::mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(&bars->tmem_base, F::kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abort = &bars->abort;
  pdl_wait();  // inputs may come from the previous kernel in the stream
  pdl_release();
  const uint64_t lim = tc::wait_limit_of(a.status);

  if (warp == 0) {
    if (lane == 0) {
      tc::prefetch_tmap(&tm_ki);
      tc::prefetch_tmap(&tm_qi);
      int stage = 0, nq = 0, cur_q = -1;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // per stage: a load was issued, with this parity
      for (long long t = t_begin; t < t_end && !*abort; ++t) {
        const Tile tl = tile_of(t, tiles_per_q, F::kTileRows);
        if (tl.q != cur_q) {
          const int slot = nq % F::kQSlots;
          const uint32_t qph = (nq / F::kQSlots) & 1;
          if (!tc::mbar_wait(&bars->qempty[slot], qph ^ 1, abort, a.status, lim)) break;
          tc::mbar_arrive_expect_tx(&bars->qfull[slot], kQBytes);
          for (int bx = 0; bx < F::kKBoxes; ++bx)
            tc::tma_load_2d(q_buf + slot * kQBytes + bx * F::kQBox, &tm_qi, bx * 64, tl.q * kG * kHi,
                            &bars->qfull[slot]);
          ++nq;
          cur_q = tl.q;
        }
        if (!tc::mbar_wait(&bars->empty[stage], phase ^ 1, abort, a.status, lim)) break;
        tc::mbar_arrive_expect_tx(&bars->full[stage], kTileBytes);
        const int row = (tl.q * kG / a.q_per_seq) * a.N_max + tl.j0;
        for (int bx = 0; bx < 2; ++bx)  // bf16: dims 64 bx.., E4M3: rows 128 bx..
          tc::tma_load_2d(stage_buf + stage * kTileBytes + bx * F::kBoxBytes, &tm_ki, kFp8 ? 0 : 64 * bx,
                          kFp8 ? row + 128 * bx : row, &bars->full[stage]);
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      // Drain: every load issued must have landed before the CTA may exit.
      // A phase that was already consumed completes the wait at once.
      for (int s = 0; s < kStages; ++s)
        if (issued_mask & (1u << s)) tc::mbar_drain(&bars->full[s], (issued_phase >> s) & 1);
      for (int i = nq - 1; i >= 0 && i >= nq - F::kQSlots; --i)
        tc::mbar_drain(&bars->qfull[i % F::kQSlots], (i / F::kQSlots) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = F::kIdesc;
      int stage = 0, acc = 0, nq = 0, cur_q = -1, slot = 0;
      uint32_t phase = 0, accph = 0;
      for (long long t = t_begin; t < t_end && !*abort; ++t) {
        const Tile tl = tile_of(t, tiles_per_q, F::kTileRows);
        if (tl.q != cur_q) {
          if (cur_q >= 0) tc::commit(&bars->qempty[slot]);  // old head block free once its MMAs finish
          slot = nq % F::kQSlots;
          if (!tc::mbar_wait(&bars->qfull[slot], (nq / F::kQSlots) & 1, abort, a.status, lim)) break;
          ++nq;
          cur_q = tl.q;
        }
        if (!tc::mbar_wait(&bars->accempty[acc], accph ^ 1, abort, a.status, lim)) break;
        if (!tc::mbar_wait(&bars->full[stage], phase, abort, a.status, lim)) break;
        tc::fence_after_sync();
        const uint32_t a_base = tc::smem_u32(stage_buf + stage * kTileBytes);
        const uint32_t b_base = tc::smem_u32(q_buf + slot * kQBytes);
#pragma unroll
        for (int sub = 0; sub < F::kSub; ++sub) {
#pragma unroll
          for (int kk = 0; kk < F::kKSteps; ++kk) {  // 32 bytes of K per MMA, 4 per 128-byte box
            const uint32_t box = kFp8 ? sub : (kk >> 2);
            const uint64_t ad = tc::sw128_desc(a_base + box * F::kBoxBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = tc::sw128_desc(b_base + (kk >> 2) * F::kQBox + (kk & 3) * 32, 16, 1024);
            const uint32_t d = tmem + acc * F::kAccCols + 64 * sub;
            if constexpr (kFp8)
              tc::mma_f8(d, ad, bd, idesc, kk > 0);
            else
              tc::mma_bf16(d, ad, bd, idesc, kk > 0);
          }
        }
        tc::commit(&bars->empty[stage]);
        tc::commit(&bars->accfull[acc]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
        if (++acc == 2) {
          acc = 0;
          accph ^= 1;
        }
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      tc::commit(&bars->mma_done);
      tc::mbar_drain(&bars->mma_done, 0);
    }
  } else if constexpr (kG > 1) {
    // Query groups: thread `row` owns one entry's 4 x 64 head products. Each
    // epilogue warp keeps its own copy of the group's head weights in shared
    // memory (no warp waits on another when the group changes).
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    constexpr int kGW = kG / (F::kEpiWarps / 4);  // queries of the group this warp reduces
    const int g0 = kGW * ((warp - 2) >> 2);
    float *wq = w_buf + (warp - 2) * (kG * kHi + kG);
    int *nq = reinterpret_cast<int *>(wq + kG * kHi);  // the group's visible counts
    int acc = 0, cur_g = -1;
    uint32_t accph = 0;
    for (long long t = t_begin; t < t_end && !*abort; ++t) {
      const Tile tl = tile_of(t, tiles_per_q, F::kTileRows);
      if (tl.q != cur_g) {
        __syncwarp();  // every lane is done with the previous group's weights
        for (int i = lane; i < kG * kHi; i += 32) wq[i] = __ldg(a.wi + (size_t)tl.q * kG * kHi + i);
        if (lane < kG) {
          const int raw = a.n_cmp[tl.q * kG + lane];
          if ((raw < 0 || raw > a.N_max) && row == lane) raise_status(a.status, CSA_STATUS_BAD_COUNT);
          nq[lane] = raw < 0 ? 0 : (raw > a.N_max ? a.N_max : raw);
        }
        __syncwarp();
        cur_g = tl.q;
      }
      const bool ok = tc::mbar_wait(&bars->accfull[acc], accph, abort, a.status, lim);
      if (!__all_sync(0xffffffffu, ok)) break;  // keep the warp converged for tcgen05.ld
      tc::fence_after_sync();
      const int j = tl.j0 + row;
      // The group's 64 head products of query g are loaded while those of
      // query g - 1 are reduced (two register buffers); the reduction runs
      // as 8 independent chains.
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + acc * F::kAccCols + 64 * g0;
      uint32_t v[2][2][32];
      tc::tmem_ld32(tbase, v[0][0]);
      tc::tmem_ld32(tbase + 32, v[0][1]);
      tc::tmem_ld_wait();
      tc::tmem_regs_ready(v[0][0]);
      tc::tmem_regs_ready(v[0][1]);
#pragma unroll
      for (int gi = 0; gi < kGW; ++gi) {
        const int b = gi & 1, g = g0 + gi;
        if (gi + 1 < kGW) {
          tc::tmem_ld32(tbase + 64 * (gi + 1), v[b ^ 1][0]);
          tc::tmem_ld32(tbase + 64 * (gi + 1) + 32, v[b ^ 1][1]);
        }
        const float *wg = wq + g * kHi;
        float p[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) p[c] = 0.f;
#pragma unroll
        for (int h = 0; h < 32; ++h) p[h & 7] = fmaf(wg[h], fmaxf(__uint_as_float(v[b][0][h]), 0.f), p[h & 7]);
#pragma unroll
        for (int h = 0; h < 32; ++h)
          p[h & 7] = fmaf(wg[32 + h], fmaxf(__uint_as_float(v[b][1][h]), 0.f), p[h & 7]);
        const float s = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
        if (j < nq[g]) a.scores[(size_t)(tl.q * kG + g) * a.N_max + j] = s;
        if (gi + 1 < kGW) {
          tc::tmem_ld_wait();
          tc::tmem_regs_ready(v[b ^ 1][0]);
          tc::tmem_regs_ready(v[b ^ 1][1]);
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->accempty[acc]);
      if (++acc == 2) {
        acc = 0;
        accph ^= 1;
      }
    }
  } else {
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int sub = (warp - 2) >> 2;  // the tile's 128-entry block this warp reduces
    const int row = quarter * 32 + lane;
    int acc = 0, cur_q = -1, cur_n = 0;
    uint32_t accph = 0;
    float w[kHi];
    float sk_next = 1.f;
    auto load_sk = [&](long long tt) {  // key scale of tile tt's row of this thread (1 past the cache)
      const Tile tn = tile_of(tt, tiles_per_q, F::kTileRows);
      const int j = tn.j0 + 128 * sub + row;
      sk_next = j < a.N_max ? __ldg(a.sk + (size_t)(tn.q / a.q_per_seq) * a.N_max + j) : 1.f;
    };
    if constexpr (kFp8) {
      if (t_begin < t_end) load_sk(t_begin);
    }
    for (long long t = t_begin; t < t_end && !*abort; ++t) {
      const Tile tl = tile_of(t, tiles_per_q, F::kTileRows);
      if (tl.q != cur_q) {
        const int raw = a.n_cmp[tl.q];
        if ((raw < 0 || raw > a.N_max) && row == 0) raise_status(a.status, CSA_STATUS_BAD_COUNT);
        cur_n = raw < 0 ? 0 : (raw > a.N_max ? a.N_max : raw);
#pragma unroll
        for (int h = 0; h < kHi; h += 4) {
          float4 v = __ldg(reinterpret_cast<const float4 *>(a.wi + (size_t)tl.q * kHi + h));
          if constexpr (kFp8) {  // the query scales fold into the head weights
            const float4 sc = __ldg(reinterpret_cast<const float4 *>(a.sq + (size_t)tl.q * kHi + h));
            v.x *= sc.x;
            v.y *= sc.y;
            v.z *= sc.z;
            v.w *= sc.w;
          }
          w[h] = v.x;
          w[h + 1] = v.y;
          w[h + 2] = v.z;
          w[h + 3] = v.w;
        }
        cur_q = tl.q;
      }
      // E4M3: the key scales of this tile were loaded one tile ahead; start
      // the next tile's now, so their latency hides behind this tile's work.
      const float skv = sk_next;
      if constexpr (kFp8) {
        if (t + 1 < t_end) load_sk(t + 1);
      }
      const bool ok = tc::mbar_wait(&bars->accfull[acc], accph, abort, a.status, lim);
      if (!__all_sync(0xffffffffu, ok)) break;  // keep the warp converged for tcgen05.ld
      tc::fence_after_sync();
      float sc;
      {
        uint32_t v0[32], v1[32];
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + acc * F::kAccCols + 64 * sub;
        tc::tmem_ld32(taddr, v0);
        tc::tmem_ld32(taddr + 32, v1);
        tc::tmem_ld_wait();
        float s = 0.f;
#pragma unroll
        for (int h = 0; h < 32; ++h) s = fmaf(w[h], fmaxf(__uint_as_float(v0[h]), 0.f), s);
#pragma unroll
        for (int h = 0; h < 32; ++h) s = fmaf(w[32 + h], fmaxf(__uint_as_float(v1[h]), 0.f), s);
        sc = s;
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&bars->accempty[acc]);
      {
        const int j = tl.j0 + 128 * sub + row;
        if (j < cur_n) a.scores[(size_t)tl.q * a.N_max + j] = kFp8 ? sc * skv : sc;
      }
      if (++acc == 2) {
        acc = 0;
        accph ^= 1;
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, F::kTmemCols);
  }
}

int num_sms_cached() { return device_sm_count(); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

namespace {

// *taken stays false when no tensor map can describe these pointers (the
// generic kernel then serves the call).
template <bool kFp8, int kG>
cudaError_t launch_tc(const ScoreArgs &a, cudaStream_t stream, bool *taken) {
  using F = Fmt<kFp8, kG>;
  CUtensorMap tm_ki, tm_qi;
  const int esz = kFp8 ? 1 : 2, box = kFp8 ? 128 : 64;
  auto mk = kFp8 ? make_tmap_u8_2d : make_tmap_bf16_2d;
  if (!mk(&tm_ki, a.ki, kDi, (uint64_t)a.B * a.N_max, kDi * esz, box, 128)) return cudaSuccess;
  if (!mk(&tm_qi, a.qi, kDi, (uint64_t)a.Q * kHi, kDi * esz, box, kG * kHi)) return cudaSuccess;
  const int tiles_per_q = (a.N_max + F::kTileRows - 1) / F::kTileRows;
  const long long total = (long long)(a.Q / kG) * tiles_per_q;
  long long grid = num_sms_cached();
  if (grid > total) grid = total;
  const long long per_cta = (total + grid - 1) / grid;
  grid = (total + per_cta - 1) / per_cta;
  static DeviceOnce attr;
  once_per_device(attr, [] {
    cudaFuncSetAttribute(index_scores_tc_kernel<kFp8, kG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem_bytes<kFp8, kG>());
  });
  *taken = true;
  return launch_pdl(index_scores_tc_kernel<kFp8, kG>, dim3((unsigned)grid), dim3(F::kThreads), smem_bytes<kFp8, kG>(),
                    stream, tm_ki, tm_qi, a, tiles_per_q, total, per_cta);
}

}  // namespace

cudaError_t launch_index_scores_tc(const ScoreArgs &a, cudaStream_t stream, bool *taken) {
  *taken = false;
  const bool fp8 = a.dtype == CSA_DTYPE_E4M3;
  if (!(fp8 || a.dtype == CSA_DTYPE_BF16) || a.Hi != kHi || a.Di != kDi) return cudaSuccess;
  if (!aligned16(a.qi) || !aligned16(a.ki) || (reinterpret_cast<uintptr_t>(a.wi) & 15)) return cudaSuccess;
  if (fp8 && (reinterpret_cast<uintptr_t>(a.sq) & 15)) return cudaSuccess;
  // Groups of 4 queries of one sequence share each key tile (prefill).
  const bool groups = !fp8 && a.q_per_seq % 4 == 0 && a.Q % 4 == 0;
  return fp8 ? launch_tc<true, 1>(a, stream, taken) : groups ? launch_tc<false, 4>(a, stream, taken)
                                                           : launch_tc<false, 1>(a, stream, taken);
}

}  // namespace csa
