// One decode step of a CSA or HCA layer in a single persistent kernel:
// the cache append (A1), the indexer scores (A2), the top-k selection (A3)
// and the attention over the selection or all entries plus the window and
// the sink (A4 / A5), with the same arithmetic as the separate kernels
// ("DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: compressed
// entries, indexer top-k, sliding window, attention sink; section 2: K = V).
//
// Why one kernel. In CSA decode the indexer key scan moves 84-98 % of the
// step's bytes and runs at HBM speed, while the selection and the attention
// of a query are latency-bound chains of a few microseconds each. As separate
// kernels they run one after the other, and the latency-bound ones leave HBM
// idle. Here every CTA (one per SM) pulls tasks from device-side queues as
// their inputs become ready, so the selection and attention of the queries
// whose keys are scanned run while the keys of later queries stream in; only
// the last query's chain is exposed after the scan.
//
// Tasks (all of one CTA's 13 worker warps, one at a time):
//   APPEND  (b, j)      entry j of sequence b's new window: pool + RMSNorm (+ RoPE)
//   SCORE   chunk       4 key tiles of one query: tcgen05 scorer pipeline
//   TOPK1   (q, g)      top-k of segment g of query q's scores (the whole list
//                       when it has one segment)
//   TOPK2   q           top-k of the segments' winners
//   MQA     (qv, s)     attention split s of query q's 64-head group: the
//                       window rows (CSA split 0), a run of selected rows, or
//                       a run of dense rows (HCA); writes an unnormalised
//                       (m, l, O) partial
//   MERGE   (qv, p)     part p of the output from all splits' partials + sink
// Scheduling. Tasks without inputs from other tasks (APPEND, the attention
// splits over the window (CSA) or over dense rows that need no appended
// entry (HCA), and SCORE chunks in query-major order) form one static list
// dealt round-robin to the CTAs: no claiming, and queries finish their scans
// in order. A task whose inputs come from other tasks is pushed into a
// device-side ready queue by the task that completes its last input (a
// dependency counter raised with acquire-release atomics); CTAs take queued
// tasks before static ones. A task is only ever queued once ready, so no CTA
// waits on work that nobody has started.
//
// Roles. Warps 0-12 do the tasks (the scorer pipeline uses warp 0 lane 0 as
// TMA producer, warp 8 as MMA issuer, warps 9-12 as epilogue; the attention
// uses warps 0-7 as loaders, warp 8 as MMA issuer, warps 9-12 for the
// softmax); warp 13 takes a task from the ready queue while the current one
// runs and leaves it in a shared-memory mailbox.
//
// Every wait is bounded (2 s); a timeout raises CSA_STATUS_WAIT_TIMEOUT and a
// global abort flag that makes every CTA stop claiming. The last CTA to exit
// returns all counters to zero for the next launch.
#include "block_select.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace csa {

namespace {

// ------------------------------------------------------------------ shape
constexpr int kWorkers = 416;               // warps 0..12
constexpr int kThreads = kWorkers + 32;     // + the scheduler warp
constexpr int kSchedWarp = 13;
constexpr int kBarSoft = 1, kBarWork = 2, kBarEpi = 3;  // named barriers (0 is __syncthreads)

// attention (same geometry as the stand-alone tensor-core MQA)
constexpr int kH = 64, kD = 512, kRows = 64;
constexpr uint32_t kBoxBytes = kRows * 128;     // 64 rows x 64 dims: 8 KB
constexpr uint32_t kTileBytes = 8 * kBoxBytes;  // 64 rows x 512 dims: 64 KB
constexpr uint32_t kQBoxBytes = kH * 128;
constexpr uint32_t kQBytes = 8 * kQBoxBytes;    // 64 heads x 512 dims: 64 KB
constexpr uint32_t kPBytes = kRows * kH * 2;    // 8 KB
constexpr int kLoadWarps = 8, kWarpsPerBuf = 4, kRowsPerWarp = kRows / kWarpsPerBuf;
constexpr int kMmaWarp = 8, kSoftWarp0 = 9;
constexpr uint32_t kTmemCols = 512, kColO = 0, kColS = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kMaxSplits = 32;
constexpr int kAhead = 1;  // rounds of tiles prefetched into L2 ahead of their load (see the stand-alone kernel)

// scorer (indexer 64 heads x 128 dims)
constexpr int kHi = 64, kDi = 128;
constexpr int kStages = 5;
template <bool kFp8>
struct SF {
  static constexpr int kSub = kFp8 ? 2 : 1;             // 128-row MMA blocks per tile
  static constexpr int kTileRows = 128 * kSub;
  static constexpr int kKBoxes = kFp8 ? 1 : 2;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  static constexpr uint32_t kBoxBytes = 128 * 128;
  static constexpr uint32_t kTileBytes = 2 * kBoxBytes;  // 32 KB
  static constexpr uint32_t kQBytes = kHi * kDi * (kFp8 ? 1 : 2);
  static constexpr uint32_t kQBox = kQBytes / kKBoxes;
  static constexpr uint32_t kAccCols = 64 * kSub;
  static constexpr uint32_t kIdesc = kFp8 ? tc::idesc_e4m3(128, 64) : tc::idesc_bf16(128, 64, 0, 0);
};

// One region of shared memory serves each task in turn.
constexpr uint32_t kRegionBytes = 2 * kTileBytes + kQBytes + 2 * kPBytes;  // 208 KB
static_assert(kStages * SF<false>::kTileBytes + 2 * SF<false>::kQBytes + 4 * 64 * 4 <= kRegionBytes, "scorer view");
constexpr int kHist1 = 13;  // private histogram copies of a segment selection (one per worker warp)
constexpr int kHist2 = 2;   // ... of the winners' selection
constexpr int kSegMax = 16384;                                                 // TOPK1 keys (largest segment)
constexpr int kCandCap = ((int)(kRegionBytes / 4) - kHist2 * bsel::kBins) / 2;  // TOPK2 keys + positions
static_assert(kSegMax * 4 + kHist1 * bsel::kBins * 4 <= kRegionBytes, "segment selection view");

// task types
enum : int { T_NONE = 0, T_EXIT, T_APPEND, T_SCORE, T_TOPK1, T_TOPK2, T_MQA, T_MERGE };
// counters at the head of the counter block (K_HEAD, K_RESERVE: one 8-byte word)
enum : int { K_HEAD = 0, K_RESERVE = 1, K_STATIC = 4, K_ABORT = 8, K_EXIT = 9, kCtrHead = 16 };

// meta flags of a scorer tile
constexpr int M_LAST = 1, M_SENTINEL = 2;

struct Hdr {
  // scorer pipeline
  uint64_t full[kStages], empty[kStages], qfull[2], qempty[2], accfull[2], accempty[2];
  int4 smeta[kStages];
  int4 ameta[2];
  // attention pipeline
  uint64_t q_full, kv_full[2], kv_empty[2], s_full[2], p_full[2], pv_done[4], o_done;
  uint64_t mma_drain;
  float red[4][kH];
  alignas(16) float mref[kH];
  float alpha[kH];
  float lsum[kH];
  int need[4];
  int rescale;
  const bf16 *rowp[kLoadWarps][kRowsPerWarp];
  // selection
  bsel::Shared sel;
  int offs[65];
  // tasks
  int4 mb_task, cur, pending;
  int mb_full, busy, st_pre, st_done;
  uint64_t bulk;   // bulk copies into the region (top-k scores, merge partials)
  int bulk_n;      // its completed phases
  // pipeline positions carried between tasks (kept here, not in registers,
  // so that no task pays for another's state)
  int ss_stage, ss_phase, ss_nq, ss_acc, ss_accph;  // scorer ring
  uint32_t ss_imask, ss_iphase;                     // scorer stages issued, and their last parity
  int ms_LI, ms_mt, ms_mq;                          // attention tiles, tasks, query-block loads
  uint64_t wait_ns;                                  // limit of every bounded wait in this launch
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = 1024 + kRegionBytes + sizeof(Hdr);
static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");

}  // namespace

// Launch plan (host-computed) and arguments.
struct StepPlan {
  int mode;           // 0 CSA (scores + top-k + sparse attention), 1 HCA (dense attention)
  int fp8;            // indexer on E4M3 codes
  int G, QV;          // 64-head groups per query, query groups
  // scorer
  int tile_rows, tiles_per_q, chunk_tiles, chunks_per_q;
  int nseg, seg_tiles, seg_entries;
  int sstride;        // row stride of the scores (entries; a multiple of 32)
  // attention
  int win_tiles;      // CSA: window tiles at the head of each row list
  int sel_tiles;      // CSA: tiles of selected rows; HCA: 0
  int tps;            // tiles per split (selected rows / dense rows)
  int S_main;         // CSA: splits of the selected rows; HCA: splits of the dense list
  int S;              // partials per query group (CSA: 1 + S_main; HCA: S_main)
  int P;              // merge parts per query group (0: one split, no merge)
  int app_per_b;      // appended entries per sequence (0: no append)
  int app_row0;       // their first row in the compressed cache
  int dep_s0, n_dep;  // HCA: the splits holding appended rows (queued once the append is done)
  int deps_target;    // CSA: completions an attention split of a query waits for (top-k, append)
  int n_app, n_ms, n_chunks, n_static;  // the static list: appends | attention splits | score chunks
  int D;              // tasks that go through the ready queue
  int q_off;          // word offset of the ready queue (8-byte slots) in the counter block
  int n_ctr;          // counter words, queue included
};

struct StepArgs {
  // append
  CompressArgs app;
  // indexer
  const void *qi, *ki;
  const float *wi, *sq, *sk;
  const int32_t *n_cmp;
  int k;
  int32_t *idx;
  float *scores;
  // attention
  const void *q, *kv_cmp, *kv_win;
  const int32_t *win_end;
  const float *sink;
  float scale_log2;
  void *out;
  int Q, B, H, N_max, win_len, T_raw, q_per_seq;
  // workspace
  float *part_o, *part_ml;
  uint32_t *cand_key;
  int32_t *cand_idx, *cand_cnt;
  uint32_t *ctr;
  uint32_t *status;
};

namespace {

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void wbar() { asm volatile("bar.sync %0, %1;" ::"r"(kBarWork), "r"(kWorkers) : "memory"); }
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ bool bar_any(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, %2, %3, p; selp.u32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void bulk_prefetch_l2(const void *p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
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

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global to shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   tc::smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

// Bounded mbarrier wait with this launch's limit (see tc::mbar_wait).
__device__ __forceinline__ bool mwait(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t *status,
                                      uint64_t limit) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if ((i & 63) == 63) {
      const uint64_t now = tc::globaltimer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit) {
        raise_status(status, CSA_STATUS_WAIT_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void mbar_arrive_cnt(uint64_t *bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(tc::smem_u32(bar)), "r"(n) : "memory");
}

// ------------------------------------------------------------------ scheduling

// per-index counters: scored tiles per (query, segment), finished segment
// selections per query, completed inputs of a query's attention splits, and
// finished splits per query group
__device__ __forceinline__ uint32_t *ctr_seg(const StepArgs &a, const StepPlan &P) { return a.ctr + kCtrHead; }
__device__ __forceinline__ uint32_t *ctr_sel(const StepArgs &a, const StepPlan &P) {
  return a.ctr + kCtrHead + a.Q * P.nseg;
}
__device__ __forceinline__ uint32_t *ctr_deps(const StepArgs &a, const StepPlan &P) {
  return a.ctr + kCtrHead + a.Q * (P.nseg + 1);
}
__device__ __forceinline__ uint32_t *ctr_arr(const StepArgs &a, const StepPlan &P) {
  return a.ctr + kCtrHead + a.Q * (P.nseg + 2);
}
__device__ __forceinline__ unsigned long long *ready_queue(const StepArgs &a, const StepPlan &P) {
  return reinterpret_cast<unsigned long long *>(a.ctr + P.q_off);
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const void *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u64(void *p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// A queued task: type (8 bits) | a (28 bits) | b (28 bits); 0 = not yet written.
__device__ __forceinline__ unsigned long long enc_task(int type, int x, int y) {
  return (unsigned long long)type | ((unsigned long long)x << 8) | ((unsigned long long)y << 36);
}
__device__ __forceinline__ int4 dec_task(unsigned long long v) {
  return make_int4((int)(v & 0xff), (int)((v >> 8) & 0xfffffff), (int)((v >> 36) & 0xfffffff), 0);
}

// Queue n ready tasks (one thread). The slot stores are releases: whoever
// takes a task sees everything its pusher saw.
template <class F>
__device__ __forceinline__ void push_tasks(const StepArgs &a, const StepPlan &P, int n, F task_at) {
  const uint32_t slot = atomicAdd(a.ctr + K_RESERVE, (uint32_t)n);
  unsigned long long *qu = ready_queue(a, P);
  for (int i = 0; i < n; ++i) st_release_u64(qu + slot + i, task_at(i));
}

__device__ __forceinline__ int seg_tiles_of(const StepPlan &P, int g) {
  return g < P.nseg - 1 ? P.seg_tiles : P.tiles_per_q - (P.nseg - 1) * P.seg_tiles;
}

// One more completed input of query q's attention splits: the last one
// queues them (CSA: the selected-row splits of every head group).
__device__ __forceinline__ void complete_dep(const StepArgs &a, const StepPlan &P, int q) {
  if ((int)atom_add_acq_rel(ctr_deps(a, P) + q, 1u) + 1 == P.deps_target)
    push_tasks(a, P, P.G * P.S_main, [&](int i) {
      return enc_task(T_MQA, q * P.G + i / P.S_main, 1 + i % P.S_main);
    });
}

// Static task t of the round-robin list.
__device__ __forceinline__ int4 static_task(const StepPlan &P, int t) {
  if (t < P.n_app) return make_int4(T_APPEND, t, 0, 0);
  t -= P.n_app;
  if (t < P.n_ms) {
    if (P.mode == 0) return make_int4(T_MQA, t, 0, 0);  // CSA: the window split of query group t
    const int si = t / P.QV, qv = t - si * P.QV;       // HCA: split-major, skipping the queued ones
    return make_int4(T_MQA, qv, si < P.dep_s0 ? si : si + P.n_dep, 0);
  }
  return make_int4(T_SCORE, t - P.n_ms, 0, 0);
}

// The ready-queue warp: while the workers run a scoring run or wait for
// work (not busy), it takes a ticket (the next queue position, one atomic
// add: tickets never fail or retry) and waits for that position to be
// filled, then leaves the task in the mailbox. Every queued task is filled
// by a running task and taken by exactly one ticket, so a waiting ticket is
// always served; a ticket past the last queued task of the launch means EXIT.
// The workers keep taking static work while the ticket waits.
__device__ void scheduler(const StepArgs &a, const StepPlan &P, Hdr *h) {
  if ((threadIdx.x & 31) != 0) return;
  volatile int *mb_full = &h->mb_full, *busy = &h->busy, *abort = &h->abort;
  unsigned long long *qu = ready_queue(a, P);
  for (;;) {
    while (*mb_full || *busy) {  // (a busy CTA would sit on a ready task)
      if (*abort) return;
      __nanosleep(128);
    }
    const uint32_t ticket = atomicAdd(a.ctr + K_HEAD, 1u);
    int4 task = make_int4(T_EXIT, 0, 0, 0);
    if ((int)ticket < P.D) {
      unsigned long long v;
      uint64_t t0 = 0;
      for (uint32_t i = 0; (v = ld_acquire_u64(qu + ticket)) == 0; ++i) {
        if (*abort) return;
        __nanosleep(64);
        if ((i & 15) == 15) {
          if (ld_relaxed(a.ctr + K_ABORT)) break;  // another CTA gave up: EXIT
          const uint64_t now = tc::globaltimer_ns();
          if (t0 == 0) {
            t0 = now;
          } else if (now - t0 > h->wait_ns) {
            raise_status(a.status, CSA_STATUS_WAIT_TIMEOUT);
            atomicExch(a.ctr + K_ABORT, 1u);
            break;
          }
        }
      }
      if (v != 0) task = dec_task(v);
    }
    h->mb_task = task;
    __threadfence_block();
    *mb_full = 1;
    if (task.x == T_EXIT) return;
  }
}

// Worker side (thread 0): the CTA's next task. A queued task comes first,
// then the static list (claimed in order through one counter, usually one
// task ahead, see score_run); EXIT once both are exhausted. In a scoring run
// (in_run) T_NONE means: end the run, nothing claimed. Bounded.
__device__ int4 take_task(const StepArgs &a, const StepPlan &P, Hdr *h, bool in_run) {
  volatile int *mb_full = &h->mb_full, *abort = &h->abort, *busy = &h->busy;
  *busy = 0;  // between tasks: the queue warp may take a queued task
  const uint64_t t0 = tc::globaltimer_ns();
  for (;;) {
    if (*abort) return make_int4(T_EXIT, 0, 0, 0);
    if (*mb_full) {
      __threadfence_block();
      const volatile int *mt = reinterpret_cast<const volatile int *>(&h->mb_task);
      const int4 t = make_int4(mt[0], mt[1], mt[2], mt[3]);
      if (t.x != T_EXIT) {
        // the task's inputs were published at gpu scope and acquired by the queue warp
        asm volatile("fence.acq_rel.gpu;" ::: "memory");
        *busy = 1;
        __threadfence_block();
        *mb_full = 0;
        return t;
      }
      if (h->st_done) return t;  // EXIT (left in the mailbox)
    }
    if (!h->st_done) {
      const int ti = h->st_pre >= 0 ? h->st_pre : (int)atomicAdd(a.ctr + K_STATIC, 1u);
      h->st_pre = -1;
      if (ti < P.n_static) {
        const int4 t = static_task(P, ti);
        *busy = t.x != T_SCORE;
        return t;
      }
      h->st_done = 1;
      continue;
    }
    if (in_run) return make_int4(T_NONE, 0, 0, 0);  // no static work left: end the run, wait outside it
    __nanosleep(64);
    if (tc::globaltimer_ns() - t0 > 2 * h->wait_ns) {
      raise_status(a.status, CSA_STATUS_WAIT_TIMEOUT);
      *abort = 1;
      return make_int4(T_EXIT, 0, 0, 0);
    }
  }
}

// ------------------------------------------------------------------ APPEND
// Entry j of sequence b of the new raw window: the gated pool over the win
// positions, RMSNorm, and RoPE of the last rope_dims dims at the entry's
// last-token position (same definitions as csa_compress / csa_compress_rope).

__device__ __forceinline__ void unpack8(const uint4 &v, float f[8]) {
  const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ void append_task(const StepArgs &a, const StepPlan &P, Hdr *h, uint8_t *region, int task) {
  const CompressArgs &c = a.app;
  const int b = task / P.app_per_b, j = task % P.app_per_b;
  constexpr int kVec = kD / 8;                // 64 vectors of 8 dims
  constexpr int kGroups = kWorkers / kVec;    // 6 position groups
  const int tid = threadIdx.x, v = tid % kVec, g = tid / kVec;
  float *st = reinterpret_cast<float *>(region);  // [kGroups][3][8][kVec]
  float *cvec = st + kGroups * 3 * 8 * kVec;      // [kD] pooled values
  float *ssum = cvec + kD;                        // [32]
  const bf16 *kvj = static_cast<const bf16 *>(c.kv) + b * c.kv_ss + (long long)j * c.stride * kD;
  const bf16 *gj = static_cast<const bf16 *>(c.gate) + b * c.gate_ss + (long long)j * c.stride * kD;
  if (g < kGroups) {
    float m[8], l[8], acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      m[e] = -INFINITY;
      l[e] = 0.f;
      acc[e] = 0.f;
    }
    for (int i0 = g; i0 < c.win; i0 += 2 * kGroups) {
      uint4 kvv[2], gv[2];
      float4 a0[2], a1[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = i0 + u * kGroups;
        if (i < c.win) {
          kvv[u] = __ldg(reinterpret_cast<const uint4 *>(kvj + (long long)i * kD) + v);
          gv[u] = __ldg(reinterpret_cast<const uint4 *>(gj + (long long)i * kD) + v);
          a0[u] = __ldg(reinterpret_cast<const float4 *>(c.ape + (size_t)i * kD + 8 * v));
          a1[u] = __ldg(reinterpret_cast<const float4 *>(c.ape + (size_t)i * kD + 8 * v + 4));
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = i0 + u * kGroups;
        if (i < c.win) {
          float kf[8], gf[8];
          unpack8(kvv[u], kf);
          unpack8(gv[u], gf);
          const float ap[8] = {a0[u].x, a0[u].y, a0[u].z, a0[u].w, a1[u].x, a1[u].y, a1[u].z, a1[u].w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x = (gf[e] + ap[e]) * kLog2e;
            const float mx = fmaxf(m[e], x);
            const float ex = exp2f(fminf(m[e], x) - mx);
            const bool up = x > m[e];
            const float so = up ? ex : 1.f, sn = up ? 1.f : ex;
            l[e] = l[e] * so + sn;
            acc[e] = acc[e] * so + kf[e] * sn;
            m[e] = mx;
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      st[((g * 3 + 0) * 8 + e) * kVec + v] = m[e];
      st[((g * 3 + 1) * 8 + e) * kVec + v] = l[e];
      st[((g * 3 + 2) * 8 + e) * kVec + v] = acc[e];
    }
  }
  wbar();
  float ss = 0.f;
  for (int d = tid; d < kD; d += kWorkers) {
    const int vv = d / 8, e = d % 8;
    float M = -INFINITY;
    for (int gg = 0; gg < kGroups; ++gg) M = fmaxf(M, st[((gg * 3 + 0) * 8 + e) * kVec + vv]);
    float L = 0.f, A = 0.f;
    for (int gg = 0; gg < kGroups; ++gg) {
      const float mg = st[((gg * 3 + 0) * 8 + e) * kVec + vv];
      const float w = mg == -INFINITY ? 0.f : exp2f(mg - M);
      L += st[((gg * 3 + 1) * 8 + e) * kVec + vv] * w;
      A += st[((gg * 3 + 2) * 8 + e) * kVec + vv] * w;
    }
    const float cd = A / L;
    cvec[d] = cd;
    ss += cd * cd;
  }
  ss = warp_sum(ss);
  if ((tid & 31) == 0) ssum[tid >> 5] = ss;
  wbar();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kWorkers / 32; ++w) tot += ssum[w];
  const float r = 1.0f / sqrtf(tot / (float)kD + 1e-6f);
  bf16 *o = static_cast<bf16 *>(c.out) + b * c.out_ss + (long long)j * kD;
  const int d0 = kD - c.rope_dims;
  for (int p = tid; p < kD / 2; p += kWorkers) {
    const int d = 2 * p;
    float x0 = cvec[d] * r * c.norm_w[d], x1 = cvec[d + 1] * r * c.norm_w[d + 1];
    if (c.rope_dims && d >= d0) {
      const double pos = (double)((c.pos0 ? c.pos0[b] : 0) + (long long)j * c.stride + c.win - 1);
      const double ang = pos * pow(c.rope_theta, -(double)(d - d0) / c.rope_dims);
      double sn, cs;
      sincos(ang, &sn, &cs);
      const float cf = (float)cs, sf = (float)sn;
      const float y0 = x0 * cf - x1 * sf, y1 = x0 * sf + x1 * cf;
      x0 = y0;
      x1 = y1;
    }
    *reinterpret_cast<__nv_bfloat162 *>(o + d) = __floats2bfloat162_rn(x0, x1);
  }
  wbar();
  if (tid == 0 && b < a.Q) {  // (one query per sequence; sequences past Q have none)
    if (P.mode == 0) {
      complete_dep(a, P, b);
    } else if (P.n_dep > 0) {  // HCA: the splits over the new rows can start
      push_tasks(a, P, P.G * P.n_dep, [&](int i) {
        return enc_task(T_MQA, b * P.G + i / P.n_dep, P.dep_s0 + i % P.n_dep);
      });
    }
  }
}

// ------------------------------------------------------------------ SCORE
// The indexer scorer of one CTA over a run of chunks (same arithmetic and
// pipeline as index_scores_tc_kernel): warp 0 lane 0 loads key tiles and the
// query's head block by TMA, warp 8 lane 0 issues the tcgen05 MMAs into two
// TMEM accumulators, warps 9-12 reduce sum_h w_h ReLU(.) per entry. The run
// ends when the mailbox hands the producer a task of another kind: a
// sentinel then travels down the pipeline behind the last tile.

struct ScoreState {
  int stage, nq;
  uint32_t phase;
  int acc;
  uint32_t accph;
  uint32_t issued_mask, issued_phase;  // producer: per stage, a load was issued, with this parity
};

template <bool kFp8>
__device__ void score_run(const StepArgs &a, const StepPlan &P, Hdr *h, uint8_t *region, uint32_t tmem,
                          const CUtensorMap *tm_ki, const CUtensorMap *tm_qi, int4 first) {
  using F = SF<kFp8>;
  ScoreState ss{h->ss_stage, h->ss_nq, (uint32_t)h->ss_phase, h->ss_acc, (uint32_t)h->ss_accph, h->ss_imask,
                h->ss_iphase};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t *stage_buf = region;
  uint8_t *q_buf = region + kStages * F::kTileBytes;
  volatile int *abort = &h->abort;
  const uint64_t lim = h->wait_ns;
  if (warp == 0) {
    if (lane == 0) {
      int4 task = first;
      int cur_q = -1, qslot_seq = -1;
      bool ok = true;
      for (;;) {
        const int cidx = task.y;  // chunk index (query-major)
        // claim the next static task now; its index is only needed at the
        // end of the chunk, so the atomic's round trip hides behind the loads
        const int pre = h->st_done ? -1 : (int)atomicAdd(a.ctr + K_STATIC, 1u);
        const int q = cidx / P.chunks_per_q, cc = cidx - q * P.chunks_per_q;
        const int t0 = cc * P.chunk_tiles, t1 = min(P.tiles_per_q, t0 + P.chunk_tiles);
        const int g = t0 / P.seg_tiles;
        if (q != cur_q) {
          const int slot = ss.nq & 1;
          if (!mwait(&h->qempty[slot], ((ss.nq >> 1) & 1) ^ 1, abort, a.status, lim)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(&h->qfull[slot], F::kQBytes);
          for (int bx = 0; bx < F::kKBoxes; ++bx)
            tc::tma_load_2d(q_buf + slot * F::kQBytes + bx * F::kQBox, tm_qi, bx * 64, q * kHi, &h->qfull[slot]);
          qslot_seq = ss.nq++;
          cur_q = q;
        }
        for (int t = t0; t < t1; ++t) {
          if (!mwait(&h->empty[ss.stage], ss.phase ^ 1, abort, a.status, lim)) {
            ok = false;
            break;
          }
          const int flags = (t == t1 - 1 ? M_LAST : 0) | ((t1 - t0) << 8) | (g << 16);
          h->smeta[ss.stage] = make_int4(q, t * F::kTileRows, qslot_seq, flags);
          tc::mbar_arrive_expect_tx(&h->full[ss.stage], F::kTileBytes);
          const int row = (q / a.q_per_seq) * a.N_max + t * F::kTileRows;
          for (int bx = 0; bx < 2; ++bx)
            tc::tma_load_2d(stage_buf + ss.stage * F::kTileBytes + bx * F::kBoxBytes, tm_ki, kFp8 ? 0 : 64 * bx,
                            kFp8 ? row + 128 * bx : row, &h->full[ss.stage]);
          if constexpr (kFp8) {  // the tile's key scales, into L2 for the epilogue (16-byte aligned span)
            const uintptr_t lo = reinterpret_cast<uintptr_t>(a.sk + row) & ~uintptr_t(15);
            const uintptr_t hi = (reinterpret_cast<uintptr_t>(a.sk + min(row + F::kTileRows, a.B * a.N_max)) + 15) &
                                 ~uintptr_t(15);
            if (hi > lo) bulk_prefetch_l2(reinterpret_cast<const void *>(lo), (uint32_t)(hi - lo));
          }
          ss.issued_mask |= 1u << ss.stage;
          ss.issued_phase = (ss.issued_phase & ~(1u << ss.stage)) | (ss.phase << ss.stage);
          if (++ss.stage == kStages) {
            ss.stage = 0;
            ss.phase ^= 1;
          }
        }
        if (pre >= 0) h->st_pre = pre;
        if (!ok) break;
        task = take_task(a, P, h, true);
        if (task.x == T_SCORE) continue;
        // end of the run: a sentinel follows the last tile
        if (!mwait(&h->empty[ss.stage], ss.phase ^ 1, abort, a.status, lim)) {
          ok = false;
          break;
        }
        h->smeta[ss.stage] = make_int4(0, 0, 0, M_SENTINEL);
        tc::mbar_arrive(&h->full[ss.stage]);
        ss.issued_mask |= 1u << ss.stage;  // the stage's latest phase (see the drain at exit)
        ss.issued_phase = (ss.issued_phase & ~(1u << ss.stage)) | (ss.phase << ss.stage);
        if (++ss.stage == kStages) {
          ss.stage = 0;
          ss.phase ^= 1;
        }
        h->pending = task;
        break;
      }
      if (!ok) h->pending = make_int4(T_EXIT, 0, 0, 0);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      int cur_seq = -1;
      int stage = ss.stage;  // the consumer trails the producer through the same ring
      uint32_t phase = ss.phase;
      for (;;) {
        if (!mwait(&h->full[stage], phase, abort, a.status, lim)) break;
        const int4 meta = h->smeta[stage];
        if (meta.w & M_SENTINEL) {
          tc::mbar_arrive(&h->empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
          if (!mwait(&h->accempty[ss.acc], ss.accph ^ 1, abort, a.status, lim)) break;
          h->ameta[ss.acc] = meta;
          mbar_arrive_cnt(&h->accfull[ss.acc], 2);
          if (++ss.acc == 2) {
            ss.acc = 0;
            ss.accph ^= 1;
          }
          break;
        }
        if (meta.z != cur_seq) {
          if (cur_seq >= 0) tc::commit(&h->qempty[cur_seq & 1]);
          if (!mwait(&h->qfull[meta.z & 1], (meta.z >> 1) & 1, abort, a.status, lim)) break;
          cur_seq = meta.z;
        }
        if (!mwait(&h->accempty[ss.acc], ss.accph ^ 1, abort, a.status, lim)) break;
        tc::fence_after_sync();
        const uint32_t a_base = tc::smem_u32(stage_buf + stage * F::kTileBytes);
        const uint32_t b_base = tc::smem_u32(q_buf + (meta.z & 1) * F::kQBytes);
#pragma unroll
        for (int sub = 0; sub < F::kSub; ++sub) {
#pragma unroll
          for (int kk = 0; kk < F::kKSteps; ++kk) {
            const uint32_t box = kFp8 ? sub : (kk >> 2);
            const uint64_t ad = tc::sw128_desc(a_base + box * F::kBoxBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = tc::sw128_desc(b_base + (kk >> 2) * F::kQBox + (kk & 3) * 32, 16, 1024);
            const uint32_t d = tmem + ss.acc * F::kAccCols + 64 * sub;
            if constexpr (kFp8)
              tc::mma_f8(d, ad, bd, F::kIdesc, kk > 0);
            else
              tc::mma_bf16(d, ad, bd, F::kIdesc, kk > 0);
          }
        }
        tc::commit(&h->empty[stage]);
        h->ameta[ss.acc] = meta;
        tc::mbar_arrive(&h->accfull[ss.acc]);  // releases ameta
        tc::commit(&h->accfull[ss.acc]);       // the MMAs' completion
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
        if (++ss.acc == 2) {
          ss.acc = 0;
          ss.accph ^= 1;
        }
      }
      if (cur_seq >= 0) tc::commit(&h->qempty[cur_seq & 1]);  // the head block's slot is free once its MMAs are
    }
  } else if (warp >= kSoftWarp0) {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int acc = ss.acc;
    uint32_t accph = ss.accph;
    int cur_q = -1, cur_n = 0;
    // this warp's copy of the query's head weights (shared memory past the
    // stages and head blocks; every lane reads the same word: a broadcast)
    float *w = reinterpret_cast<float *>(region + kStages * F::kTileBytes + 2 * F::kQBytes) + (warp - kSoftWarp0) * kHi;
    for (;;) {
      const bool okw = mwait(&h->accfull[acc], accph, abort, a.status, lim);
      // the four epilogue warps stop together (they share a named barrier below)
      if (bar_any(kBarEpi, 128, !okw)) break;
      const int4 meta = h->ameta[acc];
      if (meta.w & M_SENTINEL) {
        tc::mbar_arrive(&h->accempty[acc]);
        if (++acc == 2) {
          acc = 0;
          accph ^= 1;
        }
        break;
      }
      const int q = meta.x, j0 = meta.y;
      if (q != cur_q) {
        const int raw = a.n_cmp[q];
        if ((raw < 0 || raw > a.N_max) && row == 0) raise_status(a.status, CSA_STATUS_BAD_COUNT);
        cur_n = raw < 0 ? 0 : (raw > a.N_max ? a.N_max : raw);
        __syncwarp();  // every lane is done with the previous query's weights
        for (int hh = lane; hh < kHi; hh += 32) {
          float v = __ldg(a.wi + (size_t)q * kHi + hh);
          if constexpr (kFp8) v *= __ldg(a.sq + (size_t)q * kHi + hh);  // the query scales fold into the weights
          w[hh] = v;
        }
        __syncwarp();
        cur_q = q;
      }
      float skv[F::kSub];  // E4M3 key scales (in L2: the producer prefetched them with the tile)
      if constexpr (kFp8) {
#pragma unroll
        for (int sub = 0; sub < F::kSub; ++sub) {
          const int j = j0 + 128 * sub + row;
          skv[sub] = j < a.N_max ? __ldg(a.sk + (size_t)(q / a.q_per_seq) * a.N_max + j) : 1.f;
        }
      }
      tc::fence_after_sync();
      float sc[F::kSub];
#pragma unroll
      for (int sub = 0; sub < F::kSub; ++sub) {
        const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + acc * F::kAccCols + 64 * sub;
        float s = 0.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // 32 heads at a time
          uint32_t v[32];
          tc::tmem_ld32(taddr + 32 * half, v);
          tc::tmem_ld_wait();
          const float4 *w4 = reinterpret_cast<const float4 *>(w + 32 * half);
#pragma unroll
          for (int h4 = 0; h4 < 8; ++h4) {
            const float4 ww = w4[h4];
            s = fmaf(ww.x, fmaxf(__uint_as_float(v[4 * h4]), 0.f), s);
            s = fmaf(ww.y, fmaxf(__uint_as_float(v[4 * h4 + 1]), 0.f), s);
            s = fmaf(ww.z, fmaxf(__uint_as_float(v[4 * h4 + 2]), 0.f), s);
            s = fmaf(ww.w, fmaxf(__uint_as_float(v[4 * h4 + 3]), 0.f), s);
          }
        }
        sc[sub] = s;
      }
      tc::fence_before_sync();
      tc::mbar_arrive(&h->accempty[acc]);
#pragma unroll
      for (int sub = 0; sub < F::kSub; ++sub) {
        const int j = j0 + 128 * sub + row;
        if (j < cur_n) a.scores[(size_t)q * P.sstride + j] = kFp8 ? sc[sub] * skv[sub] : sc[sub];
      }
      if (++acc == 2) {
        acc = 0;
        accph ^= 1;
      }
      if (meta.w & M_LAST) {
        // the chunk's scores are all stored: publish them; the chunk that
        // completes its segment queues the segment's selection
        named_sync(kBarEpi, 128);
        if (warp == kSoftWarp0 && lane == 0) {
          const int g = (meta.w >> 16) & 0xffff, nt = (meta.w >> 8) & 0xff;
          if ((int)atom_add_acq_rel(ctr_seg(a, P) + q * P.nseg + g, (uint32_t)nt) + nt == seg_tiles_of(P, g))
            push_tasks(a, P, 1, [&](int) { return enc_task(T_TOPK1, q, g); });
        }
      }
    }
  }
  // Every role has passed the sentinel (or stopped on an abort): carry the
  // ring positions over to the next run, the producer's (thread 0) for the
  // stages and head blocks, the MMA thread's for the accumulators.
  tc::fence_before_sync();
  wbar();  // every thread has read the positions it started from
  tc::fence_after_sync();
  if (threadIdx.x == 0) {
    h->ss_stage = ss.stage;
    h->ss_phase = (int)ss.phase;
    h->ss_nq = ss.nq;
    h->ss_imask = ss.issued_mask;
    h->ss_iphase = ss.issued_phase;
  }
  if (warp == kMmaWarp && lane == 0) {
    h->ss_acc = ss.acc;
    h->ss_accph = (int)ss.accph;
  }
}

// ------------------------------------------------------------------ TOPK

// Bulk-copy `bytes` (a multiple of 16) from global memory into the region
// and wait for it (all workers). The source was written by other CTAs and
// published with release semantics; the caller has acquired it.
__device__ void bulk_load(const StepArgs &a, Hdr *h, void *dst, const void *src, uint32_t bytes) {
  if (threadIdx.x == 0) {
    asm volatile("fence.proxy.async.global;" ::: "memory");  // generic-proxy writes, read by the async proxy
    tc::mbar_arrive_expect_tx(&h->bulk, bytes);
    for (uint32_t o = 0; o < bytes; o += 16384)
      bulk_g2s(static_cast<uint8_t *>(dst) + o, static_cast<const uint8_t *>(src) + o, min(16384u, bytes - o), &h->bulk);
  }
  const int n = h->bulk_n;
  mwait(&h->bulk, n & 1, &h->abort, a.status, h->wait_ns);
  wbar();
  if (threadIdx.x == 0) h->bulk_n = n + 1;
}

__device__ void topk1_task(const StepArgs &a, const StepPlan &P, Hdr *h, uint8_t *region, int q, int g) {
  uint32_t *keys = reinterpret_cast<uint32_t *>(region);
  uint32_t *hist = keys + kSegMax;
  const int n = clamp_count(a.n_cmp[q], a.N_max, threadIdx.x == 0 ? a.status : nullptr);
  const int k = a.k;
  const bool single = P.nseg == 1;
  const int j0 = g * P.seg_entries;
  const int len = max(0, min(P.seg_entries, n - j0));
  const float *s = a.scores + (size_t)q * P.sstride + j0;
  if (single && n <= k) {
    for (int i = threadIdx.x; i < k; i += kWorkers) a.idx[(size_t)q * k + i] = i < n ? i : -1;
  } else if (!single && len <= k) {
    const size_t cb = ((size_t)q * P.nseg + g) * k;
    for (int i = threadIdx.x; i < len; i += kWorkers) {
      a.cand_key[cb + i] = score_key(__ldcg(s + i));
      a.cand_idx[cb + i] = j0 + i;
    }
    if (threadIdx.x == 0) a.cand_cnt[q * P.nseg + g] = len;
  } else {
    // the segment's scores in one bulk copy (rows are 128-byte aligned), then keys in place
    bulk_load(a, h, keys, s, (uint32_t)((len + 3) & ~3) * 4);
    for (int i = threadIdx.x; i < len; i += kWorkers) keys[i] = score_key(__uint_as_float(keys[i]));
    wbar();
    if (single) {
      int32_t *out = a.idx + (size_t)q * k;
      bsel::select<kWorkers, kHist1>(h->sel, hist, keys, len, k, kBarWork,
                                     [&](uint32_t slot, int j) { out[slot] = j; });
    } else {
      const size_t cb = ((size_t)q * P.nseg + g) * k;
      bsel::select<kWorkers, kHist1>(h->sel, hist, keys, len, k, kBarWork,
                                     [&](uint32_t slot, int j) {
                                       a.cand_key[cb + slot] = keys[j];
                                       a.cand_idx[cb + slot] = j0 + j;
                                     });
      if (threadIdx.x == 0) a.cand_cnt[q * P.nseg + g] = k;
    }
  }
  wbar();
  if (threadIdx.x == 0) {
    if (single) {
      complete_dep(a, P, q);
    } else if ((int)atom_add_acq_rel(ctr_sel(a, P) + q, 1u) + 1 == P.nseg) {
      push_tasks(a, P, 1, [&](int) { return enc_task(T_TOPK2, q, 0); });
    }
  }
}

__device__ void topk2_task(const StepArgs &a, const StepPlan &P, Hdr *h, uint8_t *region, int q) {
  uint32_t *keys = reinterpret_cast<uint32_t *>(region);
  int32_t *pos = reinterpret_cast<int32_t *>(keys + kCandCap);
  uint32_t *hist = reinterpret_cast<uint32_t *>(pos + kCandCap);
  const int k = a.k;
  if (threadIdx.x < 32) {  // segment offsets (the candidates are ascending in position)
    int total = 0;
    for (int g0 = 0; g0 < P.nseg; g0 += 32) {
      const int g = g0 + (int)threadIdx.x;
      const int c = g < P.nseg ? (int)__ldcg(a.cand_cnt + q * P.nseg + g) : 0;
      int x = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if ((int)threadIdx.x >= o) x += y;
      }
      if (g < P.nseg) h->offs[g] = total + x - c;
      total += __shfl_sync(0xffffffffu, x, 31);
    }
    if (threadIdx.x == 0) h->offs[P.nseg] = total;
  }
  wbar();
  const int total = h->offs[P.nseg];
  for (int g = 0; g < P.nseg; ++g) {
    const int o = h->offs[g], c = h->offs[g + 1] - o;
    const size_t cb = ((size_t)q * P.nseg + g) * k;
    for (int i = threadIdx.x; i < c; i += kWorkers) {
      keys[o + i] = __ldcg(a.cand_key + cb + i);
      pos[o + i] = __ldcg(a.cand_idx + cb + i);
    }
  }
  wbar();
  int32_t *out = a.idx + (size_t)q * k;
  if (total <= k) {
    for (int i = threadIdx.x; i < k; i += kWorkers) out[i] = i < total ? pos[i] : -1;
  } else {
    bsel::select<kWorkers, kHist2>(h->sel, hist, keys, total, k, kBarWork,
                                   [&](uint32_t slot, int j) { out[slot] = pos[j]; });
  }
  wbar();
  if (threadIdx.x == 0) complete_dep(a, P, q);
}

// ------------------------------------------------------------------ MQA
// One split of one query group's row list through the tensor-core attention
// pipeline of the stand-alone kernel (transposed S^T / O^T products, two KV
// tile buffers, cp.async gathers for selected rows and TMA boxes for
// contiguous runs, online softmax with a lazy 2^8 rescale). The barrier
// parities continue across the CTA's attention tasks: LI counts the CTA's
// tiles, mt its tasks.

// Row list of query q. CSA: [window rows, padded to win_tiles x 64 | the k
// selected entries]; HCA: [the n visible entries, padded to a multiple of 4 |
// the window rows].
struct RowList {
  int nsel, sel_r0, win_r0, wlo, wcount, R, tiles;
};

__device__ __forceinline__ RowList row_list(const StepArgs &a, const StepPlan &P, int q, uint32_t *status) {
  RowList L;
  int e = a.win_end[q];
  if (e < 0 || e >= a.T_raw) {
    raise_status(status, CSA_STATUS_BAD_WINDOW);
    e = e < 0 ? 0 : a.T_raw - 1;
  }
  L.wlo = max(0, e - a.win_len + 1);
  L.wcount = e - L.wlo + 1;
  if (P.mode == 0) {
    L.nsel = a.k;
    L.win_r0 = 0;
    L.sel_r0 = P.win_tiles * kRows;
    L.R = L.sel_r0 + a.k;
    L.tiles = P.win_tiles + P.sel_tiles;
  } else {
    L.nsel = clamp_count(a.n_cmp[q], a.N_max, status);
    L.sel_r0 = 0;
    L.win_r0 = (L.nsel + 3) & ~3;
    L.R = L.win_r0 + L.wcount;
    L.tiles = (L.R + kRows - 1) / kRows;
  }
  return L;
}

__device__ void mqa_task(const StepArgs &a, const StepPlan &P, Hdr *h, uint8_t *region, uint32_t tmem,
                         const CUtensorMap *tm_q, const CUtensorMap *tm_cmp, const CUtensorMap *tm_win, int qv,
                         int s) {
  uint8_t *kv = region;                      // [2 tiles][8 boxes][64 rows][128 B]
  uint8_t *qs = region + 2 * kTileBytes;     // [8 boxes][64 heads][128 B]
  uint8_t *ps = qs + kQBytes;                // [2][64 rows][128 B]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = qv / P.G, hg = qv - q * P.G;
  const int b = q / a.q_per_seq;
  volatile int *abort = &h->abort;
  const uint64_t lim = h->wait_ns;
  const bool sparse = P.mode == 0;
  const RowList L = row_list(a, P, q, threadIdx.x == 0 ? a.status : nullptr);
  int t0, t1;
  if (sparse) {
    if (s == 0) {
      t0 = 0;
      t1 = P.win_tiles;
    } else {
      t0 = P.win_tiles + (s - 1) * P.tps;
      t1 = min(P.win_tiles + P.sel_tiles, t0 + P.tps);
    }
  } else {
    t0 = s * P.tps;
    t1 = min(L.tiles, t0 + P.tps);
  }
  const int ntiles = max(0, t1 - t0);
  const int LI0 = h->ms_LI, mt = h->ms_mt, mq = h->ms_mq;
  const int32_t *idxq = a.idx + (size_t)q * a.k;
  // entry at selected list position p (CSA)
  auto sel_at = [&](int p) -> int { return (int)__ldcg(idxq + p); };
  // is list row r a live row (masked otherwise)
  auto valid_row = [&](int r, int j) -> bool {
    if (sparse) {
      if (r < L.sel_r0) return r < L.wcount;
      return r - L.sel_r0 < L.nsel && j >= 0 && j < a.N_max;
    }
    return r < L.win_r0 ? r < L.nsel : r < L.R;
  };

  if (threadIdx.x < kH) {
    h->mref[threadIdx.x] = -INFINITY;
    h->alpha[threadIdx.x] = 1.f;
  }
  wbar();
  if (warp == kMmaWarp && lane == 0 && ntiles > 0) {
    asm volatile("fence.proxy.async.global;" ::: "memory");  // rows appended in this launch, read by TMA
    tc::mbar_arrive_expect_tx(&h->q_full, kQBytes);
    for (int bx = 0; bx < kD / 64; ++bx) tc::tma_load_2d(qs + bx * kQBoxBytes, tm_q, bx * 64, qv * kH, &h->q_full);
  }

  if (warp < kLoadWarps) {
    const int g = warp / kWarpsPerBuf, part = warp % kWarpsPerBuf;
    const uint32_t buf_base = tc::smem_u32(kv) + g * kTileBytes;
    if (lane == 0 && part == 0) asm volatile("fence.proxy.async.global;" ::: "memory");
    auto src_row = [&](int r) -> const bf16 * {
      if (sparse) {
        if (r < L.sel_r0)
          return r < L.wcount ? static_cast<const bf16 *>(a.kv_win) + ((size_t)b * a.T_raw + L.wlo + r) * kD
                              : nullptr;
        const int p = r - L.sel_r0;
        if (p >= L.nsel) return nullptr;
        int j = sel_at(p);
        if (j < -1 || j >= a.N_max) {
          raise_status(a.status, CSA_STATUS_BAD_INDEX);
          j = -1;
        }
        return j >= 0 ? static_cast<const bf16 *>(a.kv_cmp) + ((size_t)b * a.N_max + j) * kD : nullptr;
      }
      if (r < L.nsel) return static_cast<const bf16 *>(a.kv_cmp) + ((size_t)b * a.N_max + r) * kD;
      if (r >= L.win_r0 && r < L.R)
        return static_cast<const bf16 *>(a.kv_win) + ((size_t)b * a.T_raw + L.wlo + (r - L.win_r0)) * kD;
      return nullptr;
    };
    // a tile that is one contiguous run of rows: window rows, or dense entries
    auto is_run = [&](int r0, bool &win_run, int &src_row0) {
      if (sparse) {
        win_run = r0 < L.sel_r0;
        src_row0 = b * a.T_raw + L.wlo + r0;
        return win_run;
      }
      win_run = r0 >= L.win_r0;
      src_row0 = win_run ? b * a.T_raw + L.wlo + (r0 - L.win_r0) : b * a.N_max + r0;
      return win_run || r0 + kRows <= L.nsel;
    };
    auto prefetch_l2 = [&](int li) {
      if (li >= ntiles) return;
      const int r0 = (t0 + li) * kRows;
      bool win_run;
      int srow;
      if (is_run(r0, win_run, srow)) {
        if (lane == 0) {
          const int first = srow + kRowsPerWarp * part;
          const int limit = win_run ? (b + 1) * a.T_raw : (b + 1) * a.N_max;
          const int rows = min(kRowsPerWarp, limit - first);
          if (rows > 0) {
            const bf16 *base = static_cast<const bf16 *>(win_run ? a.kv_win : a.kv_cmp) + (size_t)first * kD;
            bulk_prefetch_l2(base, (uint32_t)rows * kD * 2);
          }
        }
      } else if (lane < kRowsPerWarp) {
        if (const bf16 *p = src_row(r0 + kRowsPerWarp * part + lane)) bulk_prefetch_l2(p, kD * 2);
      }
    };
    int last = -1;
    // this group's tiles: LI = LI0 + li with LI = g (mod 2)
    for (int li = ((g - LI0) & 1); li < ntiles; li += 2) {
      const int LI = LI0 + li;
      const int r0 = (t0 + li) * kRows;
      bool win_run;
      int srow;
      const bool run = is_run(r0, win_run, srow);
      __syncwarp();
      if (!run && lane < kRowsPerWarp) h->rowp[warp][lane] = src_row(r0 + kRowsPerWarp * part + lane);
      if (li < 2) {  // the first tile streams in order too; later tiles are prefetched kAhead rounds ahead
        if (run) prefetch_l2(li);
        for (int r = 1; r <= kAhead; ++r) prefetch_l2(li + 2 * r);
      }
      if (!__all_sync(0xffffffffu, mwait(&h->kv_empty[g], ((LI >> 1) & 1) ^ 1, abort, a.status, lim))) break;
      if (run) {
        if (part == 0 && lane == 0) {
          tc::mbar_arrive_expect_tx(&h->kv_full[g], kTileBytes);
          for (int bx = 0; bx < 8; ++bx)
            tc::tma_load_2d(kv + g * kTileBytes + bx * kBoxBytes, win_run ? tm_win : tm_cmp, 64 * bx, srow,
                            &h->kv_full[g]);
        } else {
          tc::mbar_arrive(&h->kv_full[g]);
        }
      } else {
        __syncwarp();
#pragma unroll 8
        for (int i = 0; i < 2 * kRowsPerWarp; ++i) {
          const int rw = i >> 1, c16 = lane + 32 * (i & 1);
          const int row = kRowsPerWarp * part + rw;
          const bf16 *src = h->rowp[warp][rw];
          const uint32_t dst = buf_base + (c16 >> 3) * kBoxBytes + row * 128 + (((c16 & 7) ^ (row & 7)) << 4);
          cp_async16(dst, src ? src + c16 * 8 : static_cast<const bf16 *>(a.kv_win), src != nullptr);
        }
      }
      if (li >= 2) prefetch_l2(li + 2 * kAhead);
      if (!run) {
        cp_async_wait_all();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc::mbar_arrive(&h->kv_full[g]);
      }
      last = LI;
    }
    if (part == 0 && lane == 0 && last >= 0) tc::mbar_drain(&h->kv_full[g], (last >> 1) & 1);
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16(64, 64, 0, 0);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(128, 64, 1, 1);
      const uint32_t kv_base = tc::smem_u32(kv), q_base = tc::smem_u32(qs), p_base = tc::smem_u32(ps);
      bool ok = ntiles == 0 || mwait(&h->q_full, mq & 1, abort, a.status, lim);
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
        const int LP = LI0 + np, LS = LI0 + ns;
        if (np < ns && tc::mbar_test_wait(&h->p_full[LP & 1], (LP >> 1) & 1)) {
          const int pb = LP & 1;
          tc::fence_after_sync();
          const uint64_t ad0 = ad_v + (uint64_t)((pb * kTileBytes) >> 4), bd0 = bd_p + (uint64_t)((pb * kPBytes) >> 4);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
#pragma unroll
            for (int j = 0; j < kRows / 16; ++j)
              tc::mma_bf16(tmem + kColO + 64 * m, ad0 + (uint64_t)((2 * m * kBoxBytes + j * 2048) >> 4),
                           bd0 + (uint64_t)((j * 2048) >> 4), idesc_pv, np > 0 || j > 0);
          }
          tc::commit(&h->kv_empty[pb]);
          tc::commit(&h->pv_done[LP & 3]);
          ++np;
          progressed = true;
        }
        // S^T(ns) overwrites the S^T buffer of tile ns - 2: P.V(ns - 2) must
        // have been issued, i.e. its softmax has finished reading it.
        if (ns < ntiles && ns <= np + 1 && tc::mbar_test_wait(&h->kv_full[LS & 1], (LS >> 1) & 1)) {
          const int buf = LS & 1;
          tc::fence_after_sync();
          const uint64_t ad0 = ad_kv + (uint64_t)((buf * kTileBytes) >> 4);
#pragma unroll
          for (int j = 0; j < kD / 16; ++j)
            tc::mma_bf16(tmem + kColS + 64 * buf, ad0 + (uint64_t)(((j >> 2) * kBoxBytes + (j & 3) * 32) >> 4),
                         bd_q + (uint64_t)(((j >> 2) * kQBoxBytes + (j & 3) * 32) >> 4), idesc_s, j > 0);
          tc::commit(&h->s_full[buf]);
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
      tc::commit(&h->o_done);
      tc::mbar_drain(&h->o_done, mt & 1);
      if (ntiles > 0) tc::mbar_drain(&h->q_full, mq & 1);
    }
  } else {
    // ---------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int rq = lane >> 2, cq = lane & 3;
    const int rowA = quarter * 16 + rq, rowB = rowA + 8;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const bool leader = warp == kSoftWarp0;
    float l[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) l[i] = 0.f;
    bool ok = true;
    // the selected entries of this thread's two rows of the next tile
    auto entry_of = [&](int r) -> int {
      if (!sparse || r < L.sel_r0) return 0;
      const int p = r - L.sel_r0;
      return p < L.nsel ? sel_at(p) : -1;
    };
    int idxA = 0, idxB = 0;
    if (ntiles > 0) {
      idxA = entry_of(t0 * kRows + rowA);
      idxB = entry_of(t0 * kRows + rowB);
    }
    for (int li = 0; li < ntiles; ++li) {
      const int LI = LI0 + li, buf = LI & 1;
      const bool got = __all_sync(0xffffffffu, mwait(&h->s_full[buf], (LI >> 1) & 1, abort, a.status, lim));
      tc::fence_after_sync();
      const int rA = (t0 + li) * kRows + rowA, rB = rA + 8;
      const bool validA = valid_row(rA, idxA), validB = valid_row(rB, idxB);
      if (li + 1 < ntiles) {
        idxA = entry_of(rA + kRows);
        idxB = entry_of(rB + kRows);
      }
      uint32_t v[32];
      tmem_ld_16x256b_x8(tmem + lane_off + kColS + 64 * buf, v);
      tc::tmem_ld_wait();
      const float sl2 = a.scale_log2;
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          v[4 * c + e] = __float_as_uint(validA ? __uint_as_float(v[4 * c + e]) * sl2 : -INFINITY);
          v[4 * c + 2 + e] = __float_as_uint(validB ? __uint_as_float(v[4 * c + 2 + e]) * sl2 : -INFINITY);
        }
      bool over = false;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float2 mr = *reinterpret_cast<const float2 *>(&h->mref[8 * c + 2 * cq]);
        over |= __uint_as_float(v[4 * c]) > mr.x + kRescaleLog2 || __uint_as_float(v[4 * c + 1]) > mr.y + kRescaleLog2 ||
                __uint_as_float(v[4 * c + 2]) > mr.x + kRescaleLog2 || __uint_as_float(v[4 * c + 3]) > mr.y + kRescaleLog2;
      }
      if (leader && lane == 0) h->need[(LI + 2) & 3] = 0;  // slot of tile LI + 2, last read at tile LI - 2
      if (__any_sync(0xffffffffu, over) && lane == 0) atomicOr(&h->need[LI & 3], 1);
      if (bar_any(kBarSoft, 128, !(got && ok))) {
        ok = false;
        break;
      }
      bool rescale = false;
      if (h->need[LI & 3] != 0) {
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
            for (int e = 0; e < 2; ++e) h->red[quarter][8 * c + 2 * cq + e] = mx[2 * c + e];
        }
        named_sync(kBarSoft, 128);
        if (leader) {
          bool any = false;
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int hh = 2 * lane + i;
            const float tm = fmaxf(fmaxf(h->red[0][hh], h->red[1][hh]), fmaxf(h->red[2][hh], h->red[3][hh]));
            const float mo = h->mref[hh];
            float al = 1.f;
            if (mo == -INFINITY || tm > mo + kRescaleLog2) {
              const float mn = fmaxf(mo, tm);
              al = mo == -INFINITY ? 0.f : exp2f(mo - mn);
              h->mref[hh] = mn;
              any |= mo != -INFINITY;
            }
            h->alpha[hh] = al;
          }
          any = __any_sync(0xffffffffu, any);
          if (lane == 0) h->rescale = any ? 1 : 0;
        }
        named_sync(kBarSoft, 128);
        rescale = h->rescale != 0;
        if (rescale) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float2 al = *reinterpret_cast<const float2 *>(&h->alpha[8 * c + 2 * cq]);
            l[2 * c] *= al.x;
            l[2 * c + 1] *= al.y;
          }
        }
      }
      {
        const uint32_t pbase = tc::smem_u32(ps) + buf * kPBytes + 4 * cq;
        const uint32_t swz = rowA & 7;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float2 mr = *reinterpret_cast<const float2 *>(&h->mref[8 * c + 2 * cq]);
          const float pa0 = validA ? ex2_approx(__uint_as_float(v[4 * c]) - mr.x) : 0.f;
          const float pa1 = validA ? ex2_approx(__uint_as_float(v[4 * c + 1]) - mr.y) : 0.f;
          const float pb0 = validB ? ex2_approx(__uint_as_float(v[4 * c + 2]) - mr.x) : 0.f;
          const float pb1 = validB ? ex2_approx(__uint_as_float(v[4 * c + 3]) - mr.y) : 0.f;
          __nv_bfloat162 ta = __floats2bfloat162_rn(pa0, pa1), tb = __floats2bfloat162_rn(pb0, pb1);
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
        // first (only then: see the stand-alone attention kernel; one barrier
        // per tile slot mod 4)
        ok = __all_sync(0xffffffffu, mwait(&h->pv_done[(LI - 1) & 3], ((LI - 1) >> 2) & 1, abort, a.status, lim));
        tc::fence_after_sync();
        if (ok) {
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              uint32_t w[32];
              const uint32_t ta = tmem + lane_off + kColO + 64 * m + 32 * half;
              tc::tmem_ld32(ta, w);
              tc::tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 32; ++c) w[c] = __float_as_uint(__uint_as_float(w[c]) * h->alpha[32 * half + c]);
              tmem_st32(ta, w);
            }
          }
          tmem_st_wait();
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc::fence_before_sync();
      tc::mbar_arrive(&h->p_full[buf]);
    }
    // ---- epilogue
    ok = __all_sync(0xffffffffu, ok && (ntiles == 0 || mwait(&h->o_done, mt & 1, abort, a.status, lim)));
    tc::fence_after_sync();
#pragma unroll
    for (int o = 4; o < 32; o <<= 1)
#pragma unroll
      for (int i = 0; i < 16; ++i) l[i] += __shfl_xor_sync(0xffffffffu, l[i], o);
    if (rq == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int e = 0; e < 2; ++e) h->red[quarter][8 * c + 2 * cq + e] = l[2 * c + e];
    }
    ok = !bar_any(kBarSoft, 128, !ok);
    if (leader) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int hh = 2 * lane + i;
        h->lsum[hh] = (h->red[0][hh] + h->red[1][hh]) + (h->red[2][hh] + h->red[3][hh]);
      }
    }
    named_sync(kBarSoft, 128);
    const int orow = quarter * 32 + lane;
    if (P.S > 1) {
      const size_t pidx = (size_t)qv * P.S + s;
      if (leader) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int hh = 2 * lane + i;
          a.part_ml[(pidx * 2) * kH + hh] = h->mref[hh];
          a.part_ml[(pidx * 2 + 1) * kH + hh] = h->lsum[hh];
        }
      }
      float *po = a.part_o + pidx * (size_t)kH * kD;
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + orow;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t w[32];
          if (ok && ntiles > 0) {
            tc::tmem_ld32(tmem + lane_off + kColO + 64 * m + 32 * half, w);
            tc::tmem_ld_wait();
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) w[c] = 0u;
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) po[(size_t)(32 * half + c) * kD + d] = __uint_as_float(w[c]);
        }
      }
      named_sync(kBarSoft, 128);
      if (leader && lane == 0 && (int)atom_add_acq_rel(ctr_arr(a, P) + qv, 1u) + 1 == P.S)
        push_tasks(a, P, P.P, [&](int i) { return enc_task(T_MERGE, qv, i); });
    } else if (ok) {
      if (leader) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int hh = 2 * lane + i;
          const float mr = h->mref[hh], sk = a.sink[hg * kH + hh] * kLog2e;
          const float M = fmaxf(mr, sk);
          const float wm = mr == -INFINITY ? 0.f : exp2f(mr - M);
          h->alpha[hh] = wm / (h->lsum[hh] * wm + exp2f(sk - M));
        }
      }
      named_sync(kBarSoft, 128);
      bf16 *out = static_cast<bf16 *>(a.out) + (size_t)qv * kH * kD;
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + orow;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t w[32];
          tc::tmem_ld32(tmem + lane_off + kColO + 64 * m + 32 * half, w);
          tc::tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 32; ++c)
            out[(size_t)(32 * half + c) * kD + d] = __float2bfloat16_rn(__uint_as_float(w[c]) * h->alpha[32 * half + c]);
        }
      }
    }
  }
  tc::fence_before_sync();
  wbar();  // every thread has read the positions it started from
  tc::fence_after_sync();
  if (threadIdx.x == 0) {
    h->ms_LI = LI0 + ntiles;
    h->ms_mt = mt + 1;
    h->ms_mq = mq + (ntiles > 0 ? 1 : 0);
  }
}

// ------------------------------------------------------------------ MERGE
// Part p of query group qv's output from its S partials and the sink:
//   M = max(max_s m_s, sink), L = sum_s l_s 2^(m_s - M) + 2^(sink - M),
//   out = sum_s O_s 2^(m_s - M) / L     (m and sink in log2 units).
__device__ void merge_task(const StepArgs &a, const StepPlan &P, Hdr *h, uint8_t *region, int qv, int p) {
  const int S = P.S, hg = qv % P.G;
  const int hpp = kH / P.P;                          // heads of this part
  const uint32_t slice = (uint32_t)hpp * kD * 4;     // bytes of one split's partial for them
  float *po = reinterpret_cast<float *>(region);     // [S][hpp][512]
  float *coef = po + (size_t)S * hpp * kD;           // [S][hpp]
  if (threadIdx.x == 0) {
    asm volatile("fence.proxy.async.global;" ::: "memory");
    tc::mbar_arrive_expect_tx(&h->bulk, slice * S);
    for (int r = 0; r < S; ++r)
      bulk_g2s(po + (size_t)r * hpp * kD, a.part_o + ((size_t)(qv * S + r) * kH + p * hpp) * kD, slice, &h->bulk);
  }
  const float *pml = a.part_ml + (size_t)qv * S * 2 * kH;
  if (threadIdx.x < hpp) {
    const int hh = p * hpp + threadIdx.x;
    const float sk = a.sink[hg * kH + hh] * kLog2e;
    float M = sk;
    for (int r = 0; r < S; ++r) M = fmaxf(M, __ldcg(pml + (2 * r) * kH + hh));
    float Lsum = exp2f(sk - M);
    for (int r = 0; r < S; ++r) {
      const float mr = __ldcg(pml + (2 * r) * kH + hh);
      const float w = mr == -INFINITY ? 0.f : exp2f(mr - M);
      coef[r * hpp + threadIdx.x] = w;
      Lsum += __ldcg(pml + (2 * r + 1) * kH + hh) * w;
    }
    const float inv = 1.f / Lsum;
    for (int r = 0; r < S; ++r) coef[r * hpp + threadIdx.x] *= inv;
  }
  const int n = h->bulk_n;
  mwait(&h->bulk, n & 1, &h->abort, a.status, h->wait_ns);
  wbar();
  if (threadIdx.x == 0) h->bulk_n = n + 1;
  bf16 *out = static_cast<bf16 *>(a.out) + ((size_t)qv * kH + p * hpp) * kD;
  const int groups = hpp * kD / 4;
  for (int gi = threadIdx.x; gi < groups; gi += kWorkers) {
    const int hl = gi / (kD / 4), d = 4 * (gi % (kD / 4));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < S; ++r) {
      const float c = coef[r * hpp + hl];
      const float4 v = *reinterpret_cast<const float4 *>(po + ((size_t)r * hpp + hl) * kD + d);
      acc.x = fmaf(c, v.x, acc.x);
      acc.y = fmaf(c, v.y, acc.y);
      acc.z = fmaf(c, v.z, acc.z);
      acc.w = fmaf(c, v.w, acc.w);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
    *reinterpret_cast<uint2 *>(out + hl * kD + d) =
        make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
  }
  wbar();
}

// ------------------------------------------------------------------ kernel

// 14 warps: one SM sub-partition holds four of them, so a thread may use up
// to 128 of the sub-partition's 16K registers.
template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    decode_step_kernel(const __grid_constant__ CUtensorMap tm_ki, const __grid_constant__ CUtensorMap tm_qi,
                       const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_cmp,
                       const __grid_constant__ CUtensorMap tm_win, const __grid_constant__ StepArgs a,
                       const __grid_constant__ StepPlan P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *region = smem;
  Hdr *h = reinterpret_cast<Hdr *>(smem + kRegionBytes);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&h->full[s], 1);
      tc::mbar_init(&h->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&h->qfull[s], 1);
      tc::mbar_init(&h->qempty[s], 1);
      tc::mbar_init(&h->accfull[s], 2);
      tc::mbar_init(&h->accempty[s], 4 * 32);
      tc::mbar_init(&h->kv_full[s], 32 * kWarpsPerBuf);
      tc::mbar_init(&h->kv_empty[s], 1);
      tc::mbar_init(&h->s_full[s], 1);
      tc::mbar_init(&h->p_full[s], 4 * 32);
    }
    tc::mbar_init(&h->q_full, 1);
    for (int i = 0; i < 4; ++i) tc::mbar_init(&h->pv_done[i], 1);
    tc::mbar_init(&h->o_done, 1);
    tc::mbar_init(&h->mma_drain, 1);
    for (int i = 0; i < 4; ++i) h->need[i] = 0;
    h->mb_full = 0;
    h->busy = 0;
    h->st_pre = -1;
    h->st_done = 0;
    h->bulk_n = 0;
    tc::mbar_init(&h->bulk, 1);
    h->abort = 0;
    h->ss_stage = h->ss_phase = h->ss_nq = h->ss_acc = h->ss_accph = 0;
    h->ss_imask = h->ss_iphase = 0u;
    h->ms_LI = h->ms_mt = h->ms_mq = 0;
    tc::fence_barrier_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(&h->tmem_base, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = h->tmem_base;
  pdl_wait();  // inputs and the counters may come from the previous kernel in the stream
  pdl_release();
  if (threadIdx.x == 0) {
    // bytes 8..15 of the workspace: an optional wait limit in ns (0: 2 s)
    const unsigned long long wl = *reinterpret_cast<const volatile unsigned long long *>(a.status + 2);
    h->wait_ns = wl ? wl : tc::kWaitLimitNs;
    tc::prefetch_tmap(&tm_q);
    tc::prefetch_tmap(&tm_cmp);
    tc::prefetch_tmap(&tm_win);
    if (P.mode == 0) {
      tc::prefetch_tmap(&tm_ki);
      tc::prefetch_tmap(&tm_qi);
    }
  }
  __syncthreads();

  if (warp == kSchedWarp) {
    scheduler(a, P, h);
  } else {
    int4 task = make_int4(T_NONE, 0, 0, 0);
    bool have = false;  // a task left by a scoring run
    for (;;) {
      // the region's next user may write it through TMA (the async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (threadIdx.x == 0) {
        int4 t = have ? h->pending : make_int4(T_NONE, 0, 0, 0);
        if (t.x == T_NONE) t = take_task(a, P, h, false);
        h->cur = t;
      }
      wbar();
      task = h->cur;
      have = false;
      if (task.x == T_EXIT || h->abort) break;
      switch (task.x) {
        case T_SCORE:
          score_run<kFp8>(a, P, h, region, tmem, &tm_ki, &tm_qi, task);
          have = true;
          break;
        case T_APPEND: append_task(a, P, h, region, task.y); break;
        case T_TOPK1: topk1_task(a, P, h, region, task.y, task.z); break;
        case T_TOPK2: topk2_task(a, P, h, region, task.y); break;
        case T_MQA: mqa_task(a, P, h, region, tmem, &tm_q, &tm_cmp, &tm_win, task.y, task.z); break;
        case T_MERGE: merge_task(a, P, h, region, task.y, task.z); break;
        default: break;
      }
      if (h->abort) break;
    }
    // on an abort every CTA stops claiming (the scheduler warp of this CTA
    // watches the shared flag, the others the global one)
    if (threadIdx.x == 0 && h->abort) atomicExch(a.ctr + K_ABORT, 1u);
    // no copy may still be landing in shared memory when the CTA exits (after
    // an abort some were never consumed; a consumed phase completes at once)
    if (threadIdx.x == 0) {
      for (int st = 0; st < kStages; ++st)
        if (h->ss_imask & (1u << st)) tc::mbar_drain(&h->full[st], (h->ss_iphase >> st) & 1);
      for (int i = h->ss_nq - 1; i >= 0 && i >= h->ss_nq - 2; --i) tc::mbar_drain(&h->qfull[i & 1], (i >> 1) & 1);
    }
    // every tensor-core operation this CTA issued has completed before TMEM is freed
    if (warp == kMmaWarp && (threadIdx.x & 31) == 0) {
      tc::commit(&h->mma_drain);
      tc::mbar_drain(&h->mma_drain, 0);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(a.ctr + K_EXIT, 1u) == gridDim.x - 1) {
      // the last CTA: every other CTA has finished; zero the counters for the next launch
      __threadfence();
      for (int i = 0; i < P.n_ctr; ++i) a.ctr[i] = 0u;
      __threadfence();
    }
  }
}

}  // namespace

// ====================================================================== host

namespace {

constexpr int kChunkTiles = 4;
constexpr int kSegEntries = 8192;  // top-k segment (entries; a multiple of the FP8 tile of 256)
static_assert(kSegEntries <= kSegMax, "segment keys fit the selection view");

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct Layout {
  size_t ctr, scores, cand_key, cand_idx, cand_cnt, part_o, part_ml, total;
};

// The fused plan for these arguments, or false when the fused kernel does not
// take them (the separate kernels then run).
bool make_plan(const csa_decode_step_args &s, StepPlan *P) {
  const bool csa = s.qi != nullptr;
  const bool fp8 = csa && s.index_dtype == CSA_DTYPE_E4M3;
  if (s.dtype != CSA_DTYPE_BF16 || s.D != kD || (s.H != kH && s.H != 2 * kH) || s.q_per_seq != 1) return false;
  if (!aligned16(s.q) || !aligned16(s.kv_cmp) || !aligned16(s.kv_win) || !aligned16(s.out)) return false;
  if (s.win_len > 1024 || (long long)s.Q * (s.H / kH) > (1 << 20)) return false;
  if (s.app_kv && (s.app_win > 128 || s.app_T < s.app_win || !aligned16(s.app_kv) || !aligned16(s.app_gate) ||
                   (s.app_kv_seq_stride % 8) || (s.app_gate_seq_stride % 8) || ((reinterpret_cast<uintptr_t>(s.ape) |
                   reinterpret_cast<uintptr_t>(s.norm_w)) & 15)))
    return false;
  StepPlan p{};
  p.mode = csa ? 0 : 1;
  p.fp8 = fp8;
  p.G = s.H / kH;
  p.QV = s.Q * p.G;
  if (csa) {
    if (s.Hi != kHi || s.Di != kDi || s.k < 1 || s.k > CSA_MAX_TOPK) return false;
    if (!(fp8 || s.index_dtype == CSA_DTYPE_BF16)) return false;
    if (!aligned16(s.qi) || !aligned16(s.ki) || !aligned16(s.wi) || (fp8 && !aligned16(s.sq))) return false;
    p.tile_rows = fp8 ? 256 : 128;
    p.tiles_per_q = (s.N_max + p.tile_rows - 1) / p.tile_rows;
    p.chunk_tiles = kChunkTiles;
    p.chunks_per_q = (p.tiles_per_q + kChunkTiles - 1) / kChunkTiles;
    // segments of kSegEntries: the selection of a query's earlier segments
    // runs while its later key tiles are still being scored
    // (longer for long lists, so that the winners of all segments fit one block)
    const int max_seg = kCandCap / s.k;
    int seg = (s.N_max + max_seg - 1) / max_seg;
    seg = ((seg + 1023) / 1024) * 1024;  // whole chunks of tiles (bf16 and FP8)
    p.seg_entries = seg > kSegEntries ? seg : kSegEntries;
    if (p.seg_entries > kSegMax) return false;
    p.seg_tiles = p.seg_entries / p.tile_rows;
    p.nseg = (p.tiles_per_q + p.seg_tiles - 1) / p.seg_tiles;
    if (p.nseg == 1) {
      p.seg_tiles = p.tiles_per_q;
      p.seg_entries = p.tiles_per_q * p.tile_rows;
    }
    if (p.nseg > 64 || (long long)p.nseg * s.k > kCandCap) return false;
    p.sstride = (s.N_max + 31) & ~31;
    p.win_tiles = (s.win_len + kRows - 1) / kRows;
    p.sel_tiles = (s.k + kRows - 1) / kRows;
    p.tps = 2;
    p.S_main = (p.sel_tiles + p.tps - 1) / p.tps;
    p.S = 1 + p.S_main;
  } else {
    const int rows_max = ((s.N_max + 3) & ~3) + s.win_len;
    const int tiles = (rows_max + kRows - 1) / kRows;
    int want = device_sm_count() / (p.QV > 0 ? p.QV : 1);
    want = want < 1 ? 1 : (want > kMaxSplits ? kMaxSplits : want);
    want = want > tiles ? tiles : want;
    p.tps = (tiles + want - 1) / want;
    p.S_main = (tiles + p.tps - 1) / p.tps;
    p.S = p.S_main;
  }
  if (p.S > kMaxSplits) return false;
  // merge parts: each part's slices of all S partials fit the region
  p.P = 0;
  if (p.S > 1) {
    p.P = 4;
    while ((size_t)p.S * (kH / p.P) * kD * 4 + (size_t)p.S * (kH / p.P) * 4 > kRegionBytes) p.P *= 2;
  }
  if (s.app_kv) {
    p.app_per_b = (s.app_T - s.app_win) / s.app_stride + 1;
    p.app_row0 = (int)s.app_row0;
  }
  if (!csa && p.app_per_b > 0) {  // the dense splits holding appended rows wait for the append
    const int tile0 = p.app_row0 / kRows, tile1 = (p.app_row0 + p.app_per_b - 1) / kRows;
    p.dep_s0 = tile0 / p.tps;
    const int s1 = tile1 / p.tps < p.S - 1 ? tile1 / p.tps : p.S - 1;
    p.n_dep = s1 - p.dep_s0 + 1;
  }
  p.deps_target = csa ? 1 + (p.app_per_b > 0 ? 1 : 0) : 0;
  p.n_app = p.app_per_b * s.B;
  p.n_ms = csa ? p.QV : p.QV * (p.S - p.n_dep);
  p.n_chunks = csa ? s.Q * p.chunks_per_q : 0;
  p.n_static = p.n_app + p.n_ms + p.n_chunks;
  p.D = csa ? s.Q * p.nseg + (p.nseg > 1 ? s.Q : 0) + p.QV * p.S_main : p.QV * p.n_dep;
  p.D += p.S > 1 ? p.QV * p.P : 0;
  p.q_off = (kCtrHead + s.Q * (p.nseg + 2) + p.QV + 1) & ~1;  // 8-byte aligned
  p.n_ctr = p.q_off + 2 * p.D;
  *P = p;
  return true;
}

Layout layout_of(const csa_decode_step_args &s, const StepPlan &p) {
  Layout L{};
  size_t o = 256;  // the status word (and the optional wait limit)
  L.ctr = o;
  o += align256((size_t)p.n_ctr * 4);
  if (p.mode == 0) {
    L.scores = o;
    o += align256((size_t)s.Q * p.sstride * 4);
    if (p.nseg > 1) {
      L.cand_key = o;
      o += align256((size_t)s.Q * p.nseg * s.k * 4);
      L.cand_idx = o;
      o += align256((size_t)s.Q * p.nseg * s.k * 4);
      L.cand_cnt = o;
      o += align256((size_t)s.Q * p.nseg * 4);
    }
  }
  if (p.S > 1) {
    L.part_o = o;
    o += align256((size_t)p.QV * p.S * kH * kD * 4);
    L.part_ml = o;
    o += align256((size_t)p.QV * p.S * 2 * kH * 4);
  }
  L.total = o;
  return L;
}

int sm_count_for_grid() { return device_sm_count(); }

template <bool kFp8>
cudaError_t launch_fused(const csa_decode_step_args &s, const StepPlan &p, const Layout &L, char *ws,
                         cudaStream_t stream) {
  CUtensorMap tm_ki{}, tm_qi{}, tm_q{}, tm_cmp{}, tm_win{};
  if (p.mode == 0) {
    const int esz = kFp8 ? 1 : 2, box = kFp8 ? 128 : 64;
    auto mk = kFp8 ? make_tmap_u8_2d : make_tmap_bf16_2d;
    if (!mk(&tm_ki, s.ki, kDi, (uint64_t)s.B * s.N_max, kDi * esz, box, 128)) return cudaErrorInvalidValue;
    if (!mk(&tm_qi, s.qi, kDi, (uint64_t)s.Q * kHi, kDi * esz, box, kHi)) return cudaErrorInvalidValue;
  }
  if (!make_tmap_bf16_2d(&tm_q, s.q, kD, (uint64_t)s.Q * s.H, kD * 2, 64, kH) ||
      !make_tmap_bf16_2d(&tm_cmp, s.kv_cmp, kD, (uint64_t)s.B * s.N_max, kD * 2, 64, kRows) ||
      !make_tmap_bf16_2d(&tm_win, s.kv_win, kD, (uint64_t)s.B * s.T_raw, kD * 2, 64, kRows))
    return cudaErrorInvalidValue;
  if (p.mode != 0) {  // unused by the dense attention, but must be valid maps
    tm_ki = tm_q;
    tm_qi = tm_q;
  }
  StepArgs a{};
  if (s.app_kv) {
    CompressArgs &c = a.app;
    c.kv = s.app_kv;
    c.gate = s.app_gate;
    c.ape = s.ape;
    c.norm_w = s.norm_w;
    c.out = static_cast<bf16 *>(const_cast<void *>(s.kv_cmp)) + (size_t)s.app_row0 * kD;
    c.B = s.B;
    c.T = s.app_T;
    c.D = kD;
    c.win = s.app_win;
    c.stride = s.app_stride;
    c.N = p.app_per_b;
    c.kv_ss = s.app_kv_seq_stride ? s.app_kv_seq_stride : (long long)s.app_T * kD;
    c.gate_ss = s.app_gate_seq_stride ? s.app_gate_seq_stride : (long long)s.app_T * kD;
    c.out_ss = (long long)s.N_max * kD;
    c.dtype = CSA_DTYPE_BF16;
    c.rope_dims = s.rope_dims;
    c.rope_theta = s.rope_theta;
    c.pos0 = s.pos0;
  }
  a.qi = s.qi;
  a.ki = s.ki;
  a.wi = s.wi;
  a.sq = s.sq;
  a.sk = s.sk;
  a.n_cmp = s.n_cmp;
  a.k = s.k;
  a.idx = s.idx_out;
  a.scores = p.mode == 0 ? reinterpret_cast<float *>(ws + L.scores) : nullptr;
  a.q = s.q;
  a.kv_cmp = s.kv_cmp;
  a.kv_win = s.kv_win;
  a.win_end = s.win_end;
  a.sink = s.sink;
  a.scale_log2 = s.scale * kLog2e;
  a.out = s.out;
  a.Q = s.Q;
  a.B = s.B;
  a.H = s.H;
  a.N_max = s.N_max;
  a.win_len = s.win_len;
  a.T_raw = s.T_raw;
  a.q_per_seq = s.q_per_seq;
  a.part_o = p.S > 1 ? reinterpret_cast<float *>(ws + L.part_o) : nullptr;
  a.part_ml = p.S > 1 ? reinterpret_cast<float *>(ws + L.part_ml) : nullptr;
  a.cand_key = p.nseg > 1 ? reinterpret_cast<uint32_t *>(ws + L.cand_key) : nullptr;
  a.cand_idx = p.nseg > 1 ? reinterpret_cast<int32_t *>(ws + L.cand_idx) : nullptr;
  a.cand_cnt = p.nseg > 1 ? reinterpret_cast<int32_t *>(ws + L.cand_cnt) : nullptr;
  a.ctr = reinterpret_cast<uint32_t *>(ws + L.ctr);
  a.status = reinterpret_cast<uint32_t *>(ws);
  static DeviceOnce attr;
  once_per_device(attr, [] {
    cudaFuncSetAttribute(decode_step_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    cudaFuncSetAttribute(decode_step_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  });
  return launch_pdl(decode_step_kernel<kFp8>, dim3((unsigned)sm_count_for_grid()), dim3(kThreads), kSmemBytes, stream,
                    tm_ki, tm_qi, tm_q, tm_cmp, tm_win, a, p);
}

bool nonneg_sizes(const csa_decode_step_args &s) {
  return s.Q >= 1 && s.B >= 1 && s.H >= 1 && s.D >= 1 && s.N_max >= 1 && s.win_len >= 1 && s.T_raw >= 1 &&
         s.q_per_seq >= 1 && (long long)s.B * s.q_per_seq >= s.Q;
}

// Workspace of the separate-kernel path: the calls run one after another on
// one stream, so they share it.
size_t fallback_bytes(const csa_decode_step_args &s) {
  size_t m = csa_mqa_workspace_bytes(s.Q, s.H, s.D, (s.qi ? ((s.k + 3) & ~3) : ((s.N_max + 3) & ~3)) + s.win_len);
  if (s.qi) {
    const size_t t = csa_index_topk_workspace_bytes(s.Q, s.N_max, s.k);
    m = m > t ? m : t;
  }
  return m;
}

}  // namespace

}  // namespace csa

using namespace csa;

extern "C" {

size_t csa_decode_step_workspace_bytes(const csa_decode_step_args *s) {
  if (!s || !nonneg_sizes(*s)) return 256;
  StepPlan p;
  if (s->variant == CSA_STEP_PERSISTENT && make_plan(*s, &p)) return layout_of(*s, p).total;
  return fallback_bytes(*s);
}

int csa_decode_step(const csa_decode_step_args *s, void *ws, size_t ws_bytes, csa_stream_t stream) {
  if (!s || !nonneg_sizes(*s)) return CSA_ERR_INVALID;
  if (s->variant != CSA_STEP_CHAINED && s->variant != CSA_STEP_PERSISTENT) return CSA_ERR_INVALID;
  if (!s->q || !s->kv_cmp || !s->kv_win || !s->win_end || !s->sink || !s->out || !s->n_cmp) return CSA_ERR_INVALID;
  const bool csa = s->qi != nullptr;
  if (csa && (!s->wi || !s->ki || !s->idx_out || s->k < 1 || s->k > CSA_MAX_TOPK ||
              (s->index_dtype == CSA_DTYPE_E4M3 && (!s->sq || !s->sk))))
    return CSA_ERR_INVALID;
  if (s->app_kv && (!s->app_gate || !s->ape || !s->norm_w || s->app_win < 1 || s->app_win > 128 ||
                    s->app_stride < 1 || s->app_T < s->app_win || s->app_row0 < 0))
    return CSA_ERR_INVALID;
  if (s->app_kv) {
    const long long n_new = (s->app_T - s->app_win) / s->app_stride + 1;
    if (s->app_row0 + n_new > s->N_max) return CSA_ERR_INVALID;
  }
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) || ws_bytes < csa_decode_step_workspace_bytes(s))
    return CSA_ERR_WORKSPACE;
  StepPlan p;
  cudaStream_t st = (cudaStream_t)stream;
  if (s->variant == CSA_STEP_PERSISTENT && make_plan(*s, &p)) {
    const Layout L = layout_of(*s, p);
    cudaError_t e = p.fp8 ? launch_fused<true>(*s, p, L, static_cast<char *>(ws), st)
                          : launch_fused<false>(*s, p, L, static_cast<char *>(ws), st);
    if (e == cudaSuccess) return CSA_OK;
    if (e != cudaErrorInvalidValue) {
      note_cuda_error(e);
      return CSA_ERR_CUDA;
    }
    cudaGetLastError();  // a tensor map the encoder rejected: the separate kernels serve the call
  }
  // The chained kernels, one after another on the stream (each launch a
  // programmatic dependent of the one before). CSA: scorer, append, top-k,
  // attention -- the append needs nothing the scorer writes, so it starts
  // at once, on the SMs the scorer's CTAs leave, and waits for the scorer
  // only before it exits (the top-k then follows both); HCA: append,
  // attention.
  int rc = CSA_OK;
  auto append = [&](bool late_wait) -> int {
    if (!s->app_kv) return CSA_OK;
    void *out = static_cast<char *>(const_cast<void *>(s->kv_cmp)) +
                (size_t)s->app_row0 * s->D * (s->dtype == CSA_DTYPE_F32 ? 4 : 2);
    const long long oss = (long long)s->N_max * s->D;
    return compress_call(s->app_kv, s->app_gate, s->ape, s->norm_w, s->app_stride, s->app_win, s->app_stride, out,
                         s->B, s->app_T, s->D, s->app_kv_seq_stride, s->app_gate_seq_stride, oss, s->dtype,
                         s->rope_dims, s->rope_theta, s->pos0, late_wait, st);
  };
  if (csa) {
    const bool fp8 = s->index_dtype == CSA_DTYPE_E4M3;
    rc = fp8 ? check_index_topk_fp8(static_cast<const uint8_t *>(s->qi), s->sq, s->wi,
                                    static_cast<const uint8_t *>(s->ki), s->sk, s->n_cmp, s->k, s->idx_out, s->Q,
                                    s->B, s->Hi, s->Di, s->N_max, s->q_per_seq)
             : check_index_topk(s->qi, s->wi, s->ki, s->n_cmp, s->k, s->idx_out, s->Q, s->B, s->Hi, s->Di,
                                s->N_max, s->q_per_seq, s->index_dtype);
    if (rc) return rc;
    if (ws_bytes < csa_index_topk_workspace_bytes(s->Q, s->N_max, s->k)) return CSA_ERR_WORKSPACE;
    ScoreArgs sa{s->qi, s->wi, s->ki, s->n_cmp, nullptr, s->Q, s->B, s->Hi, s->Di, s->N_max, s->q_per_seq,
                 s->index_dtype, nullptr, fp8 ? s->sq : nullptr, fp8 ? s->sk : nullptr};
    if ((rc = index_scores_into_ws(sa, ws, st))) return rc;
    if ((rc = append(true))) return rc;
    if ((rc = topk_from_ws(sa, s->k, s->idx_out, ws, ws_bytes, st))) return rc;
    // The attention loads the queries and runs the window tiles before it
    // waits for the top-k (which writes none of them).
    return attend_call(s->q, s->kv_cmp, s->idx_out, nullptr, s->kv_win, s->sink, s->scale, s->out, s->Q, s->B, s->H,
                       s->D, s->N_max, s->k, s->win_len, s->win_end, s->T_raw, s->q_per_seq, s->dtype, true, ws,
                       ws_bytes, st);
  }
  if ((rc = append(false))) return rc;
  // HCA: only the tiles holding the appended rows wait for the append (which
  // writes nothing else the attention reads); without an append, the
  // caller's kernel may write anything.
  const int n_new = s->app_kv ? (s->app_T - s->app_win) / s->app_stride + 1 : 0;
  return attend_call(s->q, s->kv_cmp, nullptr, s->n_cmp, s->kv_win, s->sink, s->scale, s->out, s->Q, s->B, s->H, s->D,
                     s->N_max, 0, s->win_len, s->win_end, s->T_raw, s->q_per_seq, s->dtype, s->app_kv != nullptr, ws,
                     ws_bytes, st, s->app_kv ? (int)s->app_row0 : -1, n_new);
}

}  // extern "C"
