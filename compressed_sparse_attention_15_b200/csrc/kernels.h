// Host-side launchers of the kernels, one translation unit per step. Every
// launcher enqueues on `stream`, returns cudaGetLastError() of its launch,
// and assumes its arguments were validated by the C-ABI layer (csa_api.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include <utility>

namespace csa {

// Process-wide count of kernel launches made by the library.
void note_launches(unsigned n);
// Remember (per host thread) a CUDA error a call returns as CSA_ERR_CUDA.
void note_cuda_error(cudaError_t e);

// Launch with programmatic stream serialization: the kernel may begin while
// its predecessor in the stream finishes (it calls pdl_wait() before reading
// inputs). cluster_x > 1 groups consecutive blocks along x into thread-block
// clusters of that size (gridDim.x must be a multiple). Counts the launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               unsigned cluster_x, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  cfg.attrs = attr;
  note_launches(1);
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
  return launch_pdl_cluster(kernel, grid, block, smem, stream, 1u, std::forward<Args>(args)...);
}

struct CompressArgs {
  const void *kv, *gate;
  const float *ape, *norm_w;
  void *out;
  int B, T, D, win, stride, N;
  long long kv_ss, gate_ss, out_ss;  // sequence strides in elements
  int dtype;
  // RoPE on the last rope_dims dims of each entry (0: none): entry j of
  // sequence b at position pos0[b] + j * stride + win - 1, pair i turning by
  // that position times rope_theta^(-2 i / rope_dims).
  int rope_dims = 0;
  double rope_theta = 0.0;
  const int64_t *pos0 = nullptr;
  // 1: the kernel before this one in the stream reads and writes none of
  // kv, gate, ape, norm_w and out (the decode step's scorer): the per-entry
  // window kernel starts at once and waits for it only before exiting (so
  // the kernels after it still follow both); 0: wait before reading anything.
  int late_wait = 0;
};
cudaError_t launch_compress(const CompressArgs &a, cudaStream_t stream);
// The indexer's compressor (pool + RMSNorm + Hadamard rotation; D in 64..512,
// a power of two): rows to a.out in a.dtype, or, with codes != nullptr, E4M3
// codes at the same offsets and one scale per entry (sequence stride scale_ss).
cudaError_t launch_index_compress(const CompressArgs &a, uint8_t *codes, float *scales, long long scale_ss,
                                  cudaStream_t stream);
// Hadamard rotation of rows x [rows, D] into out (dtype), or into E4M3 codes
// + per-row scales when codes != nullptr.
cudaError_t launch_hadamard_rows(const void *x, void *out, uint8_t *codes, float *scales, long long rows, int D,
                                 int dtype, cudaStream_t stream);

struct ScoreArgs {
  const void *qi;
  const float *wi;
  const void *ki;
  const int32_t *n_cmp;
  float *scores;
  int Q, B, Hi, Di, N_max, q_per_seq, dtype;
  uint32_t *status;
  const float *sq = nullptr;  // CSA_DTYPE_E4M3: per (query, head) scale [Q, Hi]
  const float *sk = nullptr;  // CSA_DTYPE_E4M3: per entry scale [B, N_max]
};
cudaError_t launch_index_scores(const ScoreArgs &a, cudaStream_t stream);

struct TopkArgs {
  const float *scores;
  const int32_t *n_cmp;
  int32_t *out_idx;
  int Q, N_max, k;
  uint32_t *status;
};
// scratch (may be null): device memory for the two-stage selection of long
// lists, at least topk_scratch_bytes() bytes; without it one stage is used.
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream, void *scratch, size_t scratch_bytes);
size_t topk_scratch_bytes(int Q, int N_max, int k);

// Host-side checks of csa_index_topk's arguments other than the workspace
// (CSA_OK or the code csa_index_topk would return).
int check_index_topk(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp, int k,
                     const int32_t *out_idx, int Q, int B, int Hi, int Di, int N_max, int q_per_seq, int dtype);
int check_index_topk_fp8(const uint8_t *qi8, const float *sq, const float *wi, const uint8_t *ki8, const float *sk,
                         const int32_t *n_cmp, int k, const int32_t *out_idx, int Q, int B, int Hi, int Di, int N_max,
                         int q_per_seq);
// Scores, then top-k, on `stream` (sa.scores and sa.status are set from ws),
// as one call or as its two launches (other work may go between them).
int index_topk_launch(ScoreArgs sa, int k, int32_t *out_idx, void *ws, size_t ws_bytes, cudaStream_t stream);
int index_scores_into_ws(ScoreArgs sa, void *ws, cudaStream_t stream);
int topk_from_ws(const ScoreArgs &sa, int k, int32_t *out_idx, void *ws, size_t ws_bytes, cudaStream_t stream);
// csa_compress / csa_compress_rope: checks, then the launch; late_wait sets
// CompressArgs::late_wait.
int compress_call(const void *kv, const void *gate, const float *ape, const float *norm_w, int ratio, int win,
                  int stride, void *out, int B, int T, int D, long long kv_seq_stride, long long gate_seq_stride,
                  long long out_seq_stride, int dtype, int rope_dims, double rope_theta, const int64_t *pos0,
                  bool late_wait, cudaStream_t stream);

// ---------------------------------------------------------------- per-device setup
// Kernel attributes are set, and device facts cached, once per device (a
// process may drive several GPUs, from several host threads).
constexpr int kMaxDevices = 64;

struct DeviceOnce {
  std::mutex m;
  bool done[kMaxDevices] = {};
};

// Runs fn on the current device the first time this site is reached there;
// every caller returns only after it has run.
template <class F>
inline void once_per_device(DeviceOnce &o, F fn) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    fn();
    return;
  }
  std::lock_guard<std::mutex> g(o.m);
  if (!o.done[dev]) {
    fn();
    o.done[dev] = true;
  }
}

// SM count of the current device (148 on a B200), cached per device.
inline int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

struct MqaArgs {
  const void *q, *kv_cmp, *kv_win;
  const int32_t *idx;      // null for the dense (HCA) variant
  const int32_t *n_cmp;    // dense variant: visible entries per query
  const int32_t *win_end;
  const float *sink;
  float scale;
  void *out;
  int Q, B, H, D, N_max, k, win_len, T_raw, q_per_seq, dtype;
  void *partials;          // split-K scratch inside the workspace
  size_t partial_bytes;
  uint32_t *status;
  const float *scores;     // non-null: select the top-k of these indexer scores in the kernel (idx unused)
  int32_t *idx_out;        // ... and write the selection here
  // 1: the kernel before this one in the stream writes none of q, kv_win,
  // win_end, sink and n_cmp (the decode step's top-k, or its append for
  // HCA): the tensor-core kernel loads the queries and runs the window tiles
  // before waiting for it; 0: it waits before reading anything. With early
  // set and a dense list (idx null), dep_row0 >= 0 names the only cache rows
  // that kernel writes, [dep_row0, dep_row0 + dep_rows) of every sequence:
  // only tiles holding them wait.
  int early = 0;
  int dep_row0 = -1, dep_rows = 0;
};
cudaError_t launch_mqa(const MqaArgs &a, cudaStream_t stream);
// csa_sparse_mqa (idx given) / hca_mqa (idx null, n_cmp given): checks, then
// the launch; early sets MqaArgs::early.
int attend_call(const void *q, const void *kv_cmp, const int32_t *idx, const int32_t *n_cmp, const void *kv_win,
                const float *sink, float scale, void *out, int Q, int B, int H, int D, int N_max, int k, int win_len,
                const int32_t *win_end, int T_raw, int q_per_seq, int dtype, bool early, void *ws, size_t ws_bytes,
                cudaStream_t stream, int dep_row0 = -1, int dep_rows = 0);
// Top-k selection fused into the tensor-core MQA (a.scores set); *taken is
// false when the shape or the launch plan does not allow it.
cudaError_t launch_topk_mqa_tc(const MqaArgs &a, cudaStream_t stream, bool *taken);
size_t mqa_partial_bytes(int Q, int H, int D, int rows_max);

}  // namespace csa
