// C ABI of libcsa.so (declared in include/csa.h): host-side argument checks,
// workspace carving and dispatch to the kernels. Nothing here allocates,
// frees or synchronises (except csa_workspace_status, which is documented to
// synchronise).
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

using namespace csa;

namespace csa {
static unsigned long long g_launches = 0;
void note_launches(unsigned n) { __atomic_fetch_add(&g_launches, (unsigned long long)n, __ATOMIC_RELAXED); }
static thread_local int g_last_cuda_error = 0;
void note_cuda_error(cudaError_t e) { g_last_cuda_error = (int)e; }
}  // namespace csa

namespace {

constexpr size_t kStatusBytes = 256;

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool device_ok() {
  static int cached[64];  // 0 unknown, 1 sm_100, 2 other (immutable device facts)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
  if (dev < 64 && cached[dev]) return cached[dev] == 1;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  const bool ok = major == 10 && minor == 0;
  if (dev < 64) cached[dev] = ok ? 1 : 2;
  return ok;
}

bool dtype_ok(int dtype) { return dtype == CSA_DTYPE_F32 || dtype == CSA_DTYPE_BF16; }
size_t esize(int dtype) { return dtype == CSA_DTYPE_F32 ? 4 : 2; }
bool ws_aligned(const void *ws) { return (reinterpret_cast<uintptr_t>(ws) & 255) == 0; }
bool elem_aligned(const void *p, int dtype) {
  return (reinterpret_cast<uintptr_t>(p) & (esize(dtype) - 1)) == 0;
}
uint32_t *status_of(void *ws) { return static_cast<uint32_t *>(ws); }

int cuda_rc(cudaError_t e) {
  if (e == cudaSuccess) return CSA_OK;
  note_cuda_error(e);
  return CSA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char *csa_strerror(int code) {
  switch (code) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID: return "CSA_ERR_INVALID: invalid argument (null pointer, size, alignment or ratio)";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED: needs an sm_100 device (B200)";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE: workspace too small or not 256-byte aligned";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA: a CUDA call failed";
    case CSA_ERR_DEVICE: return "CSA_ERR_DEVICE: the workspace status word is set";
    case CSA_ERR_SCRATCH_LIMIT:
      return "CSA_ERR_SCRATCH_LIMIT: the request needs more than the built-in scratch of csa_index_topk_noalloc";
    default: return "unknown csa status code";
  }
}

static int compress_common(const void *kv, const void *gate, const float *ape, const float *norm_w, int ratio,
                           int win, int stride, void *out, int B, int T, int D, long long kv_seq_stride,
                           long long gate_seq_stride, long long out_seq_stride, int dtype, int rope_dims,
                           double rope_theta, const int64_t *pos0, csa_stream_t stream, bool late_wait = false) {
  if (!kv || !gate || !ape || !norm_w || !out) return CSA_ERR_INVALID;
  if (!dtype_ok(dtype) || B < 1 || D < 1 || D > 4096 || win < 1 || win > 128 || stride < 1) return CSA_ERR_INVALID;
  if (ratio != stride || T < win) return CSA_ERR_INVALID;
  if (kv_seq_stride < 0 || gate_seq_stride < 0 || out_seq_stride < 0) return CSA_ERR_INVALID;
  if (!elem_aligned(kv, dtype) || !elem_aligned(gate, dtype) || !elem_aligned(out, dtype)) return CSA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(ape) | reinterpret_cast<uintptr_t>(norm_w)) & 3) return CSA_ERR_INVALID;
  if (rope_dims < 0 || rope_dims > D || rope_dims % 8 || (rope_dims && !(rope_theta > 1.0)) ||
      (reinterpret_cast<uintptr_t>(pos0) & 7))
    return CSA_ERR_INVALID;
  const int N = (T - win) / stride + 1;
  const long long kv_ss = kv_seq_stride ? kv_seq_stride : (long long)T * D;
  const long long g_ss = gate_seq_stride ? gate_seq_stride : (long long)T * D;
  const long long o_ss = out_seq_stride ? out_seq_stride : (long long)N * D;
  if (B > 1 && (kv_ss < (long long)T * D || g_ss < (long long)T * D || o_ss < (long long)N * D)) return CSA_ERR_INVALID;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  CompressArgs a{kv, gate, ape, norm_w, out, B, T, D, win, stride, N, kv_ss, g_ss, o_ss, dtype};
  a.rope_dims = rope_dims;
  a.rope_theta = rope_theta;
  a.pos0 = pos0;
  a.late_wait = late_wait ? 1 : 0;
  return cuda_rc(launch_compress(a, (cudaStream_t)stream));
}

int csa_compress(const void *kv, const void *gate, const float *ape, const float *norm_w, int ratio, int win,
                 int stride, void *out, int B, int T, int D, long long kv_seq_stride, long long gate_seq_stride,
                 long long out_seq_stride, int dtype, csa_stream_t stream) {
  return compress_common(kv, gate, ape, norm_w, ratio, win, stride, out, B, T, D, kv_seq_stride, gate_seq_stride,
                         out_seq_stride, dtype, 0, 0.0, nullptr, stream);
}

int csa_compress_rope(const void *kv, const void *gate, const float *ape, const float *norm_w, int ratio, int win,
                      int stride, void *out, int B, int T, int D, long long kv_seq_stride, long long gate_seq_stride,
                      long long out_seq_stride, int rope_dims, double rope_theta, const int64_t *pos0, int dtype,
                      csa_stream_t stream) {
  return compress_common(kv, gate, ape, norm_w, ratio, win, stride, out, B, T, D, kv_seq_stride, gate_seq_stride,
                         out_seq_stride, dtype, rope_dims, rope_theta, pos0, stream);
}

static bool pow2_dim(int D) { return D == 64 || D == 128 || D == 256 || D == 512; }

int csa_index_compress(const void *kv, const void *gate, const float *ape, const float *norm_w, int ratio, int win,
                       int stride, void *out, float *out_scales, int B, int T, int D, long long kv_seq_stride,
                       long long gate_seq_stride, long long out_seq_stride, int dtype, int out_dtype,
                       csa_stream_t stream) {
  if (!kv || !gate || !ape || !norm_w || !out) return CSA_ERR_INVALID;
  if (!dtype_ok(dtype) || !pow2_dim(D) || B < 1 || win < 1 || win > 128 || stride < 1) return CSA_ERR_INVALID;
  const bool fp8 = out_dtype == CSA_DTYPE_E4M3;
  if (!fp8 && out_dtype != dtype) return CSA_ERR_INVALID;
  if (fp8 && (!out_scales || (reinterpret_cast<uintptr_t>(out_scales) & 3))) return CSA_ERR_INVALID;
  if (ratio != stride || T < win) return CSA_ERR_INVALID;
  if (kv_seq_stride < 0 || gate_seq_stride < 0 || out_seq_stride < 0) return CSA_ERR_INVALID;
  if (!elem_aligned(kv, dtype) || !elem_aligned(gate, dtype) || (!fp8 && !elem_aligned(out, dtype)) ||
      (fp8 && (reinterpret_cast<uintptr_t>(out) & 1)))
    return CSA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(ape) | reinterpret_cast<uintptr_t>(norm_w)) & 3) return CSA_ERR_INVALID;
  const int N = (T - win) / stride + 1;
  const long long kv_ss = kv_seq_stride ? kv_seq_stride : (long long)T * D;
  const long long g_ss = gate_seq_stride ? gate_seq_stride : (long long)T * D;
  const long long o_ss = out_seq_stride ? out_seq_stride : (long long)N * D;
  if (B > 1 && (kv_ss < (long long)T * D || g_ss < (long long)T * D || o_ss < (long long)N * D)) return CSA_ERR_INVALID;
  if (o_ss % D) return CSA_ERR_INVALID;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  CompressArgs a{kv, gate, ape, norm_w, out, B, T, D, win, stride, N, kv_ss, g_ss, o_ss, dtype};
  return cuda_rc(launch_index_compress(a, fp8 ? static_cast<uint8_t *>(out) : nullptr, fp8 ? out_scales : nullptr,
                                       o_ss / D, (cudaStream_t)stream));
}

int csa_hadamard_rows(const void *x, void *out, float *out_scales, long long rows, int D, int dtype, int out_dtype,
                      csa_stream_t stream) {
  if (!x || !out || rows < 0 || !dtype_ok(dtype) || !pow2_dim(D)) return CSA_ERR_INVALID;
  const bool fp8 = out_dtype == CSA_DTYPE_E4M3;
  if (!fp8 && out_dtype != dtype) return CSA_ERR_INVALID;
  if (fp8 && (!out_scales || (reinterpret_cast<uintptr_t>(out_scales) & 3))) return CSA_ERR_INVALID;
  if (!elem_aligned(x, dtype) || (!fp8 && !elem_aligned(out, dtype)) || (fp8 && (reinterpret_cast<uintptr_t>(out) & 1)))
    return CSA_ERR_INVALID;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  return cuda_rc(launch_hadamard_rows(x, fp8 ? nullptr : out, fp8 ? static_cast<uint8_t *>(out) : nullptr,
                                      fp8 ? out_scales : nullptr, rows, D, dtype, (cudaStream_t)stream));
}

size_t csa_topk_workspace_bytes(int Q, int N_max, int k) {
  if (Q < 1 || N_max < 1 || k < 1) return kStatusBytes;
  return kStatusBytes + align256(topk_scratch_bytes(Q, N_max, k));
}

size_t csa_index_topk_workspace_bytes(int Q, int N_max, int k) {
  if (Q < 1 || N_max < 1) return kStatusBytes;
  return kStatusBytes + align256((size_t)Q * N_max * sizeof(float)) + align256(topk_scratch_bytes(Q, N_max, k > 0 ? k : 1));
}

static int check_scores(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp, int Q, int B, int Hi,
                        int Di, int N_max, int q_per_seq, int dtype) {
  if (!qi || !wi || !ki || !n_cmp) return CSA_ERR_INVALID;
  if (!dtype_ok(dtype) || Q < 1 || B < 1 || Hi < 1 || Hi > 128 || Di < 1 || Di > 256 || N_max < 1 ||
      N_max > (1 << 22) || q_per_seq < 1)
    return CSA_ERR_INVALID;
  if ((long long)B * q_per_seq < Q) return CSA_ERR_INVALID;
  if (!elem_aligned(qi, dtype) || !elem_aligned(ki, dtype) || (reinterpret_cast<uintptr_t>(wi) & 3) ||
      (reinterpret_cast<uintptr_t>(n_cmp) & 3))
    return CSA_ERR_INVALID;
  return CSA_OK;
}

int csa_index_scores(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp, float *scores, int Q,
                     int B, int Hi, int Di, int N_max, int q_per_seq, int dtype, void *ws, size_t ws_bytes,
                     csa_stream_t stream) {
  int rc = check_scores(qi, wi, ki, n_cmp, Q, B, Hi, Di, N_max, q_per_seq, dtype);
  if (rc) return rc;
  if (!scores || (reinterpret_cast<uintptr_t>(scores) & 3)) return CSA_ERR_INVALID;
  if (!ws || !ws_aligned(ws) || ws_bytes < kStatusBytes) return CSA_ERR_WORKSPACE;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  ScoreArgs a{qi, wi, ki, n_cmp, scores, Q, B, Hi, Di, N_max, q_per_seq, dtype, status_of(ws)};
  return cuda_rc(launch_index_scores(a, (cudaStream_t)stream));
}

int csa_topk(const float *scores, const int32_t *n_cmp, int k, int32_t *out_idx, int Q, int N_max, void *ws,
             size_t ws_bytes, csa_stream_t stream) {
  if (!scores || !n_cmp || !out_idx) return CSA_ERR_INVALID;
  if (Q < 1 || N_max < 1 || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(scores) | reinterpret_cast<uintptr_t>(n_cmp) |
       reinterpret_cast<uintptr_t>(out_idx)) & 3)
    return CSA_ERR_INVALID;
  if (!ws || !ws_aligned(ws) || ws_bytes < csa_topk_workspace_bytes(Q, N_max, k)) return CSA_ERR_WORKSPACE;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  TopkArgs a{scores, n_cmp, out_idx, Q, N_max, k, status_of(ws)};
  return cuda_rc(launch_topk(a, (cudaStream_t)stream, static_cast<char *>(ws) + kStatusBytes,
                             ws_bytes - kStatusBytes));
}

}  // extern "C"

// The host-side checks of csa_index_topk's arguments other than the
// workspace (also run by the entry point without allocation before it
// touches its built-in buffer).
int csa::check_index_topk(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp, int k,
                          const int32_t *out_idx, int Q, int B, int Hi, int Di, int N_max, int q_per_seq, int dtype) {
  int rc = check_scores(qi, wi, ki, n_cmp, Q, B, Hi, Di, N_max, q_per_seq, dtype);
  if (rc) return rc;
  if (!out_idx || (reinterpret_cast<uintptr_t>(out_idx) & 3) || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  return CSA_OK;
}

// The launches of csa_index_topk / csa_index_topk_fp8 once their arguments
// are checked: the scores into the workspace after the status page, then the
// top-k with the rest of it as scratch. (Also the decode step's chain.)
int csa::index_scores_into_ws(ScoreArgs sa, void *ws, cudaStream_t stream) {
  sa.scores = reinterpret_cast<float *>(static_cast<char *>(ws) + kStatusBytes);
  sa.status = status_of(ws);
  return cuda_rc(launch_index_scores(sa, stream));
}

int csa::topk_from_ws(const ScoreArgs &sa, int k, int32_t *out_idx, void *ws, size_t ws_bytes, cudaStream_t stream) {
  float *scores = reinterpret_cast<float *>(static_cast<char *>(ws) + kStatusBytes);
  TopkArgs ta{scores, sa.n_cmp, out_idx, sa.Q, sa.N_max, k, status_of(ws)};
  const size_t sbytes = align256((size_t)sa.Q * sa.N_max * sizeof(float));
  return cuda_rc(launch_topk(ta, stream, static_cast<char *>(ws) + kStatusBytes + sbytes, ws_bytes - kStatusBytes - sbytes));
}

int csa::index_topk_launch(ScoreArgs sa, int k, int32_t *out_idx, void *ws, size_t ws_bytes, cudaStream_t stream) {
  const int rc = index_scores_into_ws(sa, ws, stream);
  return rc ? rc : topk_from_ws(sa, k, out_idx, ws, ws_bytes, stream);
}

int csa::compress_call(const void *kv, const void *gate, const float *ape, const float *norm_w, int ratio, int win,
                       int stride, void *out, int B, int T, int D, long long kv_seq_stride, long long gate_seq_stride,
                       long long out_seq_stride, int dtype, int rope_dims, double rope_theta, const int64_t *pos0,
                       bool late_wait, cudaStream_t stream) {
  return compress_common(kv, gate, ape, norm_w, ratio, win, stride, out, B, T, D, kv_seq_stride, gate_seq_stride,
                         out_seq_stride, dtype, rope_dims, rope_theta, pos0, (csa_stream_t)stream, late_wait);
}

extern "C" {
static int check_scores_fp8(const uint8_t *qi8, const float *sq, const float *wi, const uint8_t *ki8, const float *sk,
                            const int32_t *n_cmp, int Q, int B, int Hi, int Di, int N_max, int q_per_seq);
}

int csa::check_index_topk_fp8(const uint8_t *qi8, const float *sq, const float *wi, const uint8_t *ki8, const float *sk,
                              const int32_t *n_cmp, int k, const int32_t *out_idx, int Q, int B, int Hi, int Di,
                              int N_max, int q_per_seq) {
  int rc = check_scores_fp8(qi8, sq, wi, ki8, sk, n_cmp, Q, B, Hi, Di, N_max, q_per_seq);
  if (rc) return rc;
  if (!out_idx || (reinterpret_cast<uintptr_t>(out_idx) & 3) || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  return CSA_OK;
}

extern "C" {

int csa_index_topk(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp, int k, int32_t *out_idx,
                   int Q, int B, int Hi, int Di, int N_max, int q_per_seq, int dtype, void *ws, size_t ws_bytes,
                   csa_stream_t stream) {
  int rc = check_scores(qi, wi, ki, n_cmp, Q, B, Hi, Di, N_max, q_per_seq, dtype);
  if (rc) return rc;
  if (!out_idx || (reinterpret_cast<uintptr_t>(out_idx) & 3) || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if (!ws || !ws_aligned(ws) || ws_bytes < csa_index_topk_workspace_bytes(Q, N_max, k)) return CSA_ERR_WORKSPACE;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  ScoreArgs sa{qi, wi, ki, n_cmp, nullptr, Q, B, Hi, Di, N_max, q_per_seq, dtype, status_of(ws)};
  return index_topk_launch(sa, k, out_idx, ws, ws_bytes, (cudaStream_t)stream);
}

static int check_scores_fp8(const uint8_t *qi8, const float *sq, const float *wi, const uint8_t *ki8, const float *sk,
                            const int32_t *n_cmp, int Q, int B, int Hi, int Di, int N_max, int q_per_seq) {
  if (!qi8 || !sq || !wi || !ki8 || !sk || !n_cmp) return CSA_ERR_INVALID;
  if (Q < 1 || B < 1 || Hi < 1 || Hi > 128 || Di < 1 || Di > 256 || N_max < 1 || N_max > (1 << 22) || q_per_seq < 1)
    return CSA_ERR_INVALID;
  if ((long long)B * q_per_seq < Q) return CSA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(sq) | reinterpret_cast<uintptr_t>(wi) | reinterpret_cast<uintptr_t>(sk) |
       reinterpret_cast<uintptr_t>(n_cmp)) & 3)
    return CSA_ERR_INVALID;
  return CSA_OK;
}

int csa_index_scores_fp8(const uint8_t *qi8, const float *sq, const float *wi, const uint8_t *ki8, const float *sk,
                         const int32_t *n_cmp, float *scores, int Q, int B, int Hi, int Di, int N_max, int q_per_seq,
                         void *ws, size_t ws_bytes, csa_stream_t stream) {
  int rc = check_scores_fp8(qi8, sq, wi, ki8, sk, n_cmp, Q, B, Hi, Di, N_max, q_per_seq);
  if (rc) return rc;
  if (!scores || (reinterpret_cast<uintptr_t>(scores) & 3)) return CSA_ERR_INVALID;
  if (!ws || !ws_aligned(ws) || ws_bytes < kStatusBytes) return CSA_ERR_WORKSPACE;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  ScoreArgs a{qi8, wi, ki8, n_cmp, scores, Q, B, Hi, Di, N_max, q_per_seq, CSA_DTYPE_E4M3, status_of(ws), sq, sk};
  return cuda_rc(launch_index_scores(a, (cudaStream_t)stream));
}

int csa_index_topk_fp8(const uint8_t *qi8, const float *sq, const float *wi, const uint8_t *ki8, const float *sk,
                       const int32_t *n_cmp, int k, int32_t *out_idx, int Q, int B, int Hi, int Di, int N_max,
                       int q_per_seq, void *ws, size_t ws_bytes, csa_stream_t stream) {
  int rc = check_scores_fp8(qi8, sq, wi, ki8, sk, n_cmp, Q, B, Hi, Di, N_max, q_per_seq);
  if (rc) return rc;
  if (!out_idx || (reinterpret_cast<uintptr_t>(out_idx) & 3) || k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID;
  if (!ws || !ws_aligned(ws) || ws_bytes < csa_index_topk_workspace_bytes(Q, N_max, k)) return CSA_ERR_WORKSPACE;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  ScoreArgs sa{qi8, wi, ki8, n_cmp, nullptr, Q, B, Hi, Di, N_max, q_per_seq, CSA_DTYPE_E4M3, status_of(ws), sq, sk};
  return index_topk_launch(sa, k, out_idx, ws, ws_bytes, (cudaStream_t)stream);
}

size_t csa_mqa_workspace_bytes(int Q, int H, int D, int rows_max) {
  if (Q < 1 || H < 1 || D < 1 || rows_max < 1) return kStatusBytes;
  return kStatusBytes + align256(mqa_partial_bytes(Q, H, D, rows_max));
}

static int check_mqa(const void *q, const void *kv_cmp, const void *kv_win, const float *sink, const void *out, int Q,
                     int B, int H, int D, int N_max, int win_len, const int32_t *win_end, int T_raw, int q_per_seq,
                     int dtype) {
  if (!q || !kv_cmp || !kv_win || !sink || !out || !win_end) return CSA_ERR_INVALID;
  if (!dtype_ok(dtype) || Q < 1 || B < 1 || H < 1 || H > 128 || D < 1 || D > 1024 || N_max < 1 || win_len < 1 ||
      T_raw < 1 || q_per_seq < 1)
    return CSA_ERR_INVALID;
  if ((long long)B * q_per_seq < Q) return CSA_ERR_INVALID;
  if (!elem_aligned(q, dtype) || !elem_aligned(kv_cmp, dtype) || !elem_aligned(kv_win, dtype) ||
      !elem_aligned(out, dtype) || (reinterpret_cast<uintptr_t>(sink) & 3) ||
      (reinterpret_cast<uintptr_t>(win_end) & 3))
    return CSA_ERR_INVALID;
  return CSA_OK;
}

int csa_sparse_mqa(const void *q, const void *kv_cmp, const int32_t *idx, const void *kv_win, const float *sink,
                   float scale, void *out, int Q, int B, int H, int D, int N_max, int k, int win_len,
                   const int32_t *win_end, int T_raw, int q_per_seq, int dtype, void *ws, size_t ws_bytes,
                   csa_stream_t stream) {
  return attend_call(q, kv_cmp, idx, nullptr, kv_win, sink, scale, out, Q, B, H, D, N_max, k, win_len, win_end,
                     T_raw, q_per_seq, dtype, false, ws, ws_bytes, (cudaStream_t)stream);
}

size_t csa_topk_sparse_mqa_workspace_bytes(int Q, int H, int D, int N_max, int k, int win_len) {
  if (Q < 1 || H < 1 || D < 1 || N_max < 1 || k < 1 || win_len < 0) return kStatusBytes;
  // the selection's scratch and the attention's partials are used one after the other
  const size_t t = topk_scratch_bytes(Q, N_max, k), m = mqa_partial_bytes(Q, H, D, k + win_len);
  return kStatusBytes + align256(t > m ? t : m);
}

int csa_topk_sparse_mqa(const float *scores, const int32_t *n_cmp, int k, int32_t *idx_out, const void *q,
                        const void *kv_cmp, const void *kv_win, const float *sink, float scale, void *out, int Q,
                        int B, int H, int D, int N_max, int win_len, const int32_t *win_end, int T_raw,
                        int q_per_seq, int dtype, void *ws, size_t ws_bytes, csa_stream_t stream) {
  int rc = check_mqa(q, kv_cmp, kv_win, sink, out, Q, B, H, D, N_max, win_len, win_end, T_raw, q_per_seq, dtype);
  if (rc) return rc;
  if (!scores || !n_cmp || !idx_out || k < 1 || k > CSA_MAX_TOPK || (long long)k + win_len > 65536)
    return CSA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(scores) | reinterpret_cast<uintptr_t>(n_cmp) |
       reinterpret_cast<uintptr_t>(idx_out)) & 3)
    return CSA_ERR_INVALID;
  if (!ws || !ws_aligned(ws) || ws_bytes < csa_topk_sparse_mqa_workspace_bytes(Q, H, D, N_max, k, win_len))
    return CSA_ERR_WORKSPACE;
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  char *scratch = static_cast<char *>(ws) + kStatusBytes;
  const size_t scratch_bytes = ws_bytes - kStatusBytes;
  MqaArgs a{q, kv_cmp, kv_win, nullptr, n_cmp, win_end, sink, scale, out, Q, B, H, D, N_max, k, win_len, T_raw,
            q_per_seq, dtype, scratch, scratch_bytes, status_of(ws), scores, idx_out};
  bool taken = false;
  cudaError_t e = launch_topk_mqa_tc(a, (cudaStream_t)stream, &taken);
  if (taken) return cuda_rc(e);
  TopkArgs ta{scores, n_cmp, idx_out, Q, N_max, k, status_of(ws)};
  e = launch_topk(ta, (cudaStream_t)stream, scratch, scratch_bytes);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  a.idx = idx_out;
  a.scores = nullptr;
  a.idx_out = nullptr;
  return cuda_rc(launch_mqa(a, (cudaStream_t)stream));
}

int hca_mqa(const void *q, const void *kv_cmp, const void *kv_win, const float *sink, float scale, void *out, int Q,
            int B, int H, int D, int N_max, const int32_t *n_cmp, int win_len, const int32_t *win_end, int T_raw,
            int q_per_seq, int dtype, void *ws, size_t ws_bytes, csa_stream_t stream) {
  return attend_call(q, kv_cmp, nullptr, n_cmp, kv_win, sink, scale, out, Q, B, H, D, N_max, 0, win_len, win_end,
                     T_raw, q_per_seq, dtype, false, ws, ws_bytes, (cudaStream_t)stream);
}

unsigned long long csa_launch_count(void) { return __atomic_load_n(&csa::g_launches, __ATOMIC_RELAXED); }

int csa_last_cuda_error(void) { return csa::g_last_cuda_error; }

const char *csa_cuda_error_string(int code) { return cudaGetErrorString((cudaError_t)code); }

int csa_workspace_status(void *ws, csa_stream_t stream, uint32_t *status) {
  if (!ws || !status) return CSA_ERR_INVALID;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return CSA_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return CSA_ERR_CUDA;
  *status = v;
  if (v && cudaMemset(ws, 0, sizeof(uint32_t)) != cudaSuccess) return CSA_ERR_CUDA;
  return v ? CSA_ERR_DEVICE : CSA_OK;
}

}  // extern "C"

// The checks and the launch of csa_sparse_mqa (idx given) / hca_mqa (n_cmp
// given); early: see MqaArgs::early (the decode step's chain).
int csa::attend_call(const void *q, const void *kv_cmp, const int32_t *idx, const int32_t *n_cmp, const void *kv_win,
                     const float *sink, float scale, void *out, int Q, int B, int H, int D, int N_max, int k,
                     int win_len, const int32_t *win_end, int T_raw, int q_per_seq, int dtype, bool early, void *ws,
                     size_t ws_bytes, cudaStream_t stream, int dep_row0, int dep_rows) {
  int rc = check_mqa(q, kv_cmp, kv_win, sink, out, Q, B, H, D, N_max, win_len, win_end, T_raw, q_per_seq, dtype);
  if (rc) return rc;
  if (idx) {
    if ((reinterpret_cast<uintptr_t>(idx) & 3) || k < 1 || (long long)k + win_len > 65536) return CSA_ERR_INVALID;
    if (!ws || !ws_aligned(ws) || ws_bytes < csa_mqa_workspace_bytes(Q, H, D, k + win_len)) return CSA_ERR_WORKSPACE;
  } else {
    if (!n_cmp || (reinterpret_cast<uintptr_t>(n_cmp) & 3)) return CSA_ERR_INVALID;
    if (!ws || !ws_aligned(ws) || ws_bytes < csa_mqa_workspace_bytes(Q, H, D, N_max + win_len))
      return CSA_ERR_WORKSPACE;
    k = 0;
  }
  if (!device_ok()) return CSA_ERR_UNSUPPORTED;
  MqaArgs a{q, kv_cmp, kv_win, idx, idx ? nullptr : n_cmp, win_end, sink, scale, out, Q, B, H, D, N_max, k, win_len,
            T_raw, q_per_seq, dtype, static_cast<char *>(ws) + kStatusBytes, ws_bytes - kStatusBytes, status_of(ws)};
  a.early = early ? 1 : 0;
  a.dep_row0 = dep_row0;
  a.dep_rows = dep_rows;
  return cuda_rc(launch_mqa(a, stream));
}
