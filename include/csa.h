/*
 * csa.h -- C ABI of libcsa.so: the hybrid compressed-sparse attention
 * (CSA / HCA) hot path for DeepSeek-V4-Flash shapes on NVIDIA B200 (sm_100a).
 *
 * The method is described in prose in "DeepSeek-V4 Architecture Analysis"
 * (architecture_analysis.py), INNOVATIONS section 1 "COMPRESSED SPARSE
 * ATTENTION (CSA)" and section 2 "UNIFIED HEAD DIMENSION"; the shapes come
 * from the "DeepSeek-V4-Flash" model card, table "Champs bruts du config.json"
 * (head_dim 512, 64 query heads : 1 KV head, index_n_heads 64,
 * index_head_dim 128, index_topk 512, sliding_window 128, rms_norm_eps 1e-6).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    never allocates or frees memory, never synchronises the stream, keeps no
 *    state between calls and may be called from several host threads.
 *  - Tensors are dense, row-major, in the element type `dtype`
 *    (CSA_DTYPE_BF16 or CSA_DTYPE_F32) unless the argument says float / int32.
 *    bf16 tensors whose row length is a multiple of 8 elements and whose base
 *    is 16-byte aligned take the tensor-core / vectorised kernels; everything
 *    else takes the generic kernels (same results within rounding).
 *  - All arithmetic is fp32 (inputs widened from bf16, products accumulated in
 *    fp32); outputs are rounded once to `dtype` (round to nearest even).
 *  - Every argument is checked on the host before any launch. A failed check
 *    returns a non-zero code and launches nothing.
 *  - Values that live in device memory (visible counts, indices, window ends)
 *    cannot be checked on the host: kernels clamp them to the valid range and
 *    raise a bit in the workspace status word (read with
 *    csa_workspace_status) instead of reading out of bounds.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Launches
 *    are asynchronous; a returned CSA_OK means the work was enqueued.
 *  - Workspaces: the caller passes `ws` (device memory, 256-byte aligned) of at
 *    least the size the matching *_workspace_bytes() returns. Its first 256
 *    bytes hold the status word; the library writes the rest freely. The
 *    status word must be zero before the first call (cudaMemset once); calls
 *    only ever OR bits into it.
 *  - Bounded waits: every wait of a tensor-core kernel on its own pipeline
 *    gives up after a time limit, raises CSA_STATUS_WAIT_TIMEOUT, drops the
 *    rest of its work (that output is invalid) and returns, so the context
 *    stays usable. The limit is 2 s unless bytes 8..15 of the workspace hold a
 *    non-zero uint64 number of nanoseconds (for tests of the timeout path;
 *    leave them zero otherwise).
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *csa_stream_t; /* identical to cudaStream_t */

/* Return codes. */
enum {
  CSA_OK = 0,
  CSA_ERR_INVALID = 1,     /* null pointer, bad size, bad alignment, ratio != stride, k too large */
  CSA_ERR_UNSUPPORTED = 2, /* no sm_100 device current, or an uncompiled size/dtype combination */
  CSA_ERR_WORKSPACE = 3,   /* workspace smaller than *_workspace_bytes() */
  CSA_ERR_CUDA = 4,        /* a CUDA launch or attribute call failed */
  CSA_ERR_DEVICE = 5,      /* (csa_workspace_status only) the status word is non-zero */
  CSA_ERR_SCRATCH_LIMIT = 6 /* (csa_index_topk_noalloc only) the request needs more scratch than
                               CSA_NOALLOC_SCRATCH_BYTES */
};

/* Element types of the dtype-typed tensors. */
enum { CSA_DTYPE_F32 = 0, CSA_DTYPE_BF16 = 1, CSA_DTYPE_E4M3 = 2 /* FP8 indexer entry points only */ };

/* Bits of the workspace status word. */
enum {
  CSA_STATUS_BAD_COUNT = 1u,   /* an n_cmp value was < 0 or > N_max; it was clamped */
  CSA_STATUS_BAD_INDEX = 2u,   /* an idx value was < -1 or >= N_max; the row was skipped */
  CSA_STATUS_BAD_WINDOW = 4u,  /* a win_end value was < 0 or >= T_raw; it was clamped */
  CSA_STATUS_WAIT_TIMEOUT = 8u /* a bounded pipeline wait gave up; that output is invalid */
};

/* Largest supported top-k. */
#define CSA_MAX_TOPK 2048

/* Human-readable name of a return code (static string, never NULL). */
const char *csa_strerror(int code);

/* ------------------------------------------------------------------------
 * csa_num_entries, csa_visible_counts -- how many compressed entries exist,
 * and how many a query may read.
 *
 * "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the compressor
 * folds each window of raw tokens into one entry (CSA: windows of 8 tokens
 * every 4, overlapping; HCA: 128 every 128). Entry j covers tokens
 * j*stride .. j*stride + win - 1 (the reading of the window geometry used by
 * csa_compress), and a query at position p may read it iff its whole window
 * lies at or before p:  j*stride + win - 1 <= p.  Hence
 *     n(p) = 0 if p + 1 < win,  else (p + 1 - win) / stride + 1,
 * the number of complete windows in the first p + 1 tokens.
 *
 * csa_num_entries: entries a compressor run over T tokens makes (n(T - 1));
 *   host-only, no GPU needed. Returns -1 if win < 1, stride < 1 or T < 0.
 * csa_visible_counts_host: n_cmp[q] = n(pos[q]) for q < Q on HOST arrays
 *   (pos int64, 8-byte aligned; n_cmp int32); no GPU needed.
 * csa_visible_counts: the same on DEVICE arrays, one kernel on `stream`;
 *   the result is the n_cmp argument of csa_index_topk / hca_mqa /
 *   csa_topk_sparse_mqa for queries at positions pos.
 * Negative positions count 0; counts above INT32_MAX are clamped to it.
 * Both return CSA_ERR_INVALID (Q < 0, win < 1, stride < 1, a null or
 * misaligned pointer with Q > 0) before any work, CSA_ERR_CUDA if the launch
 * fails (for example without an sm_100 device), else CSA_OK. Q = 0 does nothing.
 * ---------------------------------------------------------------------- */
long long csa_num_entries(long long T, int win, int stride);
int csa_visible_counts_host(const int64_t *pos, long long Q, int win, int stride, int32_t *n_cmp);
int csa_visible_counts(const int64_t *pos, long long Q, int win, int stride, int32_t *n_cmp, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_compress -- gated-pooling KV compressor followed by RMSNorm.
 *
 * Defined by "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: a
 * learned gated pooling folds the raw per-token KV of each window into one
 * entry ("4 tokens -> 1, with overlapping windows" for CSA, "128 tokens -> 1"
 * for HCA), using absolute position embeddings within the window and an
 * RMSNorm on the compressed output. For every sequence b, entry j over tokens
 * t = j*stride + i (i = 0..win-1) and dimension d:
 *     a[i,d]   = softmax over i of (gate[b,t,d] + ape[i,d])
 *     c[d]     = sum_i a[i,d] * kv[b,t,d]
 *     out[b,j] = c / sqrt(mean_d c[d]^2 + 1e-6) * norm_w
 * Entries j = 0 .. N-1 with N = (T - win) / stride + 1 (a trailing partial
 * window makes no entry; T < win is an error). CSA uses win 8 / stride 4,
 * HCA win 128 / stride 128.
 *
 *   kv, gate : [B, T, D] dtype; sequence b starts at b * kv_seq_stride
 *              (resp. gate_seq_stride) elements; 0 means T * D.
 *   ape      : [win, D] float32.        norm_w : [D] float32.
 *   ratio    : the compression ratio; must equal `stride`.
 *   out      : [B, N, D] dtype; sequence b starts at b * out_seq_stride
 *              elements (0 means N * D), so entries may be written straight
 *              into a larger cache.
 * Limits: 1 <= win <= 128, 1 <= stride, 1 <= D <= 4096, B >= 1.
 * ---------------------------------------------------------------------- */
int csa_compress(const void *kv, const void *gate, const float *ape, const float *norm_w,
                 int ratio, int win, int stride, void *out,
                 int B, int T, int D,
                 long long kv_seq_stride, long long gate_seq_stride, long long out_seq_stride,
                 int dtype, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_compress_rope -- csa_compress with RoPE on the entries' rope dims,
 * fused: the cache append of a decode step.
 *
 * "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1 (the compressor
 * applies "RoPE on rope dimensions of compressed KV"), section 2 (the last
 * qk_rope_head_dim = 64 of the 512 dims are the rope dims) and
 * ARCHITECTURE_SPEC (compress_rope_theta = 160000). After the pool and the
 * RMSNorm, the last rope_dims dims of entry j of sequence b are rotated in
 * adjacent pairs (d, d + 1), pair i by the angle
 *     (pos0[b] + j * stride + win - 1) * rope_theta^(-2 i / rope_dims),
 * the position of the entry's last raw token (pos0[b]: the absolute position
 * of kv[b, 0]; the angle is formed in double precision).
 * Arguments as csa_compress, plus rope_dims (a multiple of 8, <= D; 0 gives
 * csa_compress), rope_theta (> 1) and pos0 (int64 [B] device array, 8-byte
 * aligned, or NULL for all zeros). Errors as csa_compress, CSA_ERR_INVALID
 * also for a bad rope_dims / rope_theta / pos0.
 * ---------------------------------------------------------------------- */
int csa_compress_rope(const void *kv, const void *gate, const float *ape, const float *norm_w, int ratio, int win,
                      int stride, void *out, int B, int T, int D, long long kv_seq_stride, long long gate_seq_stride,
                      long long out_seq_stride, int rope_dims, double rope_theta, const int64_t *pos0, int dtype,
                      csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_index_compress -- the indexer's own KV compressor, and
 * csa_hadamard_rows -- the rotation of indexer query rows.
 *
 * "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the indexer
 * "has its own dedicated KV compressor with Hadamard rotation". Entry j is
 * csa_compress's entry (same windows, pool, RMSNorm, arguments and
 * strides) rotated by the orthonormal Sylvester-Hadamard matrix:
 *     out[b, j, :] = compress(...)[b, j, :] H_D / sqrt(D).
 * csa_hadamard_rows rotates each row of x [rows, D] the same way (the
 * indexer queries: scores are unchanged in exact arithmetic).
 * out_dtype = dtype writes rows in the input dtype. out_dtype =
 * CSA_DTYPE_E4M3 writes FP8 codes (uint8, same layout) and one float32 scale
 * per row to out_scales ([B, N] with sequence stride out_seq_stride / D, or
 * [rows]): scale = amax|row| / 448 (1 for a zero row), code = E4M3(v / scale)
 * rounded to nearest even, saturating -- the inputs of csa_index_topk_fp8
 * (the model's quantization_config: fmt e4m3, dynamic activation scales,
 * "deepseek-ai/DeepSeek-V4-Flash-0731", table "Config changes").
 * D must be 64, 128, 256 or 512; other limits and errors as csa_compress;
 * out_scales must be a 4-byte aligned device pointer for FP8 output.
 * ---------------------------------------------------------------------- */
int csa_index_compress(const void *kv, const void *gate, const float *ape, const float *norm_w, int ratio, int win,
                       int stride, void *out, float *out_scales, int B, int T, int D, long long kv_seq_stride,
                       long long gate_seq_stride, long long out_seq_stride, int dtype, int out_dtype,
                       csa_stream_t stream);
int csa_hadamard_rows(const void *x, void *out, float *out_scales, long long rows, int D, int dtype, int out_dtype,
                      csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_index_topk -- indexer scores and top-k selection of compressed entries.
 *
 * "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1, Indexer: a
 * learned scorer "selects top-k compressed positions" using "dot-product
 * attention + per-head importance weights". For query q of sequence
 * b = q / q_per_seq and every visible entry j < n_cmp[q]:
 *     s[q,j] = sum_h wi[q,h] * max(0, qi[q,h,:] . ki[b,j,:])     (no scale)
 * and out_idx[q] holds the min(k, n_cmp[q]) entries of largest score, ties
 * resolved towards the smaller j, written in ascending j, followed by -1
 * padding up to k. Scores are fp32 (bf16 products, fp32 accumulation).
 *
 *   qi      : [Q, Hi, Di] dtype.        wi : [Q, Hi] float32.
 *   ki      : [B, N_max, Di] dtype (indexer keys, one cache per sequence).
 *   n_cmp   : [Q] int32 device array, number of entries visible to query q
 *             (0 .. N_max); covers decode (all N) and causal prefill alike.
 *   out_idx : [Q, k] int32.
 * Limits: 1 <= k <= CSA_MAX_TOPK, Hi <= 128, Di <= 256, Q, B >= 1, 1 <= N_max <= 2^22,
 * B * q_per_seq >= Q.
 * Workspace: csa_index_topk_workspace_bytes(Q, N_max, k).
 * ---------------------------------------------------------------------- */
size_t csa_index_topk_workspace_bytes(int Q, int N_max, int k);
int csa_index_topk(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp,
                   int k, int32_t *out_idx,
                   int Q, int B, int Hi, int Di, int N_max, int q_per_seq, int dtype,
                   void *ws, size_t ws_bytes, csa_stream_t stream);

/* The two halves of csa_index_topk, exposed so each can be driven alone.
 * csa_index_scores writes scores[q, j] (float32, row stride N_max) for
 * j < n_cmp[q] and leaves the rest of the row untouched.
 * csa_topk selects from given float32 scores with the same rule as above
 * (-0.0 and +0.0 compare equal); it reads scores[q, j] for j < n_cmp[q] only. */
int csa_index_scores(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp,
                     float *scores, int Q, int B, int Hi, int Di, int N_max, int q_per_seq,
                     int dtype, void *ws, size_t ws_bytes, csa_stream_t stream);
size_t csa_topk_workspace_bytes(int Q, int N_max, int k);
int csa_topk(const float *scores, const int32_t *n_cmp, int k, int32_t *out_idx,
             int Q, int N_max, void *ws, size_t ws_bytes, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_index_scores_fp8 / csa_index_topk_fp8 -- the indexer on FP8 inputs.
 *
 * "deepseek-ai/DeepSeek-V4-Flash-0731", table "Config changes": the model's
 * quantization_config is fmt e4m3, quant_method fp8, dynamic activation
 * scales; "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the
 * indexer is trained quantization-aware. Keys and queries arrive as OCP FP8
 * E4M3 codes (1 byte: sign, 4-bit exponent with bias 7, 3-bit mantissa; NaN
 * at S.1111.111, no infinities) with one positive fp32 scale per row:
 *     qi[q,h,:] = sq[q,h] * e4m3(qi8[q,h,:]),  ki[b,j,:] = sk[b,j] * e4m3(ki8[b,j,:])
 * and the scores and the selection are those of csa_index_scores /
 * csa_index_topk on these values.
 *
 *   qi8 : [Q, Hi, Di] uint8 codes.   sq : [Q, Hi] float32 (> 0).
 *   wi  : [Q, Hi] float32.
 *   ki8 : [B, N_max, Di] uint8 codes. sk : [B, N_max] float32 (> 0).
 *   n_cmp, k, out_idx, scores, q_per_seq, workspace: as for the bf16 calls
 *   (csa_index_topk_workspace_bytes(Q, N_max, k) for the _topk call, 256
 *   bytes for the _scores call).
 * Limits: Hi <= 128, Di <= 256, N_max <= 2^22; the tensor-core path takes
 * Hi = 64, Di = 128 with 16-byte aligned qi8 / ki8 / wi / sq.
 * Returns CSA_ERR_INVALID (null pointer, bad shape, misaligned float or
 * int32 array, k outside 1..CSA_MAX_TOPK) or CSA_ERR_WORKSPACE before any
 * launch.
 * ---------------------------------------------------------------------- */
int csa_index_scores_fp8(const uint8_t *qi8, const float *sq, const float *wi, const uint8_t *ki8, const float *sk,
                         const int32_t *n_cmp, float *scores, int Q, int B, int Hi, int Di, int N_max, int q_per_seq,
                         void *ws, size_t ws_bytes, csa_stream_t stream);
int csa_index_topk_fp8(const uint8_t *qi8, const float *sq, const float *wi, const uint8_t *ki8, const float *sk,
                       const int32_t *n_cmp, int k, int32_t *out_idx, int Q, int B, int Hi, int Di, int N_max,
                       int q_per_seq, void *ws, size_t ws_bytes, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_sparse_mqa -- MQA over the selected compressed entries, the sliding
 * window of raw tokens and a per-head attention sink.
 *
 * "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1 (sliding window:
 * each token attends to its nearest 128 tokens; attention sink: a learnable
 * per-head scalar) and section 2 (key and value share one head_dim = 512
 * representation: K = V). For query q of sequence b = q / q_per_seq, head h:
 *     rows    = { kv_cmp[b, idx[q,r]] : idx[q,r] >= 0 }
 *             U { kv_win[b, t] : max(0, e - win_len + 1) <= t <= e },  e = win_end[q]
 *     logit_r = scale * q[q,h,:] . row_r ;  the sink adds sink[h] (unscaled)
 *               to the softmax denominator with a zero value
 *     out[q,h] = sum_r softmax_r * row_r
 * The window is not de-duplicated against compressed rows.
 *
 *   q       : [Q, H, D] dtype (RoPE already applied).
 *   kv_cmp  : [B, N_max, D] dtype compressed cache.
 *   idx     : [Q, k] int32 (-1 = unused slot).
 *   kv_win  : [B, T_raw, D] dtype raw-KV buffer holding the window tokens.
 *   win_end : [Q] int32 device array, row of kv_win holding query q's token.
 *   sink    : [H] float32.      out : [Q, H, D] dtype.
 * Limits: H <= 128, D <= 1024, k + win_len <= 65536, win_len >= 1.
 * Workspace: csa_mqa_workspace_bytes(Q, H, D, k + win_len).
 * ---------------------------------------------------------------------- */
size_t csa_mqa_workspace_bytes(int Q, int H, int D, int rows_max);
int csa_sparse_mqa(const void *q, const void *kv_cmp, const int32_t *idx, const void *kv_win,
                   const float *sink, float scale, void *out,
                   int Q, int B, int H, int D, int N_max, int k, int win_len,
                   const int32_t *win_end, int T_raw, int q_per_seq, int dtype,
                   void *ws, size_t ws_bytes, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_topk_sparse_mqa -- csa_topk followed by csa_sparse_mqa, as one call.
 *
 * "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the indexer's
 * top-k picks the compressed entries the core attention reads. Given the
 * indexer scores, this call selects with csa_topk's rule, writes the
 * selection to idx_out, and computes csa_sparse_mqa over it; results are
 * those of the two calls in sequence. Where the tensor-core attention runs
 * each query's splits as one thread-block cluster (H = 64 or 128, D = 512,
 * bf16, k <= 1024, slices of at most 32,768 scores per block), the selection
 * is made inside the attention kernel, by the cluster, and the attention
 * starts from it without a kernel boundary; otherwise the two kernels run.
 *
 *   scores  : [Q, N_max] float32 (row stride N_max); entries j < n_cmp[q] read.
 *   n_cmp   : [Q] int32 device array (0 .. N_max), visible entries per query.
 *   idx_out : [Q, k] int32, written (ascending, -1 padded, as csa_topk).
 *   q, kv_cmp, kv_win, win_end, sink, scale, out, shapes, dtype: as
 *   csa_sparse_mqa.
 * Limits: those of csa_topk and csa_sparse_mqa.
 * Workspace: csa_topk_sparse_mqa_workspace_bytes(Q, H, D, N_max, k, win_len).
 * Returns CSA_ERR_INVALID / CSA_ERR_WORKSPACE before any launch.
 * ---------------------------------------------------------------------- */
size_t csa_topk_sparse_mqa_workspace_bytes(int Q, int H, int D, int N_max, int k, int win_len);
int csa_topk_sparse_mqa(const float *scores, const int32_t *n_cmp, int k, int32_t *idx_out,
                        const void *q, const void *kv_cmp, const void *kv_win, const float *sink,
                        float scale, void *out, int Q, int B, int H, int D, int N_max, int win_len,
                        const int32_t *win_end, int T_raw, int q_per_seq, int dtype,
                        void *ws, size_t ws_bytes, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * hca_mqa -- the dense (heavily compressed, 128 tokens -> 1) variant: as
 * csa_sparse_mqa but over every visible compressed entry j < n_cmp[q]
 * instead of an index list ("DeepSeek-V4 Architecture Analysis",
 * INNOVATIONS section 1, "HCA (128:1): heavy compression for global
 * context").
 *   n_cmp : [Q] int32 device array (0 .. N_max).
 * Workspace: csa_mqa_workspace_bytes(Q, H, D, N_max + win_len).
 * ---------------------------------------------------------------------- */
int hca_mqa(const void *q, const void *kv_cmp, const void *kv_win, const float *sink,
            float scale, void *out,
            int Q, int B, int H, int D, int N_max, const int32_t *n_cmp, int win_len,
            const int32_t *win_end, int T_raw, int q_per_seq, int dtype,
            void *ws, size_t ws_bytes, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_index_topk_noalloc -- csa_index_topk for callers that cannot allocate.
 *
 * The pages have no counterpart to this call; it exists for callers that
 * cannot provide device memory of their own: a plugin that only receives the
 * input and output pointers from a host framework whose memory pools it must
 * not bypass, or a latency-bound decode loop that may not call cudaMalloc
 * (which can synchronise the device) in the middle of a step. It computes
 * exactly what csa_index_topk computes, with the same arguments minus the
 * workspace, and allocates nothing: its scratch is a buffer built into the
 * library, CSA_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU that loads
 * the library until the process exits.
 *  - Requests whose csa_index_topk_workspace_bytes(Q, N_max, k) exceeds that
 *    size return CSA_ERR_SCRATCH_LIMIT and launch nothing.
 *  - The first call on a device looks the buffer's device address up (with
 *    that device current); make that first call before any stream capture.
 *  - All calls share the one buffer and it keeps the last call's contents;
 *    calls whose work overlaps on the GPU (different streams or host
 *    threads) race on it. Device-side status bits are cleared at the start
 *    of every call and cannot be read back through this entry point.
 * ---------------------------------------------------------------------- */
#define CSA_NOALLOC_SCRATCH_BYTES (16u << 20)
int csa_index_topk_noalloc(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp, int k,
                           int32_t *out_idx, int Q, int B, int Hi, int Di, int N_max, int q_per_seq,
                           int dtype, csa_stream_t stream);

/* ------------------------------------------------------------------------
 * csa_decode_step -- one whole decode step of a CSA or HCA layer in one call:
 * the cache append, then (CSA) the indexer scores and top-k, then the
 * attention over the selection (CSA) or all visible entries (HCA) plus the
 * window and the sink.
 *
 * "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: each step
 * folds the newest raw window into the compressed cache, the indexer selects
 * the top-k compressed entries (CSA), and the core attention reads them with
 * the 128-token sliding window and the per-head sink; HCA attends to every
 * compressed entry. The results are those of the separate calls in order:
 *   1. if app_kv != NULL: csa_compress (csa_compress_rope if rope_dims > 0)
 *      of app_kv / app_gate [B, app_T, D] (sequence strides app_kv_seq_stride,
 *      app_gate_seq_stride; 0 = app_T * D) with ape [app_win, D], norm_w [D],
 *      window app_win, stride app_stride (= ratio), writing its
 *      N_new = (app_T - app_win) / app_stride + 1 entries of sequence b to
 *      kv_cmp[b, app_row0 .. app_row0 + N_new) (app_row0 + N_new <= N_max);
 *   2. CSA (qi != NULL): csa_index_topk (index_dtype CSA_DTYPE_BF16) or
 *      csa_index_topk_fp8 (CSA_DTYPE_E4M3, with sq / sk) into idx_out [Q, k],
 *      then csa_sparse_mqa over idx_out;
 *      HCA (qi == NULL): hca_mqa over the entries j < n_cmp[q].
 * Every argument keeps the meaning, layout and limits it has in those calls.
 *
 * variant = CSA_STEP_CHAINED (0): the kernels of those calls, launched as
 * one chain of programmatic dependent launches on `stream` with no host
 * synchronisation. CSA runs the scorer first and the append after it, the
 * append starting at once (the scorer reads none of what it reads or
 * writes: qi, wi, ki and n_cmp must not overlap kv_cmp, app_kv, app_gate)
 * on the SMs the scorer leaves; the top-k follows both; the attention loads
 * the queries and computes the window tiles before the top-k is done (q,
 * kv_win, win_end and sink must not be written by the caller's kernel
 * launched just before this call with programmatic dependent launch). The
 * selection is that of the separate calls; the attention outputs agree with
 * them to rounding (the window tiles are summed first).
 * variant = CSA_STEP_PERSISTENT (1), for bf16 attention with H = 64 or 128,
 * D = 512, one query per sequence (q_per_seq = 1) and the indexer shape
 * 64 x 128: ONE persistent kernel in which each SM pulls tasks (append,
 * key-tile chunks, top-k, attention splits, split merges) from device-side
 * queues as their inputs complete. Its split plans differ from the separate
 * calls', so its outputs agree with them to rounding, not bit for bit; other
 * shapes take the chained kernels.
 *
 * Workspace: csa_decode_step_workspace_bytes(args) bytes, 256-byte aligned,
 * zero-filled before the first call (cudaMemset once); the step leaves its
 * counters at zero for the next call. Bytes 0..3 hold the status word (as for
 * every call); bytes 8..15 may hold a limit in nanoseconds for the bounded
 * waits (0 = 2 s; for tests of the timeout path).
 * Calls sharing one workspace must not overlap on the GPU.
 * Returns CSA_ERR_INVALID / CSA_ERR_WORKSPACE before any launch.
 * ---------------------------------------------------------------------- */
typedef struct csa_decode_step_args {
  /* attention: as csa_sparse_mqa / hca_mqa */
  const void *q;           /* [Q, H, D] */
  const void *kv_cmp;      /* [B, N_max, D] (the append writes into it) */
  const void *kv_win;      /* [B, T_raw, D] */
  const int32_t *win_end;  /* [Q] */
  const float *sink;       /* [H] */
  void *out;               /* [Q, H, D] */
  const int32_t *n_cmp;    /* [Q] visible entries per query */
  /* indexer (CSA): qi == NULL selects HCA */
  const void *qi;          /* [Q, Hi, Di] (uint8 codes for E4M3) */
  const float *sq;         /* [Q, Hi] (E4M3 only) */
  const float *wi;         /* [Q, Hi] */
  const void *ki;          /* [B, N_max, Di] (uint8 codes for E4M3) */
  const float *sk;         /* [B, N_max] (E4M3 only) */
  int32_t *idx_out;        /* [Q, k] the selection */
  /* append (app_kv == NULL: none) */
  const void *app_kv;
  const void *app_gate;
  const float *ape;
  const float *norm_w;
  const int64_t *pos0;     /* RoPE positions (csa_compress_rope), may be NULL */
  float scale;
  int Q, B, H, D, N_max, win_len, T_raw, q_per_seq, dtype;
  int index_dtype, Hi, Di, k;
  int app_win, app_stride, app_T, rope_dims;
  long long app_kv_seq_stride, app_gate_seq_stride, app_row0;
  double rope_theta;
  int variant;             /* CSA_STEP_CHAINED or CSA_STEP_PERSISTENT */
} csa_decode_step_args;

enum { CSA_STEP_CHAINED = 0, CSA_STEP_PERSISTENT = 1 };

size_t csa_decode_step_workspace_bytes(const csa_decode_step_args *args);
int csa_decode_step(const csa_decode_step_args *args, void *ws, size_t ws_bytes, csa_stream_t stream);

/* Number of kernels this library has launched in this process so far
 * (a monotonically increasing counter, for profiling and tests). */
unsigned long long csa_launch_count(void);

/* The CUDA error code (cudaError_t) behind the last CSA_ERR_CUDA this host
 * thread received from the library (0 if none), and its text. */
int csa_last_cuda_error(void);
const char *csa_cuda_error_string(int code);

/* Synchronises `stream`, copies the workspace status word into *status and
 * clears it. Returns CSA_OK if it was zero, CSA_ERR_DEVICE if not,
 * CSA_ERR_CUDA if the copy failed. Test/debug use. */
int csa_workspace_status(void *ws, csa_stream_t stream, uint32_t *status);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H_ */
