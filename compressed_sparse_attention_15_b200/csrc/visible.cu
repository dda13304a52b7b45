// Causal visibility of compressed entries, and the entry count of a
// compressor run.
//
// "DeepSeek-V4 Architecture Analysis", INNOVATIONS section 1: the compressor
// folds each window of raw tokens into one entry (CSA: windows of 8 tokens
// every 4, overlapping; HCA: 128 tokens every 128). A query at position p may
// only read entries whose window has ended by then: entry j covers tokens
// j * stride .. j * stride + win - 1, so it is visible iff
// j * stride + win - 1 <= p, and the number of visible entries is the number
// of complete windows in the first p + 1 tokens,
//     n(p) = 0                              if p + 1 < win
//          = (p + 1 - win) / stride + 1     otherwise.
// A run over T tokens makes n(T - 1) entries.
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace {

__host__ __device__ inline long long entries_in_prefix(long long tokens, int win, int stride) {
  return tokens < win ? 0 : (tokens - win) / stride + 1;
}

__host__ __device__ inline int32_t visible_count(int64_t p, int win, int stride) {
  const long long n = p < 0 ? 0 : entries_in_prefix((long long)p + 1, win, stride);
  return n > INT32_MAX ? INT32_MAX : (int32_t)n;
}

__global__ void visible_counts_kernel(const int64_t *pos, long long Q, int win, int stride, int32_t *n_cmp) {
  csa::pdl_wait();  // positions may come from the previous kernel in the stream
  csa::pdl_release();
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < Q; q += (long long)gridDim.x * blockDim.x)
    n_cmp[q] = visible_count(pos[q], win, stride);
}

bool args_ok(const int64_t *pos, long long Q, int win, int stride, const int32_t *n_cmp) {
  if (Q < 0 || win < 1 || stride < 1) return false;
  if (Q > 0 && (!pos || !n_cmp)) return false;
  return ((reinterpret_cast<uintptr_t>(pos) & 7) | (reinterpret_cast<uintptr_t>(n_cmp) & 3)) == 0;
}

}  // namespace

extern "C" {

long long csa_num_entries(long long T, int win, int stride) {
  if (win < 1 || stride < 1 || T < 0) return -1;
  return entries_in_prefix(T, win, stride);
}

int csa_visible_counts_host(const int64_t *pos, long long Q, int win, int stride, int32_t *n_cmp) {
  if (!args_ok(pos, Q, win, stride, n_cmp)) return CSA_ERR_INVALID;
  for (long long q = 0; q < Q; ++q) n_cmp[q] = visible_count(pos[q], win, stride);
  return CSA_OK;
}

int csa_visible_counts(const int64_t *pos, long long Q, int win, int stride, int32_t *n_cmp, csa_stream_t stream) {
  if (!args_ok(pos, Q, win, stride, n_cmp)) return CSA_ERR_INVALID;
  if (Q == 0) return CSA_OK;
  const long long blocks = (Q + 255) / 256;
  const unsigned grid = (unsigned)(blocks < 1024 ? blocks : 1024);
  const cudaError_t e = csa::launch_pdl(visible_counts_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream, pos,
                                        Q, win, stride, n_cmp);
  return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // extern "C"
