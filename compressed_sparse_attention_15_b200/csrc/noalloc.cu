// csa_index_topk_noalloc: csa_index_topk for callers that cannot allocate
// device memory.
//
// Some callers have no way to hand the library a workspace: a plugin that
// only receives the input and output pointers from a host framework whose
// memory pools and accounting it must not bypass, or a real-time decode loop
// that may not block on cudaMalloc (which can synchronise the device) in the
// middle of a step. This entry point serves them with a scratch buffer that
// is part of the library image itself: a file-scope __device__ array of
// CSA_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds
// until the process exits. Nothing here calls cudaMalloc, cudaFree or any
// allocating routine.
//
// The array's host-side name is only a stand-in for the device symbol, so the
// device address is looked up once per device with cudaGetSymbolAddress (with
// that device current) the first time this entry point runs on it; make that
// first call before any stream capture. Every call shares the one array and
// its contents persist between calls: the status word is cleared at the start
// of each call, and calls whose work overlaps on the GPU (other streams, other
// host threads) race on the array.
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = CSA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// Looks up (once per device) the device address of the scratch array.
int scratch_on_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA_ERR_CUDA;
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return CSA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return CSA_OK;
}

}  // namespace

extern "C" int csa_index_topk_noalloc(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp, int k,
                                      int32_t *out_idx, int Q, int B, int Hi, int Di, int N_max, int q_per_seq,
                                      int dtype, csa_stream_t stream) {
  if (Q < 1 || N_max < 1 || k < 1) return CSA_ERR_INVALID;
  if (csa_index_topk_workspace_bytes(Q, N_max, k) > kScratchBytes) return CSA_ERR_SCRATCH_LIMIT;
  void *scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != CSA_OK) return rc;
  // The status word must start at zero; the array keeps the last call's bytes.
  if (cudaMemsetAsync(scratch, 0, 256, (cudaStream_t)stream) != cudaSuccess) return CSA_ERR_CUDA;
  return csa_index_topk(qi, wi, ki, n_cmp, k, out_idx, Q, B, Hi, Di, N_max, q_per_seq, dtype, scratch,
                        kScratchBytes, stream);
}
