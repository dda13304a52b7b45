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

// Device address of g_noalloc_scratch, per device: looked up once per device
// (the lookup runs under the lock of once_per_device, so concurrent first
// calls from several host threads see one lookup) and read lock-free after.
std::atomic<void *> g_scratch_ptr[csa::kMaxDevices];

int scratch_on_current_device(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= csa::kMaxDevices) return CSA_ERR_CUDA;
  void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    static csa::DeviceOnce once;
    csa::once_per_device(once, [dev] {
      void *a = nullptr;
      if (cudaGetSymbolAddress(&a, g_noalloc_scratch) == cudaSuccess && a)
        g_scratch_ptr[dev].store(a, std::memory_order_release);
      else
        cudaGetLastError();
    });
    p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) return CSA_ERR_CUDA;
  }
  *out = p;
  return CSA_OK;
}

}  // namespace

extern "C" int csa_index_topk_noalloc(const void *qi, const float *wi, const void *ki, const int32_t *n_cmp, int k,
                                      int32_t *out_idx, int Q, int B, int Hi, int Di, int N_max, int q_per_seq,
                                      int dtype, csa_stream_t stream) {
  if (Q < 1 || N_max < 1 || k < 1) return CSA_ERR_INVALID;
  if (csa_index_topk_workspace_bytes(Q, N_max, k) > kScratchBytes) return CSA_ERR_SCRATCH_LIMIT;
  // csa_index_topk's own argument checks, before anything is written to the
  // shared buffer: a rejected call leaves it untouched.
  const int chk = csa::check_index_topk(qi, wi, ki, n_cmp, k, out_idx, Q, B, Hi, Di, N_max, q_per_seq, dtype);
  if (chk != CSA_OK) return chk;
  void *scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != CSA_OK) return rc;
  // The status word must start at zero; the array keeps the last call's bytes.
  if (cudaMemsetAsync(scratch, 0, 256, (cudaStream_t)stream) != cudaSuccess) return CSA_ERR_CUDA;
  return csa_index_topk(qi, wi, ki, n_cmp, k, out_idx, Q, B, Hi, Di, N_max, q_per_seq, dtype, scratch,
                        kScratchBytes, stream);
}
