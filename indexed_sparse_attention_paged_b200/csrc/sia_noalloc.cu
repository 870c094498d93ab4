// sia_noalloc.cu -- stage 1 (index scores + Top-K) for callers that cannot allocate device
// memory while they run.
//
// Some callers cannot call cudaMalloc after start-up: a serving loop whose device memory is a
// fixed, preallocated arena (every request must fit in it), a host runtime written in C with no
// device allocator of its own, or a latency-critical loop where a cudaMalloc/cudaFree would
// stall it (both can synchronize the device).  sia_sparse_index_topk needs a caller-provided
// workspace for the per-position scores; this entry point instead keeps them in a file-scope
// device array of fixed size, so it allocates nothing.
//
// The array is part of the library image: every GPU that loads libsia holds it (16 MiB) until
// the process exits.  All calls share it, so calls whose kernels overlap on the GPU (different
// streams, or different host threads) race on it and must be serialised by the caller.  The
// scores are fully rewritten before they are read by every call, so nothing needs clearing.
#include <cuda_runtime.h>

#include "sia.h"

namespace {

constexpr size_t kScratchFloats = size_t(4) << 20;  // 16 MiB of fp32 scores

__device__ __align__(256) float g_score_scratch[kScratchFloats];

// Device address of g_score_scratch for each device, looked up once per device.
void* g_scratch_addr[64] = {nullptr};

}  // namespace

extern "C" sia_status sia_sparse_index_topk_noalloc(const sia_index_args* a, int32_t* dev_status,
                                                    void* stream) {
  if (!a) return SIA_ERR_INVALID_ARGUMENT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SIA_ERR_CUDA;
  if (!g_scratch_addr[dev]) {
    // first call on this device: the host-side symbol is only a stand-in, look up the real
    // device address of the array (with this device current)
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_score_scratch) != cudaSuccess || !ptr) return SIA_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  // the regular entry point checks the size: more than 16 MiB of scores (batch * n_q *
  // max_pages_per_seq * page_size * 4 bytes) fails there with SIA_ERR_WORKSPACE and a message
  // from sia_last_error(), before anything is launched
  return sia_sparse_index_topk(a, g_scratch_addr[dev], kScratchFloats * sizeof(float), dev_status, stream);
}
