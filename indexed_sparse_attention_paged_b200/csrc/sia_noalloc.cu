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
// The array belongs to this file's module.  CUDA loads modules lazily, so the 16 MiB are
// reserved on a device by the first call of this entry point there, and stay reserved until
// the process exits (or the device's context is reset).  All calls share the array, so calls
// whose kernels overlap on the GPU (different streams, or different host threads) race on it
// and must be serialised by the caller.  The scores are fully rewritten before they are read by
// every call, so nothing needs clearing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "sia.h"
#include "sia_internal.h"

namespace {

constexpr size_t kScratchFloats = size_t(4) << 20;  // 16 MiB of fp32 scores

__device__ __align__(256) float g_score_scratch[kScratchFloats];

// The array's device address, looked up once per device context.  In host code the name
// g_score_scratch is only a host-side stand-in, so the address a kernel is given must come
// from cudaGetSymbolAddress with that device current.  The context id keys the entry, so that
// a context created after a reset (which reloads the module elsewhere) gets a fresh lookup.
struct ScratchSlot {
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_mu;
ScratchSlot g_slots[64];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the calling thread's current context, or 0 when there is none or the driver cannot say.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

sia_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return sia::set_last_error(SIA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return sia::set_last_error(SIA_ERR_UNSUPPORTED, "device %d: at most 64 devices", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchSlot& slot = g_slots[dev];
  const unsigned long long id = current_context_id();
  if (slot.ptr && id != 0 && slot.ctx_id == id) {
    *out = slot.ptr;
    return SIA_OK;
  }
  // first call on this device (or in a new context): loads the module, which reserves the
  // array on the device, and resolves its device address with the device current
  void* ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_score_scratch);
  if (e != cudaSuccess || !ptr)
    return sia::set_last_error(SIA_ERR_CUDA, "cudaGetSymbolAddress of the score scratch: %s",
                               cudaGetErrorString(e));
  slot.ctx_id = current_context_id();   // the lookup made a context current if there was none
  slot.ptr = slot.ctx_id ? ptr : nullptr;   // no id: look the address up again on every call
  *out = ptr;
  return SIA_OK;
}

}  // namespace

extern "C" sia_status sia_sparse_index_topk_noalloc(const sia_index_args* a, int32_t* dev_status,
                                                    void* stream) {
  sia::set_last_error(SIA_OK, "%s", "");
  if (!a) return sia::set_last_error(SIA_ERR_INVALID_ARGUMENT, "index args are NULL");
  void* scratch = nullptr;
  const sia_status st = scratch_address(&scratch);
  if (st != SIA_OK) return st;
  // the regular entry point checks the size: more than 16 MiB of scores (batch * n_q *
  // max_pages_per_seq * page_size * 4 bytes) fails there with SIA_ERR_WORKSPACE and a message
  // from sia_last_error(), before anything is launched
  return sia_sparse_index_topk(a, scratch, kScratchFloats * sizeof(float), dev_status, stream);
}
