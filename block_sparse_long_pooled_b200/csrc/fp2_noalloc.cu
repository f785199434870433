// fp2_discover_static: block discovery that allocates nothing, for callers that cannot call
// cudaMalloc (or any allocator) at the point where they run discovery -- for example a serving
// runtime that reserves all device memory for its KV cache at start-up and forbids allocation on
// the request path, or a plain C host that has no device allocator of its own to hand us scratch.
//
// The scratch that fp2_discover takes from the caller (status word, per-row kept bitmask, per-row
// counts) lives here in one file-scope __device__ array of FP2_STATIC_SCRATCH_BYTES.  Every GPU
// that loads this library holds that array until the process exits.  The host cannot use the
// array's name as a device address, so the first call in each CUDA context looks the address up
// with cudaGetSymbolAddress (with that context's device current) and caches it per device together
// with the context's id; a call from a new context on the same device (after cudaDeviceReset, say)
// looks it up again instead of reusing a stale address.  Under CUDA's lazy module loading that
// first lookup is also when the driver loads this file's module and places the array, so the
// 8 MiB are taken from the device then: make the first call at start-up, before the caller
// reserves the rest of device memory and before any stream capture.  Every call reuses the same
// array and leaves its contents behind; the status word is cleared at the start of each call and
// the bitmask/count words a call reads are the ones it wrote, so nothing else needs clearing.  Two
// calls whose work overlaps on the GPU (different streams, or different host threads on one
// device) race on the array: serialise them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/fp2.h"

namespace fp2_internal {
fp2_status set_error(fp2_status s, const char* msg);
fp2_status discover_fixed_scratch(const fp2_problem* problem, const fp2_sparse_params* params,
                                  const fp2_pooled* pooled, const fp2_index* index, void* scratch,
                                  size_t capacity, uint32_t* status_dev, cudaStream_t st);
}  // namespace fp2_internal

static __device__ __align__(256) unsigned char g_fp2_static_scratch[FP2_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
struct Cached {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_mutex;
Cached g_cache[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the calling thread's current context (unique for the life of the process), or 0 when the
// driver cannot say.  The driver functions are looked up once through the runtime.
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
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}
}  // namespace

extern "C" FP2_API fp2_status fp2_discover_static(const fp2_problem* problem, const fp2_sparse_params* params,
                                                  const fp2_pooled* pooled, const fp2_index* index,
                                                  uint32_t* status_dev, fp2_stream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
    return fp2_internal::set_error(FP2_ERR_CUDA, "no current CUDA device");
  if (dev >= kMaxDevices)
    return fp2_internal::set_error(FP2_ERR_UNSUPPORTED,
                                   "device index exceeds the static-scratch address cache (64 devices)");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    // Before the first runtime call in this thread the context may not exist yet (id 0); the
    // lookup below creates it, and its id is taken afterwards.
    const unsigned long long id = current_context_id();
    Cached& c = g_cache[dev];
    if (c.addr == nullptr || id == 0 || c.ctx_id != id) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_fp2_static_scratch);
      if (e != cudaSuccess || p == nullptr)
        return fp2_internal::set_error(FP2_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
      c.addr = p;
      c.ctx_id = current_context_id();
    }
    scratch = c.addr;
  }
  return fp2_internal::discover_fixed_scratch(problem, params, pooled, index, scratch, FP2_STATIC_SCRATCH_BYTES,
                                              status_dev, static_cast<cudaStream_t>(stream));
}
