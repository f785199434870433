// fp2_discover_static: block discovery that allocates nothing, for callers that cannot call
// cudaMalloc (or any allocator) at the point where they run discovery -- for example a serving
// runtime that reserves all device memory for its KV cache at start-up and forbids allocation on
// the request path, or a plain C host that has no device allocator of its own to hand us scratch.
//
// The scratch that fp2_discover takes from the caller (status word, per-row kept bitmask, per-row
// counts) lives here in one file-scope __device__ array of FP2_STATIC_SCRATCH_BYTES.  Every GPU
// that loads this library holds that array until the process exits.  The host cannot use the
// array's name as a device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it; make that first call before
// any stream capture.  Every call reuses the same array and leaves its contents behind; the status
// word is cleared at the start of each call and the bitmask/count words a call reads are the ones
// it wrote, so nothing else needs clearing.  Two calls whose work overlaps on the GPU (different
// streams, or different host threads on one device) race on the array: serialise them.
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
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};
}  // namespace

extern "C" FP2_API fp2_status fp2_discover_static(const fp2_problem* problem, const fp2_sparse_params* params,
                                                  const fp2_pooled* pooled, const fp2_index* index,
                                                  uint32_t* status_dev, fp2_stream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fp2_internal::set_error(FP2_ERR_CUDA, "no current CUDA device");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_addr[dev] == nullptr) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_fp2_static_scratch);
      if (e != cudaSuccess || p == nullptr)
        return fp2_internal::set_error(FP2_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  return fp2_internal::discover_fixed_scratch(problem, params, pooled, index, scratch, FP2_STATIC_SCRATCH_BYTES,
                                              status_dev, static_cast<cudaStream_t>(stream));
}
