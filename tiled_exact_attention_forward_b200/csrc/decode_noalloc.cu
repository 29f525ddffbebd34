// fa_decode_noalloc: the split-KV decode for callers that cannot allocate
// device memory.
//
// fa_decode needs a workspace for the per-chunk partial results and leaves
// allocating it to the caller.  Some callers have no allocator to use: serving
// runtimes that plan every byte of device memory at start-up and forbid
// allocation on the request path, plugin interfaces that hand a kernel only
// its inputs and outputs, and code that must not risk the device-wide
// synchronisation a cudaMalloc/cudaFree pair can cause.  This entry point
// keeps the partials in a fixed array compiled into the library instead, so a
// call allocates nothing.
//
// The array lives in device global memory.  With lazy module loading (the
// CUDA 12 default) it is reserved on a device by the first call made there
// (or at library load when CUDA_MODULE_LOADING=EAGER) and held until the
// process exits.  Its host-side name is only a shadow of the device array, so
// every call asks the runtime for the device address in the CURRENT context
// with cudaGetSymbolAddress.  The address belongs to a context, not to a
// device: after cudaDeviceReset, or with another context made current on the
// same device, the module is loaded again at a new address, which is why no
// address is kept between calls.  Once the module is loaded the lookup is a
// table search that does not synchronise.  The first call on each device
// loads the module: make it at start-up, before any stream capture.
// All calls share the array: two calls whose kernels overlap on the GPU race
// on it.  Nothing in it needs clearing between calls, because every partial
// the combine step reads is written earlier in the same call.
#include "../../include/fa.h"
#include "common.cuh"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[FA_DECODE_NOALLOC_SCRATCH_BYTES];

}  // namespace

extern "C" fa_status fa_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                       const int32_t* seqlens, void* o, float* lse, int B, int H,
                                       int cap, int d, float scale, fa_dtype dtype, void* stream) {
  const size_t need = fa_decode_workspace_size(B, H, cap, d);
  if (need == 0 || need > static_cast<size_t>(FA_DECODE_NOALLOC_SCRATCH_BYTES)) return FA_ERR_INVALID;
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_decode_noalloc_scratch) != cudaSuccess || scratch == nullptr)
    return FA_ERR_CUDA;
  return fa_decode(q, kcache, vcache, seqlens, o, lse, B, H, cap, d, scale, dtype, scratch, need, stream);
}
