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
// The array lives in device global memory on every GPU that loads the
// library, for the life of the process.  Its host-side name is only a shadow
// of the device array, so the device address is looked up with
// cudaGetSymbolAddress -- once per device, on the first call made while that
// device is current.  That first call should come before any stream capture.
// All calls share the array: two calls whose kernels overlap on the GPU race
// on it.  Nothing in it needs clearing between calls, because every partial
// the combine step reads is written earlier in the same call.
#include <mutex>

#include "../../include/fa.h"
#include "common.cuh"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[FA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" fa_status fa_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                       const int32_t* seqlens, void* o, float* lse, int B, int H,
                                       int cap, int d, float scale, fa_dtype dtype, void* stream) {
  const size_t need = fa_decode_workspace_size(B, H, cap, d);
  if (need == 0 || need > static_cast<size_t>(FA_DECODE_NOALLOC_SCRATCH_BYTES)) return FA_ERR_INVALID;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return FA_ERR_CUDA;
  return fa_decode(q, kcache, vcache, seqlens, o, lse, B, H, cap, d, scale, dtype, scratch, need, stream);
}
