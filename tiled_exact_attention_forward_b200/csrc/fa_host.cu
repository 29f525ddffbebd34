// Host-side helpers shared by the launchers: TMA descriptor encoding through
// the driver entry point (no link against libcuda), per-device kernel
// attributes, and the device status word.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace fa {

cudaError_t take_status_host(unsigned int* out) { return take_local_status(out); }

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

}  // namespace

bool make_tmap_half_rows(void* map, const void* base, int d, long long rows_per_head, long long heads,
                         int box_rows, int f16) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows_per_head),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(rows_per_head)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(reinterpret_cast<CUtensorMap*>(map),
                  f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_f32_rows(void* map, const void* base, int d, long long rows_per_head, long long heads,
                        int box_cols, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows_per_head),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                           static_cast<cuuint64_t>(d) * 4 * static_cast<cuuint64_t>(rows_per_head)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(reinterpret_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                  const_cast<void*>(base), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t set_max_dynamic_smem(const void* func, size_t bytes) {
  // One bit per (device, kernel) pair; the kernel set is tiny and fixed.
  static std::mutex mu;
  struct Entry {
    const void* func;
    int device;
  };
  static Entry done[256];
  static int n_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].func == func && done[i].device == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  if (n_done < 256) done[n_done++] = Entry{func, dev};
  return cudaSuccess;
}

cudaError_t sm_count(int* out) {
  static std::mutex mu;
  static int cached[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int v = 0;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    cached[dev] = v;
  }
  *out = cached[dev];
  return cudaSuccess;
}

namespace {

// One CTA waits on an mbarrier that nothing ever arrives on.  The bounded wait
// must give up after `limit_cycles`, record the timeout in the status word and
// let the kernel return normally -- the same path every production kernel
// takes when a barrier stalls.
__global__ void selftest_wait_timeout_kernel(long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait_limit(smem_u32(&bar), 0, &abort_flag, limit_cycles);
  (void)ok;
}

// Evaluates the forward's exp2 cubic (exp2_poly_pair) on an array, two values
// per thread exactly as the softmax feeds it, so a test can hold the device
// function to its stated error bound.
__global__ void selftest_exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  const long long stride = 2LL * gridDim.x * blockDim.x;
  for (long long i = 2LL * (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x); i < n; i += stride) {
    const bool two = i + 1 < n;
    const uint64_t r = exp2_poly_pair(f2_pack(x[i], two ? x[i + 1] : 0.f));
    float r0, r1;
    f2_unpack(r, r0, r1);
    y[i] = r0;
    if (two) y[i + 1] = r1;
  }
}

}  // namespace

cudaError_t launch_selftest_exp2_poly(const float* x, float* y, long long n, cudaStream_t stream) {
  const long long pairs = (n + 1) / 2;
  const long long blocks = (pairs + 255) / 256;
  selftest_exp2_poly_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait_timeout(long long limit_cycles, cudaStream_t stream) {
  selftest_wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_cycles);
  return cudaGetLastError();
}

}  // namespace fa
