// Float32 forward on CUDA cores (head dimension 64 or 128, any mask).
//
// The same online-softmax algorithm as the tensor-core path ("Building Flash
// Attention from Scratch in Pure NumPy", architecture overview and Step 2),
// in float32 throughout: 32-key tiles of K and V staged in shared memory,
// one warp per query row, lane l scoring key l of the tile, the running
// (m, l, O) state kept in registers, O spread over the lanes (d/32 columns
// each).  Masks: "Build a FlashAttention-2 Inference Kernel from Scratch in
// Pure Python", Step 3.
#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace fwdf32 {

constexpr int ROWS = 16;      // query rows per CTA
constexpr int WARPS = 4;      // 4 rows per warp
constexpr int KT = 32;        // keys per tile (one per lane)

template <int D>
__global__ void __launch_bounds__(WARPS * 32)
    fwd_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                   const float* __restrict__ v, float* __restrict__ o, float* __restrict__ lse, int n,
                   int causal, int window, float scale, float sl2) {
  constexpr int E = D / 32;  // output columns per lane
  constexpr int RPW = ROWS / WARPS;
  __shared__ float qs[ROWS][D];
  __shared__ float ks[KT][D + 1];
  __shared__ float vs[KT][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * ROWS;
  const size_t head = static_cast<size_t>(bh) * n * D;

  for (int idx = threadIdx.x; idx < ROWS * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D;
    qs[r][c] = (r0 + r < n) ? q[head + static_cast<size_t>(r0 + r) * D + c] : 0.f;
  }

  float m[RPW], l[RPW], acc[RPW][E];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[r][e] = 0.f;
  }

  const int rlast = min(r0 + ROWS - 1, n - 1);
  const int key_hi = causal ? rlast + 1 : n;
  const int key_lo = window > 0 ? max(0, r0 - window + 1) : 0;
  for (int t0 = (key_lo / KT) * KT; t0 < key_hi; t0 += KT) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * D; idx += blockDim.x) {
      const int r = idx / D, c = idx % D;
      const bool in = t0 + r < n;
      ks[r][c] = in ? k[head + static_cast<size_t>(t0 + r) * D + c] : 0.f;
      vs[r][c] = in ? v[head + static_cast<size_t>(t0 + r) * D + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int rr = warp * RPW + r;
      const int i = r0 + rr;
      const int j = t0 + lane;
      float s = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) s = fmaf(qs[rr][c], ks[lane][c], s);
      s = key_visible(i, j, n, causal, window) ? s : -INFINITY;
      const float mx = warp_max(s);
      const float m_new = fmaxf(m[r], mx);
      const float ms = (m_new == -INFINITY) ? 0.f : m_new * sl2;
      const float alpha = (m[r] == -INFINITY) ? 0.f : exp2f(m[r] * sl2 - ms);
      const float p = exp2f(s * sl2 - ms);
      l[r] = l[r] * alpha + warp_sum(p);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[r][e] *= alpha;
#pragma unroll 4
      for (int kk = 0; kk < KT; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, p, kk);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[r][e] = fmaf(pk, vs[kk][lane + 32 * e], acc[r][e]);
      }
      m[r] = m_new;
    }
  }

#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int i = r0 + warp * RPW + r;
    if (i >= n) continue;
    const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[head + static_cast<size_t>(i) * D + lane + 32 * e] = acc[r][e] * inv;
    if (lane == 0 && lse != nullptr)
      lse[static_cast<size_t>(bh) * n + i] = l[r] > 0.f ? m[r] * scale + logf(l[r]) : -INFINITY;
  }
}

}  // namespace fwdf32

cudaError_t launch_fwd_f32(const FwdArgs& a, cudaStream_t stream) {
  using namespace fwdf32;
  const long long bh = static_cast<long long>(a.B) * a.H;
  if (bh > 65535) return cudaErrorInvalidValue;
  dim3 grid((a.N + ROWS - 1) / ROWS, static_cast<unsigned>(bh));
  const float* q = static_cast<const float*>(a.q);
  const float* k = static_cast<const float*>(a.k);
  const float* v = static_cast<const float*>(a.v);
  float* o = static_cast<float*>(a.o);
  if (a.d == 64)
    fwd_f32_kernel<64><<<grid, WARPS * 32, 0, stream>>>(q, k, v, o, a.lse, a.N, a.causal, a.window,
                                                        a.scale, a.scale_log2);
  else
    fwd_f32_kernel<128><<<grid, WARPS * 32, 0, stream>>>(q, k, v, o, a.lse, a.N, a.causal, a.window,
                                                         a.scale, a.scale_log2);
  return cudaGetLastError();
}

}  // namespace fa
