// Merge of partial attention results over disjoint key sets.
//
// Building Flash Attention from Scratch in Pure NumPy, architecture overview:
// the softmax over a union of key sets is a re-weighting of the partial
// softmaxes (the printed identity is garbled; restated):
//     lse = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
// Used by the context-parallel forward, where each part is one key shard's
// result (the "Extending It" roadmaps of the two pure-Python kernel pages:
// split the attention across devices, each holding part of the key/value space).
//
// HBM-bound: per row, S parts x d 16-bit values and S lse values are read once and
// d values plus one lse written.  d / 8 threads share a row, each moving 16 bytes
// per part, so a warp reads 2 (d = 128) or 4 (d = 64) whole rows per load; the
// grid is a multiple of the SM count and strides over the rows.
#include "common.cuh"
#include "kernels.h"

namespace fa {

namespace mrg {

constexpr int THREADS = 256;
constexpr int kBlocksPerSm = 8;

template <class T, int D>
__global__ void __launch_bounds__(THREADS) merge_kernel(MergeArgs a) {
  constexpr int TPR = D / 8;          // threads per row, 8 elements (16 bytes) each
  constexpr int RPB = THREADS / TPR;  // rows per block per pass
  const int sub = static_cast<int>(threadIdx.x) % TPR;
  const size_t part_vecs = static_cast<size_t>(a.rows) * (D / 8);  // uint4 per part
  const uint4* parts = static_cast<const uint4*>(a.o_parts);
  uint4* out = static_cast<uint4*>(a.o);
  for (long long row = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / TPR; row < a.rows;
       row += static_cast<long long>(gridDim.x) * RPB) {
    // Largest lse of the row; a NaN in any part marks the row.
    float M = -INFINITY;
    bool nan = false;
    for (int s = 0; s < a.S; ++s) {
      const float l = __ldg(a.lse_parts + static_cast<size_t>(s) * a.rows + row);
      nan |= (l != l);
      M = fmaxf(M, l);
    }
    const size_t v = static_cast<size_t>(row) * (D / 8) + sub;
    if (nan || M == -INFINITY) {
      // NaN in: NaN out.  No part saw a key: O = 0, lse = -inf.
      const uint32_t w = nan ? pack2<T>(__uint_as_float(0x7fc00000u), __uint_as_float(0x7fc00000u)) : 0u;
      out[v] = make_uint4(w, w, w, w);
      if (sub == 0 && a.lse) a.lse[row] = nan ? __uint_as_float(0x7fc00000u) : -INFINITY;
      continue;
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float W = 0.f;
#pragma unroll 4
    for (int s = 0; s < a.S; ++s) {
      const float w = __expf(__ldg(a.lse_parts + static_cast<size_t>(s) * a.rows + row) - M);
      if (w == 0.f) continue;  // an empty part (or one far below the rest) adds nothing
      W += w;
      float f[8];
      unpack8<T>(__ldg(parts + static_cast<size_t>(s) * part_vecs + v), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(w, f[i], acc[i]);
    }
    const float inv = 1.f / W;
    out[v] = make_uint4(pack2<T>(acc[0] * inv, acc[1] * inv), pack2<T>(acc[2] * inv, acc[3] * inv),
                        pack2<T>(acc[4] * inv, acc[5] * inv), pack2<T>(acc[6] * inv, acc[7] * inv));
    if (sub == 0 && a.lse) a.lse[row] = M + logf(W);
  }
}

template <class T, int D>
cudaError_t launch_t(const MergeArgs& a, cudaStream_t stream, int sms) {
  constexpr int RPB = THREADS / (D / 8);
  const long long need = (a.rows + RPB - 1) / RPB;
  const long long cap = static_cast<long long>(sms) * kBlocksPerSm;
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  merge_kernel<T, D><<<grid, THREADS, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace mrg

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream) {
  using namespace mrg;
  int sms = 0;
  cudaError_t e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  if (a.d == 128) return a.f16 ? launch_t<F16, 128>(a, stream, sms) : launch_t<Bf16, 128>(a, stream, sms);
  if (a.d == 64) return a.f16 ? launch_t<F16, 64>(a, stream, sms) : launch_t<Bf16, 64>(a, stream, sms);
  return cudaErrorInvalidValue;
}

}  // namespace fa
