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
// per part, so a warp reads 2 (d = 128) or 4 (d = 64) whole rows per load.  One
// pass per row: the lse and 16-byte slice of a batch of parts (of R rows) are
// loaded together (one memory round trip per batch, not one per part), then folded into
// a running (max, sum, accumulator) with an online rescale -- the same
// recurrence as the forward's softmax, applied to whole parts.  Parts with
// lse = -inf (no visible key) are read but contribute nothing: their weight is
// selected to zero, never multiplied, so whatever their O holds cannot leak in.
#include "common.cuh"
#include "kernels.h"

namespace fa {

namespace mrg {

constexpr int THREADS = 128;

// R rows per thread per pass, each with its parts loaded in batches of BATCH: the
// R x BATCH loads of a batch step are independent and in flight together.  The
// host picks (R, BATCH) from S so that about eight 16-byte loads per thread are
// outstanding whatever the part count.
template <class T, int D, int R, int BATCH>
__global__ void __launch_bounds__(THREADS) merge_kernel(MergeArgs a) {
  constexpr int TPR = D / 8;          // threads per row, 8 elements (16 bytes) each
  constexpr int RPB = THREADS / TPR;  // rows per block per row slot
  const int sub = static_cast<int>(threadIdx.x) % TPR;
  const size_t part_vecs = static_cast<size_t>(a.rows) * (D / 8);  // uint4 per part
  const uint4* parts = static_cast<const uint4*>(a.o_parts);
  uint4* out = static_cast<uint4*>(a.o);
  const long long pass = static_cast<long long>(gridDim.x) * RPB * R;
  for (long long base = static_cast<long long>(blockIdx.x) * RPB * R + threadIdx.x / TPR; base < a.rows;
       base += pass) {
    float M[R], W[R], acc[R][8];
    bool nan[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      M[r] = -INFINITY;
      W[r] = 0.f;
      nan[r] = false;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
    }
    for (int s0 = 0; s0 < a.S; s0 += BATCH) {
      float l[R][BATCH];
      uint4 o[R][BATCH];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long row = base + static_cast<long long>(r) * RPB;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const bool in = s0 + i < a.S && row < a.rows;
          const size_t s = static_cast<size_t>(s0 + i);
          l[r][i] = in ? __ldg(a.lse_parts + s * a.rows + row) : -INFINITY;
          o[r][i] = in ? __ldg(parts + s * part_vecs + static_cast<size_t>(row) * (D / 8) + sub)
                       : make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float mb = -INFINITY;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          nan[r] |= (l[r][i] != l[r][i]);
          mb = fmaxf(mb, l[r][i]);  // ignores NaN
        }
        const float m_new = fmaxf(M[r], mb);
        if (m_new == -INFINITY) continue;  // nothing visible so far
        // Rescale what was accumulated against the previous maximum.
        const float f = M[r] == -INFINITY ? 0.f : __expf(M[r] - m_new);
        W[r] *= f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][e] *= f;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const bool live = l[r][i] != -INFINITY && l[r][i] == l[r][i];
          const float w = live ? __expf(l[r][i] - m_new) : 0.f;
          W[r] += w;
          float x[8];
          unpack8<T>(o[r][i], x);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[r][e] = live ? fmaf(w, x[e], acc[r][e]) : acc[r][e];
        }
        M[r] = m_new;
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const long long row = base + static_cast<long long>(r) * RPB;
      if (row >= a.rows) break;
      const size_t v = static_cast<size_t>(row) * (D / 8) + sub;
      if (nan[r] || M[r] == -INFINITY) {
        // NaN in: NaN out.  No part saw a key: O = 0, lse = -inf.
        const uint32_t w = nan[r] ? pack2<T>(__uint_as_float(0x7fc00000u), __uint_as_float(0x7fc00000u)) : 0u;
        out[v] = make_uint4(w, w, w, w);
        if (sub == 0 && a.lse) a.lse[row] = nan[r] ? __uint_as_float(0x7fc00000u) : -INFINITY;
        continue;
      }
      const float inv = 1.f / W[r];
      out[v] = make_uint4(pack2<T>(acc[r][0] * inv, acc[r][1] * inv), pack2<T>(acc[r][2] * inv, acc[r][3] * inv),
                          pack2<T>(acc[r][4] * inv, acc[r][5] * inv), pack2<T>(acc[r][6] * inv, acc[r][7] * inv));
      if (sub == 0 && a.lse) a.lse[row] = M[r] + logf(W[r]);
    }
  }
}

template <class T, int D, int R, int BATCH>
cudaError_t launch_t(const MergeArgs& a, cudaStream_t stream, int sms) {
  constexpr int RPB = THREADS / (D / 8);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, merge_kernel<T, D, R, BATCH>, THREADS, 0);
  if (e != cudaSuccess) return e;
  const long long need = (a.rows + RPB * R - 1) / (RPB * R);
  const long long cap = static_cast<long long>(sms) * (per_sm > 0 ? per_sm : 1);
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  merge_kernel<T, D, R, BATCH><<<grid, THREADS, 0, stream>>>(a);
  return cudaGetLastError();
}

// Measured on B200 (d = 128, bf16, rows past L2; GB/s for S = 2 / 4 / 8 parts):
// 128-thread blocks with (R, BATCH) = (2, 2) for S <= 2 and (1, 4) above reached
// 5548 / 5310 / 4974, ahead of 256-thread blocks with (4, 2), (2, 4), (1, 8)
// (4907 / 4889 / 4625): fewer registers per thread, more resident warps.
template <class T, int D>
cudaError_t launch_d(const MergeArgs& a, cudaStream_t stream, int sms) {
  if (a.S <= 2) return launch_t<T, D, 2, 2>(a, stream, sms);
  return launch_t<T, D, 1, 4>(a, stream, sms);
}

}  // namespace mrg

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream) {
  using namespace mrg;
  int sms = 0;
  cudaError_t e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  if (a.d == 128) return a.f16 ? launch_d<F16, 128>(a, stream, sms) : launch_d<Bf16, 128>(a, stream, sms);
  if (a.d == 64) return a.f16 ? launch_d<F16, 64>(a, stream, sms) : launch_d<Bf16, 64>(a, stream, sms);
  return cudaErrorInvalidValue;
}

}  // namespace fa
