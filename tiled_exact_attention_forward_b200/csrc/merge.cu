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
// HBM-bound: per row, S parts x d values and S lse values are read once and d
// values plus one lse written.  The parts and the output are 16-bit, or float32
// for callers that keep their partials unrounded.  d / 8 threads share a row, each
// moving 8 elements per part (16 bytes of 16-bit values, 32 of float32), so a warp
// reads 2 (d = 128) or 4 (d = 64) whole rows per load.  One pass per row: the lse
// and slice of a batch of parts (of R rows) are
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

// Streaming 16-byte load: not kept in L1, with a 256-byte L2 fetch granularity (a
// warp reads 512 contiguous bytes of a part per load).  Measured against plain
// read-only loads (TB/s): 2 parts 5.5 either way, 4 parts 5.2 -> 5.4, 8 parts
// 4.8 -> 5.1-5.2.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Conversions between 16-byte words of the parts' type and float32: a word holds
// 8 elements of a 16-bit type or 4 of float32 (tag F32).
struct F32 {};
template <class T> struct Conv {
  static constexpr int E = 8;
  __device__ static __forceinline__ void to(const uint4& w, float* x) {
    float f[8];
    unpack8<T>(w, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = f[e];
  }
  __device__ static __forceinline__ uint4 from(const float* x) {
    return make_uint4(pack2<T>(x[0], x[1]), pack2<T>(x[2], x[3]), pack2<T>(x[4], x[5]), pack2<T>(x[6], x[7]));
  }
  __device__ static __forceinline__ uint4 nan() {
    const uint32_t w = pack2<T>(__uint_as_float(0x7fc00000u), __uint_as_float(0x7fc00000u));
    return make_uint4(w, w, w, w);
  }
};
template <> struct Conv<F32> {
  static constexpr int E = 4;
  __device__ static __forceinline__ void to(const uint4& w, float* x) {
    x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y); x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
  }
  __device__ static __forceinline__ uint4 from(const float* x) {
    return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
  }
  __device__ static __forceinline__ uint4 nan() { return make_uint4(0x7fc00000u, 0x7fc00000u, 0x7fc00000u, 0x7fc00000u); }
};

// R rows per thread per pass, each with its parts loaded in batches of BATCH: the
// R x BATCH loads of a batch step are independent and in flight together.  The
// host picks (R, BATCH) from S so that about eight 16-byte loads per thread are
// outstanding whatever the part count.
template <class T, int D, int R, int BATCH, int NV>
__global__ void __launch_bounds__(THREADS) merge_kernel(MergeArgs a) {
  using C = Conv<T>;
  constexpr int EPT = NV * C::E;        // elements per thread: NV 16-byte words
  constexpr int TPR = D / EPT;          // threads per row
  constexpr int RPB = THREADS / TPR;    // rows per block per row slot
  constexpr int WPR = D / C::E;         // 16-byte words per row
  static_assert(D % EPT == 0 && THREADS % TPR == 0, "row split");
  const int sub = static_cast<int>(threadIdx.x) % TPR;
  const size_t part_words = static_cast<size_t>(a.rows) * WPR;
  const uint4* parts = static_cast<const uint4*>(a.o_parts);
  uint4* out = static_cast<uint4*>(a.o);
  const long long pass = static_cast<long long>(gridDim.x) * RPB * R;
  for (long long base = static_cast<long long>(blockIdx.x) * RPB * R + threadIdx.x / TPR; base < a.rows;
       base += pass) {
    float M[R], W[R], acc[R][EPT];
    bool nan[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      M[r] = -INFINITY;
      W[r] = 0.f;
      nan[r] = false;
#pragma unroll
      for (int e = 0; e < EPT; ++e) acc[r][e] = 0.f;
    }
    for (int s0 = 0; s0 < a.S; s0 += BATCH) {
      float l[R][BATCH];
      uint4 o[R][BATCH][NV];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const long long row = base + static_cast<long long>(r) * RPB;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const bool in = s0 + i < a.S && row < a.rows;
          const size_t s = static_cast<size_t>(s0 + i);
          l[r][i] = in ? __ldg(a.lse_parts + s * a.rows + row) : -INFINITY;
          const uint4* src = parts + s * part_words + static_cast<size_t>(row) * WPR + sub * NV;
#pragma unroll
          for (int k = 0; k < NV; ++k) o[r][i][k] = in ? ld_stream(src + k) : make_uint4(0u, 0u, 0u, 0u);
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
        for (int e = 0; e < EPT; ++e) acc[r][e] *= f;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const bool live = l[r][i] != -INFINITY && l[r][i] == l[r][i];
          const float w = live ? __expf(l[r][i] - m_new) : 0.f;
          W[r] += w;
          float x[EPT];
#pragma unroll
          for (int k = 0; k < NV; ++k) C::to(o[r][i][k], x + k * C::E);
#pragma unroll
          for (int e = 0; e < EPT; ++e) acc[r][e] = live ? fmaf(w, x[e], acc[r][e]) : acc[r][e];
        }
        M[r] = m_new;
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const long long row = base + static_cast<long long>(r) * RPB;
      if (row >= a.rows) break;
      uint4* dst = out + static_cast<size_t>(row) * WPR + sub * NV;
      if (nan[r] || M[r] == -INFINITY) {
        // NaN in: NaN out.  No part saw a key: O = 0, lse = -inf.
#pragma unroll
        for (int k = 0; k < NV; ++k) dst[k] = nan[r] ? C::nan() : make_uint4(0u, 0u, 0u, 0u);
        if (sub == 0 && a.lse) a.lse[row] = nan[r] ? __uint_as_float(0x7fc00000u) : -INFINITY;
        continue;
      }
      const float inv = 1.f / W[r];
      float y[EPT];
#pragma unroll
      for (int e = 0; e < EPT; ++e) y[e] = acc[r][e] * inv;
#pragma unroll
      for (int k = 0; k < NV; ++k) dst[k] = C::from(y + k * C::E);
      if (sub == 0 && a.lse) a.lse[row] = M[r] + logf(W[r]);
    }
  }
}

template <class T, int D, int R, int BATCH, int NV>
cudaError_t launch_t(const MergeArgs& a, cudaStream_t stream, int sms) {
  constexpr int RPB = THREADS / (D / (NV * Conv<T>::E));
  int per_sm = 0;
  cudaError_t e =
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, merge_kernel<T, D, R, BATCH, NV>, THREADS, 0);
  if (e != cudaSuccess) return e;
  const long long need = (a.rows + RPB * R - 1) / (RPB * R);
  const long long cap = static_cast<long long>(sms) * (per_sm > 0 ? per_sm : 1);
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  merge_kernel<T, D, R, BATCH, NV><<<grid, THREADS, 0, stream>>>(a);
  return cudaGetLastError();
}

// Measured on B200 (d = 128, bf16, rows past L2; GB/s for S = 2 / 4 / 8 parts):
// 128-thread blocks with (R, BATCH) = (2, 2) for S <= 2 and (1, 4) above reached
// 5548 / 5310 / 4974, ahead of 256-thread blocks with (4, 2), (2, 4), (1, 8)
// (4907 / 4889 / 4625): fewer registers per thread, more resident warps.  Two
// 16-byte words per thread per part for 16-bit parts measured the same (within
// 2 %, either way); float32 parts take two words (8 elements) per thread.
template <class T, int D>
cudaError_t launch_d(const MergeArgs& a, cudaStream_t stream, int sms) {
  constexpr int NV = Conv<T>::E == 4 ? 2 : 1;  // 16-byte words per thread per part
  if (a.S <= 2) return launch_t<T, D, 2, 2, NV>(a, stream, sms);
  return launch_t<T, D, 1, 4, NV>(a, stream, sms);
}

}  // namespace mrg

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream) {
  using namespace mrg;
  int sms = 0;
  cudaError_t e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  if (a.f32) {
    if (a.d == 128) return launch_d<F32, 128>(a, stream, sms);
    if (a.d == 64) return launch_d<F32, 64>(a, stream, sms);
    return cudaErrorInvalidValue;
  }
  if (a.d == 128) return a.f16 ? launch_d<F16, 128>(a, stream, sms) : launch_d<Bf16, 128>(a, stream, sms);
  if (a.d == 64) return a.f16 ? launch_d<F16, 64>(a, stream, sms) : launch_d<Bf16, 64>(a, stream, sms);
  return cudaErrorInvalidValue;
}

}  // namespace fa
