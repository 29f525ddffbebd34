// Single-token decode against a padded or a paged key/value cache (bf16 or f16,
// d = 128).
//
// "Build a FlashAttention Kernel with Online Softmax and KV Cache in Pure
// Python", Step 4: the query of (b, h) attends to every cached position
// j < seqlens[b] (the cache already holds the current token).  The work is
// HBM-bound: every cached key and value row is read once, 256 bytes each.
//
// Split: CTA (chunk, h, b) scores keys [chunk * 512, chunk * 512 + 512) (paged:
// 2048-key chunks) of its sequence with the online softmax and writes a normalised partial
// (o_c, lse_c).  Each half-warp owns one key row per step (16 lanes x 16
// bytes = one 256-byte row, so a warp reads 512 contiguous bytes per load
// instruction) and keeps 8 rows of K and 8 of V in flight per thread.
// Paged cache ("Build a FlashAttention-2 Inference Kernel from Scratch in Pure
// Python", Extending It: paged KV-cache integration): the rows live in
// fixed-size blocks of a shared pool and a per-sequence block table maps the
// logical block j / block_size to its physical block; a half-warp still reads
// one whole 256-byte row per key, now at the table's address.
// Combine: lse = ln sum_c exp(lse_c), o = sum_c exp(lse_c - lse) o_c -- the
// two-softmax merge identity of "Building Flash Attention from Scratch in
// Pure NumPy" (architecture overview), restated.
#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace dec {

constexpr int D = 128;
constexpr int THREADS = 256;          // 8 warps = 16 half-warps
constexpr int HALVES = THREADS / 16;
constexpr int U = 8;                  // key rows in flight per half-warp and step
// Keys per split CTA: a paged CTA first loads its chunk's block-table entries, a
// dependent load before its first row, so it takes four times the keys to amortise
// it (measured on the paged workload: 1024-key chunks 5980 GB/s, 2048 6105, 4096 6014).
template <bool PAGED> __host__ __device__ constexpr int chunk_keys() { return PAGED ? 4 * kDecodeChunk : kDecodeChunk; }

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// T: the 16-bit type of q and the caches (Bf16 or F16).
template <bool PAGED, class T>
__global__ void __launch_bounds__(THREADS)
    decode_split_kernel(DecodeArgs a) {
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n = min(max(a.seqlens[b], 0), a.cap);
  constexpr int CHUNK = chunk_keys<PAGED>();
  const int start = c * CHUNK;
  if (start >= n) return;
  const int end = min(start + CHUNK, n);

  const int lane = threadIdx.x & 31;
  const int hw = threadIdx.x >> 4;   // half-warp 0..15 (keys start + hw + 16 i)
  const int sub = lane & 15;         // 16-byte slice of the row
  const size_t bhh = static_cast<size_t>(b) * a.H + h;

  float qf[8];
  unpack8<T>(*reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.q) + bhh * D + sub * 8), qf);
  const float sl2 = a.scale_log2;
#pragma unroll
  for (int e = 0; e < 8; ++e) qf[e] *= sl2;  // scores come out in exp2 units

  // Row r of the cache is at kb + r * D: r = key (contiguous) or, paged, the row of the
  // key's physical block (the table is read per key row; rows of a block share an entry).
  const size_t base = PAGED ? 0 : bhh * a.cap * D;
  const uint16_t* kb = static_cast<const uint16_t*>(a.kcache) + base + sub * 8;
  const uint16_t* vb = static_cast<const uint16_t*>(a.vcache) + base + sub * 8;
  const int bmask = (1 << a.block_shift) - 1;
  bool bad_block = false;
  // The chunk's block-table entries, staged once in shared memory so that no key
  // row waits on a dependent table load (at most CHUNK + 1 entries).
  __shared__ int sm_blk[PAGED ? CHUNK + 1 : 1];
  const int blk0 = start >> a.block_shift;
  if (PAGED) {
    const int32_t* table = a.block_table + static_cast<size_t>(b) * a.max_blocks;
    const int nblk = ((end - 1) >> a.block_shift) - blk0 + 1;
    for (int i = threadIdx.x; i < nblk; i += THREADS) sm_blk[i] = table[blk0 + i];
    __syncthreads();
  }

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  // The loop bound is warp-uniform (both half-warps run the same trip count), so the
  // full-warp shuffles below always see all 32 lanes; each key is checked on its own.
  const int half = (threadIdx.x >> 4) & 1;
  const int warp = threadIdx.x >> 5;
  for (int kbase = start + 2 * warp; kbase < end; kbase += HALVES * U) {
    uint4 kr[U], vr[U];
    bool live[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int key = kbase + half + u * HALVES;
      live[u] = key < end;
      size_t r = static_cast<size_t>(key);
      if (PAGED && live[u]) {
        const int phys = sm_blk[(key >> a.block_shift) - blk0];
        if (phys < 0 || phys >= a.num_blocks) {
          bad_block = true;
          live[u] = false;
        } else {
          r = ((static_cast<size_t>(phys) * a.H + h) << a.block_shift) + (key & bmask);
        }
      }
      if (live[u]) {
        kr[u] = ld_stream(kb + r * D);
        vr[u] = ld_stream(vb + r * D);
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
    float s[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float kf[8];
      unpack8<T>(kr[u], kf);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      s[u] = live[u] ? dot : -INFINITY;
    }
    float mx = s[0];
#pragma unroll
    for (int u = 1; u < U; ++u) mx = fmaxf(mx, s[u]);
    const float m_new = fmaxf(m, mx);
    // A half-warp may have no valid key in this step (and none before): keep its
    // state unchanged instead of forming (-inf) - (-inf).
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = ex2_approx(m - m_use);  // m = -inf gives 0: nothing accumulated yet
    l *= alpha;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float p = ex2_approx(s[u] - m_use);
      l += p;
      float vf[8];
      unpack8<T>(vr[u], vf);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(p, vf[e], acc[e]);
    }
    m = m_new;
  }

  if (PAGED && bad_block) atomicOr(&g_status, kStatusBadBlock);

  // Merge the 16 half-warp states (exp2 units) through shared memory.
  __shared__ float sm_m[HALVES], sm_l[HALVES];
  __shared__ float sm_acc[HALVES][D];
  if (sub == 0) {
    sm_m[hw] = m;
    sm_l[hw] = l;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) sm_acc[hw][sub * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    const int e = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < HALVES; ++i) M = fmaxf(M, sm_m[i]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int i = 0; i < HALVES; ++i) {
      const float w = (sm_m[i] == -INFINITY) ? 0.f : ex2_approx(sm_m[i] - M);
      L = fmaf(sm_l[i], w, L);
      O = fmaf(sm_acc[i][e], w, O);
    }
    const size_t row = bhh * a.max_chunks + c;
    a.ws_o[row * D + e] = O / L;
    if (e == 0) a.ws_lse[row] = (M + log2f(L)) * 0.69314718055994531f;  // natural log
  }
}

template <bool PAGED, class T>
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeArgs a) {
  const size_t bhh = blockIdx.x;
  const int b = static_cast<int>(bhh / a.H);
  const int n = min(max(a.seqlens[b], 0), a.cap);
  constexpr int CHUNK = chunk_keys<PAGED>();
  const int chunks = (n + CHUNK - 1) / CHUNK;
  const int e = threadIdx.x;
  uint16_t* o = static_cast<uint16_t*>(a.o) + bhh * D;
  if (chunks == 0) {
    o[e] = to16<T>(0.f);
    if (e == 0 && a.lse) a.lse[bhh] = -INFINITY;
    return;
  }
  const float* ls = a.ws_lse + bhh * a.max_chunks;
  const float* os = a.ws_o + bhh * a.max_chunks * D;
  float M = -INFINITY;
  for (int c = 0; c < chunks; ++c) M = fmaxf(M, ls[c]);
  float W = 0.f, O = 0.f;
  for (int c = 0; c < chunks; ++c) {
    const float w = __expf(ls[c] - M);
    W += w;
    O = fmaf(w, os[static_cast<size_t>(c) * D + e], O);
  }
  o[e] = to16<T>(O / W);
  if (e == 0 && a.lse) a.lse[bhh] = M + logf(W);
}

}  // namespace dec

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  using namespace dec;
  if (a.H > 65535 || a.B > 65535) return cudaErrorInvalidValue;
  // a.max_chunks counts kDecodeChunk-key chunks (it sizes the workspace); a paged
  // CTA takes four of them.
  const bool paged = a.block_table != nullptr;
  const dim3 grid(paged ? (a.max_chunks + 3) / 4 : a.max_chunks, a.H, a.B);
  if (paged)
    (a.f16 ? decode_split_kernel<true, F16> : decode_split_kernel<true, Bf16>)<<<grid, THREADS, 0, stream>>>(a);
  else
    (a.f16 ? decode_split_kernel<false, F16> : decode_split_kernel<false, Bf16>)<<<grid, THREADS, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned rows = static_cast<unsigned>(a.B * a.H);
  if (paged)
    (a.f16 ? decode_combine_kernel<true, F16> : decode_combine_kernel<true, Bf16>)<<<rows, D, 0, stream>>>(a);
  else
    (a.f16 ? decode_combine_kernel<false, F16> : decode_combine_kernel<false, Bf16>)<<<rows, D, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t take_status_decode(unsigned int* out) { return take_local_status(out); }

}  // namespace fa
