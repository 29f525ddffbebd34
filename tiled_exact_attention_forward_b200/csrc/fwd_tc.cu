// Forward pass on the 5th-generation tensor cores (sm_100a): tcgen05 MMAs with
// fp32 accumulators in tensor memory, K/V tiles streamed by TMA through a
// shared-memory ring, and the online softmax in registers.
//
// Algorithm ("Building Flash Attention from Scratch in Pure NumPy",
// architecture overview and Step 2): for each 128-row query tile, keep a row
// max m, row sum l and unnormalised output O; for each 128-key tile
// S = Q K^T, m_new = max(m, rowmax S), P = exp(S - m_new),
// l = exp(m - m_new) l + rowsum P, O = exp(m - m_new) O + P V; finally
// O / l and lse = m + ln l.  Masks and tile skipping follow "Build a
// FlashAttention-2 Inference Kernel from Scratch in Pure Python", Step 3.
//
// B200 design:
//   * One CTA owns two query tiles (256 rows) of one (batch, head) and
//     streams the union of their key ranges once.  Key tiles that the causal
//     or window mask hides from every row of a query tile are never loaded
//     for it; only tiles that straddle a mask edge (or the ragged end of the
//     sequence) get the per-element mask.
//   * Warp roles (320 threads): warps 0-3 and 4-7 are two softmax
//     warpgroups, one per query tile (thread = one query row = one TMEM
//     lane); warp 8 allocates tensor memory and issues every MMA from one
//     thread; warp 9 issues the TMA loads.
//   * Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each.
//     The softmax writes P (bf16 pairs) over the first 64 columns of its S
//     tile, and O += P V reads P straight from tensor memory (A operand in
//     TMEM), so P never touches shared memory.
//   * MMA issue order per key tile j (ping-pong):
//       PV0(j), S0(j+1), PV1(j), S1(j+1)
//     so one tile's softmax overlaps the other tile's MMAs.  MMAs of one
//     thread complete in issue order, so when S_t(j) is complete, PV_t(j-1)
//     is too: the softmax may then rescale O_t without a further wait.
//   * Lazy rescale: the running max m moves (and O, l are rescaled) only
//     when the new row max exceeds it by more than 2^8 in exp2 units; P is
//     then at most 256, exact in the final O / l.
//   * exp2 with scale*log2(e) folded into one FFMA per score.
#include "common.cuh"
#include "kernels.h"

namespace fa {

namespace fwdtc {

constexpr int BM = 128;                 // query rows per tile
constexpr int BN = 128;                 // keys per tile
constexpr int D = 128;                  // head dimension
constexpr int NS = 4;                   // K/V ring stages (K and V tiles interleaved)
constexpr int TILE_BYTES = BM * D * 2;  // one 128 x 128 bf16 tile = 32 KiB
constexpr int HALF_BYTES = TILE_BYTES / 2;  // one 64-column half (a 128-byte-swizzled box)
constexpr int NUM_THREADS = 320;
constexpr int MMA_WARP = 8;
constexpr int TMA_WARP = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Smem {
  // 1024-byte aligned by construction (the dynamic buffer is aligned at runtime).
  uint8_t q[2][TILE_BYTES];
  uint8_t kv[NS][TILE_BYTES];
  uint64_t q_full[2];
  uint64_t kv_full[NS];
  uint64_t kv_empty[NS];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

// Key-tile range [lo, hi) a query tile starting at row r0 must visit.
__device__ __forceinline__ void key_tile_range(int r0, int n, int causal, int window, int& lo,
                                               int& hi) {
  const int rlast = min(r0 + BM - 1, n - 1);
  hi = causal ? (rlast / BN + 1) : (n + BN - 1) / BN;
  const int first_key = window > 0 ? r0 - window + 1 : 0;
  lo = first_key > 0 ? first_key / BN : 0;
  if (lo > hi) lo = hi;
}

// Does key tile j need the per-element mask for rows r0..r0+BM-1?
__device__ __forceinline__ bool tile_needs_mask(int j, int r0, int n, int causal, int window) {
  const int k0 = j * BN, k1 = j * BN + BN - 1;
  const int rlast = min(r0 + BM - 1, n - 1);
  return (k1 >= n) || (causal && k1 > r0) || (window > 0 && k0 <= rlast - window);
}

__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
    const uint64_t a = smem_desc_sw128(q_smem + off, 16, 1024);
    const uint64_t b = smem_desc_sw128(k_smem + off, 16, 1024);
    mma_ss(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_smem,
                                         bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(BM, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    // V tile: [64-column half][128 keys][64 cols]; a K step of 16 keys = 16 rows.
    const uint64_t b = smem_desc_sw128(v_smem + kk * 16 * 128, HALF_BYTES, 1024);
    mma_ts(d_tmem, p_tmem + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, FwdArgs args) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BH = args.B * args.H;
  const int n = args.N;
  const int num_pairs = (n + 2 * BM - 1) / (2 * BM);
  // Heaviest work first: with a causal mask the last query tiles see the most keys.
  const int pair = num_pairs - 1 - static_cast<int>(blockIdx.x) / BH;
  const int bh = static_cast<int>(blockIdx.x) % BH;

  int r0[2], lo_t[2], hi_t[2];
  r0[0] = pair * 2 * BM;
  r0[1] = r0[0] + BM;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (r0[t] < n) {
      key_tile_range(r0[t], n, args.causal, args.window, lo_t[t], hi_t[t]);
    } else {
      lo_t[t] = hi_t[t] = 0;
    }
  }
  const bool has1 = r0[1] < n;
  const int lo = has1 ? min(lo_t[0], lo_t[1]) : lo_t[0];
  const int hi = has1 ? max(hi_t[0], hi_t[1]) : hi_t[0];

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&sm.q_full[t]), 1);
      mbar_init(smem_u32(&sm.s_full[t]), 1);
      mbar_init(smem_u32(&sm.p_full[t]), BM);
      mbar_init(smem_u32(&sm.o_full[t]), 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&sm.kv_full[s]), 1);
      mbar_init(smem_u32(&sm.kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.mma_done), 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == TMA_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int nt = has1 ? 2 : 1;
      for (int t = 0; t < nt; ++t) {
        const uint32_t bar = smem_u32(&sm.q_full[t]);
        mbar_arrive_expect_tx(bar, TILE_BYTES);
        tma_load_3d(smem_u32(sm.q[t]), &tm_q, bar, 0, r0[t], bh);
        tma_load_3d(smem_u32(sm.q[t]) + HALF_BYTES, &tm_q, bar, 64, r0[t], bh);
      }
      const int total = 2 * (hi - lo);
      int issued = 0;
      for (int idx = 0; idx < total; ++idx) {
        const int s = idx % NS;
        if (idx >= NS) {
          if (!mbar_wait(smem_u32(&sm.kv_empty[s]), ((idx / NS) - 1) & 1, abort_flag)) break;
        }
        const int j = lo + (idx >> 1);
        const CUtensorMap* tm = (idx & 1) ? &tm_v : &tm_k;
        const uint32_t bar = smem_u32(&sm.kv_full[s]);
        mbar_arrive_expect_tx(bar, TILE_BYTES);
        tma_load_3d(smem_u32(sm.kv[s]), tm, bar, 0, j * BN, bh);
        tma_load_3d(smem_u32(sm.kv[s]) + HALF_BYTES, tm, bar, 64, j * BN, bh);
        issued = idx + 1;
      }
      // Drain: every copy issued must land before the CTA may exit.
      for (int idx = max(0, issued - NS); idx < issued; ++idx)
        mbar_wait_drain(smem_u32(&sm.kv_full[idx % NS]), (idx / NS) & 1);
      for (int t = 0; t < nt; ++t) mbar_wait_drain(smem_u32(&sm.q_full[t]), 0);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS[2] = {tmem + 0, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 384};
      const uint32_t q_s[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      int it[2] = {0, 0};
      bool ok = true;
      auto act = [&](int t, int j) { return j >= lo_t[t] && j < hi_t[t]; };
      auto stage_of = [&](int idx) { return idx % NS; };
      auto parity_of = [&](int idx) { return static_cast<uint32_t>((idx / NS) & 1); };

      ok = mbar_wait(smem_u32(&sm.q_full[0]), 0, abort_flag);
      if (ok && has1) ok = mbar_wait(smem_u32(&sm.q_full[1]), 0, abort_flag);
      if (ok && hi > lo) {
        // Prologue: S_t(lo) for both tiles.
        int kidx = 0;
        ok = mbar_wait(smem_u32(&sm.kv_full[stage_of(kidx)]), parity_of(kidx), abort_flag);
        if (ok) {
          tc_fence_after();
          const uint32_t ks = smem_u32(sm.kv[stage_of(kidx)]);
          for (int t = 0; t < 2; ++t)
            if (act(t, lo)) {
              issue_qk(tS[t], q_s[t], ks);
              tc_commit(smem_u32(&sm.s_full[t]));
            }
          tc_commit(smem_u32(&sm.kv_empty[stage_of(kidx)]));
        }
        for (int j = lo; ok && j < hi; ++j) {
          const int vidx = 2 * (j - lo) + 1;
          const int nidx = vidx + 1;
          const bool has_next = j + 1 < hi;
          ok = mbar_wait(smem_u32(&sm.kv_full[stage_of(vidx)]), parity_of(vidx), abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vs = smem_u32(sm.kv[stage_of(vidx)]);
          // Tile 0: PV0(j), then S0(j+1).
          if (act(0, j)) {
            ok = mbar_wait(smem_u32(&sm.p_full[0]), it[0] & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            issue_pv(tO[0], tS[0], vs, it[0] > 0);
            ++it[0];
            if (j == hi_t[0] - 1) tc_commit(smem_u32(&sm.o_full[0]));
          }
          uint32_t ks = 0;
          if (has_next) {
            ok = mbar_wait(smem_u32(&sm.kv_full[stage_of(nidx)]), parity_of(nidx), abort_flag);
            if (!ok) break;
            tc_fence_after();
            ks = smem_u32(sm.kv[stage_of(nidx)]);
            if (act(0, j + 1)) {
              issue_qk(tS[0], q_s[0], ks);
              tc_commit(smem_u32(&sm.s_full[0]));
            }
          }
          // Tile 1: PV1(j), then S1(j+1).
          if (act(1, j)) {
            ok = mbar_wait(smem_u32(&sm.p_full[1]), it[1] & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            issue_pv(tO[1], tS[1], vs, it[1] > 0);
            ++it[1];
            if (j == hi_t[1] - 1) tc_commit(smem_u32(&sm.o_full[1]));
          }
          tc_commit(smem_u32(&sm.kv_empty[stage_of(vidx)]));
          if (has_next) {
            if (act(1, j + 1)) {
              issue_qk(tS[1], q_s[1], ks);
              tc_commit(smem_u32(&sm.s_full[1]));
            }
            tc_commit(smem_u32(&sm.kv_empty[stage_of(nidx)]));
          }
        }
      }
      // All MMAs issued by this thread must complete before TMEM is freed.
      tc_commit(smem_u32(&sm.mma_done));
      mbar_wait_drain(smem_u32(&sm.mma_done), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;  // query tile of this warpgroup
    const int wq = warp & 3;  // warp within the warpgroup -> TMEM lanes 32*wq..
    const int row = wq * 32 + lane;
    const int row_g = r0[t] + row;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * 128;
    const float sl2 = args.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    int it = 0;
    if (t == 0 || has1) {
      for (int j = lo_t[t]; j < hi_t[t]; ++j, ++it) {
        ok = mbar_wait_warp(smem_u32(&sm.s_full[t]), it & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        uint32_t s[BN];
        FA_TMEM_LD32(tS + 0, (s + 0));
        FA_TMEM_LD32(tS + 32, (s + 32));
        FA_TMEM_LD32(tS + 64, (s + 64));
        FA_TMEM_LD32(tS + 96, (s + 96));
        tmem_ld_wait();
        if (tile_needs_mask(j, r0[t], n, args.causal, args.window)) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (!key_visible(row_g, j * BN + c, n, args.causal, args.window))
              s[c] = __float_as_uint(-INFINITY);
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; ++c) mx = fmaxf(mx, __uint_as_float(s[c]));
        const float m_new = fmaxf(m, mx);
        // (m_new - m) is +inf on the first visible tile and NaN while the row is
        // still empty; only the former moves the reference max.
        const bool need = (m_new - m) * sl2 > kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx((m - m_new) * sl2);
          m = m_new;
          l *= alpha;
        }
        const float ms = (m == -INFINITY) ? 0.f : m * sl2;
        float rs = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // P columns [32h, 32h + 32) hold keys [64h, 64h + 64); S there is already in registers.
          uint32_t p[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(s[64 * h + 2 * c]), sl2, -ms));
            const float p1 = ex2_approx(fmaf(__uint_as_float(s[64 * h + 2 * c + 1]), sl2, -ms));
            rs += p0 + p1;
            p[c] = pack_bf16x2(p0, p1);
          }
          FA_TMEM_ST32(tS + 32 * h, p);
        }
        if (it > 0 && __any_sync(0xffffffffu, need)) {
          // O_t's last update (PV_t(j-1)) is complete: S_t(j) was issued after it.  The
          // rescale happens after P is stored (S is no longer live) and before p_full.
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            FA_TMEM_LD32(tO + 32 * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            FA_TMEM_ST32(tO + 32 * c, r);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.p_full[t]));
        l += rs;
      }
      // Epilogue: O / l in bf16 and lse = m * scale + ln l.
      if (ok && hi_t[t] > lo_t[t]) ok = mbar_wait_warp(smem_u32(&sm.o_full[t]), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16* orow =
            reinterpret_cast<__nv_bfloat16*>(args.o) + (static_cast<size_t>(bh) * n + row_g) * D;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          FA_TMEM_LD32(tO + 32 * c, r);
          tmem_ld_wait();
          if (row_g < n) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(r[8 * v4 + 0]) * inv, __uint_as_float(r[8 * v4 + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(r[8 * v4 + 2]) * inv, __uint_as_float(r[8 * v4 + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(r[8 * v4 + 4]) * inv, __uint_as_float(r[8 * v4 + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(r[8 * v4 + 6]) * inv, __uint_as_float(r[8 * v4 + 7]) * inv);
              dst[v4] = w;
            }
          }
        }
        if (row_g < n && args.lse != nullptr)
          args.lse[static_cast<size_t>(bh) * n + row_g] =
              l > 0.f ? m * args.scale + logf(l) : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fwdtc

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t stream) {
  using namespace fwdtc;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_rows(&tq, a.q, D, a.N, static_cast<long long>(a.B) * a.H, BM) ||
      !make_tmap_bf16_rows(&tk, a.k, D, a.N, static_cast<long long>(a.B) * a.H, BN) ||
      !make_tmap_bf16_rows(&tv, a.v, D, a.N, static_cast<long long>(a.B) * a.H, BN))
    return cudaErrorInvalidValue;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(fwd_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  const int num_pairs = (a.N + 2 * BM - 1) / (2 * BM);
  const long long grid = static_cast<long long>(num_pairs) * a.B * a.H;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  fwd_tc_kernel<<<static_cast<unsigned>(grid), NUM_THREADS, kSmemBytes, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace fa
