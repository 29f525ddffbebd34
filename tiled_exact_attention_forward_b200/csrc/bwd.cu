// Backward pass (bf16 or f16, d = 128) on the tensor cores.
//
// "Building Flash Attention from Scratch in Pure NumPy", Step 4: precompute
// D = rowsum(dO * O); then for each key tile, loop over the query tiles that
// can see it, recompute the probabilities from the saved row statistic and
// accumulate the gradients.  That page's own dK/dQ lines are declared
// simplified; the exact gradients of the forward are used instead:
//     P = exp(S * scale - lse),  dV += P^T dO,  dP = dO V^T,
//     dS = P * (dP - D),  dK += scale * dS^T Q,  dQ += scale * dS K.
//
// Kernels: bwd_pre (D and zeroed fp32 dQ accumulator), bwd_main (below),
// bwd_post (dQ fp32 -> the inputs' 16-bit type).
//
// bwd_main, one CTA per (batch*head, 128-key tile), 576 threads, the CTAs dealt
// in groups of 8 heads (low key tiles first within a group) so the CTAs in flight
// keep a few heads' Q, dO and dQ accumulator in L2:
//   * warp 17 loads K and V once, then (Q_i, dO_i) pairs by TMA into a
//     two-stage ring;
//   * warp 16 allocates tensor memory and issues the MMAs: a warp-uniform loop,
//     each block of MMAs one asm statement issued by an elected lane;
//   * warps 0-7 turn S^T, dP^T into P^T and dS^T: warp w handles the key rows
//     of TMEM lane quarter w%4 and, in each 64-query half of the tile, the 32
//     queries selected by w/4 -- two threads per key row, the halves one after
//     the other (the first half's dV and dK MMAs run under the second half).
//     P^T and dS^T go back into tensor memory as 16-bit pairs (operands of the
//     dV and dK MMAs) and dS^T also into shared memory (operand of the dQ MMA);
//   * warps 8-15 read dQ_i out of tensor memory (two threads per query row,
//     64 columns each), stage it in the finished (Q_i, dO_i) ring slot and add
//     it into the fp32 accumulator with TMA bulk reduce-adds, so no per-thread
//     global atomics compete with the P/dS warps' shared-memory traffic; at the
//     end warps 0-7 write dV and warps 8-15 write dK.
// Tensor memory (512 columns): [S^T -> P^T, later dQ_i] [dP^T -> dS^T] [dV] [dK].
// Keys are the MMA rows of S^T = K Q^T and dP^T = V dO^T, so P^T and dS^T
// land with keys on lanes -- exactly the A operands dV and dK need.
#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace bwd {

constexpr int BM = 128;  // keys per CTA (MMA rows)
constexpr int BQ = 128;  // queries per inner tile
constexpr int D = 128;
constexpr int TILE_BYTES = 128 * D * 2;
constexpr int HALF_BYTES = TILE_BYTES / 2;
constexpr int NUM_THREADS = 576;
constexpr int GROUP = 256;  // threads of the P/dS group and of the dQ group
constexpr int MMA_WARP = 16;
constexpr int TMA_WARP = 17;

struct Smem {
  uint8_t k[TILE_BYTES];
  uint8_t v[TILE_BYTES];
  uint8_t q[2][TILE_BYTES];
  uint8_t dout[2][TILE_BYTES];
  uint8_t ds[TILE_BYTES];  // dS as [query half][key][64 queries], 128-byte swizzle
  float lse2[2][BQ];       // lse * log2(e) of the query tile (+inf past N)
  float delta[2][BQ];
  uint64_t kv_full;
  uint64_t qdo_full[2];
  uint64_t qdo_empty[2];
  uint64_t s_full, dp_full, ds_ready, dq_full, dq_free, acc_done;
  uint32_t tmem_base;
  int abort_flag;
};
constexpr size_t kSmemBytes = sizeof(Smem);
static_assert(kSmemBytes <= 232448, "backward shared memory exceeds the sm_100 limit");

__device__ __forceinline__ void q_tile_range(int kt, int n, int causal, int window, int& lo, int& hi) {
  const int k0 = kt * BM;
  const int k1 = min(k0 + BM - 1, n - 1);
  const int ntiles = (n + BQ - 1) / BQ;
  lo = causal ? k0 / BQ : 0;
  hi = ntiles;
  if (window > 0) hi = min(hi, (k1 + window - 1) / BQ + 1);
  if (lo > hi) lo = hi;
}

__device__ __forceinline__ bool tile_needs_mask(int kt, int qi, int n, int causal, int window) {
  const int k0 = kt * BM, k1 = k0 + BM - 1;
  const int q0 = qi * BQ, q1 = q0 + BQ - 1;
  return (k1 >= n) || (causal && q0 < k1) || (window > 0 && q1 - k0 >= window);
}

// The MMA warp runs warp-uniformly; each 128-deep K block of MMAs is one asm
// statement (one elect, descriptor low words stepped by immediates: mma8_ss,
// mma4_ts), which issues as fast as the tensor core retires them, where one asm
// statement per MMA did not.
__device__ __forceinline__ void commit_elect(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}
// Low word of a 128-byte-swizzled descriptor (start address, leading-byte offset);
// the high word (stride 1024, version, swizzle) is kDescHi for every tile here.
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr, uint32_t lbo) {
  return static_cast<uint32_t>(smem_desc_sw128(saddr, lbo, 1024));
}
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);

// A = [rows][d] tile, K-major; B = [rows][d] tile, K-major: D[128x128] = A B^T.
template <class T>
__device__ __forceinline__ void issue_abT(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo) {
  constexpr uint32_t h = HALF_BYTES >> 4, idesc = idesc_f32acc<T>(128, 128, 0, 0);
  static_assert(D / 16 == 8, "one 8-MMA block");
  mma8_ss<idesc, 2, 4, 6, h, h + 2, h + 4, h + 6>(d_tmem, a_lo, b_lo, kDescHi, 0u);
}

// D[128 x d] (+)= A[tmem, 128 keys x 64 queries of half H, 16-bit] * B, B = [128 rows (K)][d]
// tile (MN-major), rows 64H .. 64H + 63.  The A columns of queries [16k, 16k + 16) sit at
// TMEM columns 64 (k / 4) + 32 ((k % 4) / 2) + 8 (k % 2) (16-bit pairs), where the P/dS
// thread that owns those queries wrote them over S^T / dP^T columns it had read; B's K step
// k is 16 rows = 2 KiB on.
template <int H, class T>
__device__ __forceinline__ void issue_tmemA_b_half(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                                   uint32_t accumulate) {
  constexpr uint32_t idesc = idesc_f32acc<T>(128, D, 0, 1), c0 = 64 * H, o0 = (4 * H * 2048) >> 4;
  mma4_ts<idesc, c0, c0 + 8, c0 + 32, c0 + 40, o0, o0 + 128, o0 + 256, o0 + 384>(d_tmem, a_tmem, b_lo, kDescHi,
                                                                                accumulate);
}

// dQ[128 queries x d] = dS (A, MN-major in smem) * K (B, MN-major in smem); K step k
// is 16 rows = 2 KiB on in both.
template <class T>
__device__ __forceinline__ void issue_dq(uint32_t d_tmem, uint32_t ds_lo, uint32_t k_lo) {
  constexpr uint32_t idesc = idesc_f32acc<T>(128, D, 1, 1);
  static_assert(BM / 16 == 8, "one 8-MMA block");
  mma8_ss<idesc, 128, 256, 384, 512, 640, 768, 896>(d_tmem, ds_lo, k_lo, kDescHi, 0u);
}

// T: the 16-bit type of Q, K, V, dO, P, dS and the gradients (Bf16 or F16).
template <class T>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, BwdArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(&g_status, kStatusTimeout);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = args.N;
  const int BH = args.B * args.H;
  const int nkt = (n + BM - 1) / BM;
  // CTAs go out in groups of kHeadGroup heads: within a group, low key tiles (which see
  // the most query tiles under a causal mask) first, across the group's heads.  The
  // CTAs in flight then cover about kHeadGroup heads, whose Q, dO and fp32 dQ
  // accumulator stay in L2, instead of every head at once; a simulated list schedule
  // of the causal workload keeps the same makespan as key-tile-major over all heads.
  constexpr int kHeadGroup = 8;
  const int g = BH < kHeadGroup ? BH : kHeadGroup;
  const int full = BH / g, rem = BH % g;
  const int idx = static_cast<int>(blockIdx.x);
  int kt, bh;
  if (idx < full * g * nkt) {
    const int grp = idx / (g * nkt), r = idx % (g * nkt);
    kt = r / g;
    bh = grp * g + r % g;
  } else {
    const int r = idx - full * g * nkt;
    kt = r / rem;
    bh = full * g + r % rem;
  }
  int qlo, qhi;
  q_tile_range(kt, n, args.causal, args.window, qlo, qhi);
  const int nq = qhi - qlo;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.kv_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&sm.qdo_full[s]), 1);
      // Two arrivals free a (Q, dO) slot: the MMAs that read it, and the TMA reduce
      // that read the dQ staged in it afterwards.
      mbar_init(smem_u32(&sm.qdo_empty[s]), 2);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.dp_full), 1);
    mbar_init(smem_u32(&sm.ds_ready), GROUP);
    mbar_init(smem_u32(&sm.dq_full), 1);
    mbar_init(smem_u32(&sm.dq_free), GROUP);
    mbar_init(smem_u32(&sm.acc_done), 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 384;

  if (warp == TMA_WARP) {
    if (lane == 0 && nq > 0) {
      const uint32_t kvb = smem_u32(&sm.kv_full);
      mbar_arrive_expect_tx(kvb, 2 * TILE_BYTES);
      tma_load_3d(smem_u32(sm.k), &tm_k, kvb, 0, kt * BM, bh);
      tma_load_3d(smem_u32(sm.k) + HALF_BYTES, &tm_k, kvb, 64, kt * BM, bh);
      tma_load_3d(smem_u32(sm.v), &tm_v, kvb, 0, kt * BM, bh);
      tma_load_3d(smem_u32(sm.v) + HALF_BYTES, &tm_v, kvb, 64, kt * BM, bh);
      int issued = 0;
      for (int idx = 0; idx < nq; ++idx) {
        const int s = idx & 1;
        if (idx >= 2 && !mbar_wait(smem_u32(&sm.qdo_empty[s]), ((idx >> 1) - 1) & 1, abort_flag)) break;
        const int row = (qlo + idx) * BQ;
        const uint32_t b = smem_u32(&sm.qdo_full[s]);
        mbar_arrive_expect_tx(b, 2 * TILE_BYTES);
        tma_load_3d(smem_u32(sm.q[s]), &tm_q, b, 0, row, bh);
        tma_load_3d(smem_u32(sm.q[s]) + HALF_BYTES, &tm_q, b, 64, row, bh);
        tma_load_3d(smem_u32(sm.dout[s]), &tm_do, b, 0, row, bh);
        tma_load_3d(smem_u32(sm.dout[s]) + HALF_BYTES, &tm_do, b, 64, row, bh);
        issued = idx + 1;
      }
      mbar_wait_drain(kvb, 0);
      for (int idx = max(0, issued - 2); idx < issued; ++idx)
        mbar_wait_drain(smem_u32(&sm.qdo_full[idx & 1]), (idx >> 1) & 1);
    }
  } else if (warp == MMA_WARP) {
    // Warp-uniform loop; MMAs and commits from one elected lane.  Waits on the K/V
    // and (Q, dO) barriers need no tcgen05 fence (TMA data); waits on barriers the
    // P/dS and dQ warps arrive on (after their tcgen05 loads/stores) do.
    if (nq > 0) {
      const uint32_t kd = desc_lo(smem_u32(sm.k), 16), vd = desc_lo(smem_u32(sm.v), 16);
      const uint32_t dsd = desc_lo(smem_u32(sm.ds), HALF_BYTES), kmn = desc_lo(smem_u32(sm.k), HALF_BYTES);
      auto qd = [&](int s) { return desc_lo(smem_u32(sm.q[s]), 16); };
      auto dod = [&](int s) { return desc_lo(smem_u32(sm.dout[s]), 16); };
      auto qmn = [&](int s) { return desc_lo(smem_u32(sm.q[s]), HALF_BYTES); };
      auto domn = [&](int s) { return desc_lo(smem_u32(sm.dout[s]), HALF_BYTES); };
      bool ok = mbar_wait_warp(smem_u32(&sm.kv_full), 0, abort_flag);
      if (ok) ok = mbar_wait_warp(smem_u32(&sm.qdo_full[0]), 0, abort_flag);
      if (ok) {
        issue_abT<T>(tmem + T_S, kd, qd(0));
        commit_elect(smem_u32(&sm.s_full));
        issue_abT<T>(tmem + T_DP, vd, dod(0));
        commit_elect(smem_u32(&sm.dp_full));
      }
      for (int idx = 0; ok && idx < nq; ++idx) {
        const int s = idx & 1;
        // dV and dK for query half 0 as soon as its P^T and dS^T are in TMEM (they run
        // while the P/dS warps work on half 1), then half 1 (two ds_ready phases per
        // query tile: parity 0, then 1).
        ok = mbar_wait_warp(smem_u32(&sm.ds_ready), 0, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_tmemA_b_half<0, T>(tmem + T_DV, tmem + T_S, domn(s), idx > 0 ? 1u : 0u);
        issue_tmemA_b_half<0, T>(tmem + T_DK, tmem + T_DP, qmn(s), idx > 0 ? 1u : 0u);
        ok = mbar_wait_warp(smem_u32(&sm.ds_ready), 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_tmemA_b_half<1, T>(tmem + T_DV, tmem + T_S, domn(s), 1u);
        issue_tmemA_b_half<1, T>(tmem + T_DK, tmem + T_DP, qmn(s), 1u);
        commit_elect(smem_u32(&sm.qdo_empty[s]));
        issue_dq<T>(tmem + T_S, dsd, kmn);
        commit_elect(smem_u32(&sm.dq_full));
        if (idx + 1 < nq) {
          const int s1 = (idx + 1) & 1;
          ok = mbar_wait_warp(smem_u32(&sm.qdo_full[s1]), ((idx + 1) >> 1) & 1, abort_flag);
          if (!ok) break;
          // S^T of the next tile first (its columns hold dQ until the read-out frees
          // them): the P/dS warps start on P^T as soon as it lands, and dP^T, needed
          // only for dS^T, follows it (measured 0.5 % faster than dP^T first).
          ok = mbar_wait_warp(smem_u32(&sm.dq_free), idx & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_abT<T>(tmem + T_S, kd, qd(s1));
          commit_elect(smem_u32(&sm.s_full));
          issue_abT<T>(tmem + T_DP, vd, dod(s1));
          commit_elect(smem_u32(&sm.dp_full));
        }
      }
      commit_elect(smem_u32(&sm.acc_done));
      mbar_wait_drain(smem_u32(&sm.acc_done), 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // -------------------------------------------------- P^T and dS^T (thread = key row x 32 queries
    // of each query half, the halves one after the other)
    const int hc = warp >> 2;  // which 32 queries of a half (and, at the end, which dV columns)
    const int row = (warp & 3) * 32 + lane;
    const int key = kt * BM + row;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tSb = tmem + lane_off + T_S + 32 * hc, tDPb = tmem + lane_off + T_DP + 32 * hc;
    const float sl2 = args.scale_log2;
    const float* lse_g = args.lse + static_cast<size_t>(bh) * n;
    const float* del_g = args.ws_delta + static_cast<size_t>(bh) * n;
    const int gt = threadIdx.x;  // 0..255: loads row statistic gt & 127 (lse if < 128, else D)
    bool ok = true;
    // Prefetch the first tile's row statistics.
    float stat_next = 0.f;
    auto load_stat = [&](int qt) {
      const int qi = qt * BQ + (gt & 127);
      if (gt < 128) {
        float v = INFINITY;  // past N: P = 2^(-inf) = 0
        if (qi < n) {
          const float l = lse_g[qi];
          v = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
        }
        return v;
      }
      return qi < n ? del_g[qi] : 0.f;
    };
    if (nq > 0) stat_next = load_stat(qlo);
    for (int idx = 0; idx < nq; ++idx) {
      const int s = idx & 1;
      if (gt < 128) sm.lse2[s][gt] = stat_next; else sm.delta[s][gt - 128] = stat_next;
      named_bar_sync(1, GROUP);
      if (idx + 1 < nq) stat_next = load_stat(qlo + idx + 1);
      const int qt = qlo + idx;
      const bool masked = tile_needs_mask(kt, qt, n, args.causal, args.window);
      ok = mbar_wait(smem_u32(&sm.s_full), idx & 1, abort_flag);
      if (ok) ok = mbar_wait(smem_u32(&sm.dp_full), idx & 1, abort_flag);
      // One decision for the whole group: it meets at named barrier 1 every step.
      ok = named_bar_all(ok, 2, GROUP);
      if (!ok) break;
      tc_fence_after();
      for (int h = 0; h < 2; ++h) {
        const uint32_t tS = tSb + 64 * h, tDP = tDPb + 64 * h;
        // Visible queries of this key row form one interval [q_lo, q_hi) of its 32.
        int q_lo = 0, q_hi = 32;
        if (masked) {
          const int qbase = qt * BQ + 64 * h + 32 * hc;
          if (args.causal) q_lo = max(0, key - qbase);
          if (args.window > 0) q_hi = min(32, key + args.window - qbase);
          q_hi = min(q_hi, n - qbase);  // queries past N have lse2 = +inf anyway
          if (key >= n) q_hi = 0;
          q_hi = max(q_hi, q_lo);  // an empty interval keeps nothing
        }
        const float4* l4 = reinterpret_cast<const float4*>(&sm.lse2[s][64 * h + 32 * hc]);
        const float4* d4 = reinterpret_cast<const float4*>(&sm.delta[s][64 * h + 32 * hc]);
        uint8_t* ds_row = sm.ds + h * HALF_BYTES + row * 128;
        // 16 query columns per step keeps S^T, dP^T and both outputs in registers.
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sr[16], dr[16];
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
              : "=r"(sr[0]), "=r"(sr[1]), "=r"(sr[2]), "=r"(sr[3]), "=r"(sr[4]), "=r"(sr[5]), "=r"(sr[6]), "=r"(sr[7]),
                "=r"(sr[8]), "=r"(sr[9]), "=r"(sr[10]), "=r"(sr[11]), "=r"(sr[12]), "=r"(sr[13]), "=r"(sr[14]), "=r"(sr[15])
              : "r"(tS + 16 * c));
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
              : "=r"(dr[0]), "=r"(dr[1]), "=r"(dr[2]), "=r"(dr[3]), "=r"(dr[4]), "=r"(dr[5]), "=r"(dr[6]), "=r"(dr[7]),
                "=r"(dr[8]), "=r"(dr[9]), "=r"(dr[10]), "=r"(dr[11]), "=r"(dr[12]), "=r"(dr[13]), "=r"(dr[14]), "=r"(dr[15])
              : "r"(tDP + 16 * c));
          tmem_ld_wait();
          uint32_t pp[8], dd[8];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float4 lv = l4[4 * c + e4];
            const float4 dv = d4[4 * c + e4];
            const float lq[4] = {lv.x, lv.y, lv.z, lv.w};
            const float dq[4] = {dv.x, dv.y, dv.z, dv.w};
            float pv[4], dsv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int e = 4 * e4 + u;
              float p = ex2_approx(fmaf(__uint_as_float(sr[e]), sl2, -lq[u]));
              if (masked) p = keep_or_zero(p, 16 * c + e, q_lo, q_hi);
              pv[u] = p;
              dsv[u] = p * (__uint_as_float(dr[e]) - dq[u]);
            }
            pp[2 * e4] = pack2<T>(pv[0], pv[1]);
            pp[2 * e4 + 1] = pack2<T>(pv[2], pv[3]);
            dd[2 * e4] = pack2<T>(dsv[0], dsv[1]);
            dd[2 * e4 + 1] = pack2<T>(dsv[2], dsv[3]);
          }
          // P^T over this thread's S^T columns [8c, 8c + 8) (already read), dS^T likewise
          // over its dP^T columns.
          asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(tS + 8 * c),
                       "r"(pp[0]), "r"(pp[1]), "r"(pp[2]), "r"(pp[3]), "r"(pp[4]), "r"(pp[5]), "r"(pp[6]), "r"(pp[7])
                       : "memory");
          asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(tDP + 8 * c),
                       "r"(dd[0]), "r"(dd[1]), "r"(dd[2]), "r"(dd[3]), "r"(dd[4]), "r"(dd[5]), "r"(dd[6]), "r"(dd[7])
                       : "memory");
          // dS (queries 64h + 32hc + 16c .. +15 of this key row) into the swizzled
          // MN-major tile.
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int chunk = (4 * hc + 2 * c + u) ^ (row & 7);
            *reinterpret_cast<uint4*>(ds_row + chunk * 16) =
                make_uint4(dd[4 * u], dd[4 * u + 1], dd[4 * u + 2], dd[4 * u + 3]);
          }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.ds_ready));
      }
    }
    // Epilogue: dV rows (64 columns per thread).
    if (ok && nq > 0) ok = mbar_wait_warp(smem_u32(&sm.acc_done), 0, abort_flag);
    uint16_t* dst = static_cast<uint16_t*>(args.dv) + (static_cast<size_t>(bh) * n + key) * D + 64 * hc;
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        if (nq > 0) {
          FA_TMEM_LD32(tmem + lane_off + T_DV + 64 * hc + 32 * c, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        if (key < n) {
          uint4* o4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            o4[v4] = make_uint4(pack2<T>(__uint_as_float(r[8 * v4]), __uint_as_float(r[8 * v4 + 1])),
                                pack2<T>(__uint_as_float(r[8 * v4 + 2]), __uint_as_float(r[8 * v4 + 3])),
                                pack2<T>(__uint_as_float(r[8 * v4 + 4]), __uint_as_float(r[8 * v4 + 5])),
                                pack2<T>(__uint_as_float(r[8 * v4 + 6]), __uint_as_float(r[8 * v4 + 7])));
        }
      }
    }
  } else {
    // -------------------------------------------------- dQ read-out (thread = query row x 64 columns)
    const int hc = (warp - 8) >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float scale = args.scale;
    const int gt = threadIdx.x - 256;  // 0..255 within the dQ group
    bool ok = true;
    for (int idx = 0; idx < nq; ++idx) {
      ok = mbar_wait_warp(smem_u32(&sm.dq_full), idx & 1, abort_flag);
      tc_fence_after();
      const int q0 = (qlo + idx) * BQ;
      uint32_t r[64];
      FA_TMEM_LD32(tmem + lane_off + T_S + 64 * hc, r);
      FA_TMEM_LD32(tmem + lane_off + T_S + 64 * hc + 32, (r + 32));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.dq_free));  // TMEM read: the next S^T may overwrite it
      // Stage in the (Q, dO) slot of this query tile -- its last readers, the dV and
      // dK MMAs, completed before dQ -- as four 32-column x 128-row float boxes,
      // 128-byte swizzled, reduced into the fp32 accumulator by the TMA (rows past N
      // are skipped by the TMA).  The slot is handed back to the loader once the TMA
      // has read the staging; it refills it two query tiles later.
      const int s = idx & 1;
      if (ok) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          uint8_t* box = (hc == 0 ? sm.q[s] : sm.dout[s]) + b * (BQ * 128) + row * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const int e = 32 * b + 4 * ch;
            *reinterpret_cast<float4*>(box + ((ch ^ (row & 7)) * 16)) =
                make_float4(__uint_as_float(r[e]) * scale, __uint_as_float(r[e + 1]) * scale,
                            __uint_as_float(r[e + 2]) * scale, __uint_as_float(r[e + 3]) * scale);
          }
        }
        fence_proxy_async_smem();
      }
      ok = named_bar_all(ok, 3, GROUP);
      if (gt == 0) {
        if (ok) {
          tma_reduce_add_3d(&tm_dq, smem_u32(sm.q[s]), 0, q0, bh);
          tma_reduce_add_3d(&tm_dq, smem_u32(sm.q[s]) + BQ * 128, 32, q0, bh);
          tma_reduce_add_3d(&tm_dq, smem_u32(sm.dout[s]), 64, q0, bh);
          tma_reduce_add_3d(&tm_dq, smem_u32(sm.dout[s]) + BQ * 128, 96, q0, bh);
          bulk_commit();
          bulk_wait_read0();
        }
        mbar_arrive(smem_u32(&sm.qdo_empty[s]));
      }
      if (!ok) break;
    }
    if (gt == 0) bulk_wait0();  // every reduce-add has landed before the CTA ends
    // Epilogue: dK rows (scaled, 64 columns per thread).
    if (ok && nq > 0) ok = mbar_wait_warp(smem_u32(&sm.acc_done), 0, abort_flag);
    const int key = kt * BM + row;
    uint16_t* dst = static_cast<uint16_t*>(args.dk) + (static_cast<size_t>(bh) * n + key) * D + 64 * hc;
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        if (nq > 0) {
          FA_TMEM_LD32(tmem + lane_off + T_DK + 64 * hc + 32 * c, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        if (key < n) {
          uint4* o4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            o4[v4] = make_uint4(
                pack2<T>(__uint_as_float(r[8 * v4]) * scale, __uint_as_float(r[8 * v4 + 1]) * scale),
                pack2<T>(__uint_as_float(r[8 * v4 + 2]) * scale, __uint_as_float(r[8 * v4 + 3]) * scale),
                pack2<T>(__uint_as_float(r[8 * v4 + 4]) * scale, __uint_as_float(r[8 * v4 + 5]) * scale),
                pack2<T>(__uint_as_float(r[8 * v4 + 6]) * scale, __uint_as_float(r[8 * v4 + 7]) * scale));
        }
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

// D = rowsum(dO * O) in fp32 and a zeroed dQ accumulator; 16 lanes per row.
template <class T>
__global__ void __launch_bounds__(256) bwd_pre_kernel(BwdArgs a, long long rows) {
  const long long row = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 4;
  const int sub = threadIdx.x & 15;
  float s = 0.f;
  if (row < rows) {
    float of[8], gf[8];
    unpack8<T>(*reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.o) + row * D + sub * 8), of);
    unpack8<T>(*reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.dout) + row * D + sub * 8), gf);
#pragma unroll
    for (int i = 0; i < 8; ++i) s = fmaf(of[i], gf[i], s);
    float4* acc = reinterpret_cast<float4*>(a.ws_dq + row * D + sub * 8);
    acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (row < rows && sub == 0) a.ws_delta[row] = s;
}

// dQ accumulator (already scaled) -> T; 8 elements per thread.
template <class T>
__global__ void __launch_bounds__(256) bwd_post_kernel(BwdArgs a, long long n8) {
  const long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n8) return;
  const float4* src = reinterpret_cast<const float4*>(a.ws_dq) + 2 * i;
  const float4 x = src[0], y = src[1];
  reinterpret_cast<uint4*>(a.dq)[i] =
      make_uint4(pack2<T>(x.x, x.y), pack2<T>(x.z, x.w), pack2<T>(y.x, y.y), pack2<T>(y.z, y.w));
}

}  // namespace bwd

template <class T>
cudaError_t launch_bwd_t(const BwdArgs& a, cudaStream_t stream) {
  using namespace bwd;
  const long long bh = static_cast<long long>(a.B) * a.H;
  const long long rows = bh * a.N;
  CUtensorMap tq, tk, tv, tdo, tdq;
  if (!make_tmap_half_rows(&tq, a.q, D, a.N, bh, BQ, a.f16) || !make_tmap_half_rows(&tk, a.k, D, a.N, bh, BM, a.f16) ||
      !make_tmap_half_rows(&tv, a.v, D, a.N, bh, BM, a.f16) ||
      !make_tmap_half_rows(&tdo, a.dout, D, a.N, bh, BQ, a.f16) ||
      !make_tmap_f32_rows(&tdq, a.ws_dq, D, a.N, bh, 32, BQ))
    return cudaErrorInvalidValue;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(bwd_main_kernel<T>), kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long pre_blocks = (rows * 16 + 255) / 256;
  if (pre_blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  bwd_pre_kernel<T><<<static_cast<unsigned>(pre_blocks), 256, 0, stream>>>(a, rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long nkt = (a.N + BM - 1) / BM;
  bwd_main_kernel<T><<<static_cast<unsigned>(nkt * bh), NUM_THREADS, kSmemBytes, stream>>>(tq, tk, tv, tdo, tdq, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long n8 = rows * D / 8;
  bwd_post_kernel<T><<<static_cast<unsigned>((n8 + 255) / 256), 256, 0, stream>>>(a, n8);
  return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  return a.f16 ? launch_bwd_t<F16>(a, stream) : launch_bwd_t<Bf16>(a, stream);
}

cudaError_t take_status_bwd(unsigned int* out) { return take_local_status(out); }

}  // namespace fa
