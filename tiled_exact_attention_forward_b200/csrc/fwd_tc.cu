// Forward pass on the 5th-generation tensor cores (sm_100a), bf16 or f16 inputs
// (one kernel template; P is formed in the inputs' type): tcgen05 MMAs with
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
//   * Warp roles (608 threads): warps 0-7 and 8-15 are the softmax warps of
//     query tiles 0 and 1 (two threads per query row = TMEM lane, one per
//     64-column half, in warps i and i + 4 of the tile, exchanging row max and
//     sum through shared memory behind a 64-thread barrier per warp pair);
//     warp 16 allocates tensor memory and issues every MMA from one thread;
//     warp 17 streams K/V through the ring by TMA and warp 18 loads the Q
//     tiles, each as soon as its slot frees.
//   * Items are dealt to a persistent grid of one CTA per SM, heaviest first.
//     With a causal mask tile 0 of an item ends one key tile before tile 1;
//     S_0 of the next item's first key tile is then issued at once, so tile
//     0's softmax warps do not idle across the item boundary.  (Issuing the
//     two tiles' MMAs independently -- polled, or from two threads -- was
//     measured slower: the two softmaxes then overlap and contend for the
//     same pipes, where the fixed order below keeps them alternating.)
//   * Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each.
//     The softmax writes P (16-bit pairs) over the first 64 columns of its S
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
//   * exp2 with scale*log2(e) folded into one packed (f32x2) FMA per score
//     pair.  One pair in eight takes 2^x from a cubic on the FMA pipe instead
//     of the special-function unit, whose rate (16 results per clock per SM)
//     otherwise equals the MMA rate for d = 128; more than that loads the FMA
//     and issue slots more than it relieves the ex2 unit (measured).
#include "common.cuh"
#include "kernels.h"

namespace fa {

namespace fwdtc {

constexpr int BM = 128;                 // query rows per tile
constexpr int BN = 128;                 // keys per tile
constexpr int D = 128;                  // head dimension
constexpr int NS = 4;                   // K/V ring stages (K and V tiles interleaved)
constexpr int TILE_BYTES = BM * D * 2;  // one 128 x 128 16-bit tile = 32 KiB
constexpr int HALF_BYTES = TILE_BYTES / 2;  // one 64-column half (a 128-byte-swizzled box)
constexpr int NUM_THREADS = 608;     // 16 softmax warps + MMA warp + K/V TMA warp + Q TMA warp
constexpr int WG_THREADS = 256;      // one softmax warpgroup pair per query tile
constexpr int MMA_WARP = 16;
constexpr int TMA_WARP = 17;         // K/V stream
constexpr int QLD_WARP = 18;         // Q tiles: loaded as soon as their slot frees
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kPolyPairs = 1;  // of every 8 score pairs, those exponentiated on the FMA pipe

struct Smem {
  // 1024-byte aligned by construction (the dynamic buffer is aligned at runtime).
  uint8_t q[2][TILE_BYTES];
  uint8_t kv[NS][TILE_BYTES];
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[NS];
  uint64_t kv_empty[NS];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t o_free[2];
  uint64_t mma_done;
  // Row statistics exchanged between the two threads of a row (column halves):
  // [tile][step parity][half][row].
  float xmax[2][2][2][BM];
  float xsum[2][2][BM];
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

// Positions: query row i sits at position i + q_off of the key sequence (q_off = 0
// and Nk = N for self-attention; a context-parallel shard passes the distance
// between its query rows and the key shard).  Key j of [0, Nk) is visible to row i
// iff (!causal || j <= i + q_off) && (window == 0 || j > i + q_off - window).

// The sizes and mask of one launch, held in registers (a reference to the kernel
// parameter itself would force a copy of it to local memory).
struct Geom {
  int N, Nk, q_off, causal, window;
};

// Key-tile range [lo, hi) a query tile starting at row r0 must visit (empty when
// no row of the tile sees any key).
template <bool OFFSET>
__device__ __forceinline__ void key_tile_range(int r0, const Geom& a, int& lo, int& hi) {
  const int rlast = min(r0 + BM - 1, a.N - 1);
  const int p0 = r0 + a.q_off, p1 = rlast + a.q_off;  // positions of the first and last row
  const int nkt = (a.Nk + BN - 1) / BN;
  if (!OFFSET)  // rlast < N = Nk: the causal bound needs no clamp
    hi = a.causal ? (rlast / BN + 1) : nkt;
  else
    hi = a.causal ? (p1 < 0 ? 0 : min(nkt, p1 / BN + 1)) : nkt;
  const int first_key = a.window > 0 ? p0 - a.window + 1 : 0;
  lo = first_key > 0 ? first_key / BN : 0;
  if (lo > hi) lo = hi;
}

// Does key tile j need the per-element mask for rows r0..r0+BM-1?
__device__ __forceinline__ bool tile_needs_mask(int j, int r0, const Geom& a) {
  const int k0 = j * BN, k1 = j * BN + BN - 1;
  const int rlast = min(r0 + BM - 1, a.N - 1);
  const int p0 = r0 + a.q_off, p1 = rlast + a.q_off;
  return (k1 >= a.Nk) || (a.causal && k1 > p0) || (a.window > 0 && k0 <= p1 - a.window);
}

// 128-byte-swizzled shared-memory matrix descriptor as two 32-bit words: the
// start address field (address >> 4, 14 bits) and the leading-byte offset in
// the low word, stride offset, version and swizzle mode in the high word.  Shared
// addresses stay below 2^18, so stepping through a tile is one add on the low
// word with no carry out of the address field.
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr, uint32_t lbo) { return (saddr >> 4) | ((lbo >> 4) << 16); }
__host__ __device__ constexpr uint32_t desc_hi(uint32_t sbo) { return (sbo >> 4) | (1u << 14) | (2u << 29); }
__device__ __forceinline__ uint64_t desc_of(uint32_t lo, uint32_t hi) {
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// S = Q K^T: Q and K tiles K-major ([64-column half][128 rows][64 cols]); a K step
// of 16 columns is 32 bytes inside a half, the second half 16 KiB further on.
template <class T>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo) {
  constexpr uint32_t idesc = idesc_f32acc<T>(BM, BN, 0, 0);
  constexpr uint32_t hi = desc_hi(1024);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
    mma_ss(d_tmem, desc_of(q_lo + off, hi), desc_of(k_lo + off, hi), idesc, kk > 0 ? 1u : 0u);
  }
}

// O += P V: V tile MN-major ([64-column half][128 keys][64 cols]); a K step of 16
// keys is 16 rows = 2 KiB.  P of keys [64h, 64h + 64) sits in S columns
// [64h, 64h + 32) (16-bit pairs).
template <class T>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_lo, bool accumulate) {
  constexpr uint32_t idesc = idesc_f32acc<T>(BM, D, 0, 1);
  constexpr uint32_t hi = desc_hi(1024);
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    const uint32_t a_col = (kk >> 2) * 64 + (kk & 3) * 8;
    mma_ts(d_tmem, p_tmem + a_col, desc_of(v_lo + ((kk * 16 * 128) >> 4), hi), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
  }
}

// One unit of work: two 128-row query tiles (rows [256p, 256p + 256)) of one
// (batch, head), with the key-tile range each of them must visit.  A tile that
// exists but sees no key (possible only with a query offset) is inactive: no Q
// load, no MMA; its softmax warps write O = 0 and lse = -inf directly.
struct Item {
  int bh;
  int r0[2];
  int lo_t[2], hi_t[2];
  int lo, hi;  // union of the active tiles' ranges (empty if none is active)
  bool has1;   // tile 1 exists (rows below N)
  __device__ __forceinline__ bool active(int t) const { return lo_t[t] < hi_t[t]; }
};

// OFFSET: the launch may have a query offset or Nk != N (context-parallel shards),
// so tiles can be inactive.  Self-attention (OFFSET false) has every existing tile
// active: its diagonal key tile is always visible.
template <bool OFFSET>
__device__ __forceinline__ Item make_item(int lin, int BH, int num_pairs, const Geom& a) {
  Item it;
  // Heaviest work first: with a causal mask the last query tiles see the most keys.
  const int pair = num_pairs - 1 - lin / BH;
  it.bh = lin % BH;
  it.r0[0] = pair * 2 * BM;
  it.r0[1] = it.r0[0] + BM;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (it.r0[t] < a.N) {
      key_tile_range<OFFSET>(it.r0[t], a, it.lo_t[t], it.hi_t[t]);
    } else {
      it.lo_t[t] = it.hi_t[t] = 0;
    }
  }
  it.has1 = it.r0[1] < a.N;
  if (!OFFSET) {
    it.lo = it.has1 ? min(it.lo_t[0], it.lo_t[1]) : it.lo_t[0];
    it.hi = it.has1 ? max(it.hi_t[0], it.hi_t[1]) : it.hi_t[0];
  } else if (it.active(0) && it.active(1)) {
    it.lo = min(it.lo_t[0], it.lo_t[1]);
    it.hi = max(it.hi_t[0], it.hi_t[1]);
  } else {
    const int t = it.active(1) ? 1 : 0;
    it.lo = it.active(t) ? it.lo_t[t] : 0;
    it.hi = it.active(t) ? it.hi_t[t] : 0;
  }
  return it;
}

// Item index of round k for this CTA: items are sorted heaviest first and
// dealt in a snake order (0..G-1, then G-1..0, ...) so every CTA gets a
// similar total.  Returns -1 past the end.
__device__ __forceinline__ int item_of(int k, int total) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int lin = k * G + ((k & 1) ? (G - 1 - c) : c);
  return lin < total ? lin : -1;
}

// T: the 16-bit type of Q, K, V, P and O (Bf16 or F16).  OFFSET: see make_item.
template <class T, bool OFFSET>
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
  const int total = num_pairs * BH;
  const Geom geo{args.N, OFFSET ? args.Nk : args.N, OFFSET ? args.q_off : 0, args.causal, args.window};
  // Is tile t of an item to be computed?  (Without an offset: whenever it exists.)
  auto active = [](const Item& it, int t) { return OFFSET ? it.active(t) : (t == 0 || it.has1); };

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&sm.q_full[t]), 1);
      mbar_init(smem_u32(&sm.q_empty[t]), 1);
      mbar_init(smem_u32(&sm.s_full[t]), 1);
      mbar_init(smem_u32(&sm.p_full[t]), WG_THREADS);
      mbar_init(smem_u32(&sm.o_full[t]), 1);
      mbar_init(smem_u32(&sm.o_free[t]), WG_THREADS);
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

  if (warp == QLD_WARP) {
    // ------------------------------------------------------------ Q loader
    // A warp of its own, so the next item's Q tile goes out as soon as the last
    // S MMA of the current item has read the slot, ahead of the K/V stream.
    if (lane == 0) {
      int nq[2] = {0, 0};  // Q tiles loaded so far, per slot
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int lin = item_of(k, total);
        if (lin < 0) break;
        const Item it = make_item<OFFSET>(lin, BH, num_pairs, geo);
        for (int t = 0; t < 2 && ok; ++t) {
          if (!active(it, t)) continue;
          if (nq[t] > 0) ok = mbar_wait(smem_u32(&sm.q_empty[t]), (nq[t] - 1) & 1, abort_flag);
          if (!ok) break;
          const uint32_t bar = smem_u32(&sm.q_full[t]);
          mbar_arrive_expect_tx(bar, TILE_BYTES);
          tma_load_3d(smem_u32(sm.q[t]), &tm_q, bar, 0, it.r0[t], it.bh);
          tma_load_3d(smem_u32(sm.q[t]) + HALF_BYTES, &tm_q, bar, 64, it.r0[t], it.bh);
          ++nq[t];
        }
      }
      for (int t = 0; t < 2; ++t)
        if (nq[t] > 0) mbar_wait_drain(smem_u32(&sm.q_full[t]), (nq[t] - 1) & 1);
    }
  } else if (warp == TMA_WARP) {
    // ------------------------------------------------------------ K/V producer
    if (lane == 0) {
      int kvi = 0;         // K/V ring fills so far (K and V interleaved)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int lin = item_of(k, total);
        if (lin < 0) break;
        const Item it = make_item<OFFSET>(lin, BH, num_pairs, geo);
        for (int idx = 0; ok && idx < 2 * (it.hi - it.lo); ++idx, ++kvi) {
          const int s = kvi % NS;
          if (kvi >= NS) ok = mbar_wait(smem_u32(&sm.kv_empty[s]), ((kvi / NS) - 1) & 1, abort_flag);
          if (!ok) break;
          const int j = it.lo + (idx >> 1);
          const CUtensorMap* tm = (idx & 1) ? &tm_v : &tm_k;
          const uint32_t bar = smem_u32(&sm.kv_full[s]);
          mbar_arrive_expect_tx(bar, TILE_BYTES);
          tma_load_3d(smem_u32(sm.kv[s]), tm, bar, 0, j * BN, it.bh);
          tma_load_3d(smem_u32(sm.kv[s]) + HALF_BYTES, tm, bar, 64, j * BN, it.bh);
        }
      }
      // Drain: every copy issued must land before the CTA may exit.
      for (int i = max(0, kvi - NS); i < kvi; ++i) mbar_wait_drain(smem_u32(&sm.kv_full[i % NS]), (i / NS) & 1);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS[2] = {tmem + 0, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 384};
      // Descriptor low words of the Q slots (K-major, leading-byte offset 16).
      const uint32_t q_s[2] = {desc_lo(smem_u32(sm.q[0]), 16), desc_lo(smem_u32(sm.q[1]), 16)};
      int nq[2] = {0, 0};    // Q tiles consumed, per slot
      bool q_ready[2] = {false, false};  // slot t holds the tile now in use and was waited for
      int npv[2] = {0, 0};   // PV MMAs issued, per tile slot (p_full phase)
      int nout[2] = {0, 0};  // items finished, per tile slot (o_full / o_free phase)
      int kvi = 0;
      bool ok = true;
      bool s0_ahead = false;  // S_0(lo) of this item was issued during the previous item
      auto stage_of = [&](int i) { return i % NS; };
      auto parity_of = [&](int i) { return static_cast<uint32_t>((i / NS) & 1); };
      // S_t(j) of item `it`: waits for the item's Q tile on first use; the item's last
      // S_t releases the Q slot to the loader.
      auto issue_s = [&](const Item& it, int t, int j, uint32_t ks) -> bool {
        if (!q_ready[t]) {
          if (!mbar_wait(smem_u32(&sm.q_full[t]), nq[t] & 1, abort_flag)) return false;
          ++nq[t];
          q_ready[t] = true;
          tc_fence_after();
        }
        issue_qk<T>(tS[t], q_s[t], ks);
        tc_commit(smem_u32(&sm.s_full[t]));
        if (j == it.hi_t[t] - 1) {
          tc_commit(smem_u32(&sm.q_empty[t]));
          q_ready[t] = false;
        }
        return true;
      };
      for (int k = 0; ok; ++k) {
        const int lin = item_of(k, total);
        if (lin < 0) break;
        const Item it = make_item<OFFSET>(lin, BH, num_pairs, geo);
        auto act = [&](int t, int j) { return j >= it.lo_t[t] && j < it.hi_t[t]; };
        // PV_t(j): the first one of an item overwrites O_t, so the previous item's
        // epilogue must have read it out; the last one publishes O_t.
        auto issue_o = [&](int t, int j, uint32_t vs) -> bool {
          if (j == it.lo_t[t] && nout[t] > 0) {
            if (!mbar_wait(smem_u32(&sm.o_free[t]), (nout[t] - 1) & 1, abort_flag)) return false;
          }
          if (!mbar_wait(smem_u32(&sm.p_full[t]), npv[t] & 1, abort_flag)) return false;
          tc_fence_after();
          issue_pv<T>(tO[t], tS[t], vs, j > it.lo_t[t]);
          ++npv[t];
          if (j == it.hi_t[t] - 1) {
            tc_commit(smem_u32(&sm.o_full[t]));
            ++nout[t];
          }
          return true;
        };
        if (it.hi <= it.lo) {  // no active tile: nothing to issue
          if (OFFSET) continue;
          break;
        }
        // Prologue: S_t(lo) for both tiles (S_0(lo) may already be in flight).
        ok = mbar_wait(smem_u32(&sm.kv_full[stage_of(kvi)]), parity_of(kvi), abort_flag);
        if (!ok) break;
        tc_fence_after();
        {
          const uint32_t ks = desc_lo(smem_u32(sm.kv[stage_of(kvi)]), 16);
          for (int t = 0; t < 2 && ok; ++t)
            if (act(t, it.lo) && !(t == 0 && s0_ahead)) ok = issue_s(it, t, it.lo, ks);
          if (!ok) break;
          tc_commit(smem_u32(&sm.kv_empty[stage_of(kvi)]));
          ++kvi;
          s0_ahead = false;
        }
        for (int j = it.lo; ok && j < it.hi; ++j) {
          const int vidx = kvi;            // V_j
          const int nidx = kvi + 1;        // K_{j+1}
          const bool has_next = j + 1 < it.hi;
          ok = mbar_wait(smem_u32(&sm.kv_full[stage_of(vidx)]), parity_of(vidx), abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vs = desc_lo(smem_u32(sm.kv[stage_of(vidx)]), HALF_BYTES);
          if (act(0, j) && !(ok = issue_o(0, j, vs))) break;
          uint32_t ks = 0;
          if (has_next) {
            ok = mbar_wait(smem_u32(&sm.kv_full[stage_of(nidx)]), parity_of(nidx), abort_flag);
            if (!ok) break;
            tc_fence_after();
            ks = desc_lo(smem_u32(sm.kv[stage_of(nidx)]), 16);
            if (act(0, j + 1) && !(ok = issue_s(it, 0, j + 1, ks))) break;
          }
          if (act(1, j) && !(ok = issue_o(1, j, vs))) break;
          tc_commit(smem_u32(&sm.kv_empty[stage_of(vidx)]));
          if (has_next) {
            if (act(1, j + 1) && !(ok = issue_s(it, 1, j + 1, ks))) break;
            tc_commit(smem_u32(&sm.kv_empty[stage_of(nidx)]));
          }
          kvi += has_next ? 2 : 1;
          // Causal masks end tile 0 one key tile before tile 1.  Its softmax warps
          // would then idle until tile 1 finishes, so S_0 of the next item's first
          // key tile goes out now: K(lo') is the ring entry after V(hi - 1), and
          // ring entry kvi + 1 - NS has been consumed already.
          if (j == it.hi - 2 && it.has1 && !act(0, j + 1)) {
            const int lin2 = item_of(k + 1, total);
            if (lin2 >= 0) {
              const Item nx = make_item<OFFSET>(lin2, BH, num_pairs, geo);
              if (active(nx, 0) && nx.lo_t[0] == nx.lo) {
                ok = mbar_wait(smem_u32(&sm.kv_full[stage_of(kvi + 1)]), parity_of(kvi + 1), abort_flag);
                if (!ok) break;
                tc_fence_after();
                if (!(ok = issue_s(nx, 0, nx.lo, desc_lo(smem_u32(sm.kv[stage_of(kvi + 1)]), 16)))) break;
                s0_ahead = true;
              }
            }
          }
        }
      }
      // All MMAs issued by this thread must complete before TMEM is freed.
      tc_commit(smem_u32(&sm.mma_done));
      mbar_wait_drain(smem_u32(&sm.mma_done), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    // 8 warps per query tile: warp i of the tile reads TMEM lanes 32*(i%4).. (one row
    // per thread) and columns [64h, 64h + 64) with h = i/4, so two threads share a
    // row and exchange its max and sum through shared memory.
    const int t = warp >> 3;         // query tile slot
    const int wi = warp & 7;
    const int hc = wi >> 2;          // column half
    const int row = (wi & 3) * 32 + lane;
    // The two threads of a row sit in warps wi and wi + 4 (same TMEM lanes); only
    // that warp pair exchanges, on a 64-thread named barrier of its own.
    const int bar_id = 3 + 4 * t + (wi & 3);
    constexpr int kBarThreads = 64;
    const uint32_t lane_off = static_cast<uint32_t>((wi & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128 + 64 * hc;
    const uint32_t tO = tmem + lane_off + 256 + t * 128 + 64 * hc;
    const float sl2 = args.scale_log2;
    int ns = 0;    // S tiles consumed (s_full phase)
    int nout = 0;  // items finished (o_full phase)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int lin = item_of(k, total);
      if (lin < 0) break;
      const Item item = make_item<OFFSET>(lin, BH, num_pairs, geo);
      if (t == 1 && !item.has1) continue;
      const int r0 = item.r0[t];
      const int row_g = r0 + row;
      if (OFFSET && !item.active(t)) {
        // No row of this tile sees a key: O = 0, lse = -inf.
        if (row_g < n) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(args.o) +
                                                (static_cast<size_t>(item.bh) * n + row_g) * D + 64 * hc);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
          if (hc == 0 && args.lse != nullptr) args.lse[static_cast<size_t>(item.bh) * n + row_g] = -INFINITY;
        }
        continue;
      }
      const int row_p = row_g + geo.q_off;  // the row's position in the key sequence
      float m = -INFINITY, l = 0.f;  // l: this thread's half of the row sum
      bool nan_row = false;
      for (int j = item.lo_t[t]; j < item.hi_t[t]; ++j, ++ns) {
        ok = mbar_wait_warp(smem_u32(&sm.s_full[t]), ns & 1, abort_flag);
        tc_fence_after();
        uint32_t s[64];
        FA_TMEM_LD32(tS + 0, (s + 0));
        FA_TMEM_LD32(tS + 32, (s + 32));
        tmem_ld_wait();
        const bool masked = tile_needs_mask(j, r0, geo);
        if (masked) {
          // Visible keys of this row form one interval; columns of this half are 64h + c.
          const int base = j * BN + 64 * hc;
          int c_hi = min(64, geo.Nk - base);
          if (args.causal) c_hi = min(c_hi, row_p - base + 1);
          const int c_lo = args.window > 0 ? max(0, row_p - args.window + 1 - base) : 0;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < c_lo || c >= c_hi) s[c] = __float_as_uint(-INFINITY);
        }
        // Half-row max: eight chains of 3-input max; NaN-propagating so a NaN score
        // marks the row (its output is NaN at the end).
        float mm[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          mm[q] = fmax3_nan(__uint_as_float(s[q]), __uint_as_float(s[q + 8]), -INFINITY);
#pragma unroll
        for (int c = 16; c < 64; c += 16)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            mm[q] = fmax3_nan(mm[q], __uint_as_float(s[c + q]), __uint_as_float(s[c + 8 + q]));
        const float hm = fmax3_nan(fmax3_nan(mm[0], mm[1], mm[2]), fmax3_nan(mm[3], mm[4], mm[5]),
                                   fmax3_nan(mm[6], mm[7], -INFINITY));
        sm.xmax[t][ns & 1][hc][row] = hm;
        // Barrier of the tile's 256 threads: both halves' maxima are visible, and the
        // whole group agrees on whether to go on.
        ok = named_bar_all(ok, bar_id, kBarThreads);
        if (!ok) break;
        const float mx = fmax3_nan(hm, sm.xmax[t][ns & 1][hc ^ 1][row], -INFINITY);
        nan_row |= (mx != mx);
        const float m_new = fmaxf(m, mx);  // ignores a NaN mx
        // (m_new - m) is +inf on the first visible tile and NaN while the row is
        // still empty; only the former moves the reference max.  Both halves of a
        // row take the same decision from the same numbers.
        const bool need = (m_new - m) * sl2 > kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx((m - m_new) * sl2);
          m = m_new;
          l *= alpha;
        }
        const float ms = (m == -INFINITY) ? 0.f : m * sl2;
        // P = 2^(s * scale * log2(e) - m * scale * log2(e)) -> 16-bit pairs over this
        // half's first 32 S columns (already read).  Scores go in pairs through the
        // packed f32x2 FMA; kPolyPairs of every 8 pairs take 2^x from the cubic on
        // the FMA pipe, the rest from the special-function unit, so both pipes share
        // the exponentials.
        const uint64_t sl2x2 = f2_pack(sl2, sl2), nms2 = f2_pack(-ms, -ms);
        uint64_t acc_a = f2_pack(0.f, 0.f), acc_b = f2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t p[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[32 * c + e]), __uint_as_float(s[32 * c + e + 1])),
                                       sl2x2, nms2);
            uint64_t p2;
            if (((e >> 1) & 7) >= 8 - kPolyPairs) {
              p2 = exp2_poly_pair(x2);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
            }
            if (e & 2) acc_b = f2_add(acc_b, p2); else acc_a = f2_add(acc_a, p2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            p[e >> 1] = pack2<T>(p0, p1);
          }
          asm volatile(
              "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
                  tS + 16 * c),
              "r"(p[0]), "r"(p[1]), "r"(p[2]), "r"(p[3]), "r"(p[4]), "r"(p[5]), "r"(p[6]), "r"(p[7]),
              "r"(p[8]), "r"(p[9]), "r"(p[10]), "r"(p[11]), "r"(p[12]), "r"(p[13]), "r"(p[14]), "r"(p[15])
              : "memory");
        }
        if (j > item.lo_t[t] && __any_sync(0xffffffffu, need)) {
          // O_t's last update (PV_t(j-1)) is complete: S_t(j) was issued after it.
#pragma unroll
          for (int c = 0; c < 2; ++c) {
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
        {
          float a0, a1, b0, b1;
          f2_unpack(acc_a, a0, a1);
          f2_unpack(acc_b, b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
      }
      if (!ok) break;
      // Epilogue: O / l in 16 bits and lse = m * scale + ln l.  O_t is read out first and
      // released (o_free) so the next item's PV can start while the stores drain.
      ok = mbar_wait_warp(smem_u32(&sm.o_full[t]), nout & 1, abort_flag);
      ++nout;
      tc_fence_after();
      uint32_t o[64];
      FA_TMEM_LD32(tO + 0, (o + 0));
      FA_TMEM_LD32(tO + 32, (o + 32));
      tmem_ld_wait();
      tc_fence_before();
      sm.xsum[t][hc][row] = l;
      ok = named_bar_all(ok, bar_id, kBarThreads);
      mbar_arrive(smem_u32(&sm.o_free[t]));
      if (!ok) break;
      float lt = l + sm.xsum[t][hc ^ 1][row];
      // The sums may be read again only after the next item's first exchange barrier.
      // A row whose max is still -inf saw no key: its sum is only the cubic's floor
      // for masked scores (< 1e-38 each), not probability mass.
      if (OFFSET && m == -INFINITY) lt = 0.f;
      if (nan_row) lt = __uint_as_float(0x7fc00000u);  // NaN input: NaN output row
      const float inv = lt > 0.f ? 1.f / lt : (lt == 0.f ? 0.f : lt);
      if (row_g < n) {
        uint16_t* orow = reinterpret_cast<uint16_t*>(args.o) +
                              (static_cast<size_t>(item.bh) * n + row_g) * D + 64 * hc;
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4) {
          uint4 w;
          w.x = pack2<T>(__uint_as_float(o[8 * v4 + 0]) * inv, __uint_as_float(o[8 * v4 + 1]) * inv);
          w.y = pack2<T>(__uint_as_float(o[8 * v4 + 2]) * inv, __uint_as_float(o[8 * v4 + 3]) * inv);
          w.z = pack2<T>(__uint_as_float(o[8 * v4 + 4]) * inv, __uint_as_float(o[8 * v4 + 5]) * inv);
          w.w = pack2<T>(__uint_as_float(o[8 * v4 + 6]) * inv, __uint_as_float(o[8 * v4 + 7]) * inv);
          dst[v4] = w;
        }
        if (hc == 0 && args.lse != nullptr)
          args.lse[static_cast<size_t>(item.bh) * n + row_g] =
              lt > 0.f ? m * args.scale + logf(lt) : (lt == 0.f ? -INFINITY : lt);
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
  const long long heads = static_cast<long long>(a.B) * a.H;
  if (!make_tmap_half_rows(&tq, a.q, D, a.N, heads, BM, a.f16) ||
      !make_tmap_half_rows(&tk, a.k, D, a.Nk, heads, BN, a.f16) ||
      !make_tmap_half_rows(&tv, a.v, D, a.Nk, heads, BN, a.f16))
    return cudaErrorInvalidValue;
  const bool offset = a.q_off != 0 || a.Nk != a.N;
  auto kernel = offset ? (a.f16 ? fwd_tc_kernel<F16, true> : fwd_tc_kernel<Bf16, true>)
                       : (a.f16 ? fwd_tc_kernel<F16, false> : fwd_tc_kernel<Bf16, false>);
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long items = static_cast<long long>((a.N + 2 * BM - 1) / (2 * BM)) * heads;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  int sms = 0;
  e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  kernel<<<grid, NUM_THREADS, kSmemBytes, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

cudaError_t take_status_fwd_tc(unsigned int* out) { return take_local_status(out); }

}  // namespace fa
