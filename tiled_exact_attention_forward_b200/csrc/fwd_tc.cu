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
//   * Warp roles (512 threads, four warpgroups):
//       warpgroups 0 and 1 -- the softmax of query tiles 0 and 1: one thread
//         per query row (= TMEM lane), all 128 score columns in registers, so
//         the row max and sum need no exchange between threads;
//       warpgroup 2 -- the epilogue: reads O out of TMEM, divides by the row
//         sum, stages O (16-bit) in shared memory and writes it with TMA stores,
//         and stores lse, so the softmax warps go straight on to the next item's
//         first tile;
//       warpgroup 3 -- warp 12 allocates tensor memory and issues every MMA,
//         warp 13 streams K/V through the ring by TMA, warp 14 loads the Q
//         tiles (each as soon as its slot frees) and prefetches the next item's
//         Q tiles into L2.
//     The MMA warp runs its whole loop warp-uniformly and issues each 8-MMA
//     block (one asm statement) and each commit from one elected lane; a warp
//     that branches with one active lane issues slower (measured), so the
//     issuer keeps its control flow uniform and its waits and commits few:
//     per key tile one wait per K/V ring entry (TMA data: no tcgen05 fence),
//     one P wait per tile, one commit per S and per ring entry.
//     Registers are split with setmaxnreg: 192 per softmax thread, 64 per
//     epilogue thread and 64 for warpgroup 3 (256*192 + 128*64 + 128*64 =
//     65536, the block's launch budget of 512 threads x 128).  The host
//     refuses to launch unless the compiled kernel has exactly that budget.
//   * Items are dealt to a persistent grid of one CTA per SM, heaviest first
//     (with a causal window: the full-window items first, head by head, so the
//     CTAs in flight share a few heads' K/V in L2).
//     With a causal mask tile 0 of an item ends one key tile before tile 1;
//     S_0 of the next item's first key tile is then issued at once, so tile
//     0's softmax warps do not idle across the item boundary.
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
//     pair, 2^x from the special-function unit (a cubic on the FMA pipe can
//     take a share of the pairs: FA_FWD_POLY_PAIRS, off by default -- see
//     kPolyPairs).
#include "common.cuh"
#include "kernels.h"

namespace fa {

namespace fwdtc {

// The same value in all 32 columns (one register for every operand).
#define FA_TMEM_ST32_SAME(taddr, v)                                                                 \
  asm volatile(                                                                                     \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1," \
      "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr), "r"(v)                          \
      : "memory")

constexpr int BM = 128;                 // query rows per tile
constexpr int BN = 128;                 // keys per tile
constexpr int D = 128;                  // head dimension
constexpr int NS = 4;                   // K/V ring stages (K and V tiles interleaved)
constexpr int TILE_BYTES = BM * D * 2;  // one 128 x 128 16-bit tile = 32 KiB
constexpr int HALF_BYTES = TILE_BYTES / 2;  // one 64-column half (a 128-byte-swizzled box)
constexpr int NUM_THREADS = 512;     // 4 warpgroups: softmax 0, softmax 1, epilogue, MMA/TMA
constexpr int WG_THREADS = 128;      // one warpgroup: one thread per row of a query tile
constexpr int EPI_WG = 2;            // epilogue warpgroup (warps 8-11)
constexpr int MMA_WARP = 12;
constexpr int TMA_WARP = 13;         // K/V stream
constexpr int QLD_WARP = 14;         // Q tiles: loaded as soon as their slot frees
constexpr int kEpiBar = 1;           // named barrier of the epilogue warpgroup
constexpr int kSoftmaxRegs = 192;    // 128 scores + exp2 pipeline, no spills
constexpr int kEpilogueRegs = 64;
constexpr int kOtherRegs = 64;
constexpr int kLaunchRegs = 128;     // 65536 / NUM_THREADS: what the split draws on
static_assert(2 * WG_THREADS * kSoftmaxRegs + WG_THREADS * kEpilogueRegs + WG_THREADS * kOtherRegs <=
                  NUM_THREADS * kLaunchRegs,
              "register split exceeds the launch budget");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Of every 8 score pairs, those exponentiated by the cubic on the FMA pipe instead
// of the special-function unit.  With one softmax thread per row the warp is
// bound by instruction issue, not by the ex2 unit, and the cubic only adds
// instructions: measured on B200 (causal prefill / sliding window TFLOP/s),
// 0 -> 727-732 / 1085, 1 -> 715 / 1071, 2 -> 707 / 1056.  Kept as a build option.
#ifndef FA_FWD_POLY_PAIRS
#define FA_FWD_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = FA_FWD_POLY_PAIRS;

struct Smem {
  // 1024-byte aligned by construction (the dynamic buffer is aligned at runtime).
  uint8_t q[2][TILE_BYTES];
  uint8_t kv[NS][TILE_BYTES];
  uint8_t ostage[HALF_BYTES];  // epilogue: 64 output columns of a tile, 128-byte swizzled
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t kv_full[NS];
  uint64_t kv_empty[NS];
  uint64_t s_full[2];
  uint64_t p_full[2];   // P stored in TMEM (and O rescaled if it had to be)
  uint64_t o_full[2];   // last PV of an item complete
  uint64_t o_free[2];   // epilogue has read O out of TMEM
  uint64_t st_full[2];  // softmax has published the item's row statistics
  uint64_t st_empty[2]; // epilogue has read them
  uint64_t mma_done;
  // Row statistics of a finished item, softmax -> epilogue: [tile][row].
  float stat_m[2][BM];
  float stat_l[2][BM];
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

// tcgen05.commit from one elected lane of a warp that executes it uniformly.
__device__ __forceinline__ void commit_elect(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

// S = Q K^T: Q and K tiles K-major ([64-column half][128 rows][64 cols]); a K step
// of 16 columns is 32 bytes inside a half, the second half 16 KiB further on.
template <class T>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {
  constexpr uint32_t h = HALF_BYTES >> 4, idesc = idesc_f32acc<T>(BM, BN, 0, 0);
  static_assert(D / 16 == 8, "one 8-MMA block per S tile");
  mma8_ss<idesc, 2, 4, 6, h, h + 2, h + 4, h + 6>(d_tmem, desc_lo(q_addr, 16), desc_lo(k_addr, 16), desc_hi(1024), 0u);
}

// O += P V: V tile MN-major ([64-column half][128 keys][64 cols]); a K step of
// 16 keys is 16 rows = 2 KiB.  P of keys [2c, 2c + 1] sits in S column c (16-bit
// pairs), so the A operand of K step kk starts at column 8 kk.  The first step
// accumulates only when `accumulate` is set (the first PV of an item overwrites O).
template <class T>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_addr, uint32_t accumulate) {
  static_assert(BN / 16 == 8, "one 8-MMA block per PV");
  constexpr uint32_t idesc = idesc_f32acc<T>(BM, D, 0, 1), col_step = 8, v_step = (16 * 128) >> 4;
  mma8_ts<idesc, col_step, v_step>(d_tmem, p_tmem, desc_lo(v_addr, HALF_BYTES), desc_hi(1024), accumulate);
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
  // With a causal sliding window every pair from `pf` on sees a full window (equal
  // weight): those come first and head by head, so the CTAs in flight share the
  // K/V of a few heads in L2 instead of the windows of every head; the lighter
  // pairs at the start of each sequence follow, heaviest first.  Without a window
  // pf = num_pairs and the order is pair-major over all heads.
  const int pf = (!OFFSET && a.causal && a.window > 0) ? min(num_pairs, (a.window - 1 + 2 * BM - 1) / (2 * BM))
                                                       : num_pairs;
  const int nfull = num_pairs - pf;
  int pair;
  if (lin < BH * nfull) {
    it.bh = lin / nfull;
    pair = num_pairs - 1 - lin % nfull;
  } else {
    const int rest = lin - BH * nfull;
    pair = pf - 1 - rest / BH;
    it.bh = rest % BH;
  }
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
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  FwdArgs args) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;
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
      mbar_init(smem_u32(&sm.st_full[t]), WG_THREADS);
      mbar_init(smem_u32(&sm.st_empty[t]), WG_THREADS);
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
    tma_prefetch_desc(&tm_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (wg == 3) {
    regs_dec<kOtherRegs>();
    if (warp == QLD_WARP) {
      // ---------------------------------------------------------- Q loader
      // A warp of its own, so the next item's Q tile goes out as soon as the last
      // S MMA of the current item has read the slot, ahead of the K/V stream.  The
      // item after that has its Q tiles prefetched into L2 meanwhile (issued after
      // the current item's loads: at launch that keeps a third item's Q tiles out of
      // the first DRAM burst, measured 1.5-2 % faster on the 2K causal prefill).
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
          const int lin2 = item_of(k + 1, total);
          if (ok && lin2 >= 0) {
            const Item nx = make_item<OFFSET>(lin2, BH, num_pairs, geo);
            for (int t = 0; t < 2; ++t) {
              if (!active(nx, t)) continue;
              tma_prefetch_l2_3d(&tm_q, 0, nx.r0[t], nx.bh);
              tma_prefetch_l2_3d(&tm_q, 64, nx.r0[t], nx.bh);
            }
          }
        }
        for (int t = 0; t < 2; ++t)
          if (nq[t] > 0) mbar_wait_drain(smem_u32(&sm.q_full[t]), (nq[t] - 1) & 1);
      }
    } else if (warp == TMA_WARP) {
      // ---------------------------------------------------------- K/V producer
      if (lane == 0) {
        int kvi = 0;  // K/V ring fills so far (K and V interleaved)
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
      // ---------------------------------------------------------- MMA issuer
      // The whole warp runs this loop (warp-uniform waits); MMAs and commits are
      // issued by one elected lane.
      {
        // Phase bits of the per-tile barriers, bit t for tile slot t:
        //   Q_PH  q_full phase to wait for next      QRDY  slot t holds the tile in use
        //   PV_PH p_full phase                       O_USED an item has used O_t before
        //   O_PH  o_free phase of the last item that finished on tile t
        enum : uint32_t { Q_PH = 0, QRDY = 2, PV_PH = 4, O_USED = 6, O_PH = 8 };
        uint32_t ph = 0;
        int kvi = 0;
        bool ok = true;
        bool s0_ahead = false;  // S_0(lo) of this item was issued during the previous item
        auto bit = [&](uint32_t b) { return (ph >> b) & 1u; };
        auto stage_addr = [&](int i) { return smem_u32(sm.kv[i % NS]); };
        // K/V tiles arrive by TMA: the barrier's completion orders the copy before
        // the MMAs' reads (no tcgen05 fence needed, unlike data another thread's
        // tcgen05 instructions produced).
        auto wait_kv = [&](int i) {
          return mbar_wait_warp(smem_u32(&sm.kv_full[i % NS]), static_cast<uint32_t>((i / NS) & 1), abort_flag);
        };
        // S_t(j): waits for the item's Q tile on first use; the item's last S_t
        // (last == true) releases the Q slot to the loader.
        auto issue_s = [&](int t, bool last, uint32_t k_addr) -> bool {
          if (!bit(QRDY + t)) {
            if (!mbar_wait_warp(smem_u32(&sm.q_full[t]), bit(Q_PH + t), abort_flag)) return false;
            ph ^= 1u << (Q_PH + t);
            ph |= 1u << (QRDY + t);
          }
          issue_qk<T>(tmem + 128 * t, smem_u32(sm.q[t]), k_addr);
          commit_elect(smem_u32(&sm.s_full[t]));
          if (last) {
            commit_elect(smem_u32(&sm.q_empty[t]));
            ph &= ~(1u << (QRDY + t));
          }
          return true;
        };
        // PV_t(j) once P_t(j) is in TMEM.  The first PV of an item (first == true)
        // overwrites O_t, so the epilogue must have read the previous item's O_t
        // out; the last one (last == true) publishes O_t.
        auto issue_o = [&](int t, bool first, bool last, uint32_t v_addr) -> bool {
          if (first && bit(O_USED + t)) {
            if (!mbar_wait_warp(smem_u32(&sm.o_free[t]), bit(O_PH + t), abort_flag)) return false;
            ph ^= 1u << (O_PH + t);
          }
          if (!mbar_wait_warp(smem_u32(&sm.p_full[t]), bit(PV_PH + t), abort_flag)) return false;
          tc_fence_after();
          issue_pv<T>(tmem + 256 + 128 * t, tmem + 128 * t, v_addr, first ? 0u : 1u);
          ph ^= 1u << (PV_PH + t);
          if (last) {
            commit_elect(smem_u32(&sm.o_full[t]));
            ph |= 1u << (O_USED + t);
          }
          return true;
        };
        for (int k = 0; ok; ++k) {
          const int lin = item_of(k, total);
          if (lin < 0) break;
          const Item it = make_item<OFFSET>(lin, BH, num_pairs, geo);
          auto act = [&](int t, int j) { return j >= it.lo_t[t] && j < it.hi_t[t]; };
          if (it.hi <= it.lo) {  // no active tile: nothing to issue
            if (OFFSET) continue;
            break;
          }
          // Prologue: S_t(lo) for both tiles (S_0(lo) may already be in flight).
          if (!(ok = wait_kv(kvi))) break;
          if (act(0, it.lo) && !s0_ahead && !(ok = issue_s(0, it.lo == it.hi_t[0] - 1, stage_addr(kvi)))) break;
          if (act(1, it.lo) && !(ok = issue_s(1, it.lo == it.hi_t[1] - 1, stage_addr(kvi)))) break;
          commit_elect(smem_u32(&sm.kv_empty[kvi % NS]));
          ++kvi;
          s0_ahead = false;
          for (int j = it.lo; ok && j < it.hi; ++j) {
            const int vidx = kvi;      // V_j
            const int nidx = kvi + 1;  // K_{j+1}
            const bool has_next = j + 1 < it.hi;
            if (!(ok = wait_kv(vidx))) break;
            // K_{j+1} is waited for before PV_0(j), so S_0(j+1) follows PV_0(j) into the
            // tensor pipe with nothing between them (measured 1.7 % faster).
            if (has_next && !(ok = wait_kv(nidx))) break;
            if (act(0, j) && !(ok = issue_o(0, j == it.lo_t[0], j == it.hi_t[0] - 1, stage_addr(vidx)))) break;
            if (has_next && act(0, j + 1) && !(ok = issue_s(0, j + 1 == it.hi_t[0] - 1, stage_addr(nidx)))) break;
            if (act(1, j) && !(ok = issue_o(1, j == it.lo_t[1], j == it.hi_t[1] - 1, stage_addr(vidx)))) break;
            commit_elect(smem_u32(&sm.kv_empty[vidx % NS]));
            if (has_next) {
              if (act(1, j + 1) && !(ok = issue_s(1, j + 1 == it.hi_t[1] - 1, stage_addr(nidx)))) break;
              commit_elect(smem_u32(&sm.kv_empty[nidx % NS]));
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
                  const bool last = nx.lo == nx.hi_t[0] - 1;
                  if (!(ok = wait_kv(kvi + 1))) break;
                  if (!(ok = issue_s(0, last, stage_addr(kvi + 1)))) break;
                  s0_ahead = true;
                }
              }
            }
          }
        }
        // All MMAs issued by this warp must complete before TMEM is freed.
        commit_elect(smem_u32(&sm.mma_done));
        mbar_wait_drain(smem_u32(&sm.mma_done), 0);
      }
      __syncwarp();
    }
  } else if (wg == EPI_WG) {
    // ------------------------------------------------------------ epilogue
    // Thread = one row of each query tile (TMEM lane 32 (warp % 4) + lane): waits
    // for the item's last PV and the softmax's row statistics, reads O_t out of
    // TMEM in 32-column chunks, frees O_t for the next item, and stores O / l in
    // 16 bits and lse = m * scale + ln l.
    regs_dec<kEpilogueRegs>();
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t stage = smem_u32(sm.ostage);
    const bool leader = threadIdx.x == EPI_WG * WG_THREADS;  // issues the TMA stores
    bool pending = false;  // leader: a TMA store may still be reading the staging buffer
    int nfull[2] = {0, 0};
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int lin = item_of(k, total);
      if (lin < 0) break;
      const Item item = make_item<OFFSET>(lin, BH, num_pairs, geo);
      for (int t = 0; t < 2 && ok; ++t) {
        if (t == 1 && !item.has1) continue;
        const int row_g = item.r0[t] + row;
        uint16_t* orow = reinterpret_cast<uint16_t*>(args.o) + (static_cast<size_t>(item.bh) * n + row_g) * D;
        if (OFFSET && !item.active(t)) {
          // No row of this tile sees a key: O = 0, lse = -inf.
          if (row_g < n) {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
            if (args.lse != nullptr) args.lse[static_cast<size_t>(item.bh) * n + row_g] = -INFINITY;
          }
          continue;
        }
        ok = mbar_wait_warp(smem_u32(&sm.o_full[t]), nfull[t] & 1, abort_flag);
        if (ok) ok = mbar_wait_warp(smem_u32(&sm.st_full[t]), nfull[t] & 1, abort_flag);
        // The four epilogue warps meet at named barriers below: decide together.
        ok = named_bar_all(ok, kEpiBar, WG_THREADS);
        if (!ok) break;
        ++nfull[t];
        tc_fence_after();
        const float m = sm.stat_m[t][row];
        float lt = sm.stat_l[t][row];
        mbar_arrive(smem_u32(&sm.st_empty[t]));
        // A row whose max is still -inf saw no key: its sum is only the cubic's floor
        // for masked scores (< 1e-38 each), not probability mass.  A NaN sum marks a
        // NaN input: the row comes out NaN.
        if (OFFSET && m == -INFINITY && lt == lt) lt = 0.f;
        const float inv = lt > 0.f ? 1.f / lt : (lt == 0.f ? 0.f : lt);
        const uint32_t tO = tmem + lane_off + 256 + t * 128;
        // O / l goes out through shared memory and one TMA store per 64-column half:
        // a thread storing its own 256-byte row to global memory touches 32 cache
        // lines per warp instruction, and that traffic was measured to stall the
        // softmax warps' TMEM and ex2 work at every item boundary.  The TMA store
        // also clips the rows past N.
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // The staging buffer is free once the previous TMA store has read it.
          if (leader && pending) bulk_wait_read0();
          named_bar_sync(kEpiBar, WG_THREADS);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            FA_TMEM_LD32(tO + 64 * h + 32 * c, o);
            tmem_ld_wait();
            if (h == 1 && c == 1) {
              tc_fence_before();
              mbar_arrive(smem_u32(&sm.o_free[t]));
            }
            // 16-byte chunk cc of this row's 128 bytes sits at chunk cc ^ (row % 8)
            // (the 128-byte swizzle the tensor map expects).
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const int cc = 4 * c + v4;
              const uint32_t dst = stage + row * 128 + ((cc ^ (row & 7)) << 4);
              const uint32_t w0 = pack2<T>(__uint_as_float(o[8 * v4 + 0]) * inv, __uint_as_float(o[8 * v4 + 1]) * inv);
              const uint32_t w1 = pack2<T>(__uint_as_float(o[8 * v4 + 2]) * inv, __uint_as_float(o[8 * v4 + 3]) * inv);
              const uint32_t w2 = pack2<T>(__uint_as_float(o[8 * v4 + 4]) * inv, __uint_as_float(o[8 * v4 + 5]) * inv);
              const uint32_t w3 = pack2<T>(__uint_as_float(o[8 * v4 + 6]) * inv, __uint_as_float(o[8 * v4 + 7]) * inv);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                           : "memory");
            }
          }
          fence_proxy_async_smem();
          named_bar_sync(kEpiBar, WG_THREADS);
          if (leader) {
            tma_store_3d(&tm_o, stage, 64 * h, item.r0[t], item.bh);
            bulk_commit();
            pending = true;
          }
        }
        if (row_g < n && args.lse != nullptr)
          args.lse[static_cast<size_t>(item.bh) * n + row_g] =
              lt > 0.f ? m * args.scale + logf(lt) : (lt == 0.f ? -INFINITY : lt);
      }
    }
    if (leader && pending) bulk_wait0();  // every output store completes before exit
  } else {
    // ------------------------------------------------------------ softmax warps
    // Warpgroup t is the softmax of query tile slot t: thread = row (TMEM lane
    // 32 (warp % 4) + lane), all 128 score columns of the key tile in registers.
    regs_inc<kSoftmaxRegs>();
    const int t = wg;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * 128;
    const float sl2 = args.scale_log2;
    int ns = 0;     // S tiles consumed (s_full phase)
    int nst = 0;    // items published (st_full / st_empty phase)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int lin = item_of(k, total);
      if (lin < 0) break;
      const Item item = make_item<OFFSET>(lin, BH, num_pairs, geo);
      if (!active(item, t)) continue;  // the epilogue writes an inactive tile's rows
      const int r0 = item.r0[t];
      const int row_p = r0 + row + geo.q_off;  // the row's position in the key sequence
      float m = -INFINITY, l = 0.f;
      bool nan_row = false;
      for (int j = item.lo_t[t]; j < item.hi_t[t]; ++j, ++ns) {
        ok = mbar_wait_warp(smem_u32(&sm.s_full[t]), ns & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (tile_needs_mask(j, r0, geo)) {
          // Visible keys of this row form one interval [c_lo, c_hi) of the tile's
          // columns.  The mask is applied in tensor memory, 32 columns at a time,
          // before the single pass below reads S, so the unrolled main pass carries no
          // mask code.  These few instructions run while the other tile's softmax
          // keeps the sub-partition's issue slot busy, so each one counts: the general
          // rolled loop costs ~275 cycles per chunk there, the diagonal case below
          // half as much in all (measured 1578 -> 812 cycles per diagonal tile).
          const int base = j * BN;
          const int wq = warp & 3;
          if (geo.causal && geo.window <= 0 && base == r0 + geo.q_off && base + BN <= geo.Nk) {
            // The causal diagonal tile: row 32 wq + lane keeps columns up to itself, so
            // this warp's own 32-column chunk keeps e <= lane, the chunks before it are
            // whole and the chunks after it are hidden.  No votes, no per-chunk tests.
            uint32_t r[32];
            FA_TMEM_LD32(tS + 32 * wq, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = e <= lane ? r[e] : __float_as_uint(-INFINITY);
            FA_TMEM_ST32(tS + 32 * wq, r);
            const uint32_t ninf = __float_as_uint(-INFINITY);
#pragma unroll 1
            for (int c = wq + 1; c < BN / 32; ++c) FA_TMEM_ST32_SAME(tS + 32 * c, ninf);
            tmem_st_wait();
          } else {
            int c_hi = min(BN, geo.Nk - base);
            if (geo.causal) c_hi = min(c_hi, row_p - base + 1);
            const int c_lo = geo.window > 0 ? max(0, row_p - geo.window + 1 - base) : 0;
            c_hi = max(c_hi, c_lo);  // an empty interval keeps nothing
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
              // Chunks that every row of the warp sees whole need no change; chunks no
              // row of the warp sees at all are overwritten with -inf without being
              // read; only a chunk the mask edge crosses is selected element by element.
              if (__all_sync(0xffffffffu, c_lo <= 32 * c && c_hi >= 32 * c + 32)) continue;
              uint32_t r[32];
              if (__all_sync(0xffffffffu, c_hi <= 32 * c || c_lo >= 32 * c + 32)) {
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(-INFINITY);
              } else {
                FA_TMEM_LD32(tS + 32 * c, r);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = keep_or_ninf(r[e], 32 * c + e, c_lo, c_hi);
              }
              FA_TMEM_ST32(tS + 32 * c, r);
            }
            tmem_st_wait();
          }
        }
        uint32_t s[BN];
        FA_TMEM_LD32(tS + 0, (s + 0));
        FA_TMEM_LD32(tS + 32, (s + 32));
        FA_TMEM_LD32(tS + 64, (s + 64));
        FA_TMEM_LD32(tS + 96, (s + 96));
        tmem_ld_wait();
        // Row max: eight chains of 3-input max; NaN-propagating so a NaN score marks
        // the row (its output is NaN at the end).
        float mm[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          mm[q] = fmax3_nan(__uint_as_float(s[q]), __uint_as_float(s[q + 8]), -INFINITY);
#pragma unroll
        for (int c = 16; c < BN; c += 16)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            mm[q] = fmax3_nan(mm[q], __uint_as_float(s[c + q]), __uint_as_float(s[c + 8 + q]));
        const float mx = fmax3_nan(fmax3_nan(mm[0], mm[1], mm[2]), fmax3_nan(mm[3], mm[4], mm[5]),
                                   fmax3_nan(mm[6], mm[7], -INFINITY));
        nan_row |= (mx != mx);
        const float m_new = fmaxf(m, mx);  // ignores a NaN mx
        // (m_new - m) is +inf on the first visible tile and NaN while the row is
        // still empty; only the former moves the reference max.
        const bool need = (m_new - m) * sl2 > kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx((m - m_new) * sl2);
          m = m_new;
          l *= alpha;
        }
        if (j > item.lo_t[t] && __any_sync(0xffffffffu, need)) {
          // O_t's last update (PV_t(j-1)) is complete: S_t(j) was issued after it.
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            FA_TMEM_LD32(tO + 32 * c, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            FA_TMEM_ST32(tO + 32 * c, r);
          }
        }
        const float ms = (m == -INFINITY) ? 0.f : m * sl2;
        // P = 2^(s * scale * log2(e) - m * scale * log2(e)) -> 16-bit pairs in S columns
        // [0, 64) (already read).  Scores go in pairs through the packed f32x2 FMA;
        // kPolyPairs of every 8 pairs take 2^x from the cubic on the FMA pipe, the rest
        // from the special-function unit, so both pipes share the exponentials.
        const uint64_t sl2x2 = f2_pack(sl2, sl2), nms2 = f2_pack(-ms, -ms);
        uint64_t acc[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
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
            acc[(e >> 1) & 3] = f2_add(acc[(e >> 1) & 3], p2);
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
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.p_full[t]));
        {
          const uint64_t s01 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
          float a0, a1;
          f2_unpack(s01, a0, a1);
          l += a0 + a1;
        }
      }
      if (!ok) break;
      // Publish the item's row statistics for the epilogue (the previous item's
      // must have been read first).
      if (nst > 0) ok = mbar_wait_warp(smem_u32(&sm.st_empty[t]), (nst - 1) & 1, abort_flag);
      if (!ok) break;
      sm.stat_m[t][row] = m;
      sm.stat_l[t][row] = nan_row ? __uint_as_float(0x7fc00000u) : l;
      mbar_arrive(smem_u32(&sm.st_full[t]));
      ++nst;
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
  CUtensorMap tq, tk, tv, to;
  const long long heads = static_cast<long long>(a.B) * a.H;
  if (!make_tmap_half_rows(&tq, a.q, D, a.N, heads, BM, a.f16) ||
      !make_tmap_half_rows(&tk, a.k, D, a.Nk, heads, BN, a.f16) ||
      !make_tmap_half_rows(&tv, a.v, D, a.Nk, heads, BN, a.f16) ||
      !make_tmap_half_rows(&to, a.o, D, a.N, heads, BM, a.f16))
    return cudaErrorInvalidValue;
  const bool offset = a.q_off != 0 || a.Nk != a.N;
  auto kernel = offset ? (a.f16 ? fwd_tc_kernel<F16, true> : fwd_tc_kernel<Bf16, true>)
                       : (a.f16 ? fwd_tc_kernel<F16, false> : fwd_tc_kernel<Bf16, false>);
  // The register split draws on the 128 registers per thread the block is launched
  // with; with fewer, setmaxnreg.inc would wait forever, so never launch then.
  cudaFuncAttributes fattr{};
  cudaError_t e = cudaFuncGetAttributes(&fattr, reinterpret_cast<const void*>(kernel));
  if (e != cudaSuccess) return e;
  if (fattr.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long items = static_cast<long long>((a.N + 2 * BM - 1) / (2 * BM)) * heads;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  int sms = 0;
  e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
  kernel<<<grid, NUM_THREADS, kSmemBytes, stream>>>(tq, tk, tv, to, a);
  return cudaGetLastError();
}

cudaError_t take_status_fwd_tc(unsigned int* out) { return take_local_status(out); }

}  // namespace fa
