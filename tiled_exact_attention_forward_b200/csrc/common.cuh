// Shared device helpers: status word, bounded barrier waits, and thin inline
// PTX wrappers for the sm_100a asynchronous machinery (mbarrier, TMA, tcgen05
// / TMEM).  Everything here is written from the PTX ISA's instruction
// descriptions; nothing is generated.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Device status word (bit flags), read and cleared by fa_get_device_status().
// The library is built as whole-program device code, one module per source
// file (separate compilation would make ptxas ignore the per-warpgroup
// register budgets of setmaxnreg), so each source file that launches kernels
// has a status word of its own and exports a take_status_* accessor for it.
enum : unsigned { kStatusTimeout = 1u };
namespace {
__device__ unsigned int g_status = 0;

// Read and clear this source file's status word.  Call after the work that may
// have set it has completed.
[[maybe_unused]] cudaError_t take_local_status(unsigned int* out) {
  unsigned int word = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&word, g_status, sizeof(word));
  if (e != cudaSuccess) return e;
  if (word != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *out = word;
  return cudaSuccess;
}
}  // namespace

// A wait that has not completed after this many SM clock cycles (about two
// seconds at the B200's clocks) is treated as a hang: the kernel records
// kStatusTimeout and unwinds instead of spinning forever.
constexpr long long kWaitLimitCycles = 4000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false when the
// CTA-wide abort flag is (or becomes) set, or the wait times out (which sets
// the flag and the device status word).  Callers unwind on false.
__device__ __forceinline__ bool mbar_wait_limit(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                long long limit_cycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit_cycles) {
      *abort_flag = 1;
      atomicOr(&g_status, kStatusTimeout);
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  return mbar_wait_limit(bar, parity, abort_flag, kWaitLimitCycles);
}

// The same wait for code that continues with warp-collective instructions
// (tcgen05.ld/st, shuffles): every lane of the warp must call it, and all lanes
// get the same answer, so a partial failure can never split the warp.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// Barrier of `nthreads` threads (whole warps) on named barrier `id` (1..15).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// AND of `v` over the `nthreads` threads (whole warps) that use named barrier `id`.
__device__ __forceinline__ bool named_bar_all(bool v, int id, int nthreads) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Bounded wait that ignores the abort flag: used only while draining copies
// that are already in flight, which complete on their own.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicOr(&g_status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 3-D tiled load global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Prefetch a 3-D tile of a tensor map into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_l2_3d(const void* tmap, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

// 3-D tiled store shared -> global (bulk-group completion).
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// 3-D tiled reduce-add shared -> global (element type from the tensor map).
__device__ __forceinline__ void tma_reduce_add_3d(const void* tmap, uint32_t src, int x, int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Make generic-proxy shared-memory writes visible to the async proxy (TMA, MMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- batched MMA issue

// A 128-deep K block (eight kind::f16 MMAs of K = 16) from one asm statement:
// the warp runs it uniformly, one elected lane issues, and the descriptors'
// 32-bit low words (start address >> 4, leading-byte offset) step by
// compile-time offsets.  Shared-memory addresses stay below 2^18, so the
// 14-bit address field never carries into the offset field.  Issued this way
// the MMAs keep pace with the tensor core (64.7 cycles per 128 x 128 x 16 on
// B200); one asm statement per MMA, each with its own elect and 64-bit
// descriptor adds, issued one every 84 cycles.
//
// Both operands in shared memory; A and B advance by the same offsets
// (O1..O7, in 16-byte units).  The first MMA accumulates only if acc0 != 0.
template <uint32_t IDESC, uint32_t O1, uint32_t O2, uint32_t O3, uint32_t O4, uint32_t O5, uint32_t O6,
          uint32_t O7>
__device__ __forceinline__ void mma8_ss(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t hi, uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b32 a1, b1;\n\t.reg .b64 ad, bd;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %4, %4;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "mov.b64 ad, {%1, %3};\n\tmov.b64 bd, {%2, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, p;\n\t"
      "add.u32 a1, %1, %6;\n\tadd.u32 b1, %2, %6;\n\tmov.b64 ad, {a1, %3};\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, t;\n\t"
      "add.u32 a1, %1, %7;\n\tadd.u32 b1, %2, %7;\n\tmov.b64 ad, {a1, %3};\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, t;\n\t"
      "add.u32 a1, %1, %8;\n\tadd.u32 b1, %2, %8;\n\tmov.b64 ad, {a1, %3};\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, t;\n\t"
      "add.u32 a1, %1, %9;\n\tadd.u32 b1, %2, %9;\n\tmov.b64 ad, {a1, %3};\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, t;\n\t"
      "add.u32 a1, %1, %10;\n\tadd.u32 b1, %2, %10;\n\tmov.b64 ad, {a1, %3};\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, t;\n\t"
      "add.u32 a1, %1, %11;\n\tadd.u32 b1, %2, %11;\n\tmov.b64 ad, {a1, %3};\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, t;\n\t"
      "add.u32 a1, %1, %12;\n\tadd.u32 b1, %2, %12;\n\tmov.b64 ad, {a1, %3};\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, t;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(hi), "r"(acc0), "n"(IDESC), "n"(O1), "n"(O2), "n"(O3), "n"(O4), "n"(O5),
      "n"(O6), "n"(O7)
      : "memory");
}
// A from tensor memory: A's column advances by CA per MMA, B's low word by OB
// (16-byte units).
template <uint32_t IDESC, uint32_t CA, uint32_t OB>
__device__ __forceinline__ void mma8_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi, uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b32 a1, b1;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %4, %4;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "mov.b64 bd, {%2, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %5, p;\n\t"
      "add.u32 a1, %1, %6;\n\tadd.u32 b1, %2, %13;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t"
      "add.u32 a1, %1, %7;\n\tadd.u32 b1, %2, %14;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t"
      "add.u32 a1, %1, %8;\n\tadd.u32 b1, %2, %15;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t"
      "add.u32 a1, %1, %9;\n\tadd.u32 b1, %2, %16;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t"
      "add.u32 a1, %1, %10;\n\tadd.u32 b1, %2, %17;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t"
      "add.u32 a1, %1, %11;\n\tadd.u32 b1, %2, %18;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t"
      "add.u32 a1, %1, %12;\n\tadd.u32 b1, %2, %19;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(acc0), "n"(IDESC), "n"(CA), "n"(2 * CA), "n"(3 * CA), "n"(4 * CA),
      "n"(5 * CA), "n"(6 * CA), "n"(7 * CA), "n"(OB), "n"(2 * OB), "n"(3 * OB), "n"(4 * OB), "n"(5 * OB),
      "n"(6 * OB), "n"(7 * OB)
      : "memory");
}

// Four kind::f16 MMAs with A from tensor memory, per-step A column offsets
// CA0..CA3 and B low-word offsets OB0..OB3 (16-byte units); the first MMA
// accumulates only if acc0 != 0.
template <uint32_t IDESC, uint32_t CA0, uint32_t CA1, uint32_t CA2, uint32_t CA3, uint32_t OB0, uint32_t OB1,
          uint32_t OB2, uint32_t OB3>
__device__ __forceinline__ void mma4_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t hi, uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b32 a1, b1;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %4, %4;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "add.u32 a1, %1, %6;\n\tadd.u32 b1, %2, %10;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, p;\n\t"
      "add.u32 a1, %1, %7;\n\tadd.u32 b1, %2, %11;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t"
      "add.u32 a1, %1, %8;\n\tadd.u32 b1, %2, %12;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t"
      "add.u32 a1, %1, %9;\n\tadd.u32 b1, %2, %13;\n\tmov.b64 bd, {b1, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], bd, %5, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(hi), "r"(acc0), "n"(IDESC), "n"(CA0), "n"(CA1), "n"(CA2), "n"(CA3), "n"(OB0),
      "n"(OB1), "n"(OB2), "n"(OB3)
      : "memory");
}

// ---------------------------------------------------------------- register split
// Move this warpgroup's per-thread register budget up or down (all four warps of
// the warpgroup execute the same instruction).  The budgets of all warpgroups
// must add up to at most the registers the block was launched with.
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once all previously issued tcgen05 async ops of this thread complete.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem], kind::f16, A read from tensor memory.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The two 16-bit input types of kind::f16 MMAs.  One type parameter gives both
// the A and the B format of an MMA, so a kernel never mixes them.
struct Bf16 { static constexpr uint32_t kFormat = 1; };
struct F16 { static constexpr uint32_t kFormat = 0; };

// Instruction descriptor for kind::f16 with A and B of type T and fp32 D.
//   bits 4-5 D format (1 = f32), 7-9 A format and 10-12 B format (0 = f16,
//   1 = bf16), 15 A major (0 = K), 16 B major (0 = K, 1 = MN),
//   17-22 N >> 3, 24-28 M >> 4.
template <class T>
__host__ __device__ constexpr uint32_t idesc_f32acc(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (T::kFormat << 7) | (T::kFormat << 10) | (uint32_t(a_mn_major) << 15) |
         (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
  return idesc_f32acc<Bf16>(M, N, a_mn_major, b_mn_major);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   bits 0-13 start address >> 4, 16-29 leading-dimension byte offset >> 4,
//   32-45 stride-dimension byte offset >> 4, 46-47 version (1 on sm_100),
//   49-51 base offset (0: tiles are 1024-byte aligned), 61-63 layout
//   (2 = 128-byte swizzle).
// K-major tiles (rows of 128 bytes, 8-row groups 1024 bytes apart): lbo is
// unused (16), sbo = 1024.  MN-major tiles: lbo = distance between 64-element
// MN chunks, sbo = distance between 8-row K groups.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t desc = 0;
  desc |= uint64_t((saddr >> 4) & 0x3FFFu);
  desc |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  desc |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  desc |= uint64_t(1) << 46;
  desc |= uint64_t(2) << 61;
  return desc;
}

// TMEM loads/stores: 32 lanes x 32 bits, repeated over 32 consecutive columns.
// Thread t of the warp sees lane (base lane + t); register i holds column
// (base column + i).
#define FA_TMEM_LD32(taddr, r)                                                                      \
  asm volatile(                                                                                     \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"  \
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),         \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),     \
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),  \
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),  \
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])                                          \
      : "r"(taddr))

#define FA_TMEM_ST32(taddr, r)                                                                      \
  asm volatile(                                                                                     \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"   \
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr), \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),       \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), \
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),          \
      "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]),          \
      "r"(r[30]), "r"(r[31])                                                                        \
      : "memory")

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- math
// 2^x on the special-function unit (approximate, flushes denormals; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Pack two floats to bf16x2 (round to nearest even): `lo` in bits 0-15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// The same for f16x2.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
template <class T> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<Bf16>(float lo, float hi) { return pack_bf16x2(lo, hi); }
template <> __device__ __forceinline__ uint32_t pack2<F16>(float lo, float hi) { return pack_f16x2(lo, hi); }

// Eight 16-bit values (one 16-byte load) to float.
template <class T> __device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]);
template <> __device__ __forceinline__ void unpack8<Bf16>(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
template <> __device__ __forceinline__ void unpack8<F16>(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xffffu)));
    f[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
  }
}
// One float to the 16-bit type (round to nearest even), as raw bits.
template <class T> __device__ __forceinline__ unsigned short to16(float x);
template <> __device__ __forceinline__ unsigned short to16<Bf16>(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
template <> __device__ __forceinline__ unsigned short to16<F16>(float x) { return __half_as_ushort(__float2half_rn(x)); }

// ---------------------------------------------------------------- packed fp32 (sm_100 f32x2)
// Two floats in one 64-bit register pair; fma/add/sub/mul.rn.f32x2 process both
// in one instruction.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max of three floats that is NaN when any input is NaN.
__device__ __forceinline__ float fmax3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair of floats on the FMA pipe (no special-function unit):
// x = j + f with j = round(x) (the 1.5 * 2^23 rounding trick) and
// f in [-0.5, 0.5]; 2^f from a cubic fitted for minimum relative error on that
// interval (max 7.5e-5; derivation in fit_exp2_poly.py); 2^j added to the
// exponent field.  x is clamped to >= -126.5 so 2^j stays a normal scale: for
// x below that the result is a tiny positive number (< 1e-38) instead of 0,
// far under bf16's resolution of P.  A NaN input does NOT come out as NaN
// (the clamp drops it); callers that must propagate NaN check for it apart.
__device__ __forceinline__ uint64_t exp2_poly_pair(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x2 = f2_pack(fmaxf(x0, -126.5f), fmaxf(x1, -126.5f));
  const uint64_t kMagic = f2_pack(12582912.0f, 12582912.0f);
  const uint64_t t = f2_add(x2, kMagic);       // integer part in the low mantissa bits
  const uint64_t j = f2_sub(t, kMagic);        // round(x)
  const uint64_t f = f2_sub(x2, j);            // in [-0.5, 0.5]
  uint64_t p = f2_fma(f2_pack(0.055171623826026917f, 0.055171623826026917f), f,
                      f2_pack(0.24261116981506348f, 0.24261116981506348f));
  p = f2_fma(p, f, f2_pack(0.6932610273361206f, 0.6932610273361206f));
  p = f2_fma(p, f, f2_pack(0.9999280571937561f, 0.9999280571937561f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  // bits(t) = bits(1.5 * 2^23) + j; shifting left by 23 leaves exactly j << 23.
  const uint32_t r0 = (__float_as_uint(t0) << 23) + __float_as_uint(p0);
  const uint32_t r1 = (__float_as_uint(t1) << 23) + __float_as_uint(p1);
  return f2_pack(__uint_as_float(r0), __uint_as_float(r1));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// x if lo <= c < hi, else -inf (as raw bits), without a branch: the caller's
// bounds differ from lane to lane, and a per-element `if` there compiles to
// divergent branches that cost far more than the compare and select.
__device__ __forceinline__ uint32_t keep_or_ninf(uint32_t x, int c, int lo, int hi) {
  uint32_t r;
  asm("{\n\t.reg .pred p;\n\t"
      "setp.lt.u32 p, %1, %2;\n\t"
      "selp.b32 %0, %3, 0xff800000, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(c - lo)), "r"(static_cast<uint32_t>(hi - lo)), "r"(x));
  return r;
}

// x if lo <= c < hi, else 0, without a branch (see keep_or_ninf).
__device__ __forceinline__ float keep_or_zero(float x, int c, int lo, int hi) {
  float r;
  asm("{\n\t.reg .pred p;\n\t"
      "setp.lt.u32 p, %1, %2;\n\t"
      "selp.f32 %0, %3, 0f00000000, p;\n\t}"
      : "=f"(r)
      : "r"(static_cast<uint32_t>(c - lo)), "r"(static_cast<uint32_t>(hi - lo)), "f"(x));
  return r;
}

// Visibility rule of the mask (see fa.h).
__device__ __forceinline__ bool key_visible(int i, int j, int n, int causal, int window) {
  return j < n && (!causal || j <= i) && (window <= 0 || j > i - window);
}

}  // namespace fa
