// Internal launch interface between the C ABI (fa_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fa {

struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;  // may be null
  int B, H, N, d;     // N: query rows per head
  int causal, window;
  float scale;       // natural units
  float scale_log2;  // scale * log2(e)
  int f16;           // 16-bit inputs/outputs are f16 (else bf16)
  int Nk;            // key rows per head (N for self-attention)
  int q_off;         // position of query row 0 in the key sequence (0 for self-attention)
};

struct DecodeArgs {
  const void* q;
  const void* kcache;
  const void* vcache;
  const int32_t* seqlens;
  void* o;
  float* lse;  // may be null
  int B, H, cap, d;
  float scale, scale_log2;
  float* ws_o;    // [B*H][max_chunks][d] normalised chunk outputs
  float* ws_lse;  // [B*H][max_chunks] chunk logsumexp
  int max_chunks;
  // Paged cache (block_table != null): kcache/vcache are block pools
  // [num_blocks][H][1 << block_shift][d]; key j of sequence b sits in physical
  // block block_table[b * max_blocks + (j >> block_shift)].  cap = max_blocks << block_shift.
  const int32_t* block_table;
  int block_shift, max_blocks, num_blocks;
  int f16;  // q, caches and o are f16 (else bf16)
};

// Device status bit of a paged decode that met a block id outside [0, num_blocks)
// (the block is skipped, never read).
constexpr unsigned kStatusBadBlock = 2u;

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  int B, H, N, d;
  int causal, window;
  float scale, scale_log2;
  float* ws_delta;  // [B*H*N] rowsum(dO * O)
  float* ws_dq;     // [B*H*N*d] fp32 dQ accumulator
  int f16;          // 16-bit tensors are f16 (else bf16)
};

// Merge of partial results over disjoint key sets (context parallelism).
struct MergeArgs {
  const void* o_parts;     // [S][rows][d] 16-bit (or float32 with f32), each part normalised
  const float* lse_parts;  // [S][rows]; -inf marks a part that saw no key
  void* o;                 // [rows][d], the parts' type
  float* lse;              // [rows], may be null
  long long rows;          // B * H * N
  int S, d;
  int f16;
  int f32;                 // float32 parts and output
};

// Decode: keys per split chunk (one CTA each).
constexpr int kDecodeChunk = 512;

inline int decode_max_chunks(int cap) { return (cap + kDecodeChunk - 1) / kDecodeChunk; }

// Host helpers (fa_host.cu).
// A 3-D TMA map over a 16-bit (bf16, or f16 when f16 != 0) [heads][rows_per_head][d]
// array: boxes of 64 columns x box_rows rows, 128-byte swizzle, rows past the end
// read as zero.
bool make_tmap_half_rows(void* map, const void* base, int d, long long rows_per_head,
                         long long heads, int box_rows, int f16);
// The same over a float32 array, boxes of box_cols (32: 128 bytes) x box_rows.
bool make_tmap_f32_rows(void* map, const void* base, int d, long long rows_per_head,
                        long long heads, int box_cols, int box_rows);
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per device and kernel.
cudaError_t set_max_dynamic_smem(const void* func, size_t bytes);
// Number of SMs of the current device (cached per device).
cudaError_t sm_count(int* out);

// Read and clear the device status word of each source file that has one.
cudaError_t take_status_host(unsigned int* out);
cudaError_t take_status_fwd_tc(unsigned int* out);
cudaError_t take_status_bwd(unsigned int* out);
cudaError_t take_status_decode(unsigned int* out);

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t stream);
cudaError_t launch_fwd_f32(const FwdArgs& a, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream);
cudaError_t launch_selftest_wait_timeout(long long limit_cycles, cudaStream_t stream);
cudaError_t launch_selftest_exp2_poly(const float* x, float* y, long long n, cudaStream_t stream);

}  // namespace fa
