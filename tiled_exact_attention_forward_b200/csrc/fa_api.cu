// The C ABI declared in include/fa.h: argument validation on the host, then
// one or more kernel launches on the caller's stream.  No device memory is
// allocated here; workspaces come from the caller.
#include <math.h>
#include <stdint.h>

#include "../../include/fa.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr float kLog2e = 1.4426950408889634f;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(d)); }

fa_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return FA_OK;
  if (e == cudaErrorInvalidValue) return FA_ERR_INVALID;
  return FA_ERR_CUDA;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool sizes_ok(long long B, long long H, long long N) {
  return B >= 1 && H >= 1 && N >= 1 && B * H <= (1LL << 31) / 2 && N <= (1LL << 30);
}

}  // namespace

extern "C" {

int fa_version(void) { return 104; }

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID: return "FA_ERR_INVALID: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: no kernel for this dtype/head dimension";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA launch or runtime error";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a kernel gave up waiting on an internal barrier";
  }
  return "unknown fa_status";
}

fa_status fa_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                     int N, int d, float scale, int causal, int window, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID;
  if (!sizes_ok(B, H, N) || window < 0 || (causal != 0 && causal != 1)) return FA_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse && !aligned(lse, 4)))
    return FA_ERR_INVALID;
  fa::FwdArgs a{};
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.B = B; a.H = H; a.N = N; a.d = d;
  a.Nk = N; a.q_off = 0;
  a.causal = causal; a.window = window;
  a.scale = resolve_scale(scale, d);
  a.scale_log2 = a.scale * kLog2e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16 || dtype == FA_FP16) {
    if (d != 128) return FA_ERR_UNSUPPORTED;
    a.f16 = dtype == FA_FP16;
    return from_cuda(fa::launch_fwd_tc(a, st));
  }
  if (dtype == FA_FP32) {
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    return from_cuda(fa::launch_fwd_f32(a, st));
  }
  return FA_ERR_UNSUPPORTED;
}

fa_status fa_forward_offset(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                            int H, int Nq, int Nk, int q_offset, int d, float scale, int causal,
                            int window, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID;
  // Positions (row + q_offset, minus window, minus a key index) must stay inside int.
  constexpr int kLimit = 1 << 29;
  if (!sizes_ok(B, H, Nq) || Nk < 1 || Nq > kLimit || Nk > kLimit || q_offset > kLimit ||
      q_offset < -kLimit || window < 0 || window > kLimit || (causal != 0 && causal != 1))
    return FA_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse && !aligned(lse, 4)))
    return FA_ERR_INVALID;
  if ((dtype != FA_BF16 && dtype != FA_FP16) || d != 128) return FA_ERR_UNSUPPORTED;
  fa::FwdArgs a{};
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.B = B; a.H = H; a.N = Nq; a.d = d;
  a.Nk = Nk; a.q_off = q_offset;
  a.causal = causal; a.window = window;
  a.scale = resolve_scale(scale, d);
  a.scale_log2 = a.scale * kLog2e;
  a.f16 = dtype == FA_FP16;
  return from_cuda(fa::launch_fwd_tc(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_merge(const void* o_parts, const float* lse_parts, int S, void* o, float* lse, int B,
                   int H, int N, int d, fa_dtype dtype, void* stream) {
  if (!o_parts || !lse_parts || !o) return FA_ERR_INVALID;
  if (S < 1 || S > (1 << 16) || !sizes_ok(B, H, N)) return FA_ERR_INVALID;
  if (!aligned(o_parts, 16) || !aligned(o, 16) || !aligned(lse_parts, 4) || (lse && !aligned(lse, 4)))
    return FA_ERR_INVALID;
  if ((dtype != FA_BF16 && dtype != FA_FP16 && dtype != FA_FP32) || (d != 64 && d != 128)) return FA_ERR_UNSUPPORTED;
  fa::MergeArgs a{};
  a.o_parts = o_parts; a.lse_parts = lse_parts; a.o = o; a.lse = lse;
  a.rows = static_cast<long long>(B) * H * N;
  a.S = S; a.d = d;
  a.f16 = dtype == FA_FP16;
  a.f32 = dtype == FA_FP32;
  return from_cuda(fa::launch_merge(a, static_cast<cudaStream_t>(stream)));
}

size_t fa_decode_workspace_size(int B, int H, int cap, int d) {
  if (B < 1 || H < 1 || cap < 1 || d < 1) return 0;
  const size_t chunks = static_cast<size_t>(fa::decode_max_chunks(cap));
  const size_t rows = static_cast<size_t>(B) * H * chunks;
  return round_up(rows * d * sizeof(float), 256) + round_up(rows * sizeof(float), 256);
}

fa_status fa_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                    void* o, float* lse, int B, int H, int cap, int d, float scale, fa_dtype dtype,
                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !kcache || !vcache || !seqlens || !o || !workspace) return FA_ERR_INVALID;
  if (!sizes_ok(B, H, cap)) return FA_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(o, 16) ||
      !aligned(seqlens, 4) || !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
    return FA_ERR_INVALID;
  if ((dtype != FA_BF16 && dtype != FA_FP16) || d != 128) return FA_ERR_UNSUPPORTED;
  if (workspace_bytes < fa_decode_workspace_size(B, H, cap, d)) return FA_ERR_INVALID;
  fa::DecodeArgs a{};
  a.q = q; a.kcache = kcache; a.vcache = vcache; a.seqlens = seqlens; a.o = o; a.lse = lse;
  a.B = B; a.H = H; a.cap = cap; a.d = d;
  a.scale = resolve_scale(scale, d);
  a.scale_log2 = a.scale * kLog2e;
  a.max_chunks = fa::decode_max_chunks(cap);
  a.f16 = dtype == FA_FP16;
  const size_t rows = static_cast<size_t>(B) * H * a.max_chunks;
  a.ws_o = static_cast<float*>(workspace);
  a.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                      round_up(rows * d * sizeof(float), 256));
  return from_cuda(fa::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_decode_paged(const void* q, const void* kpool, const void* vpool, const int32_t* block_table,
                          const int32_t* seqlens, void* o, float* lse, int B, int H, int num_blocks,
                          int block_size, int max_blocks, int d, float scale, fa_dtype dtype, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!q || !kpool || !vpool || !block_table || !seqlens || !o || !workspace) return FA_ERR_INVALID;
  if (num_blocks < 1 || max_blocks < 1 || block_size < 1 || block_size > 4096 ||
      (block_size & (block_size - 1)) != 0)
    return FA_ERR_INVALID;
  const long long cap = static_cast<long long>(max_blocks) * block_size;
  if (!sizes_ok(B, H, cap)) return FA_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(kpool, 16) || !aligned(vpool, 16) || !aligned(o, 16) ||
      !aligned(block_table, 4) || !aligned(seqlens, 4) || !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
    return FA_ERR_INVALID;
  if ((dtype != FA_BF16 && dtype != FA_FP16) || d != 128) return FA_ERR_UNSUPPORTED;
  if (workspace_bytes < fa_decode_workspace_size(B, H, static_cast<int>(cap), d)) return FA_ERR_INVALID;
  fa::DecodeArgs a{};
  a.q = q; a.kcache = kpool; a.vcache = vpool; a.seqlens = seqlens; a.o = o; a.lse = lse;
  a.B = B; a.H = H; a.cap = static_cast<int>(cap); a.d = d;
  a.scale = resolve_scale(scale, d);
  a.scale_log2 = a.scale * kLog2e;
  a.max_chunks = fa::decode_max_chunks(a.cap);
  a.f16 = dtype == FA_FP16;
  const size_t rows = static_cast<size_t>(B) * H * a.max_chunks;
  a.ws_o = static_cast<float*>(workspace);
  a.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + round_up(rows * d * sizeof(float), 256));
  a.block_table = block_table;
  a.block_shift = 0;
  while ((1 << a.block_shift) < block_size) ++a.block_shift;
  a.max_blocks = max_blocks;
  a.num_blocks = num_blocks;
  return from_cuda(fa::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

size_t fa_backward_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  const size_t rows = static_cast<size_t>(B) * H * N;
  return round_up(rows * sizeof(float), 256) + round_up(rows * d * sizeof(float), 256);
}

fa_status fa_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                      float scale, int causal, int window, fa_dtype dtype, void* workspace,
                      size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID;
  if (!sizes_ok(B, H, N) || window < 0 || (causal != 0 && causal != 1)) return FA_ERR_INVALID;
  const void* ptrs16[] = {q, k, v, o, dout, dq, dk, dv};
  for (const void* p : ptrs16)
    if (!aligned(p, 16)) return FA_ERR_INVALID;
  if (!aligned(lse, 4) || !aligned(workspace, 256)) return FA_ERR_INVALID;
  if ((dtype != FA_BF16 && dtype != FA_FP16) || d != 128) return FA_ERR_UNSUPPORTED;
  if (workspace_bytes < fa_backward_workspace_size(B, H, N, d)) return FA_ERR_INVALID;
  fa::BwdArgs a{};
  a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.B = B; a.H = H; a.N = N; a.d = d;
  a.causal = causal; a.window = window;
  a.scale = resolve_scale(scale, d);
  a.scale_log2 = a.scale * kLog2e;
  a.f16 = dtype == FA_FP16;
  const size_t rows = static_cast<size_t>(B) * H * N;
  a.ws_delta = static_cast<float*>(workspace);
  a.ws_dq = reinterpret_cast<float*>(static_cast<char*>(workspace) + round_up(rows * sizeof(float), 256));
  return from_cuda(fa::launch_bwd(a, static_cast<cudaStream_t>(stream)));
}

fa_status fa_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 1 || limit_cycles > 4000000000LL) return FA_ERR_INVALID;
  return from_cuda(fa::launch_selftest_wait_timeout(limit_cycles, static_cast<cudaStream_t>(stream)));
}

fa_status fa_selftest_exp2_poly(const float* x, float* y, long long n, void* stream) {
  if (!x || !y || n < 1 || !aligned(x, 4) || !aligned(y, 4)) return FA_ERR_INVALID;
  return from_cuda(fa::launch_selftest_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream)));
}

fa_status fa_get_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return FA_ERR_CUDA;
  // Each source file's kernels record into a status word of their own; gather
  // (and clear) all of them.
  unsigned int word = 0;
  for (auto take : {fa::take_status_host, fa::take_status_fwd_tc, fa::take_status_bwd, fa::take_status_decode}) {
    unsigned int w = 0;
    e = take(&w);
    if (e != cudaSuccess) return FA_ERR_CUDA;
    word |= w;
  }
  if (word & fa::kStatusTimeout) return FA_ERR_TIMEOUT;
  if (word & fa::kStatusBadBlock) return FA_ERR_INVALID;
  return FA_OK;
}

}  // extern "C"
