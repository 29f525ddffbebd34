"""The C ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

import tiled_exact_attention_forward_b200 as fa
from tiled_exact_attention_forward_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    return re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)


def test_header_declares_the_abi():
    names = declared_functions()
    assert set(names) == set(fa.EXPORTED_SYMBOLS), names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    for code in range(5):
        assert lib.fa_status_string(code).startswith(b"FA_")
    assert lib.fa_status_string(99) == b"unknown fa_status"
    # 1.04: fa_merge accepts float32 partials; 1.03 added fa_selftest_exp2_poly to
    # 1.02 (fa_forward_offset, fa_merge), which added to 1.01 (fa_decode_paged, FA_FP16).
    assert lib.fa_version() == 104


P = ctypes.c_void_p
GOOD = P(0x100000)       # 16-byte aligned, never dereferenced: validation fails first
MISALIGNED = P(0x100008)


def fwd(lib, q=GOOD, k=GOOD, v=GOOD, o=GOOD, lse=None, B=1, H=1, N=128, d=128, causal=0,
        window=0, dtype=fa.FA_BF16):
    return lib.fa_forward(q, k, v, o, lse, B, H, N, d, 0.0, causal, window, dtype, None)


def test_forward_rejects_bad_arguments(lib):
    assert fwd(lib, q=None) == fa.FA_ERR_INVALID
    assert fwd(lib, o=None) == fa.FA_ERR_INVALID
    assert fwd(lib, B=0) == fa.FA_ERR_INVALID
    assert fwd(lib, H=-1) == fa.FA_ERR_INVALID
    assert fwd(lib, N=0) == fa.FA_ERR_INVALID
    assert fwd(lib, window=-1) == fa.FA_ERR_INVALID
    assert fwd(lib, causal=2) == fa.FA_ERR_INVALID
    assert fwd(lib, k=MISALIGNED) == fa.FA_ERR_INVALID
    assert fwd(lib, lse=P(0x100002)) == fa.FA_ERR_INVALID
    assert fwd(lib, d=64) == fa.FA_ERR_UNSUPPORTED          # bf16 needs d = 128
    assert fwd(lib, d=96, dtype=fa.FA_FP32) == fa.FA_ERR_UNSUPPORTED
    assert fwd(lib, dtype=7) == fa.FA_ERR_UNSUPPORTED


def test_forward_offset_rejects_bad_arguments(lib):
    def fo(q=GOOD, lse=None, Nq=128, Nk=200, off=0, d=128, causal=1, window=0, dtype=fa.FA_BF16):
        return lib.fa_forward_offset(q, GOOD, GOOD, GOOD, lse, 1, 2, Nq, Nk, off, d, 0.0, causal,
                                     window, dtype, None)

    assert fo(q=None) == fa.FA_ERR_INVALID
    assert fo(Nq=0) == fa.FA_ERR_INVALID
    assert fo(Nk=0) == fa.FA_ERR_INVALID
    assert fo(Nk=(1 << 29) + 1) == fa.FA_ERR_INVALID
    assert fo(off=(1 << 29) + 1) == fa.FA_ERR_INVALID
    assert fo(off=-(1 << 29) - 1) == fa.FA_ERR_INVALID
    assert fo(window=(1 << 29) + 1) == fa.FA_ERR_INVALID
    assert fo(window=-1) == fa.FA_ERR_INVALID
    assert fo(causal=3) == fa.FA_ERR_INVALID
    assert fo(q=MISALIGNED) == fa.FA_ERR_INVALID
    assert fo(lse=P(0x100001)) == fa.FA_ERR_INVALID
    assert fo(d=64) == fa.FA_ERR_UNSUPPORTED
    assert fo(dtype=fa.FA_FP32) == fa.FA_ERR_UNSUPPORTED


def test_merge_rejects_bad_arguments(lib):
    def mg(parts=GOOD, lse_parts=GOOD, S=3, o=GOOD, N=100, d=128, dtype=fa.FA_BF16):
        return lib.fa_merge(parts, lse_parts, S, o, None, 2, 3, N, d, dtype, None)

    assert mg(parts=None) == fa.FA_ERR_INVALID
    assert mg(lse_parts=None) == fa.FA_ERR_INVALID
    assert mg(o=None) == fa.FA_ERR_INVALID
    assert mg(S=0) == fa.FA_ERR_INVALID
    assert mg(S=(1 << 16) + 1) == fa.FA_ERR_INVALID
    assert mg(N=0) == fa.FA_ERR_INVALID
    assert mg(parts=MISALIGNED) == fa.FA_ERR_INVALID
    assert mg(lse_parts=P(0x100002)) == fa.FA_ERR_INVALID
    assert mg(d=96) == fa.FA_ERR_UNSUPPORTED
    assert mg(dtype=7) == fa.FA_ERR_UNSUPPORTED  # no such dtype (float32 partials are supported)
    assert mg(dtype=fa.FA_FP32, d=96) == fa.FA_ERR_UNSUPPORTED


def test_decode_rejects_bad_arguments(lib):
    ws = lib.fa_decode_workspace_size(2, 3, 1000, 128)
    assert ws > 0 and ws % 256 == 0
    assert lib.fa_decode_workspace_size(0, 3, 1000, 128) == 0

    def dec(q=GOOD, seqlens=GOOD, ws_ptr=GOOD, ws_bytes=ws, cap=1000, d=128, dtype=fa.FA_BF16):
        return lib.fa_decode(q, GOOD, GOOD, seqlens, GOOD, None, 2, 3, cap, d, 0.0, dtype,
                             ws_ptr, ws_bytes, None)

    assert dec(q=None) == fa.FA_ERR_INVALID
    assert dec(seqlens=None) == fa.FA_ERR_INVALID
    assert dec(ws_ptr=None) == fa.FA_ERR_INVALID
    assert dec(ws_ptr=P(0x100010)) == fa.FA_ERR_INVALID      # workspace must be 256-aligned
    assert dec(ws_bytes=ws - 1) == fa.FA_ERR_INVALID
    assert dec(cap=0) == fa.FA_ERR_INVALID
    assert dec(d=64) == fa.FA_ERR_UNSUPPORTED
    assert dec(dtype=fa.FA_FP32) == fa.FA_ERR_UNSUPPORTED


def test_backward_rejects_bad_arguments(lib):
    ws = lib.fa_backward_workspace_size(1, 2, 300, 128)
    assert ws >= (2 * 300 * 4) + (2 * 300 * 128 * 4) and ws % 256 == 0

    def bwd(lse=GOOD, ws_ptr=GOOD, ws_bytes=ws, N=300, d=128, window=0):
        return lib.fa_backward(GOOD, GOOD, GOOD, GOOD, GOOD, lse, GOOD, GOOD, GOOD, 1, 2, N, d,
                               0.0, 1, window, fa.FA_BF16, ws_ptr, ws_bytes, None)

    assert bwd(lse=None) == fa.FA_ERR_INVALID
    assert bwd(ws_bytes=ws - 256) == fa.FA_ERR_INVALID
    assert bwd(ws_ptr=None) == fa.FA_ERR_INVALID
    assert bwd(window=-3) == fa.FA_ERR_INVALID
    assert bwd(N=0) == fa.FA_ERR_INVALID
    assert bwd(d=64) == fa.FA_ERR_UNSUPPORTED


def test_python_binding_refuses_cpu_tensors():
    import torch

    q = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward(q, q, q)


def test_shard_forward_and_merge_refuse_cpu_tensors():
    import torch

    q = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward_offset(q, q, q, 0)
    with pytest.raises(ValueError):
        fa.merge(q[None], torch.zeros(1, 1, 1, 8))


def test_forward_host_checks_its_inputs_before_touching_the_device():
    import torch

    q = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward_host(q.transpose(2, 3), q, q)  # not contiguous
    with pytest.raises(ValueError):
        fa.forward_host(q, q[:, :1], q)  # shapes differ


def test_forward_backward_host_checks_its_inputs():
    import torch

    q = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward_backward_host(q, q, q, q.float())  # dout dtype differs


def test_decode_paged_rejects_bad_arguments(lib):
    ws = lib.fa_decode_workspace_size(2, 3, 64 * 16, 128)

    def dec(table=GOOD, ws_ptr=GOOD, ws_bytes=ws, num_blocks=10, bs=16, max_blocks=64, d=128):
        return lib.fa_decode_paged(GOOD, GOOD, GOOD, table, GOOD, GOOD, None, 2, 3, num_blocks, bs,
                                   max_blocks, d, 0.0, fa.FA_BF16, ws_ptr, ws_bytes, None)

    assert dec(table=None) == fa.FA_ERR_INVALID
    assert dec(ws_ptr=None) == fa.FA_ERR_INVALID
    assert dec(ws_bytes=ws - 1) == fa.FA_ERR_INVALID
    assert dec(bs=24) == fa.FA_ERR_INVALID           # not a power of two
    assert dec(bs=0) == fa.FA_ERR_INVALID
    assert dec(bs=8192) == fa.FA_ERR_INVALID         # above 4096
    assert dec(num_blocks=0) == fa.FA_ERR_INVALID
    assert dec(max_blocks=0) == fa.FA_ERR_INVALID
    assert dec(d=64) == fa.FA_ERR_UNSUPPORTED


def test_decode_noalloc_rejects_sizes_beyond_its_array(lib):
    # The size check runs before any CUDA call, so the pointers (never
    # dereferenced) can be fake; on a machine with a GPU nothing is launched
    # either, because the sizes are refused first.
    limit = 8 << 20
    B, H, cap, d = 64, 32, 8192, 128          # ~17 MB of partials
    assert lib.fa_decode_workspace_size(B, H, cap, d) > limit
    st = lib.fa_decode_noalloc(GOOD, GOOD, GOOD, GOOD, GOOD, None, B, H, cap, d, 0.0, fa.FA_BF16, None)
    assert st == fa.FA_ERR_INVALID
    assert lib.fa_decode_workspace_size(1016, 1, cap, d) <= limit < lib.fa_decode_workspace_size(1017, 1, cap, d)
    st = lib.fa_decode_noalloc(GOOD, GOOD, GOOD, GOOD, GOOD, None, 1017, 1, cap, d, 0.0, fa.FA_BF16, None)
    assert st == fa.FA_ERR_INVALID
    assert lib.fa_decode_noalloc(GOOD, GOOD, GOOD, GOOD, GOOD, None, 0, 1, cap, d, 0.0, fa.FA_BF16,
                                 None) == fa.FA_ERR_INVALID


def test_decode_noalloc_within_its_array_reaches_the_runtime_without_a_gpu(lib):
    # Sizes inside the array pass the size check and reach the CUDA runtime,
    # which on a machine without a GPU fails the address lookup: FA_ERR_CUDA,
    # not FA_ERR_INVALID.  Skipped where a GPU exists, since the fake pointers
    # would then reach a kernel.
    import torch

    if torch.cuda.is_available():
        pytest.skip("fake pointers must not reach a GPU")
    st = lib.fa_decode_noalloc(GOOD, GOOD, GOOD, GOOD, GOOD, None, 1016, 1, 8192, 128, 0.0,
                               fa.FA_BF16, None)
    assert st == fa.FA_ERR_CUDA
