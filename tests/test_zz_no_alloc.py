"""fa_decode_noalloc: the decode entry point for callers that cannot allocate.

Some callers have no allocator on their request path (serving runtimes that fix
all device memory at start-up, plugin interfaces that pass only inputs and
outputs), so this entry point keeps its scratch in an array built into the
library.  Its results must match fa_decode's (the workspace version) on two
calls in a row -- the second call reuses the array the first one filled.
A further test checks that calls after the first take no device memory.  Sizes
beyond the array are refused on the host before any CUDA call; that check is
tested without a GPU in test_abi_host.py, so no fake pointer ever reaches a GPU
here.  This file sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from gpu_helpers import assert_lse_close, assert_output_close, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    import tiled_exact_attention_forward_b200 as fa

    lib = fa.library()
    B, H, cap, d = 8, 16, 3000, 128
    q, kc, vc, _ = workloads.decode_inputs(B, H, cap, d, 1, cap, seed=17, device="cuda")
    lens = torch.tensor([1, 511, 512, 513, 1777, 2999, 3000, 64], dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    o_ref, lse_ref = fa.decode(q, kc, vc, lens)
    torch.cuda.synchronize()
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.fa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(lens), _p(o), _p(lse), B, H, cap, d,
                                   0.0, fa.FA_BF16, stream)
        assert st == fa.FA_OK, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert fa.device_status() == fa.FA_OK
        assert_output_close(o, o_ref, f"no-alloc decode O, call {call}")
        assert_lse_close(lse, lse_ref, f"no-alloc decode lse, call {call}")
        # A second, different problem between the two calls must not leak into the next one.
        if call == 0:
            q2 = torch.randn_like(q.float()).to(q.dtype)
            o2 = torch.empty_like(q)
            assert lib.fa_decode_noalloc(_p(q2), _p(kc), _p(vc), _p(lens), _p(o2), None, B, H, cap,
                                         d, 0.0, fa.FA_BF16, stream) == fa.FA_OK


def test_noalloc_decode_allocates_nothing_after_its_first_call():
    # The point of the entry point: once the first call on a device has loaded
    # the library's module (and with it the scratch array), further calls take
    # no device memory.  The device's free bytes must not move across calls.
    import tiled_exact_attention_forward_b200 as fa

    lib = fa.library()
    B, H, cap, d = 4, 8, 2048, 128
    q, kc, vc, lens = workloads.decode_inputs(B, H, cap, d, 1, cap, seed=23, device="cuda")
    o = torch.empty_like(q)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        assert lib.fa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(lens), _p(o), None, B, H, cap, d,
                                     0.0, fa.FA_BF16, stream) == fa.FA_OK

    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert fa.device_status() == fa.FA_OK
    assert free1 == free0, f"free device memory moved by {free0 - free1} bytes"
