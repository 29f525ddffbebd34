"""float16 inputs: the same kernels (tcgen05 kind::f16 with f16 operands, P and dS
formed in f16), checked against the float64 oracle like the bf16 path."""
import numpy as np
import pytest
import torch

import oracle
import tiled_exact_attention_forward_b200 as fa
import workloads
from gpu_helpers import assert_grad_close, assert_lse_close, assert_output_close, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]
F16 = torch.float16


@pytest.mark.parametrize("N", [1, 129, 300, 640])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 130)])
def test_fp16_forward(N, causal, window):
    q, k, v = workloads.forward_inputs(2, 3, N, 128, F16, seed=200 + N, device="cpu")
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), causal=causal, window=window)
    torch.cuda.synchronize()
    assert o.dtype == F16 and fa.device_status() == fa.FA_OK
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, causal, window)
    assert_output_close(o, O_ref, f"fp16 O N={N}")
    assert_lse_close(lse, lse_ref, f"fp16 lse N={N}")


def test_fp16_forward_many_items_per_cta():
    q, k, v = workloads.forward_inputs(4, 40, 640, 128, F16, seed=210, device="cpu")
    o, lse = fa.forward(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, True, 0)
    assert_output_close(o, O_ref, "fp16 O many items")
    assert_lse_close(lse, lse_ref, "fp16 lse many items")


def test_fp16_same_values_as_bf16_path_within_rounding():
    """Inputs exactly representable in both types: the two kernels agree to their
    output rounding (f16 carries 3 more mantissa bits than bf16)."""
    q, k, v = workloads.forward_inputs(1, 4, 500, 128, torch.bfloat16, seed=211, device="cuda")
    o_b, l_b = fa.forward(q, k, v, causal=True)
    o_h, l_h = fa.forward(q.half(), k.half(), v.half(), causal=True)
    assert (o_b.float() - o_h.float()).abs().max() <= 2e-2
    assert (l_b - l_h).abs().max() <= 1e-3


def test_fp16_decode_and_paged_decode():
    q, kc, vc, lens = workloads.decode_inputs(5, 3, 1300, 128, 1, 1300, F16, seed=212, device="cpu")
    o, lse = fa.decode(q.cuda(), kc.cuda(), vc.cuda(), lens.cuda())
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.decode_forward(q, kc, vc, lens.numpy(), None)
    assert o.dtype == F16
    assert_output_close(o, o_ref, "fp16 decode O")
    assert_lse_close(lse, lse_ref, "fp16 decode lse")
    q, kp, vp, table, lens = workloads.paged_decode_inputs(5, 3, 16, 90, 128, 1, 1400, F16, seed=213,
                                                           device="cpu")
    o, lse = fa.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), lens.cuda())
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    o_ref, lse_ref = oracle.decode_paged_forward(q, kp, vp, table.numpy(), lens.numpy(), None)
    assert_output_close(o, o_ref, "fp16 paged decode O")
    assert_lse_close(lse, lse_ref, "fp16 paged decode lse")


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 130)])
def test_fp16_backward(causal, window):
    q, k, v, dO = workloads.forward_inputs(1, 2, 300, 128, F16, seed=214, device="cpu", with_dout=True)
    qd, kd, vd = (t.cuda().requires_grad_() for t in (q, k, v))
    o = fa.attention(qd, kd, vd, causal=causal, window=window)
    (o.float() * dO.cuda().float()).sum().backward()
    assert qd.grad.dtype == F16 and fa.device_status() == fa.FA_OK
    rq, rk, rv = oracle.attention_backward(q, k, v, dO, None, causal, window)
    assert_grad_close(qd.grad, rq, "fp16 dQ")
    assert_grad_close(kd.grad, rk, "fp16 dK")
    assert_grad_close(vd.grad, rv, "fp16 dV")
