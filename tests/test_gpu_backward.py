"""Backward parity on the GPU: gradients from the CUDA library (which
recomputes P from the forward's lse) against the oracle's analytic gradient."""
import pytest
import torch

import oracle
import tiled_exact_attention_forward_b200 as fa
import workloads
from gpu_helpers import assert_grad_close, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


def run_fwd_bwd(q, k, v, dO, causal, window, scale=None):
    o, lse = fa.forward(q, k, v, causal=causal, window=window, scale=scale)
    dq, dk, dv = fa.backward(q, k, v, o, dO, lse, causal=causal, window=window, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return dq, dk, dv


@pytest.mark.parametrize("N", [1, 100, 128, 129, 300, 512])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 130), (False, 200), (True, 1)])
def test_backward_small(N, causal, window):
    q, k, v, dO = workloads.forward_inputs(1, 2, N, 128, torch.bfloat16, seed=100 + N, device="cpu",
                                           with_dout=True)
    dq, dk, dv = run_fwd_bwd(q.cuda(), k.cuda(), v.cuda(), dO.cuda(), causal, window)
    rq, rk, rv = oracle.attention_backward(q, k, v, dO, None, causal, window)
    tag = f"N={N} causal={causal} window={window}"
    assert_grad_close(dq, rq, "dQ " + tag)
    assert_grad_close(dk, rk, "dK " + tag)
    assert_grad_close(dv, rv, "dV " + tag)


@pytest.mark.parametrize("chunks", [1, 3, 100])
def test_forward_backward_host_pipelined(chunks):
    """forward_backward_host runs the 2 x 3 heads in `chunks` groups (clamped to 6),
    reusing one backward workspace across them; gradients equal the oracle's and the
    forward outputs equal the device call's."""
    q, k, v, dO = workloads.forward_inputs(2, 3, 300, 128, torch.bfloat16, seed=43, device="cpu",
                                           with_dout=True)
    q, k, v, dO = (t.pin_memory() for t in (q, k, v, dO))
    o, lse, dq, dk, dv = fa.forward_backward_host(q, k, v, dO, causal=True, window=0, chunks=chunks)
    assert not dq.is_cuda and fa.device_status() == fa.FA_OK
    o_d, lse_d = fa.forward(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert torch.equal(o, o_d.cpu()) and torch.equal(lse, lse_d.cpu())
    rq, rk, rv = oracle.attention_backward(q, k, v, dO, None, True, 0)
    assert_grad_close(dq, rq, f"dQ chunks={chunks}")
    assert_grad_close(dk, rk, f"dK chunks={chunks}")
    assert_grad_close(dv, rv, f"dV chunks={chunks}")


@pytest.mark.parametrize("causal,window", [(True, 0), (False, 90)])
def test_autograd_binding(causal, window):
    """fa.attention as a torch.autograd function: loss = sum(o * dO), so the
    gradients reaching q, k, v are the backward of the forward at dO."""
    q, k, v, dO = workloads.forward_inputs(2, 2, 200, 128, torch.bfloat16, seed=47, device="cpu",
                                           with_dout=True)
    qd, kd, vd = (t.cuda().requires_grad_() for t in (q, k, v))
    o = fa.attention(qd, kd, vd, causal=causal, window=window)
    o_ref, _ = fa.forward(qd.detach(), kd.detach(), vd.detach(), causal=causal, window=window)
    assert torch.equal(o.detach(), o_ref)
    (o.float() * dO.cuda().float()).sum().backward()
    assert fa.device_status() == fa.FA_OK
    rq, rk, rv = oracle.attention_backward(q, k, v, dO, None, causal, window)
    assert_grad_close(qd.grad, rq, "autograd dQ")
    assert_grad_close(kd.grad, rk, "autograd dK")
    assert_grad_close(vd.grad, rv, "autograd dV")


def test_backward_explicit_scale():
    q, k, v, dO = workloads.forward_inputs(2, 1, 260, 128, torch.bfloat16, seed=8, device="cpu",
                                           with_dout=True)
    dq, dk, dv = run_fwd_bwd(q.cuda(), k.cuda(), v.cuda(), dO.cuda(), True, 0, scale=0.07)
    rq, rk, rv = oracle.attention_backward(q, k, v, dO, 0.07, True, 0)
    assert_grad_close(dq, rq, "dQ")
    assert_grad_close(dk, rk, "dK")
    assert_grad_close(dv, rv, "dV")


def test_full_size_fwd_bwd_workload_sampled():
    """Full-size causal forward+backward; the oracle recomputes whole sampled heads."""
    w = workloads.WORKLOADS["causal_fwd_bwd"]
    q, k, v, dO = workloads.workload_inputs(w, device="cuda")
    dq, dk, dv = run_fwd_bwd(q, k, v, dO, w.causal, w.window, w.scale)
    for b, h in [(0, 0), (w.B - 1, w.H - 1)]:
        rq, rk, rv = oracle.attention_backward(q[b, h].cpu(), k[b, h].cpu(), v[b, h].cpu(),
                                               dO[b, h].cpu(), w.scale, w.causal, w.window)
        assert_grad_close(dq[b, h], rq, f"dQ head ({b},{h})")
        assert_grad_close(dk[b, h], rk, f"dK head ({b},{h})")
        assert_grad_close(dv[b, h], rv, f"dV head ({b},{h})")
    for g in (dq, dk, dv):
        assert torch.isfinite(g.float()).all()
