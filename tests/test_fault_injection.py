"""Fault injection without faulting the GPU.

"Building Flash Attention from Scratch in Pure NumPy" (extension 4) proposes
corrupting 5% of the K entries and checking the output against a numerical
bound.  The bound used here holds for ANY finite K: each output row is a convex
combination of the visible V rows, so it lies inside their column-wise
[min, max].  Non-finite inputs must propagate (NaN rows) without hanging.
The timeout path of the bounded barrier waits is exercised by a self-test
kernel that waits on a barrier nothing completes.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def corrupt(k: torch.Tensor, frac: float, seed: int, magnitude: float = 60.0) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    kc = k.clone()
    mask = torch.rand(kc.shape, generator=g) < frac
    vals = (torch.rand(kc.shape, generator=g) * 2 - 1) * magnitude
    kc[mask] = vals[mask].to(kc.dtype)
    return kc


def hull_violation(O, V, causal, window):
    """Largest distance of an output entry outside the [min, max] of its visible V rows."""
    O = np.asarray(O, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N = V.shape[-2]
    worst = 0.0
    for i in range(N):
        lo_j = max(0, i - window + 1) if window > 0 else 0
        hi_j = i + 1 if causal else N
        rows = V[..., lo_j:hi_j, :]
        vmin, vmax = rows.min(axis=-2), rows.max(axis=-2)
        o = O[..., i, :]
        worst = max(worst, float(np.maximum(vmin - o, 0).max()), float(np.maximum(o - vmax, 0).max()))
    return worst


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 9)])
def test_oracle_convex_hull_under_corrupted_keys(causal, window):
    q, k, v = workloads.forward_inputs(1, 2, 40, 8, torch.float32, seed=3)
    kc = corrupt(k, 0.05, seed=1)
    O, _ = oracle.attention_forward(q, kc, v, None, causal, window)
    assert hull_violation(O, v.numpy(), causal, window) < 1e-12


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 300)])
def test_kernel_convex_hull_under_corrupted_keys(causal, window):
    import tiled_exact_attention_forward_b200 as fa

    q, k, v = workloads.forward_inputs(2, 2, 700, 128, torch.bfloat16, seed=21)
    kc = corrupt(k, 0.05, seed=2)
    o, lse = fa.forward(q.cuda(), kc.cuda(), v.cuda(), causal=causal, window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    # bf16 output rounding: half an ulp of the largest |V| (2^-8 relative) is allowed.
    slack = float(v.abs().max()) * 2.0 ** -8
    assert hull_violation(o.float().cpu().numpy(), v.float().numpy(), causal, window) <= slack
    O_ref, lse_ref = oracle.attention_forward(q, kc, v, None, causal, window)
    assert np.abs(o.double().cpu().numpy() - O_ref).max() <= 2e-2
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() <= 2e-3 * 60


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_kernel_nan_input_propagates_without_hang():
    import tiled_exact_attention_forward_b200 as fa

    q, k, v = workloads.forward_inputs(1, 1, 384, 128, torch.bfloat16, seed=4, device="cuda")
    k[0, 0, 200, 5] = float("nan")
    o, lse = fa.forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    bad = ~torch.isfinite(o.float()).all(dim=-1)[0, 0]
    assert not bad[:200].any()        # rows that cannot see key 200 are untouched
    assert bad[200:].all()            # rows that see it are NaN


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_bounded_wait_reports_timeout_and_context_survives():
    import tiled_exact_attention_forward_b200 as fa

    assert fa.device_status() == fa.FA_OK
    assert fa.selftest_wait_timeout(20_000_000) == fa.FA_OK   # ~10 ms of waiting
    assert fa.device_status() == fa.FA_ERR_TIMEOUT
    assert fa.device_status() == fa.FA_OK                     # the record was cleared
    q, k, v = workloads.forward_inputs(1, 1, 256, 128, torch.bfloat16, seed=5, device="cuda")
    o, lse = fa.forward(q, k, v, causal=True)                  # the context still works
    torch.cuda.synchronize()
    O_ref, _ = oracle.attention_forward(q, k, v, None, True, 0)
    assert np.abs(o.double().cpu().numpy() - O_ref).max() <= 2e-2
