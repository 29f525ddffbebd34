"""Forward parity on the GPU: the CUDA library (through the C ABI) against the
float64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import tiled_exact_attention_forward_b200 as fa
import workloads
from gpu_helpers import (FP32_ATOL, assert_lse_close, assert_output_close, requires_cuda,
                         to64)

pytestmark = [pytest.mark.gpu, requires_cuda]

MASKS = [(False, 0), (True, 0), (True, 1), (True, 128), (True, 129), (True, 200), (False, 77)]


def run_fwd(q, k, v, causal, window, scale=None):
    o, lse = fa.forward(q, k, v, causal=causal, window=window, scale=scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return o, lse


@pytest.mark.parametrize("N", [1, 64, 127, 128, 129, 255, 256, 300, 640])
@pytest.mark.parametrize("causal,window", MASKS)
def test_bf16_forward_small(N, causal, window):
    q, k, v = workloads.forward_inputs(2, 3, N, 128, torch.bfloat16, seed=N + 7 * window, device="cpu")
    o, lse = run_fwd(q.cuda(), k.cuda(), v.cuda(), causal, window)
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, causal, window)
    assert_output_close(o, O_ref, f"O N={N} causal={causal} window={window}")
    assert_lse_close(lse, lse_ref, f"lse N={N} causal={causal} window={window}")


@pytest.mark.parametrize("causal,window", [(True, 0), (True, 200), (False, 0), (False, 300)])
def test_bf16_forward_many_items_per_cta(causal, window):
    """160 heads x 3 row pairs = 480 work items for at most 148 persistent CTAs, so
    every CTA walks several items and crosses item boundaries (where the next
    item's first S may be issued early); N = 640 leaves the last pair with a single
    query tile."""
    q, k, v = workloads.forward_inputs(4, 40, 640, 128, torch.bfloat16, seed=31 + window, device="cpu")
    o, lse = run_fwd(q.cuda(), k.cuda(), v.cuda(), causal, window)
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, causal, window)
    assert_output_close(o, O_ref, f"O many items causal={causal} window={window}")
    assert_lse_close(lse, lse_ref, f"lse many items causal={causal} window={window}")


@pytest.mark.parametrize("window", [1, 64, 255, 256, 257, 511, 513, 1100, 5000])
def test_bf16_forward_causal_window_item_order(window):
    """Causal sliding windows deal the items whose 256 rows all see a full window
    first, head by head, then the rest pair-major.  Windows around the 256-row item
    size move the split point (every item full at window 1, none at a window longer
    than the sequence); each item must still be computed exactly once."""
    q, k, v = workloads.forward_inputs(2, 40, 1100, 128, torch.bfloat16, seed=53 + window, device="cpu")
    o, lse = run_fwd(q.cuda(), k.cuda(), v.cuda(), True, window)
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, True, window)
    assert_output_close(o, O_ref, f"O causal window={window}")
    assert_lse_close(lse, lse_ref, f"lse causal window={window}")


@pytest.mark.parametrize("chunks", [1, 4, 6, 100])
def test_forward_host_pipelined_over_head_groups(chunks):
    """forward_host splits the 2 x 3 heads into `chunks` groups (clamped to 6) whose
    copies and kernels overlap on three streams; results equal the oracle's."""
    q, k, v = workloads.forward_inputs(2, 3, 300, 128, torch.bfloat16, seed=41, device="cpu")
    q, k, v = (t.pin_memory() for t in (q, k, v))
    o, lse = fa.forward_host(q, k, v, causal=True, window=100, chunks=chunks)
    assert not o.is_cuda and o.shape == q.shape and lse.shape == (2, 3, 300)
    assert fa.device_status() == fa.FA_OK
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, True, 100)
    assert_output_close(o, O_ref, f"forward_host O chunks={chunks}")
    assert_lse_close(lse, lse_ref, f"forward_host lse chunks={chunks}")


def test_bf16_forward_explicit_scale_and_no_lse():
    q, k, v = workloads.forward_inputs(1, 2, 200, 128, torch.bfloat16, seed=11, device="cuda")
    o = torch.empty_like(q)
    st = fa.library().fa_forward(fa._ptr(q), fa._ptr(k), fa._ptr(v), fa._ptr(o), None, 1, 2, 200,
                                 128, 0.05, 1, 0, fa.FA_BF16, fa._stream(q.device))
    assert st == fa.FA_OK
    torch.cuda.synchronize()
    O_ref, _ = oracle.attention_forward(q, k, v, 0.05, True, 0)
    assert_output_close(o, O_ref, "O scale=0.05")


def test_bf16_forward_large_scores():
    # Scores of order +-100 exercise the lazy rescale of the running max.
    q, k, v = workloads.forward_inputs(1, 2, 700, 128, torch.bfloat16, seed=5, device="cpu")
    q = (q.float() * 8).to(torch.bfloat16)
    o, lse = run_fwd(q.cuda(), k.cuda(), v.cuda(), True, 0)
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, True, 0)
    assert_output_close(o, O_ref, "O large scores")
    assert_lse_close(lse, lse_ref, "lse large scores")


def test_bf16_forward_deterministic():
    q, k, v = workloads.forward_inputs(2, 4, 1000, 128, torch.bfloat16, seed=3, device="cuda")
    o1, l1 = run_fwd(q, k, v, True, 300)
    o2, l2 = run_fwd(q, k, v, True, 300)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 37, 128, 300])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 50), (False, 20)])
def test_fp32_forward(d, N, causal, window):
    q, k, v = workloads.forward_inputs(2, 2, N, d, torch.float32, seed=N + d, device="cpu")
    o, lse = run_fwd(q.cuda(), k.cuda(), v.cuda(), causal, window)
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, causal, window)
    err = np.abs(to64(o) - O_ref).max()
    assert err <= FP32_ATOL, err
    assert_lse_close(lse, lse_ref, "fp32 lse", tol=FP32_ATOL)


def test_single_head_fp32_workload():
    w = workloads.WORKLOADS["single_head_fp32"]
    q, k, v = workloads.workload_inputs(w, device="cpu")
    o, lse = run_fwd(q.cuda(), k.cuda(), v.cuda(), w.causal, w.window, w.scale)
    O_ref, lse_ref = oracle.attention_forward(q, k, v, w.scale, w.causal, w.window)
    assert np.abs(to64(o) - O_ref).max() <= FP32_ATOL
    assert_lse_close(lse, lse_ref, "lse", tol=FP32_ATOL)


def _sampled_rows(N, rng, extra=24):
    fixed = [0, 1, 127, 128, 129, 255, 256, 257, N // 2, N - 129, N - 128, N - 2, N - 1]
    rnd = rng.integers(0, N, extra).tolist()
    return np.unique(np.clip(np.array(fixed + rnd), 0, N - 1))


@pytest.mark.parametrize("name", ["causal_prefill", "sliding_window_long"])
def test_full_size_workload_sampled(name):
    """Full-size workload, in the launch configuration the benchmark times;
    the oracle checks sampled rows of sampled heads (each row needs every key)."""
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.workload_inputs(w, device="cuda")
    o, lse = run_fwd(q, k, v, w.causal, w.window, w.scale)
    rng = np.random.default_rng(0)
    heads = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 3)]
    for b, h in heads:
        rows = _sampled_rows(w.N, rng)
        O_ref, lse_ref = oracle.attention_forward_rows(q[b, h].cpu(), k[b, h].cpu(), v[b, h].cpu(),
                                                       rows, w.scale, w.causal, w.window)
        assert_output_close(o[b, h][rows], O_ref, f"{name} O head ({b},{h})")
        assert_lse_close(lse[b, h][rows], lse_ref, f"{name} lse head ({b},{h})")
    # Every row of every head is finite.
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
