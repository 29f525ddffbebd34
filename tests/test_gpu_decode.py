"""Decode parity on the GPU against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import tiled_exact_attention_forward_b200 as fa
import workloads
from gpu_helpers import assert_lse_close, assert_output_close, requires_cuda

pytestmark = [pytest.mark.gpu, requires_cuda]


def run_decode(q, kc, vc, seqlens, scale=None):
    o, lse = fa.decode(q, kc, vc, seqlens, scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return o, lse


def test_decode_edge_lengths_nan_padding():
    """Lengths at the chunk edges, 1 and the full capacity; cache rows past each
    length hold NaN, so any read beyond a sequence shows up in the output."""
    cap = 1537
    lens = [1, 7, 511, 512, 513, 1024, 1536, 1537]
    B, H = len(lens), 3
    g = torch.Generator().manual_seed(9)
    q = torch.randn(B, H, 128, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, H, cap, 128, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, H, cap, 128, generator=g).to(torch.bfloat16)
    for b, n in enumerate(lens):
        kc[b, :, n:] = float("nan")
        vc[b, :, n:] = float("nan")
    seqlens = torch.tensor(lens, dtype=torch.int32)
    o, lse = run_decode(q.cuda(), kc.cuda(), vc.cuda(), seqlens.cuda())
    o_ref, lse_ref = oracle.decode_forward(q, kc, vc, seqlens.numpy(), None)
    assert_output_close(o, o_ref, "decode O")
    assert_lse_close(lse, lse_ref, "decode lse")


def test_decode_zero_and_clamped_lengths():
    B, H, cap = 3, 2, 700
    q, kc, vc, _ = workloads.decode_inputs(B, H, cap, 128, 1, cap, seed=4, device="cpu")
    seqlens = torch.tensor([0, 900, 300], dtype=torch.int32)  # 900 is clamped to the capacity
    o, lse = run_decode(q.cuda(), kc.cuda(), vc.cuda(), seqlens.cuda())
    o_ref, lse_ref = oracle.decode_forward(q, kc, vc, np.array([0, cap, 300]), None)
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert_output_close(o[1:], o_ref[1:], "decode O")
    assert_lse_close(lse, lse_ref, "decode lse")


def test_decode_matches_forward_last_row():
    """Decode of token n-1 equals the last row of the causal forward kernel."""
    B, H, n = 2, 4, 777
    q, k, v = workloads.forward_inputs(B, H, n, 128, torch.bfloat16, seed=12, device="cuda")
    o_f, lse_f = fa.forward(q, k, v, causal=True)
    seqlens = torch.full((B,), n, dtype=torch.int32, device="cuda")
    o_d, lse_d = run_decode(q[:, :, n - 1].contiguous(), k, v, seqlens)
    assert_output_close(o_d, o_f[:, :, n - 1], "decode vs forward last row")
    assert_lse_close(lse_d, lse_f[:, :, n - 1], "decode vs forward lse")


def test_full_size_decode_workload_sampled():
    w = workloads.WORKLOADS["kv_cache_decode"]
    q, kc, vc, seqlens = workloads.workload_inputs(w, device="cuda")
    o, lse = run_decode(q, kc, vc, seqlens, w.scale)
    lens = seqlens.cpu().numpy()
    rng = np.random.default_rng(1)
    bs = sorted(set([int(np.argmin(lens)), int(np.argmax(lens))] + rng.integers(0, w.B, 4).tolist()))
    for b in bs:
        hs = [0, w.H - 1, int(rng.integers(0, w.H))]
        n = int(lens[b])
        sub_k = kc[b:b + 1, hs, :n].cpu()
        sub_v = vc[b:b + 1, hs, :n].cpu()
        o_ref, lse_ref = oracle.decode_forward(q[b:b + 1, hs].cpu(), sub_k, sub_v, np.array([n]),
                                               w.scale)
        assert_output_close(o[b:b + 1, hs], o_ref, f"decode b={b}")
        assert_lse_close(lse[b:b + 1, hs], lse_ref, f"decode lse b={b}")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
