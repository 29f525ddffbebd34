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


def run_paged(q, kp, vp, table, seqlens, scale=None):
    o, lse = fa.decode_paged(q, kp, vp, table, seqlens, scale)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return o, lse


@pytest.mark.parametrize("bs", [1, 16, 64, 256])
def test_decode_paged_edge_lengths(bs):
    """Lengths 0, 1, around a block and around the 512-key chunk, and the full
    capacity; blocks shuffled through the pool, the unused rows of each last block
    NaN and unused table entries -1, so any stray read shows in the output."""
    max_blocks = -(-1100 // bs)
    lens = [0, 1, bs - 1 if bs > 1 else 2, bs, bs + 1, 511, 512, 513, max_blocks * bs]
    q, kp, vp, table, _ = workloads.paged_decode_inputs(len(lens), 3, bs, max_blocks, 128, 1, 1,
                                                         seed=20 + bs, device="cpu")
    # Re-draw a layout for these exact lengths (the generator's lengths are random).
    g = torch.Generator().manual_seed(bs)
    nblk = [-(-n // bs) for n in lens]
    perm = torch.randperm(sum(nblk), generator=g)
    kp = torch.randn(sum(nblk), 3, bs, 128, generator=g).to(torch.bfloat16)
    vp = torch.randn(sum(nblk), 3, bs, 128, generator=g).to(torch.bfloat16)
    table = torch.full((len(lens), max_blocks), -1, dtype=torch.int32)
    i = 0
    for b, n in enumerate(lens):
        table[b, :nblk[b]] = perm[i:i + nblk[b]].to(torch.int32)
        i += nblk[b]
        if n % bs:
            last = int(table[b, nblk[b] - 1])
            kp[last, :, n % bs:] = float("nan")
            vp[last, :, n % bs:] = float("nan")
    seqlens = torch.tensor(lens, dtype=torch.int32)
    o, lse = run_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), seqlens.cuda())
    o_ref, lse_ref = oracle.decode_paged_forward(q, kp, vp, table.numpy(), seqlens.numpy(), None)
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert_output_close(o[1:], o_ref[1:], f"paged decode O bs={bs}")
    assert_lse_close(lse, lse_ref, f"paged decode lse bs={bs}")


def test_decode_paged_matches_padded_cache():
    """The same rows as a padded cache and as a shuffled pool give the same result up
    to the order of the final merge (paged decode splits the keys into 1024-key
    chunks, padded decode into 512-key chunks)."""
    B, H, bs, max_blocks = 4, 2, 32, 40
    q, kp, vp, table, lens = workloads.paged_decode_inputs(B, H, bs, max_blocks, 128, 100, bs * max_blocks,
                                                           seed=7, device="cuda")
    cap = bs * max_blocks
    kc = torch.zeros(B, H, cap, 128, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    for b in range(B):
        for t in range(-(-int(lens[b]) // bs)):
            kc[b, :, t * bs:(t + 1) * bs] = kp[int(table[b, t])]
            vc[b, :, t * bs:(t + 1) * bs] = vp[int(table[b, t])]
    o_p, lse_p = run_paged(q, kp, vp, table, lens)
    o_c, lse_c = run_decode(q, kc, vc, lens)
    # Both are fp32 results (equal up to the merge order) rounded to bf16, so each
    # pair of outputs is at most one bf16 ulp apart, measured at the larger of the two.
    a, b = o_p.double().cpu().numpy(), o_c.double().cpu().numpy()
    mag = np.maximum(np.maximum(np.abs(a), np.abs(b)), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    assert np.all(np.abs(a - b) <= ulp), float((np.abs(a - b) / ulp).max())
    assert (lse_p - lse_c).abs().max() <= 1e-5


def test_decode_paged_out_of_range_block_is_reported_and_skipped():
    """A used table entry outside the pool is never dereferenced: the kernel skips
    that block, records FA_ERR_INVALID, and every other sequence is unaffected."""
    B, H, bs, max_blocks = 3, 2, 16, 8
    q, kp, vp, table, lens = workloads.paged_decode_inputs(B, H, bs, max_blocks, 128, 40, 120,
                                                           seed=11, device="cpu")
    bad = table.clone()
    bad[1, 0] = kp.shape[0] + 1000
    o, lse = fa.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), bad.cuda(), lens.cuda())
    assert fa.device_status() == fa.FA_ERR_INVALID
    assert fa.device_status() == fa.FA_OK   # the record was cleared
    o_ref, lse_ref = oracle.decode_paged_forward(q, kp, vp, table.numpy(), lens.numpy(), None)
    keep = [0, 2]
    assert_output_close(o[keep], o_ref[keep], "other sequences O")
    assert_lse_close(lse[keep], lse_ref[keep], "other sequences lse")


def test_full_size_paged_decode_workload_sampled():
    """The paged decode workload at full size, in the benchmark's launch
    configuration; the oracle checks sampled (sequence, head) pairs."""
    w = workloads.WORKLOADS["paged_kv_decode"]
    q, kp, vp, table, lens = workloads.workload_inputs(w, device="cuda")
    o, lse = run_paged(q, kp, vp, table, lens, w.scale)
    for b in (0, 17, w.B - 1):
        nb = -(-int(lens[b]) // w.block_size)
        tb = table[b:b + 1, :nb].cpu()
        ids = tb[0].long()
        sub_k, sub_v = kp[ids.cuda()].cpu(), vp[ids.cuda()].cpu()
        local = torch.arange(nb, dtype=torch.int32).reshape(1, nb)
        o_ref, lse_ref = oracle.decode_paged_forward(q[b:b + 1].cpu(), sub_k, sub_v, local.numpy(),
                                                     lens[b:b + 1].cpu().numpy(), w.scale)
        assert_output_close(o[b:b + 1], o_ref, f"paged full-size O seq {b}")
        assert_lse_close(lse[b:b + 1], lse_ref, f"paged full-size lse seq {b}")
    assert torch.isfinite(o.float()).all()


def test_decode_bindings_reject_mismatched_dtypes():
    """A cache of another dtype than q is refused before any launch."""
    q = torch.zeros(1, 2, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(1, 2, 64, 128, dtype=torch.float16, device="cuda")
    lens = torch.full((1,), 64, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        fa.decode(q, kc, kc, lens)
    table = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        fa.decode_paged(q, kc.view(4, 2, 16, 128), kc.view(4, 2, 16, 128), table, lens)
