"""Context parallelism on the GPU: the key-shard forward (fa_forward_offset) and
the merge (fa_merge) through the C ABI against the float64 oracle, and the
ring's steps of every rank, run on one device, against the oracle's full
forward."""
import dataclasses
import os
import sys

import numpy as np
import pytest
import torch

import oracle
import tiled_exact_attention_forward_b200 as fa
import workloads
from gpu_helpers import assert_lse_close, assert_output_close, requires_cuda, to64
from tiled_exact_attention_forward_b200 import context_parallel as cp

pytestmark = [pytest.mark.gpu, requires_cuda]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _qkv(B, H, Nq, Nk, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, H, Nq, 128), generator=g).to(dtype)
    k = torch.randn((B, H, Nk, 128), generator=g).to(dtype)
    v = torch.randn((B, H, Nk, 128), generator=g).to(dtype)
    return q, k, v


def _check_offset(q, k, v, off, causal, window, what):
    o, lse = fa.forward_offset(q.cuda(), k.cuda(), v.cuda(), off, causal=causal, window=window)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    O_ref, lse_ref = oracle.attention_forward_offset(q, k, v, off, None, causal, window)
    assert_output_close(o, O_ref, f"O {what}")
    live = np.isfinite(lse_ref)
    got = lse.cpu().numpy()
    assert np.all(np.isneginf(got[~live])), f"lse of rows with no visible key {what}"
    assert torch.all(o.cpu()[torch.from_numpy(~live)] == 0), f"O of rows with no visible key {what}"
    if live.any():
        assert_lse_close(lse.cpu()[torch.from_numpy(live)], lse_ref[live], f"lse {what}")


# (Nq, Nk, q_offset, causal, window): offsets that put the key shard before, on and
# after the queries; ragged lengths; windows that leave whole query tiles (even whole
# two-tile items) without a visible key, and a first tile without keys before a
# second one with keys.
CASES = [
    (300, 200, 0, True, 0),
    (300, 200, 100, True, 0),
    (300, 200, 250, True, 0),
    (300, 200, -50, True, 0),
    (300, 200, -400, True, 0),       # every row before every key: all empty
    (300, 200, 150, False, 0),
    (300, 200, 150, False, 120),
    (300, 200, 320, True, 130),
    (700, 256, 0, True, 100),        # rows >= 355 see nothing: tiles 3-5 inactive
    (500, 300, -150, True, 0),       # tile 0 inactive, tile 1 active
    (500, 300, -300, True, 0),       # item 0 empty, item 1 active
    (129, 1000, 871, True, 0),
    (256, 129, 4096, False, 0),
]


@pytest.mark.parametrize("Nq,Nk,off,causal,window", CASES)
def test_forward_offset_small(Nq, Nk, off, causal, window):
    q, k, v = _qkv(2, 3, Nq, Nk, torch.bfloat16, seed=Nq + Nk + abs(off) + window)
    _check_offset(q, k, v, off, causal, window, f"Nq={Nq} Nk={Nk} off={off} causal={causal} w={window}")


def test_forward_offset_fp16():
    q, k, v = _qkv(2, 2, 400, 300, torch.float16, seed=9)
    _check_offset(q, k, v, 200, True, 250, "fp16")


@pytest.mark.parametrize("off,window", [(0, 100), (-150, 0), (200, 0)])
def test_forward_offset_many_items_with_inactive_tiles(off, window):
    """160 heads x 3 two-tile items for at most 148 persistent CTAs: CTAs walk
    active and inactive tiles and empty items in one pass of their pipelines."""
    q, k, v = _qkv(4, 40, 700, 256, torch.bfloat16, seed=77 + window)
    _check_offset(q, k, v, off, True, window, f"many items off={off} window={window}")


def test_forward_offset_zero_is_forward():
    q, k, v = (t.cuda() for t in _qkv(2, 3, 517, 517, torch.bfloat16, seed=5))
    o1, l1 = fa.forward(q, k, v, causal=True, window=200)
    o2, l2 = fa.forward_offset(q, k, v, 0, causal=True, window=200)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_forward_offset_rejects_bad_arguments():
    q, k, v = (t.cuda() for t in _qkv(1, 1, 64, 64, torch.bfloat16, seed=1))
    with pytest.raises(fa.FAError):
        fa.forward_offset(q, k, v, 1 << 30)
    with pytest.raises(fa.FAError):
        fa.forward_offset(q.float(), k.float(), v.float(), 0)
    with pytest.raises(ValueError):
        fa.forward_offset(q, k[:, :, :, :64].contiguous(), v, 0)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("S", [1, 3, 6])
def test_merge_matches_oracle(dtype, d, S):
    B, H, N = 2, 3, 333
    g = torch.Generator().manual_seed(S * d)
    o_parts = torch.randn((S, B, H, N, d), generator=g).to(dtype)
    lse_parts = (torch.randn((S, B, H, N), generator=g) * 4).float()
    # Parts that saw no key for some rows, and one row no part saw.
    lse_parts[0, 0, 0, ::3] = -float("inf")
    if S > 1:
        lse_parts[S - 1, 1, 2, 5::7] = -float("inf")
    lse_parts[:, 1, 1, 10] = -float("inf")
    o, lse = fa.merge(o_parts.cuda(), lse_parts.cuda())
    torch.cuda.synchronize()
    O_ref, lse_ref = oracle.merge_partials(o_parts, lse_parts)
    assert_output_close(o, O_ref, f"merged O S={S} d={d}")
    live = np.isfinite(lse_ref)
    assert np.all(np.isneginf(lse.cpu().numpy()[~live]))
    assert torch.all(o.cpu()[1, 1, 10] == 0)
    assert_lse_close(lse.cpu()[torch.from_numpy(live)], lse_ref[live], f"merged lse S={S} d={d}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("S", [1, 2, 5, 8])
def test_merge_float32_partials_match_oracle(d, S):
    """float32 partials merge in float32 throughout: the result is within float32
    rounding of the float64 merge (the 16-bit tolerances do not apply)."""
    B, H, N = 2, 3, 257
    g = torch.Generator().manual_seed(100 + S * d)
    o_parts = torch.randn((S, B, H, N, d), generator=g, dtype=torch.float64)
    lse_parts = torch.randn((S, B, H, N), generator=g, dtype=torch.float64) * 4
    lse_parts[0, 0, 0, ::3] = -float("inf")
    lse_parts[:, 1, 1, 10] = -float("inf")
    o_p32, l_p32 = o_parts.float(), lse_parts.float()
    o, lse = fa.merge(o_p32.cuda(), l_p32.cuda())
    torch.cuda.synchronize()
    assert o.dtype == torch.float32
    # The oracle merges exactly the float32 values the kernel read.
    O_ref, lse_ref = oracle.merge_partials(o_p32.double(), l_p32.double())
    assert_output_close(o, O_ref, f"float32 merge S={S} d={d}", max_tol=5e-5, mean_tol=1e-6)
    live = np.isfinite(lse_ref)
    assert np.all(np.isneginf(lse.cpu().numpy()[~live]))
    assert torch.all(o.cpu()[1, 1, 10] == 0)
    assert_lse_close(lse.cpu()[torch.from_numpy(live)], lse_ref[live], f"float32 merge lse S={S}", tol=5e-5)


def test_merge_float32_empty_parts_never_leak():
    """A float32 part with lse = -inf for a row is not read into the result, even
    when its O holds NaN there."""
    S, B, H, N, d = 3, 1, 2, 64, 128
    g = torch.Generator().manual_seed(7)
    o_parts = torch.randn((S, B, H, N, d), generator=g)
    lse_parts = torch.randn((S, B, H, N), generator=g)
    lse_parts[1, :, :, ::2] = -float("inf")
    o_parts[1, :, :, ::2] = float("nan")
    o, lse = fa.merge(o_parts.cuda(), lse_parts.cuda())
    torch.cuda.synchronize()
    clean = o_parts.clone()
    clean[1, :, :, ::2] = 0.0
    O_ref, lse_ref = oracle.merge_partials(clean.double(), lse_parts.double())
    assert_output_close(o, O_ref, "float32 merge with empty parts", max_tol=5e-5, mean_tol=1e-6)
    assert_lse_close(lse.cpu(), lse_ref, "float32 merge lse with empty parts", tol=5e-5)


def test_merge_propagates_nan():
    o_parts = torch.randn((2, 1, 1, 8, 128)).to(torch.bfloat16)
    lse_parts = torch.zeros((2, 1, 1, 8))
    lse_parts[1, 0, 0, 3] = float("nan")
    o, lse = fa.merge(o_parts.cuda(), lse_parts.cuda())
    torch.cuda.synchronize()
    assert torch.isnan(o[0, 0, 3].float()).all() and torch.isnan(lse[0, 0, 3])
    assert torch.isfinite(o[0, 0, :3].float()).all() and torch.isfinite(lse[0, 0, 4:]).all()


def _emulated_ring(q, k, v, G, causal, window, balanced):
    """Every rank's ring steps on this device, with the driver's own schedule."""
    B, H, N, d = q.shape
    m = cp.n_chunks(G, balanced)
    C = N // m
    chunks = [[t[:, :, a * C:(a + 1) * C].contiguous() for a in range(m)] for t in (q, k, v)]
    res = {}
    for r in range(G):
        plan = cp.ring_schedule(r, G, C, causal, window, balanced)
        for qi, a in enumerate(cp.rank_chunks(r, G, balanced)):
            parts = [(cp.rank_chunks(st.shard, G, balanced)[p.k_chunk], p.q_offset)
                     for st in plan for p in st.partials if p.q_chunk == qi]
            o_p = torch.empty((len(parts), B, H, C, d), dtype=q.dtype, device="cuda")
            l_p = torch.empty((len(parts), B, H, C), dtype=torch.float32, device="cuda")
            for i, (c, off) in enumerate(parts):
                fa.forward_offset(chunks[0][a], chunks[1][c], chunks[2][c], off, causal=causal, window=window,
                                  out=o_p[i], lse=l_p[i])
            res[a] = fa.merge(o_p, l_p) if len(parts) > 1 else (o_p[0], l_p[0])
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    return torch.cat([res[a][0] for a in range(m)], dim=2), torch.cat([res[a][1] for a in range(m)], dim=2)


@pytest.mark.parametrize("G,balanced", [(2, False), (4, False), (2, True), (4, True)])
@pytest.mark.parametrize("causal,window", [(True, 0), (True, 300), (False, 0), (False, 200), (True, 1)])
def test_emulated_ring_matches_full_forward(G, balanced, causal, window):
    q, k, v = workloads.forward_inputs(2, 3, 1024, 128, torch.bfloat16, seed=G + window, device="cpu")
    o, lse = _emulated_ring(q.cuda(), k.cuda(), v.cuda(), G, causal, window, balanced)
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, causal, window)
    what = f"ring G={G} balanced={balanced} causal={causal} window={window}"
    assert_output_close(o, O_ref, what)
    assert_lse_close(lse, lse_ref, what)


def test_context_parallel_forward_without_process_group_is_forward():
    q, k, v = (t.cuda() for t in _qkv(1, 4, 640, 640, torch.bfloat16, seed=12))
    o1, l1 = cp.context_parallel_forward(q, k, v, causal=True)
    o2, l2 = fa.forward(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_full_size_context_parallel_workload_sampled():
    """The benchmark's 16K causal context over 4 ring ranks (balanced layout: 8 chunks),
    in the launch configuration the benchmark times; sampled rows of sampled heads
    against the oracle."""
    sys.path.insert(0, ROOT)
    import bench

    w = workloads.WORKLOADS["context_parallel_causal"]
    step, (qs, ks, vs), (outs, lses), _ = bench.context_parallel_emulated(w, torch.device("cuda", 0), fa)
    step()
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    q, k, v = (torch.cat(t, dim=2) for t in (qs, ks, vs))
    o, lse = torch.cat(outs, dim=2), torch.cat(lses, dim=2)
    rng = np.random.default_rng(1)
    C = w.N // cp.n_chunks(w.shards, w.balanced)  # chunk boundaries are where the partials meet
    fixed = [0, 1, C - 1, C, C + 1, 2 * C + 127, 3 * C - 1, 3 * C, 5 * C, w.N - C, w.N - 1]
    rows = np.unique(np.concatenate([fixed, rng.integers(0, w.N, 16)]))
    for h in (0, w.H // 2, w.H - 1):
        O_ref, lse_ref = oracle.attention_forward_rows(q[0, h].cpu(), k[0, h].cpu(), v[0, h].cpu(), rows,
                                                       w.scale, w.causal, w.window)
        assert_output_close(o[0, h][rows], O_ref, f"context parallel O head {h}")
        assert_lse_close(lse[0, h][rows], lse_ref, f"context parallel lse head {h}")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("S", [3, 5, 8, 9])
def test_merge_empty_parts_never_leak(S):
    """Parts with lse = -inf are not part of the result, whatever their O holds
    (here NaN and inf), across the kernel's batches of four parts."""
    B, H, N, d = 1, 2, 200, 128
    g = torch.Generator().manual_seed(40 + S)
    o_parts = torch.randn((S, B, H, N, d), generator=g).to(torch.bfloat16)
    lse_parts = (torch.randn((S, B, H, N), generator=g) * 4).float()
    for s in range(0, S, 2):  # every other part empty for a third of the rows
        lse_parts[s, :, :, s % 3::3] = -float("inf")
        o_parts[s, :, :, s % 3::3] = float("nan") if s % 4 == 0 else float("inf")
    lse_parts[:, 0, 1, 7] = -float("inf")  # one row no part saw
    o, lse = fa.merge(o_parts.cuda(), lse_parts.cuda())
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    clean = torch.where(torch.isneginf(lse_parts)[..., None], torch.zeros_like(o_parts), o_parts)
    O_ref, lse_ref = oracle.merge_partials(clean, lse_parts)
    assert torch.isfinite(o.float()).all()
    assert torch.all(o[0, 1, 7] == 0) and torch.isneginf(lse[0, 1, 7])
    assert_output_close(o, O_ref, f"merge S={S} with empty parts")
    live = np.isfinite(lse_ref)
    assert_lse_close(lse.cpu()[torch.from_numpy(live)], lse_ref[live], f"merge lse S={S}")


@pytest.mark.parametrize("name", ["merge_parts_2", "merge_parts_4", "merge_parts_8", "merge_parts_4_fp32"])
def test_full_size_merge_workload_sampled(name):
    """The merge benchmark workloads at full size, in the benchmark's launch
    configuration; the oracle merges sampled rows."""
    w = workloads.WORKLOADS[name]
    o_parts, lse_parts = workloads.workload_inputs(w, device="cuda")
    o, lse = fa.merge(o_parts, lse_parts)
    torch.cuda.synchronize()
    assert fa.device_status() == fa.FA_OK
    rows = np.unique(np.concatenate([[0, 1, w.N - 1], np.random.default_rng(5).integers(0, w.N, 64)]))
    for h in (0, w.H - 1):
        O_ref, lse_ref = oracle.merge_partials(o_parts[:, 0, h, rows].cpu(), lse_parts[:, 0, h, rows].cpu())
        assert_output_close(o[0, h, rows], O_ref, f"{name} O head {h}")
        assert_lse_close(lse[0, h, rows], lse_ref, f"{name} lse head {h}")
    assert torch.isfinite(o.float()).all()
