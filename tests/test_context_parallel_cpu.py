"""Host logic of the context-parallel (ring) forward, on CPU.

The ring driver takes its compute as two callables; here they are the float64
oracle's key-shard forward and merge, so the exchange (gloo ranks, world size 2
and 3), the schedule and the merge bookkeeping are checked end to end against
the oracle's full forward without a GPU.  The CUDA compute is checked on the
GPU in test_gpu_context_parallel.py.
"""
import itertools
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

import oracle
from tiled_exact_attention_forward_b200 import context_parallel as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MASKS = [(False, 0), (True, 0), (True, 5), (False, 7), (True, 1), (True, 40)]


def _brute_visible(n_q, n_k, off, causal, window):
    for i in range(n_q):
        p = i + off
        for j in range(n_k):
            if (not causal or j <= p) and (window <= 0 or j > p - window):
                return True
    return False


def test_visible_matches_brute_force():
    for n_q, n_k in [(1, 1), (3, 5), (7, 2), (4, 4)]:
        for off in range(-12, 13):
            for causal, window in MASKS + [(False, 1), (True, 3)]:
                assert cp.visible(n_q, n_k, off, causal, window) == \
                    _brute_visible(n_q, n_k, off, causal, window), (n_q, n_k, off, causal, window)


def _pairs_of_plan(world, chunk, causal, window, balanced):
    """(query chunk, key chunk) pairs each rank computes, from its schedule."""
    out = {}
    for r in range(world):
        mine = cp.rank_chunks(r, world, balanced)
        for st in cp.ring_schedule(r, world, chunk, causal, window, balanced):
            theirs = cp.rank_chunks(st.shard, world, balanced) if st.shard >= 0 else ()
            for p in st.partials:
                a, c = mine[p.q_chunk], theirs[p.k_chunk]
                assert p.q_offset == (a - c) * chunk
                out.setdefault(r, []).append((a, c))
    return out


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("balanced", [False, True])
def test_ring_schedule_computes_every_visible_pair_once(world, balanced):
    C = 8
    m = cp.n_chunks(world, balanced)
    held = sorted(a for r in range(world) for a in cp.rank_chunks(r, world, balanced))
    assert held == list(range(m))  # the layout partitions the sequence
    for causal, window in MASKS:
        pairs = _pairs_of_plan(world, C, causal, window, balanced)
        got = sorted(x for r in pairs for x in pairs[r])
        want = sorted((a, c) for a in range(m) for c in range(m)
                      if _brute_visible(C, C, (a - c) * C, causal, window))
        assert got == want, (world, balanced, causal, window)


@pytest.mark.parametrize("world", [2, 3, 4, 8])
@pytest.mark.parametrize("balanced", [False, True])
def test_ring_sends_match_receives(world, balanced):
    for causal, window in MASKS:
        plans = [cp.ring_schedule(r, world, 8, causal, window, balanced) for r in range(world)]
        for r in range(world):
            nxt = (r + 1) % world
            for t in range(world - 1):
                assert plans[r][t].send == plans[nxt][t].recv, (r, t, causal, window)
                if plans[nxt][t].recv:
                    # The receiver holds at step t + 1 what the sender held at step t.
                    assert plans[nxt][t + 1].shard == plans[r][t].shard
            assert not plans[r][world - 1].send and not plans[r][world - 1].recv


def test_causal_ring_stops_forwarding_shards_nobody_ahead_sees():
    # Contiguous causal layout: shard s is seen by ranks s .. world - 1 only, so it
    # is passed on only until it reaches the last rank (and the last rank's own shard
    # is never sent).
    world = 4
    plans = [cp.ring_schedule(r, world, 8, True, 0, False) for r in range(world)]
    sends = [(r, t, plans[r][t].shard) for r in range(world) for t in range(world) if plans[r][t].send]
    assert all(s <= r for r, t, s in sends)
    assert not any(r == world - 1 for r, t, s in sends)
    assert len(sends) == 6  # shard 0 three hops, shard 1 two, shard 2 one
    # Balanced causal layout: every rank's later chunk sees every shard, so all travel.
    plans = [cp.ring_schedule(r, world, 8, True, 0, True) for r in range(world)]
    assert sum(st.send for p in plans for st in p) == world * (world - 1)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_balanced_causal_layout_balances_the_ranks(world):
    """Visible (query, key) pairs per rank under a causal mask: the balanced layout
    keeps the largest rank within 1.1x of the mean (the contiguous one does not)."""
    N = 128 * world

    def loads(balanced):
        C = N // cp.n_chunks(world, balanced)
        out = []
        for r in range(world):
            n = 0
            mine = cp.rank_chunks(r, world, balanced)
            for st in cp.ring_schedule(r, world, C, True, 0, balanced):
                theirs = cp.rank_chunks(st.shard, world, balanced) if st.shard >= 0 else ()
                for p in st.partials:
                    ok = oracle.allowed_mask(C, C, True, 0, q_pos=np.arange(C) + p.q_offset)
                    n += int(ok.sum())
            out.append(n)
        return np.array(out)

    bal, con = loads(True), loads(False)
    assert bal.sum() == con.sum()
    assert bal.max() <= 1.1 * bal.mean(), bal
    assert con.max() > 1.4 * con.mean(), con


def test_shard_rows_reassembles_the_sequence():
    x = torch.arange(2 * 48 * 3, dtype=torch.float64).reshape(1, 2, 48, 3)
    for world in (1, 2, 3, 4):
        for balanced in (False, True):
            m = cp.n_chunks(world, balanced)
            C = 48 // m
            parts = {}
            for r in range(world):
                rows = cp.shard_rows(x, r, world, balanced)
                for i, a in enumerate(cp.rank_chunks(r, world, balanced)):
                    parts[a] = rows[:, :, i * C:(i + 1) * C]
            assert torch.equal(torch.cat([parts[a] for a in range(m)], dim=2), x)


def _oracle_partial(q, k, v, q_offset, causal, window, scale, out, lse):
    O, L = oracle.attention_forward_offset(q, k, v, q_offset, scale, causal, window)
    out.copy_(torch.from_numpy(O))
    lse.copy_(torch.from_numpy(L))


def _oracle_merge(o_parts, lse_parts):
    O, L = oracle.merge_partials(o_parts.numpy(), lse_parts.numpy())
    return torch.from_numpy(O), torch.from_numpy(L)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, balanced, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, C, d = 2, 2, 7, 4
        N = C * cp.n_chunks(world, balanced)
        g = torch.Generator().manual_seed(7)
        q, k, v = (torch.randn((B, H, N, d), generator=g, dtype=torch.float64) for _ in range(3))
        ring = cp.RingForward(_oracle_partial, _oracle_merge, balanced=balanced)
        errs = []
        for causal, window in MASKS:
            o, lse = ring(*(cp.shard_rows(t, rank, world, balanced).contiguous() for t in (q, k, v)),
                          causal, window, 0.5)
            O_ref, lse_ref = oracle.attention_forward(q, k, v, 0.5, causal, window)
            O_mine = cp.shard_rows(torch.from_numpy(O_ref), rank, world, balanced).numpy()
            L_mine = cp.shard_rows(torch.from_numpy(lse_ref)[..., None], rank, world, balanced)[..., 0].numpy()
            errs.append((float(np.abs(o.numpy() - O_mine).max()), float(np.abs(lse.numpy() - L_mine).max())))
        tdist.barrier()
        out[rank] = errs
    finally:
        tdist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("balanced", [False, True])
def test_ring_forward_gloo_matches_full_forward(world, balanced):
    """The ring over gloo ranks, with the oracle's key-shard forward
    (attention_forward_offset) for every chunk pair and its merge, equals the
    oracle's full forward on every rank's rows, in both layouts."""
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, balanced, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == list(range(world))
    for r in range(world):
        for (eo, el), mask in zip(res[r], MASKS):
            # lse partials travel as float32: errors of order 1e-7 relative.
            assert eo < 1e-5 and el < 1e-5, (r, mask, eo, el)


def test_ring_forward_single_process_is_plain_forward():
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn((1, 2, 9, 4), generator=g, dtype=torch.float64) for _ in range(3))
    o, lse = cp.RingForward(_oracle_partial, _oracle_merge)(q, k, v, True, 4, None)
    O_ref, lse_ref = oracle.attention_forward(q, k, v, None, True, 4)
    assert np.abs(o.numpy() - O_ref).max() < 1e-12
    assert np.abs(lse.numpy() - lse_ref).max() < 1e-6


def test_bench_plan_partitions_the_visible_pairs():
    """The key-chunk partials of all ranks cover each visible (query, key) pair of
    the whole sequence exactly once, so the ring's work is the full forward's."""
    import dataclasses

    sys.path.insert(0, ROOT)
    import bench
    import workloads

    w0 = workloads.WORKLOADS["context_parallel_causal"]
    assert (w0.N, w0.shards, w0.causal, w0.balanced) == (16384, 4, True, True)
    C, plans = bench.context_parallel_plan(w0)
    assert C == 2048 and [sum(len(st.partials) for st in p) for p in plans] == [9, 9, 9, 9]
    for balanced in (False, True):
        for causal, window in MASKS + [(True, 70), (False, 0)]:
            w = dataclasses.replace(w0, N=96, shards=4, causal=causal, window=window, balanced=balanced)
            C, plans = bench.context_parallel_plan(w)
            total = 0
            for r, plan in enumerate(plans):
                for st in plan:
                    for p in st.partials:
                        ok = oracle.allowed_mask(C, C, causal, window, q_pos=np.arange(C) + p.q_offset)
                        total += int(ok.sum())
            assert total == bench.allowed_pairs(96, causal, window), (balanced, causal, window)


def test_ring_forward_checks_shapes_before_any_exchange():
    q = torch.zeros((1, 2, 8, 4), dtype=torch.float64)
    ring = cp.RingForward(_oracle_partial, _oracle_merge)
    with pytest.raises(ValueError):
        ring(q, q[:, :, :4], q)
    with pytest.raises(ValueError):
        ring(q, q.transpose(2, 3).contiguous().transpose(2, 3), q)


def test_bench_ring_accounting():
    """With N GPUs the bench runs one shard per rank: the whole job's launches per
    step are the visible partials plus the merges, and the emulated one-GPU plan
    of the same shard count launches exactly as many kernels."""
    import dataclasses

    sys.path.insert(0, ROOT)
    import bench
    import workloads

    w = workloads.WORKLOADS["context_parallel_causal"]
    # Balanced causal, 4 ranks (8 chunks): rank r's chunks r and 7 - r see r + 1 and
    # 8 - r key chunks; every chunk with more than one partial is merged (all but chunk 0).
    assert bench.ring_launches_per_step(w, 4) == 36 + 7
    assert bench.ring_launches_per_step(w, 1) == 3 + 1
    assert bench.ring_launches_per_step(w, 2) == 10 + 3
    wc = dataclasses.replace(w, balanced=False)
    assert bench.ring_launches_per_step(wc, 4) == 13  # partials 1 + 2 + 3 + 4, merges on ranks 1-3
    for world in (2, 4, 8):
        for ww in (dataclasses.replace(w, shards=world), dataclasses.replace(wc, shards=world)):
            import torch as _t  # noqa: F401  (the emulated plan is built without a device here)
            _, plans = bench.context_parallel_plan(ww)
            from tiled_exact_attention_forward_b200 import context_parallel as cpm
            want = 0
            for r, p in enumerate(plans):
                counts = [0] * len(cpm.rank_chunks(r, world, ww.balanced))
                for st in p:
                    for q_ in st.partials:
                        counts[q_.q_chunk] += 1
                want += sum(counts) + sum(c > 1 for c in counts)
            assert bench.ring_launches_per_step(ww, world) == want
