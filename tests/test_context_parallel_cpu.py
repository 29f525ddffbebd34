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


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_ring_schedule_covers_every_shard_once(world):
    Ns = 8
    for rank, (causal, window) in itertools.product(range(world), MASKS):
        sched = cp.ring_schedule(rank, world, Ns, causal, window)
        assert [s.step for s in sched] == list(range(world))
        assert sorted(s.shard for s in sched) == list(range(world))
        assert sched[0].shard == rank and sched[0].q_offset == 0 and sched[0].visible
        for s in sched:
            assert s.q_offset == (rank - s.shard) * Ns
            if causal:
                # Shards after this rank's queries are never computed.
                assert s.visible == (s.shard <= rank and
                                     (window <= 0 or (rank - s.shard) * Ns <= Ns + window - 2))


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


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, Ns, d = 2, 2, 11, 4
        N = Ns * world
        g = torch.Generator().manual_seed(7)
        q, k, v = (torch.randn((B, H, N, d), generator=g, dtype=torch.float64) for _ in range(3))
        sl = slice(rank * Ns, (rank + 1) * Ns)
        ring = cp.RingForward(_oracle_partial, _oracle_merge)
        errs = []
        for causal, window in MASKS:
            o, lse = ring(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                          causal, window, 0.5)
            O_ref, lse_ref = oracle.attention_forward(q, k, v, 0.5, causal, window)
            errs.append((float(np.abs(o.numpy() - O_ref[:, :, sl]).max()),
                         float(np.abs(lse.numpy() - lse_ref[:, :, sl]).max())))
        tdist.barrier()
        out[rank] = errs
    finally:
        tdist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_forward_gloo_matches_full_forward(world):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
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
    """The key-shard partials of all ranks cover each visible (query, key) pair of
    the whole sequence exactly once, so the ring's work is the full forward's."""
    import dataclasses

    sys.path.insert(0, ROOT)
    import bench
    import workloads

    w0 = workloads.WORKLOADS["context_parallel_causal"]
    assert (w0.N, w0.shards, w0.causal) == (16384, 4, True)
    Ns, plans = bench.context_parallel_plan(w0)
    assert Ns == 4096 and [len(p) for p in plans] == [1, 2, 3, 4]
    for causal, window in MASKS + [(True, 70), (False, 0)]:
        w = dataclasses.replace(w0, N=96, shards=4, causal=causal, window=window)
        Ns, plans = bench.context_parallel_plan(w)
        total = 0
        for r, plan in enumerate(plans):
            for st in plan:
                ok = oracle.allowed_mask(Ns, Ns, causal, window, q_pos=np.arange(Ns) + st.q_offset)
                total += int(ok.sum())
        assert total == bench.allowed_pairs(96, causal, window), (causal, window)


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
    # Causal, 4 shards: partials 1 + 2 + 3 + 4, merges on ranks 1-3.
    assert bench.ring_launches_per_step(w, 4) == 13
    assert bench.ring_launches_per_step(w, 1) == 1
    assert bench.ring_launches_per_step(w, 2) == 4
    for world in (2, 4, 8):
        ww = dataclasses.replace(w, shards=world)
        _, plans = bench.context_parallel_plan(ww)
        assert bench.ring_launches_per_step(w, world) == \
            sum(len(p) for p in plans) + sum(len(p) > 1 for p in plans)
