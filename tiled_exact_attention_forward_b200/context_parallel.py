"""Context-parallel (ring) attention forward over torch.distributed ranks.

Both pure-Python kernel pages end with a roadmap that splits attention across
devices so the context can outgrow one device's memory ("Build a
FlashAttention-2 Inference Kernel from Scratch in Pure Python", Extending It:
distributed tensor parallelism; "Build a FlashAttention Kernel with Online
Softmax and KV Cache in Pure Python", Extending It: horizontal scaling, each
worker holding part of the key/value space).  Reading taken here: the
sequence is cut into `world` contiguous shards of equal length Ns; rank r
holds rows [r Ns, (r + 1) Ns) of Q, K and V for every head.  The key/value
shards travel once around the ring (rank r sends to r + 1 and receives from
r - 1), and at step t rank r holds the keys of shard s = (r - t) mod world,
whose first key sits (r - s) Ns positions before its first query.  Each
visible shard gives one partial (O_s, lse_s) from the key-shard forward; the
partials merge with the identity of "Building Flash Attention from Scratch in
Pure NumPy" (architecture overview):
    lse = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.

The exchange of step t + 1 is posted before the compute of step t, so the
transfer runs (on the communication library's own stream) while the tensor
cores work; the result for each rank's own query shard is exact, whatever the
order in which the shards arrive.

The compute is passed in as two callables, so the same driver runs with the
CUDA library (``context_parallel_forward``) and, in the CPU tests, with any
other implementation of the same two functions.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


def visible(n_q: int, n_k: int, q_offset: int, causal: bool, window: int) -> bool:
    """Does any of n_q query rows (row i at position i + q_offset) see any of
    keys 0 .. n_k - 1 under the mask (causal: j <= p; window w > 0: j > p - w)?"""
    if n_q < 1 or n_k < 1:
        return False
    # Rows whose window still reaches key n_k - 1 or earlier: p - w + 1 <= n_k - 1.
    last_row = n_q - 1 if window <= 0 else min(n_q - 1, n_k + window - 2 - q_offset)
    # Rows that see key 0 or later under causality: p >= 0.
    first_row = max(0, -q_offset) if causal else 0
    return first_row <= last_row


@dataclass(frozen=True)
class RingStep:
    step: int      # 0 .. world - 1
    shard: int     # key/value shard held at this step
    q_offset: int  # first query position minus first key position
    visible: bool  # does any query of this rank see any key of the shard


def ring_schedule(rank: int, world: int, shard_len: int, causal: bool, window: int) -> list[RingStep]:
    """The shards rank `rank` holds, step by step, and which of them it computes."""
    out = []
    for t in range(world):
        s = (rank - t) % world
        off = (rank - s) * shard_len
        out.append(RingStep(t, s, off, visible(shard_len, shard_len, off, causal, window)))
    return out


def _peer(group, r: int) -> int:
    return r if group is None else dist.get_global_rank(group, r)


class RingForward:
    """Ring attention over the ranks of `group` (the default group if None).

    partial(q, k, v, q_offset, causal, window, scale, out, lse) writes one key
    shard's normalised output and row logsumexp into `out` and `lse`;
    merge(o_parts, lse_parts) returns the merged (o, lse).
    """

    def __init__(self, partial, merge, group=None):
        self.partial = partial
        self.merge = merge
        self.group = group

    def __call__(self, q, k, v, causal: bool = False, window: int = 0, scale=None):
        if q.shape != k.shape or q.shape != v.shape:
            raise ValueError("each rank holds equal-length shards: q, k, v of one shape [B, H, Ns, d]")
        if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
            # Checked before the first exchange is posted: a peer may already be waiting on it.
            raise ValueError("q, k, v must be contiguous")
        world = dist.get_world_size(self.group) if dist.is_initialized() else 1
        rank = dist.get_rank(self.group) if dist.is_initialized() else 0
        B, H, Ns, d = q.shape
        sched = ring_schedule(rank, world, Ns, causal, window)
        n_parts = sum(st.visible for st in sched)
        o_parts = torch.empty((n_parts, B, H, Ns, d), dtype=q.dtype, device=q.device)
        lse_parts = torch.empty((n_parts, B, H, Ns), dtype=torch.float32, device=q.device)
        cur = (k, v)
        i = 0
        for st in sched:
            pending = None
            if st.step + 1 < world:
                # Post the next exchange before this step's compute.
                nxt = tuple(torch.empty_like(t) for t in cur)
                ops = [dist.P2POp(dist.isend, t, _peer(self.group, (rank + 1) % world), self.group)
                       for t in cur]
                ops += [dist.P2POp(dist.irecv, t, _peer(self.group, (rank - 1) % world), self.group)
                        for t in nxt]
                pending = (nxt, dist.batch_isend_irecv(ops))
            if st.visible:
                self.partial(q, cur[0], cur[1], st.q_offset, causal, window, scale,
                             o_parts[i], lse_parts[i])
                i += 1
            if pending is not None:
                for req in pending[1]:
                    req.wait()
                cur = pending[0]
        if n_parts == 1:
            return o_parts[0], lse_parts[0]
        return self.merge(o_parts, lse_parts)


def _cuda_partial(q, k, v, q_offset, causal, window, scale, out, lse):
    from . import forward_offset

    forward_offset(q, k, v, q_offset, causal=causal, window=window, scale=scale, out=out, lse=lse)


def _cuda_merge(o_parts, lse_parts):
    from . import merge

    return merge(o_parts, lse_parts)


def context_parallel_forward(q, k, v, causal: bool = False, window: int = 0, scale=None, group=None):
    """The attention of this rank's query shard over the whole sequence.

    q, k, v: this rank's shard [B, H, Ns, d] (bf16 or fp16, d = 128) on its CUDA
    device; the ranks of `group` hold consecutive shards in rank order.  Returns
    (o, lse) for the local query rows.  The exchange uses the process group's
    backend (NCCL over NVLink between GPUs); every partial and the merge run in
    the CUDA library.  With no process group (or one rank) this is the plain
    forward.
    """
    return RingForward(_cuda_partial, _cuda_merge, group)(q, k, v, causal, window, scale)
