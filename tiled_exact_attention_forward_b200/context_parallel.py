"""Context-parallel (ring) attention forward over torch.distributed ranks.

Both pure-Python kernel pages end with a roadmap that splits attention across
devices so the context can outgrow one device's memory ("Build a
FlashAttention-2 Inference Kernel from Scratch in Pure Python", Extending It:
distributed tensor parallelism; "Build a FlashAttention Kernel with Online
Softmax and KV Cache in Pure Python", Extending It: horizontal scaling, each
worker holding part of the key/value space).  No page says how; the readings
taken here:

* The sequence is cut into equal chunks of C rows.  In the contiguous layout
  there are `world` chunks and rank r holds chunk r.  In the balanced layout
  there are 2 world chunks and rank r holds chunks r and 2 world - 1 - r (in
  that order): under a causal mask every rank then has the same number of
  visible (query, key) pairs, where the contiguous layout gives rank r work in
  proportion to r + 1/2.
* A rank's chunks of K and V form its shard, which travels once around the
  ring (rank r sends to r + 1 and receives from r - 1); at step t rank r holds
  the shard of rank s = (r - t) mod world.  A shard is passed on only while some
  rank further along the ring still sees a key of it.
* Each (query chunk, key chunk) pair with a visible key gives one partial
  (O, lse) from the key-shard forward, its query offset being the distance
  between the two chunks' first positions.  The partials of a query chunk merge
  with the identity of "Building Flash Attention from Scratch in Pure NumPy"
  (architecture overview):
      lse = ln sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.

The exchange of step t + 1 is posted before the compute of step t, so the
transfer runs (on the communication library's own stream) while the tensor
cores work; the result for each rank's own query rows is exact, whatever the
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


def rank_chunks(rank: int, world: int, balanced: bool) -> tuple[int, ...]:
    """Sequence chunks held by `rank`, in the order of its local rows."""
    return (rank, 2 * world - 1 - rank) if balanced else (rank,)


def n_chunks(world: int, balanced: bool) -> int:
    return 2 * world if balanced else world


@dataclass(frozen=True)
class Partial:
    q_chunk: int   # index into this rank's chunks
    k_chunk: int   # index into the held shard's chunks
    q_offset: int  # first query position minus first key position


@dataclass(frozen=True)
class RingStep:
    step: int                        # 0 .. world - 1
    shard: int                       # rank whose key/value shard is held (-1: none)
    partials: tuple[Partial, ...]    # visible (query chunk, key chunk) pairs
    send: bool                       # pass the held shard on to rank + 1
    recv: bool                       # receive the next shard from rank - 1

    @property
    def visible(self) -> bool:
        return bool(self.partials)


def _partials(rank: int, shard: int, world: int, chunk: int, causal: bool, window: int,
              balanced: bool) -> tuple[Partial, ...]:
    out = []
    for qi, a in enumerate(rank_chunks(rank, world, balanced)):
        for ki, c in enumerate(rank_chunks(shard, world, balanced)):
            off = (a - c) * chunk
            if visible(chunk, chunk, off, causal, window):
                out.append(Partial(qi, ki, off))
    return tuple(out)


def _sees(rank: int, shard: int, world: int, chunk: int, causal: bool, window: int, balanced: bool) -> bool:
    return bool(_partials(rank, shard, world, chunk, causal, window, balanced))


def ring_schedule(rank: int, world: int, chunk: int, causal: bool, window: int,
                  balanced: bool = False) -> list[RingStep]:
    """What rank `rank` holds, computes, sends and receives at each ring step.

    Every rank evaluates the same predicate for each hand-over (does any rank
    still ahead of the shard see it?), so sender and receiver always agree."""
    def forwarded(holder: int, s: int, t: int) -> bool:
        # After step t the shard moves on; ranks holder + 1 .. holder + (world - 1 - t)
        # would still get it.
        return any(_sees((holder + u) % world, s, world, chunk, causal, window, balanced)
                   for u in range(1, world - t))

    out = []
    holding = True  # rank holds its own shard at step 0
    for t in range(world):
        s = (rank - t) % world
        held = s if holding else -1
        parts = _partials(rank, s, world, chunk, causal, window, balanced) if holding else ()
        send = holding and t + 1 < world and forwarded(rank, s, t)
        s_next = (rank - t - 1) % world
        recv = t + 1 < world and forwarded((rank - 1) % world, s_next, t)
        out.append(RingStep(t, held, parts, send, recv))
        holding = recv
    return out


def shard_rows(x: torch.Tensor, rank: int, world: int, balanced: bool) -> torch.Tensor:
    """The rows of a full-sequence tensor [..., N, d] that rank `rank` holds, in its
    local order (N must split into the layout's chunks)."""
    n = x.shape[-2]
    m = n_chunks(world, balanced)
    if n % m:
        raise ValueError(f"sequence length {n} does not split into {m} equal chunks")
    c = n // m
    return torch.cat([x[..., a * c:(a + 1) * c, :] for a in rank_chunks(rank, world, balanced)], dim=-2)


def _peer(group, r: int) -> int:
    return r if group is None else dist.get_global_rank(group, r)


class RingForward:
    """Ring attention over the ranks of `group` (the default group if None).

    partial(q, k, v, q_offset, causal, window, scale, out, lse) writes one key
    chunk's normalised output and row logsumexp into `out` and `lse`;
    merge(o_parts, lse_parts) returns the merged (o, lse).  With balanced=True
    each rank holds chunks r and 2 world - 1 - r of the sequence (see the module
    docstring); otherwise chunk r.
    """

    def __init__(self, partial, merge, group=None, balanced: bool = False):
        self.partial = partial
        self.merge = merge
        self.group = group
        self.balanced = balanced

    def __call__(self, q, k, v, causal: bool = False, window: int = 0, scale=None):
        if q.shape != k.shape or q.shape != v.shape:
            raise ValueError("each rank holds equal-length shards: q, k, v of one shape [B, H, Ns, d]")
        if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
            # Checked before the first exchange is posted: a peer may already be waiting on it.
            raise ValueError("q, k, v must be contiguous")
        world = dist.get_world_size(self.group) if dist.is_initialized() else 1
        rank = dist.get_rank(self.group) if dist.is_initialized() else 0
        B, H, Ns, d = q.shape
        nloc = len(rank_chunks(rank, world, self.balanced))
        if Ns % nloc:
            raise ValueError(f"a shard of {Ns} rows does not split into {nloc} equal chunks")
        C = Ns // nloc
        sched = ring_schedule(rank, world, C, causal, window, self.balanced)

        def split(x):
            return [x[:, :, i * C:(i + 1) * C].contiguous() for i in range(nloc)] if nloc > 1 else [x]

        qs = split(q)
        counts = [0] * nloc
        for st in sched:
            for p in st.partials:
                counts[p.q_chunk] += 1
        o_parts = [torch.empty((max(n, 1), B, H, C, d), dtype=q.dtype, device=q.device) for n in counts]
        lse_parts = [torch.empty((max(n, 1), B, H, C), dtype=torch.float32, device=q.device) for n in counts]
        used = [0] * nloc
        cur = split(k) + split(v)  # this rank's K chunks, then its V chunks
        for st in sched:
            pending = None
            if st.send or st.recv:
                # Post the next exchange before this step's compute.
                ops, nxt = [], None
                if st.send:
                    ops += [dist.P2POp(dist.isend, t, _peer(self.group, (rank + 1) % world), self.group)
                            for t in cur]
                if st.recv:
                    nxt = [torch.empty((B, H, C, d), dtype=q.dtype, device=q.device) for _ in range(2 * nloc)]
                    ops += [dist.P2POp(dist.irecv, t, _peer(self.group, (rank - 1) % world), self.group)
                            for t in nxt]
                pending = (nxt, dist.batch_isend_irecv(ops))
            for p in st.partials:
                i = used[p.q_chunk]
                self.partial(qs[p.q_chunk], cur[p.k_chunk], cur[nloc + p.k_chunk], p.q_offset, causal, window,
                             scale, o_parts[p.q_chunk][i], lse_parts[p.q_chunk][i])
                used[p.q_chunk] += 1
            if pending is not None:
                for req in pending[1]:
                    req.wait()
                cur = pending[0] if pending[0] is not None else cur
        outs, lses = [], []
        for c in range(nloc):
            if counts[c] == 0:  # no visible key at all (cannot happen for a self-attention mask)
                outs.append(torch.zeros((B, H, C, d), dtype=q.dtype, device=q.device))
                lses.append(torch.full((B, H, C), float("-inf"), dtype=torch.float32, device=q.device))
            elif counts[c] == 1:
                outs.append(o_parts[c][0])
                lses.append(lse_parts[c][0])
            else:
                o_c, l_c = self.merge(o_parts[c], lse_parts[c])
                outs.append(o_c)
                lses.append(l_c)
        if nloc == 1:
            return outs[0], lses[0]
        return torch.cat(outs, dim=2), torch.cat(lses, dim=2)


def _cuda_partial(q, k, v, q_offset, causal, window, scale, out, lse):
    from . import forward_offset

    forward_offset(q, k, v, q_offset, causal=causal, window=window, scale=scale, out=out, lse=lse)


def _cuda_merge(o_parts, lse_parts):
    from . import merge

    return merge(o_parts, lse_parts)


def context_parallel_forward(q, k, v, causal: bool = False, window: int = 0, scale=None, group=None,
                             balanced: bool = False):
    """The attention of this rank's query rows over the whole sequence.

    q, k, v: this rank's rows [B, H, Ns, d] (bf16 or fp16, d = 128) on its CUDA
    device -- chunk r of `world` (balanced=False) or chunks r and 2 world - 1 - r
    of 2 world, concatenated (balanced=True; see ``shard_rows``).  Returns
    (o, lse) for the local query rows, in the same order.  The exchange uses the
    process group's backend (NCCL over NVLink between GPUs); every partial and
    the merge run in the CUDA library.  With no process group (or one rank)
    this is the plain forward.
    """
    return RingForward(_cuda_partial, _cuda_merge, group, balanced)(q, k, v, causal, window, scale)
