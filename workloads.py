"""Seeded synthetic inputs for the attention workloads.

This module holds shapes, seeds and random draws only -- none of the
attention arithmetic.  Both sides of every parity check (the float64 oracle
and the CUDA library) read tensors made here, so a result never depends on
which side generated its own inputs.

Recipe: a ``torch.Generator`` seeded with the workload's seed draws, in order,
q, k, v (and dO for the backward) as float32 standard normals, which are then
rounded to the workload's dtype.  The decode workload first draws its
per-sequence cache lengths from a CPU generator (uniform integers in
[lo, hi]), then q and the two caches; the paged decode workload draws the same
lengths, a random placement of the blocks in the pool (CPU generator, seed + 1),
then q and the two pools.  Draws on a CUDA device use torch's CUDA
generator with the same seed; those values differ from the CPU stream, which
does not matter because both sides read the same tensors.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BF16 = torch.bfloat16
FP32 = torch.float32


@dataclass(frozen=True)
class Workload:
    """One named attention workload (shapes, masks, dtype, seed)."""

    name: str
    kind: str            # "forward", "decode", "paged_decode", "forward_backward" or "context_parallel"
    B: int
    H: int
    N: int               # sequence length (decode: cache capacity)
    d: int
    dtype: torch.dtype
    seed: int
    causal: bool = False
    window: int = 0
    seqlen_lo: int = 0   # decode only: per-sequence cache length range
    seqlen_hi: int = 0
    block_size: int = 0  # paged decode only: rows per cache block
    shards: int = 0      # context parallel only: sequence shards (ranks of the ring)
    balanced: bool = False  # context parallel only: rank r holds chunks r and 2 shards - 1 - r
    parts: int = 0       # merge only: partial results merged per row
    notes: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("single_head_fp32", "forward", 1, 1, 128, 64, FP32, 0,
                 notes="single-head fp32 forward, non-causal"),
        Workload("causal_prefill", "forward", 4, 16, 2048, 128, BF16, 1, causal=True,
                 notes="causal prefill forward, bf16 in / fp32 accumulate"),
        Workload("sliding_window_long", "forward", 1, 32, 16384, 128, BF16, 2,
                 causal=True, window=4096,
                 notes="long-context causal sliding window (i-4096 < j <= i)"),
        Workload("kv_cache_decode", "decode", 64, 32, 8192, 128, BF16, 3,
                 seqlen_lo=512, seqlen_hi=8192,
                 notes="single-token decode, padded cache capacity 8192"),
        Workload("causal_fwd_bwd", "forward_backward", 2, 16, 4096, 128, BF16, 4,
                 causal=True, notes="causal forward + recompute backward"),
        Workload("causal_prefill_fp16", "forward", 4, 16, 2048, 128, torch.float16, 1, causal=True,
                 notes="the causal prefill forward with float16 inputs"),
        Workload("paged_kv_decode", "paged_decode", 64, 32, 8192, 128, BF16, 3,
                 seqlen_lo=512, seqlen_hi=8192, block_size=16,
                 notes="single-token decode against a paged cache: 16-row blocks, "
                       "shuffled in one pool, the lengths of kv_cache_decode"),
        Workload("merge_parts_2", "merge", 1, 32, 16384, 128, BF16, 6, parts=2,
                 notes="merge of 2 partial results per row (the context-parallel combine), "
                       "524288 rows of d = 128"),
        Workload("merge_parts_4", "merge", 1, 16, 16384, 128, BF16, 6, parts=4,
                 notes="merge of 4 partial results per row, 262144 rows of d = 128"),
        Workload("merge_parts_8", "merge", 1, 8, 16384, 128, BF16, 6, parts=8,
                 notes="merge of 8 partial results per row, 131072 rows of d = 128"),
        Workload("merge_parts_4_fp32", "merge", 1, 16, 16384, 128, FP32, 6, parts=4,
                 notes="merge of 4 float32 partial results per row, 262144 rows of d = 128"),
        Workload("context_parallel_causal", "context_parallel", 1, 32, 16384, 128, BF16, 5,
                 causal=True, shards=4, balanced=True,
                 notes="causal forward of a 16K context over 4 ring ranks, each holding sequence "
                       "chunks r and 7 - r of 8 (equal causal work per rank); on one GPU every "
                       "rank's ring steps (key-chunk partials, then the merges) run in turn"),
    ]
}


def _gen(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    return g


def randn(shape, dtype, gen: torch.Generator, device) -> torch.Tensor:
    """float32 N(0,1) draw rounded to ``dtype`` (round-to-nearest-even)."""
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def forward_inputs(B, H, N, d, dtype=BF16, seed=0, device="cpu", with_dout=False):
    """q, k, v (and dO) of shape [B, H, N, d], contiguous, i.i.d. N(0,1)."""
    g = _gen(seed, device)
    q = randn((B, H, N, d), dtype, g, device)
    k = randn((B, H, N, d), dtype, g, device)
    v = randn((B, H, N, d), dtype, g, device)
    if with_dout:
        dO = randn((B, H, N, d), dtype, g, device)
        return q, k, v, dO
    return q, k, v


def decode_seqlens(B, lo, hi, seed) -> torch.Tensor:
    """Per-sequence cache lengths, uniform integers in [lo, hi] (int32, CPU)."""
    g = _gen(seed, "cpu")
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def decode_inputs(B, H, cap, d, lo, hi, dtype=BF16, seed=0, device="cpu",
                  pad_value: float | None = None):
    """q [B,H,d], kcache/vcache [B,H,cap,d], seqlens [B] (int32, on ``device``).

    Cache rows at positions >= seqlens[b] are also random unless ``pad_value``
    is given, in which case they are filled with it (NaN makes any read past a
    sequence's length visible in the output).
    """
    seqlens = decode_seqlens(B, lo, hi, seed)
    g = _gen(seed, device)
    q = randn((B, H, d), dtype, g, device)
    kc = torch.empty((B, H, cap, d), dtype=dtype, device=device)
    vc = torch.empty((B, H, cap, d), dtype=dtype, device=device)
    for b in range(B):  # per sequence, to bound the float32 staging buffer
        kc[b] = randn((H, cap, d), dtype, g, device)
        vc[b] = randn((H, cap, d), dtype, g, device)
    if pad_value is not None:
        for b in range(B):
            n = int(seqlens[b])
            kc[b, :, n:] = pad_value
            vc[b, :, n:] = pad_value
    return q, kc, vc, seqlens.to(device)


def paged_decode_inputs(B, H, block_size, max_blocks, d, lo, hi, dtype=BF16, seed=0, device="cpu",
                        pad_value: float | None = None):
    """q [B,H,d], kpool/vpool [num_blocks,H,block_size,d], block_table [B,max_blocks]
    and seqlens [B] (int32, on ``device``).

    Sequence b holds ceil(seqlens[b] / block_size) blocks; all sequences' blocks
    are placed in one pool in a seeded random order (as a long-running cache
    fragments), and the table maps each logical block to its place.  Table
    entries past a sequence's blocks are -1.  Pool rows past a sequence's length
    (the tail of its last block) are random unless ``pad_value`` is given.
    """
    seqlens = decode_seqlens(B, lo, hi, seed)
    nblk = [(int(n) + block_size - 1) // block_size for n in seqlens]
    if max(nblk) > max_blocks:
        raise ValueError("a sequence needs more than max_blocks blocks")
    num_blocks = max(1, sum(nblk))
    perm = torch.randperm(num_blocks, generator=_gen(seed + 1, "cpu"))
    table = torch.full((B, max_blocks), -1, dtype=torch.int32)
    first = 0
    for b in range(B):
        table[b, :nblk[b]] = perm[first:first + nblk[b]].to(torch.int32)
        first += nblk[b]
    g = _gen(seed, device)
    q = randn((B, H, d), dtype, g, device)
    kpool = randn((num_blocks, H, block_size, d), dtype, g, device)
    vpool = randn((num_blocks, H, block_size, d), dtype, g, device)
    if pad_value is not None:
        for b in range(B):
            n = int(seqlens[b])
            if n % block_size:
                last = int(table[b, nblk[b] - 1])
                kpool[last, :, n % block_size:] = pad_value
                vpool[last, :, n % block_size:] = pad_value
    return q, kpool, vpool, table.to(device), seqlens.to(device)


def merge_inputs(S, B, H, N, d, dtype=BF16, seed=0, device="cpu"):
    """o_parts [S, B, H, N, d] (N(0,1) rounded to dtype) and lse_parts [S, B, H, N]
    float32 (3 N(0,1), so the parts' weights differ widely)."""
    g = _gen(seed, device)
    o_parts = randn((S, B, H, N, d), dtype, g, device)
    lse_parts = randn((S, B, H, N), torch.float32, g, device) * 3.0
    return o_parts, lse_parts


def workload_inputs(w: Workload, device="cpu", **kw):
    """Inputs of a named workload at its full size."""
    if w.kind == "decode":
        return decode_inputs(w.B, w.H, w.N, w.d, w.seqlen_lo, w.seqlen_hi, w.dtype,
                             w.seed, device, **kw)
    if w.kind == "merge":
        return merge_inputs(w.parts, w.B, w.H, w.N, w.d, w.dtype, w.seed, device)
    if w.kind == "paged_decode":
        return paged_decode_inputs(w.B, w.H, w.block_size, w.N // w.block_size, w.d, w.seqlen_lo,
                                   w.seqlen_hi, w.dtype, w.seed, device, **kw)
    return forward_inputs(w.B, w.H, w.N, w.d, w.dtype, w.seed, device,
                          with_dout=(w.kind == "forward_backward"))

