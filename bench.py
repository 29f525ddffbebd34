"""Benchmark of the tiled exact attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one pass of the hot path over one batch of synthetic input:
  causal_prefill (default): fa_forward on B=4, H=16, N=2048, d=128, bf16, causal
  sliding_window_long:      fa_forward on B=1, H=32, N=16384, d=128, window 4096
  kv_cache_decode:          fa_decode, batch 64 x 32 heads, cache lengths U[512, 8192]
  paged_kv_decode:          fa_decode_paged, the same lengths in shuffled 16-row blocks of one pool
  causal_fwd_bwd:           fa_forward + fa_backward on B=2, H=16, N=4096, d=128
Inputs are seeded N(0,1) draws (``workloads.py``), resident in HBM before the
timed region.  The L2 (126 MB) is flushed between timed steps by writing a
256 MiB buffer outside the timed events.  Throughput counts only the (query,
key) pairs the mask allows: 4*d FLOPs per pair forward, 10*d backward;
decode counts the bytes of the K/V rows it must read plus q and o (paged: plus
the block-table entries it uses).

Prints one JSON line (rank 0).  With --gpus N > 1 each rank runs its own
independent batch (weak scaling, no collective on the data path); value = all
ranks' work / the slowest rank's time.  Launched without torchrun, --gpus N > 1
starts the N ranks itself through torch.distributed.run; it stops with an error
(exit 2, no result line) when fewer than N GPUs are visible or when --gpus
differs from the launcher's WORLD_SIZE.

--impl reference times the float64 CPU oracle (the only other
implementation of this method) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
_CPU_THREADS = str(os.cpu_count() or 1)
for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_v, _CPU_THREADS)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------- work counts
def allowed_pairs(N: int, causal: bool, window: int) -> int:
    """(query, key) pairs one head's mask allows, in closed form per row."""
    i = np.arange(N, dtype=np.int64)
    hi = i + 1 if causal else np.full(N, N, dtype=np.int64)
    lo = np.maximum(0, i - window + 1) if window > 0 else np.zeros(N, dtype=np.int64)
    return int(np.maximum(0, hi - lo).sum())


def forward_flops(w) -> float:
    return 4.0 * w.d * allowed_pairs(w.N, w.causal, w.window) * w.B * w.H


def backward_flops(w) -> float:
    return 10.0 * w.d * allowed_pairs(w.N, w.causal, w.window) * w.B * w.H


DECODE_KINDS = ("decode", "paged_decode")
BYTE_KINDS = DECODE_KINDS + ("merge",)  # workloads measured in GB/s against copy bandwidth


def merge_row_bytes(w) -> int:
    """Bytes per merged row: every part's O row and lse, the merged row and lse."""
    es = torch.finfo(w.dtype).bits // 8
    return w.parts * (es * w.d + 4) + es * w.d + 4


def merge_bytes(w) -> float:
    """Bytes one merge reads and writes."""
    return float(w.B * w.H * w.N) * merge_row_bytes(w)


def decode_bytes(w, seqlens) -> float:
    n = np.minimum(np.asarray(seqlens, dtype=np.int64), w.N)
    rows = float(n.sum()) * w.H
    table = 4.0 * float((-(-n // w.block_size)).sum()) if w.kind == "paged_decode" else 0.0
    return rows * w.d * 2 * 2 + 2 * w.B * w.H * w.d * 2 + table  # K + V rows, q + o, table


def dtype_name(dtype) -> str:
    """The arithmetic input type of a workload as the bench line names it."""
    return {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}[dtype]


# ----------------------------------------------------------------------------- measurement helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def source_hash(names):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tiled_exact_attention_forward_b200", "csrc")
    for n in sorted(names):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, sources):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary (profiles/dram_traffic.json), if its kernel source is current."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_hash") != source_hash(sources):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile

            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.path is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        smax = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] > 0.5 * smax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, s in enumerate(r[2]) if s.lower() == "active"})
        return {"sm_mhz": float(np.median([r[0] for r in loaded])), "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


def cpu_threads_used():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        n = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else int(_CPU_THREADS)
    except Exception:  # noqa: BLE001
        return int(_CPU_THREADS)


def cpu_model() -> str:
    """The host CPU's model name (Linux), or the platform's processor string."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


# ----------------------------------------------------------------------------- oracle (CPU) timing
def oracle_sample(w, budget_s=12.0):
    """Time the float64 oracle on whole heads of the workload until ~budget_s.

    Returns (value in the workload's unit, sample description)."""
    import oracle

    gen = torch.Generator().manual_seed(w.seed)
    t_total, units, heads = 0.0, 0.0, 0
    while t_total < budget_s and heads < w.B * w.H:
        if w.kind == "decode":
            n = int(workloads.decode_seqlens(w.B, w.seqlen_lo, w.seqlen_hi, w.seed)[heads % w.B])
            q = torch.randn(1, 1, w.d, generator=gen).to(w.dtype)
            kc = torch.randn(1, 1, n, w.d, generator=gen).to(w.dtype)
            vc = torch.randn(1, 1, n, w.d, generator=gen).to(w.dtype)
            t0 = time.perf_counter()
            oracle.decode_forward(q, kc, vc, np.array([n]), w.scale)
            t_total += time.perf_counter() - t0
            units += n * w.d * 2 * 2 + 2 * w.d * 2
        elif w.kind == "merge":
            rows = 4096
            o_p = torch.randn((w.parts, rows, w.d), generator=gen).to(w.dtype)
            l_p = torch.randn((w.parts, rows), generator=gen) * 3.0
            t0 = time.perf_counter()
            oracle.merge_partials(o_p, l_p)
            t_total += time.perf_counter() - t0
            units += rows * merge_row_bytes(w)
        elif w.kind == "paged_decode":
            n = int(workloads.decode_seqlens(w.B, w.seqlen_lo, w.seqlen_hi, w.seed)[heads % w.B])
            nb = -(-n // w.block_size)
            q = torch.randn(1, 1, w.d, generator=gen).to(w.dtype)
            kp = torch.randn(nb, 1, w.block_size, w.d, generator=gen).to(w.dtype)
            vp = torch.randn(nb, 1, w.block_size, w.d, generator=gen).to(w.dtype)
            table = torch.randperm(nb, generator=gen).reshape(1, nb)
            t0 = time.perf_counter()
            oracle.decode_paged_forward(q, kp, vp, table, np.array([n]), w.scale)
            t_total += time.perf_counter() - t0
            units += n * w.d * 2 * 2 + 2 * w.d * 2 + 4 * nb
        else:
            q, k, v = (torch.randn(w.N, w.d, generator=gen).to(w.dtype) for _ in range(3))
            t0 = time.perf_counter()
            o, lse = oracle.attention_forward(q, k, v, w.scale, w.causal, w.window)
            if w.kind == "forward_backward":
                oracle.attention_backward(q, k, v, torch.randn(w.N, w.d, generator=gen).to(w.dtype),
                                          w.scale, w.causal, w.window)
            t_total += time.perf_counter() - t0
            per = 4.0 * w.d * allowed_pairs(w.N, w.causal, w.window)
            if w.kind == "forward_backward":
                per *= 3.5
            units += per
        heads += 1
    rate = units / t_total
    if w.kind == "merge":
        return rate / 1e9, f"{heads} blocks of 4096 rows x {w.parts} parts (float64), {t_total:.1f} s"
    if w.kind in DECODE_KINDS:
        return rate / 1e9, f"{heads} of {w.B * w.H} (sequence, head) decodes, {t_total:.1f} s"
    return rate / 1e12, f"{heads} of {w.B * w.H} heads (full N x N float64 per head), {t_total:.1f} s"


# ----------------------------------------------------------------------------- GPU arm
# What the roofline's duration covers, per workload kind, and (for a step of several
# launches whose dominant kernel can be timed on its own call) that call and its units.
ROOF_TIMED = {
    "forward": "the fwd_tc_kernel launch (one per step)",
    "forward_backward": "one fa_backward call (bwd_pre, bwd_main, bwd_post), timed apart from the forward",
    "decode": "one fa_decode call (split and combine kernels)",
    "paged_decode": "one fa_decode_paged call (split and combine kernels)",
    "merge": "the merge_kernel launch (one per step)",
    "context_parallel": "the whole ring step (every key-chunk partial and merge)",
}
ROOF_CALL = {}  # kind -> (callable, units per call), filled by make_step


def make_step(w, dev, rank=0, world=1):
    """Returns (step_fn, e2e_fn, units_per_step, unit, metric, launches_per_step, kernel, sources).

    units and launches are this rank's share: the whole job is world x units."""
    import tiled_exact_attention_forward_b200 as fa

    if w.kind == "paged_decode":
        q, kp, vp, table, seqlens = workloads.workload_inputs(w, device=dev)
        ws = torch.empty(fa.decode_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H), dtype=torch.float32, device=dev)
        units = decode_bytes(w, seqlens.cpu().numpy()) / 1e9

        def step():
            fa.decode_paged(q, kp, vp, table, seqlens, w.scale, workspace=ws, out=o, lse=lse)

        # End to end: the step's own inputs (new query, lengths, block table) go up and
        # the output comes back; the block pool stays resident as it would in serving.
        q_h, s_h, t_h = (t.cpu().pin_memory() for t in (q, seqlens, table))
        o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        l_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

        def e2e():
            q.copy_(q_h, non_blocking=True)
            seqlens.copy_(s_h, non_blocking=True)
            table.copy_(t_h, non_blocking=True)
            fa.decode_paged(q, kp, vp, table, seqlens, w.scale, workspace=ws, out=o, lse=lse)
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)

        h2d = sum(t.numel() * t.element_size() for t in (q_h, s_h, t_h))
        d2h = o_h.numel() * o_h.element_size() + l_h.numel() * 4
        return (step, e2e, units, "GB/s", "decode GB/s", 2, "decode_split_kernel",
                ["decode.cu", "common.cuh", "kernels.h"], h2d, d2h)

    if w.kind == "merge":
        o_parts, lse_parts = workloads.workload_inputs(w, device=dev)
        o = torch.empty(o_parts.shape[1:], dtype=o_parts.dtype, device=dev)
        lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=dev)

        def step():
            fa.merge(o_parts, lse_parts, out=o, lse=lse)

        # End to end: the parts go up, the merged rows and lse come back.
        h_in = [t.cpu().pin_memory() for t in (o_parts, lse_parts)]
        h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, lse)]

        def e2e():
            o_parts.copy_(h_in[0], non_blocking=True)
            lse_parts.copy_(h_in[1], non_blocking=True)
            fa.merge(o_parts, lse_parts, out=o, lse=lse)
            h_out[0].copy_(o, non_blocking=True)
            h_out[1].copy_(lse, non_blocking=True)

        h2d = sum(t.numel() * t.element_size() for t in h_in)
        d2h = sum(t.numel() * t.element_size() for t in h_out)
        return (step, e2e, merge_bytes(w) / 1e9, "GB/s", "merge GB/s", 1, "merge_kernel",
                ["merge.cu", "common.cuh", "kernels.h"], h2d, d2h)

    if w.kind == "decode":
        q, kc, vc, seqlens = workloads.workload_inputs(w, device=dev)
        ws = torch.empty(fa.decode_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H), dtype=torch.float32, device=dev)
        units = decode_bytes(w, seqlens.cpu().numpy()) / 1e9

        def step():
            fa.decode(q, kc, vc, seqlens, w.scale, workspace=ws, out=o, lse=lse)

        # End to end: a decode step's own inputs (the new query and the lengths) go up,
        # the output comes back; the cache stays resident as it would in serving.
        q_h = q.cpu().pin_memory()
        s_h = seqlens.cpu().pin_memory()
        o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        l_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

        def e2e():
            q.copy_(q_h, non_blocking=True)
            seqlens.copy_(s_h, non_blocking=True)
            fa.decode(q, kc, vc, seqlens, w.scale, workspace=ws, out=o, lse=lse)
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)

        h2d = q_h.numel() * q_h.element_size() + s_h.numel() * 4
        d2h = o_h.numel() * o_h.element_size() + l_h.numel() * 4
        return (step, e2e, units, "GB/s", "decode GB/s", 2, "decode_split_kernel",
                ["decode.cu", "common.cuh", "kernels.h"], h2d, d2h)

    if w.kind == "context_parallel":
        if world > 1:
            return _ring_step(w, dev, fa, rank, world)
        return _context_parallel_step(w, dev, fa)

    with_bwd = w.kind == "forward_backward"
    ins = workloads.workload_inputs(w, device=dev)
    q, k, v = ins[:3]
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    flops = forward_flops(w) + (backward_flops(w) if with_bwd else 0.0)
    if with_bwd:
        dO = ins[3]
        ws = torch.empty(fa.backward_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def step():
        fa.forward(q, k, v, w.causal, w.window, w.scale, out=o, lse=lse)
        if with_bwd:
            fa.backward(q, k, v, o, dO, lse, w.causal, w.window, w.scale, workspace=ws, dq=dq, dk=dk, dv=dv)

    if with_bwd:
        def bwd_only():
            fa.backward(q, k, v, o, dO, lse, w.causal, w.window, w.scale, workspace=ws, dq=dq, dk=dk, dv=dv)

        ROOF_CALL["forward_backward"] = (bwd_only, backward_flops(w) / 1e12)

    host_in = [t.cpu().pin_memory() for t in ins]
    outs = [o, lse] + ([dq, dk, dv] if with_bwd else [])
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]

    # The public host-buffer calls: copies in, kernels and copies out pipelined over
    # head groups; each returns once the results are in host memory.
    if with_bwd:
        def e2e():
            fa.forward_backward_host(*host_in[:4], w.causal, w.window, w.scale, device=dev)
    else:
        def e2e():
            fa.forward_host(*host_in[:3], w.causal, w.window, w.scale, device=dev)

    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    metric = "attention TFLOP/s (fwd+bwd, unmasked FLOPs)" if with_bwd else \
        "attention TFLOP/s (fwd, unmasked FLOPs)"
    return (step, e2e, flops / 1e12, "TFLOP/s", metric, 4 if with_bwd else 1,
            "bwd_main_kernel" if with_bwd else "fwd_tc_kernel",
            ["bwd.cu" if with_bwd else "fwd_tc.cu", "common.cuh", "kernels.h"], h2d, d2h)


def context_parallel_plan(w, world=None):
    """Per rank of the ring: its steps with the visible key-chunk partials.

    Returns (chunk length, plans) with plans[r] the ring_schedule of rank r."""
    from tiled_exact_attention_forward_b200 import context_parallel as cp

    world = world or w.shards
    m = cp.n_chunks(world, w.balanced)
    if w.N % m:
        raise ValueError(f"{w.name}: N = {w.N} does not split into {m} equal chunks")
    C = w.N // m
    return C, [cp.ring_schedule(r, world, C, w.causal, w.window, w.balanced) for r in range(world)]


def ring_launches_per_step(w, world: int) -> int:
    """Kernel launches of the whole job per ring step: every rank's visible key-chunk
    partials plus one merge per query chunk that has more than one partial."""
    from tiled_exact_attention_forward_b200 import context_parallel as cp

    _, plans = context_parallel_plan(w, world)
    total = 0
    for r, plan in enumerate(plans):
        counts = [0] * len(cp.rank_chunks(r, world, w.balanced))
        for st in plan:
            for p in st.partials:
                counts[p.q_chunk] += 1
        total += sum(counts) + sum(c > 1 for c in counts)
    return total


def context_parallel_emulated(w, dev, fa):
    """All ranks of the ring on one device: each rank's chunks of q, k, v, the
    key-chunk partials it computes and the merges.  The exchange itself (NCCL
    send/receive between GPUs) is not part of it: one GPU has no peer.
    Returns (step, inputs (q, k, v chunk lists), results (o, lse chunk lists), launches)."""
    from tiled_exact_attention_forward_b200 import context_parallel as cp

    q, k, v = workloads.workload_inputs(w, device=dev)
    C, plans = context_parallel_plan(w)
    m = cp.n_chunks(w.shards, w.balanced)
    cut = [[t[:, :, a * C:(a + 1) * C].contiguous() for a in range(m)] for t in (q, k, v)]
    del q, k, v
    qs, ks, vs = cut
    jobs = []  # per (rank, local query chunk): the list of (key chunk, q_offset)
    for r, plan in enumerate(plans):
        mine = cp.rank_chunks(r, w.shards, w.balanced)
        for qi, a in enumerate(mine):
            parts = [(cp.rank_chunks(st.shard, w.shards, w.balanced)[p.k_chunk], p.q_offset)
                     for st in plan for p in st.partials if p.q_chunk == qi]
            jobs.append((a, parts))
    jobs.sort(key=lambda job: job[0])  # results in sequence order: chunk a of every rank
    o_parts = [torch.empty((len(p), w.B, w.H, C, w.d), dtype=w.dtype, device=dev) for _, p in jobs]
    l_parts = [torch.empty((len(p), w.B, w.H, C), dtype=torch.float32, device=dev) for _, p in jobs]
    outs = [torch.empty_like(qs[a]) if len(p) > 1 else o_parts[i][0] for i, (a, p) in enumerate(jobs)]
    lses = [torch.empty((w.B, w.H, C), dtype=torch.float32, device=dev) if len(p) > 1 else l_parts[i][0]
            for i, (a, p) in enumerate(jobs)]

    def step():
        for i, (a, parts) in enumerate(jobs):
            for n, (c, off) in enumerate(parts):
                fa.forward_offset(qs[a], ks[c], vs[c], off, w.causal, w.window, w.scale,
                                  out=o_parts[i][n], lse=l_parts[i][n])
            if len(parts) > 1:
                fa.merge(o_parts[i], l_parts[i], out=outs[i], lse=lses[i])

    launches = sum(len(p) + (len(p) > 1) for _, p in jobs)
    return step, (qs, ks, vs), (outs, lses), launches


def _context_parallel_step(w, dev, fa):
    step, (qs, ks, vs), (outs, lses), launches = context_parallel_emulated(w, dev, fa)
    host_in = [t.cpu().pin_memory() for t in qs + ks + vs]
    dev_in = qs + ks + vs
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs + lses]
    dev_out = outs + lses

    # End to end: every rank's chunks go up from pinned host memory, the ring steps
    # run, and every rank's output rows and lse come back.
    def e2e():
        for d_, h_ in zip(dev_in, host_in):
            d_.copy_(h_, non_blocking=True)
        step()
        for h_, d_ in zip(host_out, dev_out):
            h_.copy_(d_, non_blocking=True)
        torch.cuda.current_stream(dev).synchronize()

    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    return (step, e2e, forward_flops(w) / 1e12, "TFLOP/s", "attention TFLOP/s (fwd, unmasked FLOPs)",
            launches, "fwd_tc_kernel", ["fwd_tc.cu", "common.cuh", "kernels.h"], h2d, d2h)


def _ring_step(w, dev, fa, rank, world):
    """The context-parallel ring across the ranks of the job: the sequence is cut
    into chunks, rank r holds its chunks of q, k and v (r, or r and 2 world - 1 - r
    for the balanced layout), and each step is one context_parallel_forward
    (key-chunk partials, NCCL exchange of the K/V shards around the ring, merges).
    Every rank draws the same seeded full inputs and keeps its own rows.  The total
    work is the whole sequence's, whatever `world` is."""
    from tiled_exact_attention_forward_b200 import context_parallel as cp

    q, k, v = workloads.workload_inputs(w, device=dev)
    qs, ks, vs = (cp.shard_rows(t, rank, world, w.balanced).contiguous() for t in (q, k, v))
    del q, k, v
    out = {}

    def step():
        out["o"], out["lse"] = cp.context_parallel_forward(qs, ks, vs, w.causal, w.window, w.scale,
                                                           balanced=w.balanced)

    host_in = [t.cpu().pin_memory() for t in (qs, ks, vs)]
    step()
    torch.cuda.synchronize(dev)
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (out["o"], out["lse"])]

    # End to end: this rank's rows go up from pinned host memory, the ring runs, and
    # its output rows and lse come back.
    def e2e():
        for d_, h_ in zip((qs, ks, vs), host_in):
            d_.copy_(h_, non_blocking=True)
        step()
        for h_, d_ in zip(host_out, (out["o"], out["lse"])):
            h_.copy_(d_, non_blocking=True)
        torch.cuda.current_stream(dev).synchronize()

    # Launches of the whole job per step, shared evenly (the line reports world x this).
    launches = ring_launches_per_step(w, world) / world
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    return (step, e2e, forward_flops(w) / 1e12 / world, "TFLOP/s", "attention TFLOP/s (fwd, unmasked FLOPs)",
            launches, "fwd_tc_kernel", ["fwd_tc.cu", "common.cuh", "kernels.h"], h2d, d2h)


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank values (the slowest rank sets the time)."""
    import torch.distributed as tdist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Work of all ranks (weak scaling: each rank its own batch) per second."""
    return units_per_rank * world / (ms / 1e3)


def timed_loop(fn, steps, warmup, flush, stream):
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    # `warmup` untimed steps (with their flushes) queued directly ahead of the timed
    # ones: the GPU is busy, at its working clocks, when the first timed step starts.
    # (After the idle gap of starting the clock sampler, the first step measured about
    # twice the others.)
    for _ in range(warmup):
        flush.add_(1)
        fn()
    for i in range(steps):
        flush.add_(1)  # 256 MiB write: evicts the previous step's data from L2 (not timed)
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def run_gpu(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    import tiled_exact_attention_forward_b200 as fa

    fa.library()
    w = resolve_workload(args)
    (step, e2e, units, unit, metric, launches, kernel, sources, h2d, d2h) = make_step(w, dev, rank, world)
    ring = w.kind == "context_parallel" and world > 1
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    dist = world > 1
    if dist:
        import torch.distributed as tdist

    def barrier():
        if dist:
            tdist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    with ClockSampler(local_rank) as clk:
        times = timed_loop(step, args.steps, 2, flush, stream)
    barrier()
    if fa.device_status(dev) != fa.FA_OK:
        raise RuntimeError("a kernel reported a device-side timeout")
    ms = float(np.mean(times))
    e2e_times = timed_loop(e2e, max(3, args.steps // 2), 2, flush, stream)
    barrier()
    e2e_ms = float(np.mean(e2e_times))
    if dist:
        ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)
    value = whole_job_rate(units, world, ms)
    e2e_value = whole_job_rate(units, world, e2e_ms)
    hbm, tflops, peak_kind = load_peaks()
    roof_units, roof_ms = units, ms
    if w.kind in ROOF_CALL:
        # The dominant kernel's own call, timed like the steps (L2 flushed between
        # calls); its inputs are the last timed step's.
        fn, roof_units = ROOF_CALL[w.kind]
        roof_ms = float(np.mean(timed_loop(fn, args.steps, 2, flush, stream)))
        barrier()
        if dist:
            roof_ms = max_over_ranks([roof_ms], device=dev)[0]
    if unit == "GB/s":
        roof = {"bound": "hbm", "achieved": roof_units / (roof_ms / 1e3), "peak": hbm, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": roof_units / (roof_ms / 1e3), "peak": tflops, "unit": "TFLOP/s"}
    roof["timed"] = ROOF_TIMED.get(w.kind, "the step")
    roof["ms"] = roof_ms
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = f"{peak_kind} ({'copy bandwidth' if unit == 'GB/s' else 'cuBLAS bf16 burst'})"
    roof["kernel"] = kernel
    roof["traffic"] = profiled_traffic(kernel, w.name, sources)
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms,
        "ms_per_step_spread": {"p50": float(np.median(times)), "min": float(np.min(times)),
                               "max": float(np.max(times))},
        "higher_is_better": True, "scaling": "strong" if ring else "weak",
        "vs_baseline": None, "dtype": dtype_name(w.dtype), "data": "synthetic (seeded N(0,1), workloads.py)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                   "window": w.window, "global_batch": w.B if ring else w.B * world, "seq_len": w.N,
                   "parallelism": (f"context-parallel ring x{world}" if ring else
                                   f"replicas x{world}" if world > 1 else "single GPU"),
                   "l2": "flushed between timed steps (256 MiB write, untimed)",
                   **({"block_size": w.block_size} if w.block_size else {}),
                   **({"shards": world, "layout": "balanced" if w.balanced else "contiguous",
                       "ring": "one shard per GPU, NCCL exchange inside the timed steps"}
                      if ring else
                      {"shards": w.shards, "layout": "balanced" if w.balanced else "contiguous",
                       "ring": "every rank's steps on one GPU, exchange not timed"}
                      if w.shards else {})},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(round(launches * (world if ring else 1) * args.steps)),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample = oracle_sample(w)
        line["cpu_baseline"] = {"value": v, "unit": unit, "cores": cpu_threads_used(), "kind": "oracle",
                                "sample": sample, "cpu": cpu_model()}
    return line


def resolve_workload(args):
    """The named workload, with the batch/head overrides used for small profiling runs."""
    import dataclasses

    w = workloads.WORKLOADS[args.workload]
    changes = {k: v for k, v in (("B", args.B), ("H", args.H)) if v is not None}
    return dataclasses.replace(w, **changes) if changes else w


def run_reference(args):
    w = resolve_workload(args)
    t0 = time.perf_counter()
    vals = []
    samples = []
    for i in range(args.warmup + args.steps):
        v, sample = oracle_sample(w, budget_s=args.ref_budget)
        if i >= args.warmup:
            vals.append(v)
            samples.append(sample)
    unit = "GB/s" if w.kind in BYTE_KINDS else "TFLOP/s"
    value = float(np.mean(vals))
    metric = {"decode": "decode GB/s", "paged_decode": "decode GB/s", "merge": "merge GB/s",
              "forward_backward": "attention TFLOP/s (fwd+bwd, unmasked FLOPs)"} \
        .get(w.kind, "attention TFLOP/s (fwd, unmasked FLOPs)")
    return {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1))",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                   "window": w.window,
                   **({"block_size": w.block_size} if w.block_size else {}),
                   **({"shards": w.shards, "layout": "balanced" if w.balanced else "contiguous",
                       "ring": "the oracle takes the whole sequence at once (same result)"}
                      if w.shards else {})},
        "cpu_baseline": {"kind": "oracle", "value": value, "unit": unit, "cores": cpu_threads_used(),
                         "sample": samples[-1] if samples else "", "cpu": cpu_model()},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t0,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="causal_prefill", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=4.0)
    ap.add_argument("--B", type=int, default=None, help="override the workload's batch (profiling)")
    ap.add_argument("--H", type=int, default=None, help="override the workload's heads (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    launched = "WORLD_SIZE" in os.environ

    if args.impl == "reference":
        # The CPU oracle runs on rank 0 only; other ranks exit without work.
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    problem = launch_problem(args.gpus, world if launched else None, gpu_count())
    if problem:
        print(f"bench.py: {problem}", file=sys.stderr, flush=True)
        return 2
    if not launched and args.gpus > 1:
        # One process per GPU: start the ranks ourselves (the same command line).
        return subprocess.call(torchrun_command(args.gpus, sys.argv[1:]))

    if world > 1:
        import datetime

        import torch.distributed as tdist

        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    try:
        line = run_gpu(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as tdist

            tdist.destroy_process_group()
    return 0


def gpu_count() -> int:
    return torch.cuda.device_count() if torch.cuda.is_available() else 0


def launch_problem(gpus: int, world_env, n_devices: int):
    """Why this launch cannot run (a message), or None.

    gpus: --gpus; world_env: WORLD_SIZE when launched by torchrun, else None;
    n_devices: CUDA devices visible to this process."""
    if gpus < 1:
        return f"--gpus must be >= 1, got {gpus}"
    if world_env is not None and world_env != gpus:
        return f"--gpus {gpus} does not match the launcher's WORLD_SIZE {world_env}"
    if world_env is None and gpus > n_devices:
        return f"--gpus {gpus} needs {gpus} CUDA devices, {n_devices} visible"
    return None


def torchrun_command(gpus: int, argv):
    """The command that runs this script once per GPU on this node."""
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


if __name__ == "__main__":
    sys.exit(main())
