"""The seeded input recipe and the benchmark's JSON contract (CPU only)."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_forward_inputs_are_seeded_and_shaped():
    a = workloads.forward_inputs(2, 3, 17, 128, torch.bfloat16, seed=5, with_dout=True)
    b = workloads.forward_inputs(2, 3, 17, 128, torch.bfloat16, seed=5, with_dout=True)
    c = workloads.forward_inputs(2, 3, 17, 128, torch.bfloat16, seed=6, with_dout=True)
    for x, y in zip(a, b):
        assert x.shape == (2, 3, 17, 128) and x.dtype == torch.bfloat16 and x.is_contiguous()
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])
    # q, k, v, dO are four different draws, each roughly N(0, 1).
    assert not torch.equal(a[0], a[1])
    x = a[0].float()
    assert abs(float(x.mean())) < 0.05 and abs(float(x.std()) - 1.0) < 0.05


def test_decode_inputs_lengths_and_padding():
    q, kc, vc, lens = workloads.decode_inputs(5, 2, 300, 128, 1, 300, seed=3, pad_value=float("nan"))
    assert q.shape == (5, 2, 128) and kc.shape == (5, 2, 300, 128) and lens.dtype == torch.int32
    for b in range(5):
        n = int(lens[b])
        assert 1 <= n <= 300
        assert torch.isfinite(kc[b, :, :n].float()).all()
        assert torch.isnan(kc[b, :, n:].float()).all()


def test_decode_workload_lengths_match_the_recorded_draw():
    w = workloads.WORKLOADS["kv_cache_decode"]
    lens = workloads.decode_seqlens(w.B, w.seqlen_lo, w.seqlen_hi, w.seed)
    assert lens.shape == (64,) and int(lens.min()) >= 512 and int(lens.max()) <= 8192
    assert int(lens.sum()) == 264373  # the seed-3 draw every decode number here is quoted on


def test_paged_decode_inputs_place_every_block_once():
    q, kp, vp, table, lens = workloads.paged_decode_inputs(5, 2, 16, 20, 128, 1, 300, seed=3,
                                                           pad_value=float("nan"))
    nblk = [(int(n) + 15) // 16 for n in lens]
    assert kp.shape == (sum(nblk), 2, 16, 128) and table.shape == (5, 20) and table.dtype == torch.int32
    used = torch.cat([table[b, :nblk[b]] for b in range(5)])
    assert sorted(used.tolist()) == list(range(sum(nblk)))      # a permutation of the pool
    for b in range(5):
        assert (table[b, nblk[b]:] == -1).all()
        n = int(lens[b])
        for t in range(nblk[b]):
            blk = kp[int(table[b, t])].float()
            rows = min(16, n - 16 * t)
            assert torch.isfinite(blk[:, :rows]).all() and torch.isnan(blk[:, rows:]).all()
    # Same lengths as the padded-cache decode workload draws.
    w = workloads.WORKLOADS["paged_kv_decode"]
    assert torch.equal(workloads.decode_seqlens(w.B, w.seqlen_lo, w.seqlen_hi, w.seed),
                       workloads.decode_seqlens(64, 512, 8192, 3))


def test_named_workloads():
    W = workloads.WORKLOADS
    assert (W["single_head_fp32"].N, W["single_head_fp32"].d, W["single_head_fp32"].dtype) == (128, 64, torch.float32)
    assert (W["causal_prefill"].B, W["causal_prefill"].H, W["causal_prefill"].N) == (4, 16, 2048)
    assert (W["sliding_window_long"].N, W["sliding_window_long"].window) == (16384, 4096)
    assert (W["causal_fwd_bwd"].B, W["causal_fwd_bwd"].N, W["causal_fwd_bwd"].kind) == (2, 4096, "forward_backward")


def test_flop_counts_match_closed_forms():
    sys.path.insert(0, ROOT)
    import bench

    # causal: N (N + 1) / 2 visible pairs; window w: sum_i min(i + 1, w).
    assert bench.allowed_pairs(2048, True, 0) == 2048 * 2049 // 2
    assert bench.allowed_pairs(16384, True, 4096) == sum(min(i + 1, 4096) for i in range(16384))
    assert bench.allowed_pairs(100, False, 0) == 100 * 100
    # window without causal: only the left bound j > i - w applies.
    assert bench.allowed_pairs(100, False, 7) == sum(100 - max(0, i - 6) for i in range(100))
    w = workloads.WORKLOADS["causal_prefill"]
    assert bench.forward_flops(w) == pytest.approx(68.753031168e9)
    # Decode bytes: K and V rows (256 B each per head) + q + o; paged adds 4 B per used block.
    wd, wp = workloads.WORKLOADS["kv_cache_decode"], workloads.WORKLOADS["paged_kv_decode"]
    lens = np.array([512, 8192, 1000])
    base = lens.sum() * 32 * 128 * 2 * 2 + 2 * 64 * 32 * 128 * 2
    assert bench.decode_bytes(wd, lens) == base
    assert bench.decode_bytes(wp, lens) == base + 4 * (32 + 512 + 63)
    # Merge bytes per row: S parts of d values and an lse, plus the merged row and lse.
    rows = 16 * 16384
    assert bench.merge_bytes(workloads.WORKLOADS["merge_parts_4"]) == rows * (4 * (256 + 4) + 260)
    assert bench.merge_bytes(workloads.WORKLOADS["merge_parts_4_fp32"]) == rows * (4 * (512 + 4) + 516)


@pytest.mark.parametrize("workload,unit", [("single_head_fp32", "TFLOP/s"), ("paged_kv_decode", "GB/s")])
def test_reference_arm_prints_one_json_line(workload, unit):
    env = dict(os.environ)
    env.pop("RANK", None)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-budget", "0.5", "--workload", workload],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "cpu_baseline",
                "e2e", "config"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == unit
    assert d["config"]["workload"] == workload
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert np.isfinite(d["value"])


def test_bench_line_names_the_workload_dtype():
    import bench

    W = workloads.WORKLOADS
    assert bench.dtype_name(W["causal_prefill"].dtype) == "bf16"
    assert bench.dtype_name(W["causal_prefill_fp16"].dtype) == "f16"
    assert bench.dtype_name(W["single_head_fp32"].dtype) == "f32"


def test_bench_launch_checks():
    import bench

    assert "needs 1 CUDA devices" in bench.launch_problem(1, None, 0)
    assert bench.launch_problem(2, None, 8) is None
    assert bench.launch_problem(2, 2, 8) is None
    assert "WORLD_SIZE" in bench.launch_problem(2, 3, 8)
    assert "needs 2 CUDA devices" in bench.launch_problem(2, None, 1)
    assert bench.launch_problem(0, None, 8) is not None
    cmd = bench.torchrun_command(4, ["--gpus", "4", "--steps", "2"])
    assert cmd[1:3] == ["-m", "torch.distributed.run"] and "--nproc-per-node=4" in cmd
    assert "--master-addr=127.0.0.1" in cmd and cmd[-3:] == ["4", "--steps", "2"]


def test_bench_multi_gpu_request_without_gpus_fails_cleanly():
    """On a machine without enough GPUs, --gpus 2 must not print a one-GPU result."""
    import subprocess
    import sys

    import torch

    if torch.cuda.is_available() and torch.cuda.device_count() >= 2:
        pytest.skip("this machine has two GPUs")
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 2, (r.returncode, r.stderr[-2000:])
    assert r.stdout.strip() == ""
    assert "needs 2 CUDA devices" in r.stderr
