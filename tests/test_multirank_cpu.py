"""The multi-rank host logic of the benchmark, as world-size-2 gloo ranks on CPU.

With several GPUs each rank times its own independent batch (no collective on
the data path); the only cross-rank steps are the barrier and the max of the
per-rank times.  Those run here without a GPU.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as tdist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [1.0 + rank, 10.0 - 3 * rank]   # rank 1 is slower in the first entry
        got = bench.max_over_ranks(ms)
        tdist.barrier()
        out[rank] = got + [bench.whole_job_rate(2.0, world, got[0])]
    finally:
        tdist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        assert res[r][:2] == [2.0, 10.0]
        assert res[r][2] == pytest.approx(2.0 * 2 / 2e-3)


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
