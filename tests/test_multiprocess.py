"""The N>1 host logic of bench.py, with world-size-2 gloo ranks on CPU.

On GPUs every rank runs its own replica batch and NCCL carries only the
timing maximum and the byte/token sums; the same code runs here over gloo.
"""

import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r: 10*(r+1) ms for 1e9*(r+1) bytes and 100*(r+1) tokens
        res = bench.combine_over_ranks(10.0 * (rank + 1), 1e9 * (rank + 1), 100 * (rank + 1),
                                       "cpu")
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_combine_over_ranks_gloo_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        results = dict(out)
    for rank in range(world):
        max_ms, gbs, tps = results[rank]
        assert max_ms == 20.0                      # the slowest rank's time
        assert gbs == pytest.approx(3e9 / 0.020 / 1e9)   # all ranks' bytes over it
        assert tps == pytest.approx(300 / 0.020)


def test_combine_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    max_ms, gbs, tps = bench.combine_over_ranks(4.0, 8e9, 64, "cpu")
    assert (max_ms, gbs, tps) == (4.0, pytest.approx(2000.0), pytest.approx(16000.0))


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--steps", "3", "--warmup", "1"], env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip() == ""


def test_reference_arm_rank0_prints_the_contract_line():
    """Rank 0 of the reference arm (the fp64 oracle on host cores) prints one
    JSON line with the keys the bench contract asks of that arm."""
    import json

    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                         text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "mixed_2048"
