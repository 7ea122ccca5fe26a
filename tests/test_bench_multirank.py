"""The bench's multi-rank path on CPU: two gloo ranks (world_size 2) check the max-over-
ranks timing and the whole-job rate, and that the reference arm prints only on rank 0."""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from tests.ports import free_port

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]                 # rank 1 is the slower one
        slowest = bench.max_over_ranks(local_ms, world)
        out[rank] = (slowest, bench.whole_job_tokens_per_s(4096, world, slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world, port = 2, free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        slowest, rate = res[r]
        assert slowest == 5.0
        assert rate == pytest.approx(2 * 4096 / 5e-3)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.whole_job_tokens_per_s(100, 1, 10.0) == pytest.approx(1e4)


def test_reference_arm_silent_on_nonzero_rank():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
