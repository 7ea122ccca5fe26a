"""The host side of expert parallelism across processes, on CPU: two gloo ranks
(world_size 2) exchange their window handles through ep.exchange_windows, which checks
that every rank agrees on the shapes that fix the window layout before any peer mapping
would be opened.  (Opening CUDA IPC mappings needs two GPUs; the device side of the EP
layer is covered by the one-device emulation in test_gpu_ep.py.)"""
import os
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out, case):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from dispatch_combine_grouped_b200 import ep
    from moe_inputs import small_config
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        P = 3 if case == "world" else 2
        cfg = small_config("ep_host", N=64, d=128, E=8, S=1, k=2, I=64, P=P)
        cap = 128 + (rank if case == "capacity" else 0)
        handle = bytes([rank + 1]) * 64  # stands in for a CUDA IPC handle
        try:
            out[rank] = ("ok", ep.exchange_windows(cfg, cap, rank, handle, 256 * rank))
        except ValueError as e:
            out[rank] = ("error", str(e))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(case):
    world, port = 2, 29617 + os.getpid() % 1000 + hash(case) % 50
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out, case), nprocs=world, join=True)
        return dict(out)


def test_window_handles_gathered_in_rank_order():
    res = _run("agree")
    for r in range(2):
        kind, table = res[r]
        assert kind == "ok"
        assert table == [(bytes([1]) * 64, 0), (bytes([2]) * 64, 256)]


def test_ranks_that_disagree_on_capacity_both_refuse():
    res = _run("capacity")
    for r in range(2):
        kind, msg = res[r]
        assert kind == "error" and "capacity" in msg


def test_group_size_must_equal_P():
    res = _run("world")
    for r in range(2):
        kind, msg = res[r]
        assert kind == "error" and "P = 3" in msg
