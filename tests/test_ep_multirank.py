"""The host side of expert parallelism across processes, on CPU: two gloo ranks
(world_size 2) exchange their window handles through ep.exchange_windows, which checks
that every rank agrees on the shapes that fix the window layout before any peer mapping
would be opened, and map the windows through ep.map_windows with a fake of the mapping
call.  Failures are made on the host (a refused mapping, a missing handle): every rank
must raise together and unmap what it mapped.  (The real CUDA IPC mapping runs in
test_gpu_ep_ipc.py; the device side of the EP layer in test_gpu_ep.py.)"""
import os
import sys

import torch.multiprocessing as mp

from tests.ports import free_port

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
    world, port = 2, free_port()
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


def _map_rank(rank, world, port, out, case):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from dispatch_combine_grouped_b200 import ep
    from moe_inputs import small_config
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        closed = []

        def open_fn(hb, o):  # a fake of the mapping call: rank 1 cannot map
            if case == "open" and rank == 1:
                raise OSError("mapping refused")
            return 1000 * (hb[0]) + o

        try:
            if case == "handle":
                cfg = small_config("ep_host", N=64, d=128, E=8, S=1, k=2, I=64, P=2)
                ep.exchange_windows(cfg, 128, rank, None if rank == 0 else b"x" * 64, 0,
                                    error="rank 0: no handle" if rank == 0 else None)
                out[rank] = ("ok", None)
            else:
                table = [(bytes([1]) * 64, 0), (bytes([2]) * 64, 256)]
                ptrs, opened = ep.map_windows(table, rank, 7, open_fn, lambda p, o: closed.append(p))
                out[rank] = ("ok", ptrs)
        except RuntimeError as e:
            out[rank] = ("error", str(e), closed)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run_map(case):
    world, port = 2, free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_map_rank, args=(world, port, out, case), nprocs=world, join=True)
        return dict(out)


def test_window_mapping_succeeds_in_rank_order():
    res = _run_map("none")
    assert res[0] == ("ok", [7, 2256]) and res[1] == ("ok", [1000, 7])


def test_a_failed_mapping_makes_every_rank_raise_and_unmap():
    res = _run_map("open")
    for r in range(2):
        assert res[r][0] == "error" and "rank 1 could not map the window of rank 0" in res[r][1]
    assert res[0][2] == [2256]   # rank 0 had mapped rank 1's window and unmapped it
    assert res[1][2] == []


def test_a_missing_handle_makes_every_rank_raise():
    res = _run_map("handle")
    for r in range(2):
        assert res[r][0] == "error" and "rank 0: no handle" in res[r][1]
