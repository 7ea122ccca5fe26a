"""The CUDA IPC window mapping of the expert-parallel path (moe_ep_ipc_handle / _open /
_close, ep.ipc_group), with two processes on one GPU.

Rank 1 maps rank 0's window through CUDA IPC and runs only kernels that wait for
nothing: the count exchange (moe_ep_notify) and the dispatch (moe_ep_dispatch, with
destinations computed on the host from the oracle's EP layout).  The host orders the
two processes with gloo barriers after device synchronisation, so no kernel ever waits
on another process's kernel.  Rank 0 then checks, in its own window, the count row,
the received rows, gates and flags that rank 1 stored through the mapping.
"""
import os
import sys

import pytest
import torch.multiprocessing as mp

from tests.ports import free_port

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def _proc(rank, port, out):
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from dispatch_combine_grouped_b200 import ep
    import dispatch_combine_grouped_b200 as moe
    from moe_inputs import make_inputs, small_config
    from oracle import moe_oracle as O

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2)
    torch.cuda.set_device(0)
    try:
        cfg = small_config("ep_ipc", cfg_id=120, N=256, d=256, E=8, S=0, k=2, I=64, P=2)
        n = cfg.N // 2
        rc = cfg.replace(N=n)
        cap = cfg.N * cfg.k
        inp = make_inputs(cfg, device="cuda", with_experts=False)
        xs = [inp["x"][r * n:(r + 1) * n] for r in range(2)]
        routed = [moe.route(rc, xs[r], inp["w_gate"], inp["bias"]) for r in range(2)]
        ids = [rt[1] for rt in routed]
        lay = O.ep_layout([i.cpu().numpy() for i in ids], cfg.E, cfg.P, None, cap)
        window = ep.alloc_window(rc, cap)
        torch.cuda.synchronize()
        dist.barrier()
        grp, close = ep.ipc_group(rc, cap, window)
        assert grp.windows[rank] == window.data_ptr()
        dist.barrier()
        if rank == 1:
            ws = ep.alloc_ws(rc, cap)
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            ep.notify(rc, grp, ids[1], ws, status)              # count row 1 into both windows
            h = ep.Handle(rc, grp.local_experts)
            h.dest[:n * cfg.k].copy_(torch.from_numpy(lay["dest"][1].astype(np.int32)))
            ep.dispatch(rc, grp, xs[1], routed[1][2], h)        # rows into both windows
            torch.cuda.synchronize()
            out["status1"] = int(status.item())
        dist.barrier()
        if rank == 0:
            v = ep.window_views(rc, cap, window)
            want = np.bincount(ids[1].cpu().numpy().reshape(-1), minlength=cfg.E)
            res = {"cnt_row": bool(np.array_equal(v["cnt_tab"][1].cpu().numpy(), want)),
                   "cnt_flag": int(v["cnt_flag"][1].item()), "disp_flag": int(v["disp_flag"][1].item()),
                   "own_step": int(v["step"].item())}
            rows_ok = True
            for row, (i, a) in enumerate(lay["recv"][0]):
                if i != 1:
                    continue
                rows_ok &= bool(torch.equal(v["x_recv"][row], xs[1][a // cfg.k]))
                rows_ok &= bool(v["gate"][row].item() == routed[1][2].reshape(-1)[a].item())
            res["rows"] = rows_ok
            res["n_rows_from_1"] = int((lay["recv"][0][:, 0] == 1).sum()) if len(lay["recv"][0]) else 0
            out["rank0"] = res
        dist.barrier()
        close()
        torch.cuda.synchronize()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ipc_mapped_window_receives_counts_and_rows():
    port = free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_proc, args=(port, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res["status1"] == 0
    r0 = res["rank0"]
    assert r0["cnt_row"], "count row stored through the IPC mapping"
    assert r0["cnt_flag"] == 1 and r0["disp_flag"] == 1, r0
    assert r0["own_step"] == 0, "rank 0 ran no step"
    assert r0["n_rows_from_1"] > 0 and r0["rows"], "received rows and gates stored through the IPC mapping"
