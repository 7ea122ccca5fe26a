"""Expert parallelism across GPUs: binding of libmoe's moe_ep_* calls (include/moe.h).

Argument marshalling only: every step of the EP layer runs in libmoe's kernels.  What
this module adds is the plumbing around them:
  - windows: one device buffer per rank, mapped into every other rank's address space
    (``ipc_group``: CUDA IPC handles exchanged over a torch.distributed process group),
    or, for P ranks emulated on one device, P buffers of one process (``emulated_groups``);
  - host-side checks that every rank agrees on the shapes that fix the window layout.

The EP layer follows the ep_deepep explainer §2-3 (each rank is a source of tokens and
the owner of some experts; dispatch to the owners, combine back to the sources) and the
DeepEP notes §2-3 (counts first, then the all-to-all as a transpose).
"""
from __future__ import annotations

import ctypes

import torch

from . import binding as B

N_OFFSETS = 11
OFFSET_NAMES = ["cnt_flag", "disp_flag", "done_flag", "step", "disp_ctr", "err_step", "cnt_tab", "gate", "scale",
                "x_recv", "out_recv"]
MAX_RANKS = 32


def owned_experts(E: int, P: int, rank: int, expert_owner=None) -> list[int]:
    """Experts rank ``rank`` owns, ascending: expert_owner[e] == rank, or e // (E / P)."""
    if expert_owner is None:
        per = E // P
        return list(range(rank * per, (rank + 1) * per))
    owner = [int(v) for v in (expert_owner.tolist() if hasattr(expert_owner, "tolist") else expert_owner)]
    return [e for e in range(E) if owner[e] == rank]


def window_bytes(cfg, capacity: int) -> int:
    c = B.c_config(cfg)
    return B.load().moe_ep_window_bytes(ctypes.byref(c), capacity)


def workspace_bytes(cfg, capacity: int) -> int:
    c = B.c_config(cfg)
    return B.load().moe_ep_workspace_bytes(ctypes.byref(c), capacity)


def window_offsets(cfg, capacity: int) -> dict:
    c = B.c_config(cfg)
    arr = (ctypes.c_size_t * N_OFFSETS)()
    B._check(B.load().moe_ep_window_layout(ctypes.byref(c), capacity, arr), "moe_ep_window_layout")
    return dict(zip(OFFSET_NAMES, [int(v) for v in arr]))


def alloc_window(cfg, capacity: int, device="cuda") -> torch.Tensor:
    """A zeroed window for this rank (uint8; torch allocations are 512-byte aligned)."""
    nbytes = window_bytes(cfg, capacity)
    if nbytes == 0:
        B.check_config(cfg)
        raise ValueError("capacity must be >= 1")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def window_views(cfg, capacity: int, window: torch.Tensor) -> dict:
    """Tensor views of a window's parts (for inspection)."""
    o = window_offsets(cfg, capacity)
    dt = B._dtype(cfg)
    eb = torch.empty(0, dtype=dt).element_size()
    P, E, d, S, N = cfg.P, cfg.E, cfg.d, cfg.S, cfg.N

    def view(off, n, dtype):
        es = torch.empty(0, dtype=dtype).element_size()
        return window[off:off + n * es].view(dtype)

    return dict(cnt_flag=view(o["cnt_flag"], MAX_RANKS, torch.int64),
                disp_flag=view(o["disp_flag"], MAX_RANKS, torch.int64),
                done_flag=view(o["done_flag"], MAX_RANKS, torch.int64),
                step=view(o["step"], 1, torch.int64),
                err_step=view(o["err_step"], 1, torch.int64),
                cnt_tab=view(o["cnt_tab"], P * E, torch.int32).view(P, E),
                gate=view(o["gate"], capacity, torch.float32),
                scale=view(o["scale"], capacity, torch.float32),
                x_recv_fp8=window[o["x_recv"]:o["x_recv"] + capacity * d].view(capacity, d),
                x_recv_mx_sf=window[o["x_recv"] + capacity * d:o["x_recv"] + capacity * d + capacity * (d // 32)]
                .view(capacity, d // 32),
                x_recv=window[o["x_recv"]:o["x_recv"] + capacity * d * eb].view(dt).view(capacity, d),
                out_recv=window[o["out_recv"]:o["out_recv"] + (capacity + S * N) * d * eb].view(dt)
                .view(capacity + S * N, d))


class Group:
    """moe_ep_group: this rank, the receive capacity, its expert count and every rank's
    window address as mapped in this process."""

    def __init__(self, rank: int, capacity: int, local_experts: int, windows):
        self.rank, self.capacity, self.local_experts = rank, capacity, local_experts
        self.windows = [int(w) for w in windows]
        self._arr = (ctypes.c_void_p * len(self.windows))(*self.windows)
        self.c = B.CEpGroup(rank, capacity, local_experts, self._arr)


class Handle:
    """moe_ep_handle: this rank's destinations and its owned experts' receive rows."""

    def __init__(self, cfg, local_experts: int, device="cuda"):
        L = local_experts
        self.dest = torch.empty(max(cfg.N * cfg.k, 1), dtype=torch.int32, device=device)
        self.owner_n_e = torch.empty(max(L, 1), dtype=torch.int32, device=device)
        self.owner_off = torch.empty(L + 1, dtype=torch.int32, device=device)
        self.n_dest, self.L = cfg.N * cfg.k, L
        self.c = B.CEpHandle(self.dest.data_ptr(), self.owner_n_e.data_ptr(), self.owner_off.data_ptr())

    def as_dict(self):
        return dict(dest=self.dest[:self.n_dest], owner_n_e=self.owner_n_e[:self.L], owner_off=self.owner_off)


def workspace_bytes_fp8(cfg, capacity: int) -> int:
    c = B.c_config(cfg)
    return B.load().moe_ep_workspace_bytes_fp8(ctypes.byref(c), capacity)


def workspace_bytes_mx(cfg, capacity: int) -> int:
    c = B.c_config(cfg)
    return B.load().moe_ep_workspace_bytes_mx(ctypes.byref(c), capacity)


def alloc_ws(cfg, capacity: int, device="cuda", fp8=False, mx=False) -> torch.Tensor:
    n = workspace_bytes_mx(cfg, capacity) if mx else (workspace_bytes_fp8(cfg, capacity) if fp8
                                                      else workspace_bytes(cfg, capacity))
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def emulated_groups(cfg, capacity: int, expert_owner=None, device="cuda", rank_cfgs=None):
    """P ranks of one process on one device: P zeroed windows and one Group per rank over
    the same window table.  rank_cfgs[r] (default cfg) is rank r's configuration: its N
    sizes the shared rows of its window.  Every rank's step must then be issued so that
    each wait finds its flags already set (all ranks' notify, then all layouts, all
    dispatches, all expert FFNs, all combines, on one stream): the kernels of different
    ranks never wait on one another."""
    rank_cfgs = rank_cfgs or [cfg] * cfg.P
    windows = [alloc_window(rank_cfgs[r], capacity, device) for r in range(cfg.P)]
    ptrs = [w.data_ptr() for w in windows]
    groups = [Group(r, capacity, len(owned_experts(cfg.E, cfg.P, r, expert_owner)), ptrs) for r in range(cfg.P)]
    return groups, windows


def _agree(values: dict, process_group=None) -> list:
    """all_gather_object of ``values``; raises unless every rank sent the same shape keys."""
    import torch.distributed as dist
    world = dist.get_world_size(process_group)
    got = [None] * world
    dist.all_gather_object(got, values, group=process_group)
    keys = [k for k in values if k not in ("rank", "handle", "offset", "error")]
    for r, v in enumerate(got):
        for k in keys:
            if v[k] != values[k]:
                raise ValueError(f"EP ranks disagree on {k}: rank {r} has {v[k]}, this rank {values[k]}")
        if v["rank"] != r:
            raise ValueError(f"EP rank {r} calls itself rank {v['rank']}")
    return got


def exchange_windows(cfg, capacity: int, rank: int, handle, offset: int, process_group=None,
                     error: str | None = None) -> list:
    """Gather every rank's (IPC handle, offset) after checking that all ranks agree on the
    shapes that fix the window layout (P, E, d, dtype, S, capacity).  A rank that could not
    get its handle passes error=...: every rank then raises with it.  Host logic only."""
    c = B.c_config(cfg)
    mine = dict(rank=rank, P=c.P, E=c.E, d=c.d, dtype=c.dtype, S=c.n_shared, capacity=capacity,
                handle=bytes(handle) if handle is not None else None, offset=int(offset), error=error)
    got = _agree(mine, process_group)
    errors = [g["error"] for g in got if g["error"]]
    if errors:
        raise RuntimeError("; ".join(errors))
    if len(got) != c.P:
        raise ValueError(f"process group has {len(got)} ranks, the configuration P = {c.P}")
    return [(g["handle"], g["offset"]) for g in got]


def map_windows(table, rank: int, own_ptr: int, open_fn, close_fn, process_group=None):
    """Map every other rank's window: open_fn(handle, offset) -> address (raises on
    failure), close_fn(address, offset) unmaps.  Collective: every rank learns whether
    every rank mapped every window, and if one failed all ranks unmap what they mapped and
    raise, so that no rank goes on to a collective the others have abandoned.  Returns
    (addresses in rank order, [(address, offset) opened here])."""
    import torch.distributed as dist
    ptrs, opened, failed = [], [], None
    for r, (hb, o) in enumerate(table):
        if r == rank:
            ptrs.append(own_ptr)
            continue
        try:
            p = open_fn(hb, o)
        except Exception as e:  # noqa: BLE001  (reported to every rank below)
            failed = f"rank {rank} could not map the window of rank {r}: {e}"
            break
        opened.append((p, o))
        ptrs.append(p)
    reports = [None] * dist.get_world_size(process_group)
    dist.all_gather_object(reports, failed, group=process_group)
    if any(reports):
        for p, o in opened:
            close_fn(p, o)
        raise RuntimeError("; ".join(m for m in reports if m))
    return ptrs, opened


def ipc_group(cfg, capacity: int, window: torch.Tensor, expert_owner=None, process_group=None):
    """One process per GPU: map every rank's window through CUDA IPC.  Collective over the
    process group.  Returns (Group, close), close() unmapping the peers' windows.  All
    ranks must have zeroed their windows and passed a barrier before the first step."""
    import torch.distributed as dist
    lib = B.load()
    rank = dist.get_rank(process_group)
    h = (ctypes.c_char * 64)()
    off = ctypes.c_size_t(0)
    err = None
    if lib.moe_ep_ipc_handle(ctypes.c_void_p(window.data_ptr()), h, ctypes.byref(off)) != B.MOE_OK:
        err = f"rank {rank}: moe_ep_ipc_handle: {lib.moe_last_error().decode()}"
    table = exchange_windows(cfg, capacity, rank, None if err else bytes(h), off.value, process_group, error=err)

    def open_fn(hb, o):
        buf = (ctypes.c_char * 64).from_buffer_copy(hb)
        p = ctypes.c_void_p(0)
        if lib.moe_ep_ipc_open(buf, o, ctypes.byref(p)) != B.MOE_OK:
            raise RuntimeError(lib.moe_last_error().decode())
        return p.value

    def close_fn(p, o):
        lib.moe_ep_ipc_close(ctypes.c_void_p(p), o)

    ptrs, opened = map_windows(table, rank, window.data_ptr(), open_fn, close_fn, process_group)

    def close():
        for p, o in opened:
            B._check(lib.moe_ep_ipc_close(ctypes.c_void_p(p), o), "moe_ep_ipc_close")
        opened.clear()

    grp = Group(rank, capacity, len(owned_experts(cfg.E, cfg.P, rank, expert_owner)), ptrs)
    return grp, close


def notify(cfg, grp: Group, topk_ids, ws, status=None):
    """Starts this rank's next step (moe_ep_notify)."""
    c = B.c_config(cfg)
    B._check(B.load().moe_ep_notify(ctypes.byref(c), ctypes.byref(grp.c), B._p(topk_ids), B._p(status),
                                    B._p(ws), ws.numel(), B._stream()), "moe_ep_notify")


def layout(cfg, grp: Group, topk_ids, handle: Handle, ws, expert_owner=None, status=None):
    c = B.c_config(cfg)
    B._check(B.load().moe_ep_layout(ctypes.byref(c), ctypes.byref(grp.c), B._p(expert_owner),
                                    B._p(topk_ids), ctypes.byref(handle.c), B._p(status), B._p(ws), ws.numel(),
                                    B._stream()), "moe_ep_layout")
    return handle


def dispatch(cfg, grp: Group, x, topk_w, handle: Handle):
    c = B.c_config(cfg)
    B._check(B.load().moe_ep_dispatch(ctypes.byref(c), ctypes.byref(grp.c), B._p(x), B._p(topk_w),
                                      ctypes.byref(handle.c), B._stream()), "moe_ep_dispatch")


def expert_ffn(cfg, grp: Group, x, w13, w2, handle: Handle, ws, status=None):
    c = B.c_config(cfg)
    B._check(B.load().moe_ep_expert_ffn(ctypes.byref(c), ctypes.byref(grp.c), B._p(x), B._p(w13),
                                        B._p(w2), ctypes.byref(handle.c), B._p(status), B._p(ws), ws.numel(),
                                        B._stream()), "moe_ep_expert_ffn")


def combine(cfg, grp: Group, handle: Handle, y=None, status=None, device="cuda"):
    c = B.c_config(cfg)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=B._dtype(cfg), device=device)
    B._check(B.load().moe_ep_combine(ctypes.byref(c), ctypes.byref(grp.c), ctypes.byref(handle.c), B._p(y),
                                     B._p(status), B._stream()), "moe_ep_combine")
    return y


def layer_forward(cfg, grp: Group, x, w_gate, bias, w13, w2, ws, expert_owner=None, y=None,
                  handle: Handle | None = None, status=None, side_stream=None):
    """The layer on this rank (moe_ep_layer_forward): route, notify, layout, dispatch,
    expert FFN, combine; with side_stream (a torch.cuda.Stream) the shared experts run
    there (moe_ep_layer_forward_overlapped).  With P > 1 every rank must run the same
    sequence of steps."""
    c = B.c_config(cfg)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=B._dtype(cfg), device=x.device)
    args = [ctypes.byref(c), ctypes.byref(grp.c), B._p(x), B._p(w_gate), B._p(bias), B._p(expert_owner), B._p(w13),
            B._p(w2), B._p(y), ctypes.byref(handle.c) if handle is not None else None, B._p(status), B._p(ws),
            ws.numel(), B._stream()]
    if side_stream is None:
        B._check(B.load().moe_ep_layer_forward(*args), "moe_ep_layer_forward")
    else:
        B._check(B.load().moe_ep_layer_forward_overlapped(*args, ctypes.c_void_p(side_stream.cuda_stream)),
                 "moe_ep_layer_forward_overlapped")
    return y


def dispatch_fp8(cfg, grp: Group, x_q, x_scale, topk_w, handle: Handle):
    """FP8 payload: e4m3 token rows (d bytes) with each token's scale beside its rows."""
    c = B.c_config(cfg)
    B._check(B.load().moe_ep_dispatch_fp8(ctypes.byref(c), ctypes.byref(grp.c), B._p(x_q), B._p(x_scale),
                                          B._p(topk_w), ctypes.byref(handle.c), B._stream()), "moe_ep_dispatch_fp8")


def expert_ffn_fp8(cfg, grp: Group, x_q, x_scale, w13_q, w13_scale, w2_q, w2_scale, handle: Handle, ws, status=None):
    c = B.c_config(cfg)
    B._check(B.load().moe_ep_expert_ffn_fp8(ctypes.byref(c), ctypes.byref(grp.c), B._p(x_q), B._p(x_scale),
                                            B._p(w13_q), B._p(w13_scale), B._p(w2_q), B._p(w2_scale),
                                            ctypes.byref(handle.c), B._p(status), B._p(ws), ws.numel(),
                                            B._stream()), "moe_ep_expert_ffn_fp8")


def layer_forward_fp8(cfg, grp: Group, x, w_gate, bias, w13_q, w13_scale, w2_q, w2_scale, ws, expert_owner=None,
                      y=None, handle: Handle | None = None, status=None, side_stream=None):
    """The layer on this rank with FP8 dispatch and experts, bf16 combine
    (moe_ep_layer_forward_fp8, or ..._overlapped with side_stream); ws from
    alloc_ws(..., fp8=True)."""
    c = B.c_config(cfg)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=torch.bfloat16, device=x.device)
    args = [ctypes.byref(c), ctypes.byref(grp.c), B._p(x), B._p(w_gate), B._p(bias), B._p(expert_owner),
            B._p(w13_q), B._p(w13_scale), B._p(w2_q), B._p(w2_scale), B._p(y),
            ctypes.byref(handle.c) if handle is not None else None, B._p(status), B._p(ws), ws.numel(), B._stream()]
    if side_stream is None:
        B._check(B.load().moe_ep_layer_forward_fp8(*args), "moe_ep_layer_forward_fp8")
    else:
        B._check(B.load().moe_ep_layer_forward_fp8_overlapped(*args, ctypes.c_void_p(side_stream.cuda_stream)),
                 "moe_ep_layer_forward_fp8_overlapped")
    return y


def dispatch_mx(cfg, grp: Group, x_q, x_sf, topk_w, handle: Handle):
    """MX payload: e4m3 token rows (d bytes) and their E8M0 scale rows (d/32 bytes)."""
    c = B.c_config(cfg)
    B._check(B.load().moe_ep_dispatch_mx(ctypes.byref(c), ctypes.byref(grp.c), B._p(x_q), B._p(x_sf),
                                         B._p(topk_w), ctypes.byref(handle.c), B._stream()), "moe_ep_dispatch_mx")


def expert_ffn_mx(cfg, grp: Group, x_q, x_sf, w13_q, w13_sf, w2_q, w2_sf, handle: Handle, ws, status=None):
    c = B.c_config(cfg)
    B._check(B.load().moe_ep_expert_ffn_mx(ctypes.byref(c), ctypes.byref(grp.c), B._p(x_q), B._p(x_sf),
                                           B._p(w13_q), B._p(w13_sf), B._p(w2_q), B._p(w2_sf),
                                           ctypes.byref(handle.c), B._p(status), B._p(ws), ws.numel(),
                                           B._stream()), "moe_ep_expert_ffn_mx")


def layer_forward_mx(cfg, grp: Group, x, w_gate, bias, w13_q, w13_sf, w2_q, w2_sf, ws, expert_owner=None, y=None,
                     handle: Handle | None = None, status=None, side_stream=None):
    """The layer on this rank with MX dispatch and experts, bf16 combine
    (moe_ep_layer_forward_mx, or ..._overlapped with side_stream); ws from
    alloc_ws(..., mx=True)."""
    c = B.c_config(cfg)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=torch.bfloat16, device=x.device)
    args = [ctypes.byref(c), ctypes.byref(grp.c), B._p(x), B._p(w_gate), B._p(bias), B._p(expert_owner),
            B._p(w13_q), B._p(w13_sf), B._p(w2_q), B._p(w2_sf), B._p(y),
            ctypes.byref(handle.c) if handle is not None else None, B._p(status), B._p(ws), ws.numel(), B._stream()]
    if side_stream is None:
        B._check(B.load().moe_ep_layer_forward_mx(*args), "moe_ep_layer_forward_mx")
    else:
        B._check(B.load().moe_ep_layer_forward_mx_overlapped(*args, ctypes.c_void_p(side_stream.cuda_stream)),
                 "moe_ep_layer_forward_mx_overlapped")
    return y
