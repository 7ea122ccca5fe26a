"""Thin ctypes binding over libmoe's C ABI (include/moe.h).

Argument marshalling only: tensors are passed as device pointers with the current torch
CUDA stream, and every step of the layer runs in libmoe's CUDA kernels.  Buffers the
ABI leaves to the caller are allocated here with torch (device memory is plumbing); the
library itself allocates nothing.  If libmoe.so is missing or fails to load, importing
this module raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIB=checked selects the bounds-checked build (libmoe_checked.so, see moe_checks_*)
LIB_PATH = os.path.join(_HERE, "libmoe_checked.so" if os.environ.get("MOE_LIB") == "checked" else "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_BAD_INDEX, \
    MOE_ERR_TIMEOUT = range(7)
MOE_F32, MOE_BF16 = 0, 1
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1
GROUPS = {"all": 0, "routed": 1, "shared": 2}

# every symbol include/moe.h declares
EXPORTED = ["moe_version", "moe_status_string", "moe_last_error", "moe_checks_enabled", "moe_checks_register",
            "moe_check_config",
            "moe_layout_workspace_bytes", "moe_workspace_bytes", "moe_route", "moe_dispatch_layout",
            "moe_dispatch_layout_noalloc",
            "moe_permute", "moe_permute_staged", "moe_grouped_ffn", "moe_expert_fc1", "moe_expert_fc2",
            "moe_routed_ffn", "moe_shared_ffn", "moe_layer_forward_overlapped", "moe_selftest_bounded_wait",
            "moe_combine", "moe_combine_staged",
            "moe_layer_forward", "moe_eplb_plan", "moe_eplb_workspace_bytes", "moe_eplb_assign",
            "moe_eplb_place_weights", "moe_quantize_fp8", "moe_permute_fp8", "moe_grouped_ffn_fp8",
            "moe_workspace_bytes_fp8", "moe_layer_forward_fp8", "moe_capacity_drop", "moe_capacity_rows",
            "moe_layer_forward_fp8_overlapped", "moe_workspace_bytes_chunked", "moe_layer_forward_chunked",
            "moe_ep_window_bytes", "moe_ep_window_layout",
            "moe_ep_workspace_bytes", "moe_ep_ipc_handle", "moe_ep_ipc_open", "moe_ep_ipc_close", "moe_ep_notify",
            "moe_ep_layout", "moe_ep_dispatch", "moe_ep_expert_ffn", "moe_ep_combine", "moe_ep_layer_forward",
            "moe_ep_workspace_bytes_fp8", "moe_ep_dispatch_fp8", "moe_ep_expert_ffn_fp8", "moe_ep_layer_forward_fp8",
            "moe_ep_layer_forward_overlapped", "moe_ep_layer_forward_fp8_overlapped",
            "moe_quantize_mx", "moe_permute_mx", "moe_grouped_ffn_mx", "moe_workspace_bytes_mx",
            "moe_layer_forward_mx", "moe_layer_forward_mx_overlapped", "moe_ep_workspace_bytes_mx",
            "moe_ep_dispatch_mx", "moe_ep_expert_ffn_mx", "moe_ep_layer_forward_mx",
            "moe_ep_layer_forward_mx_overlapped"]


class CConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ["N", "d", "E", "k", "I", "n_shared", "P", "n_groups", "topk_groups", "score",
                 "renormalize", "dtype", "bias_mode"]]


LAYOUT_FIELDS = ["n_e", "expert_off", "C", "send_off", "recv_off", "tok2send", "send2row", "ret2tok",
                 "tok2row", "row2tok", "tile_off"]


class CLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LAYOUT_FIELDS]


class CEpGroup(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32), ("capacity", ctypes.c_int32), ("local_experts", ctypes.c_int32),
                ("windows", ctypes.POINTER(ctypes.c_void_p))]


class CEpHandle(ctypes.Structure):
    _fields_ = [("dest", ctypes.c_void_p), ("owner_n_e", ctypes.c_void_p), ("owner_off", ctypes.c_void_p)]


class MoEError(RuntimeError):
    def __init__(self, status, where, detail=""):
        self.status = status
        super().__init__(f"{where}: status {status} ({_status_text(status)}) {detail}".strip())


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libmoe.so not found at {path}; build it with "
                          f"`python -m dispatch_combine_grouped_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cfgp, layp = ctypes.POINTER(CConfig), ctypes.POINTER(CLayout)
    sig = {
        "moe_version": (i32, []),
        "moe_status_string": (ctypes.c_char_p, [i32]),
        "moe_last_error": (ctypes.c_char_p, []),
        "moe_checks_enabled": (i32, []),
        "moe_checks_register": (i32, [vp]),
        "moe_check_config": (i32, [cfgp]),
        "moe_layout_workspace_bytes": (sz, [cfgp]),
        "moe_workspace_bytes": (sz, [cfgp]),
        "moe_route": (i32, [cfgp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_dispatch_layout": (i32, [cfgp, vp, vp, layp, vp, vp, sz, vp]),
        "moe_dispatch_layout_noalloc": (i32, [cfgp, vp, vp, layp, vp, vp]),
        "moe_permute": (i32, [cfgp, layp, vp, vp, vp]),
        "moe_permute_staged": (i32, [cfgp, layp, vp, vp, vp, vp]),
        "moe_grouped_ffn": (i32, [cfgp, layp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_expert_fc1": (i32, [cfgp, layp, vp, vp, vp, vp, i32, vp]),
        "moe_expert_fc2": (i32, [cfgp, layp, vp, vp, vp, vp, i32, vp]),
        "moe_routed_ffn": (i32, [cfgp, layp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_shared_ffn": (i32, [cfgp, vp, vp, vp, vp, vp, vp]),
        "moe_layer_forward_overlapped": (i32, [cfgp, vp, vp, vp, vp, vp, vp, vp, layp, vp, vp, sz, vp, vp]),
        "moe_selftest_bounded_wait": (i32, [vp, ctypes.c_uint64, vp]),
        "moe_combine": (i32, [cfgp, layp, vp, vp, vp, vp]),
        "moe_combine_staged": (i32, [cfgp, layp, vp, vp, vp, vp, vp]),
        "moe_layer_forward": (i32, [cfgp, vp, vp, vp, vp, vp, vp, vp, layp, vp, vp, sz, vp]),
        "moe_eplb_plan": (i32, [i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]),
        "moe_eplb_workspace_bytes": (sz, [cfgp]),
        "moe_eplb_assign": (i32, [cfgp, vp, vp, vp, i32, vp, vp, vp, sz, vp]),
        "moe_eplb_place_weights": (i32, [vp, i32, i32, i32, sz, vp, vp, vp]),
        "moe_quantize_fp8": (i32, [vp, ctypes.c_int64, i32, vp, vp, vp]),
        "moe_permute_fp8": (i32, [cfgp, layp, vp, vp, vp]),
        "moe_grouped_ffn_fp8": (i32, [cfgp, layp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "moe_workspace_bytes_fp8": (sz, [cfgp]),
        "moe_quantize_mx": (i32, [vp, ctypes.c_int64, i32, vp, vp, vp]),
        "moe_permute_mx": (i32, [cfgp, layp, vp, vp, vp, vp, vp]),
        "moe_grouped_ffn_mx": (i32, [cfgp, layp] + [vp] * 14),
        "moe_workspace_bytes_mx": (sz, [cfgp]),
        "moe_layer_forward_mx": (i32, [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, layp, vp, vp, sz, vp]),
        "moe_layer_forward_mx_overlapped": (i32, [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, layp, vp, vp, sz, vp, vp]),
        "moe_layer_forward_fp8": (i32, [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, layp, vp, vp, sz, vp]),
        "moe_capacity_drop": (i32, [cfgp, vp, i32, vp, vp, vp, sz, vp]),
        "moe_capacity_rows": (i32, [cfgp, ctypes.c_double, ctypes.POINTER(i32)]),
        "moe_workspace_bytes_chunked": (sz, [cfgp, i32]),
        "moe_layer_forward_chunked": (i32, [cfgp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]),
        "moe_layer_forward_fp8_overlapped": (i32, [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, layp, vp, vp, sz, vp,
                                                   vp]),
    }
    grpp, hdp = ctypes.POINTER(CEpGroup), ctypes.POINTER(CEpHandle)
    sig.update({
        "moe_ep_window_bytes": (sz, [cfgp, i32]),
        "moe_ep_window_layout": (i32, [cfgp, i32, vp]),
        "moe_ep_workspace_bytes": (sz, [cfgp, i32]),
        "moe_ep_ipc_handle": (i32, [vp, vp, ctypes.POINTER(sz)]),
        "moe_ep_ipc_open": (i32, [vp, sz, ctypes.POINTER(vp)]),
        "moe_ep_ipc_close": (i32, [vp, sz]),
        "moe_ep_notify": (i32, [cfgp, grpp, vp, vp, vp, sz, vp]),
        "moe_ep_layout": (i32, [cfgp, grpp, vp, vp, hdp, vp, vp, sz, vp]),
        "moe_ep_dispatch": (i32, [cfgp, grpp, vp, vp, hdp, vp]),
        "moe_ep_expert_ffn": (i32, [cfgp, grpp, vp, vp, vp, hdp, vp, vp, sz, vp]),
        "moe_ep_combine": (i32, [cfgp, grpp, hdp, vp, vp, vp]),
        "moe_ep_layer_forward": (i32, [cfgp, grpp, vp, vp, vp, vp, vp, vp, vp, hdp, vp, vp, sz, vp]),
        "moe_ep_workspace_bytes_mx": (sz, [cfgp, i32]),
        "moe_ep_dispatch_mx": (i32, [cfgp, grpp, vp, vp, vp, hdp, vp]),
        "moe_ep_expert_ffn_mx": (i32, [cfgp, grpp, vp, vp, vp, vp, vp, vp, hdp, vp, vp, sz, vp]),
        "moe_ep_layer_forward_mx": (i32, [cfgp, grpp, vp, vp, vp, vp, vp, vp, vp, vp, vp, hdp, vp, vp, sz, vp]),
        "moe_ep_layer_forward_mx_overlapped": (i32, [cfgp, grpp, vp, vp, vp, vp, vp, vp, vp, vp, vp, hdp, vp, vp, sz,
                                                     vp, vp]),
        "moe_ep_workspace_bytes_fp8": (sz, [cfgp, i32]),
        "moe_ep_dispatch_fp8": (i32, [cfgp, grpp, vp, vp, vp, hdp, vp]),
        "moe_ep_expert_ffn_fp8": (i32, [cfgp, grpp, vp, vp, vp, vp, vp, vp, hdp, vp, vp, sz, vp]),
        "moe_ep_layer_forward_fp8": (i32, [cfgp, grpp, vp, vp, vp, vp, vp, vp, vp, vp, vp, hdp, vp, vp, sz, vp]),
        "moe_ep_layer_forward_overlapped": (i32, [cfgp, grpp, vp, vp, vp, vp, vp, vp, vp, hdp, vp, vp, sz, vp, vp]),
        "moe_ep_layer_forward_fp8_overlapped": (i32, [cfgp, grpp, vp, vp, vp, vp, vp, vp, vp, vp, vp, hdp, vp, vp, sz,
                                                      vp, vp]),
    })
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _status_text(s):
    try:
        return load().moe_status_string(s).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(status, where):
    if status != MOE_OK:
        detail = load().moe_last_error().decode()
        raise MoEError(status, where, detail)


def c_config(cfg) -> CConfig:
    """moe_config from a workload description (moe_inputs.MoEConfig or any object with
    the same attribute names)."""
    score = cfg.score if isinstance(cfg.score, int) else \
        {"softmax": MOE_SCORE_SOFTMAX, "sigmoid": MOE_SCORE_SIGMOID}[cfg.score]
    dtype = cfg.dtype if isinstance(cfg.dtype, int) else {"f32": MOE_F32, "bf16": MOE_BF16}[cfg.dtype]
    bias_mode = getattr(cfg, "bias_mode", "logits")
    bias_mode = bias_mode if isinstance(bias_mode, int) else {"logits": 0, "selection": 1}[bias_mode]
    return CConfig(cfg.N, cfg.d, cfg.E, cfg.k, cfg.I, cfg.S, cfg.P, cfg.n_groups, cfg.topk_groups,
                   score, int(bool(cfg.renormalize)), dtype, bias_mode)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype(cfg):
    return torch.float32 if c_config(cfg).dtype == MOE_F32 else torch.bfloat16


class Layout:
    """Caller-owned layout arrays (int32, on the device) and their C view."""

    def __init__(self, cfg, device="cuda"):
        A, E, P, S = cfg.N * cfg.k, cfg.E, cfg.P, cfg.S
        sizes = dict(n_e=E, expert_off=E + 1, C=P * P, send_off=P * P, recv_off=P + 1, tok2send=A,
                     send2row=A, ret2tok=A, tok2row=A, row2tok=A, tile_off=E + S + 1)
        self.t = {k: torch.empty(max(v, 1), dtype=torch.int32, device=device) for k, v in sizes.items()}
        self.sizes = sizes
        self.c = CLayout(*[self.t[k].data_ptr() for k in LAYOUT_FIELDS])

    def __getitem__(self, key):
        return self.t[key][:self.sizes[key]]

    def as_dict(self):
        return {k: self[k] for k in LAYOUT_FIELDS}


def selftest_bounded_wait(status, limit_ns=20_000_000):
    """Run the bounded-wait self-test kernel; it writes MOE_ERR_TIMEOUT into ``status``."""
    _check(load().moe_selftest_bounded_wait(_p(status), limit_ns, _stream()), "moe_selftest_bounded_wait")


def version() -> int:
    return load().moe_version()


def checks_enabled() -> bool:
    """True when the loaded library is the bounds-checked build."""
    return bool(load().moe_checks_enabled())


def checks_register(word):
    """Register a device int32 tensor (or None) that the bounds-checked build records
    failed index checks into (MOE_ERR_BAD_INDEX)."""
    _check(load().moe_checks_register(_p(word)), "moe_checks_register")


def check_config(cfg):
    c = c_config(cfg)
    _check(load().moe_check_config(ctypes.byref(c)), "moe_check_config")


def workspace_bytes(cfg) -> int:
    c = c_config(cfg)
    return load().moe_workspace_bytes(ctypes.byref(c))


def layout_workspace_bytes(cfg) -> int:
    c = c_config(cfg)
    return load().moe_layout_workspace_bytes(ctypes.byref(c))


def route(cfg, x, w_gate, bias=None, out=None):
    """-> (logits [N,E] fp32, topk_ids [N,k] int32, topk_w [N,k] fp32)"""
    c = c_config(cfg)
    if out is None:
        dev = x.device
        out = (torch.empty(cfg.N, cfg.E, dtype=torch.float32, device=dev),
               torch.empty(cfg.N, cfg.k, dtype=torch.int32, device=dev),
               torch.empty(cfg.N, cfg.k, dtype=torch.float32, device=dev))
    logits, ids, w = out
    _check(load().moe_route(ctypes.byref(c), _p(x), _p(w_gate), _p(bias), _p(logits), _p(ids), _p(w),
                            _stream()), "moe_route")
    return logits, ids, w


def dispatch_layout(cfg, topk_ids, expert_owner=None, status=None, layout=None, ws=None):
    c = c_config(cfg)
    lib = load()
    layout = layout or Layout(cfg, topk_ids.device)
    nbytes = lib.moe_layout_workspace_bytes(ctypes.byref(c))
    if ws is None:
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=topk_ids.device)
    _check(lib.moe_dispatch_layout(ctypes.byref(c), _p(expert_owner), _p(topk_ids), ctypes.byref(layout.c),
                                   _p(status), _p(ws), ws.numel(), _stream()), "moe_dispatch_layout")
    return layout


def dispatch_layout_noalloc(cfg, topk_ids, expert_owner=None, status=None, layout=None):
    """moe_dispatch_layout_noalloc: the layout with the library's built-in scratch (no
    workspace argument; for callers that cannot allocate device memory)."""
    c = c_config(cfg)
    layout = layout or Layout(cfg, topk_ids.device)
    _check(load().moe_dispatch_layout_noalloc(ctypes.byref(c), _p(expert_owner), _p(topk_ids),
                                              ctypes.byref(layout.c), _p(status), _stream()),
           "moe_dispatch_layout_noalloc")
    return layout


def permute(cfg, layout, x, out=None):
    c = c_config(cfg)
    if out is None:
        out = torch.empty(cfg.N * cfg.k, cfg.d, dtype=x.dtype, device=x.device)
    _check(load().moe_permute(ctypes.byref(c), ctypes.byref(layout.c), _p(x), _p(out), _stream()),
           "moe_permute")
    return out


def permute_staged(cfg, layout, x):
    c = c_config(cfg)
    send = torch.empty(cfg.N * cfg.k, cfg.d, dtype=x.dtype, device=x.device)
    out = torch.empty_like(send)
    _check(load().moe_permute_staged(ctypes.byref(c), ctypes.byref(layout.c), _p(x), _p(send), _p(out),
                                     _stream()), "moe_permute_staged")
    return send, out


def grouped_ffn(cfg, layout, x_perm, x, w13, w2, topk_w=None, h=None, out=None):
    """-> (h [A+S*N, I], out [A+S*N, d]) in the config dtype."""
    c = c_config(cfg)
    rows = cfg.N * cfg.k + cfg.S * cfg.N
    dt, dev = _dtype(cfg), x_perm.device
    if h is None:
        h = torch.empty(rows, cfg.I, dtype=dt, device=dev)
    if out is None:
        out = torch.empty(rows, cfg.d, dtype=dt, device=dev)
    _check(load().moe_grouped_ffn(ctypes.byref(c), ctypes.byref(layout.c), _p(x_perm), _p(x), _p(w13), _p(w2),
                                  _p(topk_w), _p(h), _p(out), _stream()), "moe_grouped_ffn")
    return h, out


def expert_fc1(cfg, layout, x_perm, x, w13, h=None, groups="all", stream=None):
    c = c_config(cfg)
    if h is None:
        dev = (x_perm if x_perm is not None else x).device
        h = torch.empty(cfg.N * cfg.k + cfg.S * cfg.N, cfg.I, dtype=_dtype(cfg), device=dev)
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    lay = ctypes.byref(layout.c) if layout is not None else None
    _check(load().moe_expert_fc1(ctypes.byref(c), lay, _p(x_perm), _p(x), _p(w13), _p(h), GROUPS[groups], st),
           "moe_expert_fc1")
    return h


def expert_fc2(cfg, layout, h, w2, topk_w=None, out=None, groups="all", stream=None):
    c = c_config(cfg)
    if out is None:
        out = torch.empty(cfg.N * cfg.k + cfg.S * cfg.N, cfg.d, dtype=_dtype(cfg), device=h.device)
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    lay = ctypes.byref(layout.c) if layout is not None else None
    _check(load().moe_expert_fc2(ctypes.byref(c), lay, _p(h), _p(w2), _p(topk_w), _p(out), GROUPS[groups], st),
           "moe_expert_fc2")
    return out


def routed_ffn(cfg, layout, x_perm, w13, w2, topk_w=None, h=None, out=None):
    c = c_config(cfg)
    rows = cfg.N * cfg.k + cfg.S * cfg.N
    if h is None:
        h = torch.empty(rows, cfg.I, dtype=_dtype(cfg), device=x_perm.device)
    if out is None:
        out = torch.empty(rows, cfg.d, dtype=_dtype(cfg), device=x_perm.device)
    _check(load().moe_routed_ffn(ctypes.byref(c), ctypes.byref(layout.c), _p(x_perm), _p(w13), _p(w2), _p(topk_w),
                                 _p(h), _p(out), _stream()), "moe_routed_ffn")
    return h, out


def shared_ffn(cfg, x, w13, w2, h, out, stream=None):
    """Shared experts into rows [A, A+S*N) of h and out, on ``stream`` (default: current)."""
    c = c_config(cfg)
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    _check(load().moe_shared_ffn(ctypes.byref(c), _p(x), _p(w13), _p(w2), _p(h), _p(out), st), "moe_shared_ffn")
    return h, out


def combine(cfg, layout, out_rows, topk_w=None, y=None):
    c = c_config(cfg)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=out_rows.dtype, device=out_rows.device)
    _check(load().moe_combine(ctypes.byref(c), ctypes.byref(layout.c), _p(out_rows), _p(topk_w), _p(y),
                              _stream()), "moe_combine")
    return y


def combine_staged(cfg, layout, out_rows, topk_w=None):
    c = c_config(cfg)
    ret = torch.empty(cfg.N * cfg.k, cfg.d, dtype=out_rows.dtype, device=out_rows.device)
    y = torch.empty(cfg.N, cfg.d, dtype=out_rows.dtype, device=out_rows.device)
    _check(load().moe_combine_staged(ctypes.byref(c), ctypes.byref(layout.c), _p(out_rows), _p(topk_w), _p(ret),
                                     _p(y), _stream()), "moe_combine_staged")
    return ret, y


def alloc_workspace(cfg, device="cuda"):
    return torch.empty(max(workspace_bytes(cfg), 1), dtype=torch.uint8, device=device)


def layer_forward_overlapped(cfg, x, w_gate, bias, expert_owner, w13, w2, side_stream, y=None, ws=None, layout=None,
                             status=None):
    """moe_layer_forward_overlapped: shared experts on ``side_stream`` (a torch.cuda.Stream)."""
    c = c_config(cfg)
    if ws is None:
        ws = alloc_workspace(cfg, x.device)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=x.dtype, device=x.device)
    lay = ctypes.byref(layout.c) if layout is not None else None
    _check(load().moe_layer_forward_overlapped(ctypes.byref(c), _p(x), _p(w_gate), _p(bias), _p(expert_owner),
                                               _p(w13), _p(w2), _p(y), lay, _p(status), _p(ws), ws.numel(), _stream(),
                                               ctypes.c_void_p(side_stream.cuda_stream)),
           "moe_layer_forward_overlapped")
    return y


def workspace_bytes_chunked(cfg, n_chunks: int) -> int:
    c = c_config(cfg)
    return load().moe_workspace_bytes_chunked(ctypes.byref(c), int(n_chunks))


def layer_forward_chunked(cfg, n_chunks, x, w_gate, bias, expert_owner, w13, w2, side_stream, y=None, ws=None,
                          status=None):
    """moe_layer_forward_chunked: the layer as a pipeline over n_chunks token chunks (layout
    and permute on the current stream, expert FFN on ``side_stream``)."""
    c = c_config(cfg)
    if ws is None:
        ws = torch.empty(max(workspace_bytes_chunked(cfg, n_chunks), 1), dtype=torch.uint8, device=x.device)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=x.dtype, device=x.device)
    _check(load().moe_layer_forward_chunked(ctypes.byref(c), int(n_chunks), _p(x), _p(w_gate), _p(bias),
                                            _p(expert_owner), _p(w13), _p(w2), _p(y), _p(status), _p(ws), ws.numel(),
                                            _stream(), ctypes.c_void_p(side_stream.cuda_stream)),
           "moe_layer_forward_chunked")
    return y


def layer_forward(cfg, x, w_gate, bias, expert_owner, w13, w2, y=None, ws=None, layout=None, status=None):
    """The whole layer through moe_layer_forward; -> y [N, d]."""
    c = c_config(cfg)
    if ws is None:
        ws = alloc_workspace(cfg, x.device)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=x.dtype, device=x.device)
    lay = ctypes.byref(layout.c) if layout is not None else None
    _check(load().moe_layer_forward(ctypes.byref(c), _p(x), _p(w_gate), _p(bias), _p(expert_owner), _p(w13),
                                    _p(w2), _p(y), lay, _p(status), _p(ws), ws.numel(), _stream()),
           "moe_layer_forward")
    return y


# ---------------------------------------------------------------- redundant expert slots (EPLB)
def _np_ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def eplb_plan(load_per_expert, R: int, P: int) -> dict:
    """moe_eplb_plan (host): copies per expert, slot tables and planned owner loads.
    Returns int32/int64 NumPy arrays: copies [E], replica_off [E+1], replica_slots [E+R],
    slot_expert [E+R], slot_owner [E+R], owner_load [P]."""
    import numpy as np
    load_np = np.ascontiguousarray(np.asarray(load_per_expert, dtype=np.int64))
    E = len(load_np)
    out = {"copies": np.zeros(E, np.int32), "replica_off": np.zeros(E + 1, np.int32),
           "replica_slots": np.zeros(E + R, np.int32), "slot_expert": np.zeros(E + R, np.int32),
           "slot_owner": np.zeros(E + R, np.int32), "owner_load": np.zeros(P, np.int64)}
    _check(load().moe_eplb_plan(E, R, P, _np_ptr(load_np), _np_ptr(out["copies"]), _np_ptr(out["replica_off"]),
                                _np_ptr(out["replica_slots"]), _np_ptr(out["slot_expert"]),
                                _np_ptr(out["slot_owner"]), _np_ptr(out["owner_load"])), "moe_eplb_plan")
    return out


def physical_config(cfg, R: int):
    """The configuration of the E + R physical slots (same sizes, plain top-k grouping:
    the slots are never routed to directly)."""
    import dataclasses
    return dataclasses.replace(cfg, E=cfg.E + R, n_groups=1, topk_groups=1)


def eplb_workspace_bytes(cfg) -> int:
    c = c_config(cfg)
    return load().moe_eplb_workspace_bytes(ctypes.byref(c))


def eplb_assign(cfg, topk_ids, replica_off, replica_slots, n_slots: int, status=None, out=None, ws=None):
    """moe_eplb_assign: physical slot ids [N, k] int32 for the logical ids (device)."""
    c = c_config(cfg)
    lib = load()
    dev = topk_ids.device
    if out is None:
        out = torch.empty_like(topk_ids)
    if ws is None:
        ws = torch.empty(max(lib.moe_eplb_workspace_bytes(ctypes.byref(c)), 1), dtype=torch.uint8, device=dev)
    _check(lib.moe_eplb_assign(ctypes.byref(c), _p(topk_ids), _p(replica_off), _p(replica_slots), n_slots,
                               _p(out), _p(status), _p(ws), ws.numel(), _stream()), "moe_eplb_assign")
    return out


def eplb_place_weights(slot_expert, E: int, n_shared: int, w):
    """moe_eplb_place_weights: [n_slots + n_shared, ...] copy of w [E + n_shared, ...] whose
    slot s holds expert slot_expert[s] (host int array)."""
    import numpy as np
    se = np.ascontiguousarray(np.asarray(slot_expert, dtype=np.int32))
    n_slots = len(se)
    out = torch.empty((n_slots + n_shared,) + tuple(w.shape[1:]), dtype=w.dtype, device=w.device)
    expert_bytes = w[0].numel() * w.element_size()
    _check(load().moe_eplb_place_weights(_np_ptr(se), n_slots, E, n_shared, expert_bytes, _p(w), _p(out),
                                         _stream()), "moe_eplb_place_weights")
    return out


# ---------------------------------------------------------------- FP8 (e4m3) expert path
def quantize_fp8(src, out=None, scale=None):
    """moe_quantize_fp8: per-row e4m3 codes (uint8, same shape) and fp32 scales of a bf16
    tensor whose last dimension is the row."""
    rows = src.numel() // src.shape[-1]
    cols = src.shape[-1]
    if out is None:
        out = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    if scale is None:
        scale = torch.empty(src.shape[:-1], dtype=torch.float32, device=src.device)
    _check(load().moe_quantize_fp8(_p(src), rows, cols, _p(out), _p(scale), _stream()), "moe_quantize_fp8")
    return out, scale


def permute_fp8(cfg, layout, x_q, out=None):
    c = c_config(cfg)
    if out is None:
        out = torch.empty(cfg.N * cfg.k, cfg.d, dtype=torch.uint8, device=x_q.device)
    _check(load().moe_permute_fp8(ctypes.byref(c), ctypes.byref(layout.c), _p(x_q), _p(out), _stream()),
           "moe_permute_fp8")
    return out


def grouped_ffn_fp8(cfg, layout, x_q_perm, x_q, x_scale, w13_q, w13_scale, w2_q, w2_scale, topk_w=None,
                    h=None, h_q=None, h_scale=None, out=None):
    """-> (h bf16, h_q e4m3, h_scale, out bf16) over [A + S*N] rows."""
    c = c_config(cfg)
    dev = x_q_perm.device
    rows = cfg.N * cfg.k + cfg.S * cfg.N
    h = h if h is not None else torch.empty(rows, cfg.I, dtype=torch.bfloat16, device=dev)
    h_q = h_q if h_q is not None else torch.empty(rows, cfg.I, dtype=torch.uint8, device=dev)
    h_scale = h_scale if h_scale is not None else torch.empty(rows, dtype=torch.float32, device=dev)
    out = out if out is not None else torch.empty(rows, cfg.d, dtype=torch.bfloat16, device=dev)
    _check(load().moe_grouped_ffn_fp8(ctypes.byref(c), ctypes.byref(layout.c), _p(x_q_perm), _p(x_q), _p(x_scale),
                                      _p(w13_q), _p(w13_scale), _p(w2_q), _p(w2_scale), _p(topk_w), _p(h), _p(h_q),
                                      _p(h_scale), _p(out), _stream()), "moe_grouped_ffn_fp8")
    return h, h_q, h_scale, out


def workspace_bytes_fp8(cfg) -> int:
    c = c_config(cfg)
    return load().moe_workspace_bytes_fp8(ctypes.byref(c))


def layer_forward_fp8(cfg, x, w_gate, bias, expert_owner, w13_q, w13_scale, w2_q, w2_scale, y=None, ws=None,
                      layout=None, status=None, side_stream=None):
    """moe_layer_forward_fp8, or moe_layer_forward_fp8_overlapped when side_stream is given."""
    c = c_config(cfg)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = torch.empty(max(workspace_bytes_fp8(cfg), 1), dtype=torch.uint8, device=x.device)
    args = [ctypes.byref(c), _p(x), _p(w_gate), _p(bias), _p(expert_owner), _p(w13_q), _p(w13_scale), _p(w2_q),
            _p(w2_scale), _p(y), ctypes.byref(layout.c) if layout is not None else None, _p(status), _p(ws),
            ws.numel(), _stream()]
    if side_stream is None:
        _check(load().moe_layer_forward_fp8(*args), "moe_layer_forward_fp8")
    else:
        _check(load().moe_layer_forward_fp8_overlapped(*args, ctypes.c_void_p(side_stream.cuda_stream)),
               "moe_layer_forward_fp8_overlapped")
    return y


# ---------------------------------------------------------------- MX (block-scaled e4m3) expert path
def quantize_mx(src, out=None, sf=None):
    """moe_quantize_mx: e4m3 codes (uint8, same shape) and E8M0 scale bytes (uint8, last
    dimension / 32) of a bf16 tensor whose last dimension is the row."""
    rows = src.numel() // src.shape[-1]
    cols = src.shape[-1]
    if out is None:
        out = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    if sf is None:
        sf = torch.empty(src.shape[:-1] + (cols // 32,), dtype=torch.uint8, device=src.device)
    _check(load().moe_quantize_mx(_p(src), rows, cols, _p(out), _p(sf), _stream()), "moe_quantize_mx")
    return out, sf


def permute_mx(cfg, layout, x_q, x_sf, out=None, sf_out=None):
    c = c_config(cfg)
    A = cfg.N * cfg.k
    if out is None:
        out = torch.empty(A, cfg.d, dtype=torch.uint8, device=x_q.device)
    if sf_out is None:
        sf_out = torch.empty(A, cfg.d // 32, dtype=torch.uint8, device=x_q.device)
    _check(load().moe_permute_mx(ctypes.byref(c), ctypes.byref(layout.c), _p(x_q), _p(x_sf), _p(out), _p(sf_out),
                                 _stream()), "moe_permute_mx")
    return out, sf_out


def grouped_ffn_mx(cfg, layout, x_q_perm, x_sf_perm, x_q, x_sf, w13_q, w13_sf, w2_q, w2_sf, topk_w=None,
                   h=None, h_q=None, h_sf=None, out=None):
    """-> (h bf16, h_q e4m3, h_sf E8M0, out bf16) over [A + S*N] rows."""
    c = c_config(cfg)
    dev = x_q_perm.device
    rows = cfg.N * cfg.k + cfg.S * cfg.N
    h = h if h is not None else torch.empty(rows, cfg.I, dtype=torch.bfloat16, device=dev)
    h_q = h_q if h_q is not None else torch.empty(rows, cfg.I, dtype=torch.uint8, device=dev)
    h_sf = h_sf if h_sf is not None else torch.empty(rows, cfg.I // 32, dtype=torch.uint8, device=dev)
    out = out if out is not None else torch.empty(rows, cfg.d, dtype=torch.bfloat16, device=dev)
    _check(load().moe_grouped_ffn_mx(ctypes.byref(c), ctypes.byref(layout.c), _p(x_q_perm), _p(x_sf_perm), _p(x_q),
                                     _p(x_sf), _p(w13_q), _p(w13_sf), _p(w2_q), _p(w2_sf), _p(topk_w), _p(h),
                                     _p(h_q), _p(h_sf), _p(out), _stream()), "moe_grouped_ffn_mx")
    return h, h_q, h_sf, out


def workspace_bytes_mx(cfg) -> int:
    c = c_config(cfg)
    return load().moe_workspace_bytes_mx(ctypes.byref(c))


def layer_forward_mx(cfg, x, w_gate, bias, expert_owner, w13_q, w13_sf, w2_q, w2_sf, y=None, ws=None, layout=None,
                     status=None, side_stream=None):
    """moe_layer_forward_mx on the current stream, or moe_layer_forward_mx_overlapped when
    side_stream is given."""
    c = c_config(cfg)
    if y is None:
        y = torch.empty(cfg.N, cfg.d, dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = torch.empty(max(workspace_bytes_mx(cfg), 1), dtype=torch.uint8, device=x.device)
    args = [ctypes.byref(c), _p(x), _p(w_gate), _p(bias), _p(expert_owner), _p(w13_q), _p(w13_sf), _p(w2_q),
            _p(w2_sf), _p(y), ctypes.byref(layout.c) if layout is not None else None, _p(status), _p(ws), ws.numel(),
            _stream()]
    if side_stream is None:
        _check(load().moe_layer_forward_mx(*args), "moe_layer_forward_mx")
    else:
        _check(load().moe_layer_forward_mx_overlapped(*args, ctypes.c_void_p(side_stream.cuda_stream)),
               "moe_layer_forward_mx_overlapped")
    return y


# ---------------------------------------------------------------- capacity factor
def capacity_of(factor: float, cfg) -> int:
    """moe_capacity_rows: ceil(factor * N * k / E), the uniform share of one expert times
    the factor (computed by the library)."""
    c = c_config(cfg)
    out = ctypes.c_int32(0)
    _check(load().moe_capacity_rows(ctypes.byref(c), float(factor), ctypes.byref(out)), "moe_capacity_rows")
    return int(out.value)


def capacity_drop(cfg, topk_ids, capacity: int, status=None, out=None, ws=None):
    """moe_capacity_drop: topk_ids with the assignments past each expert's first
    `capacity` (ascending a) set to -1."""
    c = c_config(cfg)
    lib = load()
    if out is None:
        out = torch.empty_like(topk_ids)
    if ws is None:
        ws = torch.empty(max(lib.moe_eplb_workspace_bytes(ctypes.byref(c)), 1), dtype=torch.uint8,
                         device=topk_ids.device)
    _check(lib.moe_capacity_drop(ctypes.byref(c), _p(topk_ids), int(capacity), _p(out), _p(status), _p(ws),
                                 ws.numel(), _stream()), "moe_capacity_drop")
    return out

