"""The C ABI library (CPU only): it loads, exports every function include/moe.h declares,
and its host-side validation works without a GPU (no kernel is launched here)."""
import ctypes
import os
import re
import subprocess

import pytest

import dispatch_combine_grouped_b200 as moe
from dispatch_combine_grouped_b200 import binding
from moe_inputs import CONFIGS, small_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_what_binding_expects():
    assert declared_functions() == sorted(binding.EXPORTED)


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(binding.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert set(declared_functions()) <= exported


def test_library_is_sm100a_only():
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", binding.LIB_PATH],
                         capture_output=True, text=True).stdout
    archs = set(re.findall(r"sm_\d+a?", out))
    assert archs == {"sm_100a"}, archs


def test_host_validation_without_gpu():
    for cfg in CONFIGS.values():
        moe.check_config(cfg)
        assert moe.workspace_bytes(cfg) > 0
    bad = [dict(k=9), dict(E=512), dict(P=64), dict(d=100), dict(N=-1), dict(n_groups=3),
           dict(n_groups=4, topk_groups=5), dict(S=9)]
    for kw in bad:
        with pytest.raises(moe.MoEError):
            moe.check_config(CONFIGS["fine"].replace(**kw))


def test_workspace_covers_all_buffers():
    cfg = CONFIGS["wide"]
    A, S = cfg.N * cfg.k, cfg.S
    need = A * cfg.d * 2 + (A + S * cfg.N) * (cfg.I + cfg.d) * 2
    assert moe.workspace_bytes(cfg) >= need
    assert moe.layout_workspace_bytes(small_config(N=7, k=2, E=8, P=2)) > 0


def test_calls_reject_null_without_launching():
    cfg = binding.c_config(small_config(N=8, d=64, E=8, S=0, k=2, I=64, P=2))
    lib = binding.load()
    assert lib.moe_route(ctypes.byref(cfg), None, None, None, None, None, None, None) == binding.MOE_ERR_INVALID_ARG
    lay = binding.CLayout()
    assert lib.moe_dispatch_layout(ctypes.byref(cfg), None, None, ctypes.byref(lay), None, None, 0, None) \
        == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(ctypes.byref(cfg), None, None, None, None, None, None, None, None, None, None, 0,
                                 None) == binding.MOE_ERR_WORKSPACE
