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
    bad = [dict(k=9), dict(E=513), dict(P=64), dict(d=100), dict(N=-1), dict(n_groups=3),
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


def test_router_takes_at_most_256_experts():
    """Layout and expert calls accept up to 512 experts (physical slots); the router 256.
    The check happens on the host before anything launches."""
    cfg = small_config(N=8, d=64, E=288, S=0, k=2, I=64, P=2)
    moe.check_config(cfg)
    c = binding.c_config(cfg)
    lib = binding.load()
    assert lib.moe_route(ctypes.byref(c), None, None, None, None, None, None, None) == binding.MOE_ERR_UNSUPPORTED
    assert lib.moe_layer_forward(ctypes.byref(c), None, None, None, None, None, None, None, None, None, None, 0,
                                 None) == binding.MOE_ERR_UNSUPPORTED


def test_eplb_plan_matches_the_oracle_on_the_host():
    """moe_eplb_plan is host code: its tables equal the oracle's plan (same steps, written
    independently), for random and skewed loads."""
    import numpy as np
    from oracle import eplb as EP
    rng = np.random.default_rng(11)
    cases = [(4, 2, 3, np.array([10, 4, 3, 1]))]
    for E, R, P in [(8, 4, 4), (16, 16, 8), (32, 0, 8), (128, 16, 16), (256, 32, 32), (6, 3, 9), (64, 0, 8)]:
        cases.append((E, R, P, rng.zipf(1.3, size=E).astype(np.int64) % 100000))
        cases.append((E, R, P, rng.integers(0, 5, size=E)))
    for E, R, P, load in cases:
        got = moe.eplb_plan(load, R, P)
        ref = EP.plan(load, R, P)
        for key in ("copies", "replica_off", "replica_slots", "slot_expert", "slot_owner", "owner_load"):
            assert got[key].tolist() == ref[key].tolist(), (E, R, P, key)


def test_eplb_calls_reject_bad_arguments_without_launching():
    import numpy as np
    lib = binding.load()
    with pytest.raises(moe.MoEError):
        moe.eplb_plan(np.ones(8), 3, 4)  # 11 slots over 4 owners
    with pytest.raises(moe.MoEError):
        moe.eplb_plan(np.ones(500), 20, 4)  # 520 slots
    c = binding.c_config(small_config(N=8, d=64, E=8, S=0, k=2, I=64, P=2))
    assert lib.moe_eplb_workspace_bytes(ctypes.byref(c)) > 0
    assert lib.moe_eplb_assign(ctypes.byref(c), None, None, None, 12, None, None, None, 0, None) \
        == binding.MOE_ERR_INVALID_ARG
    assert lib.moe_eplb_assign(ctypes.byref(c), None, None, None, 4, None, None, None, 0, None) \
        == binding.MOE_ERR_INVALID_ARG  # fewer slots than experts
    se = np.array([0, 1, 9], dtype=np.int32)  # expert 9 does not exist
    assert lib.moe_eplb_place_weights(ctypes.c_void_p(se.ctypes.data), 3, 8, 0, 16, ctypes.c_void_p(16),
                                      ctypes.c_void_p(16), None) == binding.MOE_ERR_INVALID_ARG



def test_capacity_rows_matches_the_oracle():
    """moe_capacity_rows (host) equals the oracle's ceil(factor * N * k / E)."""
    from oracle import moe_oracle as O
    for name in ("fine", "wide", "hot", "hot_cal", "tiny"):
        cfg = CONFIGS[name]
        for factor in (0.0, 0.5, 0.8, 1.0, 1.25, 1.3333, 2.0, 7.77):
            assert moe.capacity_of(factor, cfg) == O.capacity(factor, cfg.N, cfg.k, cfg.E), (name, factor)
    for bad in (-1.0, -1e-9, float("nan"), float("inf")):
        with pytest.raises(moe.MoEError) as e:
            moe.capacity_of(bad, CONFIGS["fine"])
        assert e.value.status == binding.MOE_ERR_INVALID_ARG


def test_noalloc_layout_refusals_say_why():
    """moe_dispatch_layout_noalloc refuses on the host (nothing is launched) and records
    the reason for moe_last_error, like the other entry points."""
    lib = binding.load()
    fake = ctypes.c_void_p(256)  # never dereferenced: every case below is refused first
    lay = binding.CLayout(*([256] * len(binding.LAYOUT_FIELDS)))
    big = binding.c_config(small_config(N=40000, d=64, E=256, S=0, k=8, I=64, P=32))
    assert lib.moe_dispatch_layout_noalloc(ctypes.byref(big), None, fake, ctypes.byref(lay), None, None) \
        == binding.MOE_ERR_UNSUPPORTED
    assert b"2 MiB" in lib.moe_last_error()
    small = binding.c_config(small_config(N=8, d=64, E=8, S=0, k=2, I=64, P=3))
    assert lib.moe_dispatch_layout_noalloc(ctypes.byref(small), None, fake, ctypes.byref(lay), None, None) \
        == binding.MOE_ERR_INVALID_ARG
    assert b"E % P" in lib.moe_last_error()
    small = binding.c_config(small_config(N=8, d=64, E=8, S=0, k=2, I=64, P=2))
    assert lib.moe_dispatch_layout_noalloc(ctypes.byref(small), None, fake, ctypes.byref(binding.CLayout()), None,
                                           None) == binding.MOE_ERR_INVALID_ARG
    assert b"non-NULL" in lib.moe_last_error()


def test_checked_build_loads_and_says_so():
    """libmoe_checked.so (-DMOE_CHECKS) exports the same symbols and reports itself as the
    bounds-checked build; the normal library does not."""
    import sys
    spec_root = ROOT
    b = __import__("importlib").util.spec_from_file_location(
        "_moe_build", os.path.join(spec_root, "dispatch_combine_grouped_b200", "build.py"))
    mod = __import__("importlib").util.module_from_spec(b)
    b.loader.exec_module(mod)
    path = mod.build(checked=True)
    lib = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(lib, name), name
    lib.moe_checks_enabled.restype = ctypes.c_int32
    assert lib.moe_checks_enabled() == 1
    assert binding.load().moe_checks_enabled() == 0
    assert lib.moe_checks_register(None) == binding.MOE_OK
    code = ("import dispatch_combine_grouped_b200 as m; import sys; "
            "sys.exit(0 if m.checks_enabled() and m.binding.LIB_PATH.endswith('libmoe_checked.so') else 3)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=dict(os.environ, MOE_LIB="checked"),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]


def test_mx_calls_refuse_unsupported_shapes_without_launching():
    """The MX entry points refuse, before any launch and with a reason: rows whose length
    is not a multiple of 32 (one E8M0 scale per 32 values), d % 512 != 0 or I % 128 != 0,
    an fp32 configuration, and NULL operands; the MX workspace covers the codes and scales."""
    lib = binding.load()
    assert lib.moe_quantize_mx(ctypes.c_void_p(16), 4, 48, ctypes.c_void_p(16), ctypes.c_void_p(16), None) \
        == binding.MOE_ERR_INVALID_ARG
    assert b"32" in lib.moe_last_error()
    assert lib.moe_quantize_mx(None, 4, 64, None, None, None) == binding.MOE_ERR_INVALID_ARG
    for kw, want in ((dict(d=256), binding.MOE_ERR_UNSUPPORTED), (dict(I=192), binding.MOE_ERR_UNSUPPORTED),
                     (dict(dtype="f32"), binding.MOE_ERR_UNSUPPORTED)):
        c = binding.c_config(small_config(N=8, d=512, E=8, S=1, k=2, I=128, P=2).replace(**kw))
        assert lib.moe_layer_forward_mx(ctypes.byref(c), None, None, None, None, None, None, None, None, None, None,
                                        None, None, 0, None) == want, kw
        assert lib.moe_grouped_ffn_mx(ctypes.byref(c), None, *([None] * 14)) == want, kw
    c = binding.c_config(small_config(N=8, d=512, E=8, S=1, k=2, I=128, P=2))
    lay = binding.CLayout()
    assert lib.moe_grouped_ffn_mx(ctypes.byref(c), ctypes.byref(lay), *([None] * 14)) == binding.MOE_ERR_INVALID_ARG
    wide = CONFIGS["wide"]
    A, S = wide.N * wide.k, wide.S
    need = A * wide.d * (1 + 1 / 32) + (A + S * wide.N) * (wide.I * (1 + 1 / 32) + wide.d * 2)
    assert moe.workspace_bytes_mx(wide) >= need
