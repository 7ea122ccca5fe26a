"""Host side of the expert-parallel binding, on CPU: the window's parts are laid out in
order without overlap and sized as the C ABI states, every rank computes the same offsets
whatever its own token count, and expert ownership follows the placement."""
import numpy as np
import pytest

from dispatch_combine_grouped_b200 import ep
from moe_inputs import small_config


@pytest.mark.parametrize("dtype,eb", [("bf16", 2), ("f32", 4)])
def test_window_parts_in_order_and_sized(dtype, eb):
    cfg = small_config("w", N=100, d=128, E=24, S=2, k=3, I=64, P=4, dtype=dtype)
    cap = 333
    o = ep.window_offsets(cfg, cap)
    names = ep.OFFSET_NAMES
    assert [o[n] for n in names] == sorted(o[n] for n in names)
    sizes = {"cnt_flag": 8 * ep.MAX_RANKS, "disp_flag": 8 * ep.MAX_RANKS, "done_flag": 8 * ep.MAX_RANKS, "step": 8,
             "disp_ctr": 4, "err_step": 8, "cnt_tab": 4 * cfg.P * cfg.E, "gate": 4 * cap, "scale": 4 * cap,
             "x_recv": cap * cfg.d * eb, "out_recv": (cap + cfg.S * cfg.N) * cfg.d * eb}
    for a, b in zip(names, names[1:]):
        assert o[a] + sizes[a] <= o[b], (a, b)
    for n in ["cnt_tab", "gate", "scale", "x_recv", "out_recv"]:
        assert o[n] % 256 == 0, n
    total = ep.window_bytes(cfg, cap)
    assert o["out_recv"] + sizes["out_recv"] <= total
    # another rank's token count changes only the size of the shared rows at the end
    o2 = ep.window_offsets(cfg.replace(N=7), cap)
    assert o2 == o
    assert ep.window_bytes(cfg.replace(N=7), cap) < total


def test_invalid_capacity_has_no_window():
    cfg = small_config("w", N=10, d=64, E=8, S=0, k=2, I=64, P=2)
    assert ep.window_bytes(cfg, 0) == 0 and ep.workspace_bytes(cfg, 0) == 0
    with pytest.raises(ValueError):
        ep.alloc_window(cfg, 0, device="cpu")


def test_owned_experts_follow_the_placement():
    assert ep.owned_experts(8, 4, 2) == [4, 5]
    table = np.array([3, 0, 3, 1, 0, 2, 2, 3])
    got = [ep.owned_experts(8, 4, r, table) for r in range(4)]
    assert got == [[1, 4], [3], [5, 6], [0, 2, 7]]
    assert sorted(sum(got, [])) == list(range(8))


def test_fp8_workspace_holds_more_than_bf16():
    cfg = small_config("w", N=64, d=128, E=8, S=1, k=2, I=64, P=2)
    assert ep.workspace_bytes_fp8(cfg, 200) > ep.workspace_bytes(cfg, 200) > 0
