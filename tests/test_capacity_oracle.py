"""Pins of the capacity-factor variant of the oracle (dropped assignments) against a
hand-worked layout, the special cases no-drop and drop-all, and the output equation.

Source: the ep_deepep explainer §4 ("容量因子与负载不均衡决定长尾": a capacity factor caps
the tokens one expert receives per round; the excess may be dropped), §3 and §6 for the
layout itself.
"""
import json
import os

import numpy as np

from moe_inputs import make_inputs, small_config
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "capacity_example.json")


def check_worked_example():
    g = json.load(open(GOLDEN))
    kept = O.capacity_keep(g["ids"], g["E"], g["capacity"])
    assert kept.tolist() == g["kept_ids"]
    lay = O.dispatch_layout(kept, g["E"], g["P"])
    for key in ("n_e", "expert_off", "C", "send_off", "recv_off", "tok2send", "send2row", "ret2tok", "tok2row",
                "row2tok"):
        assert lay[key].tolist() == g[key], key


def test_worked_example():
    check_worked_example()


def test_capacity_formula():
    assert O.capacity(1.0, 4096, 6, 64) == 384
    assert O.capacity(1.25, 4096, 6, 64) == 480
    assert O.capacity(1.1, 100, 3, 7) == 48  # ceil(47.14...)


def test_large_capacity_drops_nothing_and_zero_capacity_drops_everything():
    rng = np.random.default_rng(0)
    ids = np.stack([rng.permutation(8)[:2] for _ in range(50)])
    n_max = np.bincount(ids.reshape(-1)).max()
    assert np.array_equal(O.capacity_keep(ids, 8, n_max), ids)
    assert np.array_equal(O.dispatch_layout(O.capacity_keep(ids, 8, n_max), 8, 4)["tok2row"],
                          O.dispatch_layout(ids, 8, 4)["tok2row"])
    none = O.capacity_keep(ids, 8, 0)
    assert (none == -1).all()
    lay = O.dispatch_layout(none, 8, 4)
    assert lay["n_e"].sum() == 0 and (lay["tok2row"] == -1).all() and lay["expert_off"][-1] == 0


def test_kept_assignments_are_the_first_of_each_expert():
    rng = np.random.default_rng(1)
    ids = np.stack([rng.permutation(16)[:4] for _ in range(200)])
    cap = 30
    kept = O.capacity_keep(ids, 16, cap).reshape(-1)
    flat = ids.reshape(-1)
    for e in range(16):
        pos = np.flatnonzero(flat == e)
        assert np.array_equal(np.flatnonzero(kept == e), pos[:cap])
    lay = O.dispatch_layout(kept.reshape(ids.shape), 16, 4)
    live = np.flatnonzero(kept >= 0)
    assert np.array_equal(np.sort(lay["tok2row"][live]), np.arange(len(live)))
    assert np.array_equal(lay["row2tok"][lay["tok2row"][live]], live)
    assert np.array_equal(lay["send2row"][lay["tok2send"][live]], lay["tok2row"][live])
    assert lay["C"].sum() == len(live)


def check_layout_path_with_drops(factor):
    """permute -> experts -> combine over the kept rows equals the output equation with
    the dropped assignments left out."""
    cfg = small_config(cfg_id=97, N=60, d=24, E=8, S=1, k=2, I=16, P=4, dtype="f32")
    inp = make_inputs(cfg, device="cpu")
    ref = O.moe_layer(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["w13"], inp["w2"])
    kept = O.capacity_keep(ref["ids"], cfg.E, O.capacity(factor, cfg.N, cfg.k, cfg.E))
    lay = O.dispatch_layout(kept, cfg.E, cfg.P, None, cfg.S)
    o = O.experts_on_rows(O.permute(inp["x"], lay, cfg.k), lay, inp["w13"], inp["w2"], cfg.E)
    shared = [O.swiglu_expert(inp["x"], inp["w13"][cfg.E + s], inp["w2"][cfg.E + s]) for s in range(cfg.S)]
    y = O.combine(o, lay, ref["gates"], cfg.N, cfg.k, shared)
    y_direct = O.moe_tokens_direct(cfg, inp["x"], kept, ref["gates"], inp["w13"], inp["w2"], np.arange(cfg.N))
    np.testing.assert_allclose(y, y_direct, rtol=1e-12, atol=1e-12)
    return (kept == -1).sum()


def test_layout_path_with_drops():
    assert check_layout_path_with_drops(0.8) > 0
    assert check_layout_path_with_drops(1.0) >= 0
