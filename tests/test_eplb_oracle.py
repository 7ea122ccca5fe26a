"""Pins of the EPLB oracle (redundant expert slots) against facts fixed independently of
its code: a hand-worked example, brute-force optimality of the copy counts, the
invariants the pages state (a replica serves the router's chosen logical expert; copies
share its load), and the layer's output, which replicas must not change.

Source: "Wide EP：当 MoE Expert Parallel 横跨几十张 GPU", sections "为什么要把 EP 做宽",
"Expert 副本在 Wide EP 中还有整除作用" and "Group-limited routing".
"""
import itertools
import json
import os

import numpy as np
import pytest

from moe_inputs import make_inputs, small_config
from oracle import eplb as EP
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "eplb_example.json")


def check_worked_example():
    g = json.load(open(GOLDEN))
    pl = EP.plan(g["load"], g["R"], g["P"])
    for key in ("copies", "owner_loads", "slot_expert", "slot_owner", "replica_off", "replica_slots"):
        assert pl[key if key != "owner_loads" else "owner_load"].tolist() == g[key], key
    assert EP.assign(g["ids"], pl["replica_off"], pl["replica_slots"]).tolist() == g["phys_ids"]


def test_worked_example():
    check_worked_example()


def check_copy_counts_optimal(E, R, load):
    """Reading 1 minimises max_e load_e / r_e: compare with every way to hand out R copies."""
    r = EP.replica_counts(load, R)
    assert r.sum() == E + R and r.min() >= 1
    best = None
    for extra in itertools.product(range(R + 1), repeat=E):
        if sum(extra) != R:
            continue
        worst = max(load[e] / (1 + extra[e]) for e in range(E))
        best = worst if best is None else min(best, worst)
    assert max(load[e] / r[e] for e in range(E)) == pytest.approx(best, rel=0, abs=1e-12)


@pytest.mark.parametrize("E,R", [(2, 3), (3, 2), (4, 3), (4, 4)])
def test_copy_counts_are_optimal(E, R):
    rng = np.random.default_rng(E * 10 + R)
    for _ in range(20):
        load = rng.integers(0, 50, size=E)
        check_copy_counts_optimal(E, R, load)


def test_plan_is_a_valid_placement():
    rng = np.random.default_rng(3)
    for E, R, P in [(8, 4, 4), (16, 16, 8), (32, 0, 8), (128, 16, 16), (256, 32, 32), (6, 3, 9)]:
        load = rng.zipf(1.3, size=E).astype(np.int64)
        pl = EP.plan(load, R, P)
        S, per = E + R, (E + R) // P
        assert np.bincount(pl["slot_expert"], minlength=E).tolist() == pl["copies"].tolist()
        assert (pl["slot_owner"] == np.arange(S) // per).all()
        for e in range(E):
            slots = pl["replica_slots"][pl["replica_off"][e]:pl["replica_off"][e + 1]]
            assert len(set(slots.tolist())) == len(slots) and (pl["slot_expert"][slots] == e).all()
            if pl["copies"][e] <= P:  # copies of one expert land on distinct owners here
                assert len(set(pl["slot_owner"][slots].tolist())) == len(slots)
        assert sorted(pl["replica_slots"].tolist()) == list(range(S))
        assert pl["owner_load"].sum() == load.sum()


def test_identity_replicas_are_the_plain_routing():
    """R = 0 with the identity slot table: every assignment keeps its expert id."""
    rng = np.random.default_rng(5)
    ids = rng.integers(0, 16, size=(50, 4))
    assert (EP.assign(ids, np.arange(17), np.arange(16)) == ids).all()


def test_assignment_keeps_the_expert_and_splits_its_load():
    rng = np.random.default_rng(6)
    E, R, P, N, k = 16, 8, 8, 300, 4
    ids = np.stack([rng.permutation(E)[:k] for _ in range(N)])
    load = np.bincount(ids.reshape(-1), minlength=E)
    pl = EP.plan(load, R, P)
    phys = EP.assign(ids, pl["replica_off"], pl["replica_slots"])
    assert (pl["slot_expert"][phys] == ids).all()  # the router's choice is kept
    n_slot = np.bincount(phys.reshape(-1), minlength=E + R)
    for e in range(E):
        per = n_slot[pl["replica_slots"][pl["replica_off"][e]:pl["replica_off"][e + 1]]]
        assert per.sum() == load[e] and per.max() - per.min() <= 1
        # the plan's copy loads are exactly the rows the assignment delivers
        assert per.tolist() == [EP.copy_load(load[e], len(per), c) for c in range(len(per))]
    n_owner = np.bincount(pl["slot_owner"][phys.reshape(-1)], minlength=P)
    assert n_owner.tolist() == pl["owner_load"].tolist()


def check_layer_unchanged_by_replicas(R):
    """The layer over E + R physical slots with copied weights equals the logical layer
    (float64, exactly: every row meets the same weights)."""
    cfg = small_config(cfg_id=96, N=40, d=24, E=8, S=1, k=2, I=16, P=4, dtype="f32")
    inp = make_inputs(cfg, device="cpu")
    ref = O.moe_layer(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["w13"], inp["w2"])
    pl = EP.plan(np.bincount(ref["ids"].reshape(-1), minlength=cfg.E), R, cfg.P)
    phys = EP.assign(ref["ids"], pl["replica_off"], pl["replica_slots"])
    Ep = cfg.E + R
    lay = O.dispatch_layout(phys, Ep, cfg.P, None, cfg.S)
    w13p = EP.physical_weights(inp["w13"], pl["slot_expert"], cfg.E)
    w2p = EP.physical_weights(inp["w2"], pl["slot_expert"], cfg.E)
    o = O.experts_on_rows(O.permute(inp["x"], lay, cfg.k), lay, w13p, w2p, Ep)
    shared = [O.swiglu_expert(inp["x"], w13p[Ep + s], w2p[Ep + s]) for s in range(cfg.S)]
    y = O.combine(o, lay, ref["gates"], cfg.N, cfg.k, shared)
    np.testing.assert_array_equal(y, ref["y"])


@pytest.mark.parametrize("R", [0, 4, 8])
def test_layer_unchanged_by_replicas(R):
    check_layer_unchanged_by_replicas(R)
