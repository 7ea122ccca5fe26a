"""Pins of the oracle's expert-parallel layout (oracle.moe_oracle.ep_layout), on CPU.

The definition (owner j receives, for each of its experts in ascending id, the
assignments of source 0, then source 1, ..., each in ascending local index) is pinned
against: the hand-worked 4-token example (values derived on paper), the one-GPU layout
whose virtual sources are the ranks (written independently: send buffer -> transpose ->
stable sort by expert), and invariants on unequal shards and capacity cuts.
"""
import json
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def test_worked_example_two_ranks():
    """ep_deepep explainer §3/§6 and DeepEP notes §2 on the 4-token example: rank 0 holds
    t0, t1 and rank 1 holds t2, t3; owner 0 receives e0 {t0s0, t3s1} then e1 {t0s1, t1s0,
    t2s0}, owner 1 receives e2 {t2s1, t3s0} then e3 {t1s1}."""
    g = json.load(open(os.path.join(HERE, "golden", "worked_example_4tok.json")))
    ids = np.array(g["topk_ids"])
    lay = O.ep_layout([ids[:2], ids[2:]], E=4, P=2)
    cap = lay["capacity"]
    assert cap == 5  # owner 0 receives 5 rows, owner 1 three
    tok2row, recv_off = np.array(g["tok2row"]), np.array(g["recv_off"])
    owner = np.array([0, 0, 1, 1])
    flat = ids.reshape(-1)
    want = owner[flat] * cap + tok2row - recv_off[owner[flat]]
    assert np.array_equal(np.concatenate(lay["dest"]), want)
    assert np.array_equal(lay["dest"][0], [0, 2, 3, 7]) and np.array_equal(lay["dest"][1], [4, 5, 6, 1])
    assert np.array_equal(lay["cnt"], [[1, 2, 0, 1], [1, 1, 2, 0]])
    assert np.array_equal(lay["R"], np.diff(recv_off))
    assert np.array_equal(lay["owner_n_e"][0], [2, 3]) and np.array_equal(lay["owner_off"][0], [0, 2, 5])
    assert np.array_equal(lay["owner_n_e"][1], [2, 1]) and np.array_equal(lay["owner_off"][1], [0, 2, 3])
    # receive rows as (source, local a)
    assert lay["recv"][0].tolist() == [[0, 0], [1, 3], [0, 1], [0, 2], [1, 0]]
    assert lay["recv"][1].tolist() == [[1, 1], [1, 2], [0, 3]]


@pytest.mark.parametrize("seed", range(6))
def test_equal_shards_match_one_gpu_layout(seed):
    rng = np.random.default_rng(seed)
    P = [2, 4, 3][seed % 3]
    E = P * int(rng.integers(2, 6))
    k = int(rng.integers(1, min(4, E) + 1))
    n = int(rng.integers(1, 40))
    N = n * P
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(N)])
    if seed % 2:  # dropped assignments
        ids[rng.random(ids.shape) < 0.2] = -1
    owner = rng.integers(0, P, size=E) if seed >= 3 else None
    glob = O.dispatch_layout(ids, E, P, owner)
    lay = O.ep_layout([ids[i * n:(i + 1) * n] for i in range(P)], E, P, owner)
    cap = lay["capacity"]
    own = O.default_owner(E, P) if owner is None else owner
    flat = ids.reshape(-1)
    for i in range(P):
        for a in range(n * k):
            ga, e = i * n * k + a, flat[i * n * k + a]
            if e < 0:
                assert lay["dest"][i][a] == -1
                continue
            j = own[e]
            assert lay["dest"][i][a] == j * cap + glob["tok2row"][ga] - glob["recv_off"][j]
    assert np.array_equal(lay["R"], np.diff(glob["recv_off"]))
    for j in range(P):
        mine = lay["owned"][j]
        assert np.array_equal(lay["owner_n_e"][j], glob["n_e"][mine])
        assert np.array_equal(lay["owner_off"][j][:-1], glob["expert_off"][mine] - glob["recv_off"][j])
        assert lay["owner_off"][j][-1] == lay["R"][j]


@pytest.mark.parametrize("seed", range(4))
def test_unequal_shards_and_capacity(seed):
    rng = np.random.default_rng(100 + seed)
    P, E, k = 3, 9, 2
    ns = [int(v) for v in rng.integers(0, 30, size=P)]
    ids = [np.stack([rng.choice(E, size=k, replace=False) for _ in range(n)]) if n else np.zeros((0, k), int)
           for n in ns]
    full = O.ep_layout(ids, E, P)
    cap = max(1, int(full["R"].max()) - 3) if seed % 2 else None
    lay = O.ep_layout(ids, E, P, capacity=cap)
    cap = lay["capacity"]
    own = O.default_owner(E, P)
    for j in range(P):
        rows = lay["recv"][j]
        assert len(rows) == lay["R"][j]
        # order: expert id, then source, then local a (strictly increasing keys)
        keys = [(ids[i].reshape(-1)[a], i, a) for i, a in rows]
        assert keys == sorted(keys) and len(set(keys)) == len(keys)
        assert all(own[e] == j for e, _, _ in keys)
        received = min(int(lay["R"][j]), cap)
        assert lay["owner_n_e"][j].sum() == received and lay["owner_off"][j][-1] == received
        got = sorted(int(d) - j * cap for i in range(P) for d in lay["dest"][i] if d >= 0 and d // cap == j)
        assert got == list(range(received))
    assert np.array_equal(lay["cnt"].sum(axis=0),
                          np.bincount(np.concatenate([x.reshape(-1) for x in ids]), minlength=E))


def test_cross_rank_volume_matches_the_pages_estimate():
    """ep_deepep explainer, the EP communication estimate: with experts spread evenly over P
    ranks and routing independent of the token's rank, a fraction (P-1)/P of each rank's
    k assignments per token leaves the rank, each way.  Uniform random routing on 8 ranks."""
    rng = np.random.default_rng(7)
    P, E, k, n = 8, 64, 6, 512
    ids = [np.stack([rng.choice(E, size=k, replace=False) for _ in range(n)]) for _ in range(P)]
    lay = O.ep_layout(ids, E, P)
    cap = lay["capacity"]
    for r in range(P):
        dest = lay["dest"][r]
        leaving = int(((dest >= 0) & (dest // cap != r)).sum())   # rows the oracle sends to other owners
        assert abs(leaving / (n * k) - (P - 1) / P) < 0.03
    # and every assignment is received exactly once
    assert int(lay["R"].sum()) == P * n * k


def test_wide_ep_slot_arithmetic():
    """Wide EP page, 'why make EP wide': 256 experts + 32 redundant copies = 288 slots, 9 per
    rank on 32 ranks; the oracle's placement gives every owner exactly that many slots."""
    from oracle import eplb as L
    load = np.random.default_rng(3).integers(1, 1000, size=256)
    plan = L.plan(load, R=32, P=32)
    assert len(plan["slot_expert"]) == 288
    assert np.bincount(plan["slot_owner"], minlength=32).tolist() == [9] * 32
    assert sorted(np.bincount(plan["slot_expert"], minlength=256).tolist())[-1] >= 2  # hot experts copied
