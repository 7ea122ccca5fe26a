"""Pins for the CPU oracle (CPU only).

Each test ties the oracle to something other than itself: the hand-worked example and
the transpose figure under tests/golden/, closed forms, invariants the pages state,
brute force on tiny inputs, and special cases that reduce to library routines.
"""
import json
import math
import os

import numpy as np
import torch

from oracle import moe_oracle as O
from moe_inputs import MoEConfig, make_inputs, small_config

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- worked example (golden)
def check_worked_selection():
    g = _load("worked_example_4tok.json")
    z = np.array(g["logits"], dtype=np.float64)
    ids = O.select_experts(z, 2)
    assert ids.tolist() == g["topk_ids"]
    gates = O.gate_weights(z, ids, "softmax", True)
    np.testing.assert_allclose(gates, np.array(g["gates"]), rtol=0, atol=1e-12)


def check_worked_layout():
    g = _load("worked_example_4tok.json")
    lay = O.dispatch_layout(np.array(g["topk_ids"]), E=4, P=2)
    for key in ["n_e", "expert_off", "C", "send_off", "recv_off", "tok2send", "send2row",
                "ret2tok", "tok2row", "row2tok"]:
        assert lay[key].tolist() == g[key], key


def check_worked_output():
    g = _load("worked_example_4tok.json")
    ids = np.array(g["topk_ids"])
    gates = np.array(g["gates"])
    lay = O.dispatch_layout(ids, E=4, P=2)
    x = np.array([[1.0, -2.0], [0.5, 3.0], [-1.5, 0.25], [2.0, 1.0]])
    xp = O.permute(x, lay, 2)
    expert_of_row = ids.reshape(-1)[lay["row2tok"]]
    o = (expert_of_row + 1.0)[:, None] * xp          # scalar experts (e+1) * x
    y = O.combine(o, lay, gates, 4, 2)
    m = np.array(g["scalar_expert_multiplier"])
    np.testing.assert_allclose(y, m[:, None] * x, rtol=0, atol=1e-12)


def test_worked_example_selection_and_gates():
    check_worked_selection()


def test_worked_example_layout():
    check_worked_layout()


def test_worked_example_output():
    check_worked_output()


def test_transpose_figure_p3():
    """Each of 3 sources sends one row to each owner; owners receive source-major."""
    g = _load("a2a_transpose_p3.json")
    P = g["P"]
    # token 3i + ((j + i) % 3) of source i goes to expert j (= owner j, one expert per owner),
    # so the source must re-bucket its tokens by owner.
    ids = np.zeros((9, 1), dtype=np.int64)
    label = {}
    for i in range(P):
        for j in range(P):
            t = 3 * i + (j + i) % 3
            ids[t, 0] = j
            label[t] = f"{i}->{j}"
    lay = O.dispatch_layout(ids, E=3, P=3)
    send = [None] * 9
    for a in range(9):
        send[lay["tok2send"][a]] = label[a]
    assert [send[3 * i:3 * i + 3] for i in range(3)] == g["send_blocks"]
    recv = [None] * 9
    for a in range(9):
        recv[lay["tok2row"][a]] = label[a]
    ro = lay["recv_off"]
    assert [recv[ro[j]:ro[j + 1]] for j in range(3)] == g["recv_blocks"]


# ---------------------------------------------------------------- closed forms for gates
def test_gate_closed_forms():
    # sigmoid: sigma(0) = 1/2, sigma(ln 3) = 3/4 -> renormalised 0.4, 0.6
    z = np.array([[0.0, math.log(3.0), -5.0]])
    ids = np.array([[1, 0]])
    np.testing.assert_allclose(O.gate_weights(z, ids, "sigmoid", True), [[0.6, 0.4]], atol=1e-15)
    np.testing.assert_allclose(O.gate_weights(z, ids, "sigmoid", False), [[0.75, 0.5]], atol=1e-15)
    # softmax without renormalisation over equal logits: 1/E each
    z = np.zeros((2, 8))
    ids = np.array([[0, 1, 2], [5, 6, 7]])
    np.testing.assert_allclose(O.gate_weights(z, ids, "softmax", False), np.full((2, 3), 1 / 8), atol=1e-15)
    # softmax over [ln 1, ln 2, ln 5] -> 1/8, 2/8, 5/8
    z = np.log(np.array([[1.0, 2.0, 5.0]]))
    ids = np.array([[2, 1]])
    np.testing.assert_allclose(O.gate_weights(z, ids, "softmax", False), [[5 / 8, 2 / 8]], atol=1e-15)
    np.testing.assert_allclose(O.gate_weights(z, ids, "softmax", True), [[5 / 7, 2 / 7]], atol=1e-15)


# ---------------------------------------------------------------- brute force selection
def check_selection_brute_force(seed=0):
    rng = np.random.default_rng(seed)
    for (E, k, G, tg) in [(8, 2, 1, 1), (8, 3, 1, 1), (6, 1, 1, 1), (8, 2, 4, 2), (8, 3, 4, 2),
                          (8, 2, 2, 1), (6, 2, 3, 2)]:
        keys = rng.integers(-2, 3, size=(48, E)).astype(np.float64)   # many ties
        keys[::5] = rng.normal(size=(len(keys[::5]), E))
        a = O.select_experts(keys, k, G, tg)
        b = O.brute_force_select(keys, k, G, tg)
        assert np.array_equal(a, b), (E, k, G, tg)


def test_selection_brute_force():
    check_selection_brute_force()


def test_group_limited_hand_case():
    # 4 groups of 2. Group maxima: g0=1, g1=9, g2=9, g3=8 -> keep groups 1,2 (tie 9/9, both kept)
    # with topk_groups=2; top-3 among experts 2..5: keys [5,9,9,0] -> 3, 4 (tie -> lower), 2
    keys = np.array([[1, 0, 5, 9, 9, 0, 8, 7.5]])
    assert O.select_experts(keys, 3, 4, 2).tolist() == [[3, 4, 2]]
    # expert 6 (key 8) beats expert 2 (key 5) globally but its group is not kept
    assert O.select_experts(keys, 3, 1, 1).tolist() == [[3, 4, 6]]


# ---------------------------------------------------------------- layout invariants
def _random_routing(rng, N, E, k):
    # distinct experts per token, random order, skewed so some experts are empty
    p = rng.dirichlet(np.full(E, 0.3))
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(N)])
    return ids


LAYOUT_CASES = [(1, 4, 1, 1), (7, 8, 2, 2), (33, 8, 2, 4), (64, 16, 4, 4), (129, 32, 8, 8),
                (10, 12, 3, 4), (5, 8, 2, 8)]


def check_layout_invariants(ids, E, P, owner=None):
    N, k = ids.shape
    A = N * k
    lay = O.dispatch_layout(ids, E, P, owner)
    own = O.default_owner(E, P) if owner is None else np.asarray(owner)
    src = O.source_of_token(N, P)
    n_e, C = lay["n_e"], lay["C"]
    assert n_e.sum() == A                                   # sum_e n_e = N k
    shard_sizes = np.bincount(src, minlength=P)
    assert np.array_equal(C.sum(axis=1), k * shard_sizes)    # every token sends k
    R = np.array([n_e[own == j].sum() for j in range(P)])
    assert np.array_equal(C.sum(axis=0), R)                  # R_r = sum_i C_ir
    assert np.array_equal(np.diff(lay["recv_off"]), R)
    t2r, t2s = lay["tok2row"], lay["tok2send"]
    assert sorted(t2r.tolist()) == list(range(A))
    assert sorted(t2s.tolist()) == list(range(A))
    assert np.array_equal(lay["row2tok"][t2r], np.arange(A))
    assert np.array_equal(lay["send2row"][t2s], t2r)         # send2row o tok2send = tok2row
    assert np.array_equal(lay["ret2tok"][t2s], np.arange(A)) # ret2tok o tok2send = id
    flat = ids.reshape(-1)
    for e in range(E):
        rows = lay["row2tok"][lay["expert_off"][e]:lay["expert_off"][e] + n_e[e]]
        assert np.all(flat[rows] == e)
        assert np.all(np.diff(rows) > 0)                     # ascending (token, slot)
    for i in range(P):
        for j in range(P):
            s0 = lay["send_off"][i, j]
            blk = lay["ret2tok"][s0:s0 + C[i, j]]
            assert np.all(src[blk // k] == i) and np.all(own[flat[blk]] == j)
            assert np.all(np.diff(blk) > 0)
    return lay


def test_layout_invariants():
    rng = np.random.default_rng(1)
    for (N, E, k, P) in LAYOUT_CASES:
        ids = _random_routing(rng, N, E, k)
        check_layout_invariants(ids, E, P)
        own = rng.permutation(np.arange(E) % P)              # arbitrary placement
        check_layout_invariants(ids, E, P, own)


def check_layout_naive_ranks(seed=2):
    """Every map against an O(A^2) count written from the definitions."""
    rng = np.random.default_rng(seed)
    for (N, E, k, P) in LAYOUT_CASES:
        ids = _random_routing(rng, N, E, k)
        own = rng.permutation(np.arange(E) % P) if seed % 2 == 0 else O.default_owner(E, P)
        lay = O.dispatch_layout(ids, E, P, own)
        flat = ids.reshape(-1)
        A = N * k
        src = O.source_of_token(N, P)[np.arange(A) // k]
        dst = np.asarray(own)[flat]
        order_key = [(own[e], e) for e in range(E)]
        for a in range(A):
            e = flat[a]
            base = sum(int((flat == f).sum()) for f in range(E) if order_key[f] < order_key[e])
            assert lay["tok2row"][a] == base + int((flat[:a] == e).sum())
            before = int(sum(((src == i2) & (dst == j2)).sum()
                             for i2 in range(P) for j2 in range(P) if (i2, j2) < (src[a], dst[a])))
            same = int(((src[:a] == src[a]) & (dst[:a] == dst[a])).sum())
            assert lay["tok2send"][a] == before + same


def test_layout_naive_ranks():
    check_layout_naive_ranks(2)
    check_layout_naive_ranks(3)


def test_layout_matches_stable_argsort_for_contiguous_owners():
    rng = np.random.default_rng(4)
    for (N, E, k, P) in LAYOUT_CASES:
        ids = _random_routing(rng, N, E, k)
        lay = O.dispatch_layout(ids, E, P)
        assert np.array_equal(lay["row2tok"], np.argsort(ids.reshape(-1), kind="stable"))
        assert np.array_equal(lay["expert_off"][:-1],
                              np.concatenate([[0], np.cumsum(lay["n_e"])[:-1]]))


def test_tile_prefix():
    ids = np.array([[0]] * 130 + [[2]] * 5)
    lay = O.dispatch_layout(ids, E=3, P=1, S=2)
    assert lay["tile_off"].tolist() == [0, 2, 2, 3, 5, 7]   # ceil(130/128)=2, 0, 1, 2 x ceil(135/128)


# ---------------------------------------------------------------- identity / round trip
def check_round_trip(score="softmax", renorm=True, seed=5):
    rng = np.random.default_rng(seed)
    N, E, k, P, d = 37, 8, 3, 4, 5
    x = rng.normal(size=(N, d))
    z = rng.normal(size=(N, E))
    ids = O.select_experts(z, k)
    g = O.gate_weights(z, ids, score, renorm)
    lay = O.dispatch_layout(ids, E, P)
    y = O.combine(O.permute(x, lay, k), lay, g, N, k)        # identity experts
    np.testing.assert_allclose(y, x * g.sum(axis=1, keepdims=True), rtol=1e-14, atol=1e-14)
    return y, x, g


def test_round_trip_identity():
    y, x, g = check_round_trip("softmax", True)
    np.testing.assert_allclose(y, x, rtol=1e-13, atol=1e-13)  # renormalised gates sum to 1
    check_round_trip("sigmoid", True)
    check_round_trip("softmax", False)
    check_round_trip("sigmoid", False)


# ---------------------------------------------------------------- library special cases
def _torch_swiglu(x, w13, w2):
    x, w13, w2 = (torch.as_tensor(np.asarray(a, dtype=np.float64)) for a in (x, w13, w2))
    I = w13.shape[0] // 2
    h = torch.nn.functional.silu(x @ w13[:I].T) * (x @ w13[I:].T)
    return (h @ w2.T).numpy()


def check_dense_special_case():
    """E=1, k=1, no shared expert: the layer is one dense SwiGLU MLP (gate = 1)."""
    cfg = small_config(cfg_id=91, N=19, d=24, E=1, S=0, k=1, I=16, P=1, dtype="f32")
    inp = make_inputs(cfg)
    out = O.moe_layer(cfg, inp["x"], inp["w_gate"], None, inp["w13"], inp["w2"])
    ref = _torch_swiglu(inp["x"].double(), inp["w13"][0].double(), inp["w2"][0].double())
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def test_dense_special_case():
    check_dense_special_case()


def check_expert_vs_torch():
    rng = np.random.default_rng(6)
    x = rng.normal(size=(9, 12))
    w13 = rng.normal(size=(2 * 7, 12))
    w2 = rng.normal(size=(12, 7))
    np.testing.assert_allclose(O.swiglu_expert(x, w13, w2), _torch_swiglu(x, w13, w2), rtol=1e-12, atol=1e-12)


def test_expert_vs_torch():
    check_expert_vs_torch()


def check_shared_expert_additive():
    """With gates forced to 0 the layer output is exactly the shared experts' sum."""
    cfg = small_config(cfg_id=92, N=11, d=16, E=4, S=2, k=2, I=8, P=2, dtype="f32")
    inp = make_inputs(cfg)
    x = O.f64(inp["x"])
    w13, w2 = O.f64(inp["w13"]), O.f64(inp["w2"])
    ids = O.select_experts(O.router_logits(x, inp["w_gate"]), 2)
    y = O.moe_tokens_direct(cfg, x, ids, np.zeros((11, 2)), w13, w2, range(11))
    ref = _torch_swiglu(x, w13[4], w2[4]) + _torch_swiglu(x, w13[5], w2[5])
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_shared_expert_additive():
    check_shared_expert_additive()


# ---------------------------------------------------------------- two formulations agree
def check_layout_path_equals_equation(cfg):
    inp = make_inputs(cfg)
    out = O.moe_layer(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["w13"], inp["w2"],
                      inp["expert_owner"])
    direct = O.moe_tokens_direct(cfg, inp["x"], out["ids"], out["gates"], inp["w13"], inp["w2"],
                                 np.arange(cfg.N))
    np.testing.assert_allclose(out["y"], direct, rtol=1e-12, atol=1e-12)


def test_layout_path_equals_output_equation():
    check_layout_path_equals_equation(small_config(cfg_id=93, N=41, d=32, E=8, S=1, k=2, I=24, P=4))
    check_layout_path_equals_equation(small_config(cfg_id=94, N=24, d=16, E=16, S=0, k=4, I=8, P=4,
                                                   n_groups=4, topk_groups=2, score="sigmoid"))


def test_permutation_invariance():
    cfg = small_config(cfg_id=95, N=30, d=16, E=8, S=1, k=2, I=12, P=4, dtype="f32")
    inp = make_inputs(cfg)
    perm = np.random.default_rng(7).permutation(cfg.N)
    a = O.moe_layer(cfg, inp["x"], inp["w_gate"], None, inp["w13"], inp["w2"])["y"]
    b = O.moe_layer(cfg, inp["x"][perm], inp["w_gate"], None, inp["w13"], inp["w2"])["y"]
    np.testing.assert_allclose(b, a[perm], rtol=1e-12, atol=1e-12)


def test_imbalance_and_page_arithmetic():
    assert O.imbalance([1, 1, 4, 2]) == 2.0
    # Wide EP: 256 routed + 32 redundant slots over 32 / 144 ranks (E_local = (E+R)/P_e)
    assert (256 + 32) // 32 == 9 and (256 + 32) // 144 == 2
    # decode concurrency for 16 rows per expert: N_active >= 16 * 256 / 8 = 512
    assert 16 * 256 // 8 == 512
    # tiny config: mean n_e = N k / E
    lay = O.dispatch_layout(np.arange(512).reshape(256, 2) % 8, E=8, P=2)
    assert lay["n_e"].mean() == 256 * 2 / 8


def check_correction_bias():
    """The bias steers the selection only: keys z + b pick (1, 0) over z's own (0, 2);
    the renormalised softmax gates then come from z: (e^0, e^1) / (e^0 + e^1)."""
    cfg = MoEConfig("cb", 0, N=1, d=3, E=3, S=0, k=2, I=8, P=1, score="softmax", renormalize=True,
                    dtype="f32", bias="zipf", bias_mode="selection")
    x = np.array([[1.0, 0.0, 0.5]])
    w_gate = np.eye(3)                                     # z = x
    bias = np.array([0.0, 2.0, 0.0])
    keys = O.router_logits(x, w_gate, bias)
    ids = O.select_experts(keys, 2)
    assert ids.tolist() == [[1, 0]]
    g = O.gate_weights(O.gate_logits(cfg, x, w_gate, bias), ids, cfg.score, cfg.renormalize)
    e = math.e
    np.testing.assert_allclose(g, [[1 / (1 + e), e / (1 + e)]], atol=1e-15)
    # the default mode feeds the bias to the gates too
    g2 = O.gate_weights(O.gate_logits(cfg.replace(bias_mode="logits"), x, w_gate, bias), ids, "softmax", True)
    np.testing.assert_allclose(g2, [[e ** 2 / (e ** 2 + e), e / (e ** 2 + e)]], atol=1e-15)


def test_correction_bias_closed_form():
    check_correction_bias()
