"""GPU parity at the five full workload sizes (the bench's launch configuration).

Routing and layout are checked completely (bit-exact against the oracle run on the
GPU's fp32 logits).  The grouped GEMMs are checked on rows chosen so that every tile
they run is compared with the oracle: for every routed expert and every shared expert,
the first and the last row of each 128-row block of its rows (so every 256-row CTA-pair
tile, both CTAs of it, and every 0..128-row tail tile), element by element, for h (the
SwiGLU activations after FC1) and for the gate-scaled FC2 rows.  y is checked on sampled
tokens that the oracle computes one by one from the output equation.
"""
import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import CONFIGS
from oracle import moe_oracle as O
from tests.gpu_cases import (assert_close_fro, assert_close_rel, assert_layout_equal, check_route, gpu_inputs,
                             layout_to_numpy, run_steps)

pytestmark = pytest.mark.gpu

FULL = ["fine", "wide", "decode", "hot", "hot_cal"]
SAMPLE_TOKENS = {"fine": 8, "wide": 4, "decode": 4, "hot": 8, "hot_cal": 8}
BLOCK = 128  # row block of the grouped GEMM tiles (a CTA-pair tile spans two)


def block_edge_rows(r0, n):
    """The first and the last row of every 128-row block of the rows [r0, r0 + n)."""
    rows = []
    for b0 in range(r0, r0 + n, BLOCK):
        rows += [b0, min(b0 + BLOCK, r0 + n) - 1]
    return sorted(set(rows))


def check_every_tile(cfg, inp, res, ref, gates):
    """h and gate-scaled FC2 rows of every group's block edges against the float64 SwiGLU
    expert ([EP-DeepEP] §2 Expert_e; [MoE-IV] §4.1 FC1, activation, FC2)."""
    A, N, k, I = cfg.N * cfg.k, cfg.N, cfg.k, cfg.I
    x64 = O.f64(inp["x"])
    g_flat = gates.reshape(-1)
    checked, experts = 0, 0
    groups = [(e, int(ref["expert_off"][e]), int(ref["n_e"][e])) for e in range(cfg.E)]
    groups += [(cfg.E + s, A + s * N, N) for s in range(cfg.S)]
    for e, r0, n in groups:
        if n == 0:
            continue
        rows = np.array(block_edge_rows(r0, n))
        if e < cfg.E:
            a = ref["row2tok"][rows]              # assignment of each row
            tok, gate = a // k, g_flat[a]
        else:
            tok, gate = rows - r0, np.ones(len(rows))
        w13 = O.f64(inp["w13"][e])
        xr = x64[tok]
        h_ref = O.silu(xr @ w13[:I].T) * (xr @ w13[I:].T)
        o_ref = (h_ref @ O.f64(inp["w2"][e]).T) * gate[:, None]
        idx = torch.tensor(rows, device="cuda")
        assert_close_rel(res["h"][idx], h_ref, what=f"{cfg.name} h of group {e}")
        assert_close_fro(res["out"][idx], o_ref, what=f"{cfg.name} FC2 x gate of group {e}")
        checked += len(rows)
        experts += 1
    return checked, experts


@pytest.mark.parametrize("name", FULL)
def test_full_config(name):
    cfg = CONFIGS[name]
    inp = gpu_inputs(cfg)
    res = run_steps(cfg, inp)
    ids, n_diff = check_route(cfg, inp, res, 1e-3)
    print(f"{name}: tokens routed differently by fp64 selection: {n_diff}")
    ref = O.dispatch_layout(ids, cfg.E, cfg.P, inp["expert_owner"], cfg.S)
    lay = layout_to_numpy(res["layout"])
    assert_layout_equal(lay, ref, cfg.P)
    if name.startswith("hot"):
        R = np.diff(ref["recv_off"])
        print(f"{name}: max/mean n_e = {O.imbalance(ref['n_e']):.2f}, owner max/mean = {O.imbalance(R):.2f}")

    rng = np.random.default_rng(0)
    A = cfg.N * cfg.k
    a_s = rng.choice(A, size=min(A, 2048), replace=False)
    xp = res["x_perm"][torch.tensor(ref["tok2row"][a_s], device="cuda")]
    assert torch.equal(xp, inp["x"][torch.tensor(a_s // cfg.k, device="cuda")]), "permute rows"

    # every tile of the grouped GEMMs: block-edge rows of every group, element by element
    g_all = O.gate_weights(O.gate_logits(cfg, inp["x"], inp["w_gate"], inp["bias"]), ids, cfg.score,
                           cfg.renormalize)
    n_rows, n_groups = check_every_tile(cfg, inp, res, ref, g_all)
    print(f"{name}: {n_rows} rows of h and FC2 output checked over {n_groups} groups")
    assert n_groups == int((ref["n_e"] > 0).sum()) + cfg.S

    tokens = np.sort(rng.choice(cfg.N, size=SAMPLE_TOKENS[name], replace=False))
    z64 = O.gate_logits(cfg, inp["x"][torch.tensor(tokens, device="cuda")], inp["w_gate"], inp["bias"])
    g64 = O.gate_weights(z64, ids[tokens], cfg.score, cfg.renormalize)
    gates = np.zeros((cfg.N, cfg.k))
    gates[tokens] = g64
    y_ref = O.moe_tokens_direct(cfg, inp["x"], ids, gates, inp["w13"], inp["w2"], tokens)
    assert_close_fro(res["y"][torch.tensor(tokens, device="cuda")], y_ref, what=f"{name} sampled y")

    # the fused entry point runs the same kernels: bit-identical output
    y = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"])
    torch.cuda.synchronize()
    assert torch.equal(y, res["y"])


@pytest.mark.parametrize("name,P", [("wide", 8), ("fine", 8)])
def test_full_config_expert_parallel_emulated(name, P):
    """The expert-parallel path at full size with P ranks emulated on one GPU (the
    `bench.py --ep P` configuration): the EP layout of every rank bit-exact against the
    oracle's, sampled received rows and gates bit-exact, and y bit-identical to the
    one-GPU layer (itself checked against the oracle above)."""
    from dispatch_combine_grouped_b200 import ep
    cfg = CONFIGS[name].replace(P=P)
    inp = gpu_inputs(cfg)
    n = cfg.N // P
    rc = cfg.replace(N=n)
    cap = 2 * -(-cfg.N * cfg.k // P)
    groups, windows = ep.emulated_groups(rc, cap)
    ws = [ep.alloc_ws(rc, cap) for _ in range(P)]
    hd = [ep.Handle(rc, cfg.E // P) for _ in range(P)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    E, S = cfg.E, cfg.S
    xs = [inp["x"][r * n:(r + 1) * n] for r in range(P)]
    routed = [moe.route(rc, xs[r], inp["w_gate"], inp["bias"]) for r in range(P)]
    for r in range(P):
        ep.notify(rc, groups[r], routed[r][1], ws[r], status)
    for r in range(P):
        ep.layout(rc, groups[r], routed[r][1], hd[r], ws[r], None, status)
    for r in range(P):
        ep.dispatch(rc, groups[r], xs[r], routed[r][2], hd[r])
    for r in range(P):
        idx = torch.tensor(list(range(r * E // P, (r + 1) * E // P)) + list(range(E, E + S)), device="cuda")
        ep.expert_ffn(rc, groups[r], xs[r], inp["w13"].index_select(0, idx), inp["w2"].index_select(0, idx), hd[r],
                      ws[r], status)
    ys = [ep.combine(rc, groups[r], hd[r], status=status) for r in range(P)]
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    lay = O.ep_layout([rt[1].cpu().numpy() for rt in routed], cfg.E, P, None, cap)
    rng = np.random.default_rng(1)
    for r in range(P):
        h = hd[r].as_dict()
        assert np.array_equal(h["dest"].cpu().numpy(), lay["dest"][r]), f"dest of rank {r}"
        assert np.array_equal(h["owner_n_e"].cpu().numpy(), lay["owner_n_e"][r])
        assert np.array_equal(h["owner_off"].cpu().numpy(), lay["owner_off"][r])
        v = ep.window_views(rc, cap, windows[r])
        assert np.array_equal(v["cnt_tab"].cpu().numpy(), lay["cnt"])
        rows = lay["recv"][r]
        pick = rng.choice(len(rows), size=min(256, len(rows)), replace=False)
        for q in pick:
            i, a = rows[q]
            assert torch.equal(v["x_recv"][q], xs[i][a // cfg.k]), f"received row {q} of owner {r}"
            assert v["gate"][q].item() == routed[i][2].reshape(-1)[a].item()
    y1 = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], None, inp["w13"], inp["w2"])
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys), y1)
