"""GPU parity of the capacity-factor variant (dropped assignments) through the C ABI.

The capacity cut and the layout with dropped assignments are compared with the oracle
bit for bit (every map, including the -1 marks); the layer over the kept assignments is
compared with the output equation with the dropped ones left out.

Source: the ep_deepep explainer §4 (capacity factor; the excess is dropped), §3 and §6.
"""
import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import CONFIGS, small_config
from oracle import moe_oracle as O
from tests.gpu_cases import assert_close_fro, assert_layout_equal, gpu_inputs, layout_to_numpy

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cap", [0, 1, 17, 60, 10 ** 6])
def test_capacity_cut_and_layout_match_oracle(cap):
    E, P, N, k = 16, 4, 500, 4
    rng = np.random.default_rng(cap % 1000)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(N)])
    ids[rng.random(N) < 0.3, 0] = 0  # a hot expert
    cfg = small_config("cap", N=N, d=64, E=E, S=1, k=k, I=64, P=P)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kept = moe.capacity_drop(cfg, torch.tensor(ids, dtype=torch.int32, device="cuda"), cap, status=status)
    lay = moe.dispatch_layout(cfg, kept, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    kept_ref = O.capacity_keep(ids, E, cap)
    assert np.array_equal(kept.cpu().numpy(), kept_ref)
    ref = O.dispatch_layout(kept_ref, E, P, None, cfg.S)
    assert_layout_equal(layout_to_numpy(lay), ref, P)


SMALL = [
    small_config("c_bf16", cfg_id=88, N=700, d=256, E=16, S=1, k=4, I=128, P=8),
    small_config("c_bf16_pairs", cfg_id=89, N=640, d=4096, E=8, S=1, k=2, I=192, P=4),
    small_config("c_f32", cfg_id=98, N=129, d=96, E=8, S=0, k=2, I=72, P=4, dtype="f32"),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
@pytest.mark.parametrize("factor", [0.0, 0.7, 1.0, 1.25])
def test_layer_with_capacity(cfg, factor):
    inp = gpu_inputs(cfg)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    kept = moe.capacity_drop(cfg, ids, moe.capacity_of(factor, cfg), status=status)
    lay = moe.dispatch_layout(cfg, kept, inp["expert_owner"], status=status)
    xp = moe.permute(cfg, lay, inp["x"])
    h, out = moe.grouped_ffn(cfg, lay, xp, inp["x"], inp["w13"], inp["w2"], topk_w=w)
    y = moe.combine(cfg, lay, out)
    # the staged movement (explicit send / return buffers) gives the same bits
    _, xp2 = moe.permute_staged(cfg, lay, inp["x"])
    _, y2 = moe.combine_staged(cfg, lay, out)
    torch.cuda.synchronize()
    assert status.item() == 0
    A_kept = int(lay["expert_off"][-1])
    assert torch.equal(xp[:A_kept], xp2[:A_kept]) and torch.equal(y, y2)
    ids_np = ids.cpu().numpy().astype(np.int64)
    kept_ref = O.capacity_keep(ids_np, cfg.E, O.capacity(factor, cfg.N, cfg.k, cfg.E))
    assert np.array_equal(kept.cpu().numpy(), kept_ref)
    print(f"{cfg.name} factor {factor}: {(kept_ref < 0).sum()} of {kept_ref.size} assignments dropped")
    gates = O.gate_weights(O.gate_logits(cfg, inp["x"], inp["w_gate"], inp["bias"]), ids_np, cfg.score,
                           cfg.renormalize)
    y_ref = O.moe_tokens_direct(cfg, inp["x"], kept_ref, gates, inp["w13"], inp["w2"], np.arange(cfg.N))
    assert_close_fro(y, y_ref, what=f"{cfg.name} factor {factor}")


def test_full_size_hot_with_capacity():
    """The skewed workload at full size with capacity factor 1.25: the cut and the layout
    bit-exact, sampled tokens of y against the output equation."""
    cfg = CONFIGS["hot_cal"]
    inp = gpu_inputs(cfg)
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    kept = moe.capacity_drop(cfg, ids, moe.capacity_of(1.25, cfg))
    lay = moe.dispatch_layout(cfg, kept, inp["expert_owner"])
    xp = moe.permute(cfg, lay, inp["x"])
    h, out = moe.grouped_ffn(cfg, lay, xp, inp["x"], inp["w13"], inp["w2"], topk_w=w)
    y = moe.combine(cfg, lay, out)
    torch.cuda.synchronize()
    ids_np = ids.cpu().numpy().astype(np.int64)
    kept_ref = O.capacity_keep(ids_np, cfg.E, O.capacity(1.25, cfg.N, cfg.k, cfg.E))
    assert np.array_equal(kept.cpu().numpy(), kept_ref)
    ref = O.dispatch_layout(kept_ref, cfg.E, cfg.P, inp["expert_owner"].cpu().numpy(), cfg.S)
    assert_layout_equal(layout_to_numpy(lay), ref, cfg.P)
    print(f"hot_cal capacity 1.25: {(kept_ref < 0).sum()} of {kept_ref.size} assignments dropped, "
          f"max/mean n_e {O.imbalance(ref['n_e']):.2f}")
    tokens = np.sort(np.random.default_rng(0).choice(cfg.N, 8, replace=False))
    z = O.gate_logits(cfg, inp["x"][torch.tensor(tokens, device="cuda")], inp["w_gate"], inp["bias"])
    g = np.zeros((cfg.N, cfg.k))
    g[tokens] = O.gate_weights(z, ids_np[tokens], cfg.score, cfg.renormalize)
    y_ref = O.moe_tokens_direct(cfg, inp["x"], kept_ref, g, inp["w13"], inp["w2"], tokens)
    assert_close_fro(y[torch.tensor(tokens, device="cuda")], y_ref, what="hot_cal sampled y")


def test_capacity_then_replicas():
    """Dropped assignments stay dropped through the replica assignment; the layer over the
    slots with the dropped ones gives the layer without copies, bit for bit."""
    cfg = SMALL[0]
    R = 8
    inp = gpu_inputs(cfg)
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    kept = moe.capacity_drop(cfg, ids, moe.capacity_of(0.8, cfg))
    n_e = torch.bincount(kept.reshape(-1)[kept.reshape(-1) >= 0].long(), minlength=cfg.E).cpu().numpy()
    plan = moe.eplb_plan(n_e, R, cfg.P)
    phys = moe.eplb_assign(cfg, kept, torch.tensor(plan["replica_off"], device="cuda"),
                           torch.tensor(plan["replica_slots"], device="cuda"), cfg.E + R)
    torch.cuda.synchronize()
    assert torch.equal(phys < 0, kept < 0)
    pcfg = moe.physical_config(cfg, R)
    w13p = moe.eplb_place_weights(plan["slot_expert"], cfg.E, cfg.S, inp["w13"])
    w2p = moe.eplb_place_weights(plan["slot_expert"], cfg.E, cfg.S, inp["w2"])
    lay = moe.dispatch_layout(pcfg, phys)
    xp = moe.permute(pcfg, lay, inp["x"])
    _, out = moe.grouped_ffn(pcfg, lay, xp, inp["x"], w13p, w2p, topk_w=w)
    y = moe.combine(pcfg, lay, out)
    lay0 = moe.dispatch_layout(cfg, kept)
    xp0 = moe.permute(cfg, lay0, inp["x"])
    _, out0 = moe.grouped_ffn(cfg, lay0, xp0, inp["x"], inp["w13"], inp["w2"], topk_w=w)
    y0 = moe.combine(cfg, lay0, out0)
    torch.cuda.synchronize()
    assert torch.equal(y, y0)
