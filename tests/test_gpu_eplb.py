"""GPU parity of the redundant expert slots (EPLB) path through the C ABI.

The replica assignment and the layout over E + R physical slots are compared with the
oracle bit for bit; the layer computed over the slots (with copied weights) must give
the output of the layer without copies, and match the float64 oracle.

Source: "Wide EP：当 MoE Expert Parallel 横跨几十张 GPU", sections "为什么要把 EP 做宽",
"Expert 副本在 Wide EP 中还有整除作用", "三种负载必须同时平衡".
"""
import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import CONFIGS, small_config
from oracle import eplb as EP
from oracle import moe_oracle as O
from tests.gpu_cases import assert_close_fro, assert_layout_equal, gpu_inputs, layout_to_numpy

pytestmark = pytest.mark.gpu


def _tables(plan):
    return (torch.tensor(plan["replica_off"], dtype=torch.int32, device="cuda"),
            torch.tensor(plan["replica_slots"], dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("E,R,P,N,k", [(8, 0, 4, 300, 2), (8, 4, 4, 300, 2), (16, 8, 8, 1000, 4),
                                       (64, 8, 8, 4096, 6), (256, 32, 32, 2048, 8), (8, 4, 4, 0, 2)])
def test_assign_matches_oracle(E, R, P, N, k):
    rng = np.random.default_rng(E + R + N)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(N)]) if N else np.zeros((0, k), np.int64)
    load = np.bincount(ids.reshape(-1), minlength=E) * (1 + rng.integers(0, 3, size=E))  # a stale plan
    plan = moe.eplb_plan(load, R, P)
    cfg = small_config("eplb", N=N, d=64, E=E, S=0, k=k, I=64, P=P)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ro, rs = _tables(plan)
    phys = moe.eplb_assign(cfg, torch.tensor(ids, dtype=torch.int32, device="cuda"), ro, rs, E + R, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = EP.assign(ids, plan["replica_off"], plan["replica_slots"])
    assert np.array_equal(phys.cpu().numpy(), ref)


def test_assign_reports_bad_ids():
    E, R, P = 8, 4, 4
    plan = moe.eplb_plan(np.arange(E) + 1, R, P)
    cfg = small_config("eplb_bad", N=16, d=64, E=E, S=0, k=2, I=64, P=P)
    ids = torch.zeros(16, 2, dtype=torch.int32, device="cuda")
    ids[:, 1] = 1
    ids[3, 0] = 9  # no such expert
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ro, rs = _tables(plan)
    phys = moe.eplb_assign(cfg, ids, ro, rs, E + R, status=status)
    torch.cuda.synchronize()
    assert status.item() == moe.binding.MOE_ERR_BAD_INDEX
    assert int(phys.min()) >= 0 and int(phys.max()) < E + R


def _layer_with_replicas(cfg, inp, R):
    """route -> plan (from this batch's counts) -> assign -> layout / permute / FFN over the
    E + R slots with copied weights -> combine."""
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    n_e = torch.bincount(ids.reshape(-1).long(), minlength=cfg.E).cpu().numpy()
    plan = moe.eplb_plan(n_e, R, cfg.P)
    ro, rs = _tables(plan)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    phys = moe.eplb_assign(cfg, ids, ro, rs, cfg.E + R, status=status)
    pcfg = moe.physical_config(cfg, R)
    w13p = moe.eplb_place_weights(plan["slot_expert"], cfg.E, cfg.S, inp["w13"])
    w2p = moe.eplb_place_weights(plan["slot_expert"], cfg.E, cfg.S, inp["w2"])
    lay = moe.dispatch_layout(pcfg, phys, None, status=status)
    xp = moe.permute(pcfg, lay, inp["x"])
    h, out = moe.grouped_ffn(pcfg, lay, xp, inp["x"], w13p, w2p, topk_w=w)
    y = moe.combine(pcfg, lay, out)
    torch.cuda.synchronize()
    assert status.item() == 0
    return dict(ids=ids, w=w, plan=plan, phys=phys, layout=lay, y=y)


SMALL = [
    small_config("e_bf16", cfg_id=82, N=700, d=256, E=16, S=1, k=4, I=128, P=8),
    small_config("e_bf16_pairs", cfg_id=83, N=640, d=4096, E=8, S=1, k=2, I=192, P=4),
    small_config("e_f32", cfg_id=84, N=129, d=96, E=8, S=0, k=2, I=72, P=4, dtype="f32"),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
@pytest.mark.parametrize("R", [0, 4, 8])
def test_layer_with_replicas_equals_layer_without(cfg, R):
    if (cfg.E + R) % cfg.P:
        pytest.skip("slots must divide over the owners")
    inp = gpu_inputs(cfg)
    res = _layer_with_replicas(cfg, inp, R)
    ids = res["ids"].cpu().numpy().astype(np.int64)
    # the assignment and the layout over the slots, bit for bit
    phys_ref = EP.assign(ids, res["plan"]["replica_off"], res["plan"]["replica_slots"])
    assert np.array_equal(res["phys"].cpu().numpy(), phys_ref)
    ref_lay = O.dispatch_layout(phys_ref, cfg.E + R, cfg.P, None, cfg.S)
    assert_layout_equal(layout_to_numpy(res["layout"]), ref_lay, cfg.P)
    # the output: equal to the layer without copies, and to the float64 layer
    y_plain = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], None, inp["w13"], inp["w2"])
    torch.cuda.synchronize()
    assert torch.equal(res["y"], y_plain)
    gates = O.gate_weights(O.gate_logits(cfg, inp["x"], inp["w_gate"], inp["bias"]), ids, cfg.score,
                           cfg.renormalize)
    y_ref = O.moe_tokens_direct(cfg, inp["x"], ids, gates, inp["w13"], inp["w2"], np.arange(cfg.N))
    assert_close_fro(res["y"], y_ref, what=f"{cfg.name} R={R}")


@pytest.mark.parametrize("name,R", [("hot_cal", 16), ("hot", 16)])
def test_full_size_skewed_routing_with_replicas(name, R):
    """Skewed workloads at full size: copies of the hot experts take the owner imbalance
    down; the output is unchanged."""
    cfg = CONFIGS[name]
    inp = gpu_inputs(cfg)
    res = _layer_with_replicas(cfg, inp, R)
    ref_lay = O.dispatch_layout(res["phys"].cpu().numpy(), cfg.E + R, cfg.P, None, cfg.S)
    assert_layout_equal(layout_to_numpy(res["layout"]), ref_lay, cfg.P)
    n_e = torch.bincount(res["ids"].reshape(-1).long(), minlength=cfg.E).cpu().numpy()
    plain = O.dispatch_layout(res["ids"].cpu().numpy(), cfg.E, cfg.P, inp["expert_owner"].cpu().numpy(), cfg.S)
    before = O.imbalance(np.diff(plain["recv_off"]))
    after = O.imbalance(np.diff(ref_lay["recv_off"]))
    print(f"{name}: owner max/mean {before:.2f} -> {after:.2f} with {R} copies; "
          f"expert max/mean {O.imbalance(n_e):.2f} -> {O.imbalance(ref_lay['n_e']):.2f}")
    assert after < before
    y_plain = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"],
                                inp["w2"])
    torch.cuda.synchronize()
    assert torch.equal(res["y"], y_plain)


@pytest.mark.parametrize("R", [8, 16])
def test_mx_layer_with_replicas_equals_mx_layer_without(R):
    """Redundant slots on the MXFP8 path: the slots carry copies of the MX codes and scale
    rows (eplb_place_weights moves any per-expert bytes), and the MX layer over the E + R
    slots gives the MX layer without copies, bit for bit."""
    cfg = small_config("e_mx", cfg_id=139, N=700, d=512, E=16, S=1, k=4, I=128, P=8)
    inp = gpu_inputs(cfg)
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    n_e = torch.bincount(ids.reshape(-1).long(), minlength=cfg.E).cpu().numpy()
    plan = moe.eplb_plan(n_e, R, cfg.P)
    ro, rs = _tables(plan)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    phys = moe.eplb_assign(cfg, ids, ro, rs, cfg.E + R, status=status)
    pcfg = moe.physical_config(cfg, R)
    w13_q, w13_sf = moe.quantize_mx(inp["w13"])
    w2_q, w2_sf = moe.quantize_mx(inp["w2"])
    place = [moe.eplb_place_weights(plan["slot_expert"], cfg.E, cfg.S, t) for t in (w13_q, w13_sf, w2_q, w2_sf)]
    lay = moe.dispatch_layout(pcfg, phys, None, status=status)
    x_q, x_sf = moe.quantize_mx(inp["x"])
    xp, xp_sf = moe.permute_mx(pcfg, lay, x_q, x_sf)
    _, _, _, out = moe.grouped_ffn_mx(pcfg, lay, xp, xp_sf, x_q, x_sf, *place, topk_w=w)
    y = moe.combine(pcfg, lay, out)
    y_plain = moe.layer_forward_mx(cfg, inp["x"], inp["w_gate"], inp["bias"], None, w13_q, w13_sf, w2_q, w2_sf)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(y, y_plain)


def test_fp8_layer_with_replicas_equals_fp8_layer_without():
    """The same on the row-scaled FP8 path: slot copies of the e4m3 codes and row scales."""
    R = 8
    cfg = small_config("e_f8", cfg_id=140, N=700, d=256, E=16, S=1, k=4, I=128, P=8)
    inp = gpu_inputs(cfg)
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    n_e = torch.bincount(ids.reshape(-1).long(), minlength=cfg.E).cpu().numpy()
    plan = moe.eplb_plan(n_e, R, cfg.P)
    ro, rs = _tables(plan)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    phys = moe.eplb_assign(cfg, ids, ro, rs, cfg.E + R, status=status)
    pcfg = moe.physical_config(cfg, R)
    w13_q, w13_s = moe.quantize_fp8(inp["w13"])
    w2_q, w2_s = moe.quantize_fp8(inp["w2"])
    place = [moe.eplb_place_weights(plan["slot_expert"], cfg.E, cfg.S, t) for t in (w13_q, w13_s, w2_q, w2_s)]
    lay = moe.dispatch_layout(pcfg, phys, None, status=status)
    x_q, x_s = moe.quantize_fp8(inp["x"])
    xp = moe.permute_fp8(pcfg, lay, x_q)
    _, _, _, out = moe.grouped_ffn_fp8(pcfg, lay, xp, x_q, x_s, *place, topk_w=w)
    y = moe.combine(pcfg, lay, out)
    y_plain = moe.layer_forward_fp8(cfg, inp["x"], inp["w_gate"], inp["bias"], None, w13_q, w13_s, w2_q, w2_s)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(y, y_plain)
