"""Shared helpers for the GPU parity tests: run the CUDA path step by step through the
C ABI and the oracle on the same seeded inputs, and compare."""
import numpy as np
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import make_inputs
from oracle import moe_oracle as O

# floating-point tolerance vs the float64 oracle (bf16 storage, fp32 accumulation)
MAX_ABS = 2e-2
REL_FRO = 5e-3


def assert_close_fro(got, ref, max_abs=MAX_ABS, rel_fro=REL_FRO, what=""):
    got = O.f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    err = np.abs(got - ref)
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= max_abs, f"{what}: max abs err {err.max():.3e} > {max_abs}"
    assert fro <= rel_fro, f"{what}: rel Frobenius err {fro:.3e} > {rel_fro}"
    return float(err.max()), float(fro)


def assert_close_rel(got, ref, rel=1e-2, rel_fro=REL_FRO, what=""):
    """For bf16 intermediates of any magnitude: |err| <= rel * max(|ref|, 1) elementwise
    (bf16 keeps 8 significant bits: rounding alone is up to 2^-9 of the value) and the
    relative Frobenius error bound."""
    got = O.f64(got)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    worst = (np.abs(got - ref) / np.maximum(np.abs(ref), 1.0)).max()
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert worst <= rel, f"{what}: scaled err {worst:.3e} > {rel}"
    assert fro <= rel_fro, f"{what}: rel Frobenius err {fro:.3e} > {rel_fro}"


def layout_to_numpy(layout):
    return {k: v.cpu().numpy().astype(np.int64) for k, v in layout.as_dict().items()}


def assert_layout_equal(gpu, ref, P):
    for key in ["n_e", "expert_off", "recv_off", "tok2send", "send2row", "ret2tok", "tok2row", "row2tok",
                "tile_off"]:
        assert np.array_equal(gpu[key], ref[key].reshape(-1)), key
    assert np.array_equal(gpu["C"].reshape(P, P), ref["C"]), "C"
    assert np.array_equal(gpu["send_off"].reshape(P, P), ref["send_off"]), "send_off"


def gpu_inputs(cfg, seed_offset=0):
    return make_inputs(cfg, device="cuda", seed_offset=seed_offset)


def run_steps(cfg, inp, status=None):
    """The layer step by step through the C ABI; returns every intermediate."""
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    layout = moe.dispatch_layout(cfg, ids, inp["expert_owner"], status=status)
    x_perm = moe.permute(cfg, layout, inp["x"])
    h, out = moe.grouped_ffn(cfg, layout, x_perm, inp["x"], inp["w13"], inp["w2"], topk_w=w)
    y = moe.combine(cfg, layout, out)
    torch.cuda.synchronize()
    return dict(logits=logits, ids=ids, w=w, layout=layout, x_perm=x_perm, h=h, out=out, y=y)


def check_route(cfg, inp, res, logit_tol):
    """Stages (i)-(iii) of the near-tie protocol."""
    z64 = O.router_logits(inp["x"], inp["w_gate"], inp["bias"])
    zgate = O.gate_logits(cfg, inp["x"], inp["w_gate"], inp["bias"])
    zg = res["logits"].cpu().numpy()
    assert np.abs(zg.astype(np.float64) - z64).max() <= logit_tol, "router logits"
    ids_ref = O.select_experts(zg, cfg.k, cfg.n_groups, cfg.topk_groups)   # on the GPU's fp32 logits
    ids = res["ids"].cpu().numpy().astype(np.int64)
    assert np.array_equal(ids, ids_ref), "top-k ids (selection on the same fp32 logits)"
    g_ref = O.gate_weights(zgate, ids, cfg.score, cfg.renormalize)
    np.testing.assert_allclose(res["w"].cpu().numpy(), g_ref, rtol=0, atol=1e-5)
    # report how many tokens the oracle's own fp64 selection would route differently
    ids64 = O.select_experts(z64, cfg.k, cfg.n_groups, cfg.topk_groups)
    return ids, int((np.sort(ids64, 1) != np.sort(ids, 1)).any(1).sum())
