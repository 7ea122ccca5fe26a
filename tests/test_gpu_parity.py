"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Bit-exact for ids, counts, offsets and maps; within the stated float tolerance
(max abs <= 2e-2, relative Frobenius <= 5e-3 vs float64) for logits-derived gates,
expert outputs and y.
"""
import json
import os

import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import CONFIGS, small_config
from oracle import moe_oracle as O
from tests.gpu_cases import (assert_close_fro, assert_close_rel, assert_layout_equal, check_route, gpu_inputs,
                             layout_to_numpy, run_steps)

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden")

# small cases spanning several 128-row tiles, ragged tails, empty experts, shared experts,
# group-limited routing, custom placements and d / I not multiples of 128
SMALL = [
    small_config("s_bf16_plain", cfg_id=70, N=257, d=200, E=8, S=1, k=2, I=136, P=2),
    small_config("s_bf16_norenorm", cfg_id=71, N=300, d=256, E=16, S=2, k=3, I=264, P=4, renormalize=False),
    small_config("s_bf16_grouped", cfg_id=72, N=190, d=192, E=32, S=1, k=4, I=128, P=8, n_groups=8,
                 topk_groups=3, score="sigmoid"),
    small_config("s_bf16_tiny_n", cfg_id=73, N=7, d=64, E=8, S=0, k=2, I=64, P=2),
    small_config("s_bf16_pairs", cfg_id=79, N=700, d=4096, E=8, S=1, k=2, I=200, P=4),
    small_config("s_bf16_corrbias", cfg_id=81, N=333, d=256, E=32, S=1, k=4, I=128, P=8, n_groups=8,
                 topk_groups=3, score="sigmoid", bias="zipf", bias_alpha=0.7, bias_mode="selection"),
    small_config("s_bf16_one_tok", cfg_id=74, N=1, d=128, E=64, S=1, k=6, I=96, P=8),
    # 257 groups (256 routed + 1 shared) with a skewed router: one expert with a CTA-pair
    # tile and a tail, a few with one pair tile, most with 0..4 rows (d = 4096 selects the
    # CTA-pair kernel); exercises the group table and tile decode beyond 64 groups
    small_config("s_bf16_e256_skew", cfg_id=82, N=640, d=4096, E=256, S=1, k=4, I=128, P=32, bias="zipf",
                 bias_alpha=0.5),
    small_config("s_f32", cfg_id=75, N=129, d=96, E=8, S=1, k=2, I=72, P=4, dtype="f32"),
    small_config("s_f32_grouped", cfg_id=76, N=64, d=64, E=16, S=0, k=4, I=40, P=4, n_groups=4, topk_groups=2,
                 score="sigmoid", dtype="f32"),
    CONFIGS["tiny"],
]


def _ids(cfg):
    return [c.name for c in cfg]


@pytest.mark.parametrize("cfg", SMALL, ids=_ids(SMALL))
def test_small_end_to_end(cfg):
    inp = gpu_inputs(cfg)
    res = run_steps(cfg, inp)
    # logits: bf16 operands with fp32 accumulation, or an fp32 dot product (d <= 128 here)
    tol = 1e-3 if cfg.dtype == "bf16" else 1e-5
    ids, _ = check_route(cfg, inp, res, tol)
    lay = layout_to_numpy(res["layout"])
    ref = O.dispatch_layout(ids, cfg.E, cfg.P, None, cfg.S)
    assert_layout_equal(lay, ref, cfg.P)
    if cfg.name == "s_bf16_e256_skew":  # the case reaches what it is meant to
        n_e = ref["n_e"]
        print("n_e max", n_e.max(), "> 128:", int((n_e > 128).sum()), "1..4:", int(((n_e > 0) & (n_e <= 4)).sum()))
        assert (n_e > 128).sum() >= 1 and ((n_e > 0) & (n_e <= 4)).sum() >= 100
    # permute: bit copy
    xp_ref = O.permute(inp["x"], ref, cfg.k)
    assert np.array_equal(O.f64(res["x_perm"]), xp_ref)
    # full oracle on the GPU's routing (gates from the fp64 logits)
    g64 = O.gate_weights(O.gate_logits(cfg, inp["x"], inp["w_gate"], inp["bias"]), ids, cfg.score, cfg.renormalize)
    o_ref = O.experts_on_rows(xp_ref, ref, inp["w13"], inp["w2"], cfg.E)
    A = cfg.N * cfg.k
    # h (FC1 + SwiGLU) of every routed row against the float64 activations
    for e in range(cfg.E):
        n, r0 = ref["n_e"][e], ref["expert_off"][e]
        if n == 0:
            continue
        w13 = O.f64(inp["w13"][e])
        hh = O.silu(xp_ref[r0:r0 + n] @ w13[:cfg.I].T) * (xp_ref[r0:r0 + n] @ w13[cfg.I:].T)
        assert_close_rel(res["h"][r0:r0 + n], hh, what=f"h expert {e}")
    o_gpu = O.f64(res["out"][:A])
    # the GPU applied the gate in FC2: compare against gate-scaled oracle rows
    gate_of_row = g64.reshape(-1)[ref["row2tok"]]
    assert_close_fro(o_gpu, o_ref * gate_of_row[:, None], what="routed expert rows x gate")
    shared = [O.swiglu_expert(inp["x"], inp["w13"][cfg.E + s], inp["w2"][cfg.E + s]) for s in range(cfg.S)]
    for s in range(cfg.S):
        assert_close_fro(res["out"][A + s * cfg.N:A + (s + 1) * cfg.N], shared[s], what=f"shared {s}")
    y_ref = O.combine(o_ref, ref, g64, cfg.N, cfg.k, shared)
    assert_close_fro(res["y"], y_ref, what="y")


@pytest.mark.parametrize("cfg", SMALL[:3] + SMALL[5:6], ids=_ids(SMALL[:3] + SMALL[5:6]))
def test_fused_forward_matches_steps_bitwise(cfg):
    inp = gpu_inputs(cfg)
    res = run_steps(cfg, inp)
    lay = moe.Layout(cfg)
    y = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"],
                          layout=lay)
    torch.cuda.synchronize()
    assert torch.equal(y, res["y"])
    for k, v in lay.as_dict().items():
        assert torch.equal(v, res["layout"][k]), k
    y2 = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"])
    torch.cuda.synchronize()
    assert torch.equal(y2, y), "run-to-run determinism"


@pytest.mark.parametrize("cfg", SMALL[:3] + SMALL[5:6], ids=_ids(SMALL[:3] + SMALL[5:6]))
def test_staged_movement_matches_fused(cfg):
    inp = gpu_inputs(cfg)
    res = run_steps(cfg, inp)
    lay = res["layout"]
    send, xp = moe.permute_staged(cfg, lay, inp["x"])
    ret, y = moe.combine_staged(cfg, lay, res["out"])
    torch.cuda.synchronize()
    assert torch.equal(xp, res["x_perm"])
    assert torch.equal(y, res["y"])
    ref = layout_to_numpy(lay)
    A = cfg.N * cfg.k
    a = np.arange(A)
    # the send buffer holds x[a // k] at slot tok2send[a] (sources bucketed by owner)
    assert np.array_equal(O.f64(send)[ref["tok2send"]], O.f64(inp["x"])[a // cfg.k])
    assert np.array_equal(O.f64(ret), O.f64(res["out"][:A])[ref["send2row"]])


def test_worked_example_layout_on_gpu():
    g = json.load(open(os.path.join(GOLD, "worked_example_4tok.json")))
    cfg = small_config("worked", N=4, d=64, E=4, S=0, k=2, I=64, P=2)
    ids = torch.tensor(g["topk_ids"], dtype=torch.int32, device="cuda")
    lay = layout_to_numpy(moe.dispatch_layout(cfg, ids))
    for key in ["n_e", "expert_off", "recv_off", "tok2send", "send2row", "ret2tok", "tok2row", "row2tok"]:
        assert lay[key].tolist() == g[key], key
    assert lay["C"].tolist() == sum(g["C"], [])
    assert lay["send_off"].tolist() == sum(g["send_off"], [])


LAYOUT_CASES = [(1, 4, 1, 1), (7, 8, 2, 2), (33, 8, 2, 4), (129, 32, 8, 8), (1000, 64, 6, 8),
                (4096, 256, 8, 32), (3000, 128, 8, 16), (5, 8, 2, 8), (2049, 16, 1, 4)]


@pytest.mark.parametrize("shape", LAYOUT_CASES)
@pytest.mark.parametrize("custom_owner", [False, True])
def test_layout_random_bit_exact(shape, custom_owner):
    N, E, k, P = shape
    rng = np.random.default_rng(N * 7 + E)
    p = rng.dirichlet(np.full(E, 0.3))
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(N)])
    owner = rng.permutation(np.arange(E) % P).astype(np.int32) if custom_owner else None
    cfg = small_config("lay", N=N, d=64, E=E, S=1, k=k, I=64, P=P)
    lay = moe.dispatch_layout(cfg, torch.tensor(ids, dtype=torch.int32, device="cuda"),
                              None if owner is None else torch.tensor(owner, device="cuda"))
    ref = O.dispatch_layout(ids, E, P, owner, 1)
    assert_layout_equal(layout_to_numpy(lay), ref, P)


def test_round_trip_identity_on_gpu():
    """Identity experts: combine(permute(x)) with renormalised gates returns x (fp32)."""
    cfg = small_config("rt", cfg_id=77, N=333, d=128, E=16, S=0, k=4, I=64, P=4, dtype="f32")
    inp = gpu_inputs(cfg)
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"])
    lay = moe.dispatch_layout(cfg, ids)
    xp = moe.permute(cfg, lay, inp["x"])
    y = moe.combine(cfg, lay, xp, topk_w=w)
    torch.cuda.synchronize()
    gsum = w.double().sum(1, keepdim=True).cpu().numpy()
    np.testing.assert_allclose(O.f64(y), O.f64(inp["x"]) * gsum, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(O.f64(y), O.f64(inp["x"]), rtol=1e-5, atol=1e-5)


def test_bad_expert_id_sets_status():
    cfg = small_config("bad", N=64, d=64, E=8, S=0, k=2, I=64, P=2)
    ids = torch.zeros(64, 2, dtype=torch.int32, device="cuda")
    ids[:, 1] = 1
    ids[5, 0] = 8      # out of range
    ids[9, 1] = -3     # out of range
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lay = moe.dispatch_layout(cfg, ids, status=status)
    torch.cuda.synchronize()
    assert status.item() == 5  # MOE_ERR_BAD_INDEX
    # the maps stay permutations (no out-of-bounds write happened)
    t2r = lay["tok2row"].cpu().numpy()
    assert sorted(t2r.tolist()) == list(range(128))


def test_host_errors():
    cfg = small_config("err", N=64, d=64, E=8, S=0, k=2, I=64, P=2)
    ids = torch.zeros(64, 2, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        moe.dispatch_layout(cfg, ids, ws=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 3  # MOE_ERR_WORKSPACE
    with pytest.raises(moe.MoEError) as e:
        moe.check_config(cfg.replace(d=60))   # 120 bytes per row: not a multiple of 16
    assert e.value.status == 2
    with pytest.raises(moe.MoEError) as e:
        moe.dispatch_layout(cfg.replace(P=3), ids)  # E % P != 0 without a placement table
    assert e.value.status == 1


def test_empty_batch():
    cfg = small_config("empty", N=0, d=64, E=8, S=1, k=2, I=64, P=2)
    ids = torch.zeros(0, 2, dtype=torch.int32, device="cuda")
    lay = moe.dispatch_layout(cfg, ids)
    torch.cuda.synchronize()
    assert lay["n_e"].sum().item() == 0 and lay["C"].sum().item() == 0
    assert lay["expert_off"].tolist() == [0] * 9


def _ids_with_counts(counts, N, k, seed):
    """Distinct experts per token with exact per-expert counts (greedy by remaining count)."""
    rem = list(counts)
    rows = []
    for _ in range(N):
        order = sorted(range(len(rem)), key=lambda e: (-rem[e], e))[:k]
        for e in order:
            rem[e] -= 1
        rows.append(order)
    assert all(r == 0 for r in rem)
    ids = np.array(rows)
    rng = np.random.default_rng(seed)
    ids = ids[rng.permutation(N)]
    for t in range(N):  # random slot order inside each token
        ids[t] = ids[t][rng.permutation(k)]
    return ids


def test_ffn_pair_and_tail_row_splits():
    """Groups of 256 (one pair tile), 300 (pair + 44-row tail), 400 (two pair tiles,
    the second 144/256 full), 128 and 95 (tails only), 1, 0 rows, plus a shared expert of
    640 rows (512 in pairs + a 128-row tail).  d = 4096 selects the CTA-pair kernel."""
    counts = [256, 300, 400, 128, 1, 0, 95, 100]
    cfg = small_config("splits", cfg_id=78, N=640, d=4096, E=8, S=1, k=2, I=192, P=4)
    inp = gpu_inputs(cfg)
    ids = _ids_with_counts(counts, cfg.N, cfg.k, 3)
    ids_t = torch.tensor(ids, dtype=torch.int32, device="cuda")
    gates = torch.rand(cfg.N, cfg.k, generator=torch.Generator().manual_seed(5)).float().cuda()
    lay = moe.dispatch_layout(cfg, ids_t)
    xp = moe.permute(cfg, lay, inp["x"])
    h, out = moe.grouped_ffn(cfg, lay, xp, inp["x"], inp["w13"], inp["w2"], topk_w=gates)
    torch.cuda.synchronize()
    ref = O.dispatch_layout(ids, cfg.E, cfg.P, None, cfg.S)
    assert layout_to_numpy(lay)["n_e"].tolist() == counts
    o_ref = O.experts_on_rows(O.permute(inp["x"], ref, cfg.k), ref, inp["w13"], inp["w2"], cfg.E)
    g_row = O.f64(gates).reshape(-1)[ref["row2tok"]]
    A = cfg.N * cfg.k
    assert_close_fro(out[:A], o_ref * g_row[:, None], what="routed rows")
    shared = O.swiglu_expert(inp["x"], inp["w13"][cfg.E], inp["w2"][cfg.E])
    assert_close_fro(out[A:], shared, what="shared rows")
    # h (FC1 output) against the float64 SwiGLU activations, for every routed row
    xp64 = O.permute(inp["x"], ref, cfg.k)
    for e in range(cfg.E):
        n, r0 = ref["n_e"][e], ref["expert_off"][e]
        if n == 0:
            continue
        w13 = O.f64(inp["w13"][e])
        hh = O.silu(xp64[r0:r0 + n] @ w13[:cfg.I].T) * (xp64[r0:r0 + n] @ w13[cfg.I:].T)
        assert_close_rel(h[r0:r0 + n], hh, what=f"h expert {e}")


@pytest.mark.parametrize("cfg", [SMALL[1], SMALL[4], SMALL[5]], ids=_ids([SMALL[1], SMALL[4], SMALL[5]]))
def test_overlapped_forward_and_split_ffn_match_bitwise(cfg):
    """Shared experts on a side stream give the same bits as the one-stream forward, and
    moe_routed_ffn + moe_shared_ffn write exactly what moe_grouped_ffn writes."""
    inp = gpu_inputs(cfg)
    res = run_steps(cfg, inp)
    side = torch.cuda.Stream()
    lay = moe.Layout(cfg)
    y = moe.layer_forward_overlapped(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"],
                                     inp["w2"], side, layout=lay)
    torch.cuda.synchronize()
    assert torch.equal(y, res["y"])
    assert torch.equal(lay["tok2row"], res["layout"]["tok2row"])
    h, out = moe.routed_ffn(cfg, res["layout"], res["x_perm"], inp["w13"], inp["w2"], topk_w=res["w"])
    moe.shared_ffn(cfg, inp["x"], inp["w13"], inp["w2"], h, out)
    torch.cuda.synchronize()
    assert torch.equal(h, res["h"]) and torch.equal(out, res["out"])


def test_bounded_wait_gives_up_and_context_stays_usable():
    """A wait on a barrier that nothing arrives on ends after its limit with
    MOE_ERR_TIMEOUT in the status word; the GPU keeps working afterwards."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.selftest_bounded_wait(status, limit_ns=50_000_000)  # 50 ms
    torch.cuda.synchronize()
    assert status.item() == 6  # MOE_ERR_TIMEOUT
    cfg = small_config("after", N=64, d=64, E=8, S=0, k=2, I=64, P=2)
    ids = torch.zeros(64, 2, dtype=torch.int32, device="cuda")
    ids[:, 1] = 1
    lay = moe.dispatch_layout(cfg, ids)
    torch.cuda.synchronize()
    assert lay["n_e"].tolist()[:2] == [64, 64]


def test_bad_owner_table_sets_status():
    cfg = small_config("badown", N=32, d=64, E=8, S=0, k=2, I=64, P=2)
    ids = torch.stack([torch.arange(32) % 8, (torch.arange(32) + 1) % 8], 1).to(torch.int32).cuda()
    owner = torch.tensor([0, 1, 0, 1, 0, 1, 5, 1], dtype=torch.int32, device="cuda")  # 5 >= P
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lay = moe.dispatch_layout(cfg, ids, owner, status=status)
    torch.cuda.synchronize()
    assert status.item() == 5
    assert sorted(lay["tok2row"].cpu().tolist()) == list(range(64))


@pytest.mark.parametrize("cfg", [SMALL[1], SMALL[5]], ids=_ids([SMALL[1], SMALL[5]]))
def test_forward_captures_into_cuda_graph(cfg):
    """moe_layer_forward launches only device work on its stream (no host sync, no
    allocation), so it captures into a CUDA graph; replays give the eager result."""
    inp = gpu_inputs(cfg)
    ws = moe.alloc_workspace(cfg)
    y_eager = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"],
                                inp["w2"], ws=ws)
    torch.cuda.synchronize()
    y = torch.empty_like(y_eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"],
                          y=y, ws=ws)  # warm-up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"],
                              inp["w2"], y=y, ws=ws)
    for _ in range(2):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_eager)


@pytest.mark.parametrize("cfg", [SMALL[1], SMALL[4]], ids=_ids([SMALL[1], SMALL[4]]))
def test_overlapped_forward_captures_into_cuda_graph(cfg):
    """moe_layer_forward_overlapped forks the shared experts onto the side stream with
    events, so a capture on the calling stream pulls the side stream in; replays give the
    one-stream forward's bits (the bench times this replay as the graph step)."""
    inp = gpu_inputs(cfg)
    ws = moe.alloc_workspace(cfg)
    args = (cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"])
    y_ref = moe.layer_forward(*args, ws=ws)
    torch.cuda.synchronize()
    y = torch.empty_like(y_ref)
    s, side = torch.cuda.Stream(), torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        moe.layer_forward_overlapped(*args, side, y=y, ws=ws)  # warm-up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            moe.layer_forward_overlapped(*args, side, y=y, ws=ws)
    for _ in range(2):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref)
    del g
