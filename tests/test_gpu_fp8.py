"""GPU parity of the FP8 (e4m3) expert path through the C ABI, staged so that every
quantised code is compared bit for bit and every float result against the float64
oracle built on the same codes.

  (i)   x, W13, W2 quantisation: codes and scales bit-exact (both sides divide in fp32);
  (ii)  FP8 dispatch payload: x_q_perm rows are the token rows, bit for bit;
  (iii) FC1 + SwiGLU: h (bf16) vs the oracle on the codes, float tolerance;
  (iv)  h quantisation: codes and scales of the GPU's own h, bit-exact;
  (v)   FC2 x gate: out vs the oracle on the GPU's h codes, float tolerance;
  (vi)  combine: y vs the oracle's sum of (v) plus the shared experts;
and the fused moe_layer_forward_fp8 gives the staged result bit for bit.
"""
import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import CONFIGS, small_config
from oracle import fp8 as F
from oracle import moe_oracle as O
from tests.gpu_cases import assert_close_fro, assert_close_rel, gpu_inputs

pytestmark = pytest.mark.gpu


def _np(t):
    return t.cpu().numpy()


def test_quantisation_is_bit_exact():
    g = torch.Generator().manual_seed(0)
    x = (torch.randn(300, 2048, generator=g) * torch.logspace(-3, 3, 300)[:, None]).to(torch.bfloat16)
    x[5] = 0
    x[6, ::7] = 0
    xd = x.cuda()
    q, s = moe.quantize_fp8(xd)
    torch.cuda.synchronize()
    q_ref, s_ref = F.quantize_rows(x.float().numpy())
    assert np.array_equal(_np(s), s_ref)
    assert np.array_equal(_np(q), q_ref)


def _staged(cfg, inp):
    E, S = cfg.E, cfg.S
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    lay = moe.dispatch_layout(cfg, ids, inp["expert_owner"])
    x_q, x_s = moe.quantize_fp8(inp["x"])
    w13_q, w13_s = moe.quantize_fp8(inp["w13"])
    w2_q, w2_s = moe.quantize_fp8(inp["w2"])
    xp = moe.permute_fp8(cfg, lay, x_q)
    h, h_q, h_s, out = moe.grouped_ffn_fp8(cfg, lay, xp, x_q, x_s, w13_q, w13_s, w2_q, w2_s, topk_w=w)
    y = moe.combine(cfg, lay, out)
    torch.cuda.synchronize()
    return dict(ids=ids, w=w, lay=lay, x_q=x_q, x_s=x_s, w13_q=w13_q, w13_s=w13_s, w2_q=w2_q, w2_s=w2_s, xp=xp,
                h=h, h_q=h_q, h_s=h_s, out=out, y=y)


SMALL = [
    small_config("f8_small", cfg_id=85, N=700, d=256, E=16, S=1, k=4, I=128, P=8),
    small_config("f8_ragged", cfg_id=86, N=333, d=512, E=8, S=2, k=2, I=208, P=4, score="sigmoid"),
    small_config("f8_wide_d", cfg_id=87, N=300, d=4096, E=8, S=1, k=2, I=192, P=4),
    # d = 4096 with groups over 128 rows: 256-row CTA-pair tiles plus one-CTA tails
    small_config("f8_pairs", cfg_id=99, N=640, d=4096, E=8, S=1, k=2, I=192, P=4),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
def test_fp8_layer_staged(cfg):
    inp = gpu_inputs(cfg)
    r = _staged(cfg, inp)
    E, S, N, k, I = cfg.E, cfg.S, cfg.N, cfg.k, cfg.I
    A = N * k
    # (i) quantisation of x and of every weight row
    xq_ref, xs_ref = F.quantize_rows(inp["x"].float().cpu().numpy())
    assert np.array_equal(_np(r["x_q"]), xq_ref) and np.array_equal(_np(r["x_s"]), xs_ref)
    w13 = inp["w13"].float().cpu().numpy()
    w2 = inp["w2"].float().cpu().numpy()
    w13q_ref, w13s_ref = F.quantize_rows(w13.reshape(-1, cfg.d))
    w2q_ref, w2s_ref = F.quantize_rows(w2.reshape(-1, I))
    assert np.array_equal(_np(r["w13_q"]).reshape(-1, cfg.d), w13q_ref)
    assert np.array_equal(_np(r["w13_s"]).reshape(-1), w13s_ref)
    assert np.array_equal(_np(r["w2_q"]).reshape(-1, I), w2q_ref)
    assert np.array_equal(_np(r["w2_s"]).reshape(-1), w2s_ref)
    # (ii) the FP8 dispatch payload
    row2tok = _np(r["lay"]["row2tok"])
    assert np.array_equal(_np(r["xp"]), xq_ref[row2tok // k])
    # (iii) FC1 on the codes, per expert (routed rows in layout order, then shared rows)
    n_e, off = _np(r["lay"]["n_e"]), _np(r["lay"]["expert_off"])
    w13q = w13q_ref.reshape(E + S, 2 * I, cfg.d)
    w13s = w13s_ref.reshape(E + S, 2 * I)
    h_ref = np.zeros((A + S * N, I))
    for e in range(E):
        if n_e[e]:
            rows = slice(off[e], off[e] + n_e[e])
            tok = row2tok[rows] // k
            h_ref[rows] = F.fc1(xq_ref[tok], xs_ref[tok], w13q[e], w13s[e], I)
    for s in range(S):
        h_ref[A + s * N:A + (s + 1) * N] = F.fc1(xq_ref, xs_ref, w13q[E + s], w13s[E + s], I)
    assert_close_rel(r["h"], h_ref, what=f"{cfg.name} h")
    # (iv) the GPU's h quantised on both sides
    hq_ref, hs_ref = F.quantize_rows(r["h"].float().cpu().numpy())
    assert np.array_equal(_np(r["h_q"]), hq_ref) and np.array_equal(_np(r["h_s"]), hs_ref)
    # (v) FC2 x gate on the GPU's h codes
    w2q = w2q_ref.reshape(E + S, cfg.d, I)
    w2s = w2s_ref.reshape(E + S, cfg.d)
    gate_row = O.f64(r["w"]).reshape(-1)[row2tok]
    o_ref = np.zeros((A + S * N, cfg.d))
    for e in range(E):
        if n_e[e]:
            rows = slice(off[e], off[e] + n_e[e])
            o_ref[rows] = F.fc2(hq_ref[rows], hs_ref[rows], w2q[e], w2s[e]) * gate_row[rows, None]
    for s in range(S):
        rows = slice(A + s * N, A + (s + 1) * N)
        o_ref[rows] = F.fc2(hq_ref[rows], hs_ref[rows], w2q[E + s], w2s[E + s])
    assert_close_fro(r["out"], o_ref, what=f"{cfg.name} out")
    # (vi) combine
    tok2row = _np(r["lay"]["tok2row"])
    y_ref = sum(o_ref[tok2row[np.arange(N) * k + j]] for j in range(k))
    for s in range(S):
        y_ref = y_ref + o_ref[A + s * N:A + (s + 1) * N]
    assert_close_fro(r["y"], y_ref, what=f"{cfg.name} y")
    # FP8 against the unquantised float64 layer (reported: e4m3 keeps 3 mantissa bits)
    gates = O.gate_weights(O.gate_logits(cfg, inp["x"], inp["w_gate"], inp["bias"]), _np(r["ids"]).astype(np.int64),
                           cfg.score, cfg.renormalize)
    y64 = O.moe_tokens_direct(cfg, inp["x"], _np(r["ids"]).astype(np.int64), gates, inp["w13"], inp["w2"],
                              np.arange(N))
    rel = np.linalg.norm(O.f64(r["y"]) - y64) / np.linalg.norm(y64)
    print(f"{cfg.name}: FP8 layer vs unquantised float64 layer, relative Frobenius error {rel:.4f}")
    assert rel < 0.1
    # the fused entry point runs the same kernels; with the shared experts on a side
    # stream it gives the same bits
    y = moe.layer_forward_fp8(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], r["w13_q"],
                              r["w13_s"], r["w2_q"], r["w2_s"])
    y_ov = moe.layer_forward_fp8(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], r["w13_q"],
                                 r["w13_s"], r["w2_q"], r["w2_s"], side_stream=torch.cuda.Stream())
    torch.cuda.synchronize()
    assert torch.equal(y, r["y"]) and torch.equal(y_ov, r["y"])


@pytest.mark.parametrize("name", ["fine", "hot_cal"])
def test_fp8_full_size_sampled(name):
    """Full-size workloads (fine: one-CTA tiles; hot_cal: CTA-pair tiles): x quantisation
    bit-exact, the weight codes of the sampled experts bit-exact, sampled rows of h and out
    against the oracle on the same codes, fused == staged."""
    cfg = CONFIGS[name]
    inp = gpu_inputs(cfg)
    r = _staged(cfg, inp)
    k, I, E = cfg.k, cfg.I, cfg.E
    xq_ref, xs_ref = F.quantize_rows(inp["x"].float().cpu().numpy())
    assert np.array_equal(_np(r["x_q"]), xq_ref)
    row2tok = _np(r["lay"]["row2tok"])
    n_e, off = _np(r["lay"]["n_e"]), _np(r["lay"]["expert_off"])
    rng = np.random.default_rng(0)
    w13q = _np(r["w13_q"]).reshape(E + cfg.S, 2 * I, cfg.d)
    w13s = _np(r["w13_s"]).reshape(E + cfg.S, 2 * I)
    w2q = _np(r["w2_q"]).reshape(E + cfg.S, cfg.d, I)
    w2s = _np(r["w2_s"]).reshape(E + cfg.S, cfg.d)
    hq = _np(r["h_q"])
    hs = _np(r["h_s"])
    for e in rng.choice(np.flatnonzero(n_e > 0), 6, replace=False):
        wq_ref, ws_ref = F.quantize_rows(inp["w13"][e].float().cpu().numpy())
        assert np.array_equal(w13q[e], wq_ref) and np.array_equal(w13s[e], ws_ref)
        rows = off[e] + rng.choice(n_e[e], min(8, n_e[e]), replace=False)
        tok = row2tok[rows] // k
        assert_close_rel(r["h"][torch.tensor(rows)], F.fc1(xq_ref[tok], xs_ref[tok], w13q[e], w13s[e], I),
                         what=f"h expert {e}")
        g = O.f64(r["w"]).reshape(-1)[row2tok[rows]]
        assert_close_fro(r["out"][torch.tensor(rows)], F.fc2(hq[rows], hs[rows], w2q[e], w2s[e]) * g[:, None],
                         what=f"out expert {e}")
    y = moe.layer_forward_fp8(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], r["w13_q"],
                              r["w13_s"], r["w2_q"], r["w2_s"])
    torch.cuda.synchronize()
    assert torch.equal(y, r["y"])


def test_fp8_forward_is_deterministic_and_graph_capturable():
    """Two runs give the same bits; the fused FP8 forward captured in a CUDA graph and
    replayed gives them too (the workspace and the weights are set up before capture)."""
    cfg = SMALL[3]
    inp = gpu_inputs(cfg)
    w13_q, w13_s = moe.quantize_fp8(inp["w13"])
    w2_q, w2_s = moe.quantize_fp8(inp["w2"])
    ws = torch.empty(moe.workspace_bytes_fp8(cfg), dtype=torch.uint8, device="cuda")
    args = (cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], w13_q, w13_s, w2_q, w2_s)
    y1 = moe.layer_forward_fp8(*args, ws=ws)
    y2 = moe.layer_forward_fp8(*args, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    y3 = torch.empty_like(y1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.layer_forward_fp8(*args, y=y3, ws=ws)  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    y3.zero_()
    with torch.cuda.graph(graph):
        moe.layer_forward_fp8(*args, y=y3, ws=ws)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(y3, y1)
