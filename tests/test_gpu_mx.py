"""GPU parity of the block-scaled (MX) e4m3 expert path through the C ABI.

Staged, so that every code and every scale byte is compared bit for bit and every float
result against the float64 oracle:
  (i)   x, W13, W2 MX quantisation: codes and E8M0 scale bytes bit-exact;
  (ii)  MX dispatch payload: code rows and scale rows are the token rows, bit for bit;
  (iii) FC1 + SwiGLU: h (bf16) vs the oracle's block-scaled product on the oracle's codes;
  (iv)  h quantisation: codes and scale bytes of the GPU's h, bit-exact (the quantiser on
        the values the path stores);
  (v)   FC2 x gate: out vs the oracle on those h codes;
and end to end: y vs the oracle's whole MX layer computed from the seeded inputs alone (h
rounded to bf16 where the path stores it, then quantised by the oracle), plus the fused
moe_layer_forward_mx giving the staged result bit for bit.
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


def test_mx_quantisation_is_bit_exact():
    g = torch.Generator().manual_seed(0)
    x = (torch.randn(300, 2048, generator=g) * torch.logspace(-30, 30, 300)[:, None]).to(torch.bfloat16)
    x[5] = 0
    x[6, 64:96] = 0                             # one all-zero block inside a row
    x[7, ::3] = 0
    x[8, :32] = torch.tensor([448.0, -500.0, 2.0 ** -133] * 10 + [1.0, -1.0]).to(torch.bfloat16)
    x[9] = torch.randn(2048, generator=g).to(torch.bfloat16) * 2.0 ** -126  # subnormal fp32 values
    q, sf = moe.quantize_mx(x.cuda())
    torch.cuda.synchronize()
    q_ref, sf_ref = F.quantize_mx(x.float().numpy())
    assert np.array_equal(_np(sf), sf_ref)
    assert np.array_equal(_np(q), q_ref)


def _staged(cfg, inp):
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    lay = moe.dispatch_layout(cfg, ids, inp["expert_owner"])
    x_q, x_sf = moe.quantize_mx(inp["x"])
    w13_q, w13_sf = moe.quantize_mx(inp["w13"])
    w2_q, w2_sf = moe.quantize_mx(inp["w2"])
    xp, xp_sf = moe.permute_mx(cfg, lay, x_q, x_sf)
    h, h_q, h_sf, out = moe.grouped_ffn_mx(cfg, lay, xp, xp_sf, x_q, x_sf, w13_q, w13_sf, w2_q, w2_sf, topk_w=w)
    y = moe.combine(cfg, lay, out)
    torch.cuda.synchronize()
    return dict(ids=ids, w=w, lay=lay, x_q=x_q, x_sf=x_sf, w13_q=w13_q, w13_sf=w13_sf, w2_q=w2_q, w2_sf=w2_sf,
                xp=xp, xp_sf=xp_sf, h=h, h_q=h_q, h_sf=h_sf, out=out, y=y)


def _to_bf16(a):
    """float64 -> bf16 (round to nearest even) -> float64: what the path stores h as."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


SMALL = [
    small_config("mx_small", cfg_id=130, N=700, d=512, E=16, S=1, k=4, I=256, P=8),
    # FC1 output tiles of 96 columns and FC2 tiles of 192 with ragged last tiles, two shared experts
    small_config("mx_ragged", cfg_id=131, N=333, d=1024, E=8, S=2, k=2, I=640, P=4, score="sigmoid"),
    small_config("mx_wide_d", cfg_id=132, N=300, d=4096, E=8, S=1, k=2, I=256, P=4),
    # no shared expert, groups of 0..few rows
    small_config("mx_sparse", cfg_id=133, N=40, d=512, E=32, S=0, k=2, I=128, P=4),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
def test_mx_layer_staged(cfg):
    inp = gpu_inputs(cfg)
    r = _staged(cfg, inp)
    E, S, N, k, I, d = cfg.E, cfg.S, cfg.N, cfg.k, cfg.I, cfg.d
    A = N * k
    # (i) quantisation of x and of every weight row
    xq_ref, xsf_ref = F.quantize_mx(inp["x"].float().cpu().numpy())
    assert np.array_equal(_np(r["x_q"]), xq_ref) and np.array_equal(_np(r["x_sf"]), xsf_ref)
    w13q_ref, w13sf_ref = F.quantize_mx(inp["w13"].float().cpu().numpy().reshape(-1, d))
    w2q_ref, w2sf_ref = F.quantize_mx(inp["w2"].float().cpu().numpy().reshape(-1, I))
    assert np.array_equal(_np(r["w13_q"]).reshape(-1, d), w13q_ref)
    assert np.array_equal(_np(r["w13_sf"]).reshape(-1, d // 32), w13sf_ref)
    assert np.array_equal(_np(r["w2_q"]).reshape(-1, I), w2q_ref)
    assert np.array_equal(_np(r["w2_sf"]).reshape(-1, I // 32), w2sf_ref)
    # (ii) the MX dispatch payload
    row2tok = _np(r["lay"]["row2tok"])
    assert np.array_equal(_np(r["xp"]), xq_ref[row2tok // k])
    assert np.array_equal(_np(r["xp_sf"]), xsf_ref[row2tok // k])
    # (iii) FC1 on the oracle's codes, per expert (routed rows in layout order, then shared)
    n_e, off = _np(r["lay"]["n_e"]), _np(r["lay"]["expert_off"])
    w13q = w13q_ref.reshape(E + S, 2 * I, d)
    w13sf = w13sf_ref.reshape(E + S, 2 * I, d // 32)
    h_ref = np.zeros((A + S * N, I))
    for e in range(E):
        if n_e[e]:
            rows = slice(off[e], off[e] + n_e[e])
            tok = row2tok[rows] // k
            h_ref[rows] = F.fc1_mx(xq_ref[tok], xsf_ref[tok], w13q[e], w13sf[e], I)
    for s in range(S):
        h_ref[A + s * N:A + (s + 1) * N] = F.fc1_mx(xq_ref, xsf_ref, w13q[E + s], w13sf[E + s], I)
    assert_close_rel(r["h"], h_ref, what=f"{cfg.name} h")
    # (iv) the quantiser on the GPU's stored h
    hq_gpu_ref, hsf_gpu_ref = F.quantize_mx(r["h"].float().cpu().numpy())
    assert np.array_equal(_np(r["h_q"]), hq_gpu_ref) and np.array_equal(_np(r["h_sf"]), hsf_gpu_ref)
    # (v) FC2 x gate on those codes
    w2q = w2q_ref.reshape(E + S, d, I)
    w2sf = w2sf_ref.reshape(E + S, d, I // 32)
    gate_row = O.f64(r["w"]).reshape(-1)[row2tok]

    def fc2_all(hq, hsf):
        o = np.zeros((A + S * N, d))
        for e in range(E):
            if n_e[e]:
                rows = slice(off[e], off[e] + n_e[e])
                o[rows] = F.fc2_mx(hq[rows], hsf[rows], w2q[e], w2sf[e]) * gate_row[rows, None]
        for s in range(S):
            rows = slice(A + s * N, A + (s + 1) * N)
            o[rows] = F.fc2_mx(hq[rows], hsf[rows], w2q[E + s], w2sf[E + s])
        return o

    assert_close_fro(r["out"], fc2_all(hq_gpu_ref, hsf_gpu_ref), what=f"{cfg.name} out")
    # end to end from the seeded inputs alone: the oracle's own h, rounded to bf16 where the
    # path stores it, quantised by the oracle, FC2, combine
    hq_ref, hsf_ref = F.quantize_mx(_to_bf16(h_ref).astype(np.float32))
    o_ref = fc2_all(hq_ref, hsf_ref)
    tok2row = _np(r["lay"]["tok2row"])
    y_ref = sum(o_ref[tok2row[np.arange(N) * k + j]] for j in range(k))
    for s in range(S):
        y_ref = y_ref + o_ref[A + s * N:A + (s + 1) * N]
    assert_close_fro(r["y"], y_ref, what=f"{cfg.name} y (oracle end to end)")
    # MX against the unquantised float64 layer (reported)
    gates = O.gate_weights(O.gate_logits(cfg, inp["x"], inp["w_gate"], inp["bias"]), _np(r["ids"]).astype(np.int64),
                           cfg.score, cfg.renormalize)
    y64 = O.moe_tokens_direct(cfg, inp["x"], _np(r["ids"]).astype(np.int64), gates, inp["w13"], inp["w2"],
                              np.arange(N))
    rel = np.linalg.norm(O.f64(r["y"]) - y64) / np.linalg.norm(y64)
    print(f"{cfg.name}: MX layer vs unquantised float64 layer, relative Frobenius error {rel:.4f}")
    assert rel < 0.1
    # the fused entry point runs the same kernels; with the shared experts on a side stream
    # it gives the same bits
    y = moe.layer_forward_mx(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], r["w13_q"],
                             r["w13_sf"], r["w2_q"], r["w2_sf"])
    y_ov = moe.layer_forward_mx(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], r["w13_q"],
                                r["w13_sf"], r["w2_q"], r["w2_sf"], side_stream=torch.cuda.Stream())
    torch.cuda.synchronize()
    assert torch.equal(y, r["y"]) and torch.equal(y_ov, r["y"])


@pytest.mark.parametrize("name", ["fine", "wide", "decode", "hot_cal"])
def test_mx_full_size_sampled(name):
    """Full-size workloads: x quantisation bit-exact, the sampled experts' weight codes and
    scales bit-exact, sampled rows of h and out against the oracle (covering first and last
    rows of the sampled groups, and of the shared experts), fused == staged."""
    cfg = CONFIGS[name]
    inp = gpu_inputs(cfg)
    r = _staged(cfg, inp)
    k, I, E, d = cfg.k, cfg.I, cfg.E, cfg.d
    xq_ref, xsf_ref = F.quantize_mx(inp["x"].float().cpu().numpy())
    assert np.array_equal(_np(r["x_q"]), xq_ref) and np.array_equal(_np(r["x_sf"]), xsf_ref)
    row2tok = _np(r["lay"]["row2tok"])
    n_e, off = _np(r["lay"]["n_e"]), _np(r["lay"]["expert_off"])
    rng = np.random.default_rng(0)
    hq, hsf = _np(r["h_q"]), _np(r["h_sf"])
    busy = np.flatnonzero(n_e > 0)
    for e in rng.choice(busy, min(5, len(busy)), replace=False):
        w13q_ref, w13sf_ref = F.quantize_mx(inp["w13"][e].float().cpu().numpy())
        w2q_ref, w2sf_ref = F.quantize_mx(inp["w2"][e].float().cpu().numpy())
        assert np.array_equal(_np(r["w13_q"][e]), w13q_ref) and np.array_equal(_np(r["w13_sf"][e]), w13sf_ref)
        assert np.array_equal(_np(r["w2_q"][e]), w2q_ref) and np.array_equal(_np(r["w2_sf"][e]), w2sf_ref)
        local = np.unique(np.concatenate([[0, n_e[e] - 1], rng.choice(n_e[e], min(6, n_e[e]), replace=False)]))
        rows = off[e] + local
        tok = row2tok[rows] // k
        assert_close_rel(r["h"][torch.tensor(rows)], F.fc1_mx(xq_ref[tok], xsf_ref[tok], w13q_ref, w13sf_ref, I),
                         what=f"h expert {e}")
        g = O.f64(r["w"]).reshape(-1)[row2tok[rows]]
        assert_close_fro(r["out"][torch.tensor(rows)], F.fc2_mx(hq[rows], hsf[rows], w2q_ref, w2sf_ref) * g[:, None],
                         what=f"out expert {e}")
    A = cfg.N * k
    for s_ in range(cfg.S):  # the shared experts: sampled token rows, first and last included
        e = E + s_
        w13q_ref, w13sf_ref = F.quantize_mx(inp["w13"][e].float().cpu().numpy())
        w2q_ref, w2sf_ref = F.quantize_mx(inp["w2"][e].float().cpu().numpy())
        tok = np.unique(np.concatenate([[0, cfg.N - 1], rng.choice(cfg.N, min(6, cfg.N), replace=False)]))
        rows = A + s_ * cfg.N + tok
        assert_close_rel(r["h"][torch.tensor(rows)], F.fc1_mx(xq_ref[tok], xsf_ref[tok], w13q_ref, w13sf_ref, I),
                         what=f"h shared expert {s_}")
        assert_close_fro(r["out"][torch.tensor(rows)], F.fc2_mx(hq[rows], hsf[rows], w2q_ref, w2sf_ref),
                         what=f"out shared expert {s_}")
    y = moe.layer_forward_mx(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], r["w13_q"],
                             r["w13_sf"], r["w2_q"], r["w2_sf"])
    torch.cuda.synchronize()
    assert torch.equal(y, r["y"])


def test_mx_rejects_unsupported_shapes():
    cfg = small_config("mx_bad", cfg_id=134, N=64, d=256, E=8, S=0, k=2, I=128, P=2)  # d % 512 != 0
    inp = gpu_inputs(cfg)
    x_q, x_sf = moe.quantize_mx(inp["x"])
    w13_q, w13_sf = moe.quantize_mx(inp["w13"])
    w2_q, w2_sf = moe.quantize_mx(inp["w2"])
    with pytest.raises(moe.MoEError):
        moe.layer_forward_mx(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], w13_q, w13_sf, w2_q,
                             w2_sf)


@pytest.mark.parametrize("factor", [0.0, 0.7])
def test_mx_layer_with_capacity_drops(factor):
    """Assignments dropped by a capacity factor (id -1) take no row: the MX permute skips
    them and y equals the oracle's MX layer over the kept assignments (factor 0: the shared
    expert alone)."""
    cfg = SMALL[0]
    inp = gpu_inputs(cfg)
    E, S, N, k, I, d = cfg.E, cfg.S, cfg.N, cfg.k, cfg.I, cfg.d
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    kept = moe.capacity_drop(cfg, ids, moe.capacity_of(factor, cfg), status=status)
    lay = moe.dispatch_layout(cfg, kept, inp["expert_owner"], status=status)
    x_q, x_sf = moe.quantize_mx(inp["x"])
    w13_q, w13_sf = moe.quantize_mx(inp["w13"])
    w2_q, w2_sf = moe.quantize_mx(inp["w2"])
    xp, xp_sf = moe.permute_mx(cfg, lay, x_q, x_sf)
    h, h_q, h_sf, out = moe.grouped_ffn_mx(cfg, lay, xp, xp_sf, x_q, x_sf, w13_q, w13_sf, w2_q, w2_sf, topk_w=w)
    y = moe.combine(cfg, lay, out)
    torch.cuda.synchronize()
    assert status.item() == 0
    kept_np = kept.cpu().numpy().astype(np.int64)
    assert (kept_np < 0).any()
    xq_ref, xsf_ref = F.quantize_mx(inp["x"].float().cpu().numpy())
    w13q, w13sf = F.quantize_mx(inp["w13"].float().cpu().numpy().reshape(-1, d))
    w2q, w2sf = F.quantize_mx(inp["w2"].float().cpu().numpy().reshape(-1, I))
    w13q, w13sf = w13q.reshape(E + S, 2 * I, d), w13sf.reshape(E + S, 2 * I, d // 32)
    w2q, w2sf = w2q.reshape(E + S, d, I), w2sf.reshape(E + S, d, I // 32)
    gates = O.f64(w)

    def expert(e, toks):  # the MX expert on token rows, h rounded to bf16 and quantised
        hh = F.fc1_mx(xq_ref[toks], xsf_ref[toks], w13q[e], w13sf[e], I)
        hq, hs = F.quantize_mx(_to_bf16(hh).astype(np.float32))
        return F.fc2_mx(hq, hs, w2q[e], w2sf[e])

    y_ref = np.zeros((N, d))
    for e in range(E):
        t, j = np.nonzero(kept_np == e)
        if len(t):
            y_ref[t] += expert(e, t) * gates[t, j][:, None]
    for s in range(S):
        y_ref += expert(E + s, np.arange(N))
    assert_close_fro(y, y_ref, what=f"MX layer with capacity factor {factor}")


def test_mx_forward_is_deterministic_and_graph_capturable():
    """Two runs give the same bits; the MX forward, one-stream and overlapped, captured in a
    CUDA graph and replayed gives them too (workspace and weights set up before capture)."""
    cfg = SMALL[1]
    inp = gpu_inputs(cfg)
    w13_q, w13_sf = moe.quantize_mx(inp["w13"])
    w2_q, w2_sf = moe.quantize_mx(inp["w2"])
    ws = torch.empty(moe.workspace_bytes_mx(cfg), dtype=torch.uint8, device="cuda")
    args = (cfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], w13_q, w13_sf, w2_q, w2_sf)
    y1 = moe.layer_forward_mx(*args, ws=ws)
    y2 = moe.layer_forward_mx(*args, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    side = torch.cuda.Stream()
    for overlapped in (False, True):
        kw = dict(side_stream=side) if overlapped else {}
        y3 = torch.empty_like(y1)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            moe.layer_forward_mx(*args, y=y3, ws=ws, **kw)  # warm-up on the capture stream
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            moe.layer_forward_mx(*args, y=y3, ws=ws, **kw)
        for _ in range(2):
            y3.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(y3, y1)
        del g
