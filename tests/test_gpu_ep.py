"""Expert parallelism across GPUs (moe_ep_*) with P ranks emulated on one device.

Every rank has its own window and the window table holds all of them, so each rank's
kernels store into and load from the other ranks' windows exactly as they would through
peer mappings.  The ranks' calls are issued stage by stage on one stream (all notifies,
then all layouts, dispatches, expert FFNs and combines), so every wait finds its flags
already set: no kernel waits on another.

Compared with the oracle element by element: the EP layout (destinations, owner rows),
the count table, received rows and gates in every window (bit-exact), and y (float
tolerance); and y against the one-GPU layer on the concatenated batch (bit-exact).
"""
import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from dispatch_combine_grouped_b200 import ep
from moe_inputs import small_config
from oracle import moe_oracle as O
from tests.gpu_cases import assert_close_fro, gpu_inputs

pytestmark = pytest.mark.gpu

CASES = [
    (small_config("ep_bf16", cfg_id=90, N=512, d=256, E=16, S=1, k=4, I=128, P=4), None),
    (small_config("ep_pairs", cfg_id=91, N=1024, d=4096, E=8, S=1, k=2, I=256, P=2), None),
    (small_config("ep_f32", cfg_id=92, N=256, d=128, E=8, S=0, k=2, I=64, P=2, dtype="f32"), None),
    (small_config("ep_grouped_owner", cfg_id=93, N=384, d=192, E=32, S=2, k=4, I=96, P=4, n_groups=4,
                  topk_groups=2, score="sigmoid"), "random"),
    (small_config("ep_unequal", cfg_id=94, N=512, d=256, E=16, S=1, k=4, I=128, P=4), [200, 0, 57, 255]),
]


def _owner(cfg, spec):
    if spec != "random":
        return None
    g = torch.Generator().manual_seed(cfg.cfg_id)
    return torch.randint(0, cfg.P, (cfg.E,), generator=g, dtype=torch.int32).cuda()


def _shards(cfg, spec):
    if isinstance(spec, list):
        return spec
    return [cfg.N // cfg.P] * cfg.P


class Emulated:
    """P ranks on one device: windows, groups, per-rank weights, workspaces and handles."""

    def __init__(self, cfg, shards, owner=None, capacity=None):
        self.cfg, self.shards, self.owner = cfg, shards, owner
        self.capacity = capacity or cfg.N * cfg.k
        self.rcfg = [cfg.replace(N=n) for n in shards]
        self.groups, self.windows = ep.emulated_groups(self.rcfg[0], self.capacity, owner, rank_cfgs=self.rcfg)
        self.owned = [ep.owned_experts(cfg.E, cfg.P, r, owner.cpu() if owner is not None else None)
                      for r in range(cfg.P)]
        self.ws = [ep.alloc_ws(c, self.capacity) for c in self.rcfg]
        self.handles = [ep.Handle(c, len(o)) for c, o in zip(self.rcfg, self.owned)]
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def weights(self, inp):
        E, S = self.cfg.E, self.cfg.S
        out = []
        for o in self.owned:
            idx = torch.tensor(list(o) + list(range(E, E + S)), dtype=torch.long, device="cuda")
            out.append((inp["w13"].index_select(0, idx).contiguous(), inp["w2"].index_select(0, idx).contiguous()))
        return out

    def launch(self, xs, ids, w, wts, ys):
        """One EP step of every rank, stage by stage (no synchronisation: capturable)."""
        P = self.cfg.P
        for r in range(P):
            ep.notify(self.rcfg[r], self.groups[r], ids[r], self.ws[r], self.status)
        for r in range(P):
            ep.layout(self.rcfg[r], self.groups[r], ids[r], self.handles[r], self.ws[r], self.owner, self.status)
        for r in range(P):
            ep.dispatch(self.rcfg[r], self.groups[r], xs[r], w[r], self.handles[r])
        for r in range(P):
            ep.expert_ffn(self.rcfg[r], self.groups[r], xs[r], wts[r][0], wts[r][1], self.handles[r], self.ws[r],
                          self.status)
        for r in range(P):
            ep.combine(self.rcfg[r], self.groups[r], self.handles[r], y=ys[r], status=self.status)

    def step(self, inp, ids=None, w=None):
        cfg, P = self.cfg, self.cfg.P
        starts = np.concatenate([[0], np.cumsum(self.shards)])
        xs = [inp["x"][starts[r]:starts[r + 1]] for r in range(P)]
        if ids is None:
            routed = [moe.route(self.rcfg[r], xs[r], inp["w_gate"], inp["bias"]) for r in range(P)]
            ids = [rt[1] for rt in routed]
            w = [rt[2] for rt in routed]
        ys = [torch.empty(c.N, c.d, dtype=c.torch_dtype, device="cuda") for c in self.rcfg]
        self.launch(xs, ids, w, self.weights(inp), ys)
        torch.cuda.synchronize()
        return dict(xs=xs, ids=ids, w=w, y=torch.cat(ys))


def check_windows(em, res, lay):
    """Count tables, received rows and gates in every window, bit-exact."""
    cfg = em.cfg
    for j in range(cfg.P):
        v = ep.window_views(em.rcfg[j], em.capacity, em.windows[j])
        assert np.array_equal(v["cnt_tab"].cpu().numpy(), lay["cnt"]), f"count table of rank {j}"
        rows = lay["recv"][j][:em.capacity]
        R = len(rows)
        if R == 0:
            continue
        x_want = torch.stack([res["xs"][i][a // cfg.k] for i, a in rows])
        g_want = torch.stack([res["w"][i].reshape(-1)[a] for i, a in rows])
        assert torch.equal(v["x_recv"][:R], x_want), f"received rows of owner {j}"
        assert torch.equal(v["gate"][:R], g_want), f"gates of owner {j}"


def check_handles(em, lay):
    for r in range(em.cfg.P):
        h = em.handles[r].as_dict()
        assert np.array_equal(h["dest"].cpu().numpy(), lay["dest"][r]), f"dest of rank {r}"
        assert np.array_equal(h["owner_n_e"].cpu().numpy(), lay["owner_n_e"][r]), f"owner_n_e of rank {r}"
        assert np.array_equal(h["owner_off"].cpu().numpy(), lay["owner_off"][r]), f"owner_off of rank {r}"


def y_oracle(cfg, inp, ids_all, owner, routed_ids=None):
    """routed_ids: the router's choice before any drop; the gates come from it (a kept
    assignment keeps its gate), the rows from ids_all."""
    ref = O.dispatch_layout(ids_all, cfg.E, cfg.P, owner, cfg.S)
    g64 = O.gate_weights(O.gate_logits(cfg, inp["x"], inp["w_gate"], inp["bias"]),
                         ids_all if routed_ids is None else routed_ids, cfg.score, cfg.renormalize)
    xp = O.permute(inp["x"], ref, cfg.k)
    o = O.experts_on_rows(xp, ref, inp["w13"], inp["w2"], cfg.E)
    shared = [O.swiglu_expert(inp["x"], inp["w13"][cfg.E + s], inp["w2"][cfg.E + s]) for s in range(cfg.S)]
    return O.combine(o, ref, g64, cfg.N, cfg.k, shared)


@pytest.mark.parametrize("cfg,spec", CASES, ids=[c.name for c, _ in CASES])
def test_ep_step_matches_oracle(cfg, spec):
    inp = gpu_inputs(cfg)
    owner = _owner(cfg, spec)
    em = Emulated(cfg, _shards(cfg, spec), owner)
    res = em.step(inp)
    assert int(em.status.item()) == 0
    own_np = owner.cpu().numpy() if owner is not None else None
    lay = O.ep_layout([i.cpu().numpy() for i in res["ids"]], cfg.E, cfg.P, own_np, em.capacity)
    check_handles(em, lay)
    check_windows(em, res, lay)
    ids_all = torch.cat(res["ids"]).cpu().numpy()
    assert_close_fro(res["y"], y_oracle(cfg, inp, ids_all, own_np), what="EP y")
    # the one-GPU layer on the concatenated batch gives the same y, bit for bit
    y1 = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], owner, inp["w13"], inp["w2"])
    torch.cuda.synchronize()
    assert torch.equal(res["y"], y1)


def test_ep_epochs_reuse_windows():
    """Three steps on the same windows with different inputs: flags only grow, nothing is reset."""
    cfg, _ = CASES[0]
    em = Emulated(cfg, _shards(cfg, None))
    for epoch in (1, 2, 3):
        inp = gpu_inputs(cfg, seed_offset=epoch)
        res = em.step(inp)
        assert int(em.status.item()) == 0
        y1 = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], None, inp["w13"], inp["w2"])
        torch.cuda.synchronize()
        assert torch.equal(res["y"], y1), f"epoch {epoch}"
        flags = ep.window_views(em.rcfg[0], em.capacity, em.windows[0])
        assert flags["cnt_flag"][:cfg.P].tolist() == [epoch] * cfg.P
        assert flags["disp_flag"][:cfg.P].tolist() == [epoch] * cfg.P
        assert flags["done_flag"][:cfg.P].tolist() == [epoch] * cfg.P
        assert flags["step"].tolist() == [epoch]


def test_ep_capacity_overflow_drops_rows_in_bounds():
    """capacity below an owner's load: rows past it are not received, every rank reports
    MOE_ERR_WORKSPACE, and nothing outside the windows is written (guard bands)."""
    cfg, _ = CASES[0]
    inp = gpu_inputs(cfg)
    rcfg = cfg.replace(N=cfg.N // cfg.P)
    probe = Emulated(cfg, _shards(cfg, None))
    res0 = probe.step(inp)
    lay_full = O.ep_layout([i.cpu().numpy() for i in res0["ids"]], cfg.E, cfg.P)
    cap = int(lay_full["R"].max()) - 7
    em = Emulated(cfg, _shards(cfg, None), capacity=cap)
    # windows with 4 KiB guard bands on both sides
    nbytes, G = ep.window_bytes(rcfg, cap), 4096
    raws = [torch.full((nbytes + 2 * G,), 0xA5, dtype=torch.uint8, device="cuda") for _ in range(cfg.P)]
    for r in raws:
        r[G:G + nbytes].zero_()
    em.windows = [r[G:G + nbytes] for r in raws]
    em.groups = [ep.Group(r, cap, len(em.owned[r]), [w.data_ptr() for w in em.windows]) for r in range(cfg.P)]
    res = em.step(inp, ids=res0["ids"], w=res0["w"])
    assert int(em.status.item()) == moe.binding.MOE_ERR_WORKSPACE
    lay = O.ep_layout([i.cpu().numpy() for i in res["ids"]], cfg.E, cfg.P, None, cap)
    check_handles(em, lay)
    check_windows(em, res, lay)
    for r in raws:
        assert bool((r[:G] == 0xA5).all()) and bool((r[G + nbytes:] == 0xA5).all()), "guard band written"


def test_ep_dropped_assignments():
    """Capacity-factor drops (-1 ids) take no row anywhere and add nothing to y."""
    cfg, _ = CASES[0]
    inp = gpu_inputs(cfg)
    em = Emulated(cfg, _shards(cfg, None))
    n = cfg.N // cfg.P
    routed = [moe.route(cfg.replace(N=n), inp["x"][r * n:(r + 1) * n], inp["w_gate"], inp["bias"])
              for r in range(cfg.P)]
    ids = [moe.capacity_drop(cfg.replace(N=n), rt[1], 20) for rt in routed]
    w = [rt[2] for rt in routed]
    res = em.step(inp, ids=ids, w=w)
    assert int(em.status.item()) == 0
    lay = O.ep_layout([i.cpu().numpy() for i in ids], cfg.E, cfg.P, None, em.capacity)
    assert any((i.cpu().numpy() == -1).any() for i in ids)
    check_handles(em, lay)
    check_windows(em, res, lay)
    ids_all = torch.cat(ids).cpu().numpy()
    routed_all = torch.cat([rt[1] for rt in routed]).cpu().numpy()
    assert_close_fro(res["y"], y_oracle(cfg, inp, ids_all, None, routed_all), what="EP y with drops")
    # the one-GPU steps on the same kept ids and gates give the same y, bit for bit
    lay1 = moe.dispatch_layout(cfg, torch.cat(ids))
    xp = moe.permute(cfg, lay1, inp["x"])
    _, out = moe.grouped_ffn(cfg, lay1, xp, inp["x"], inp["w13"], inp["w2"], topk_w=torch.cat(w))
    y1 = moe.combine(cfg, lay1, out)
    torch.cuda.synchronize()
    assert torch.equal(res["y"], y1)


def test_ep_one_rank_layer_forward_matches_one_gpu_layer():
    """P = 1: moe_ep_layer_forward (router + the five steps in one call), and its overlapped
    form (shared experts on a side stream), equal moe_layer_forward."""
    cfg = small_config("ep_p1", cfg_id=95, N=300, d=256, E=16, S=1, k=4, I=128, P=1)
    inp = gpu_inputs(cfg)
    cap = cfg.N * cfg.k
    groups, windows = ep.emulated_groups(cfg, cap)
    ws = ep.alloc_ws(cfg, cap)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    h = ep.Handle(cfg, cfg.E)
    side = torch.cuda.Stream()
    for epoch in (1, 2, 3):
        y = ep.layer_forward(cfg, groups[0], inp["x"], inp["w_gate"], inp["bias"], inp["w13"], inp["w2"], ws,
                             handle=h, status=status, side_stream=side if epoch == 3 else None)
        y1 = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], None, inp["w13"], inp["w2"])
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(y, y1), f"epoch {epoch}"
    assert int(ep.window_views(cfg, cap, windows[0])["step"].item()) == 3


def test_ep_wait_times_out_and_context_stays_usable():
    """Rank 0 starts a second step that no other rank starts: its layout's bounded wait for
    the count rows gives up (2 s), MOE_ERR_TIMEOUT is reported, no destination is written,
    and the context still runs."""
    cfg, _ = CASES[0]
    inp = gpu_inputs(cfg)
    em = Emulated(cfg, _shards(cfg, None))
    res = em.step(inp)
    assert int(em.status.item()) == 0
    rc = em.rcfg[0]
    ep.notify(rc, em.groups[0], res["ids"][0], em.ws[0], em.status)
    ep.layout(rc, em.groups[0], res["ids"][0], em.handles[0], em.ws[0], None, em.status)
    torch.cuda.synchronize()
    assert int(em.status.item()) == moe.binding.MOE_ERR_TIMEOUT
    assert bool((em.handles[0].as_dict()["dest"] == -1).all())
    z = torch.ones(1024, device="cuda") * 2
    assert float(z.sum().item()) == 2048.0


def test_ep_failed_dispatch_fails_the_step_on_every_rank():
    """Rank 1 skips its dispatch in one step: every owner's bounded wait for it gives up,
    each owner publishes its "done" with the error mark, and every rank's combine reports
    MOE_ERR_TIMEOUT on its own status and leaves y unwritten, instead of summing rows of
    owners whose inputs did not all arrive.  The next step runs normally again."""
    cfg, _ = CASES[0]
    inp = gpu_inputs(cfg)
    em = Emulated(cfg, _shards(cfg, None))
    res = em.step(inp)
    assert int(em.status.item()) == 0
    P, wts = cfg.P, em.weights(inp)
    st = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(P)]
    ys = [torch.full((c.N, c.d), 7.0, dtype=c.torch_dtype, device="cuda") for c in em.rcfg]
    for r in range(P):
        ep.notify(em.rcfg[r], em.groups[r], res["ids"][r], em.ws[r], st[r])
    for r in range(P):
        ep.layout(em.rcfg[r], em.groups[r], res["ids"][r], em.handles[r], em.ws[r], None, st[r])
    for r in range(P):
        if r != 1:
            ep.dispatch(em.rcfg[r], em.groups[r], res["xs"][r], res["w"][r], em.handles[r])
    for r in range(P):
        ep.expert_ffn(em.rcfg[r], em.groups[r], res["xs"][r], wts[r][0], wts[r][1], em.handles[r], em.ws[r], st[r])
    for r in range(P):
        ep.combine(em.rcfg[r], em.groups[r], em.handles[r], y=ys[r], status=st[r])
    torch.cuda.synchronize()
    for r in range(P):
        assert int(st[r].item()) == moe.binding.MOE_ERR_TIMEOUT, f"status of rank {r}"
        assert bool((ys[r] == 7.0).all()), f"y of rank {r} was written"
        v = ep.window_views(em.rcfg[r], em.capacity, em.windows[r])
        assert int(v["err_step"].item()) == int(v["step"].item()) == 2
        assert int(v["done_flag"][r].item()) == 2 - 2 ** 63   # epoch 2 with the error mark (int64 view)
    again = em.step(inp)
    assert int(em.status.item()) == 0
    assert torch.equal(again["y"], res["y"])


def test_ep_host_errors():
    cfg, _ = CASES[0]
    rc = cfg.replace(N=cfg.N // cfg.P)
    em = Emulated(cfg, _shards(cfg, None))
    ids = torch.zeros(rc.N, rc.k, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError):   # rank outside [0, P)
        ep.notify(rc, ep.Group(cfg.P, em.capacity, 4, em.groups[0].windows), ids, em.ws[0])
    with pytest.raises(moe.MoEError):   # capacity 0
        ep.notify(rc, ep.Group(0, 0, 4, em.groups[0].windows), ids, em.ws[0])
    with pytest.raises(moe.MoEError):   # small workspace
        ep.notify(rc, em.groups[0], ids, em.ws[0][:16])
    with pytest.raises(moe.MoEError):   # unaligned window
        bad = list(em.groups[0].windows)
        bad[1] += 16
        ep.notify(rc, ep.Group(0, em.capacity, 4, bad), ids, em.ws[0])
    assert int(em.groups[0].windows[0]) and all(ep.window_views(rc, em.capacity, w)["step"].item() == 0
                                                 for w in em.windows), "a refused call launched nothing"


def test_ep_step_captured_in_cuda_graph():
    """The emulated step of all ranks captured once and replayed with new inputs: the step
    number lives in the windows, so each replay is a new step with correct waits."""
    cfg, _ = CASES[0]
    em = Emulated(cfg, _shards(cfg, None))
    P, n = cfg.P, cfg.N // cfg.P
    inp = gpu_inputs(cfg)
    x = inp["x"].clone()
    xs = [x[r * n:(r + 1) * n] for r in range(P)]
    routed = [moe.route(em.rcfg[r], xs[r], inp["w_gate"], inp["bias"]) for r in range(P)]
    ids, w = [rt[1] for rt in routed], [rt[2] for rt in routed]
    wts = em.weights(inp)
    ys = [torch.empty(n, cfg.d, dtype=torch.bfloat16, device="cuda") for _ in range(P)]

    def body():
        for r in range(P):
            moe.route(em.rcfg[r], xs[r], inp["w_gate"], inp["bias"], out=routed[r])
        em.launch(xs, ids, w, wts, ys)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        body()  # eager step 1
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        body()
    for rep in range(3):
        new = gpu_inputs(cfg, seed_offset=10 + rep)["x"]
        x.copy_(new)
        g.replay()
        torch.cuda.synchronize()
        assert int(em.status.item()) == 0
        y1 = moe.layer_forward(cfg, new, inp["w_gate"], inp["bias"], None, inp["w13"], inp["w2"])
        torch.cuda.synchronize()
        assert torch.equal(torch.cat(ys), y1), f"replay {rep}"
    steps = [int(ep.window_views(em.rcfg[r], em.capacity, em.windows[r])["step"].item()) for r in range(P)]
    assert steps == [4] * P   # one eager step + three replays (the capture itself launches nothing)


FP8_CASES = [
    (small_config("ep_f8", cfg_id=96, N=512, d=256, E=16, S=1, k=4, I=128, P=4), None),
    (small_config("ep_f8_pairs", cfg_id=97, N=1024, d=4096, E=8, S=1, k=2, I=256, P=2), None),
    (small_config("ep_f8_owner", cfg_id=98, N=384, d=192, E=32, S=2, k=4, I=96, P=4, n_groups=4, topk_groups=2,
                  score="sigmoid"), "random"),
]


@pytest.mark.parametrize("cfg,spec", FP8_CASES, ids=[c.name for c, _ in FP8_CASES])
def test_ep_fp8_step_matches_one_gpu_fp8_layer(cfg, spec):
    """FP8 dispatch (e4m3 rows + token scales over the peer windows), FP8 expert FFN on the
    owners, bf16 combine: the received codes and scales are the quantised token rows bit
    for bit, and y equals the one-GPU FP8 layer bit for bit."""
    inp = gpu_inputs(cfg)
    owner = _owner(cfg, spec)
    em = Emulated(cfg, _shards(cfg, spec), owner)
    em.ws = [ep.alloc_ws(c, em.capacity, fp8=True) for c in em.rcfg]
    P, n = cfg.P, cfg.N // cfg.P
    w13_q, w13_s = moe.quantize_fp8(inp["w13"])
    w2_q, w2_s = moe.quantize_fp8(inp["w2"])
    xs = [inp["x"][r * n:(r + 1) * n] for r in range(P)]
    routed = [moe.route(em.rcfg[r], xs[r], inp["w_gate"], inp["bias"]) for r in range(P)]
    ids, w = [rt[1] for rt in routed], [rt[2] for rt in routed]
    qs = [moe.quantize_fp8(x) for x in xs]
    E, S = cfg.E, cfg.S
    ys = []
    for r in range(P):
        ep.notify(em.rcfg[r], em.groups[r], ids[r], em.ws[r], em.status)
    for r in range(P):
        ep.layout(em.rcfg[r], em.groups[r], ids[r], em.handles[r], em.ws[r], owner, em.status)
    for r in range(P):
        ep.dispatch_fp8(em.rcfg[r], em.groups[r], qs[r][0], qs[r][1], w[r], em.handles[r])
    for r in range(P):
        idx = torch.tensor(list(em.owned[r]) + list(range(E, E + S)), dtype=torch.long, device="cuda")
        ep.expert_ffn_fp8(em.rcfg[r], em.groups[r], qs[r][0], qs[r][1], w13_q.index_select(0, idx),
                          w13_s.index_select(0, idx), w2_q.index_select(0, idx), w2_s.index_select(0, idx),
                          em.handles[r], em.ws[r], em.status)
    for r in range(P):
        ys.append(ep.combine(em.rcfg[r], em.groups[r], em.handles[r], status=em.status))
    torch.cuda.synchronize()
    assert int(em.status.item()) == 0
    own_np = owner.cpu().numpy() if owner is not None else None
    lay = O.ep_layout([i.cpu().numpy() for i in ids], cfg.E, cfg.P, own_np, em.capacity)
    check_handles(em, lay)
    for j in range(P):
        v = ep.window_views(em.rcfg[j], em.capacity, em.windows[j])
        rows = lay["recv"][j]
        R = len(rows)
        if R == 0:
            continue
        assert torch.equal(v["x_recv_fp8"][:R], torch.stack([qs[i][0][a // cfg.k] for i, a in rows]))
        assert torch.equal(v["scale"][:R], torch.stack([qs[i][1][a // cfg.k] for i, a in rows]))
        assert torch.equal(v["gate"][:R], torch.stack([w[i].reshape(-1)[a] for i, a in rows]))
    y1 = moe.layer_forward_fp8(cfg, inp["x"], inp["w_gate"], inp["bias"], owner, w13_q, w13_s, w2_q, w2_s)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys), y1)


def test_ep_fp8_layer_forward_one_rank():
    """P = 1: moe_ep_layer_forward_fp8 and its overlapped form equal moe_layer_forward_fp8."""
    cfg = small_config("ep_f8_p1", cfg_id=99, N=300, d=256, E=16, S=1, k=4, I=128, P=1)
    inp = gpu_inputs(cfg)
    cap = cfg.N * cfg.k
    groups, windows = ep.emulated_groups(cfg, cap)
    ws = ep.alloc_ws(cfg, cap, fp8=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w13_q, w13_s = moe.quantize_fp8(inp["w13"])
    w2_q, w2_s = moe.quantize_fp8(inp["w2"])
    side = torch.cuda.Stream()
    for step in range(3):
        y = ep.layer_forward_fp8(cfg, groups[0], inp["x"], inp["w_gate"], inp["bias"], w13_q, w13_s, w2_q, w2_s, ws,
                                 status=status, side_stream=side if step == 2 else None)
        y1 = moe.layer_forward_fp8(cfg, inp["x"], inp["w_gate"], inp["bias"], None, w13_q, w13_s, w2_q, w2_s)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(y, y1)


def test_ep_with_redundant_expert_slots():
    """EPLB across ranks (Wide EP: redundant copies of hot experts balance the owners'
    receive load): each rank maps its logical ids to physical slots (moe_eplb_assign on
    its own assignments), the EP path runs over the E + R slots with the plan's slot
    owners and slot weights, and y equals the one-GPU layer over the logical experts bit
    for bit (copies hold identical weights)."""
    cfg = small_config("ep_eplb", cfg_id=110, N=512, d=256, E=16, S=1, k=4, I=128, P=4, bias="zipf",
                       bias_alpha=0.6)
    inp = gpu_inputs(cfg)
    R, P, n = 4, cfg.P, cfg.N // cfg.P
    _, ids_all, _ = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    n_e = torch.bincount(ids_all.reshape(-1).long(), minlength=cfg.E).cpu().numpy()
    plan = moe.eplb_plan(n_e, R, P)
    pcfg = moe.physical_config(cfg, R)
    owner = torch.tensor(plan["slot_owner"], dtype=torch.int32, device="cuda")
    rep_off = torch.tensor(plan["replica_off"], dtype=torch.int32, device="cuda")
    rep_slots = torch.tensor(plan["replica_slots"], dtype=torch.int32, device="cuda")
    phys_inp = dict(inp, w13=moe.eplb_place_weights(plan["slot_expert"], cfg.E, cfg.S, inp["w13"]),
                    w2=moe.eplb_place_weights(plan["slot_expert"], cfg.E, cfg.S, inp["w2"]))
    em = Emulated(pcfg, [n] * P, owner)
    rcfg = cfg.replace(N=n)
    ids, w = [], []
    for r in range(P):
        _, i_r, w_r = moe.route(rcfg, inp["x"][r * n:(r + 1) * n], inp["w_gate"], inp["bias"])
        ids.append(moe.eplb_assign(rcfg, i_r, rep_off, rep_slots, cfg.E + R))
        w.append(w_r)
    res = em.step(phys_inp, ids=ids, w=w)
    assert int(em.status.item()) == 0
    lay = O.ep_layout([i.cpu().numpy() for i in ids], pcfg.E, P, owner.cpu().numpy(), em.capacity)
    check_handles(em, lay)
    check_windows(em, res, lay)
    y1 = moe.layer_forward(cfg, inp["x"], inp["w_gate"], inp["bias"], None, inp["w13"], inp["w2"])
    torch.cuda.synchronize()
    assert torch.equal(res["y"], y1)
    # the plan balances the owners' receive rows at least as well as the contiguous placement
    base = O.ep_layout([ids_all[r * n:(r + 1) * n].cpu().numpy() for r in range(P)], cfg.E, P)
    print("owner receive rows, contiguous:", base["R"].tolist(), "with", R, "copies:", lay["R"].tolist())
    assert lay["R"].max() <= base["R"].max()


@pytest.mark.parametrize("cfg", [
    small_config("ep_p32", cfg_id=111, N=32 * 24, d=128, E=64, S=1, k=4, I=64, P=32),
    small_config("ep_e512", cfg_id=112, N=256, d=128, E=512, S=0, k=8, I=64, P=8),
], ids=["P32", "E512"])
def test_ep_at_size_limits(cfg):
    """The largest rank count (P = 32) and the largest expert-slot count (E = 512, ids and
    gates given directly, as a caller mapping to physical slots would): EP layout and
    windows against the oracle, y bit-identical to the one-GPU steps on the same ids."""
    inp = gpu_inputs(cfg)
    P, n = cfg.P, cfg.N // cfg.P
    g = torch.Generator(device="cuda").manual_seed(cfg.cfg_id)
    ids_all = torch.stack([torch.randperm(cfg.E, generator=g, device="cuda")[:cfg.k] for _ in range(cfg.N)])
    ids_all = ids_all.to(torch.int32).contiguous()
    w_all = torch.rand(cfg.N, cfg.k, generator=g, device="cuda")
    ids = [ids_all[r * n:(r + 1) * n].contiguous() for r in range(P)]
    w = [w_all[r * n:(r + 1) * n].contiguous() for r in range(P)]
    em = Emulated(cfg, [n] * P)
    res = em.step(inp, ids=ids, w=w)
    assert int(em.status.item()) == 0
    lay = O.ep_layout([i.cpu().numpy() for i in ids], cfg.E, P, None, em.capacity)
    check_handles(em, lay)
    check_windows(em, res, lay)
    lay1 = moe.dispatch_layout(cfg, ids_all)
    xp = moe.permute(cfg, lay1, inp["x"])
    _, out = moe.grouped_ffn(cfg, lay1, xp, inp["x"], inp["w13"], inp["w2"], topk_w=w_all)
    y1 = moe.combine(cfg, lay1, out)
    torch.cuda.synchronize()
    assert torch.equal(res["y"], y1)


MX_CASES = [
    (small_config("ep_mx", cfg_id=136, N=512, d=512, E=16, S=1, k=4, I=128, P=4), None),
    (small_config("ep_mx_owner", cfg_id=137, N=384, d=1024, E=32, S=2, k=4, I=256, P=4, n_groups=4, topk_groups=2,
                  score="sigmoid"), "random"),
]


@pytest.mark.parametrize("cfg,spec", MX_CASES, ids=[c.name for c, _ in MX_CASES])
def test_ep_mx_step_matches_one_gpu_mx_layer(cfg, spec):
    """MX dispatch (e4m3 rows + their E8M0 scale rows over the peer windows), MX expert FFN
    on the owners, bf16 combine: the received codes and scale rows are the quantised token
    rows bit for bit, and y equals the one-GPU MX layer bit for bit."""
    inp = gpu_inputs(cfg)
    owner = _owner(cfg, spec)
    em = Emulated(cfg, _shards(cfg, spec), owner)
    em.ws = [ep.alloc_ws(c, em.capacity, mx=True) for c in em.rcfg]
    P, n = cfg.P, cfg.N // cfg.P
    w13_q, w13_sf = moe.quantize_mx(inp["w13"])
    w2_q, w2_sf = moe.quantize_mx(inp["w2"])
    xs = [inp["x"][r * n:(r + 1) * n] for r in range(P)]
    routed = [moe.route(em.rcfg[r], xs[r], inp["w_gate"], inp["bias"]) for r in range(P)]
    ids, w = [rt[1] for rt in routed], [rt[2] for rt in routed]
    qs = [moe.quantize_mx(x) for x in xs]
    E, S = cfg.E, cfg.S
    ys = []
    for r in range(P):
        ep.notify(em.rcfg[r], em.groups[r], ids[r], em.ws[r], em.status)
    for r in range(P):
        ep.layout(em.rcfg[r], em.groups[r], ids[r], em.handles[r], em.ws[r], owner, em.status)
    for r in range(P):
        ep.dispatch_mx(em.rcfg[r], em.groups[r], qs[r][0], qs[r][1], w[r], em.handles[r])
    for r in range(P):
        idx = torch.tensor(list(em.owned[r]) + list(range(E, E + S)), dtype=torch.long, device="cuda")
        ep.expert_ffn_mx(em.rcfg[r], em.groups[r], qs[r][0], qs[r][1], w13_q.index_select(0, idx),
                         w13_sf.index_select(0, idx), w2_q.index_select(0, idx), w2_sf.index_select(0, idx),
                         em.handles[r], em.ws[r], em.status)
    for r in range(P):
        ys.append(ep.combine(em.rcfg[r], em.groups[r], em.handles[r], status=em.status))
    torch.cuda.synchronize()
    assert int(em.status.item()) == 0
    own_np = owner.cpu().numpy() if owner is not None else None
    lay = O.ep_layout([i.cpu().numpy() for i in ids], cfg.E, cfg.P, own_np, em.capacity)
    check_handles(em, lay)
    for j in range(P):
        v = ep.window_views(em.rcfg[j], em.capacity, em.windows[j])
        rows = lay["recv"][j]
        R = len(rows)
        if R == 0:
            continue
        assert torch.equal(v["x_recv_fp8"][:R], torch.stack([qs[i][0][a // cfg.k] for i, a in rows]))
        assert torch.equal(v["x_recv_mx_sf"][:R], torch.stack([qs[i][1][a // cfg.k] for i, a in rows]))
        assert torch.equal(v["gate"][:R], torch.stack([w[i].reshape(-1)[a] for i, a in rows]))
    y1 = moe.layer_forward_mx(cfg, inp["x"], inp["w_gate"], inp["bias"], owner, w13_q, w13_sf, w2_q, w2_sf)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys), y1)


def test_ep_mx_layer_forward_one_rank():
    """P = 1: moe_ep_layer_forward_mx and its overlapped form equal moe_layer_forward_mx."""
    cfg = small_config("ep_mx_p1", cfg_id=138, N=300, d=512, E=16, S=1, k=4, I=128, P=1)
    inp = gpu_inputs(cfg)
    cap = cfg.N * cfg.k
    groups, windows = ep.emulated_groups(cfg, cap)
    ws = ep.alloc_ws(cfg, cap, mx=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w13_q, w13_sf = moe.quantize_mx(inp["w13"])
    w2_q, w2_sf = moe.quantize_mx(inp["w2"])
    side = torch.cuda.Stream()
    for step in range(3):
        y = ep.layer_forward_mx(cfg, groups[0], inp["x"], inp["w_gate"], inp["bias"], w13_q, w13_sf, w2_q, w2_sf, ws,
                                status=status, side_stream=side if step == 2 else None)
        y1 = moe.layer_forward_mx(cfg, inp["x"], inp["w_gate"], inp["bias"], None, w13_q, w13_sf, w2_q, w2_sf)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(y, y1)
