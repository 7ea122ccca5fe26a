"""Seeded random sweeps on the GPU against the oracle.

Layout and movement: random N, E (up to 512 slots), k (up to 8), P (up to 32), owner
tables and capacity drops; the layout must equal the oracle's bit for bit, the permute is
a bit copy, and the combine of given rows matches the float64 sum of the same rows.

Expert parallelism (ranks emulated on one device, see test_gpu_ep.py): random unequal
shards (some empty), owner tables, drops and capacities; every rank's EP layout and every
window's received rows against the oracle, y against the one-GPU steps bit for bit.
"""
import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from dispatch_combine_grouped_b200 import ep
from moe_inputs import small_config
from oracle import moe_oracle as O
from tests.gpu_cases import assert_layout_equal, gpu_inputs, layout_to_numpy

pytestmark = pytest.mark.gpu


def _random_ids(rng, N, E, k, drop):
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(N)]).astype(np.int32) if N else \
        np.zeros((0, k), np.int32)
    if drop and N:
        ids[rng.random(ids.shape) < drop] = -1
    return ids


@pytest.mark.parametrize("seed", range(12))
def test_random_layout_and_movement(seed):
    rng = np.random.default_rng(1000 + seed)
    P = int(rng.choice([1, 2, 4, 8, 16, 32]))
    E = P * int(rng.integers(1, max(2, 512 // P) + 1))
    E = min(E, 512)
    k = int(rng.integers(1, min(8, E) + 1))
    N = int(rng.integers(0, 3000))
    d = int(rng.choice([64, 128, 200, 256]))
    cfg = small_config(f"rnd{seed}", cfg_id=200 + seed, N=N, d=d, E=E, S=int(rng.integers(0, 3)), k=k, I=64, P=P)
    owner_np = rng.integers(0, P, size=E).astype(np.int32) if seed % 3 == 0 else None
    owner = torch.tensor(owner_np, device="cuda") if owner_np is not None else None
    ids_np = _random_ids(rng, N, E, k, drop=0.15 if seed % 2 else 0.0)
    ids = torch.tensor(ids_np, device="cuda").reshape(N, k)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lay = moe.dispatch_layout(cfg, ids, owner, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = O.dispatch_layout(ids_np, E, P, owner_np, cfg.S)
    assert_layout_equal(layout_to_numpy(lay), ref, P)
    if N == 0:
        return
    x = torch.randn(N, d, device="cuda").to(torch.bfloat16)
    xp = moe.permute(cfg, lay, x)
    torch.cuda.synchronize()
    kept = ref["tok2row"] >= 0
    assert torch.equal(xp[torch.tensor(ref["tok2row"][kept], device="cuda")],
                       x[torch.tensor(np.flatnonzero(kept) // k, device="cuda")])
    rows = N * k + cfg.S * N
    out = torch.randn(rows, d, device="cuda").to(torch.bfloat16)
    y = moe.combine(cfg, lay, out)
    torch.cuda.synchronize()
    o64 = O.f64(out)
    shared = [o64[N * k + s * N:N * k + (s + 1) * N] for s in range(cfg.S)]
    y_ref = O.combine(o64[:N * k], ref, np.ones((N, k)), N, k, shared)
    # one bf16 rounding (2^-9 relative) of an fp32 sum of at most k + S bf16 rows (fp32
    # rounding, about 1e-6 absolute at these magnitudes)
    np.testing.assert_allclose(O.f64(y), y_ref, rtol=2 ** -8, atol=1e-5)


@pytest.mark.parametrize("seed", range(6))
def test_random_expert_parallel_step(seed):
    rng = np.random.default_rng(2000 + seed)
    P = int(rng.choice([2, 3, 4, 8]))
    E = P * int(rng.integers(1, 5))
    k = int(rng.integers(1, min(4, E) + 1))
    S = int(rng.integers(0, 2))
    shards = [int(v) for v in rng.integers(0, 90, size=P)]
    shards[int(rng.integers(0, P))] = 0          # one rank without tokens
    N = sum(shards)
    cfg = small_config(f"eprnd{seed}", cfg_id=300 + seed, N=max(N, 1), d=128, E=E, S=S, k=k, I=64, P=P)
    inp = gpu_inputs(cfg)
    owner_np = rng.integers(0, P, size=E).astype(np.int32) if seed % 2 else None
    owner = torch.tensor(owner_np, device="cuda") if owner_np is not None else None
    ids_np = [_random_ids(rng, n, E, k, drop=0.1 if seed % 3 == 0 else 0.0) for n in shards]
    flat = np.concatenate([i.reshape(-1) for i in ids_np] + [np.zeros(0, np.int64)]).astype(np.int64)
    flat_load = np.bincount(flat[flat >= 0], minlength=E)
    own = owner_np if owner_np is not None else np.arange(E) // (E // P)
    need = int(np.bincount(own, weights=flat_load, minlength=P).max())
    cap = max(1, need - (5 if seed % 2 else 0))  # odd seeds: a capacity a little short
    rcfg = [cfg.replace(N=n) for n in shards]
    groups, windows = ep.emulated_groups(rcfg[0], cap, owner, rank_cfgs=rcfg)
    owned = [ep.owned_experts(E, P, r, owner_np) for r in range(P)]
    ws = [ep.alloc_ws(c, cap) for c in rcfg]
    hd = [ep.Handle(c, len(o)) for c, o in zip(rcfg, owned)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    starts = np.concatenate([[0], np.cumsum(shards)])
    xs = [inp["x"][starts[r]:starts[r + 1]] for r in range(P)]
    ids = [torch.tensor(i, device="cuda").reshape(n, k) for i, n in zip(ids_np, shards)]
    w = [torch.rand(n, k, device="cuda") for n in shards]
    for r in range(P):
        ep.notify(rcfg[r], groups[r], ids[r], ws[r], status)
    for r in range(P):
        ep.layout(rcfg[r], groups[r], ids[r], hd[r], ws[r], owner, status)
    for r in range(P):
        ep.dispatch(rcfg[r], groups[r], xs[r], w[r], hd[r])
    for r in range(P):
        idx = torch.tensor(list(owned[r]) + list(range(E, E + S)), dtype=torch.long, device="cuda")
        ep.expert_ffn(rcfg[r], groups[r], xs[r], inp["w13"].index_select(0, idx), inp["w2"].index_select(0, idx),
                      hd[r], ws[r], status)
    ys = [ep.combine(rcfg[r], groups[r], hd[r], status=status) for r in range(P)]
    torch.cuda.synchronize()
    lay = O.ep_layout(ids_np, E, P, owner_np, cap)
    overflow = bool((lay["R"] > cap).any())
    assert int(status.item()) == (moe.binding.MOE_ERR_WORKSPACE if overflow else 0)
    for r in range(P):
        h = hd[r].as_dict()
        assert np.array_equal(h["dest"].cpu().numpy(), lay["dest"][r]), f"dest of rank {r}"
        assert np.array_equal(h["owner_n_e"].cpu().numpy(), lay["owner_n_e"][r])
        assert np.array_equal(h["owner_off"].cpu().numpy(), lay["owner_off"][r])
        v = ep.window_views(rcfg[r], cap, windows[r])
        rows = lay["recv"][r][:cap]
        if len(rows):
            assert torch.equal(v["x_recv"][:len(rows)], torch.stack([xs[i][a // k] for i, a in rows]))
    if overflow or N == 0:
        return
    ids_all = torch.cat(ids)
    lay1 = moe.dispatch_layout(cfg.replace(N=N), ids_all, owner)
    xp = moe.permute(cfg.replace(N=N), lay1, inp["x"][:N])
    _, out = moe.grouped_ffn(cfg.replace(N=N), lay1, xp, inp["x"][:N], inp["w13"], inp["w2"], topk_w=torch.cat(w))
    y1 = moe.combine(cfg.replace(N=N), lay1, out)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys), y1)
