"""GPU test of moe_dispatch_layout_noalloc, the layout entry point for callers that
cannot allocate device memory (a plugin inside a runtime that owns every device buffer,
a serving loop that must never call cudaMalloc, a service whose memory budget is fixed at
start-up).  Its scratch is an array built into the library.

It must return exactly what moe_dispatch_layout returns with a caller workspace, on two
or more calls in a row: each later call reuses the array the previous one left behind,
with a different routing and size, so stale contents would show.  The sizes include the
documented limit (N*k = 131072 assignments with E = 256, P = 32) and the hot-spot
workload's shape.  This file is collected last.
"""
import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import small_config

pytestmark = pytest.mark.gpu


def _routing(N, E, k, seed):
    """Distinct experts per token drawn from a skewed popularity (vectorised Gumbel top-k)."""
    rng = np.random.default_rng(seed)
    logp = np.log(rng.dirichlet(np.full(E, 0.5)) + 1e-12)
    keys = logp[None, :] + rng.gumbel(size=(N, E))
    ids = np.argsort(-keys, axis=1)[:, :k]
    return torch.tensor(ids, dtype=torch.int32, device="cuda")


def _check_same(cfg, ids, owner=None):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = moe.dispatch_layout_noalloc(cfg, ids, owner, status=status)
    ref = moe.dispatch_layout(cfg, ids, owner)
    torch.cuda.synchronize()
    assert status.item() == 0
    for key, v in ref.as_dict().items():   # integer maps: bit-exact
        assert torch.equal(got[key], v), (cfg.name, key)


def test_noalloc_layout_matches_workspace_layout_in_a_row():
    cases = [
        (small_config("noalloc_a", N=3000, d=64, E=128, S=1, k=8, I=64, P=16), 11),
        (small_config("noalloc_b", N=517, d=64, E=64, S=0, k=6, I=64, P=8), 12),
        # the documented limit: 131072 assignments, E = 256, P = 32 (1.72 MB of scratch)
        (small_config("noalloc_limit", N=16384, d=64, E=256, S=1, k=8, I=64, P=32), 13),
        # the hot-spot workload's shape: N = 16384, top-8 of 128 experts, 16 owners
        (small_config("noalloc_hot", N=16384, d=64, E=128, S=0, k=8, I=64, P=16), 14),
        (small_config("noalloc_c", N=5, d=64, E=8, S=0, k=2, I=64, P=2), 15),
    ]
    assert moe.layout_workspace_bytes(cases[2][0]) <= 2 << 20
    for cfg, seed in cases:  # calls in a row on the shared built-in scratch
        _check_same(cfg, _routing(cfg.N, cfg.E, cfg.k, seed))
    # a custom placement table at the limit, after the others
    cfg = cases[2][0]
    owner = torch.tensor(np.random.default_rng(3).permutation(np.arange(cfg.E) % cfg.P), dtype=torch.int32,
                         device="cuda")
    _check_same(cfg, _routing(cfg.N, cfg.E, cfg.k, 16), owner)


def test_noalloc_rejects_sizes_beyond_the_array():
    cfg = small_config("noalloc_big", N=40000, d=64, E=256, S=0, k=8, I=64, P=32)
    assert moe.layout_workspace_bytes(cfg) > 2 << 20
    ids = torch.zeros(cfg.N, cfg.k, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        moe.dispatch_layout_noalloc(cfg, ids)
    assert e.value.status == 2  # MOE_ERR_UNSUPPORTED
    assert "2 MiB" in str(e.value)  # the refusal says why (moe_last_error)
