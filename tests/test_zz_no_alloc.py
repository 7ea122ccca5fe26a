"""GPU test of moe_dispatch_layout_noalloc, the layout entry point for callers that
cannot allocate device memory (its scratch is an array built into the library).

It must return exactly what moe_dispatch_layout returns with a caller workspace, on two
calls in a row: the second call reuses the array the first one left behind, with a
different routing and size, so stale contents would show.  This file is collected last.
"""
import numpy as np
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import small_config

pytestmark = pytest.mark.gpu


def _routing(N, E, k, seed):
    rng = np.random.default_rng(seed)
    p = rng.dirichlet(np.full(E, 0.5))
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(N)])
    return torch.tensor(ids, dtype=torch.int32, device="cuda")


def test_noalloc_layout_matches_workspace_layout_twice():
    cases = [
        (small_config("noalloc_a", N=3000, d=64, E=128, S=1, k=8, I=64, P=16), 11),
        (small_config("noalloc_b", N=517, d=64, E=64, S=0, k=6, I=64, P=8), 12),
    ]
    for cfg, seed in cases:  # two calls in a row on the shared built-in scratch
        ids = _routing(cfg.N, cfg.E, cfg.k, seed)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = moe.dispatch_layout_noalloc(cfg, ids, status=status)
        ref = moe.dispatch_layout(cfg, ids)
        torch.cuda.synchronize()
        assert status.item() == 0
        for key, v in ref.as_dict().items():   # integer maps: bit-exact
            assert torch.equal(got[key], v), (cfg.name, key)


def test_noalloc_rejects_sizes_beyond_the_array():
    cfg = small_config("noalloc_big", N=40000, d=64, E=256, S=0, k=8, I=64, P=32)
    ids = torch.zeros(cfg.N, cfg.k, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        moe.dispatch_layout_noalloc(cfg, ids)
    assert e.value.status == 2  # MOE_ERR_UNSUPPORTED
