"""The layer as a pipeline over token chunks (moe_layer_forward_chunked; the ep_deepep
explainer §7, pipelined overlap of dispatch, experts and combine over micro-batches).

Each chunk is routed in the one router launch and then laid out, permuted, run through
its experts and combined on its own; every token's rows are computed by the same kernels
in the same k order as in the unchunked layer, so y must be bit-identical to
moe_layer_forward for any chunk count, including counts that do not divide N and chunks
that are empty.  One case is also compared with the float64 oracle, and the host-side
refusals are checked.
"""
import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from moe_inputs import CONFIGS, small_config
from oracle import moe_oracle as O
from tests.gpu_cases import assert_close_fro, gpu_inputs

pytestmark = pytest.mark.gpu

CASES = [
    small_config("ch_plain", cfg_id=70, N=257, d=200, E=8, S=1, k=2, I=136, P=2),
    small_config("ch_grouped", cfg_id=72, N=190, d=192, E=32, S=1, k=4, I=128, P=8, n_groups=8, topk_groups=3,
                 score="sigmoid"),
    small_config("ch_pairs", cfg_id=79, N=700, d=4096, E=8, S=1, k=2, I=200, P=4),
    small_config("ch_e256", cfg_id=82, N=640, d=4096, E=256, S=1, k=4, I=128, P=32, bias="zipf", bias_alpha=0.5),
    small_config("ch_f32", cfg_id=75, N=129, d=96, E=8, S=1, k=2, I=72, P=4, dtype="f32"),
    small_config("ch_tiny_n", cfg_id=73, N=5, d=64, E=8, S=0, k=2, I=64, P=2),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_chunked_forward_is_bit_identical(cfg):
    inp = gpu_inputs(cfg)
    args = (inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"])
    y_ref = moe.layer_forward(cfg, *args)
    side = torch.cuda.Stream()
    for n_chunks in (1, 2, 3, 5, 8):
        y = moe.layer_forward_chunked(cfg, n_chunks, *args, side)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), (cfg.name, n_chunks)


def test_chunked_forward_against_the_oracle():
    cfg = CASES[1]
    inp = gpu_inputs(cfg)
    logits, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    y = moe.layer_forward_chunked(cfg, 3, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"],
                                  inp["w2"], torch.cuda.Stream())
    torch.cuda.synchronize()
    ref = O.moe_layer(cfg, inp["x"], inp["w_gate"], inp["bias"], inp["w13"], inp["w2"],
                      select_keys=logits.cpu().numpy())
    assert_close_fro(y, ref["y"], what="chunked y")


def test_chunked_wide_layer_bit_identical():
    """The wide workload in 2 chunks: each expert's rows fall into other tile kinds of the
    CTA-pair GEMM (full blocks, carried rows, short tiles) than in the whole batch."""
    cfg = CONFIGS["wide"]
    inp = gpu_inputs(cfg)
    args = (inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"])
    y_ref = moe.layer_forward(cfg, *args)
    y = moe.layer_forward_chunked(cfg, 2, *args, torch.cuda.Stream())
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)


def test_chunked_forward_host_errors():
    cfg = CASES[0]
    inp = gpu_inputs(cfg)
    args = (inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"])
    side = torch.cuda.Stream()
    for bad in (0, 17):
        with pytest.raises(moe.MoEError) as e:
            moe.layer_forward_chunked(cfg, bad, *args, side, ws=torch.empty(1 << 20, dtype=torch.uint8,
                                                                              device="cuda"))
        assert e.value.status == 1
    with pytest.raises(moe.MoEError) as e:
        moe.layer_forward_chunked(cfg, 2, *args, side, ws=torch.empty(1024, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 3
    assert moe.workspace_bytes_chunked(cfg, 4) >= moe.workspace_bytes(cfg)
    assert moe.workspace_bytes_chunked(cfg, 0) == 0 and moe.workspace_bytes_chunked(cfg, 17) == 0
