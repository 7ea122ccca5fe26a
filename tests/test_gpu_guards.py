"""Guard bands around every output buffer (a stand-in for a memory checker, which is not
available here): each output is the middle of a larger allocation whose 4 KiB bands on
both sides hold a fixed byte pattern; after the calls, the bands must be untouched.
Ragged shapes, the CTA-pair path, dropped assignments, redundant slots and FP8 are
covered.
"""
import math

import pytest
import torch

import dispatch_combine_grouped_b200 as moe
from dispatch_combine_grouped_b200 import binding
from moe_inputs import small_config
from tests.gpu_cases import gpu_inputs

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """Allocations with guard bands; check() asserts every band still holds the pattern."""

    def __init__(self):
        self.raws = []

    def __call__(self, shape, dtype):
        n = math.prod(shape) * torch.empty(0, dtype=dtype).element_size()
        raw = torch.full((2 * GUARD + max(n, 1),), PATTERN, dtype=torch.uint8, device="cuda")
        self.raws.append((raw, n))
        return raw[GUARD:GUARD + n].view(dtype).view(shape)

    def layout(self, cfg):
        lay = moe.Layout(cfg)
        for k, size in lay.sizes.items():
            lay.t[k] = self((max(size, 1),), torch.int32)
        lay.c = binding.CLayout(*[lay.t[k].data_ptr() for k in binding.LAYOUT_FIELDS])
        return lay

    def check(self):
        torch.cuda.synchronize()
        for i, (raw, n) in enumerate(self.raws):
            head, tail = raw[:GUARD], raw[GUARD + n:]
            assert bool((head == PATTERN).all()) and bool((tail == PATTERN).all()), f"guard band {i} written"


CASES = [
    small_config("g_ragged", cfg_id=100, N=257, d=200, E=8, S=1, k=2, I=136, P=2),
    small_config("g_pairs", cfg_id=101, N=640, d=4096, E=8, S=1, k=2, I=192, P=4),
    small_config("g_f32", cfg_id=102, N=129, d=96, E=8, S=1, k=2, I=72, P=4, dtype="f32"),
    small_config("g_many", cfg_id=103, N=1000, d=256, E=64, S=2, k=6, I=128, P=8, n_groups=8, topk_groups=4),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_bf16_path_writes_only_its_buffers(cfg):
    inp = gpu_inputs(cfg)
    g = Guarded()
    dt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    A, rows = cfg.N * cfg.k, cfg.N * cfg.k + cfg.S * cfg.N
    logits, ids, w = g((cfg.N, cfg.E), torch.float32), g((cfg.N, cfg.k), torch.int32), g((cfg.N, cfg.k), torch.float32)
    moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"], out=(logits, ids, w))
    lay = moe.dispatch_layout(cfg, ids, inp["expert_owner"], layout=g.layout(cfg))
    xp = moe.permute(cfg, lay, inp["x"], out=g((A, cfg.d), dt))
    h, out = moe.grouped_ffn(cfg, lay, xp, inp["x"], inp["w13"], inp["w2"], topk_w=w, h=g((rows, cfg.I), dt),
                             out=g((rows, cfg.d), dt))
    moe.combine(cfg, lay, out, y=g((cfg.N, cfg.d), dt))
    # dropped assignments and redundant slots on the same inputs
    kept = moe.capacity_drop(cfg, ids, moe.capacity_of(0.8, cfg), out=g((cfg.N, cfg.k), torch.int32))
    lay2 = moe.dispatch_layout(cfg, kept, inp["expert_owner"], layout=g.layout(cfg))
    xp2 = moe.permute(cfg, lay2, inp["x"], out=g((A, cfg.d), dt))
    _, out2 = moe.grouped_ffn(cfg, lay2, xp2, inp["x"], inp["w13"], inp["w2"], topk_w=w, h=g((rows, cfg.I), dt),
                              out=g((rows, cfg.d), dt))
    moe.combine(cfg, lay2, out2, y=g((cfg.N, cfg.d), dt))
    R = cfg.P
    n_e = torch.bincount(ids.reshape(-1).long(), minlength=cfg.E).cpu().numpy()
    plan = moe.eplb_plan(n_e, R, cfg.P)
    moe.eplb_assign(cfg, ids, torch.tensor(plan["replica_off"], device="cuda"),
                    torch.tensor(plan["replica_slots"], device="cuda"), cfg.E + R,
                    out=g((cfg.N, cfg.k), torch.int32))
    g.check()


@pytest.mark.parametrize("cfg", [CASES[1], small_config("g_f8", cfg_id=104, N=333, d=512, E=8, S=2, k=2, I=208,
                                                          P=4)], ids=["g_pairs", "g_f8"])
def test_fp8_path_writes_only_its_buffers(cfg):
    inp = gpu_inputs(cfg)
    g = Guarded()
    A, rows = cfg.N * cfg.k, cfg.N * cfg.k + cfg.S * cfg.N
    _, ids, w = moe.route(cfg, inp["x"], inp["w_gate"], inp["bias"])
    lay = moe.dispatch_layout(cfg, ids, inp["expert_owner"], layout=g.layout(cfg))
    x_q, x_s = moe.quantize_fp8(inp["x"], out=g((cfg.N, cfg.d), torch.uint8), scale=g((cfg.N,), torch.float32))
    E2, I2 = cfg.E + cfg.S, 2 * cfg.I
    w13_q, w13_s = moe.quantize_fp8(inp["w13"], out=g((E2, I2, cfg.d), torch.uint8), scale=g((E2, I2), torch.float32))
    w2_q, w2_s = moe.quantize_fp8(inp["w2"], out=g((E2, cfg.d, cfg.I), torch.uint8),
                                  scale=g((E2, cfg.d), torch.float32))
    xp = moe.permute_fp8(cfg, lay, x_q, out=g((A, cfg.d), torch.uint8))
    _, _, _, out = moe.grouped_ffn_fp8(cfg, lay, xp, x_q, x_s, w13_q, w13_s, w2_q, w2_s, topk_w=w,
                                       h=g((rows, cfg.I), torch.bfloat16), h_q=g((rows, cfg.I), torch.uint8),
                                       h_scale=g((rows,), torch.float32), out=g((rows, cfg.d), torch.bfloat16))
    moe.combine(cfg, lay, out, y=g((cfg.N, cfg.d), torch.bfloat16))
    g.check()
