"""Seeded synthetic inputs for one MoE layer, shared by the CUDA path's tests and the oracle.

This module holds the workload table and the random draws only. It contains none of
the layer's arithmetic (no routing, no layout, no expert math), so that the oracle and
the CUDA library can both consume its tensors without sharing any method code.

Workloads follow the shapes the pages discuss: fine-grained experts (DeepSeek MoE, 64
experts), DeepSeek-V3-style wide EP (256 experts, top-8, 8 groups), a decode batch, and
a skewed (hot-spot) router.  Draw rules: x ~ N(0, 1); router and expert weights
~ N(0, 1/d); each tensor has its own CPU/CUDA ``torch.Generator`` seeded with
``1000 * cfg_id + tensor_id`` (x=0, W_g=1, W13=2, W2=3, shared W13=4, shared W2=5),
drawn in fp32 and rounded to the config's dtype (round-to-nearest-even for bf16).
Expert weights are drawn one expert at a time so that the draw is the same however
large the stack is.
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["MoEConfig", "CONFIGS", "make_inputs", "hot_owner_table", "zipf_bias"]


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    cfg_id: int          # seed namespace
    N: int               # tokens
    d: int               # hidden size
    E: int               # routed experts
    S: int               # shared experts (always active, weight 1)
    k: int               # top-k
    I: int               # expert intermediate size (SwiGLU)
    P: int               # virtual expert-owner ranks
    n_groups: int = 1    # expert groups for group-limited routing (1 = plain top-k)
    topk_groups: int = 1 # groups kept per token
    score: str = "softmax"   # "softmax" | "sigmoid"
    renormalize: bool = True
    dtype: str = "bf16"      # "f32" | "bf16"
    bias: str = "none"       # "none" | "zipf"
    bias_alpha: float = 0.0  # b_e = alpha * ln(1 / rank_e), rank_e = e + 1
    bias_mode: str = "logits"  # "logits": bias in selection and gates | "selection": selection only
    owner: str = "contiguous"  # "contiguous" | "hot4"

    @property
    def A(self) -> int:
        return self.N * self.k

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)


# The five workloads (sizes, routing rule, placement) plus the calibrated hot-spot variant.
# hot_cal's alpha is the value found by oracle/calibrate_hot.py (max/mean n_e ~= 8 at seed 0).
CONFIGS = {
    "tiny": MoEConfig("tiny", 1, N=256, d=128, E=8, S=0, k=2, I=256, P=2,
                      score="softmax", renormalize=True, dtype="f32"),
    "fine": MoEConfig("fine", 2, N=4096, d=2048, E=64, S=2, k=6, I=1408, P=8,
                      score="softmax", renormalize=False),
    "wide": MoEConfig("wide", 3, N=8192, d=7168, E=256, S=1, k=8, I=2048, P=32,
                      n_groups=8, topk_groups=4, score="sigmoid", renormalize=True),
    "decode": MoEConfig("decode", 4, N=128, d=7168, E=256, S=1, k=8, I=2048, P=32,
                        n_groups=8, topk_groups=4, score="sigmoid", renormalize=True),
    "hot": MoEConfig("hot", 5, N=16384, d=4096, E=128, S=0, k=8, I=1536, P=16,
                     score="softmax", renormalize=True, bias="zipf", bias_alpha=3.0,
                     owner="hot4"),
    "hot_cal": MoEConfig("hot_cal", 5, N=16384, d=4096, E=128, S=0, k=8, I=1536, P=16,
                         score="softmax", renormalize=True, bias="zipf", bias_alpha=0.432861328125,
                         owner="hot4"),
}

# Reduced cases for profiler captures that must stay a few GB on the device: the wide
# layer's shapes and its n_e ~ 256 per expert with 32 experts (2.9 GB of weights), and the
# same with 4096 tokens so that the permute / combine traffic (0.5 GB) exceeds the L2.
PROFILE_CASES = {
    "wide_e32": MoEConfig("wide_e32", 6, N=1024, d=7168, E=32, S=1, k=8, I=2048, P=8,
                          n_groups=8, topk_groups=4, score="sigmoid", renormalize=True),
    "wide_e32_n4k": MoEConfig("wide_e32_n4k", 7, N=4096, d=7168, E=32, S=1, k=8, I=2048, P=8,
                              n_groups=8, topk_groups=4, score="sigmoid", renormalize=True),
}


def zipf_bias(E: int, alpha: float) -> torch.Tensor:
    """Router logit bias b_e = alpha * ln(1/rank_e) with rank_e = e + 1 (expert 0 hottest)."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    return (alpha * torch.log(1.0 / ranks)).to(torch.float32)


def hot_owner_table(E: int, P: int) -> torch.Tensor:
    """Expert -> owner placement with the 4 hottest experts on one owner.

    Owner 0 holds popularity ranks 1-4 (experts 0-3) and the 4 coldest experts
    (E-4 .. E-1); the remaining experts go round-robin over owners 1..P-1.  With
    E=128, P=16 every owner holds 8 experts.
    """
    if E % P != 0 or E < 8 or P < 2:
        raise ValueError("hot4 placement needs E % P == 0, E >= 8, P >= 2")
    owner = torch.empty(E, dtype=torch.int32)
    owner[:4] = 0
    owner[E - 4:] = 0
    mid = torch.arange(4, E - 4)
    owner[4:E - 4] = (1 + (mid - 4) % (P - 1)).to(torch.int32)
    return owner


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, gen, device, dtype):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _fill_expert_stack(dst, std, seed):
    """Fill dst[e] (one expert at a time) from one generator seeded with ``seed``."""
    g = _gen(dst.device, seed)
    for e in range(dst.shape[0]):
        dst[e] = _normal(tuple(dst.shape[1:]), std, g, dst.device, dst.dtype)


def make_inputs(cfg: MoEConfig, device="cpu", seed_offset: int = 0, with_experts: bool = True) -> dict:
    """Draw every input of the layer for ``cfg`` on ``device``.

    Returns a dict with
      x      [N, d]            activations (cfg dtype)
      w_gate [E, d]            router weight, one row per expert (cfg dtype)
      bias   [E] fp32 or None  router logit bias
      w13    [E+S, 2I, d]      expert gate rows [0, I) and up rows [I, 2I) (cfg dtype)
      w2     [E+S, d, I]       expert down projection (cfg dtype)
      expert_owner [E] int32 or None (None = contiguous owners e // (E/P))
    Shared experts are the last S entries of the stacks.
    """
    dt = cfg.torch_dtype
    base = 1000 * cfg.cfg_id + 100000 * seed_offset
    std = 1.0 / math.sqrt(cfg.d)
    out = {
        "x": _normal((cfg.N, cfg.d), 1.0, _gen(device, base + 0), device, dt),
        "w_gate": _normal((cfg.E, cfg.d), std, _gen(device, base + 1), device, dt),
        "bias": None,
        "expert_owner": None,
    }
    if cfg.bias == "zipf":
        out["bias"] = zipf_bias(cfg.E, cfg.bias_alpha).to(device)
    if cfg.owner == "hot4":
        out["expert_owner"] = hot_owner_table(cfg.E, cfg.P).to(device)
    if with_experts:
        E, S, I, d = cfg.E, cfg.S, cfg.I, cfg.d
        w13 = torch.empty((E + S, 2 * I, d), device=device, dtype=dt)
        w2 = torch.empty((E + S, d, I), device=device, dtype=dt)
        _fill_expert_stack(w13[:E], std, base + 2)
        _fill_expert_stack(w2[:E], std, base + 3)
        if S:
            _fill_expert_stack(w13[E:], std, base + 4)
            _fill_expert_stack(w2[E:], std, base + 5)
        out["w13"] = w13
        out["w2"] = w2
    return out


def small_config(name="small", **kw) -> MoEConfig:
    """A reduced workload for parity tests: same rules, sizes chosen by the caller."""
    base = dict(cfg_id=90, N=257, d=200, E=8, S=1, k=2, I=136, P=2)
    base.update(kw)
    return MoEConfig(name, **base)
