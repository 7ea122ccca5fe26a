"""Find the hot-spot bias scale alpha for which max_e n_e / mean_e n_e ~= 8 (seed 0).

Test infrastructure: runs the oracle's router and selection only.  The hot-spot workload
(N=16384, d=4096, E=128, top-8) biases the router logits by b_e = alpha * ln(1/rank_e);
with the literal alpha = 3 the hottest expert is picked by every token and the ratio
saturates at E/k = 16, so a calibrated alpha is kept beside the literal one.  The value
printed here is the one stored for the ``hot_cal`` workload in ``moe_inputs``.

    python -m oracle.calibrate_hot
"""
import numpy as np

from moe_inputs import CONFIGS, make_inputs, zipf_bias
from oracle import moe_oracle as O


def ratio(z_nobias, alpha, cfg):
    z = z_nobias + O.f64(zipf_bias(cfg.E, alpha))[None, :]
    ids = O.select_experts(z, cfg.k)
    n_e = np.bincount(ids.reshape(-1), minlength=cfg.E)
    return n_e.max() / n_e.mean(), n_e


def main(target=8.0):
    cfg = CONFIGS["hot"]
    inp = make_inputs(cfg, with_experts=False)
    z0 = O.router_logits(inp["x"], inp["w_gate"])
    lit, n_lit = ratio(z0, cfg.bias_alpha, cfg)
    print(f"literal alpha={cfg.bias_alpha}: max/mean n_e = {lit:.3f}, empty experts = {(n_lit == 0).sum()}")
    lo, hi = 0.0, 3.0
    for _ in range(12):                       # bisection on a grid of 3/4096
        mid = 0.5 * (lo + hi)
        r, _ = ratio(z0, mid, cfg)
        lo, hi = (mid, hi) if r < target else (lo, mid)
    r, n = ratio(z0, hi, cfg)
    print(f"calibrated alpha={hi!r}: max/mean n_e = {r:.3f}, empty experts = {(n == 0).sum()}")
    return hi


if __name__ == "__main__":
    main()
