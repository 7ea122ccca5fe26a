"""The bench's algorithmic work and peak choice, on CPU.

The FLOPs and bytes the bench divides by its timings are checked against the closed forms
of the layer for the five workloads: FFN FLOP = 6 (A + S N) d I, permute bytes = (N + A) d b
(each token row read once, each assignment row written once), combine bytes = (A + S N + N)
d b (each summed row read once, y written once), router FLOP = 2 N d E.  A few values are
also written out as numbers (the fine and wide workloads) so that a changed workload table
shows up here.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from moe_inputs import CONFIGS  # noqa: E402


@pytest.mark.parametrize("name", ["tiny", "fine", "wide", "decode", "hot", "hot_cal"])
def test_algorithmic_work_closed_forms(name):
    c = CONFIGS[name]
    a = bench.algorithmic(c)
    A, b = c.N * c.k, (2 if c.dtype == "bf16" else 4)
    assert a["ffn_flops"] == 6 * (A + c.S * c.N) * c.d * c.I
    assert a["fc1_flops"] + a["fc2_flops"] == a["ffn_flops"]
    assert a["fc1_flops"] == 2 * a["fc2_flops"]
    assert a["permute_bytes"] == (c.N + A) * c.d * b
    assert a["combine_bytes"] == (A + c.S * c.N + c.N) * c.d * b
    assert a["router_flops"] == 2 * c.N * c.d * c.E
    assert a["fc1_weight_bytes"] == (c.E + c.S) * 2 * c.I * c.d * b


def test_workload_numbers():
    fine, wide = bench.algorithmic(CONFIGS["fine"]), bench.algorithmic(CONFIGS["wide"])
    assert fine["ffn_flops"] == pytest.approx(566.9e9, rel=1e-3)     # 425.2 routed + 141.7 shared
    assert fine["permute_bytes"] == pytest.approx(117.4e6, rel=1e-3)
    assert wide["ffn_flops"] == pytest.approx(6494e9, rel=1e-3)      # 5772 routed + 722 shared
    assert wide["permute_bytes"] == pytest.approx(1.057e9, rel=1e-3)
    # the routed FC1 of fine, the numerator of the bench's roofline line
    c = CONFIGS["fine"]
    assert 4.0 * c.N * c.k * c.d * c.I == pytest.approx(283.47e9, rel=1e-4)


def test_peak_follows_the_clock():
    peaks = {"bf16_tflops": 1693.9, "bf16_tflops_sustained": 1400.0}
    assert bench.tensor_peak(peaks, {"sm_mhz": 1965, "sm_max_mhz": 1965}) == (1693.9, "burst")
    assert bench.tensor_peak(peaks, {"sm_mhz": 1870, "sm_max_mhz": 1965}) == (1693.9, "burst")
    assert bench.tensor_peak(peaks, {"sm_mhz": 1455, "sm_max_mhz": 1965}) == (1400.0, "sustained")
    assert bench.tensor_peak(peaks, None) == (1400.0, "sustained")


def test_whole_job_rate_and_max_over_ranks():
    assert bench.whole_job_tokens_per_s(4096, 1, 0.5) == pytest.approx(4096 / 0.5e-3)
    assert bench.whole_job_tokens_per_s(4096, 8, 0.5) == pytest.approx(8 * 4096 / 0.5e-3)
    assert bench.max_over_ranks(2.5, 1) == 2.5


def test_layer_roofline_per_workload():
    """Layer roofline: router, permute and combine at HBM bandwidth, the FFN at the slower
    of its FLOPs at the tensor peak and its touched weights at HBM.  With the measured
    peaks the wide FFN is tensor-bound (near the ridge) and the decode FFN weight-bound."""
    hbm, tc = 6454.3, 1693.9
    wide = bench.roofline_layer_ms(CONFIGS["wide"], 256, hbm, tc)
    assert wide["ffn_bound"] == "tensor"
    assert wide["parts_ms"]["ffn"] == pytest.approx(6494e9 / 1693.9e12 * 1e3, rel=2e-3)
    assert wide["parts_ms"]["permute"] == pytest.approx(1.057e9 / 6454.3e9 * 1e3, rel=2e-3)
    assert wide["ms"] == pytest.approx(sum(wide["parts_ms"].values()))
    dec = bench.roofline_layer_ms(CONFIGS["decode"], 252, hbm, tc)
    assert dec["ffn_bound"] == "hbm"
    assert dec["parts_ms"]["ffn"] == pytest.approx(253 * 3 * 7168 * 2048 * 2 / 6454.3e9 * 1e3, rel=1e-9)


def test_both_arms_describe_the_workload_identically():
    for name in ("wide", "fine", "tiny"):
        assert bench.config_dict(CONFIGS[name], 1) == bench.config_dict(CONFIGS[name], 1)
        assert set(bench.config_dict(CONFIGS[name], 1)) == {"workload", "tokens_per_gpu", "l2", "parallelism"}


def test_spec_peak_scales_with_the_clock():
    assert bench.spec_at_clock(1965) == pytest.approx(2250.0)
    assert bench.spec_at_clock(1455) == pytest.approx(2250.0 * 1455 / 1965)


def test_default_workload_is_the_wide_layer():
    import sys as _sys
    old = _sys.argv
    _sys.argv = ["bench.py"]
    try:
        assert bench.parse().workload == "wide"
    finally:
        _sys.argv = old


def test_launch_count_per_step():
    # wide: router 2, layout 3, permute 1, routed FC1/FC2 2, shared FC1/FC2 2, combine 1
    assert bench.kernel_launches_per_step(CONFIGS["wide"]) == 11
    assert bench.kernel_launches_per_step(CONFIGS["fine"]) == 2 + 3 + 1 + 2 + 2 + 1
    assert bench.kernel_launches_per_step(CONFIGS["hot"]) == 2 + 3 + 1 + 2 + 0 + 1
