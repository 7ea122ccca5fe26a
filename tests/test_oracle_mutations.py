"""Planted mistakes in the oracle (CPU only): each must make at least one pin fail.

Each mutation is applied with monkeypatch to the oracle module only, so the rest of the
suite sees the unmodified oracle.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
import tests.test_oracle_pins as pins


def _fails(check, *args):
    with pytest.raises(AssertionError):
        check(*args)


def test_ties_to_higher_index_is_caught(monkeypatch):
    # reverse the tie order: equal keys now prefer the higher index
    monkeypatch.setattr(O, "_descending_stable",
                        lambda r: (len(r) - 1 - np.argsort(-r[::-1], kind="stable")))
    _fails(pins.check_worked_selection)


def test_silu_sign_is_caught(monkeypatch):
    monkeypatch.setattr(O, "silu", lambda z: z / (1.0 + np.exp(z)))
    _fails(pins.check_expert_vs_torch)
    _fails(pins.check_dense_special_case)


def test_swapped_gate_up_is_caught(monkeypatch):
    def swapped(x_rows, w13_e, w2_e):
        w13_e = O.f64(w13_e)
        I = w13_e.shape[0] // 2
        return O.__dict__["_orig_swiglu"](x_rows, np.concatenate([w13_e[I:], w13_e[:I]]), w2_e)
    monkeypatch.setitem(O.__dict__, "_orig_swiglu", O.swiglu_expert)
    monkeypatch.setattr(O, "swiglu_expert", swapped)
    _fails(pins.check_expert_vs_torch)


def test_transposed_down_projection_is_caught(monkeypatch):
    orig = O.swiglu_expert

    def transposed(x_rows, w13_e, w2_e):
        w2 = O.f64(w2_e)
        if w2.shape[0] != w2.shape[1]:
            pytest.skip("needs a square case")
        return orig(x_rows, w13_e, w2.T)
    # use square shapes so the transposed operand still multiplies
    monkeypatch.setattr(O, "swiglu_expert", transposed)
    rng = np.random.default_rng(0)
    x = rng.normal(size=(5, 6))
    w13 = rng.normal(size=(12, 6))
    w2 = rng.normal(size=(6, 6))
    with pytest.raises(AssertionError):
        np.testing.assert_allclose(O.swiglu_expert(x, w13, w2), pins._torch_swiglu(x, w13, w2),
                                   rtol=1e-12, atol=1e-12)


def test_wrong_source_shards_are_caught(monkeypatch):
    # round-robin sources instead of contiguous shards
    monkeypatch.setattr(O, "source_of_token", lambda N, P: np.arange(N, dtype=np.int64) % P)
    _fails(pins.check_worked_layout)


def test_missing_renormalisation_is_caught(monkeypatch):
    orig = O.gate_weights
    monkeypatch.setattr(O, "gate_weights", lambda z, ids, score="softmax", renormalize=True:
                        orig(z, ids, score, False))
    _fails(pins.check_worked_selection)


def test_dropped_gate_in_combine_is_caught(monkeypatch):
    orig = O.combine
    monkeypatch.setattr(O, "combine", lambda o, lay, g, N, k, shared_out=None:
                        orig(o, lay, np.ones_like(O.f64(g)), N, k, shared_out))
    _fails(pins.check_worked_output)


def test_dropped_shared_expert_is_caught(monkeypatch):
    orig = O.moe_tokens_direct

    def no_shared(cfg, *a, **kw):
        return orig(cfg.replace(S=0), *a, **kw)
    monkeypatch.setattr(O, "moe_tokens_direct", no_shared)
    _fails(pins.check_shared_expert_additive)


def test_expert_order_by_id_only_is_caught(monkeypatch):
    # ignore the owner when ordering rows (plain argsort by expert id)
    orig = O.dispatch_layout

    def by_id(ids, E, P, expert_owner=None, S=0):
        lay = orig(ids, E, P, expert_owner, S)
        flat = O.i64(ids).reshape(-1)
        row2tok = np.argsort(flat, kind="stable")
        lay["row2tok"] = row2tok
        lay["tok2row"] = np.empty_like(row2tok)
        lay["tok2row"][row2tok] = np.arange(len(row2tok))
        return lay
    monkeypatch.setattr(O, "dispatch_layout", by_id)
    _fails(pins.check_layout_naive_ranks, 2)


def test_bias_leaking_into_gates_is_caught(monkeypatch):
    # a correction bias that also shifts the gates
    monkeypatch.setattr(O, "gate_logits", lambda cfg, x, w_gate, bias: O.router_logits(x, w_gate, bias))
    _fails(pins.check_correction_bias)


# ---- EPLB oracle (redundant expert slots)
import tests.test_eplb_oracle as eplb_pins
from oracle import eplb as EP


def test_copies_to_the_coldest_expert_are_caught(monkeypatch):
    def coldest(load, R):
        load = np.asarray(load, dtype=np.int64)
        r = np.ones(len(load), dtype=np.int64)
        for _ in range(R):
            r[int(np.argmin(load / r))] += 1
        return r
    monkeypatch.setattr(EP, "replica_counts", coldest)
    _fails(eplb_pins.check_copy_counts_optimal, 3, 2, np.array([30, 5, 1]))
    _fails(eplb_pins.check_worked_example)


def test_replica_rank_off_by_one_is_caught(monkeypatch):
    def shifted(ids, replica_off, replica_slots):
        ids = np.asarray(ids, dtype=np.int64)
        flat = ids.reshape(-1)
        out = np.empty_like(flat)
        for e in range(len(replica_off) - 1):
            rows = np.flatnonzero(flat == e)
            r = replica_off[e + 1] - replica_off[e]
            out[rows] = np.asarray(replica_slots)[replica_off[e] + (np.arange(len(rows)) + 1) % r]
        return out.reshape(ids.shape)
    monkeypatch.setattr(EP, "assign", shifted)
    _fails(eplb_pins.check_worked_example)


# ---- FP8 oracle
import tests.test_fp8_oracle as fp8_pins
from oracle import fp8 as F8


def test_fp8_ties_away_from_even_are_caught(monkeypatch):
    orig = F8.e4m3_encode

    def up(v):
        v = np.asarray(v, dtype=np.float64)
        return orig(np.nextafter(np.abs(v), np.inf) * np.where(np.signbit(v), -1, 1))
    monkeypatch.setattr(F8, "e4m3_encode", up)
    _fails(fp8_pins.test_ties_go_to_the_even_code_and_large_values_saturate)


def test_fp8_wrong_scale_is_caught(monkeypatch):
    monkeypatch.setattr(F8, "E4M3_MAX", 240.0)
    _fails(fp8_pins.test_row_quantisation)


# ---- capacity (dropped assignments)
import tests.test_capacity_oracle as cap_pins


def test_dropping_the_first_instead_of_the_last_is_caught(monkeypatch):
    def last(ids, E, cap):
        ids = O.i64(ids)
        flat = ids.reshape(-1).copy()
        for e in range(E):
            rows = np.flatnonzero(flat == e)
            flat[rows[:max(len(rows) - cap, 0)]] = -1
        return flat.reshape(ids.shape)
    monkeypatch.setattr(O, "capacity_keep", last)
    _fails(cap_pins.check_worked_example)


def test_dropped_rows_leaking_into_combine_are_caught(monkeypatch):
    orig = O.combine

    def leaky(o_rows, layout, gates, N, k, shared_out=None):
        lay = dict(layout)
        lay["tok2row"] = np.where(layout["tok2row"] < 0, 0, layout["tok2row"])
        return orig(o_rows, lay, gates, N, k, shared_out)
    monkeypatch.setattr(O, "combine", leaky)
    _fails(cap_pins.check_layout_path_with_drops, 0.8)


# ---- the expert-parallel receive order (oracle.ep_layout): each planted order mistake
# must fail one of the EP pins in tests/test_ep_oracle.py
import tests.test_ep_oracle as ep_pins  # noqa: E402


def _ep_pins_fail():
    failed = 0
    for check, args in [(ep_pins.test_worked_example_two_ranks, ()),
                        (ep_pins.test_equal_shards_match_one_gpu_layout, (1,)),
                        (ep_pins.test_equal_shards_match_one_gpu_layout, (4,)),
                        (ep_pins.test_unequal_shards_and_capacity, (0,))]:
        try:
            check(*args)
        except AssertionError:
            failed += 1
    return failed


def _receive_lists(order_sources, order_experts, order_a):
    def lists(flats, owner, E, P):
        recv = [[] for _ in range(P)]
        for e in order_experts(range(E)):
            for i, f in order_sources(list(enumerate(flats))):
                for a in order_a(np.flatnonzero(f == e)):
                    recv[int(owner[e])].append((i, int(a)))
        return recv
    return lists


@pytest.mark.parametrize("name,mut", [
    ("sources reversed", _receive_lists(lambda s: s[::-1], lambda e: e, lambda a: a)),
    ("experts descending", _receive_lists(lambda s: s, lambda e: list(e)[::-1], lambda a: a)),
    ("local index descending", _receive_lists(lambda s: s, lambda e: e, lambda a: a[::-1])),
])
def test_ep_receive_order_mistakes_are_caught(monkeypatch, name, mut):
    assert _ep_pins_fail() == 0, "the unmodified oracle passes its EP pins"
    monkeypatch.setattr(O, "_ep_receive_lists", mut)
    assert _ep_pins_fail() >= 1, name


import tests.test_mx_oracle as mx_pins


def test_mx_exponent_off_by_one_is_caught(monkeypatch):
    orig = F8.mx_block_exponent
    monkeypatch.setattr(F8, "mx_block_exponent", lambda amax: np.clip(orig(amax) + 1, -127, 127))
    _fails(mx_pins.test_block_exponent_against_brute_force)
    _fails(mx_pins.test_hand_values)


def test_mx_scale_by_column_instead_of_block_is_caught(monkeypatch):
    # a scale looked up by k % (K/32) instead of k // 32
    def tiled(codes, sf):
        return F8.e4m3_decode(codes) * np.tile(F8.e8m0_decode(sf), (1, F8.MX_BLOCK))
    monkeypatch.setattr(F8, "dequantize_mx", tiled)
    _fails(mx_pins.test_gemm_brute_force_and_block_indexing)


def test_mx_ceil_exponent_is_caught(monkeypatch):
    # the other common reading, 2^ceil(log2(amax / 448)): no saturation, a different scale
    def ceil_exp(amax):
        amax = np.asarray(amax, dtype=np.float64)
        with np.errstate(divide="ignore"):
            e = np.where(amax > 0, np.ceil(np.log2(np.where(amax > 0, amax, 1.0) / 448.0)), -127)
        return np.clip(e, -127, 127).astype(np.int64)
    monkeypatch.setattr(F8, "mx_block_exponent", ceil_exp)
    _fails(mx_pins.test_hand_values)
