"""Pins of the FP8 (e4m3) oracle against the format's definition, a library conversion,
hand-checked values and error bounds.

Source of the format reading: the e4m3 "no infinities" format (1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits, largest finite 448); the pages name FP8 dispatch and
FP8 grouped GEMMs ("MoE我们喜欢你（四）"; "Wide EP：当 MoE Expert Parallel 横跨几十张 GPU")
without fixing a format, see oracle/fp8.py.
"""
import numpy as np
import torch

from oracle import fp8 as F


def test_decode_known_values():
    assert F.e4m3_decode(0x7E) == 448.0          # largest finite
    assert F.e4m3_decode(0x38) == 1.0            # exponent 7 = bias
    assert F.e4m3_decode(0x08) == 2.0 ** -6      # smallest normal
    assert F.e4m3_decode(0x01) == 2.0 ** -9      # smallest subnormal
    assert F.e4m3_decode(0x07) == 7 / 8 * 2.0 ** -6
    assert F.e4m3_decode(0xB8) == -1.0
    assert np.isnan(F.e4m3_decode(0x7F)) and np.isnan(F.e4m3_decode(0xFF))
    vals = F.e4m3_decode(np.arange(0x7F))
    assert np.all(np.diff(vals) > 0)             # codes are ordered by value


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(F.e4m3_encode(F.e4m3_decode(codes)), codes)


def test_ties_go_to_the_even_code_and_large_values_saturate():
    assert F.e4m3_encode(1.0625) == 0x38         # halfway 1.0 / 1.125 -> even mantissa
    assert F.e4m3_encode(1.1875) == 0x3A         # halfway 1.125 / 1.25 -> even mantissa
    assert F.e4m3_encode(2.0 ** -10) == 0x00     # halfway 0 / 2^-9 -> 0
    assert F.e4m3_encode(3 * 2.0 ** -10) == 0x02  # halfway 2^-9 / 2^-8 -> even
    assert F.e4m3_encode(1e6) == 0x7E and F.e4m3_encode(-1e6) == 0xFE
    assert F.e4m3_encode(-0.0) == 0x80


def test_matches_torch_float8_conversion():
    """torch's float -> float8_e4m3fn conversion (round to nearest even) on values already
    clamped to the finite range."""
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.normal(size=20000) * 100, rng.normal(size=5000) * 1e-2,
                        F.e4m3_decode(np.arange(0x7F)) * 1.0001, F.e4m3_decode(np.arange(0x7E)) * 0.9999])
    v = np.clip(v, -448, 448).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_encode(v), ref)


def test_row_quantisation():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(50, 300)).astype(np.float32)
    x[7] = 0.0
    q, s = F.quantize_rows(x)
    assert s.dtype == np.float32 and s[7] == 1.0 and not q[7].any()
    amax_pos = np.argmax(np.abs(x), axis=1)
    for r in range(50):
        if r != 7:
            assert q[r, amax_pos[r]] & 0x7F == 0x7E  # the largest element maps to +-448
    # error bound: e4m3 keeps 3 mantissa bits, so |x - dq| <= 2^-4 |x| above the
    # subnormal range, and <= half the subnormal step (2^-10 s) below it
    dq = F.dequantize_rows(q, s)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s[:, None])
    assert np.all(np.abs(dq - x) <= bound * (1 + 1e-6))


def test_gemm_is_the_product_of_the_dequantised_operands():
    rng = np.random.default_rng(2)
    a, b = rng.normal(size=(9, 64)), rng.normal(size=(7, 64))
    qa, sa = F.quantize_rows(a)
    qb, sb = F.quantize_rows(b)
    d = F.gemm_rows(qa, sa, qb, sb)
    brute = np.array([[sum(F.e4m3_decode(qa[i, k]) * sa[i] * F.e4m3_decode(qb[j, k]) * sb[j] for k in range(64))
                       for j in range(7)] for i in range(9)])
    np.testing.assert_allclose(d, brute, rtol=1e-12, atol=1e-12)
    # and close to the unquantised product (relative error of e4m3 operands)
    assert np.linalg.norm(d - a @ b.T) / np.linalg.norm(a @ b.T) < 0.05


def test_fp8_ffn_equals_the_bf16_oracle_when_quantisation_is_exact():
    """The FP8 expert FFN (fc1 then fc2) reduces to the float64 SwiGLU expert of the main
    oracle when every operand is an e4m3 value under a scale of 1: then the codes carry the
    values exactly and only the operand path differs (codes + scales vs plain floats)."""
    from oracle import moe_oracle as O
    rng = np.random.default_rng(0)
    finite = F.e4m3_decode(np.arange(0x00, 0x7F))        # every finite non-negative e4m3 value
    small = finite[(finite > 0) & (finite <= 2.0)]
    R, d, I = 5, 32, 16

    def pick(shape):
        v = rng.choice(small, size=shape) * rng.choice([-1.0, 1.0], size=shape)
        return v, F.e4m3_encode(v)

    x, qx = pick((R, d))
    w13, qw13 = pick((2 * I, d))
    w2, qw2 = pick((d, I))
    h = F.fc1(qx, np.ones(R), qw13, np.ones(2 * I), I)
    assert np.allclose(h, O.silu(x @ w13[:I].T) * (x @ w13[I:].T), rtol=1e-15, atol=0)
    # FC2 on an h that is itself exactly representable, then the whole expert
    hv, qh = pick((R, I))
    np.testing.assert_allclose(F.fc2(qh, np.ones(R), qw2, np.ones(d)), hv @ w2.T, rtol=1e-15, atol=0)
    y_ref = O.swiglu_expert(x, w13, w2)
    np.testing.assert_allclose(h @ w2.T, y_ref, rtol=1e-12, atol=1e-12)


def test_fp8_gemm_scale_properties():
    """Properties of a scaled product that a transposed, dropped or misplaced scale breaks:
    swapping the operands transposes the result, and doubling one row's scale doubles
    exactly that row."""
    rng = np.random.default_rng(1)
    qa = rng.integers(0, 0x7F, size=(4, 8)).astype(np.uint8)
    qb = rng.integers(0, 0x7F, size=(3, 8)).astype(np.uint8)
    sa, sb = rng.uniform(0.5, 2.0, 4), rng.uniform(0.5, 2.0, 3)
    d = F.gemm_rows(qa, sa, qb, sb)
    np.testing.assert_allclose(F.gemm_rows(qb, sb, qa, sa), d.T, rtol=1e-15)
    sa2 = sa.copy()
    sa2[2] *= 2
    d2 = F.gemm_rows(qa, sa2, qb, sb)
    np.testing.assert_allclose(d2[2], 2 * d[2], rtol=1e-15)
    np.testing.assert_array_equal(np.delete(d2, 2, axis=0), np.delete(d, 2, axis=0))
