"""Pins of the block-scaled (MX) e4m3 oracle against the format's definition, torch's own
E8M0 and e4m3 conversions, brute force, hand values and error bounds.

Source of the reading: the microscaling (MX) format for FP8 elements (32-value blocks,
one E8M0 power-of-two scale per block, shared exponent floor(log2 amax) minus the
element format's largest exponent); "MoE我们喜欢你（四）" names MXFP8 as low-precision expert
compute without fixing the format, see oracle/fp8.py.
"""
import math

import numpy as np
import torch

from oracle import fp8 as F


def test_e8m0_decode_matches_torch():
    b = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(b).view(torch.float8_e8m0fnu).double().numpy()
    got = F.e8m0_decode(b)
    assert np.array_equal(got[:255], ref[:255])
    assert np.isnan(got[255]) and np.isnan(ref[255])
    assert got[127] == 1.0 and got[0] == 2.0 ** -127 and got[254] == 2.0 ** 127


def _brute_exponent(amax):
    """The unique integer e with 2^(e+8) <= amax < 2^(e+9), found by walking powers of two
    (no logarithm), then clamped to [-127, 127]; -127 for 0."""
    if amax == 0:
        return -127
    p = -160
    while 2.0 ** (p + 1) <= amax:
        p += 1
    assert 2.0 ** p <= amax < 2.0 ** (p + 1)
    return max(-127, min(127, p - 8))


def test_block_exponent_against_brute_force():
    vals = [0.0, 1.0, 0.75, 3.0, 448.0, 512.0, 2.0 ** -133, 2.0 ** -126, 2.0 ** 127, 1e-30, 7.5e37]
    for p in range(-140, 128, 7):  # powers of two and their neighbours on both sides
        vals += [2.0 ** p, np.nextafter(np.float32(2.0 ** p), np.float32(0)).item(),
                 np.nextafter(np.float32(2.0 ** p), np.float32(np.inf)).item()]
    rng = np.random.default_rng(3)
    vals += list(np.abs(rng.standard_normal(200) * 10.0 ** rng.integers(-30, 30, 200)).astype(np.float32))
    vals = [float(np.float32(v)) for v in vals if np.isfinite(np.float32(v))]
    got = F.mx_block_exponent(np.array(vals))
    assert list(got) == [_brute_exponent(v) for v in vals]


def test_hand_values():
    x = np.zeros((5, 64), dtype=np.float32)
    x[0, 0], x[0, 1:32] = 1.0, 0.5      # amax 1   -> e = -8, scale byte 119, 1.0 -> 256 = 0x78
    x[1, 0] = 3.0                       # amax 3   -> e = -7, byte 120, 3.0 -> 384 = 0x7C
    x[2, 0], x[2, 1] = 1.9, -1.0        # 1.9 * 256 = 486.4 saturates to 448 = 0x7E; -1 -> -256 = 0xF8
    x[3, 32] = 448.0                    # second block only: e = 0, byte 127, code 448 = 0x7E
    x[4, :] = 0.0                       # all-zero blocks: byte 0, codes 0
    q, s = F.quantize_mx(x)
    assert s.shape == (5, 2) and q.shape == (5, 64)
    assert list(s[:, 0]) == [119, 120, 119, 0, 0] and list(s[:, 1]) == [0, 0, 0, 127, 0]
    assert q[0, 0] == 0x78 and q[0, 1] == 0x70    # 0.5 * 256 = 128 = 2^7 -> exponent 14
    assert q[1, 0] == 0x7C and q[2, 0] == 0x7E and q[2, 1] == 0xF8 and q[3, 32] == 0x7E
    assert not q[4].any() and not q[3, :32].any()


def test_codes_match_torch_conversion():
    """Codes are torch's float -> float8_e4m3fn conversion (round to nearest even) of the
    exactly scaled values, after clamping to the finite range; scales from the brute-force
    exponent."""
    rng = np.random.default_rng(4)
    R, C = 40, 256
    x = (rng.standard_normal((R, C)) * 10.0 ** rng.integers(-8, 8, (R, 1))).astype(np.float32)
    x[3, 32:64] = 0.0
    x[5, :32] = rng.choice([-448.0, 448.0, 1e-40, -2.0 ** -133], size=32).astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()  # bf16-representable, as the path stores
    q, s = F.quantize_mx(x)
    blocks = x.reshape(R, C // 32, 32).astype(np.float64)
    e = np.array([[_brute_exponent(float(np.abs(b).max())) for b in row] for row in blocks])
    assert np.array_equal(s.astype(np.int64), e + 127)
    scaled = np.clip(blocks * np.ldexp(1.0, -e)[:, :, None], -448, 448).reshape(R, C)
    ref = torch.from_numpy(scaled.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_quantisation_error_bound():
    """|dequant - x| <= max(|x| 2^-4, X 2^-10) for every element whose scaled value is at
    most 448 (RNE with 3 mantissa bits, or the subnormal half step); a larger one saturates
    to +-448 X.  The scaled block maximum lies in [256, 512)."""
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 512)) * 10.0 ** rng.integers(-5, 5, (64, 1))).astype(np.float32)
    q, s = F.quantize_mx(x)
    X = np.repeat(F.e8m0_decode(s), 32, axis=1)
    v = F.dequantize_mx(q, s)
    scaled = np.abs(x) / X
    amax_scaled = (np.abs(x).reshape(64, 16, 32).max(axis=2) / F.e8m0_decode(s))
    assert np.all((amax_scaled >= 256) & (amax_scaled < 512))
    ok = scaled <= 448
    assert np.all(np.abs(v - x)[ok] <= np.maximum(np.abs(x) * 2.0 ** -4, X * 2.0 ** -10)[ok])
    assert np.array_equal(v[~ok], np.sign(x[~ok]) * 448 * X[~ok])


def test_exactly_representable_blocks_round_trip():
    """A block of e4m3 values times 2^e whose largest magnitude lies in [256, 448] * 2^e
    quantises to exactly those codes and that scale."""
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 0x7F, size=(30, 128)).astype(np.uint8) | (rng.integers(0, 2, (30, 128)) << 7).astype(np.uint8)
    codes[:, ::32] = 0x78 | (codes[:, ::32] & 0x80)  # every block holds +-256
    e = rng.integers(-100, 100, size=(30, 4))
    x = F.e4m3_decode(codes) * np.repeat(np.ldexp(1.0, e), 32, axis=1)
    q, s = F.quantize_mx(x.astype(np.float32))
    assert np.array_equal(s.astype(np.int64), e + 127)
    neg_zero = (codes == 0x80)  # -0 keeps its sign bit
    assert np.array_equal(q[~neg_zero], codes[~neg_zero]) and np.all(q[neg_zero] == 0x80)


def test_gemm_unit_scales_is_the_plain_e4m3_product():
    rng = np.random.default_rng(7)
    qa = rng.integers(0, 0x7F, size=(5, 96)).astype(np.uint8)
    qb = rng.integers(0, 0x7F, size=(4, 96)).astype(np.uint8)
    ones_a, ones_b = np.full((5, 3), 127, np.uint8), np.full((4, 3), 127, np.uint8)
    np.testing.assert_array_equal(F.gemm_mx(qa, ones_a, qb, ones_b), F.gemm_rows(qa, np.ones(5), qb, np.ones(4)))


def test_gemm_brute_force_and_block_indexing():
    """A triple loop over (i, j, k) with each scale looked up by k // 32; raising one block's
    scale byte by one adds exactly that block's partial dot product (a scale indexed by
    k % 32, or a transposed scale table, fails this)."""
    rng = np.random.default_rng(8)
    M, N, K = 3, 4, 96
    qa = rng.integers(0, 0x7F, size=(M, K)).astype(np.uint8) | (rng.integers(0, 2, (M, K)) << 7).astype(np.uint8)
    qb = rng.integers(0, 0x7F, size=(N, K)).astype(np.uint8)
    sa = rng.integers(110, 140, size=(M, 3)).astype(np.uint8)
    sb = rng.integers(110, 140, size=(N, 3)).astype(np.uint8)
    d = F.gemm_mx(qa, sa, qb, sb)
    va, vb = F.e4m3_decode(qa), F.e4m3_decode(qb)
    for i in range(M):
        for j in range(N):
            acc = math.fsum(va[i, k] * 2.0 ** (int(sa[i, k // 32]) - 127) * vb[j, k] * 2.0 ** (int(sb[j, k // 32]) - 127)
                            for k in range(K))
            assert abs(d[i, j] - acc) <= 1e-12 * max(1.0, abs(acc))
    sa2 = sa.copy()
    sa2[1, 2] += 1
    d2 = F.gemm_mx(qa, sa2, qb, sb)
    part = (va[1, 64:96] * 2.0 ** (int(sa[1, 2]) - 127)) @ (vb[:, 64:96] * np.repeat(
        2.0 ** (sb[:, 2:3].astype(np.int64) - 127), 32, axis=1)).T
    np.testing.assert_allclose(d2[1] - d[1], part, rtol=1e-12, atol=1e-300)
    np.testing.assert_array_equal(np.delete(d2, 1, axis=0), np.delete(d, 1, axis=0))


def test_fc1_fc2_mx_definition():
    """The expert FFN on MX operands is SwiGLU over the dequantised operands."""
    rng = np.random.default_rng(9)
    R, d, I = 6, 64, 32
    x = rng.standard_normal((R, d)).astype(np.float32)
    w13 = (rng.standard_normal((2 * I, d)) / 8).astype(np.float32)
    w2 = (rng.standard_normal((d, I)) / 8).astype(np.float32)
    qx, sx = F.quantize_mx(x)
    qw, sw = F.quantize_mx(w13)
    xv, wv = F.dequantize_mx(qx, sx), F.dequantize_mx(qw, sw)
    h = F.fc1_mx(qx, sx, qw, sw, I)
    np.testing.assert_allclose(h, F.silu(xv @ wv[:I].T) * (xv @ wv[I:].T), rtol=1e-14)
    qh, sh = F.quantize_mx(h.astype(np.float32))
    q2, s2 = F.quantize_mx(w2)
    np.testing.assert_allclose(F.fc2_mx(qh, sh, q2, s2), F.dequantize_mx(qh, sh) @ F.dequantize_mx(q2, s2).T,
                               rtol=1e-14)
    # MX keeps every block's own range: rows of very different magnitude within one row
    # of K lose no more than the e4m3 rounding (a per-row scale would flush the small block)
    y = np.concatenate([np.full(32, 1e-4), np.full(32, 1e4)]).astype(np.float32)[None]
    qy, sy = F.quantize_mx(y)
    np.testing.assert_allclose(F.dequantize_mx(qy, sy), y, rtol=2.0 ** -4)
