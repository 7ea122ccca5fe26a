"""CPU oracle for the FP8 (e4m3) variant of the expert path: row quantisation, the FP8
dispatch payload and the two grouped GEMMs with their scales.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  It shares no
code with the CUDA library and imports nothing from it.

Sources: "MoE我们喜欢你（四）：DeepEP 与 GroupedGEMM 如何拆解通信和计算瓶颈" (FP8 dispatch
payloads and FP8 grouped GEMMs as the lever on both walls), "Wide EP：当 MoE Expert
Parallel 横跨几十张 GPU" (FP8 weights and dispatch in the deployment tables); the ep_deepep
explainer §7 (low-precision dispatch, combine kept in higher precision).  The pages name
FP8 but fix neither the format nor the scaling; readings taken (listed in the design
notes):
  * format: e4m3 with no infinities (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits; largest finite 448; the all-ones pattern is NaN; subnormals down to 2^-9);
  * scaling: one fp32 scale per row of every operand (a token row of x, a row of h, an
    output row of W13 and of W2): s = amax(|row|) / 448 computed in fp32 (s = 1 for an
    all-zero row); code = round-to-nearest-even of the fp32 quotient x / s, clamped to
    +-448;
  * GEMMs: D = (sum_k qa_k qb_k) * s_row * s_col; the combine is unchanged (fp32
    accumulation, bf16 output); h is rounded to bf16 before its own quantisation, as the
    CUDA path stores it.

The block-scaled (MX) form.  "MoE我们喜欢你（四）" names MXFP8 beside FP8 as the low-precision
expert compute; the pages do not define the format, so the reading is the published
microscaling (MX) format for FP8 elements:
  * a block is 32 consecutive values along the reduction dimension (K) of one row;
  * its shared scale is a power of two X = 2^e stored as one unbiased-exponent byte
    (E8M0: byte b means 2^(b-127); 255 is NaN and never written);
  * e = floor(log2(max |v| of the block)) - 8, where 8 is the exponent of the largest power
    of two e4m3 holds (256), clamped to [-127, 127]; an all-zero block takes e = -127;
  * each element's code is the e4m3 round-to-nearest-even of v / X, saturating at +-448
    (so the largest element, whose v / X lies in [256, 512), may clip to 448);
  * a GEMM on MX operands is D = sum_k (qa_k * Xa(k // 32)) * (qb_k * Xb(k // 32)).
v / X is exact (a power-of-two scaling), so the codes are a function of the stored values.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(code) -> np.ndarray:
    """Value of every e4m3 code (uint8 array) as float64; the NaN pattern gives NaN."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def _finite_table():
    codes = np.arange(0x7F, dtype=np.int64)  # positive, 0x7F is NaN
    return codes, e4m3_decode(codes)


def e4m3_encode(v) -> np.ndarray:
    """Nearest e4m3 code (ties to the even code), saturating at +-448, for float values."""
    v = np.asarray(v, dtype=np.float64)
    codes, vals = _finite_table()  # ascending values 0 .. 448
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(vals, a, side="left")  # vals[hi-1] < a <= vals[hi]
    hi = np.clip(hi, 0, len(vals) - 1)
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    d_lo, d_hi = a - vals[lo], vals[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0))
    mag = np.where(pick_hi, codes[hi], codes[lo])
    mag = np.where(a == vals[hi], codes[hi], mag)
    return (mag | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def quantize_rows(x):
    """Per-row e4m3 quantisation (the reading above).  x: values exactly representable in
    fp32 (bf16 or fp32 storage).  Returns (codes uint8 [R, C], scales float32 [R])."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=1) if x32.shape[1] else np.zeros(x32.shape[0], np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = (x32 / scale[:, None]).astype(np.float32)  # fp32 division, as on the GPU
    return e4m3_encode(q), scale


def dequantize_rows(codes, scale) -> np.ndarray:
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, None]


def gemm_rows(qa, sa, qb, sb) -> np.ndarray:
    """D[i, j] = (sum_k a_ik b_jk) sa_i sb_j with a, b the decoded codes (float64)."""
    return (e4m3_decode(qa) @ e4m3_decode(qb).T) * np.asarray(sa, np.float64)[:, None] * \
        np.asarray(sb, np.float64)[None, :]


def silu(z):
    return z / (1.0 + np.exp(-z))


def fc1(qx_rows, sx_rows, qw13, sw13, I: int) -> np.ndarray:
    """SwiGLU activations of one expert's rows from FP8 operands (float64)."""
    z = gemm_rows(qx_rows, sx_rows, qw13, sw13)
    return silu(z[:, :I]) * z[:, I:]


def fc2(qh_rows, sh_rows, qw2, sw2) -> np.ndarray:
    return gemm_rows(qh_rows, sh_rows, qw2, sw2)


# ---------------------------------------------------------------------------------------
# Block-scaled (MX) e4m3: 32-value blocks along K, one E8M0 power-of-two scale per block.
# ---------------------------------------------------------------------------------------
MX_BLOCK = 32
E4M3_EMAX = 8  # 2^8 = 256 is the largest power of two e4m3 represents


def e8m0_decode(b) -> np.ndarray:
    """Scale of every E8M0 byte: 2^(b - 127); 255 is NaN."""
    b = np.asarray(b, dtype=np.int64)
    return np.where(b == 255, np.nan, np.ldexp(1.0, (b - 127).clip(-127, 127)))


def mx_block_exponent(amax) -> np.ndarray:
    """e of a block with largest magnitude amax (float64 array): floor(log2 amax) - 8,
    clamped to [-127, 127]; -127 for amax == 0.  np.frexp writes amax = m 2^f with m in
    [0.5, 1), so floor(log2 amax) = f - 1 exactly (subnormal amax included)."""
    amax = np.asarray(amax, dtype=np.float64)
    _, f = np.frexp(amax)
    e = np.where(amax > 0, f.astype(np.int64) - 1 - E4M3_EMAX, -127)
    return np.clip(e, -127, 127)


def quantize_mx(x):
    """MX quantisation of rows (the reading above).  x: [R, C] values exactly representable
    in fp32 (bf16 or fp32 storage), C % 32 == 0.  Returns (codes uint8 [R, C], scale bytes
    uint8 [R, C // 32])."""
    x64 = np.asarray(x, dtype=np.float32).astype(np.float64)
    R, C = x64.shape
    assert C % MX_BLOCK == 0
    blocks = x64.reshape(R, C // MX_BLOCK, MX_BLOCK)
    e = mx_block_exponent(np.abs(blocks).max(axis=2) if C else np.zeros((R, 0)))
    q = e4m3_encode(blocks * np.ldexp(1.0, -e)[:, :, None])  # exact scaling in float64
    return q.reshape(R, C), (e + 127).astype(np.uint8)


def dequantize_mx(codes, sf) -> np.ndarray:
    """Values of MX rows: code value times its block's scale (float64)."""
    scale = np.repeat(e8m0_decode(sf), MX_BLOCK, axis=1)
    return e4m3_decode(codes) * scale


def gemm_mx(qa, sa, qb, sb) -> np.ndarray:
    """D[i, j] = sum_k (qa_ik Xa_i,k//32) (qb_jk Xb_j,k//32) in float64 (the products are
    exact; only the sum rounds)."""
    return dequantize_mx(qa, sa) @ dequantize_mx(qb, sb).T


def fc1_mx(qx_rows, sx_rows, qw13, sw13, I: int) -> np.ndarray:
    """SwiGLU activations of one expert's rows from MX operands (float64)."""
    z = gemm_mx(qx_rows, sx_rows, qw13, sw13)
    return silu(z[:, :I]) * z[:, I:]


def fc2_mx(qh_rows, sh_rows, qw2, sw2) -> np.ndarray:
    return gemm_mx(qh_rows, sh_rows, qw2, sw2)
