// Block-scaled (MX) e4m3 quantisation of one 32-value block, shared by the quantisation
// kernel and the FC1 epilogue that quantises h as it produces it ("MoE我们喜欢你（四）":
// MXFP8 expert compute; the microscaling format for FP8 elements).
//
// The block's scale is X = 2^e stored as the E8M0 byte e + 127, e = floor(log2 amax) - 8
// (8: the exponent of 256, the largest power of two in e4m3), clamped to [-127, 127]
// (-127 for an all-zero block); code = round-to-nearest-even of v * 2^-e, saturating at
// +-448.  The scaling by 2^-e is exact (it only moves the exponent) unless the product
// falls below 2^-126, where every candidate code is 0 anyway.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace moe {

__device__ __forceinline__ int mx_exponent(float amax) {
  const uint32_t b = __float_as_uint(amax);
  if (b == 0u) return -127;
  const int biased = (int)(b >> 23);
  const int fl = biased > 0 ? biased - 127 : (31 - __clz((int)(b & 0x7FFFFFu))) - 149;  // floor(log2 amax)
  const int e = fl - 8;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// f: the 32 values of one block (finite); packed: their codes, 4 per word in order
// (little-endian); returns the scale byte.
__device__ __forceinline__ uint8_t mx_quantize32(const float (&f)[32], uint32_t (&packed)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(f[i]));
  const int e = mx_exponent(amax);
  const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, a normal float for e <= 119
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(f[4 * i], inv), __fmul_rn(f[4 * i + 1], inv)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(f[4 * i + 2], inv), __fmul_rn(f[4 * i + 3], inv)), __NV_SATFINITE, __NV_E4M3);
    packed[i] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
  return (uint8_t)(e + 127);
}

}  // namespace moe
