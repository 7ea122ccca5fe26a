// FP8 (e4m3) row quantisation: the payload format of the FP8 dispatch and the operand
// format of the FP8 expert GEMMs ("MoE我们喜欢你（四）": FP8 dispatch and FP8 grouped
// GEMMs; "Wide EP：当 MoE Expert Parallel 横跨几十张 GPU": FP8 weights and dispatch).
//
// One fp32 scale per row: s = amax(|row|) / 448 (s = 1 for an all-zero row), code =
// round-to-nearest-even(x / s) with saturation at +-448 (cvt.rn.satfinite).  The
// division is the IEEE fp32 one, so the codes are a function of the stored bf16 values.
// One warp per row, 16-byte loads (8 bf16) and 8-byte stores (8 codes); the row is read
// twice (max, then codes), the second time from L1/L2.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.cuh"
#include "mx.cuh"

namespace moe {

constexpr int kQuantWarps = 8;

__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_rows_kernel(const uint4* __restrict__ src, uint2* __restrict__ dst, float* __restrict__ scale,
                         long long rows, int vpr) {
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (r >= rows) return;  // whole warp leaves together
  const uint4* s = src + r * vpr;
  float amax = 0.f;
  for (int v = lane; v < vpr; v += 32) {
    const uint4 u = s[v];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (lane == 0) scale[r] = sc;
  uint2* d = dst + r * vpr;
  for (int v = lane; v < vpr; v += 32) {
    const uint4 u = s[v];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t packed[2];
#pragma unroll
    for (int q = 0; q < 4; q += 2) {
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]));
      const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[q + 1]));
      const __nv_fp8x2_storage_t lo =
          __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(f0.x, sc), __fdiv_rn(f0.y, sc)), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi =
          __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(f1.x, sc), __fdiv_rn(f1.y, sc)), __NV_SATFINITE, __NV_E4M3);
      packed[q / 2] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    d[v] = make_uint2(packed[0], packed[1]);
  }
}

cudaError_t launch_quantize_rows(const void* src, long long rows, int cols, void* dst, float* scale,
                                 cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const long long blocks = (rows + kQuantWarps - 1) / kQuantWarps;
  quantize_rows_kernel<<<(unsigned)blocks, kQuantWarps * 32, 0, st>>>(static_cast<const uint4*>(src),
                                                                      static_cast<uint2*>(dst), scale, rows, cols / 8);
  return cudaGetLastError();
}

// Block-scaled (MX) e4m3 quantisation of rows (the format and its rule: mx.cuh).
// One warp per row, one 32-value block per lane: four 16-byte loads (64 bytes, adjacent
// lanes adjacent), two 16-byte stores of codes and one scale byte per lane.
__global__ void __launch_bounds__(kQuantWarps * 32)
    quantize_mx_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, uint8_t* __restrict__ sf,
                       long long rows, int blocks_per_row) {
  const int lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  const uint4* s = src + r * blocks_per_row * 4;  // 4 x 16 bytes = 32 bf16 per block
  uint4* d = dst + r * blocks_per_row * 2;        // 2 x 16 bytes = 32 codes per block
  for (int blk = lane; blk < blocks_per_row; blk += 32) {
    uint4 u[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) u[q] = s[blk * 4 + q];
    float f[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w[4] = {u[q].x, u[q].y, u[q].z, u[q].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[h]));
        f[q * 8 + 2 * h] = t.x;
        f[q * 8 + 2 * h + 1] = t.y;
      }
    }
    uint32_t packed[8];
    const uint8_t sfb = mx_quantize32(f, packed);
    d[blk * 2] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    d[blk * 2 + 1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    sf[r * blocks_per_row + blk] = sfb;
  }
}

cudaError_t launch_quantize_mx(const void* src, long long rows, int cols, void* dst, uint8_t* sf, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const long long blocks = (rows + kQuantWarps - 1) / kQuantWarps;
  quantize_mx_kernel<<<(unsigned)blocks, kQuantWarps * 32, 0, st>>>(static_cast<const uint4*>(src),
                                                                    static_cast<uint4*>(dst), sf, rows, cols / 32);
  return cudaGetLastError();
}

}  // namespace moe
