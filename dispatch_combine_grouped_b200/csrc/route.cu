// Expert selection and gate weights from fp32 router logits.
//
// Follows the naive MoE forward of "深入浅出 DeepSeek MoE" (gate scores, then pick k
// experts), the ep_deepep explainer §2 (I_t and g_{t,e}), the Wide EP page's
// group-limited routing (keep g of G groups, then top-k inside them) and the grouped
// top-k / renormalise options named in "MoE我们喜欢你（四）" §4.2.
//
// One warp per token.  Lane l holds logits of experts l, l+32, ...; every comparison is
// on (value, index) with ties to the lower index, so the result does not depend on the
// order of the reduction.  The selection is made on exactly the fp32 logits in memory.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

struct TopkArgs {
  const float* logits;
  const float* gate_bias;  // correction bias: selection on logits, gates on logits - bias
  int32_t* ids;
  float* w;
  int N, E, k, n_groups, topk_groups, score, renorm;
};

// (va, ia) is ranked before (vb, ib): larger value first, then lower index.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

constexpr int kLanesE = kMaxE / 32;  // logits per lane

__global__ void __launch_bounds__(256) topk_kernel(TopkArgs p) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= p.N) return;  // whole warp leaves together
  const float* row = p.logits + (size_t)t * p.E;
  float v[kLanesE];
#pragma unroll
  for (int q = 0; q < kLanesE; ++q) {
    const int col = lane + 32 * q;
    v[q] = col < p.E ? row[col] : -INFINITY;
  }
  const int gsize = p.E / p.n_groups;
  int grp[kLanesE];  // group of each logit this lane holds (no division in the loops below)
#pragma unroll
  for (int q = 0; q < kLanesE; ++q) grp[q] = (lane + 32 * q) / gsize;

  // group-limited routing: keep topk_groups groups by their max logit
  uint32_t allowed = 0xffffffffu;
  if (p.n_groups > 1) {
    float gv[kMaxTopkGroups];
    int gi[kMaxTopkGroups];
#pragma unroll
    for (int q = 0; q < kMaxTopkGroups; ++q) {
      gv[q] = -INFINITY;
      gi[q] = 0x7fffffff;
    }
    for (int g = 0; g < p.n_groups; ++g) {
      float m = -INFINITY;
#pragma unroll
      for (int q = 0; q < kLanesE; ++q) {
        const int col = lane + 32 * q;
        if (col < p.E && grp[q] == g) m = fmaxf(m, v[q]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      // insert (m, g) into the kept list (uniform across the warp)
      float cv = m;
      int ci = g;
#pragma unroll
      for (int q = 0; q < kMaxTopkGroups; ++q) {
        if (q < p.topk_groups && ranks_before(cv, ci, gv[q], gi[q])) {
          float tv = gv[q];
          int ti = gi[q];
          gv[q] = cv;
          gi[q] = ci;
          cv = tv;
          ci = ti;
        }
      }
    }
    allowed = 0;
#pragma unroll
    for (int q = 0; q < kMaxTopkGroups; ++q)
      if (q < p.topk_groups) allowed |= 1u << gi[q];
  }

  // top-k: k rounds of a warp arg-max over the allowed, not yet taken logits
  uint32_t taken = 0;
  float sel_v[kMaxK];
  int sel_i[kMaxK];
#pragma unroll
  for (int s = 0; s < kMaxK; ++s) {
    sel_v[s] = -INFINITY;
    sel_i[s] = 0;
    if (s < p.k) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < kLanesE; ++q) {
        const int col = lane + 32 * q;
        const bool ok = col < p.E && !((taken >> q) & 1u) && ((allowed >> grp[q]) & 1u);
        if (ok && ranks_before(v[q], col, bv, bi)) {
          bv = v[q];
          bi = col;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ranks_before(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (bi == 0x7fffffff) bi = 0;  // only reachable with NaN logits
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      sel_v[s] = bv;
      sel_i[s] = bi;
    }
  }

  // gate inputs: the selection keys, or with a correction bias the unbiased logits
  if (p.gate_bias) {
#pragma unroll
    for (int q = 0; q < kLanesE; ++q) {
      const int col = lane + 32 * q;
      if (col < p.E) v[q] -= p.gate_bias[col];
    }
#pragma unroll
    for (int s = 0; s < kMaxK; ++s)
      if (s < p.k) sel_v[s] -= p.gate_bias[sel_i[s]];
  }

  // softmax denominator over all E (only needed without renormalisation)
  float gmax = -INFINITY, den_all = 0.f;
  if (p.score == MOE_SCORE_SOFTMAX && !p.renorm) {
#pragma unroll
    for (int q = 0; q < kLanesE; ++q) gmax = fmaxf(gmax, v[q]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
#pragma unroll
    for (int q = 0; q < kLanesE; ++q)
      if (lane + 32 * q < p.E) den_all += expf(v[q] - gmax);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den_all += __shfl_xor_sync(0xffffffffu, den_all, o);
  }
  float smax = -INFINITY;  // max of the chosen gate inputs (softmax renormalised)
#pragma unroll
  for (int s = 0; s < kMaxK; ++s)
    if (s < p.k) smax = fmaxf(smax, sel_v[s]);

  if (lane == 0) {
    float g[kMaxK];
    float sum = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxK; ++s) {
      g[s] = 0.f;
      if (s < p.k) {
        if (p.score == MOE_SCORE_SOFTMAX) {
          g[s] = p.renorm ? expf(sel_v[s] - smax) : expf(sel_v[s] - gmax) / den_all;
        } else {
          g[s] = 1.0f / (1.0f + expf(-sel_v[s]));
        }
        sum += g[s];
      }
    }
#pragma unroll
    for (int s = 0; s < kMaxK; ++s) {
      if (s < p.k) {
        p.ids[(size_t)t * p.k + s] = sel_i[s];
        p.w[(size_t)t * p.k + s] = p.renorm ? g[s] / sum : g[s];
      }
    }
  }
}

cudaError_t launch_topk(const moe_config& cfg, const float* logits, const float* gate_bias, int32_t* ids, float* w,
                        cudaStream_t st) {
  if (cfg.N == 0) return cudaSuccess;
  TopkArgs p;
  p.logits = logits;
  p.gate_bias = gate_bias;
  p.ids = ids;
  p.w = w;
  p.N = cfg.N;
  p.E = cfg.E;
  p.k = cfg.k;
  p.n_groups = cfg.n_groups;
  p.topk_groups = cfg.topk_groups;
  p.score = cfg.score;
  p.renorm = cfg.renormalize;
  const int warps = 8;
  topk_kernel<<<(cfg.N + warps - 1) / warps, warps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
