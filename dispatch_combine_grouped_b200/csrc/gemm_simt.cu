// fp32 grouped GEMM on the CUDA cores, for the fp32 configurations (the tensor-core path
// is bf16).  Same three jobs and the same group / tile scheme as the tcgen05 kernel:
// router logits (+ bias), FC1 with SwiGLU, FC2 with the gate scale.  64 x 64 output tile
// per CTA, 32-deep k slices staged in shared memory (the next slice's loads issued into
// registers before the current one is multiplied, so that their latency overlaps the
// FMAs), 4 x 4 outputs per thread, fp32 FMA in ascending k order.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int SBM = 64, SBN = 64, SBK = 32;
constexpr int kSimtThreads = 256;
constexpr int kSimtGroups = kMaxSlots + kMaxShared;

template <int MODE>
__global__ void __launch_bounds__(kSimtThreads) simt_gemm_kernel(const GemmArgs p) {
  __shared__ float As[SBK][SBM + 4];
  __shared__ float Bg[SBK][SBN + 4];
  __shared__ float Bu[SBK][SBN + 4];
  __shared__ int s_prefix[kSimtGroups + 1], s_arow[kSimtGroups], s_orow[kSimtGroups], s_rows[kSimtGroups];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.G;
  for (int g = tid; g < G; g += kSimtThreads) {
    int rows, arow, orow;
    const int gg = p.g0 + g;  // global group
    if (gg < p.E) {
      rows = p.n_e[gg];
      arow = orow = p.expert_off[gg];
      // bounds-checked build: a group must lie inside the routed rows
      if (kChecks && (rows < 0 || arow < 0 || (long long)arow + rows > p.A_routed)) {
        report(p.check, MOE_ERR_BAD_INDEX);
        rows = 0;
        arow = orow = 0;
      }
    } else {
      const int s = gg - p.E;
      rows = p.N;
      orow = p.A_routed + s * p.N;
      arow = p.shared_from_map1 ? 0 : orow;
    }
    s_rows[g] = rows;
    s_arow[g] = arow;
    s_orow[g] = orow;
  }
  __syncthreads();
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      const int v = g < G ? (s_rows[g] + SBM - 1) / SBM : 0;
      int incl = v;
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (g < G) s_prefix[g] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_prefix[G] = run;
  }
  __syncthreads();

  const int n_tiles = (p.n_out + SBN - 1) / SBN;
  const int total = s_prefix[G] * n_tiles;
  const int ty = tid / 16, tx = tid % 16;
  const float* Aall = static_cast<const float*>(p.a0);
  const float* A1 = static_cast<const float*>(p.a1);
  const float* Ball = static_cast<const float*>(p.b);

  for (int t = blockIdx.x; t < total; t += gridDim.x) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] * n_tiles <= t) lo = mid;
      else hi = mid - 1;
    }
    const int g = lo;
    const int mt = s_prefix[g + 1] - s_prefix[g];
    const int local = t - s_prefix[g] * n_tiles;
    const int n_blk = local / mt, m_blk = local - n_blk * mt;
    const int rows = s_rows[g];
    const int gz = p.g0 + g;  // global group = weight index
    const float* Abase = (gz >= p.E && p.shared_from_map1) ? A1 : Aall;
    const long long arow0 = (long long)s_arow[g] + (long long)m_blk * SBM;
    const float* W = Ball + (long long)gz * p.b_rows * p.K;
    const int n0 = n_blk * SBN;

    float accg[4][4] = {}, accu[4][4] = {};
    // this thread's share of a slice: rows / columns tid / 4, k offsets (tid % 4) * 4 and +16
    const int lr = tid / 4, kq = (tid % 4) * 4;
    float4 ra[2], rg[2], ru[2];
    auto load = [&](int k0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int kk = k0 + kq + 16 * h;
        ra[h] = rg[h] = ru[h] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (m_blk * SBM + lr < rows && kk < p.K) ra[h] = *reinterpret_cast<const float4*>(Abase + (arow0 + lr) * p.K + kk);
        if (n0 + lr < p.n_out && kk < p.K) {
          rg[h] = *reinterpret_cast<const float4*>(W + (long long)(n0 + lr) * p.K + kk);
          if (MODE == MODE_FC1) ru[h] = *reinterpret_cast<const float4*>(W + (long long)(p.I + n0 + lr) * p.K + kk);
        }
      }
    };
    load(0);
    for (int k0 = 0; k0 < p.K; k0 += SBK) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // registers -> shared memory, k-major
        const int kk = kq + 16 * h;
        As[kk + 0][lr] = ra[h].x;
        As[kk + 1][lr] = ra[h].y;
        As[kk + 2][lr] = ra[h].z;
        As[kk + 3][lr] = ra[h].w;
        Bg[kk + 0][lr] = rg[h].x;
        Bg[kk + 1][lr] = rg[h].y;
        Bg[kk + 2][lr] = rg[h].z;
        Bg[kk + 3][lr] = rg[h].w;
        if (MODE == MODE_FC1) {
          Bu[kk + 0][lr] = ru[h].x;
          Bu[kk + 1][lr] = ru[h].y;
          Bu[kk + 2][lr] = ru[h].z;
          Bu[kk + 3][lr] = ru[h].w;
        }
      }
      __syncthreads();
      if (k0 + SBK < p.K) load(k0 + SBK);  // the next slice, in flight during the FMAs below
#pragma unroll
      for (int kk = 0; kk < SBK; ++kk) {
        float a[4], bg[4], bu[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bg[j] = Bg[kk][tx * 4 + j];
          if (MODE == MODE_FC1) bu[j] = Bu[kk][tx * 4 + j];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            accg[i][j] = fmaf(a[i], bg[j], accg[i][j]);
            if (MODE == MODE_FC1) accu[i][j] = fmaf(a[i], bu[j], accu[i][j]);
          }
      }
      __syncthreads();
    }
    // epilogue
    float* out = static_cast<float*>(p.out);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = m_blk * SBM + ty * 4 + i;
      if (r >= rows) continue;
      const long long orow = (long long)s_orow[g] + r;
      float scale = 1.0f;
      if (MODE == MODE_FC2 && p.gate_w && gz < p.E) {
          const int gi = p.row2tok ? p.row2tok[orow] : (int)orow;
          scale = check_range(gi, 0, p.A_routed, p.check) ? p.gate_w[gi] : 0.0f;
        }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = n0 + tx * 4 + j;
        if (col >= p.n_out) continue;
        float v;
        if (MODE == MODE_FC1) v = silu_f32(accg[i][j]) * accu[i][j];
        else if (MODE == MODE_FC2) v = accg[i][j] * scale;
        else v = accg[i][j] + (p.bias ? p.bias[col] : 0.f);
        out[orow * p.ldo + col] = v;
      }
    }
  }
}

cudaError_t launch_simt_gemm(const GemmArgs& g, cudaStream_t st) {
  const long long rows_total = launch_rows(g);
  const long long blocks = (rows_total + SBM - 1) / SBM + g.G;
  const long long tiles = blocks * ((g.n_out + SBN - 1) / SBN);
  long long grid = 4LL * sm_count();
  if (tiles < grid) grid = tiles;
  if (grid < 1) grid = 1;
  switch (g.mode) {
    case MODE_FC1: simt_gemm_kernel<MODE_FC1><<<(unsigned)grid, kSimtThreads, 0, st>>>(g); break;
    case MODE_FC2: simt_gemm_kernel<MODE_FC2><<<(unsigned)grid, kSimtThreads, 0, st>>>(g); break;
    default: simt_gemm_kernel<MODE_ROUTER><<<(unsigned)grid, kSimtThreads, 0, st>>>(g); break;
  }
  return cudaGetLastError();
}

}  // namespace moe
