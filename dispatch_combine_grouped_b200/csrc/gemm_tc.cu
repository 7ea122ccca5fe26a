// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM, fed by TMA), bf16 or
// e4m3 (F8) operands with fp32 accumulation, one kernel family for three jobs:
//   MODE_ROUTER  logits = x W_g^T (+ b), fp32 out                ("深入浅出 DeepSeek MoE", step 1)
//   MODE_FC1     h = SiLU(X W_gate^T) * (X W_up^T), bf16 out     ("MoE我们喜欢你（四）" §4.1 FC1 + activation)
//   MODE_FC2     o = (h W_down^T) * gate(row), bf16 out          (§4.1 FC2; the combine's gate applied here)
// over "groups" of rows with variable sizes n_e that are only known on the device
// (ep_deepep explainer §2: work per expert is n_e, critical work max_e n_e).
//
// Structure (one CTA per SM, persistent, 6 warps):
//   warp 0      TMA producer: A tile [128 x 128 B] + B tile [BN x 128 B] per stage (64
//               bf16 or 128 e4m3 k values per row), 128B swizzle
//   warp 1      MMA issuer: 4 x tcgen05.mma (M=128, N=BN, K=16 bf16 / 32 e4m3) per stage;
//               owns the TMEM allocation (2 x BN fp32 columns: double-buffered accumulator)
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes, SwiGLU / gate scale / bias,
//               vectorised stores; overlaps the next tile's mainloop
// The tile schedule is computed in the kernel from n_e: each CTA builds the prefix of
// row blocks per group in shared memory and walks tiles blockIdx.x, +gridDim.x, ...
// ordered group-major, then by output-column tile, then by row block, so that the row
// blocks sharing one weight tile run at the same time and the weight streams from HBM
// about once.
//
// FC1 needs gate and up columns of the same output in one accumulator: the B tile is
// loaded as two boxes, W_gate rows [n0, n0+BN/2) and W_up rows [I+n0, I+n0+BN/2), so no
// repacking of the weights is needed.  Rows past a group's end are computed from the
// following rows (or TMA zero fill) and never stored.  Every wait is bounded.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int BM = 128;
// k per stage: 64 bf16 (128-byte rows with the 128B swizzle); narrower k-steps (64- and
// 32-byte swizzles) measured 20% and 50% slower on B200
constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr int kMaxGroupsGemm = kMaxSlots + kMaxShared;

struct SmemPlan {
  int a_bytes, b_bytes, stages, total;
};

// barriers: full/empty per stage, 2 tfull, 2 tempty, drain, then TMEM holder + abort flag
template <int STAGES>
__host__ __device__ constexpr int barrier_bytes() {
  return ((2 * STAGES + 5) * 8 + 8 + 15) & ~15;
}

template <int BN, int STAGES, int BKT, int ES>
__host__ __device__ constexpr int smem_bytes_for() {
  // 1 KB alignment slack + stages + barriers/flags + group tables
  return 1024 + STAGES * (BM * BKT * ES + BN * BKT * ES) + barrier_bytes<STAGES>() + 4 * (4 * kMaxGroupsGemm + 8);
}

struct TileDesc {
  int g, m_blk, n_blk;
};

__device__ __forceinline__ TileDesc decode_tile(int t, const int* prefix, int G, int n_tiles) {
  // largest g with prefix[g] * n_tiles <= t
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] * n_tiles <= t) lo = mid;
    else hi = mid - 1;
  }
  const int mt = prefix[lo + 1] - prefix[lo];
  const int local = t - prefix[lo] * n_tiles;
  TileDesc d;
  d.g = lo;
  d.n_blk = local / mt;
  d.m_blk = local - d.n_blk * mt;
  return d;
}

// F8: e4m3 operands (BKT = 128 k per stage, the same 128-byte rows), kind::f8f6f4 MMAs and
// the row x column scales applied to the accumulator in the epilogue.
template <int BN, int MODE, int STAGES, int BKT, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  constexpr int ES = F8 ? 1 : 2;        // bytes per element
  constexpr int ROWB = BKT * ES;        // bytes of one row of a stage
  constexpr int A_BYTES = BM * ROWB;
  constexpr int B_BYTES = BN * ROWB;
  constexpr int HALF_B = B_BYTES / 2;
  constexpr uint32_t TMEM_COLS = 2 * BN;  // BN is a power of two >= 32
  constexpr uint32_t IDESC = F8 ? idesc_e4m3_f32(BM, BN) : idesc_bf16_f32(BM, BN);
  constexpr uint32_t TX_BYTES = A_BYTES + B_BYTES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);
  int* s_prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + barrier_bytes<STAGES>());
  int* s_arow = s_prefix + (kMaxGroupsGemm + 1);
  int* s_orow = s_arow + kMaxGroupsGemm;
  int* s_rows = s_orow + kMaxGroupsGemm;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_holder, TMEM_COLS);

  // group table: rows, first A row, first output row
  for (int g = threadIdx.x; g < G; g += kThreads) {
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
  if (warp == 0) {  // exclusive prefix of row blocks per group
    int run = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      const int v = g < G ? (s_rows[g] + BM - 1) / BM : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (g < G) s_prefix[g] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_prefix[G] = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = *tmem_holder;
  const int n_tiles = (MODE == MODE_FC1) ? (p.n_out + BN / 2 - 1) / (BN / 2) : (p.n_out + BN - 1) / BN;
  const int total = s_prefix[G] * n_tiles;
  const int num_kb = (p.K + BKT - 1) / BKT;
  volatile int* abort_v = abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileDesc td = decode_tile(t, s_prefix, G, n_tiles);
        const int gz = p.g0 + td.g;  // global group = weight index
        const CUtensorMap* mapA = (gz >= p.E && p.shared_from_map1) ? &tmA1 : &tmA0;
        const int a_row = s_arow[td.g] + td.m_blk * BM;
        int b_row0, b_row1;
        if (MODE == MODE_FC1) {
          b_row0 = td.n_blk * (BN / 2);
          b_row1 = p.I + b_row0;
        } else {
          b_row0 = td.n_blk * BN;
          b_row1 = b_row0 + BN / 2;
        }
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], ph ^ 1u, abort_v)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], TX_BYTES);
          tma_load_2d(sA + stage * A_BYTES, mapA, &full[stage], kb * BKT, a_row);
          tma_load_3d(sB + stage * B_BYTES, &tmB, &full[stage], kb * BKT, b_row0, gz);
          tma_load_3d(sB + stage * B_BYTES + HALF_B, &tmB, &full[stage], kb * BKT, b_row1, gz);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        report(p.status, MOE_ERR_TIMEOUT);
        *abort_v = 1;
      }
      // drain: the last min(issued, STAGES) loads must have landed before the CTA exits
      for (int q = 0; q < STAGES && q < issued; ++q) {
        if (stage == 0) {
          stage = STAGES;
          ph ^= 1u;
        }
        --stage;
        int dummy = 0;
        mbar_wait(&full[stage], ph, &dummy);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true, any = false;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_v)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], ph, abort_v)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < ROWB / 32; ++kk) {  // 32 bytes of k per MMA
            if (F8)
              umma_e4m3(d_tmem, smem_desc_kmajor<ROWB>(a_addr + kk * 32), smem_desc_kmajor<ROWB>(b_addr + kk * 32),
                        IDESC, (kb | kk) != 0 ? 1u : 0u);
            else
              umma_bf16(d_tmem, smem_desc_kmajor<ROWB>(a_addr + kk * 32), smem_desc_kmajor<ROWB>(b_addr + kk * 32),
                        IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          any = true;
          umma_commit(&empty[stage]);  // frees the smem stage when these MMAs complete
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);  // accumulator ready for the epilogue
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (!ok) {
        report(p.status, MOE_ERR_TIMEOUT);
        *abort_v = 1;
      }
      if (any) {  // every issued MMA finished before TMEM is released
        umma_commit(drain);
        int dummy = 0;
        mbar_wait(drain, 0, &dummy);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter+32)
    const int r_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t aph = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const TileDesc td = decode_tile(t, s_prefix, G, n_tiles);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, abort_v));
      if (!ok) {
        if (lane == 0) {
          report(p.status, MOE_ERR_TIMEOUT);
          *abort_v = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      const int r = td.m_blk * BM + r_in_tile;
      const bool row_ok = r < s_rows[td.g];
      const long long orow = (long long)s_orow[td.g] + r;

      if (MODE == MODE_ROUTER) {
        float* dst = static_cast<float*>(p.out) + orow * p.ldo;
        const int col_base = td.n_blk * BN;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c0, v);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 32; q += 4) {
              const int col = col_base + c0 + q;
              float f[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                f[u] = __uint_as_float(v[q + u]);
                if (p.bias && col + u < p.n_out) f[u] += p.bias[col + u];
              }
              if (col + 4 <= p.n_out) {
                *reinterpret_cast<float4*>(dst + col) = make_float4(f[0], f[1], f[2], f[3]);
              } else {
                for (int u = 0; u < 4; ++u)
                  if (col + u < p.n_out) dst[col + u] = f[u];
              }
            }
          }
        }
      } else if (MODE == MODE_FC1) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + orow * p.ldo;
        const int col_base = td.n_blk * (BN / 2);
        float ra = 1.0f;  // FP8: scale of this row's token
        const float* sb = nullptr;
        if (F8) {
          const int gz = p.g0 + td.g;
          // token of the row: routed rows through row2tok (or their own scale in
          // a_scale_rows); a shared expert's rows are the tokens in order, after A_routed
          // and the earlier shared experts' blocks
          if (row_ok)
            ra = gz < p.E ? (p.a_scale_rows ? p.a_scale_rows[orow] : token_scale(p, orow))
                          : p.a_scale[(int)(orow - p.A_routed - (long long)(gz - p.E) * p.N)];
          sb = p.b_scale + (size_t)gz * p.b_rows;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < BN / 2; c0 += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(taddr + c0, gv);
          tmem_ld32(taddr + BN / 2 + c0, uv);
          tmem_wait_ld();
          if (F8 && row_ok) {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const int col = min(col_base + c0 + q, p.n_out - 1);
              gv[q] = __float_as_uint(__uint_as_float(gv[q]) * ra * __ldg(sb + col));
              uv[q] = __float_as_uint(__uint_as_float(uv[q]) * ra * __ldg(sb + p.I + col));
            }
          }
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 32; q += 8) {
              const int col = col_base + c0 + q;
              if (col < p.n_out) {  // n_out % 8 == 0: the whole vector is valid
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const float h0 = silu_f32(__uint_as_float(gv[q + 2 * u])) * __uint_as_float(uv[q + 2 * u]);
                  const float h1 =
                      silu_f32(__uint_as_float(gv[q + 2 * u + 1])) * __uint_as_float(uv[q + 2 * u + 1]);
                  w[u] = pack_bf16x2(h0, h1);
                }
                *reinterpret_cast<uint4*>(dst + col) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
      } else {  // MODE_FC2
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + orow * p.ldo;
        float scale = 1.0f;
        if (row_ok && p.gate_w && p.g0 + td.g < p.E) {
          const int gi = p.row2tok ? p.row2tok[orow] : (int)orow;
          scale = check_range(gi, 0, p.A_routed, p.check) ? p.gate_w[gi] : 0.0f;
        }
        const float* sb = nullptr;
        if (F8) {
          if (row_ok) scale *= p.a_scale[orow];  // FP8: scale of this h row
          sb = p.b_scale + (size_t)(p.g0 + td.g) * p.b_rows;
        }
        const int col_base = td.n_blk * BN;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c0, v);
          tmem_wait_ld();
          if (F8 && row_ok) {
#pragma unroll
            for (int q = 0; q < 32; ++q)
              v[q] = __float_as_uint(__uint_as_float(v[q]) * __ldg(sb + min(col_base + c0 + q, p.n_out - 1)));
          }
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 32; q += 8) {
              const int col = col_base + c0 + q;
              if (col < p.n_out) {
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  w[u] = pack_bf16x2(__uint_as_float(v[q + 2 * u]) * scale,
                                     __uint_as_float(v[q + 2 * u + 1]) * scale);
                *reinterpret_cast<uint4*>(dst + col) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

static CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// 2D map over [rows, K] (K contiguous; bf16, or bytes when u8), box [128 rows, box_k
// elements], swizzle = the box's row bytes.
bool make_map_a(CUtensorMap* m, const void* base, long long rows, long long K, int box_k, bool u8, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  const int es = u8 ? 1 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)K * es};
  cuuint32_t box[2] = {(cuuint32_t)box_k, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(box_k * es),
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D map over [G, R, K] (bf16, or bytes when u8), box [1, box_rows, box_k elements].
bool make_map_b(CUtensorMap* m, const void* base, long long G, long long R, long long K, int box_rows, int box_k,
                bool u8) {
  auto enc = get_encode();
  if (!enc) return false;
  const int es = u8 ? 1 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)R, (cuuint64_t)G};
  cuuint64_t strides[2] = {(cuuint64_t)K * es, (cuuint64_t)(R * K * es)};
  cuuint32_t box[3] = {(cuuint32_t)box_k, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(box_k * es),
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cache[64] = {0};
  if (dev < 64 && cache[dev]) return cache[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev < 64) cache[dev] = n;
  return n;
}

template <int BN, int MODE, int BKT, bool F8 = false>
static cudaError_t launch_bn(const GemmArgs& g, const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                             long long max_tiles, cudaStream_t st) {
  // as many stages as fit in ~192 KB, at most 16
  constexpr int ES = F8 ? 1 : 2;
  constexpr int STAGE_B = BM * BKT * ES + BN * BKT * ES;
  constexpr int STAGES = (192 * 1024 / STAGE_B) > 16 ? 16 : (192 * 1024 / STAGE_B);
  constexpr int smem = smem_bytes_for<BN, STAGES, BKT, ES>();
  auto kern = tc_gemm_kernel<BN, MODE, STAGES, BKT, F8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  long long grid = sm_count();
  if (g.max_ctas > 0 && g.max_ctas < grid) grid = g.max_ctas;
  if (max_tiles < grid) grid = max_tiles;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, kThreads, smem, st>>>(a0, a1, b, g);
  return cudaGetLastError();
}

cudaError_t launch_tc_gemm(const GemmArgs& g, int a0_rows, int a1_rows, cudaStream_t st) {
  // B box rows: half the tile (two boxes per stage)
  int BN;
  if (g.mode == MODE_ROUTER) {
    // one tile column holds every expert when that already gives ~a wave of tiles;
    // with few 128-token row blocks the experts are split over narrower tile columns
    // so that more SMs stream x
    BN = 32;
    while (BN < g.n_out) BN <<= 1;
    const long long row_blocks = ((long long)g.N + BM - 1) / BM;
    while (BN > 32 && row_blocks * ((g.n_out + BN - 1) / BN) < 120) BN >>= 1;
  } else {
    BN = 256;
  }
  const bool f8 = g.fp8 != 0 && g.mode != MODE_ROUTER;
  const int bk = f8 ? 128 : (g.mode == MODE_ROUTER ? BK : BK);  // k per stage
  CUtensorMap a0, a1, b;
  if (!make_map_a(&a0, g.a0, a0_rows, g.K, bk, f8)) return cudaErrorInvalidValue;
  if (!make_map_a(&a1, g.a1 ? g.a1 : g.a0, g.a1 ? a1_rows : a0_rows, g.K, bk, f8)) return cudaErrorInvalidValue;
  if (!make_map_b(&b, g.b, g.g0 + g.G, g.b_rows, g.K, BN / 2, bk, f8)) return cudaErrorInvalidValue;
  // upper bound on tiles: every group adds at most one partial row block
  long long rows_total = launch_rows(g);
  long long blocks = (rows_total + BM - 1) / BM + g.G;
  long long n_tiles = g.mode == MODE_FC1 ? (g.n_out + BN / 2 - 1) / (BN / 2) : (g.n_out + BN - 1) / BN;
  long long max_tiles = blocks * n_tiles;
  switch (g.mode) {
    case MODE_FC1:
      if (f8) return launch_bn<256, MODE_FC1, 128, true>(g, a0, a1, b, max_tiles, st);
      return launch_bn<256, MODE_FC1, BK>(g, a0, a1, b, max_tiles, st);
    case MODE_FC2:
      if (f8) return launch_bn<256, MODE_FC2, 128, true>(g, a0, a1, b, max_tiles, st);
      return launch_bn<256, MODE_FC2, BK>(g, a0, a1, b, max_tiles, st);
    default:
      switch (BN) {
        case 32: return launch_bn<32, MODE_ROUTER, BK>(g, a0, a1, b, max_tiles, st);
        case 64: return launch_bn<64, MODE_ROUTER, BK>(g, a0, a1, b, max_tiles, st);
        case 128: return launch_bn<128, MODE_ROUTER, BK>(g, a0, a1, b, max_tiles, st);
        case 256: return launch_bn<256, MODE_ROUTER, BK>(g, a0, a1, b, max_tiles, st);
        default: return cudaErrorInvalidValue;
      }
  }
}

}  // namespace moe
