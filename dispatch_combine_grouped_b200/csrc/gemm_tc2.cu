// Grouped FC1 / FC2 over CTA pairs: tcgen05.mma.cta_group::2 with 256 x 256 tiles.
//
// Same jobs as the one-CTA kernel in gemm_tc.cu ("MoE我们喜欢你（四）" §4.1: FC1 +
// SwiGLU, FC2 x gate, over experts of variable size n_e), for the rows of each group that
// whole 256-row pair tiles cover (pair_rows()); the remaining 0..128 rows of a group run
// afterwards as 128-row tiles of the one-CTA kernel.
//
// Why pairs: an M=256 x N=256 tile computed by two SMs needs, per SM and per 64-deep
// k-step, its own 128 rows of A (16 KB) and half of B (16 KB): 32 KB instead of the 48 KB
// a one-CTA 128 x 256 tile needs for the same MMA work.  That lowers the L2->SM operand
// rate by a third and leaves room for 6 stages (192 KB) in flight instead of 4.
//
// Roles (both CTAs of a pair, 6 warps each):
//   warp 0     TMA producer: own A rows and own half of B into own shared memory; the
//              completion bytes land on the even CTA's stage barrier
//   warp 1     even CTA: issues the pair MMAs (4 per stage) and commits to the stage and
//              accumulator barriers of both CTAs; both CTAs: TMEM alloc / dealloc
//   warps 2-5  epilogue of this CTA's 128 rows, from its own TMEM; each warp releases
//              the accumulator to both CTAs' barriers
// F8: e4m3 operands, a 128-element k-step (the same 128-byte rows), kind::f8f6f4 MMAs and
// the row x column scales applied to the accumulator in the epilogue.
// No TMA multicast is used.  Every wait is bounded (2 s); on timeout the kernel writes
// MOE_ERR_TIMEOUT and every role leaves its loop.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int PM = 256;             // rows per pair tile (128 per CTA)
constexpr int PN = 256;             // MMA N (each CTA stages PN/2 rows of B)
constexpr int PK = 64;              // k per stage
constexpr int kPairThreads = 192;
constexpr int kPairStages = 6;
constexpr int kPairGroups = kMaxSlots + kMaxShared;
constexpr int A_BYTES = 128 * PK * 2;          // 16 KB
constexpr int B_BYTES = (PN / 2) * PK * 2;     // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kPairSmem = 1024 + kPairStages * STAGE_BYTES + 256 + 4 * (4 * kPairGroups + 8);

}  // namespace

template <int MODE, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  constexpr uint32_t TMEM_COLS = 2 * PN;  // double-buffered 128 x 256 fp32 accumulator
  constexpr uint32_t IDESC = F8 ? idesc_e4m3_f32(PM, PN) : idesc_bf16_f32(PM, PN);
  constexpr int KSTEP = F8 ? 2 * PK : PK;  // elements of k per stage (128-byte rows either way)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPairStages * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kPairStages * B_BYTES);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);
  int* s_prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + 256);
  int* s_arow = s_prefix + (kPairGroups + 1);
  int* s_orow = s_arow + kPairGroups;
  int* s_rows = s_orow + kPairGroups;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int G = p.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);   // even CTA: one arrive (expect both CTAs' bytes)
      mbar_init(&empty[s], 1);  // one pair commit per use
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);   // one pair commit per use
      mbar_init(&tempty[b], 8);  // 4 epilogue warps in each CTA
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
  if (warp == 1) tmem_alloc_pair(tmem_holder, TMEM_COLS);

  // group table over the rows that pair tiles cover
  for (int g = threadIdx.x; g < G; g += kPairThreads) {
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
    s_rows[g] = rows;  // valid rows (stores are masked to these)
    s_arow[g] = arow;
    s_orow[g] = orow;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix of pair tiles (256-row blocks) per group
    int run = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      const int v = g < G ? pair_rows(s_rows[g]) / PM : 0;
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
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
  tc_fence_after();

  const uint32_t tmem_base = *tmem_holder;
  const int n_tiles = (MODE == MODE_FC1) ? (p.n_out + PN / 2 - 1) / (PN / 2) : (p.n_out + PN - 1) / PN;
  const int total = s_prefix[G] * n_tiles;
  const int num_kb = (p.K + KSTEP - 1) / KSTEP;
  const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  volatile int* abort_v = abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t lead_full0 = map_to_rank(smem_u32(&full[0]), 0);
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = pair_id; t < total && ok; t += n_pairs) {
        int lo = 0, hi = G - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (s_prefix[mid] * n_tiles <= t) lo = mid;
          else hi = mid - 1;
        }
        const int g = lo, mt = s_prefix[g + 1] - s_prefix[g];
        const int local = t - s_prefix[g] * n_tiles;
        const int n_blk = local / mt, m_blk = local - n_blk * mt;
        const int gz = p.g0 + g;  // global group = weight index
        const CUtensorMap* mapA = (gz >= p.E && p.shared_from_map1) ? &tmA1 : &tmA0;
        const int a_row = s_arow[g] + m_blk * PM + (int)rank * 128;
        // FC1: the even CTA stages the W_gate rows, the odd CTA the W_up rows of the same
        // 128 outputs, so accumulator columns [0,128) are gate and [128,256) are up
        const int b_row = (MODE == MODE_FC1) ? (rank == 0 ? n_blk * 128 : p.I + n_blk * 128)
                                             : n_blk * PN + (int)rank * 128;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], ph ^ 1u, abort_v)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
          const uint32_t bar = lead_full0 + (uint32_t)(stage * sizeof(uint64_t));
          tma_load_2d_pair(sA + stage * A_BYTES, mapA, bar, kb * KSTEP, a_row);
          tma_load_3d_pair(sB + stage * B_BYTES, &tmB, bar, kb * KSTEP, b_row, gz);
          if (++stage == kPairStages) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        report(p.status, MOE_ERR_TIMEOUT);
        *abort_v = 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true, any = false;
      for (int t = pair_id; t < total && ok; t += n_pairs) {
        if (!mbar_wait_cluster(&tempty[acc], aph ^ 1u, abort_v)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * PN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_cluster(&full[stage], ph, abort_v)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 32 bytes of k per MMA
            if (F8)
              umma_e4m3_pair(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC,
                             (kb | kk) != 0 ? 1u : 0u);
            else
              umma_bf16_pair(d_tmem, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC,
                             (kb | kk) != 0 ? 1u : 0u);
          }
          any = true;
          umma_commit_pair(&empty[stage], 0x3);  // frees this stage in both CTAs
          if (++stage == kPairStages) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);  // accumulator ready in both CTAs
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (!ok) {
        report(p.status, MOE_ERR_TIMEOUT);
        *abort_v = 1;
      }
      if (any) {  // every pair MMA finished before TMEM is released
        umma_commit_pair(drain, 0x1);
        int dummy = 0;
        mbar_wait(drain, 0, &dummy);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5, both CTAs)
    const int quarter = warp & 3;
    const int r_in_tile = quarter * 32 + lane;
    const uint32_t tempty_peer0 = map_to_rank(smem_u32(&tempty[0]), rank ^ 1u);
    int acc = 0;
    uint32_t aph = 0;
    for (int t = pair_id; t < total; t += n_pairs) {
      int lo = 0, hi = G - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_prefix[mid] * n_tiles <= t) lo = mid;
        else hi = mid - 1;
      }
      const int g = lo, mt = s_prefix[g + 1] - s_prefix[g];
      const int local = t - s_prefix[g] * n_tiles;
      const int n_blk = local / mt, m_blk = local - n_blk * mt;
      const bool ok = __all_sync(0xffffffffu, mbar_wait_cluster(&tfull[acc], aph, abort_v));
      if (!ok) {
        if (lane == 0) {
          report(p.status, MOE_ERR_TIMEOUT);
          *abort_v = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * PN);
      const int r = m_blk * PM + (int)rank * 128 + r_in_tile;
      const bool row_ok = r < s_rows[g];
      const long long orow = (long long)s_orow[g] + r;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + orow * p.ldo;
      if (MODE == MODE_FC1) {
        const int col_base = n_blk * (PN / 2);
        float ra = 1.0f;  // FP8: scale of this row's token
        const float* sb = nullptr;
        if (F8) {
          const int gz = p.g0 + g;
          // token of the row: routed rows through row2tok (or their own scale in
          // a_scale_rows); a shared expert's rows are the tokens in order, after A_routed
          // and the earlier shared experts' blocks
          if (row_ok)
            ra = gz < p.E ? (p.a_scale_rows ? p.a_scale_rows[orow] : token_scale(p, orow))
                          : p.a_scale[(int)(orow - p.A_routed - (long long)(gz - p.E) * p.N)];
          sb = p.b_scale + (size_t)gz * p.b_rows;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < PN / 2; c0 += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(taddr + c0, gv);
          tmem_ld32(taddr + PN / 2 + c0, uv);
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
              if (col < p.n_out) {
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
      } else {
        float scale = 1.0f;
        if (row_ok && p.gate_w && p.g0 + g < p.E) {
          const int gi = p.row2tok ? p.row2tok[orow] : (int)orow;
          scale = check_range(gi, 0, p.A_routed, p.check) ? p.gate_w[gi] : 0.0f;
        }
        const float* sb = nullptr;
        if (F8) {
          if (row_ok) scale *= p.a_scale[orow];  // FP8: scale of this h row
          sb = p.b_scale + (size_t)(p.g0 + g) * p.b_rows;
        }
        const int col_base = n_blk * PN;
#pragma unroll 1
        for (int c0 = 0; c0 < PN; c0 += 32) {
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
                  w[u] = pack_bf16x2(__uint_as_float(v[q + 2 * u]) * scale, __uint_as_float(v[q + 2 * u + 1]) * scale);
                *reinterpret_cast<uint4*>(dst + col) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // release this accumulator to the MMA issuer: own and peer barrier
        mbar_arrive(&tempty[acc]);
        mbar_arrive_cluster(tempty_peer0 + (uint32_t)(acc * sizeof(uint64_t)));
      }
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA releases TMEM or exits while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

cudaError_t launch_tc_gemm_pair(const GemmArgs& g, int a0_rows, int a1_rows, cudaStream_t st) {
  CUtensorMap a0, a1, b;
  const bool f8 = g.fp8 != 0;
  const int bk = f8 ? 2 * PK : PK;
  if (!make_map_a(&a0, g.a0, a0_rows, g.K, bk, f8)) return cudaErrorInvalidValue;
  if (!make_map_a(&a1, g.a1 ? g.a1 : g.a0, g.a1 ? a1_rows : a0_rows, g.K, bk, f8)) return cudaErrorInvalidValue;
  if (!make_map_b(&b, g.b, g.g0 + g.G, g.b_rows, g.K, PN / 2, bk, f8)) return cudaErrorInvalidValue;
  const long long rows_total = launch_rows(g);
  const long long pairs = (rows_total + PM - 1) / PM + g.G;
  const long long n_tiles = g.mode == MODE_FC1 ? (g.n_out + PN / 2 - 1) / (PN / 2) : (g.n_out + PN - 1) / PN;
  long long grid = (sm_count() / 2) * 2;
  if (g.max_ctas > 0 && g.max_ctas < grid) grid = (g.max_ctas / 2) * 2;
  if (2 * pairs * n_tiles < grid) grid = 2 * pairs * n_tiles;
  if (grid < 2) grid = 2;
  auto run = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)grid, kPairThreads, kPairSmem, st>>>(a0, a1, b, g);
    return cudaGetLastError();
  };
  if (g.mode == MODE_FC1) return f8 ? run(tc_gemm_pair_kernel<MODE_FC1, true>) : run(tc_gemm_pair_kernel<MODE_FC1, false>);
  return f8 ? run(tc_gemm_pair_kernel<MODE_FC2, true>) : run(tc_gemm_pair_kernel<MODE_FC2, false>);
}

}  // namespace moe
