// Block-scaled (MX) e4m3 grouped GEMM on the 5th-generation tensor cores: the expert FFN's
// two GEMMs ("MoE我们喜欢你（四）" §4.1 FC1 + SwiGLU, FC2 with the combine's gate; MXFP8 as
// the low-precision expert compute) with operands in the microscaling format: e4m3 codes
// and one E8M0 power-of-two scale per 32 values along K, in row-major arrays [rows, K/32].
// The scales are applied inside the MMA (tcgen05.mma kind::mxf8f6f4.block_scale), so the
// accumulator holds sum_k (qa Xa)(qb Xb) and the epilogue applies no scale of its own.
//
// Structure (one CTA per SM, persistent, 7 warps):
//   warp 0      TMA producer: A tile [128 rows x 128 codes] + B tile [192 rows x 128 codes]
//               per stage, 128B swizzle (the same boxes as the e4m3 kernel, B in two
//               96-row boxes: FC1 W_gate rows and the matching W_up rows)
//   warp 6      scale stager: reads the scale bytes (4 per row and stage: 128 K values) of
//               the 128 A rows and the 192 B rows from the row-major arrays, 8 stages per
//               batch of loads (32 bytes of each row, 16-byte loads when rows allow), and
//               writes them in the layout tcgen05.cp takes (32 rows x 16 bytes per 128-row
//               atom: row r at byte 16 (r % 32) + 4 (r / 32) + k-block), then arrives on
//               the stage's barrier beside the TMA bytes.  Lanes read different rows, so
//               4-byte loads cost one L1 wavefront per row each: the 16-byte form moves
//               the same bytes in a quarter of the wavefronts (measured 1270 -> 1580
//               TFLOP/s on the wide expert shapes)
//   warp 1      MMA issuer: per stage three tcgen05.cp of the atoms into TMEM (scale A: 4
//               columns, scale B: 8; every 32-lane quarter gets a copy) and 4 block-scaled
//               MMAs (M=128, N=192, K=32 each; the scale of k-block kk is byte kk of the
//               TMEM words, selected by the instruction descriptor)
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes, SwiGLU / gate, bf16 stores;
//               FC1 also quantises h to MX as it goes (a 32-column chunk of a row is one
//               MX block of h, held by one thread), so h needs no pass of its own
// TMEM: two 192-column fp32 accumulators (columns 0 and 192), the scale columns after
// them (one copy; the tcgen05 operations of a thread run in issue order, so the next
// stage's copy follows the MMAs that read the previous one).  N = 192 keeps both
// accumulators and the scales inside the 512 columns of an SM.  Every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.cuh"
#include "mx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 192;                 // accumulator columns per tile (FC1: 96 gate + 96 up)
constexpr int kBK = 128;                 // e4m3 values (bytes) of K per stage
constexpr int kStages = 5;
constexpr int kThreadsMx = 224;          // 7 warps
constexpr int kABytes = kBM * kBK;       // 16 KB
constexpr int kBBytes = kBN * kBK;       // 24 KB
constexpr int kHalfB = kBBytes / 2;      // one 96-row box
constexpr int kSfBytes = 1536;           // per stage: A atom (512) + two B atoms (2 x 512)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfaCol = 2 * kBN;    // 384: 4 columns (128 rows / 32)
constexpr uint32_t kSfbCol = kSfaCol + 8;  // 392: 8 columns (the second atom half used)
constexpr int kMaxGroupsMx = kMaxSlots + kMaxShared;
constexpr int kBarBytes = ((2 * kStages + 5) * 8 + 8 + 15) & ~15;
constexpr int kSmemMx = 1024 + kStages * (kABytes + kBBytes + kSfBytes) + kBarBytes + 4 * (4 * kMaxGroupsMx + 8);
static_assert(kSmemMx <= 232448, "shared memory of one CTA");

// Instruction descriptor of the block-scaled MMA: A and B E4M3 (format 0), K-major, scale
// format E8M0, shape M x N; sf_id selects the byte of the TMEM scale words for A and B.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N, int sf_id) {
  return ((uint32_t)sf_id << 4)          // B scale-factor id
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | (1u << 23)                    // scale format: E8M0
         | ((uint32_t)(M >> 4) << 24)    // M / 16
         | ((uint32_t)sf_id << 29);      // A scale-factor id
}

__device__ __forceinline__ void umma_mx(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t tmem_sfa, uint32_t tmem_sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tmem_sfa), "r"(tmem_sfb)
      : "memory");
}

// 32 rows x 16 bytes of shared memory into 4 TMEM columns of lanes 0-31, copied to the
// other three 32-lane quarters as well.
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Descriptor of one scale atom: 32 rows of 16 bytes, no swizzle, 8-row core matrices
// 128 bytes apart.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address
  d |= (uint64_t)(128u >> 4) << 16;         // leading byte offset (one core matrix along K)
  d |= (uint64_t)(128u >> 4) << 32;         // stride byte offset: 8 rows x 16 B
  d |= (uint64_t)1u << 46;                  // descriptor version (sm_100); layout type 0: no swizzle
  return d;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct MxTile {
  int g, m_blk, n_blk;
};

// Tiles are ordered group-major, then by output-column tile, then by row block, so that the
// row blocks sharing one weight tile run at the same time.
__device__ __forceinline__ MxTile mx_decode_tile(int t, const int* prefix, int G, int n_tiles) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // largest g with prefix[g] * n_tiles <= t
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] * n_tiles <= t) lo = mid;
    else hi = mid - 1;
  }
  const int mt = prefix[lo + 1] - prefix[lo];
  const int local = t - prefix[lo] * n_tiles;
  MxTile d;
  d.g = lo;
  d.n_blk = local / mt;
  d.m_blk = local - d.n_blk * mt;
  return d;
}

// VEC16: scale rows are 16-byte aligned (K % 512 == 0) and read 16 bytes at a time.
template <int MODE, bool VEC16>
__global__ void __launch_bounds__(kThreadsMx, 1)
    tc_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                      const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  static_assert(MODE == MODE_FC1 || MODE == MODE_FC2, "expert GEMMs only");
  constexpr uint32_t TX_BYTES = kABytes + kBBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * kABytes;
  uint8_t* sSF = sB + kStages * kBBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSF + kStages * kSfBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);
  int* s_prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + kBarBytes);
  int* s_arow = s_prefix + (kMaxGroupsMx + 1);
  int* s_orow = s_arow + kMaxGroupsMx;
  int* s_rows = s_orow + kMaxGroupsMx;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 2);  // the producer's expect_tx arrival and the scale stager's
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
  if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);

  // group table: rows, first A row, first output row
  for (int g = threadIdx.x; g < G; g += kThreadsMx) {
    int rows, arow, orow;
    const int gg = p.g0 + g;
    if (gg < p.E) {
      rows = p.n_e[gg];
      arow = orow = p.expert_off[gg];
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
  if (warp == 0) {  // exclusive prefix of 128-row blocks per group
    int run = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      const int v = g < G ? (s_rows[g] + kBM - 1) / kBM : 0;
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
  const int n_tiles = (MODE == MODE_FC1) ? (p.n_out + kBN / 2 - 1) / (kBN / 2) : (p.n_out + kBN - 1) / kBN;
  const int total = s_prefix[G] * n_tiles;
  const int num_kb = p.K / kBK;  // K % 128 == 0
  volatile int* abort_v = abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const MxTile td = mx_decode_tile(t, s_prefix, G, n_tiles);
        const int gz = p.g0 + td.g;
        const CUtensorMap* mapA = (gz >= p.E && p.shared_from_map1) ? &tmA1 : &tmA0;
        const int a_row = s_arow[td.g] + td.m_blk * kBM;
        int b_row0, b_row1;
        if (MODE == MODE_FC1) {
          b_row0 = td.n_blk * (kBN / 2);
          b_row1 = p.I + b_row0;
        } else {
          b_row0 = td.n_blk * kBN;
          b_row1 = b_row0 + kBN / 2;
        }
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], ph ^ 1u, abort_v)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], TX_BYTES);
          tma_load_2d(sA + stage * kABytes, mapA, &full[stage], kb * kBK, a_row);
          tma_load_3d(sB + stage * kBBytes, &tmB, &full[stage], kb * kBK, b_row0, gz);
          tma_load_3d(sB + stage * kBBytes + kHalfB, &tmB, &full[stage], kb * kBK, b_row1, gz);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        report(p.status, MOE_ERR_TIMEOUT);
        *abort_v = 1;
      }
      // the last min(issued, stages) loads must have landed before the CTA exits
      for (int q = 0; q < kStages && q < issued; ++q) {
        if (stage == 0) {
          stage = kStages;
          ph ^= 1u;
        }
        --stage;
        int dummy = 0;  // not cut short by an abort: the bytes must land before exit
        mbar_wait(&full[stage], ph, &dummy);
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ scale stager
    const long long kpr = p.K / 32;  // scale bytes per row
    int stage = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const MxTile td = mx_decode_tile(t, s_prefix, G, n_tiles);
      const int gz = p.g0 + td.g;
      const bool m1 = gz >= p.E && p.shared_from_map1;
      const uint8_t* sfa = m1 ? p.a1_sf : p.a0_sf;
      const long long a_last = (m1 ? p.a1_rows : p.a0_rows) - 1;
      const long long a_row = (long long)s_arow[td.g] + td.m_blk * kBM;
      const uint8_t* pa[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // rows past the tensor read its last row (never stored)
        const long long r = a_row + 32 * q + lane;
        pa[q] = sfa + (r < a_last ? r : a_last) * kpr;
      }
      const uint8_t* pb[6];
#pragma unroll
      for (int q = 0; q < 6; ++q) {
        long long r;
        if (MODE == MODE_FC1)
          r = q < 3 ? (long long)td.n_blk * (kBN / 2) + 32 * q + lane
                    : (long long)p.I + td.n_blk * (kBN / 2) + 32 * (q - 3) + lane;
        else
          r = (long long)td.n_blk * kBN + 32 * q + lane;
        if (r > p.b_rows - 1) r = p.b_rows - 1;
        pb[q] = p.b_sf + ((long long)gz * p.b_rows + r) * kpr;
      }
      // 8 stages of scale words per batch of loads: 32 bytes of each of the lane's 10 rows
      // (two 16-byte loads when rows are 16-byte aligned, K % 512 == 0; else 4-byte loads)
      for (int kb0 = 0; kb0 < num_kb && ok; kb0 += 8) {
        uint32_t va[8][4], vb[8][6];
        if (VEC16) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (kb0 + 4 * h < num_kb) {  // num_kb % 4 == 0: the 16 bytes lie inside the row
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 u = __ldg(reinterpret_cast<const uint4*>(pa[q] + 4 * kb0 + 16 * h));
                va[4 * h][q] = u.x;
                va[4 * h + 1][q] = u.y;
                va[4 * h + 2][q] = u.z;
                va[4 * h + 3][q] = u.w;
              }
#pragma unroll
              for (int q = 0; q < 6; ++q) {
                const uint4 u = __ldg(reinterpret_cast<const uint4*>(pb[q] + 4 * kb0 + 16 * h));
                vb[4 * h][q] = u.x;
                vb[4 * h + 1][q] = u.y;
                vb[4 * h + 2][q] = u.z;
                vb[4 * h + 3][q] = u.w;
              }
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (kb0 + j < num_kb) {
#pragma unroll
              for (int q = 0; q < 4; ++q) va[j][q] = __ldg(reinterpret_cast<const uint32_t*>(pa[q] + 4 * (kb0 + j)));
#pragma unroll
              for (int q = 0; q < 6; ++q) vb[j][q] = __ldg(reinterpret_cast<const uint32_t*>(pb[q] + 4 * (kb0 + j)));
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (kb0 + j < num_kb) {
            if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], ph ^ 1u, abort_v))) {
              ok = false;
              break;
            }
            uint8_t* dst = sSF + stage * kSfBytes;
            *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(va[j][0], va[j][1], va[j][2], va[j][3]);
            *reinterpret_cast<uint4*>(dst + 512 + 16 * lane) = make_uint4(vb[j][0], vb[j][1], vb[j][2], vb[j][3]);
            *reinterpret_cast<uint4*>(dst + 1024 + 16 * lane) =
                make_uint4(vb[j][4], vb[j][5], 0x7F7F7F7Fu, 0x7F7F7F7Fu);
            fence_proxy_async_smem();  // visible to tcgen05.cp (async proxy)
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[stage]);
            if (++stage == kStages) {
              stage = 0;
              ph ^= 1u;
            }
          }
        }
      }
    }
    if (!ok && lane == 0) {
      report(p.status, MOE_ERR_TIMEOUT);
      *abort_v = 1;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true, any = false;
      const uint32_t t_sfa = tmem_base + kSfaCol, t_sfb = tmem_base + kSfbCol;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort_v)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], ph, abort_v)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf_addr = smem_u32(sSF + stage * kSfBytes);
          tmem_cp_atom(t_sfa, sf_atom_desc(sf_addr));
          tmem_cp_atom(t_sfb, sf_atom_desc(sf_addr + 512));
          tmem_cp_atom(t_sfb + 4, sf_atom_desc(sf_addr + 1024));
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 32; ++kk) {  // 32 codes of K per MMA, one scale byte each
            umma_mx(d_tmem, smem_desc_kmajor<kBK>(a_addr + kk * 32), smem_desc_kmajor<kBK>(b_addr + kk * 32),
                    idesc_mx(kBM, kBN, kk), t_sfa | ((uint32_t)kk << 30), t_sfb | ((uint32_t)kk << 30),
                    (kb | kk) != 0 ? 1u : 0u);
          }
          any = true;
          umma_commit(&empty[stage]);  // frees the stage (codes and scale atoms) when these complete
          if (++stage == kStages) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
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
      const MxTile td = mx_decode_tile(t, s_prefix, G, n_tiles);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, abort_v));
      if (!ok) {
        if (lane == 0) {
          report(p.status, MOE_ERR_TIMEOUT);
          *abort_v = 1;
        }
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * kBN);
      const int r = td.m_blk * kBM + r_in_tile;
      const bool row_ok = r < s_rows[td.g];
      const long long orow = (long long)s_orow[td.g] + r;
      __nv_bfloat16* dst = p.out ? static_cast<__nv_bfloat16*>(p.out) + orow * p.ldo : nullptr;
      if (MODE == MODE_FC1) {
        const int col_base = td.n_blk * (kBN / 2);
#pragma unroll 1
        for (int c0 = 0; c0 < kBN / 2; c0 += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(taddr + c0, gv);
          tmem_ld32(taddr + kBN / 2 + c0, uv);
          tmem_wait_ld();
          // n_out % 32 == 0: a 32-column chunk is wholly inside the output or wholly past it
          if (row_ok && col_base + c0 < p.n_out) {
            uint32_t w[16];  // the chunk's h rounded to bf16, two per word
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const float h0 = silu_f32(__uint_as_float(gv[2 * u])) * __uint_as_float(uv[2 * u]);
              const float h1 = silu_f32(__uint_as_float(gv[2 * u + 1])) * __uint_as_float(uv[2 * u + 1]);
              w[u] = pack_bf16x2(h0, h1);
            }
            const int col = col_base + c0;
            if (p.out) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(dst + col + 8 * q) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
            }
            if (p.q_out) {  // the chunk is one MX block of h: quantise the stored (bf16) values
              float f[32];
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[u]));
                f[2 * u] = t.x;
                f[2 * u + 1] = t.y;
              }
              uint32_t packed[8];
              const uint8_t sfb = mx_quantize32(f, packed);
              uint4* qd = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.q_out) + orow * p.n_out + col);
              qd[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
              qd[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
              p.q_sf[orow * (p.n_out / 32) + col / 32] = sfb;
            }
          }
        }
      } else {
        float scale = 1.0f;
        if (row_ok && p.gate_w && p.g0 + td.g < p.E) {
          const int gi = p.row2tok ? p.row2tok[orow] : (int)orow;
          scale = check_range(gi, 0, p.A_routed, p.check) ? p.gate_w[gi] : 0.0f;
        }
        const int col_base = td.n_blk * kBN;
#pragma unroll 1
        for (int c0 = 0; c0 < kBN; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c0, v);
          tmem_wait_ld();
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
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

template <int MODE, bool VEC16>
cudaError_t launch_mode(const GemmArgs& g, const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                        long long max_tiles, cudaStream_t st) {
  auto kern = tc_gemm_mx_kernel<MODE, VEC16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMx);
  if (e != cudaSuccess) return e;
  long long grid = sm_count();
  if (g.max_ctas > 0 && g.max_ctas < grid) grid = g.max_ctas;
  if (max_tiles < grid) grid = max_tiles;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, kThreadsMx, kSmemMx, st>>>(a0, a1, b, g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemm_mx(const GemmArgs& g, cudaStream_t st) {
  if ((g.mode != MODE_FC1 && g.mode != MODE_FC2) || g.K % kBK != 0 || g.n_out % 32 != 0 || !g.a0_sf || !g.b_sf ||
      (g.a1 && !g.a1_sf) || g.a0_rows < 1 || g.b_rows < 1 || (g.q_out && !g.q_sf) ||
      (g.mode == MODE_FC2 && !g.out) || (g.mode == MODE_FC1 && !g.out && !g.q_out))
    return cudaErrorInvalidValue;
  CUtensorMap a0, a1, b;
  if (!make_map_a(&a0, g.a0, g.a0_rows, g.K, kBK, true)) return cudaErrorInvalidValue;
  const bool m1 = g.a1 != nullptr;
  if (!make_map_a(&a1, m1 ? g.a1 : g.a0, m1 ? g.a1_rows : g.a0_rows, g.K, kBK, true)) return cudaErrorInvalidValue;
  if (!make_map_b(&b, g.b, g.g0 + g.G, g.b_rows, g.K, kBN / 2, kBK, true)) return cudaErrorInvalidValue;
  const long long blocks = (launch_rows(g) + kBM - 1) / kBM + g.G;  // every group adds at most one partial block
  const long long n_tiles = g.mode == MODE_FC1 ? (g.n_out + kBN / 2 - 1) / (kBN / 2) : (g.n_out + kBN - 1) / kBN;
  // 16-byte scale loads need 16-byte aligned rows (K / 32 % 16 == 0) and arrays
  const bool vec = g.K % 512 == 0 && ((reinterpret_cast<uintptr_t>(g.a0_sf) | reinterpret_cast<uintptr_t>(g.a1_sf) |
                                       reinterpret_cast<uintptr_t>(g.b_sf)) & 15) == 0;
  const long long mt = blocks * n_tiles;
  if (g.mode == MODE_FC1)
    return vec ? launch_mode<MODE_FC1, true>(g, a0, a1, b, mt, st) : launch_mode<MODE_FC1, false>(g, a0, a1, b, mt, st);
  return vec ? launch_mode<MODE_FC2, true>(g, a0, a1, b, mt, st) : launch_mode<MODE_FC2, false>(g, a0, a1, b, mt, st);
}

}  // namespace moe
