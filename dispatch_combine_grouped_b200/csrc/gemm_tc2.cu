// Grouped FC1 / FC2 over CTA pairs (tcgen05.mma.cta_group::2), every row of a group in
// one pass over its weights.
//
// Same jobs as the one-CTA kernel in gemm_tc.cu ("MoE我们喜欢你（四）" §4.1: FC1 +
// SwiGLU, FC2 x gate, over experts of variable size n_e); the ep_deepep explainer §2 puts
// an expert's cost at its rows n_e, so each weight tile is streamed once for all of them.
//
// Tiles.  The N dimension of a tile is 256 weight rows (FC1: 128 gate + 128 up outputs;
// FC2: 256 outputs); each CTA of the pair stages half of them.  The M dimension covers a
// group's rows in 256-row blocks (128 per CTA, an M=256 pair MMA), and a group whose rows
// end 1..128 past a block boundary carries that remainder on its last block: each k-step
// then also issues an M=128 pair MMA (64 rows per CTA) on the same weight stage.  A group
// of at most 128 rows is one such 128-row tile.  So a tile is FULL (256 rows), CARRY (256
// + up to 128 rows) or SHORT (up to 128 rows), and no row needs a second pass over the
// weights.  (A carrying block of half the weight rows would fit its own buffer but was
// measured 40% slower: it needs a third more operand bytes per MMA cycle.)
//
// Accumulators.  TMEM holds 512 fp32 columns, seen as two buffers b of two 128-column
// regions (lo, hi).  An M=256 x N=256 accumulator fills one buffer; an M=128 x N=256
// accumulator fills one region (it keeps columns [0,128) of N on lanes 0-63 and [128,256)
// on lanes 64-127).  Tiles alternate buffers; a CARRY tile on buffer b keeps its extra
// rows in the hi region of buffer b^1, a SHORT tile uses the lo region of its buffer.  The
// MMA issuer acquires each region before a tile's first MMA and the epilogue releases each
// region as soon as it has drained it (the borrowed one first), so a CARRY tile waits only
// for one region of the tile before it, not for a whole buffer.
//
// FC1 column order: CTA r stages W_gate rows [n0 + 64r, +64) then W_up rows of the same
// outputs, so every 128-column region holds 64 gate and the matching 64 up columns per
// lane and SwiGLU needs nothing from another lane.
//
// Roles (both CTAs of a pair, 6 warps each):
//   warp 0     TMA producer: own A rows (and carried rows) and own half of B into own
//              shared memory; the completion bytes land on the even CTA's stage barrier
//   warp 1     even CTA: acquires the regions and issues the pair MMAs (4 or 8 per stage),
//              commits to the stage and accumulator barriers of both CTAs; both CTAs:
//              TMEM alloc / dealloc
//   warps 2-5  epilogue from this CTA's TMEM; each warp releases a drained region to both
//              CTAs' barriers
// F8: e4m3 operands, a 128-element k-step (the same 128-byte rows), kind::f8f6f4 MMAs and
// the row x column scales applied to the accumulator in the epilogue.
// No TMA multicast is used.  Every wait is bounded (2 s); on timeout the kernel writes
// MOE_ERR_TIMEOUT and every role leaves its loop.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int PM = 256;             // rows of a full block (128 per CTA)
constexpr int PN = 256;             // MMA N (each CTA stages PN/2 rows of B)
constexpr int PK = 64;              // k per stage (bf16; 128 for e4m3: same bytes)
constexpr int kPairThreads = 192;
constexpr int kPairStages = 6;              // A + B stages
constexpr int kTSlots = 3;                  // stages of carried (or short-tile) rows, a ring of their own
constexpr int kPairGroups = kMaxSlots + kMaxShared;
constexpr int A_BYTES = 128 * PK * 2;          // 16 KB: this CTA's 128 rows of a full block
constexpr int T_BYTES = 64 * PK * 2;           // 8 KB: this CTA's 64 carried (or short-tile) rows
constexpr int B_BYTES = (PN / 2) * PK * 2;     // 16 KB: this CTA's half of the weight tile
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kTables = 4;                     // two phase prefixes, orow, rows
constexpr int kPairSmem =
    1024 + kPairStages * STAGE_BYTES + kTSlots * T_BYTES + 256 + 4 * (kTables * kPairGroups + 16);
static_assert(kPairSmem <= 227 * 1024, "shared memory of the pair kernel");

enum TileKind { FULL = 0, CARRY = 1, SHORT = 2 };

// A group of `rows` rows: *full = 256-row blocks, the last one carrying *extra rows when
// *extra > 0; with *full = 0, one short tile of *extra rows.  Returns the group's tiles per
// weight tile in the first phase of the schedule (full blocks that carry nothing, or the
// short tile); *carry = tiles per weight tile in the second phase (the carrying block).
__host__ __device__ __forceinline__ int group_tiles(int rows, int* full, int* extra, int* carry) {
  *full = 0;
  *extra = 0;
  *carry = 0;
  if (rows <= 0) return 0;
  if (rows <= 128) {
    *extra = rows;
    return 1;
  }
  const int q = rows >> 8, r = rows & 255;
  if (r == 0) {
    *full = q;
  } else if (r > 128) {
    *full = q + 1;
  } else {
    *full = q;
    *extra = r;
    *carry = 1;
    return q - 1;
  }
  return *full;
}

struct PairTile {
  int g, n_blk, m_blk, kind, full;
};

// The schedule runs in two phases: first every FULL and SHORT tile, then every CARRY
// tile.  A carrying tile borrows TMEM from the tile before it and lends to the one after
// it on the same CTA pair, so each change between kinds costs a pipeline drain; grouping
// the carrying tiles keeps those drains to one per tile.  Inside a phase tiles are
// group-major, then weight tile, then block, so that the tiles sharing a weight tile run
// together.  prefix / prefc: exclusive prefix over groups of the tiles per weight tile of
// the first / second phase.
__device__ __forceinline__ int search_group(int t, const int* prefix, int G, int n_tiles) {
  int lo = 0, hi = G - 1;  // largest g with prefix[g] * n_tiles <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] * n_tiles <= t) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ PairTile decode_pair_tile(int t, const int* prefix, const int* prefc, const int* rows,
                                                     int G, int n_tiles) {
  PairTile d;
  const int first = prefix[G] * n_tiles;
  int ex, cy;
  if (t < first) {
    d.g = search_group(t, prefix, G, n_tiles);
    const int mt = prefix[d.g + 1] - prefix[d.g];
    const int local = t - prefix[d.g] * n_tiles;
    d.n_blk = local / mt;
    d.m_blk = local - d.n_blk * mt;
    group_tiles(rows[d.g], &d.full, &ex, &cy);
    d.kind = d.full == 0 ? SHORT : FULL;
  } else {
    const int t2 = t - first;
    d.g = search_group(t2, prefc, G, n_tiles);
    d.n_blk = t2 - prefc[d.g] * n_tiles;  // one carrying tile per weight tile
    group_tiles(rows[d.g], &d.full, &ex, &cy);
    d.m_blk = d.full - 1;
    d.kind = CARRY;
  }
  return d;
}

// Positions in the A/B stage ring and in the carried-row ring.
struct Rings {
  int stage;
  uint32_t ph;
  int ts;
  uint32_t tph;
};

// The loads of one tile (TMA producer of either CTA).  MAIN: 128 rows of a full block;
// EXTRA: 64 carried (or short-tile) rows.  The k-loop holds nothing else: the producer and
// the MMA issuer are on the critical path of every k-step.
template <int MODE, bool MAIN, bool EXTRA, int KSTEP>
__device__ __forceinline__ bool load_tile(Rings& r, int num_kb, uint64_t* full, uint64_t* empty, uint64_t* tempty,
                                          uint32_t lead_full0, bool leader, uint8_t* sA, uint8_t* sT, uint8_t* sB,
                                          const CUtensorMap* mapA, const CUtensorMap* mapT, const CUtensorMap* mapB,
                                          int a_row, int t_row, int b_row0, int b_row1, int gz,
                                          volatile int* abort_v) {
  constexpr uint32_t TX = 2u * (uint32_t)(B_BYTES + (MAIN ? A_BYTES : 0) + (EXTRA ? T_BYTES : 0));
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!mbar_wait(&empty[r.stage], r.ph ^ 1u, abort_v)) return false;
    if (EXTRA && !mbar_wait(&tempty[r.ts], r.tph ^ 1u, abort_v)) return false;
    if (leader) mbar_arrive_expect_tx(&full[r.stage], TX);
    const uint32_t bar = lead_full0 + (uint32_t)(r.stage * sizeof(uint64_t));
    if (MAIN) tma_load_2d_pair(sA + r.stage * A_BYTES, mapA, bar, kb * KSTEP, a_row);
    if (EXTRA) tma_load_2d_pair(sT + r.ts * T_BYTES, mapT, bar, kb * KSTEP, t_row);
    tma_load_3d_pair(sB + r.stage * B_BYTES, mapB, bar, kb * KSTEP, b_row0, gz);
    if (MODE == MODE_FC1) tma_load_3d_pair(sB + r.stage * B_BYTES + B_BYTES / 2, mapB, bar, kb * KSTEP, b_row1, gz);
    if (++r.stage == kPairStages) {
      r.stage = 0;
      r.ph ^= 1u;
    }
    if (EXTRA && ++r.ts == kTSlots) {
      r.ts = 0;
      r.tph ^= 1u;
    }
  }
  return true;
}

// The MMAs of one tile (even CTA, one thread): per k-step 4 pair MMAs of M=256 (MAIN)
// and / or 4 of M=128 (EXTRA) on the same weight stage, then the commits that free it.
template <bool F8, bool MAIN, bool EXTRA>
__device__ __forceinline__ bool mma_tile(Rings& r, int num_kb, uint64_t* full, uint64_t* empty, uint64_t* tempty,
                                         const uint8_t* sA, const uint8_t* sT, const uint8_t* sB, uint32_t d_main,
                                         uint32_t d_extra, volatile int* abort_v) {
  constexpr uint32_t IDESC_M = F8 ? idesc_e4m3_f32(PM, PN) : idesc_bf16_f32(PM, PN);
  constexpr uint32_t IDESC_T = F8 ? idesc_e4m3_f32(128, PN) : idesc_bf16_f32(128, PN);
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!mbar_wait_cluster(&full[r.stage], r.ph, abort_v)) return false;
    tc_fence_after();
    const uint32_t a_addr = smem_u32(sA + r.stage * A_BYTES);
    const uint32_t b_addr = smem_u32(sB + r.stage * B_BYTES);
    const uint32_t t_addr = EXTRA ? smem_u32(sT + r.ts * T_BYTES) : 0u;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {  // 32 bytes of k per MMA
      const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
      if (MAIN) {
        if (F8)
          umma_e4m3_pair(d_main, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC_M, acc);
        else
          umma_bf16_pair(d_main, smem_desc_k128(a_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC_M, acc);
      }
      if (EXTRA) {
        if (F8)
          umma_e4m3_pair(d_extra, smem_desc_k128(t_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC_T, acc);
        else
          umma_bf16_pair(d_extra, smem_desc_k128(t_addr + kk * 32), smem_desc_k128(b_addr + kk * 32), IDESC_T, acc);
      }
    }
    umma_commit_pair(&empty[r.stage], 0x3);  // frees this stage in both CTAs
    if (EXTRA) {
      umma_commit_pair(&tempty[r.ts], 0x3);  // and the carried rows' stage
      if (++r.ts == kTSlots) {
        r.ts = 0;
        r.tph ^= 1u;
      }
    }
    if (++r.stage == kPairStages) {
      r.stage = 0;
      r.ph ^= 1u;
    }
  }
  return true;
}

}  // namespace

template <int MODE, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmT0, const __grid_constant__ CUtensorMap tmT1,
                        const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  constexpr uint32_t TMEM_COLS = 2 * PN;  // two buffers of 256 columns
  constexpr int KSTEP = F8 ? 2 * PK : PK;  // elements of k per stage (128-byte rows either way)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kPairStages * A_BYTES;
  uint8_t* sT = sB + kPairStages * B_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sT + kTSlots * T_BYTES);
  uint64_t* empty = full + kPairStages;
  uint64_t* tempty = empty + kPairStages;  // [kTSlots] carried-row stage consumed
  uint64_t* tfull = tempty + kTSlots;      // [2] accumulators of the tile on buffer b complete
  uint64_t* rfree = tfull + 2;             // [4] region 2b (lo) / 2b+1 (hi) drained
  uint64_t* drain = rfree + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);
  int* s_prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + 256);
  int* s_prefc = s_prefix + (kPairGroups + 1);
  int* s_orow = s_prefc + (kPairGroups + 1);
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
    for (int s = 0; s < kTSlots; ++s) mbar_init(&tempty[s], 1);
    for (int b = 0; b < 2; ++b) mbar_init(&tfull[b], 1);  // one pair commit per use
    for (int r = 0; r < 4; ++r) mbar_init(&rfree[r], 8);  // 4 epilogue warps in each CTA
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmT0);
    tma_prefetch_desc(&tmT1);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc_pair(tmem_holder, TMEM_COLS);

  // group table: rows, first output row (the first A row is the output row, or 0 for a
  // shared expert read from the token rows)
  for (int g = threadIdx.x; g < G; g += kPairThreads) {
    int rows, orow;
    const int gg = p.g0 + g;  // global group
    if (gg < p.E) {
      rows = p.n_e[gg];
      orow = p.expert_off[gg];
      // bounds-checked build: a group must lie inside the routed rows
      if (kChecks && (rows < 0 || orow < 0 || (long long)orow + rows > p.A_routed)) {
        report(p.check, MOE_ERR_BAD_INDEX);
        rows = 0;
        orow = 0;
      }
    } else {
      rows = p.N;
      orow = p.A_routed + (gg - p.E) * p.N;
    }
    s_rows[g] = rows;  // valid rows (stores are masked to these)
    s_orow[g] = orow;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefixes of the tiles per weight tile, per phase
    int run = 0, runc = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int fb = 0, ex = 0, cy = 0;
      const int v = g < G ? group_tiles(s_rows[g], &fb, &ex, &cy) : 0;
      int incl = v, inclc = cy;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        const int uc = __shfl_up_sync(0xffffffffu, inclc, o);
        if (lane >= o) {
          incl += u;
          inclc += uc;
        }
      }
      if (g < G) {
        s_prefix[g] = run + incl - v;
        s_prefc[g] = runc + inclc - cy;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
      runc += __shfl_sync(0xffffffffu, inclc, 31);
    }
    if (lane == 0) {
      s_prefix[G] = run;
      s_prefc[G] = runc;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
  tc_fence_after();

  const uint32_t tmem_base = *tmem_holder;
  const int n_tiles = (MODE == MODE_FC1) ? (p.n_out + PN / 2 - 1) / (PN / 2) : (p.n_out + PN - 1) / PN;
  const int total = (s_prefix[G] + s_prefc[G]) * n_tiles;
  const int num_kb = (p.K + KSTEP - 1) / KSTEP;
  const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  volatile int* abort_v = abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t lead_full0 = map_to_rank(smem_u32(&full[0]), 0);
      Rings rg = {0, 0u, 0, 0u};
      bool ok = true;
      for (int t = pair_id; t < total && ok; t += n_pairs) {
        const PairTile td = decode_pair_tile(t, s_prefix, s_prefc, s_rows, G, n_tiles);
        const int g = td.g;
        const int gz = p.g0 + g;  // global group = weight index
        const bool map1 = gz >= p.E && p.shared_from_map1;
        const CUtensorMap* mapA = map1 ? &tmA1 : &tmA0;
        const CUtensorMap* mapT = map1 ? &tmT1 : &tmT0;
        const int arow = map1 ? 0 : s_orow[g];  // first A row of the group
        const int a_row = arow + td.m_blk * PM + (int)rank * 128;
        const int t_row = arow + td.full * PM + (int)rank * 64;
        // B rows this CTA stages: FC1 W_gate rows [n0 + 64r, +64) and the W_up rows of the
        // same outputs (two 64-row boxes); FC2 W_down rows [n0 + 128r, +128) (one box)
        const int b_row0 = (MODE == MODE_FC1) ? td.n_blk * 128 + (int)rank * 64 : td.n_blk * PN + (int)rank * 128;
        const int b_row1 = p.I + b_row0;
        if (td.kind == FULL)
          ok = load_tile<MODE, true, false, KSTEP>(rg, num_kb, full, empty, tempty, lead_full0, leader, sA, sT, sB,
                                                  mapA, mapT, &tmB, a_row, t_row, b_row0, b_row1, gz, abort_v);
        else if (td.kind == CARRY)
          ok = load_tile<MODE, true, true, KSTEP>(rg, num_kb, full, empty, tempty, lead_full0, leader, sA, sT, sB,
                                                 mapA, mapT, &tmB, a_row, t_row, b_row0, b_row1, gz, abort_v);
        else
          ok = load_tile<MODE, false, true, KSTEP>(rg, num_kb, full, empty, tempty, lead_full0, leader, sA, sT, sB,
                                                  mapA, mapT, &tmB, a_row, t_row, b_row0, b_row1, gz, abort_v);
      }
      if (!ok) {
        report(p.status, MOE_ERR_TIMEOUT);
        *abort_v = 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      Rings rg = {0, 0u, 0, 0u};
      uint32_t upar = 0;  // bit r: parity of region r's acquisitions so far
      bool ok = true, any = false;
      int i = 0;  // tiles of this pair so far: buffer = i & 1
      for (int t = pair_id; t < total && ok; t += n_pairs, ++i) {
        const PairTile td = decode_pair_tile(t, s_prefix, s_prefc, s_rows, G, n_tiles);
        const int b = i & 1;
        // regions this tile writes (bit mask): its buffer (both regions, or lo for a short
        // tile) and, for a carrying tile, the hi region of the other buffer
        const uint32_t need = td.kind == SHORT ? (1u << (2 * b))
                                               : ((3u << (2 * b)) | (td.kind == CARRY ? 1u << (2 * (b ^ 1) + 1) : 0u));
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (ok && ((need >> r) & 1u)) {
            if (!mbar_wait_cluster(&rfree[r], ((upar >> r) & 1u) ^ 1u, abort_v)) ok = false;
            upar ^= 1u << r;
          }
        }
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_main = tmem_base + (uint32_t)(b * PN);
        const uint32_t d_extra =
            tmem_base + (uint32_t)(td.kind == CARRY ? (b ^ 1) * PN + PN / 2 : b * PN);
        if (td.kind == FULL)
          ok = mma_tile<F8, true, false>(rg, num_kb, full, empty, tempty, sA, sT, sB, d_main, d_extra, abort_v);
        else if (td.kind == CARRY)
          ok = mma_tile<F8, true, true>(rg, num_kb, full, empty, tempty, sA, sT, sB, d_main, d_extra, abort_v);
        else
          ok = mma_tile<F8, false, true>(rg, num_kb, full, empty, tempty, sA, sT, sB, d_main, d_extra, abort_v);
        any = true;
        if (!ok) break;
        umma_commit_pair(&tfull[b], 0x3);  // accumulators ready in both CTAs
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
    const int lid = quarter * 32 + lane;  // TMEM lane this thread reads
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t rfree_peer0 = map_to_rank(smem_u32(&rfree[0]), rank ^ 1u);
    uint32_t tph = 0;  // bit b: phase of buffer b's accumulator barrier
    int i = 0;
    for (int t = pair_id; t < total; t += n_pairs, ++i) {
      const PairTile td = decode_pair_tile(t, s_prefix, s_prefc, s_rows, G, n_tiles);
      const int b = i & 1;
      const int g = td.g, gz = p.g0 + g;
      const bool ok = __all_sync(0xffffffffu, mbar_wait_cluster(&tfull[b], (tph >> b) & 1u, abort_v));
      tph ^= 1u << b;
      if (!ok) {
        if (lane == 0) {
          report(p.status, MOE_ERR_TIMEOUT);
          *abort_v = 1;
        }
        break;
      }
      tc_fence_after();
      // FP8: the scales the accumulator is multiplied by
      const float* sb = F8 ? p.b_scale + (size_t)gz * p.b_rows : nullptr;
      // output columns of the tile; the two halves of N are the two CTAs' B halves
      const int nb0 = (MODE == MODE_FC1) ? td.n_blk * 128 : td.n_blk * PN;
      constexpr int HALF = (MODE == MODE_FC1) ? 64 : 128;  // outputs per 128-column region
      // the regions to drain, in order (the borrowed one first: the next tile may be
      // waiting for it): TMEM column, row of the group, first output column, region id.
      // Carried / short-tile rows (M=128 accumulator): lane l holds row 64*rank + (l & 63)
      // of the block after the full ones, for the N half l >> 6.
      const int r_extra = td.full * PM + (int)rank * 64 + (lid & 63);
      const int c_extra = nb0 + HALF * (lid >> 6);
      const int r_main = td.m_blk * PM + (int)rank * 128 + lid;
      // slot 0: the borrowed region of a carrying tile; slot 1: hi region (a short tile's
      // lo region); slot 2: lo region of a full or carrying tile
      const bool on[3] = {td.kind == CARRY, true, td.kind != SHORT};
      const uint32_t q_col[3] = {(uint32_t)((b ^ 1) * PN + PN / 2),
                                 (uint32_t)(td.kind == SHORT ? b * PN : b * PN + PN / 2), (uint32_t)(b * PN)};
      const int q_row[3] = {r_extra, td.kind == SHORT ? r_extra : r_main, r_main};
      const int q_c0[3] = {c_extra, td.kind == SHORT ? c_extra : nb0 + HALF, nb0};
      const int q_id[3] = {2 * (b ^ 1) + 1, td.kind == SHORT ? 2 * b : 2 * b + 1, 2 * b};
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        if (on[q]) {
        // drain one 128-column region into row r of the group, outputs from column c0
        // (FC1: 64 gate + 64 up columns -> 64 outputs; FC2: 128 outputs)
        const int r = q_row[q], c0 = q_c0[q];
        const bool row_ok = r < s_rows[g];
        const long long orow = (long long)s_orow[g] + r;
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + orow * p.ldo;
        const uint32_t taddr = tmem_base + lane_off + q_col[q];
        if (MODE == MODE_FC1) {
          float ra = 1.0f;  // FP8: scale of this row's token
          if (F8 && row_ok)
            ra = gz < p.E ? (p.a_scale_rows ? p.a_scale_rows[orow] : token_scale(p, orow))
                          : p.a_scale[(int)(orow - p.A_routed - (long long)(gz - p.E) * p.N)];
#pragma unroll 1
          for (int c = 0; c < 64; c += 32) {
            uint32_t gv[32], uv[32];
            tmem_ld32(taddr + c, gv);
            tmem_ld32(taddr + 64 + c, uv);
            tmem_wait_ld();
            if (F8 && row_ok) {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const int colc = min(c0 + c + e, p.n_out - 1);
                gv[e] = __float_as_uint(__uint_as_float(gv[e]) * ra * __ldg(sb + colc));
                uv[e] = __float_as_uint(__uint_as_float(uv[e]) * ra * __ldg(sb + p.I + colc));
              }
            }
            if (row_ok) {
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                const int colo = c0 + c + e;
                if (colo < p.n_out) {
                  uint32_t w[4];
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    const float h0 = silu_f32(__uint_as_float(gv[e + 2 * u])) * __uint_as_float(uv[e + 2 * u]);
                    const float h1 =
                        silu_f32(__uint_as_float(gv[e + 2 * u + 1])) * __uint_as_float(uv[e + 2 * u + 1]);
                    w[u] = pack_bf16x2(h0, h1);
                  }
                  *reinterpret_cast<uint4*>(dst + colo) = make_uint4(w[0], w[1], w[2], w[3]);
                }
              }
            }
          }
        } else {
          float scale = 1.0f;
          if (row_ok && p.gate_w && gz < p.E) {
            const int gi = p.row2tok ? p.row2tok[orow] : (int)orow;
            scale = check_range(gi, 0, p.A_routed, p.check) ? p.gate_w[gi] : 0.0f;
          }
          if (F8 && row_ok) scale *= p.a_scale[orow];  // FP8: scale of this h row
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            uint32_t v[32];
            tmem_ld32(taddr + c, v);
            tmem_wait_ld();
            if (F8 && row_ok) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                v[e] = __float_as_uint(__uint_as_float(v[e]) * __ldg(sb + min(c0 + c + e, p.n_out - 1)));
            }
            if (row_ok) {
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                const int colo = c0 + c + e;
                if (colo < p.n_out) {
                  uint32_t w[4];
#pragma unroll
                  for (int u = 0; u < 4; ++u)
                    w[u] = pack_bf16x2(__uint_as_float(v[e + 2 * u]) * scale,
                                       __uint_as_float(v[e + 2 * u + 1]) * scale);
                  *reinterpret_cast<uint4*>(dst + colo) = make_uint4(w[0], w[1], w[2], w[3]);
                }
              }
            }
          }
        }
        // this warp is done with the region: release it on its own and the peer's barrier
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rfree[q_id[q]]);
          mbar_arrive_cluster(rfree_peer0 + (uint32_t)(q_id[q] * sizeof(uint64_t)));
        }
        }
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
  CUtensorMap a0, a1, t0, t1, b;
  const bool f8 = g.fp8 != 0;
  const int bk = f8 ? 2 * PK : PK;
  const void* a1p = g.a1 ? g.a1 : g.a0;
  const int a1r = g.a1 ? a1_rows : a0_rows;
  if (!make_map_a(&a0, g.a0, a0_rows, g.K, bk, f8, 128)) return cudaErrorInvalidValue;
  if (!make_map_a(&a1, a1p, a1r, g.K, bk, f8, 128)) return cudaErrorInvalidValue;
  if (!make_map_a(&t0, g.a0, a0_rows, g.K, bk, f8, 64)) return cudaErrorInvalidValue;
  if (!make_map_a(&t1, a1p, a1r, g.K, bk, f8, 64)) return cudaErrorInvalidValue;
  // B boxes: FC1 stages 64 gate + 64 up rows per CTA, FC2 128 rows
  if (!make_map_b(&b, g.b, g.g0 + g.G, g.b_rows, g.K, g.mode == MODE_FC1 ? 64 : 128, bk, f8))
    return cudaErrorInvalidValue;
  const long long rows_total = launch_rows(g);
  const long long m_tiles = (rows_total + 128 + PM - 1) / PM + g.G;
  const long long n_tiles = g.mode == MODE_FC1 ? (g.n_out + PN / 2 - 1) / (PN / 2) : (g.n_out + PN - 1) / PN;
  long long grid = (sm_count() / 2) * 2;
  if (g.max_ctas > 0 && g.max_ctas < grid) grid = (g.max_ctas / 2) * 2;
  if (2 * m_tiles * n_tiles < grid) grid = 2 * m_tiles * n_tiles;
  if (grid < 2) grid = 2;
  auto run = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)grid, kPairThreads, kPairSmem, st>>>(a0, a1, t0, t1, b, g);
    return cudaGetLastError();
  };
  if (g.mode == MODE_FC1) return f8 ? run(tc_gemm_pair_kernel<MODE_FC1, true>) : run(tc_gemm_pair_kernel<MODE_FC1, false>);
  return f8 ? run(tc_gemm_pair_kernel<MODE_FC2, true>) : run(tc_gemm_pair_kernel<MODE_FC2, false>);
}

}  // namespace moe
