// Dispatch layout: n_e, expert offsets, the P x P count matrix, send/receive offsets and
// the token <-> send slot <-> expert row maps, computed on the device without any host
// synchronisation.
//
// What is computed follows the ep_deepep explainer (§2 n_e, §3 source-side bucketing by
// owner, §6 the three maps), the Wide EP page (count matrix C_ij, R_r = sum_i C_ir) and
// the DeepEP notes §2 (the all-to-all as a transpose: owner j receives blocks 0->j,
// 1->j, ... in source order).
//
// How: a stable counting sort done as three launches over chunks of CH assignments.
//   1. count : per chunk, per-expert / per-owner / per-(source, owner) counts, and each
//              assignment's rank among same-expert and same-owner assignments of the
//              chunk (deterministic: warp match + per-warp counts, in assignment order)
//   2. scan  : one CTA turns the chunk counts into chunk bases, and computes n_e, C,
//              send_off, recv_off, expert_off and tile_off
//   3. maps  : every assignment's row and send slot from bases + ranks; scatter of the
//              five maps
// Ranks come from counts, never from atomic arrival order, so the result is identical
// on every run.  An id of -1 marks a dropped assignment (capacity factor): it is not
// counted, gets no row and no send slot (its tok2row / tok2send are -1), and the unused
// tails [A_kept, A) of row2tok, send2row and ret2tok are -1.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / 32;

struct LayoutWs {
  int32_t* hist_e;   // [nchunks][E]  counts, then exclusive chunk bases
  int32_t* hist_j;   // [nchunks][P]
  int32_t* hist_ij;  // [nchunks][P*P]
  int32_t* rank_e;   // [A]
  int32_t* rank_j;   // [A]
  int32_t* colpre;   // [P*P]  sum_{i' < i} C[i'][j]
};

size_t layout_ws_bytes(int A, int E, int P, int nchunks) {
  size_t n = (size_t)nchunks * (E + P + P * P) + 2 * (size_t)A + (size_t)P * P;
  return n * sizeof(int32_t) + 256;
}

static LayoutWs carve_layout_ws(void* ws, int A, int E, int P, int nchunks) {
  LayoutWs w;
  int32_t* p = reinterpret_cast<int32_t*>(ws);
  w.hist_e = p;  p += (size_t)nchunks * E;
  w.hist_j = p;  p += (size_t)nchunks * P;
  w.hist_ij = p; p += (size_t)nchunks * P * P;
  w.rank_e = p;  p += A;
  w.rank_j = p;  p += A;
  w.colpre = p;
  return w;
}

struct LayoutArgs {
  const int32_t* ids;
  const int32_t* owner;  // NULL = contiguous
  int N, k, A, E, P, S, shard, per_owner;
  int* status;
};

// Expert of assignment a; -1 marks a dropped assignment (capacity), which takes no row.
__device__ __forceinline__ int expert_of(const LayoutArgs& p, int a) {
  int e = p.ids[a];
  if (e == -1) return -1;
  if (e < 0 || e >= p.E) {
    report(p.status, MOE_ERR_BAD_INDEX);
    e = 0;
  }
  return e;
}

__device__ __forceinline__ int owner_of(const LayoutArgs& p, int e) {
  if (p.owner == nullptr) return e / p.per_owner;
  int j = p.owner[e];
  if (j < 0 || j >= p.P) {
    report(p.status, MOE_ERR_BAD_INDEX);
    j = 0;
  }
  return j;
}

__global__ void __launch_bounds__(kLayoutThreads) layout_count_kernel(LayoutArgs p, LayoutWs w) {
  __shared__ int run_e[kMaxSlots];
  __shared__ int run_j[kMaxP];
  __shared__ int wcnt_e[kLayoutWarps][kMaxSlots];
  __shared__ int wcnt_j[kLayoutWarps][kMaxP];
  __shared__ int hist_ij[kMaxP * kMaxP];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int PP = p.P * p.P;
  for (int x = tid; x < p.E; x += kLayoutThreads) {
    run_e[x] = 0;
    for (int q = 0; q < kLayoutWarps; ++q) wcnt_e[q][x] = 0;
  }
  for (int x = tid; x < p.P; x += kLayoutThreads) {
    run_j[x] = 0;
    for (int q = 0; q < kLayoutWarps; ++q) wcnt_j[q][x] = 0;
  }
  for (int x = tid; x < PP; x += kLayoutThreads) hist_ij[x] = 0;
  __syncthreads();

  const int c = blockIdx.x;
  const int a_begin = c * kLayoutChunk;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int r = 0; r < kLayoutChunk / kLayoutThreads; ++r) {
    const int a = a_begin + r * kLayoutThreads + tid;
    int e = -1, j = -1;
    if (a < p.A) {
      e = expert_of(p, a);
      if (e >= 0) j = owner_of(p, e);
    }
    const bool valid = e >= 0;  // in range and not dropped
    const unsigned me = __match_any_sync(0xffffffffu, e);
    const unsigned mj = __match_any_sync(0xffffffffu, j);
    const int lre = __popc(me & lt_mask), lrj = __popc(mj & lt_mask);
    if (valid) {
      if (lre == 0) wcnt_e[warp][e] = __popc(me);
      if (lrj == 0) wcnt_j[warp][j] = __popc(mj);
      const int i = (a / p.k) / p.shard;
      atomicAdd(&hist_ij[i * p.P + j], 1);  // a count: order of arrival does not matter
    }
    __syncthreads();
    if (valid) {
      int oe = run_e[e] + lre, oj = run_j[j] + lrj;
      for (int q = 0; q < warp; ++q) {
        oe += wcnt_e[q][e];
        oj += wcnt_j[q][j];
      }
      w.rank_e[a] = oe;
      w.rank_j[a] = oj;
    }
    __syncthreads();
    for (int x = tid; x < p.E; x += kLayoutThreads) {
      int s = 0;
      for (int q = 0; q < kLayoutWarps; ++q) {
        s += wcnt_e[q][x];
        wcnt_e[q][x] = 0;
      }
      run_e[x] += s;
    }
    for (int x = tid; x < p.P; x += kLayoutThreads) {
      int s = 0;
      for (int q = 0; q < kLayoutWarps; ++q) {
        s += wcnt_j[q][x];
        wcnt_j[q][x] = 0;
      }
      run_j[x] += s;
    }
    __syncthreads();
    if (a_begin + (r + 1) * kLayoutThreads >= p.A) break;  // uniform across the CTA
  }
  for (int x = tid; x < p.E; x += kLayoutThreads) w.hist_e[(size_t)c * p.E + x] = run_e[x];
  for (int x = tid; x < p.P; x += kLayoutThreads) w.hist_j[(size_t)c * p.P + x] = run_j[x];
  for (int x = tid; x < PP; x += kLayoutThreads) w.hist_ij[(size_t)c * PP + x] = hist_ij[x];
}

// Exclusive scan of one int per thread over a CTA of blockDim.x (multiple of 32) threads.
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  __syncthreads();
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nw ? warp_sums[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      int u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    warp_sums[lane] = s;  // inclusive scan of the warp sums
  }
  __syncthreads();
  const int base = warp > 0 ? warp_sums[warp - 1] : 0;
  if (total) *total = warp_sums[nw - 1];
  return base + incl - v;
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) layout_scan_kernel(LayoutArgs p, LayoutWs w, moe_layout L,
                                                                   int nchunks) {
  __shared__ int s_ne[kMaxSlots];
  __shared__ int s_C[kMaxP * kMaxP];
  __shared__ int s_recv[kMaxP + 1];
  const int tid = threadIdx.x;
  const int PP = p.P * p.P;

  // per-expert and per-owner chunk bases (in place), totals
  // column scans over chunks; loads are batched so that 8 are in flight at a time
  constexpr int B = 8;
  if (tid < p.E) {
    int s = 0;
    for (int c0 = 0; c0 < nchunks; c0 += B) {
      int v[B];
#pragma unroll
      for (int u = 0; u < B; ++u) v[u] = c0 + u < nchunks ? w.hist_e[(size_t)(c0 + u) * p.E + tid] : 0;
#pragma unroll
      for (int u = 0; u < B; ++u) {
        if (c0 + u < nchunks) w.hist_e[(size_t)(c0 + u) * p.E + tid] = s;
        s += v[u];
      }
    }
    s_ne[tid] = s;
    L.n_e[tid] = s;
  } else if (tid >= 512 && tid < 512 + p.P) {
    const int j = tid - 512;
    int s = 0;
    for (int c0 = 0; c0 < nchunks; c0 += B) {
      int v[B];
#pragma unroll
      for (int u = 0; u < B; ++u) v[u] = c0 + u < nchunks ? w.hist_j[(size_t)(c0 + u) * p.P + j] : 0;
#pragma unroll
      for (int u = 0; u < B; ++u) {
        if (c0 + u < nchunks) w.hist_j[(size_t)(c0 + u) * p.P + j] = s;
        s += v[u];
      }
    }
  }
  for (int x = tid; x < PP; x += kScanThreads) {
    int s = 0;
    for (int c0 = 0; c0 < nchunks; c0 += B) {
      int v[B];
#pragma unroll
      for (int u = 0; u < B; ++u) v[u] = c0 + u < nchunks ? w.hist_ij[(size_t)(c0 + u) * PP + x] : 0;
#pragma unroll
      for (int u = 0; u < B; ++u) s += v[u];
    }
    s_C[x] = s;
    L.C[x] = s;
  }
  __syncthreads();

  // send_off: exclusive scan of C in (source, owner) order
  {
    int v = tid < PP ? s_C[tid] : 0;
    int ex = block_exclusive_scan(v, nullptr);
    if (tid < PP) L.send_off[tid] = ex;
  }
  // colpre[i][j] = sum_{i' < i} C[i'][j];  R_j = column sums
  if (tid < p.P) {
    int s = 0;
    for (int i = 0; i < p.P; ++i) {
      w.colpre[i * p.P + tid] = s;
      s += s_C[i * p.P + tid];
    }
    s_recv[tid] = s;
  }
  __syncthreads();
  if (tid == 0) {
    int s = 0;
    for (int j = 0; j < p.P; ++j) {
      int r = s_recv[j];
      s_recv[j] = s;
      s += r;
    }
    s_recv[p.P] = s;
  }
  __syncthreads();
  if (tid <= p.P) L.recv_off[tid] = s_recv[tid];

  // expert_off: owners in order, experts in id order inside an owner
  if (p.owner == nullptr) {
    int v = tid < p.E ? s_ne[tid] : 0;
    int ex = block_exclusive_scan(v, nullptr);
    if (tid < p.E) L.expert_off[tid] = ex;
  } else {
    __shared__ int s_own[kMaxSlots];
    if (tid < p.E) s_own[tid] = owner_of(p, tid);
    __syncthreads();
    if (tid < p.E) {
      const int j = s_own[tid];
      int s = s_recv[j];
      for (int e2 = 0; e2 < tid; ++e2)
        if (s_own[e2] == j) s += s_ne[e2];
      L.expert_off[tid] = s;
    }
  }
  if (tid == 0) L.expert_off[p.E] = s_recv[p.P];  // rows in use (A minus dropped)

  // tile_off: prefix of ceil(rows / 128) over routed experts then shared groups
  {
    const int G = p.E + p.S;
    int v = 0;
    if (tid < p.E) v = (s_ne[tid] + kTileRows - 1) / kTileRows;
    else if (tid < G) v = (p.N + kTileRows - 1) / kTileRows;
    int total = 0;
    int ex = block_exclusive_scan(v, &total);
    if (tid < G) L.tile_off[tid] = ex;
    if (tid == 0) L.tile_off[G] = total;
  }
}

__global__ void layout_maps_kernel(LayoutArgs p, LayoutWs w, moe_layout L) {
  const int a = blockIdx.x * blockDim.x + threadIdx.x;
  if (a >= p.A) return;
  // rows and send slots past the ones in use (dropped assignments) are marked -1
  if (a >= L.recv_off[p.P]) {
    L.row2tok[a] = -1;
    L.ret2tok[a] = -1;
    L.send2row[a] = -1;
  }
  const int e = expert_of(p, a);
  if (e < 0) {
    L.tok2send[a] = -1;
    L.tok2row[a] = -1;
    return;
  }
  const int j = owner_of(p, e);
  const int c = a / kLayoutChunk;
  const int i = (a / p.k) / p.shard;
  const int row = L.expert_off[e] + w.hist_e[(size_t)c * p.E + e] + w.rank_e[a];
  const int gj = w.hist_j[(size_t)c * p.P + j] + w.rank_j[a];
  const int s = L.send_off[i * p.P + j] + gj - w.colpre[i * p.P + j];
  L.tok2send[a] = s;
  L.ret2tok[s] = a;
  L.tok2row[a] = row;
  L.row2tok[row] = a;
  L.send2row[s] = row;
}

cudaError_t launch_layout(const moe_config& cfg, const int32_t* owner, const int32_t* ids, const moe_layout& L,
                          int32_t* status, void* ws, cudaStream_t st) {
  const int A = cfg.N * cfg.k;
  const int nchunks = A > 0 ? (A + kLayoutChunk - 1) / kLayoutChunk : 0;
  LayoutWs w = carve_layout_ws(ws, A, cfg.E, cfg.P, nchunks);
  LayoutArgs p;
  p.ids = ids;
  p.owner = owner;
  p.N = cfg.N;
  p.k = cfg.k;
  p.A = A;
  p.E = cfg.E;
  p.P = cfg.P;
  p.S = cfg.n_shared;
  p.shard = cfg.N > 0 ? (cfg.N + cfg.P - 1) / cfg.P : 1;
  p.per_owner = cfg.E / cfg.P > 0 ? cfg.E / cfg.P : 1;
  p.status = status;
  if (nchunks > 0) layout_count_kernel<<<nchunks, kLayoutThreads, 0, st>>>(p, w);
  layout_scan_kernel<<<1, kScanThreads, 0, st>>>(p, w, L, nchunks);
  if (A > 0) layout_maps_kernel<<<(A + 255) / 256, 256, 0, st>>>(p, w, L);
  return cudaGetLastError();
}

}  // namespace moe
