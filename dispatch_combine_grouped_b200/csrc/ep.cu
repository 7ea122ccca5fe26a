// Expert parallelism across GPUs: the dispatch and combine all-to-all over peer memory,
// one rank per GPU, P ranks = P expert owners.
//
// What is computed follows the ep_deepep explainer (§2 the expert-parallel layer, §3 each
// source buckets its tokens by owner and the combine returns the rows to the source),
// the DeepEP notes (§2: a count exchange first, then the all-to-all as a transpose in
// which owner j receives the blocks 0->j, 1->j, ... in source order) and the Wide EP page
// (the count matrix C_ij, R_j = sum_i C_ij).  Rank r's receive rows are exactly rows
// [recv_off[r], recv_off[r+1]) of the one-GPU layout whose virtual sources are the ranks:
// expert-major in ascending id, and inside an expert by source rank, then by assignment.
//
// How (B200): no staging buffer and no library collective on the data path.
//   counts   each rank stores its per-expert counts into row r of every rank's count
//            table (peer stores), then publishes the step's epoch with a release store
//   layout   after acquiring all P rows, every rank knows where each of its assignments
//            lands: owner o, row  off_o(e) + sum_{i<r} cnt[i][e] + (rank of the
//            assignment among r's own assignments to e)
//   dispatch the permute kernel with remote destinations: each token row is read once
//            and stored straight into the owners' receive rows over NVLink, with its gate;
//            the last CTA to finish publishes the epoch to every owner
//   combine  the gather-and-sum kernel with remote sources: the owners' output rows are
//            loaded over NVLink and summed in slot order in fp32
// Flags hold epochs: each rank counts its steps in its own window (the notify kernel
// increments the count, later kernels of the step read it), so the epoch is never a
// launch argument and a captured CUDA graph replays correctly.  Flags only grow, so
// nothing is reset between steps.  Every wait is bounded (MOE_WAIT_LIMIT_NS) and
// reports MOE_ERR_TIMEOUT.  A failed wait also fails the step on every rank: the rank
// records the step in its window (err_step), and the flags it publishes later in that
// step (its dispatch to the owners, its "done" to the sources) carry an error mark (the
// top bit) beside the epoch; a wait that finds the mark for its epoch reports
// MOE_ERR_TIMEOUT and fails the step there too, so no combine sums rows of an owner
// whose inputs did not all arrive.  The mark is tied to its epoch: the next step's flags
// are plain again.
// No TMA and no multicast touches peer memory: peer traffic is plain 16-byte loads and
// stores.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kEpWarps = 8;
constexpr int kEpUnroll = 4;

__device__ __forceinline__ void st_release_sys(uint64_t* p, uint64_t v) {
  asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_acquire_sys(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Error mark on a published flag: the epoch's step failed on the publishing rank.
constexpr uint64_t kEpErr = 1ull << 63;

// One thread: wait until flags[0..n) all hold at least epoch (error marks aside).  Gives
// up after MOE_WAIT_LIMIT_NS (or 2^32 polls), reports MOE_ERR_TIMEOUT and returns false;
// also returns false with MOE_ERR_TIMEOUT when a flag carries the error mark of this
// epoch (a wait failed on the rank that published it).
__device__ bool wait_epochs(const uint64_t* flags, int n, uint64_t epoch, int* status) {
  const uint64_t t0 = global_timer_ns();
  uint64_t polls = 0;
  bool ok = true;
  for (int i = 0; i < n; ++i) {
    uint64_t v;
    while (((v = ld_acquire_sys(flags + i)) & ~kEpErr) < epoch) {
      if ((++polls & 31u) == 0u && (global_timer_ns() - t0 > MOE_WAIT_LIMIT_NS || polls > 0xffffffffull)) {
        report(status, MOE_ERR_TIMEOUT);
        return false;
      }
      __nanosleep(64);
    }
    if (v == (epoch | kEpErr)) ok = false;
  }
  if (!ok) report(status, MOE_ERR_TIMEOUT);
  return ok;
}

template <typename T>
__device__ __forceinline__ T* at(const char* base, size_t off) {
  return reinterpret_cast<T*>(const_cast<char*>(base) + off);
}

// This rank's current step (written by an earlier kernel on the same stream).
__device__ __forceinline__ uint64_t step_of(const char* own, const EpOffsets& off) {
  return *reinterpret_cast<const volatile uint64_t*>(own + off.step);
}

// The running step failed on this rank (a wait of one of its kernels gave up or met an
// error mark); later kernels of the step, on the same stream, see it.
__device__ __forceinline__ void fail_step(const char* own, const EpOffsets& off) {
  *reinterpret_cast<volatile uint64_t*>(const_cast<char*>(own) + off.err_step) = step_of(own, off);
}
__device__ __forceinline__ bool step_failed(const char* own, const EpOffsets& off) {
  return *reinterpret_cast<const volatile uint64_t*>(own + off.err_step) == step_of(own, off);
}
// The value this rank publishes for the running step: its epoch, marked if it failed.
__device__ __forceinline__ uint64_t published_epoch(const char* own, const EpOffsets& off) {
  return step_of(own, off) | (step_failed(own, off) ? kEpErr : 0ull);
}

// ---------------------------------------------------------------- count exchange
// Row `me` of every rank's count table = this rank's per-expert counts n_loc[E].
__global__ void ep_push_counts_kernel(const __grid_constant__ EpPeers peers, EpOffsets off,
                                      const int32_t* __restrict__ n_loc, int E, int P, int me) {
  for (int p = 0; p < P; ++p) {
    int32_t* row = at<int32_t>(peers.base[p], off.cnt_tab) + (size_t)me * E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) row[e] = n_loc[e];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t* step = at<uint64_t>(peers.base[me], off.step);
    const uint64_t epoch = *step + 1;  // this step
    *step = epoch;
    __threadfence_system();
    for (int p = 0; p < P; ++p) st_release_sys(at<uint64_t>(peers.base[p], off.cnt_flag) + me, epoch);
  }
}

// ---------------------------------------------------------------- layout
struct EpLayoutArgs {
  const int32_t* ids;         // [A] this rank's assignments
  const int32_t* tok2row;     // [A] local layout: row in the local expert-sorted order
  const int32_t* eoff;        // [E+1] local layout: expert offsets
  const int32_t* owner;       // [E] or NULL (contiguous, per_owner experts each)
  int E, P, me, A, capacity, local_experts, per_owner;
  const char* win;            // this rank's window
  EpOffsets off;
  int32_t* dest;              // [A] owner * capacity + row, -1 = no row
  int32_t* own_n_e;           // [local_experts]
  int32_t* own_off;           // [local_experts + 1]
  int* status;
};

constexpr int kEpLayoutThreads = 512;

__global__ void __launch_bounds__(kEpLayoutThreads) ep_layout_kernel(EpLayoutArgs a) {
  __shared__ int s_ok;
  __shared__ int n_tot[kMaxSlots];   // sum over sources of cnt[i][e]
  __shared__ int e_off[kMaxSlots];   // first row of expert e in its owner's receive rows
  __shared__ int base[kMaxSlots];    // first row of this source's block of expert e
  __shared__ int own_of[kMaxSlots];
  __shared__ int R[kMaxP];
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_ok = wait_epochs(at<uint64_t>(a.win, a.off.cnt_flag), a.P, step_of(a.win, a.off), a.status);
    if (!s_ok) fail_step(a.win, a.off);
  }
  __syncthreads();
  const int32_t* cnt = at<int32_t>(a.win, a.off.cnt_tab);
  for (int e = tid; e < a.E; e += blockDim.x) {
    int o = a.owner ? a.owner[e] : e / a.per_owner;
    if (o < 0 || o >= a.P) {
      report(a.status, MOE_ERR_BAD_INDEX);
      o = 0;
    }
    own_of[e] = o;
    int n = 0, before = 0;
    if (s_ok) {
      for (int i = 0; i < a.P; ++i) {
        const int c = cnt[(size_t)i * a.E + e];
        n += c;
        if (i < a.me) before += c;
      }
    }
    n_tot[e] = n;
    base[e] = before;
  }
  __syncthreads();
  for (int e = tid; e < a.E; e += blockDim.x) {
    const int o = own_of[e];
    int s = 0;
    for (int q = 0; q < e; ++q) s += own_of[q] == o ? n_tot[q] : 0;
    e_off[e] = s;
    base[e] += s;
  }
  for (int o = tid; o < a.P; o += blockDim.x) {
    int s = 0;
    for (int e = 0; e < a.E; ++e) s += own_of[e] == o ? n_tot[e] : 0;
    R[o] = s;
    if (s > a.capacity && blockIdx.x == 0) report(a.status, MOE_ERR_WORKSPACE);
  }
  __syncthreads();
  // destinations of this rank's assignments
  for (int i = blockIdx.x * blockDim.x + tid; i < a.A; i += gridDim.x * blockDim.x) {
    int e = a.ids[i];
    const int r = a.tok2row[i];
    int d = -1;
    if (s_ok && e != -1 && r >= 0) {
      if (e < 0 || e >= a.E) e = 0;  // the local layout counted a bad id as expert 0 (and reported it)
      const int row = base[e] + (r - a.eoff[e]);
      d = row < a.capacity ? own_of[e] * a.capacity + row : -1;
    }
    a.dest[i] = d;
  }
  if (blockIdx.x != 0) return;
  // this owner's experts, in ascending id: rows and first row (capped at capacity)
  for (int e = tid; e < a.E; e += blockDim.x) {
    if (own_of[e] != a.me) continue;
    int q = 0;
    for (int p = 0; p < e; ++p) q += own_of[p] == a.me;
    if (q >= a.local_experts) {
      report(a.status, MOE_ERR_INVALID_ARG);
      continue;
    }
    const int first = min(e_off[e], a.capacity);
    a.own_off[q] = first;
    a.own_n_e[q] = min(n_tot[e], a.capacity - first);
  }
  if (tid == 0) {
    int owned = 0;
    for (int e = 0; e < a.E; ++e) owned += own_of[e] == a.me;
    if (owned != a.local_experts) report(a.status, MOE_ERR_INVALID_ARG);
    const int rows = min(R[a.me], a.capacity);
    for (int q = owned; q < a.local_experts; ++q) {
      a.own_off[q] = rows;
      a.own_n_e[q] = 0;
    }
    a.own_off[a.local_experts] = rows;
  }
}

// ---------------------------------------------------------------- dispatch
__device__ __forceinline__ uint4 ld_nc(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Each token row of x is read once and stored into the receive rows of the owners of its
// k experts; the gate of each assignment (and, for an FP8 payload, the token's scale)
// goes beside its row.  Grid-stride over tokens.
__global__ void __launch_bounds__(kEpWarps * 32) ep_dispatch_kernel(const __grid_constant__ EpPeers peers,
                                                                     EpOffsets off, const uint4* __restrict__ x,
                                                                     const int32_t* __restrict__ dest,
                                                                     const float* __restrict__ topk_w,
                                                                     const float* __restrict__ x_scale, int N,
                                                                     int k, int vpr, int capacity, int P,
                                                                     int me, int* check,
                                                                     const uint4* __restrict__ x2, int vpr2) {
  const int lane = threadIdx.x & 31;
  for (int t = blockIdx.x * kEpWarps + (threadIdx.x >> 5); t < N; t += gridDim.x * kEpWarps) {
    int my = lane < k ? dest[(size_t)t * k + lane] : -1;
    if (!check_range(my, -1, (long long)P * capacity, check)) my = -1;  // bounds-checked build
    if (my >= 0) {
      const int o = my / capacity;
      at<float>(peers.base[o], off.gate)[my - o * capacity] = topk_w[(size_t)t * k + lane];
      if (x_scale) at<float>(peers.base[o], off.scale)[my - o * capacity] = x_scale[t];
    }
    uint4* rows[kMaxK];
    uint4* srows[kMaxK];  // MX scale rows: [capacity, vpr2] vectors after [capacity, vpr] of codes
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      const int d = __shfl_sync(0xffffffffu, my, j);
      rows[j] = nullptr;
      srows[j] = nullptr;
      if (j < k && d >= 0) {
        const int o = d / capacity;
        rows[j] = at<uint4>(peers.base[o], off.x_recv) + (size_t)(d - o * capacity) * vpr;
        if (x2) srows[j] = at<uint4>(peers.base[o], off.x_recv) + (size_t)capacity * vpr + (size_t)(d - o * capacity) * vpr2;
      }
    }
    const uint4* s = x + (size_t)t * vpr;
    for (int v0 = 0; v0 < vpr; v0 += 32 * kEpUnroll) {
      uint4 buf[kEpUnroll];
#pragma unroll
      for (int u = 0; u < kEpUnroll; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vpr) buf[u] = ld_nc(s + v);
      }
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        if (rows[j] == nullptr) continue;
#pragma unroll
        for (int u = 0; u < kEpUnroll; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < vpr) rows[j][v] = buf[u];
        }
      }
    }
    if (x2 && lane < vpr2) {  // MX: the token's scale row (vpr2 <= 32 vectors) to the same
                              // receive rows of the scale region, which follows the codes
      const uint4 u = ld_nc(x2 + (size_t)t * vpr2 + lane);
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (srows[j] != nullptr) srows[j][lane] = u;
    }
  }
  // The last CTA to finish publishes this source's epoch to every owner.  Each CTA
  // fences its stores at system scope before counting itself, and the last one fences
  // again after reading the count, so its release store covers every CTA's rows.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence_system();
    uint32_t* ctr = at<uint32_t>(peers.base[me], off.disp_ctr);
    if (atomicAdd(ctr, 1u) == gridDim.x - 1) {
      *ctr = 0;  // ready for the next launch, which is stream-ordered after this one
      const uint64_t epoch = published_epoch(peers.base[me], off);
      __threadfence_system();
      for (int p = 0; p < P; ++p) st_release_sys(at<uint64_t>(peers.base[p], off.disp_flag) + me, epoch);
    }
  }
}

// ---------------------------------------------------------------- waits and signals
__global__ void ep_wait_kernel(const char* own, EpOffsets off, size_t flag_off, int n, int* status) {
  if (threadIdx.x == 0 && !wait_epochs(at<uint64_t>(own, flag_off), n, step_of(own, off), status))
    fail_step(own, off);
}

// flag[me] = epoch in every rank's window (with the error mark if the step failed on this
// rank), after everything before this launch on the stream
__global__ void ep_signal_kernel(const __grid_constant__ EpPeers peers, EpOffsets off, size_t flag_off, int P,
                                 int me) {
  if (threadIdx.x != 0) return;
  const uint64_t epoch = published_epoch(peers.base[me], off);
  __threadfence_system();
  for (int p = 0; p < P; ++p) st_release_sys(at<uint64_t>(peers.base[p], flag_off) + me, epoch);
}

// ---------------------------------------------------------------- combine
__device__ __forceinline__ uint4 ld_peer(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <typename T>
struct EpVec;
template <>
struct EpVec<float> {
  static constexpr int n = 4;
  __device__ static void add(const uint4& q, float (&f)[8]) {
    f[0] += __uint_as_float(q.x);
    f[1] += __uint_as_float(q.y);
    f[2] += __uint_as_float(q.z);
    f[3] += __uint_as_float(q.w);
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};
template <>
struct EpVec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void add(const uint4& q, float (&f)[8]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] += __uint_as_float(w[i] << 16);
      f[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
  }
};

// y_t = sum_{j<k} out_owner(t,j)[row(t,j)] + sum_{s<S} shared_s[t]: the routed rows (gate
// already applied by FC2) are loaded from their owners' windows, the shared rows from this
// rank's own; fp32 in exactly this order, one rounding.  A warp handles one (token, 32
// vectors) item, with the k (+S) loads of a lane in flight together.
template <typename T>
__global__ void __launch_bounds__(kEpWarps * 32) ep_combine_kernel(const __grid_constant__ EpPeers peers,
                                                                    EpOffsets off, const int32_t* __restrict__ dest,
                                                                    uint4* __restrict__ y, int N, int k, int S,
                                                                    int vpr, int capacity, int P, int me,
                                                                    int* status, int* check) {
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    const char* own = peers.base[me];
    s_ok = wait_epochs(at<uint64_t>(own, off.done_flag), P, step_of(own, off), status);
    if (s_ok && step_failed(own, off)) {  // an earlier wait of this rank's step gave up
      report(status, MOE_ERR_TIMEOUT);
      s_ok = 0;
    }
    if (!s_ok) fail_step(own, off);
  }
  __syncthreads();
  if (!s_ok) return;  // y is not written
  const int lane = threadIdx.x & 31;
  const int chunks = (vpr + 31) / 32;
  const uint4* shared = at<uint4>(peers.base[me], off.out_recv) + (size_t)capacity * vpr;
  for (long long item = (long long)blockIdx.x * kEpWarps + (threadIdx.x >> 5); item < (long long)N * chunks;
       item += (long long)gridDim.x * kEpWarps) {
    const int t = (int)(item / chunks);
    const int v = (int)(item - (long long)t * chunks) * 32 + lane;
    int my = lane < k ? dest[(size_t)t * k + lane] : -1;
    if (!check_range(my, -1, (long long)P * capacity, check)) my = -1;  // bounds-checked build
    int rows[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) rows[j] = __shfl_sync(0xffffffffu, my, j);
    if (v >= vpr) continue;
    uint4 q[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k && rows[j] >= 0) {
        const int o = rows[j] / capacity;
        q[j] = ld_peer(at<uint4>(peers.base[o], off.out_recv) + (size_t)(rows[j] - o * capacity) * vpr + v);
      }
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k && rows[j] >= 0) EpVec<T>::add(q[j], acc);
    for (int s = 0; s < S; ++s) EpVec<T>::add(shared[((size_t)s * N + t) * vpr + v], acc);
    y[(size_t)t * vpr + v] = EpVec<T>::pack(acc);
  }
}

// ---------------------------------------------------------------- host side
static inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

EpOffsets ep_offsets(const moe_config& c, int capacity) {
  const size_t eb = c.dtype == MOE_BF16 ? 2 : 4;
  EpOffsets o;
  o.cnt_flag = 0;
  o.disp_flag = o.cnt_flag + kMaxP * sizeof(uint64_t);
  o.done_flag = o.disp_flag + kMaxP * sizeof(uint64_t);
  o.step = o.done_flag + kMaxP * sizeof(uint64_t);
  o.disp_ctr = o.step + sizeof(uint64_t);
  o.err_step = o.disp_ctr + sizeof(uint64_t);
  o.cnt_tab = al256(o.err_step + sizeof(uint64_t));
  o.gate = al256(o.cnt_tab + (size_t)c.P * c.E * sizeof(int32_t));
  o.scale = al256(o.gate + (size_t)capacity * sizeof(float));
  o.x_recv = al256(o.scale + (size_t)capacity * sizeof(float));
  o.out_recv = al256(o.x_recv + (size_t)capacity * c.d * eb);
  o.total = al256(o.out_recv + ((size_t)capacity + (size_t)c.n_shared * c.N) * c.d * eb);
  return o;
}

static inline unsigned ep_grid(long long items, int per_cta) {
  const long long cap = 8LL * sm_count();
  long long g = (items + per_cta - 1) / per_cta;
  if (g > cap) g = cap;
  return (unsigned)(g < 1 ? 1 : g);
}

cudaError_t launch_ep_push_counts(const EpPeers& peers, const EpOffsets& off, const int32_t* n_loc, int E, int P,
                                  int me, cudaStream_t st) {
  ep_push_counts_kernel<<<1, 256, 0, st>>>(peers, off, n_loc, E, P, me);
  return cudaGetLastError();
}

cudaError_t launch_ep_layout(const moe_config& c, const EpPeers& peers, const EpOffsets& off, int me, int capacity,
                             int local_experts, const int32_t* owner, const int32_t* ids, const moe_layout& loc,
                             int32_t* dest, int32_t* own_n_e, int32_t* own_off, int* status, cudaStream_t st) {
  EpLayoutArgs a;
  a.ids = ids;
  a.tok2row = loc.tok2row;
  a.eoff = loc.expert_off;
  a.owner = owner;
  a.E = c.E;
  a.P = c.P;
  a.me = me;
  a.A = c.N * c.k;
  a.capacity = capacity;
  a.local_experts = local_experts;
  a.per_owner = c.E / c.P > 0 ? c.E / c.P : 1;
  a.win = peers.base[me];
  a.off = off;
  a.dest = dest;
  a.own_n_e = own_n_e;
  a.own_off = own_off;
  a.status = status;
  ep_layout_kernel<<<ep_grid(a.A, kEpLayoutThreads), kEpLayoutThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const moe_config& c, const EpPeers& peers, const EpOffsets& off, int me,
                               int capacity, const void* x, const int32_t* dest, const float* topk_w,
                               const float* x_scale, int row_bytes, cudaStream_t st, const void* x2, int row_bytes2) {
  if (x2 && (row_bytes2 % 16 != 0 || row_bytes2 > 32 * 16)) return cudaErrorInvalidValue;
  ep_dispatch_kernel<<<ep_grid(c.N, kEpWarps), kEpWarps * 32, 0, st>>>(
      peers, off, static_cast<const uint4*>(x), dest, topk_w, x_scale, c.N, c.k, row_bytes / 16, capacity, c.P, me,
      check_word(), static_cast<const uint4*>(x2), x2 ? row_bytes2 / 16 : 0);
  return cudaGetLastError();
}

cudaError_t launch_ep_wait(const char* own, const EpOffsets& off, size_t flag_off, int n, int* status,
                           cudaStream_t st) {
  ep_wait_kernel<<<1, 32, 0, st>>>(own, off, flag_off, n, status);
  return cudaGetLastError();
}

cudaError_t launch_ep_signal(const EpPeers& peers, const EpOffsets& off, size_t flag_off, int P, int me,
                             cudaStream_t st) {
  ep_signal_kernel<<<1, 32, 0, st>>>(peers, off, flag_off, P, me);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const moe_config& c, const EpPeers& peers, const EpOffsets& off, int me, int capacity,
                              const int32_t* dest, void* y, int* status, cudaStream_t st) {
  const int vpr = c.d * (c.dtype == MOE_BF16 ? 2 : 4) / 16;
  const long long items = (long long)c.N * ((vpr + 31) / 32);
  const unsigned grid = ep_grid(items, kEpWarps);
  if (c.dtype == MOE_BF16)
    ep_combine_kernel<__nv_bfloat16><<<grid, kEpWarps * 32, 0, st>>>(
        peers, off, dest, static_cast<uint4*>(y), c.N, c.k, c.n_shared, vpr, capacity, c.P, me, status,
        check_word());
  else
    ep_combine_kernel<float><<<grid, kEpWarps * 32, 0, st>>>(
        peers, off, dest, static_cast<uint4*>(y), c.N, c.k, c.n_shared, vpr, capacity, c.P, me, status,
        check_word());
  return cudaGetLastError();
}

}  // namespace moe
