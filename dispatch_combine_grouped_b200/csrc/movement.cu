// Token movement: permute (dispatch) and combine, plus their two-hop "staged" forms.
//
// "MoE我们喜欢你（四）" §4 gives the pipeline permute_by_expert -> a2a dispatch ->
// grouped_gemm -> a2a combine -> unpermute_and_weighted_sum; the ep_deepep explainer §3
// says the source buckets by owner and the combine returns rows to the source, where
// they are summed by gate.  On one GPU the all-to-all is a transpose of row blocks, so
// the fused kernels compose it with the permute / unpermute through the layout maps;
// the staged kernels materialise the send (or return) buffer in between.
//
// All kernels: one warp per row (or token), 16-byte vectors, rows are d * elem bytes
// (a multiple of 16).  Permute is a bit copy and ignores the dtype.  A map entry of -1
// (a dropped assignment, an unused slot) is skipped: nothing is moved or added for it.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kMoveWarps = 8;   // warps per CTA
constexpr int kMoveUnroll = 4;  // 16-byte vectors in flight per lane per step

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Token-centric scatter: dst[map[t*k + j]] = src[t] for j < k (each source row read once).
__global__ void __launch_bounds__(kMoveWarps * 32) scatter_token_rows(const uint4* __restrict__ src,
                                                                       uint4* __restrict__ dst,
                                                                       const int32_t* __restrict__ map, int N,
                                                                       int k, int vpr, int dst_rows, int* check) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kMoveWarps + (threadIdx.x >> 5);
  if (t >= N) return;
  int my = lane < k ? map[(size_t)t * k + lane] : 0;
  if (!check_range(my, -1, dst_rows, check)) my = -1;  // bounds-checked build: skip a bad row
  int rows[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) rows[j] = __shfl_sync(0xffffffffu, my, j);
  const uint4* s = src + (size_t)t * vpr;
  for (int v0 = 0; v0 < vpr; v0 += 32 * kMoveUnroll) {
    uint4 buf[kMoveUnroll];
#pragma unroll
    for (int u = 0; u < kMoveUnroll; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vpr) buf[u] = ld_stream(s + v);
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k && rows[j] >= 0) {  // a dropped assignment (-1) has no row
        uint4* d = dst + (size_t)rows[j] * vpr;
#pragma unroll
        for (int u = 0; u < kMoveUnroll; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < vpr) d[v] = buf[u];
        }
      }
    }
  }
}

// The same scatter with 32-byte vectors (rows whose size is a multiple of 32 bytes):
// half the load / store instructions of the 16-byte version.
struct alignas(32) V32 {
  uint32_t w[8];
};

__device__ __forceinline__ V32 ld_stream32(const V32* p) {
  V32 r;
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]), "=r"(r.w[5]), "=r"(r.w[6]),
                 "=r"(r.w[7])
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st32(V32* p, const V32& v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v.w[0]), "r"(v.w[1]),
               "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]), "r"(v.w[7])
               : "memory");
}

__global__ void __launch_bounds__(kMoveWarps * 32) scatter_token_rows32(const V32* __restrict__ src,
                                                                         V32* __restrict__ dst,
                                                                         const int32_t* __restrict__ map, int N,
                                                                         int k, int vpr, int dst_rows, int* check) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kMoveWarps + (threadIdx.x >> 5);
  if (t >= N) return;
  int my = lane < k ? map[(size_t)t * k + lane] : 0;
  if (!check_range(my, -1, dst_rows, check)) my = -1;  // bounds-checked build: skip a bad row
  int rows[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) rows[j] = __shfl_sync(0xffffffffu, my, j);
  const V32* s = src + (size_t)t * vpr;
  for (int v0 = 0; v0 < vpr; v0 += 32 * kMoveUnroll) {
    V32 buf[kMoveUnroll];
#pragma unroll
    for (int u = 0; u < kMoveUnroll; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vpr) buf[u] = ld_stream32(s + v);
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k && rows[j] >= 0) {  // a dropped assignment (-1) has no row
        V32* d = dst + (size_t)rows[j] * vpr;
#pragma unroll
        for (int u = 0; u < kMoveUnroll; ++u) {
          const int v = v0 + u * 32 + lane;
          if (v < vpr) st32(d + v, buf[u]);
        }
      }
    }
  }
}

// Row gather: dst[i] = src[map[i]] for i < rows  (map == NULL: dst[map_inv...] not used)
// Row scatter: dst[map[i]] = src[i]
template <bool kScatter>
__global__ void __launch_bounds__(kMoveWarps * 32) move_rows(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                              const int32_t* __restrict__ map, int rows, int vpr,
                                                              int* check) {
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kMoveWarps + (threadIdx.x >> 5);
  if (i >= rows) return;
  const int m = map[i];
  if (m < 0) return;  // an unused slot / a dropped assignment
  if (!check_range(m, 0, rows, check)) return;  // bounds-checked build: skip a bad row
  const uint4* s = src + (size_t)(kScatter ? i : m) * vpr;
  uint4* d = dst + (size_t)(kScatter ? m : i) * vpr;
  for (int v0 = 0; v0 < vpr; v0 += 32 * kMoveUnroll) {
    uint4 buf[kMoveUnroll];
#pragma unroll
    for (int u = 0; u < kMoveUnroll; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vpr) buf[u] = ld_stream(s + v);
    }
#pragma unroll
    for (int u = 0; u < kMoveUnroll; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vpr) d[v] = buf[u];
    }
  }
}

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int n = 4;
  __device__ static void unpack(const uint4& q, float (&f)[8]) {
    f[0] = __uint_as_float(q.x);
    f[1] = __uint_as_float(q.y);
    f[2] = __uint_as_float(q.z);
    f[3] = __uint_as_float(q.w);
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void unpack(const uint4& q, float (&f)[8]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
  }
};

// y_t = sum_{j<k} g_{t,j} * routed[map[t*k+j]] + sum_{s<S} shared[s*N + t], fp32
// accumulation in exactly this order, one rounding.  A warp handles one (token, chunk of
// 64 vectors) item: each lane issues the loads of its 2 vectors for all k (+S) rows
// before using any, so up to 2*(k+S) 16-byte loads per lane are in flight.
constexpr int kCombVec = 2;

template <typename T>
__global__ void __launch_bounds__(kMoveWarps * 32) combine_kernel(const uint4* __restrict__ routed,
                                                                   const uint4* __restrict__ shared,
                                                                   const int32_t* __restrict__ map,
                                                                   const float* __restrict__ gates,
                                                                   uint4* __restrict__ y, int N, int k, int S,
                                                                   int vpr, int* check) {
  const int lane = threadIdx.x & 31;
  const int chunks = (vpr + 32 * kCombVec - 1) / (32 * kCombVec);
  const long long item = (long long)blockIdx.x * kMoveWarps + (threadIdx.x >> 5);
  if (item >= (long long)N * chunks) return;
  const int t = (int)(item / chunks);
  const int v0 = (int)(item - (long long)t * chunks) * 32 * kCombVec + lane;
  int my_row = lane < k ? map[(size_t)t * k + lane] : 0;
  if (!check_range(my_row, -1, (long long)N * k, check)) my_row = -1;  // bounds-checked build
  const float my_g = (lane < k && gates) ? gates[(size_t)t * k + lane] : 1.0f;
  int rows[kMaxK];
  float gs[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    gs[j] = __shfl_sync(0xffffffffu, my_g, j);
  }
  uint4 q[kCombVec][kMaxK];
#pragma unroll
  for (int u = 0; u < kCombVec; ++u) {
    const int v = v0 + u * 32;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k && rows[j] >= 0 && v < vpr) q[u][j] = ld_stream(routed + (size_t)rows[j] * vpr + v);
  }
#pragma unroll
  for (int u = 0; u < kCombVec; ++u) {
    const int v = v0 + u * 32;
    if (v >= vpr) continue;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k && rows[j] >= 0) {  // a dropped assignment adds nothing
        float f[8];
        Vec<T>::unpack(q[u][j], f);
#pragma unroll
        for (int i = 0; i < Vec<T>::n; ++i) acc[i] = fmaf(gs[j], f[i], acc[i]);
      }
    }
    for (int s = 0; s < S; ++s) {
      float f[8];
      Vec<T>::unpack(ld_stream(shared + ((size_t)s * N + t) * vpr + v), f);
#pragma unroll
      for (int i = 0; i < Vec<T>::n; ++i) acc[i] += f[i];
    }
    y[(size_t)t * vpr + v] = Vec<T>::pack(acc);
  }
}

// The combine with 32-byte vectors (rows whose size is a multiple of 32 bytes): one
// vector per lane per item, k (+S) loads in flight per lane; grid-stride over items with
// a grid of a few CTAs per SM (measured 10-16% faster on B200 than one short-lived CTA
// per 8 items).
template <typename T>
__global__ void __launch_bounds__(kMoveWarps * 32) combine_kernel32(const V32* __restrict__ routed,
                                                                     const V32* __restrict__ shared,
                                                                     const int32_t* __restrict__ map,
                                                                     const float* __restrict__ gates,
                                                                     V32* __restrict__ y, int N, int k, int S,
                                                                     int vpr, int* check) {
  const int lane = threadIdx.x & 31;
  const int chunks = (vpr + 31) / 32;
  for (long long item = (long long)blockIdx.x * kMoveWarps + (threadIdx.x >> 5); item < (long long)N * chunks;
       item += (long long)gridDim.x * kMoveWarps) {
    const int t = (int)(item / chunks);
    const int v = (int)(item - (long long)t * chunks) * 32 + lane;
    int my_row = lane < k ? map[(size_t)t * k + lane] : 0;
    if (!check_range(my_row, -1, (long long)N * k, check)) my_row = -1;  // bounds-checked build
    const float my_g = (lane < k && gates) ? gates[(size_t)t * k + lane] : 1.0f;
    int rows[kMaxK];
    float gs[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      rows[j] = __shfl_sync(0xffffffffu, my_row, j);
      gs[j] = __shfl_sync(0xffffffffu, my_g, j);
    }
    if (v >= vpr) continue;
    V32 q[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k && rows[j] >= 0) q[j] = ld_stream32(routed + (size_t)rows[j] * vpr + v);
    constexpr int n = Vec<T>::n;  // elements per 16 bytes
    float acc[2 * 8];
#pragma unroll
    for (int i = 0; i < 2 * n; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k && rows[j] >= 0) {  // a dropped assignment adds nothing
        float f[8];
        Vec<T>::unpack(make_uint4(q[j].w[0], q[j].w[1], q[j].w[2], q[j].w[3]), f);
#pragma unroll
        for (int i = 0; i < n; ++i) acc[i] = fmaf(gs[j], f[i], acc[i]);
        Vec<T>::unpack(make_uint4(q[j].w[4], q[j].w[5], q[j].w[6], q[j].w[7]), f);
#pragma unroll
        for (int i = 0; i < n; ++i) acc[n + i] = fmaf(gs[j], f[i], acc[n + i]);
      }
    }
    for (int s = 0; s < S; ++s) {
      const V32 sv = ld_stream32(shared + ((size_t)s * N + t) * vpr + v);
      float f[8];
      Vec<T>::unpack(make_uint4(sv.w[0], sv.w[1], sv.w[2], sv.w[3]), f);
#pragma unroll
      for (int i = 0; i < n; ++i) acc[i] += f[i];
      Vec<T>::unpack(make_uint4(sv.w[4], sv.w[5], sv.w[6], sv.w[7]), f);
#pragma unroll
      for (int i = 0; i < n; ++i) acc[n + i] += f[i];
    }
    float lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo[i] = i < n ? acc[i] : 0.f;
      hi[i] = i < n ? acc[n + i] : 0.f;
    }
    const uint4 a = Vec<T>::pack(lo), b = Vec<T>::pack(hi);
    V32 o;
    o.w[0] = a.x; o.w[1] = a.y; o.w[2] = a.z; o.w[3] = a.w;
    o.w[4] = b.x; o.w[5] = b.y; o.w[6] = b.z; o.w[7] = b.w;
    st32(y + (size_t)t * vpr + v, o);
  }
}

static inline int elem_bytes(const moe_config& c) { return c.dtype == MOE_BF16 ? 2 : 4; }
static inline int vecs_per_row(const moe_config& c) { return c.d * elem_bytes(c) / 16; }
static inline unsigned blocks_for(long long rows) { return (unsigned)((rows + kMoveWarps - 1) / kMoveWarps); }

// x_perm[tok2row[a]] = x[a / k] for rows of row_bytes bytes (a multiple of 16)
cudaError_t launch_permute_bytes(const moe_config& c, const moe_layout& L, const void* x, void* x_perm,
                                 int row_bytes, cudaStream_t st) {
  if (c.N == 0) return cudaSuccess;
  if (row_bytes % 32 == 0) {
    scatter_token_rows32<<<blocks_for(c.N), kMoveWarps * 32, 0, st>>>(
        static_cast<const V32*>(x), static_cast<V32*>(x_perm), L.tok2row, c.N, c.k, row_bytes / 32, c.N * c.k,
        check_word());
    return cudaGetLastError();
  }
  scatter_token_rows<<<blocks_for(c.N), kMoveWarps * 32, 0, st>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(x_perm), L.tok2row, c.N, c.k, row_bytes / 16, c.N * c.k,
      check_word());
  return cudaGetLastError();
}

cudaError_t launch_permute(const moe_config& c, const moe_layout& L, const void* x, void* x_perm, cudaStream_t st) {
  return launch_permute_bytes(c, L, x, x_perm, c.d * elem_bytes(c), st);
}

cudaError_t launch_permute_staged(const moe_config& c, const moe_layout& L, const void* x, void* send_buf,
                                  void* x_perm, cudaStream_t st) {
  if (c.N == 0) return cudaSuccess;
  const int vpr = vecs_per_row(c);
  const int A = c.N * c.k;
  // hop 1: each source buckets its rows by destination owner (send buffer)
  scatter_token_rows<<<blocks_for(c.N), kMoveWarps * 32, 0, st>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(send_buf), L.tok2send, c.N, c.k, vpr, A, check_word());
  // hop 2: the transpose to the owners plus the expert-local order
  move_rows<true><<<blocks_for(A), kMoveWarps * 32, 0, st>>>(
      static_cast<const uint4*>(send_buf), static_cast<uint4*>(x_perm), L.send2row, A, vpr, check_word());
  return cudaGetLastError();
}

template <typename T>
static void combine_launch(const moe_config& c, const uint4* routed, const uint4* shared, const int32_t* map,
                           const float* gates, uint4* y, cudaStream_t st) {
  const int row_bytes = c.d * elem_bytes(c);
  if (row_bytes % 32 == 0) {
    const int vpr32 = row_bytes / 32;
    const long long items = (long long)c.N * ((vpr32 + 31) / 32);
    const long long nb = blocks_for(items), cap = 4LL * sm_count();  // grid-stride: 4 CTAs per SM
    combine_kernel32<T><<<(unsigned)(nb < cap ? nb : cap), kMoveWarps * 32, 0, st>>>(
        reinterpret_cast<const V32*>(routed), reinterpret_cast<const V32*>(shared), map, gates,
        reinterpret_cast<V32*>(y), c.N, c.k, c.n_shared, vpr32, check_word());
    return;
  }
  const int vpr = vecs_per_row(c);
  const long long items = (long long)c.N * ((vpr + 32 * kCombVec - 1) / (32 * kCombVec));
  combine_kernel<T><<<blocks_for(items), kMoveWarps * 32, 0, st>>>(routed, shared, map, gates, y, c.N, c.k,
                                                                    c.n_shared, vpr, check_word());
}

cudaError_t launch_combine(const moe_config& c, const moe_layout& L, const void* out, const float* topk_w, void* y,
                           cudaStream_t st) {
  if (c.N == 0) return cudaSuccess;
  const size_t A = (size_t)c.N * c.k;
  const uint4* o = static_cast<const uint4*>(out);
  const uint4* sh = o + A * vecs_per_row(c);
  if (c.dtype == MOE_BF16)
    combine_launch<__nv_bfloat16>(c, o, sh, L.tok2row, topk_w, static_cast<uint4*>(y), st);
  else
    combine_launch<float>(c, o, sh, L.tok2row, topk_w, static_cast<uint4*>(y), st);
  return cudaGetLastError();
}

cudaError_t launch_combine_staged(const moe_config& c, const moe_layout& L, const void* out, const float* topk_w,
                                  void* ret_buf, void* y, cudaStream_t st) {
  if (c.N == 0) return cudaSuccess;
  const int vpr = vecs_per_row(c);
  const int A = c.N * c.k;
  const uint4* o = static_cast<const uint4*>(out);
  // hop 1: owners return rows in send-slot order (reverse transpose): ret[s] = out[send2row[s]]
  move_rows<false><<<blocks_for(A), kMoveWarps * 32, 0, st>>>(o, static_cast<uint4*>(ret_buf), L.send2row, A, vpr,
                                                              check_word());
  // hop 2: unpermute + weighted sum at the source through tok2send
  const uint4* sh = o + (size_t)A * vpr;
  if (c.dtype == MOE_BF16)
    combine_launch<__nv_bfloat16>(c, static_cast<const uint4*>(ret_buf), sh, L.tok2send, topk_w,
                                  static_cast<uint4*>(y), st);
  else
    combine_launch<float>(c, static_cast<const uint4*>(ret_buf), sh, L.tok2send, topk_w, static_cast<uint4*>(y),
                          st);
  return cudaGetLastError();
}

}  // namespace moe
