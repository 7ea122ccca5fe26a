// C entry points of libmoe: argument validation, workspace carving and the launch order
// of the layer's steps.  Every step runs in this library's CUDA kernels; nothing here
// computes on the host.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "kernels.cuh"

using namespace moe;

namespace {

thread_local char g_last_error[256] = "";

moe_status fail(moe_status s, const char* what) {
  snprintf(g_last_error, sizeof(g_last_error), "%s", what);
  return s;
}

moe_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return MOE_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int elem_bytes(const moe_config& c) { return c.dtype == MOE_BF16 ? 2 : 4; }

moe_status check_config(const moe_config* c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "config is NULL");
  if (c->N < 0 || c->d <= 0 || c->E <= 0 || c->k <= 0 || c->I <= 0 || c->n_shared < 0 || c->P <= 0)
    return fail(MOE_ERR_INVALID_ARG, "sizes must be positive (N >= 0)");
  if (c->n_groups <= 0 || c->topk_groups <= 0 || c->topk_groups > c->n_groups || c->E % c->n_groups != 0)
    return fail(MOE_ERR_INVALID_ARG, "need 1 <= topk_groups <= n_groups and E % n_groups == 0");
  if ((long long)c->k > (long long)c->topk_groups * (c->E / c->n_groups))
    return fail(MOE_ERR_INVALID_ARG, "k exceeds the experts of the kept groups");
  if ((c->score != MOE_SCORE_SOFTMAX && c->score != MOE_SCORE_SIGMOID) ||
      (c->dtype != MOE_F32 && c->dtype != MOE_BF16) || (c->renormalize != 0 && c->renormalize != 1) ||
      (c->bias_mode != MOE_BIAS_LOGITS && c->bias_mode != MOE_BIAS_SELECTION))
    return fail(MOE_ERR_INVALID_ARG, "score, dtype, renormalize or bias_mode out of range");
  if (c->k > kMaxK || c->E > kMaxSlots || c->P > kMaxP || c->n_groups > kMaxGroups ||
      c->topk_groups > kMaxTopkGroups || c->n_shared > kMaxShared)
    return fail(MOE_ERR_UNSUPPORTED, "k <= 8, E <= 512, P <= 32, n_groups <= 32, topk_groups <= 8, S <= 8");
  const int eb = elem_bytes(*c);
  if ((c->d * eb) % 16 != 0 || (c->I * eb) % 16 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "rows of d and I elements must be multiples of 16 bytes");
  const long long rows = (long long)c->N * c->k + (long long)c->n_shared * c->N;
  if (rows >= (1LL << 31) / 2) return fail(MOE_ERR_UNSUPPORTED, "N * (k + S) too large");
  return MOE_OK;
}

// The router (and so every call that routes) scores at most kMaxE experts; the layout,
// movement and expert calls take up to kMaxSlots (e.g. E + R physical expert slots).
moe_status check_router(const moe_config& c) {
  if (c.E > kMaxE) return fail(MOE_ERR_UNSUPPORTED, "the router scores at most 256 experts");
  return MOE_OK;
}

moe_status check_owner(const moe_config& c, const int32_t* owner) {
  if (!owner && c.E % c.P != 0) return fail(MOE_ERR_INVALID_ARG, "contiguous placement needs E % P == 0");
  return MOE_OK;
}

bool layout_complete(const moe_layout* L) {
  return L && L->n_e && L->expert_off && L->C && L->send_off && L->recv_off && L->tok2send && L->send2row &&
         L->ret2tok && L->tok2row && L->row2tok && L->tile_off;
}

size_t layout_scratch(const moe_config& c) {
  const int A = c.N * c.k;
  const int nchunks = (A + kLayoutChunk - 1) / kLayoutChunk;
  return align256(layout_ws_bytes(A, c.E, c.P, nchunks));
}

struct FwdWs {
  float* logits;
  int32_t* ids;
  float* w;
  moe_layout lay;
  void* lay_ws;
  void* x_perm;
  void* h;
  void* out;
  // FP8 forward only
  void* x_q;
  float* x_scale;
  void* h_q;
  float* h_scale;
  // MX forward only: E8M0 scale bytes, one per 32 values of a row
  uint8_t* x_sf;       // [N, d/32]
  uint8_t* x_sf_perm;  // [A, d/32]
  uint8_t* h_sf;       // [A + S*N, I/32]
  size_t total;
};

// fp8: the FP8 forward's buffers (x_perm holds e4m3 rows, plus x_q, h_q and the scales)
// mx: the MX forward's buffers (those of the FP8 forward plus the scale bytes)
FwdWs carve_forward(const moe_config& c, char* base, bool fp8 = false, bool mx = false) {
  fp8 = fp8 || mx;
  FwdWs w;
  memset(&w, 0, sizeof(w));
  const size_t A = (size_t)c.N * c.k, E = c.E, P = c.P, S = c.n_shared, eb = elem_bytes(c);
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off += align256(bytes ? bytes : 1);
    return p;
  };
  w.logits = reinterpret_cast<float*>(take((size_t)c.N * E * 4));
  w.ids = reinterpret_cast<int32_t*>(take(A * 4));
  w.w = reinterpret_cast<float*>(take(A * 4));
  w.lay.n_e = reinterpret_cast<int32_t*>(take(E * 4));
  w.lay.expert_off = reinterpret_cast<int32_t*>(take((E + 1) * 4));
  w.lay.C = reinterpret_cast<int32_t*>(take(P * P * 4));
  w.lay.send_off = reinterpret_cast<int32_t*>(take(P * P * 4));
  w.lay.recv_off = reinterpret_cast<int32_t*>(take((P + 1) * 4));
  w.lay.tok2send = reinterpret_cast<int32_t*>(take(A * 4));
  w.lay.send2row = reinterpret_cast<int32_t*>(take(A * 4));
  w.lay.ret2tok = reinterpret_cast<int32_t*>(take(A * 4));
  w.lay.tok2row = reinterpret_cast<int32_t*>(take(A * 4));
  w.lay.row2tok = reinterpret_cast<int32_t*>(take(A * 4));
  w.lay.tile_off = reinterpret_cast<int32_t*>(take((E + S + 1) * 4));
  w.lay_ws = take(layout_scratch(c));
  w.x_perm = take(A * c.d * (fp8 ? 1 : eb));
  w.h = take(mx ? 0 : (A + S * c.N) * c.I * eb);  // the MX forward quantises h in FC1's epilogue
  w.out = take((A + S * c.N) * c.d * eb);
  if (fp8) {
    w.x_q = take((size_t)c.N * c.d);
    w.x_scale = reinterpret_cast<float*>(take((size_t)c.N * 4));
    w.h_q = take((A + S * c.N) * c.I);
    w.h_scale = reinterpret_cast<float*>(take((A + S * c.N) * 4));
  }
  if (mx) {
    w.x_sf = reinterpret_cast<uint8_t*>(take((size_t)c.N * (c.d / 32)));
    w.x_sf_perm = reinterpret_cast<uint8_t*>(take(A * (c.d / 32)));
    w.h_sf = reinterpret_cast<uint8_t*>(take((A + S * c.N) * (c.I / 32)));
  }
  w.total = off;
  return w;
}

moe_status route_impl(const moe_config& c, const void* x, const void* w_gate, const float* bias, float* logits,
                      int32_t* ids, float* w, cudaStream_t st) {
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.mode = MODE_ROUTER;
  g.G = 1;
  g.E = 0;
  g.N = c.N;
  g.A_routed = 0;
  g.K = c.d;
  g.n_out = c.E;
  g.shared_from_map1 = 1;
  g.bias = bias;
  g.out = logits;
  g.ldo = c.E;
  g.a0 = x;
  g.a1 = x;
  g.b = w_gate;
  g.b_rows = c.E;
  cudaError_t e = c.dtype == MOE_BF16 ? launch_tc_gemm(g, c.N, c.N, st) : launch_simt_gemm(g, st);
  if (e != cudaSuccess) return cuda_status(e, "router GEMM");
  return cuda_status(launch_topk(c, logits, c.bias_mode == MOE_BIAS_SELECTION ? bias : nullptr, ids, w, st),
                     "top-k");
}

GemmArgs fc1_args(const moe_config& c, const moe_layout& L, const void* x_perm, const void* x, const void* w13,
                  void* h) {
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.mode = MODE_FC1;
  g.G = c.E + c.n_shared;
  g.E = c.E;
  g.N = c.N;
  g.A_routed = c.N * c.k;
  g.K = c.d;
  g.n_out = c.I;
  g.I = c.I;
  g.shared_from_map1 = 1;
  g.n_e = L.n_e;
  g.expert_off = L.expert_off;
  g.row2tok = L.row2tok;
  g.out = h;
  g.ldo = c.I;
  g.a0 = x_perm;
  g.a1 = c.n_shared > 0 ? x : nullptr;
  g.b = w13;
  g.b_rows = 2LL * c.I;
  g.check = check_word();
  return g;
}

GemmArgs fc2_args(const moe_config& c, const moe_layout& L, const void* h, const void* w2, const float* topk_w,
                  void* out) {
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.mode = MODE_FC2;
  g.G = c.E + c.n_shared;
  g.E = c.E;
  g.N = c.N;
  g.A_routed = c.N * c.k;
  g.K = c.I;
  g.n_out = c.d;
  g.I = c.I;
  g.shared_from_map1 = 0;
  g.n_e = L.n_e;
  g.expert_off = L.expert_off;
  g.row2tok = L.row2tok;
  g.gate_w = topk_w;
  g.out = out;
  g.ldo = c.d;
  g.a0 = h;
  g.b = w2;
  g.b_rows = c.d;
  g.check = check_word();
  return g;
}

// Tensor-core grouped GEMM: on CTA pairs for wide hidden sizes (d >= 4096), where every
// row of a group runs in one pass over its weights (256-row blocks, the 1..128 rows past
// the last block carried on it, or one 128-row tile for a group of at most 128 rows); with
// d = 2048 the one-CTA 128-row tiles measured faster.  A group has at most N rows, so with
// N <= 128 the one-CTA kernel runs.
cudaError_t tc_grouped(GemmArgs g, const moe_config& c, int a0_rows, int a1_rows, cudaStream_t st) {
  if (c.N > 128 && c.d >= 4096) return launch_tc_gemm_pair(g, a0_rows, a1_rows, st);
  return launch_tc_gemm(g, a0_rows, a1_rows, st);
}

// A launch over the shared experts alone runs beside the routing kernels of the same
// layer (moe_layer_forward_overlapped): it leaves this many SMs to them.
constexpr int kSharedReserveSMs = 16;

int shared_cap(const moe_config& c, int g0) {
  return (g0 >= c.E && sm_count() > 2 * kSharedReserveSMs) ? sm_count() - kSharedReserveSMs : 0;
}

moe_status fc1_impl(const moe_config& c, const moe_layout& L, const void* x_perm, const void* x, const void* w13,
                    void* h, cudaStream_t st, int g0 = 0, int G = -1) {
  GemmArgs g = fc1_args(c, L, x_perm, x, w13, h);
  g.g0 = g0;
  g.max_ctas = shared_cap(c, g0);
  if (G >= 0) g.G = G;
  if (g.G == 0) return MOE_OK;
  cudaError_t e = c.dtype == MOE_BF16 ? tc_grouped(g, c, c.N * c.k, c.N, st) : launch_simt_gemm(g, st);
  return cuda_status(e, "FC1 grouped GEMM");
}

moe_status fc2_impl(const moe_config& c, const moe_layout& L, const void* h, const void* w2, const float* topk_w,
                    void* out, cudaStream_t st, int g0 = 0, int G = -1) {
  GemmArgs g = fc2_args(c, L, h, w2, topk_w, out);
  g.g0 = g0;
  g.max_ctas = shared_cap(c, g0);
  if (G >= 0) g.G = G;
  if (g.G == 0) return MOE_OK;
  cudaError_t e = c.dtype == MOE_BF16 ? tc_grouped(g, c, c.N * c.k + c.n_shared * c.N, 0, st)
                                      : launch_simt_gemm(g, st);
  return cuda_status(e, "FC2 grouped GEMM");
}

// FP8 expert FFN over groups [g0, g0+G): FC1 on e4m3 rows -> h (bf16) -> per-row e4m3
// quantisation of h -> FC2 on e4m3 rows, on the same tile kernels as bf16.
struct Fp8Ffn {
  const void *x_q_perm, *x_q;
  const float* x_scale;
  const void* w13_q;
  const float* w13_scale;
  const void* w2_q;
  const float* w2_scale;
  const float* topk_w;
  void* h;
  void* h_q;
  float* h_scale;
  void* out;
};

moe_status ffn_fp8_impl(const moe_config& c, const moe_layout& L, const Fp8Ffn& f, cudaStream_t st, int g0 = 0,
                        int G = -1) {
  if (G < 0) G = c.E + c.n_shared - g0;
  if (G == 0) return MOE_OK;
  const long long A = (long long)c.N * c.k;
  GemmArgs g = fc1_args(c, L, f.x_q_perm, f.x_q, f.w13_q, f.h);
  g.g0 = g0;
  g.G = G;
  g.max_ctas = shared_cap(c, g0);
  g.fp8 = 1;
  g.k = c.k;
  g.a_scale = f.x_scale;
  g.b_scale = f.w13_scale;
  cudaError_t e = tc_grouped(g, c, (int)A, c.N, st);
  if (e != cudaSuccess) return cuda_status(e, "FC1 grouped GEMM (fp8)");
  // rows of h this group range wrote: all routed rows [0, A) if a routed group is in
  // range, then the N-row blocks of the shared experts in range
  const long long r0 = g0 < c.E ? 0 : A + (long long)(g0 - c.E) * c.N;
  const long long r1 = (g0 + G <= c.E) ? A : A + (long long)(g0 + G - c.E) * c.N;
  e = launch_quantize_rows(static_cast<const uint16_t*>(f.h) + r0 * c.I, r1 - r0, c.I,
                           static_cast<uint8_t*>(f.h_q) + r0 * c.I, f.h_scale + r0, st);
  if (e != cudaSuccess) return cuda_status(e, "h quantisation");
  GemmArgs g2 = fc2_args(c, L, f.h_q, f.w2_q, f.topk_w, f.out);
  g2.g0 = g0;
  g2.G = G;
  g2.max_ctas = shared_cap(c, g0);
  g2.fp8 = 1;
  g2.k = c.k;
  g2.a_scale = f.h_scale;
  g2.b_scale = f.w2_scale;
  return cuda_status(tc_grouped(g2, c, (int)(A + (long long)c.n_shared * c.N), 0, st), "FC2 grouped GEMM (fp8)");
}

// MX expert FFN over groups [g0, g0+G): FC1 on block-scaled e4m3 rows, whose epilogue
// rounds h to bf16 (stored when f.h is given) and quantises it to MX, then FC2 on
// block-scaled rows, on the block-scaled tile kernel.
struct MxFfn {
  const void* x_q_perm;
  const uint8_t* x_sf_perm;
  const void* x_q;
  const uint8_t* x_sf;
  const void* w13_q;
  const uint8_t* w13_sf;
  const void* w2_q;
  const uint8_t* w2_sf;
  const float* topk_w;
  void* h;
  void* h_q;
  uint8_t* h_sf;
  void* out;
};

moe_status ffn_mx_impl(const moe_config& c, const moe_layout& L, const MxFfn& f, cudaStream_t st, int g0 = 0,
                       int G = -1) {
  if (G < 0) G = c.E + c.n_shared - g0;
  if (G == 0) return MOE_OK;
  const long long A = (long long)c.N * c.k;
  GemmArgs g = fc1_args(c, L, f.x_q_perm, f.x_q, f.w13_q, f.h);
  g.g0 = g0;
  g.G = G;
  g.max_ctas = shared_cap(c, g0);
  g.a0_sf = f.x_sf_perm;
  g.a1_sf = f.x_sf;
  g.b_sf = f.w13_sf;
  g.a0_rows = A > 0 ? A : 1;
  g.a1_rows = c.N;
  g.q_out = f.h_q;  // h quantised by FC1's epilogue (h itself stored only when f.h is given)
  g.q_sf = f.h_sf;
  cudaError_t e = launch_tc_gemm_mx(g, st);
  if (e != cudaSuccess) return cuda_status(e, "FC1 grouped GEMM (mx)");
  GemmArgs g2 = fc2_args(c, L, f.h_q, f.w2_q, f.topk_w, f.out);
  g2.g0 = g0;
  g2.G = G;
  g2.max_ctas = shared_cap(c, g0);
  g2.a0_sf = f.h_sf;
  g2.b_sf = f.w2_sf;
  g2.a0_rows = A + (long long)c.n_shared * c.N;
  g2.a1_rows = g2.a0_rows;
  return cuda_status(launch_tc_gemm_mx(g2, st), "FC2 grouped GEMM (mx)");
}

moe_status ffn_impl(const moe_config& c, const moe_layout& L, const void* x_perm, const void* x, const void* w13,
                    const void* w2, const float* topk_w, void* h, void* out, cudaStream_t st, int g0 = 0,
                    int G = -1) {
  moe_status s = fc1_impl(c, L, x_perm, x, w13, h, st, g0, G);
  if (s != MOE_OK) return s;
  return fc2_impl(c, L, h, w2, topk_w, out, st, g0, G);
}

// ---- expert parallelism across GPUs
struct EpWs {
  moe_layout loc;  // this rank's assignments laid out with a single owner
  void* lay_ws;
  void* h;         // [capacity + S*N, I]
  // moe_ep_layer_forward only
  float* logits;
  int32_t* ids;
  float* w;
  moe_ep_handle hd;
  // FP8 only
  void* h_q;        // [capacity + S*N, I] e4m3
  float* h_scale;   // [capacity + S*N]
  void* x_q;        // [N, d] e4m3 (moe_ep_layer_forward_fp8)
  float* x_scale;   // [N]
  // MX only
  uint8_t* h_sf;    // [capacity + S*N, I/32] E8M0
  uint8_t* x_sf;    // [N, d/32] (moe_ep_layer_forward_mx)
  size_t total;
};

moe_config one_owner(const moe_config& c) {
  moe_config c1 = c;
  c1.P = 1;
  return c1;
}

// fp8: the FP8 path's buffers; mx: the MX path's (those plus the scale bytes)
EpWs carve_ep(const moe_config& c, int capacity, char* base, bool fp8 = false, bool mx = false) {
  fp8 = fp8 || mx;
  EpWs w;
  memset(&w, 0, sizeof(w));
  const size_t A = (size_t)c.N * c.k, E = c.E, S = c.n_shared, eb = elem_bytes(c);
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off += align256(bytes ? bytes : 1);
    return p;
  };
  auto i32 = [&](size_t n) { return reinterpret_cast<int32_t*>(take(n * 4)); };
  w.loc.n_e = i32(E);
  w.loc.expert_off = i32(E + 1);
  w.loc.C = i32(1);
  w.loc.send_off = i32(1);
  w.loc.recv_off = i32(2);
  w.loc.tok2send = i32(A);
  w.loc.send2row = i32(A);
  w.loc.ret2tok = i32(A);
  w.loc.tok2row = i32(A);
  w.loc.row2tok = i32(A);
  w.loc.tile_off = i32(E + S + 1);
  w.lay_ws = take(layout_scratch(one_owner(c)));
  // (the MX path quantises h in FC1's epilogue and leaves this unused; it stays so that an
  // MX workspace also satisfies the size check of the precision-independent EP calls)
  w.h = take(((size_t)capacity + S * c.N) * c.I * eb);
  w.logits = reinterpret_cast<float*>(take((size_t)c.N * E * 4));
  w.ids = i32(A);
  w.w = reinterpret_cast<float*>(take(A * 4));
  w.hd.dest = i32(A);
  w.hd.owner_n_e = i32(E);
  w.hd.owner_off = i32(E + 1);
  if (fp8) {
    const size_t rows = (size_t)capacity + S * c.N;
    w.h_q = take(rows * c.I);
    w.h_scale = reinterpret_cast<float*>(take(rows * 4));
    w.x_q = take((size_t)c.N * c.d);
    w.x_scale = reinterpret_cast<float*>(take((size_t)c.N * 4));
  }
  if (mx) {
    w.h_sf = reinterpret_cast<uint8_t*>(take(((size_t)capacity + S * c.N) * (c.I / 32)));
    w.x_sf = reinterpret_cast<uint8_t*>(take((size_t)c.N * (c.d / 32)));
  }
  w.total = off;
  return w;
}

moe_status check_ep(const moe_config* cfg, const moe_ep_group* g, EpPeers* peers) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (!g || !g->windows) return fail(MOE_ERR_INVALID_ARG, "EP group or its window table is NULL");
  const moe_config& c = *cfg;
  if (g->rank < 0 || g->rank >= c.P) return fail(MOE_ERR_INVALID_ARG, "rank outside [0, P)");
  if (g->capacity < 1 || (long long)g->capacity * c.P >= (1LL << 31) ||
      (long long)g->capacity + (long long)c.n_shared * c.N >= (1LL << 30))
    return fail(MOE_ERR_UNSUPPORTED, "need 1 <= capacity, capacity * P < 2^31 and capacity + S*N < 2^30");
  if (g->local_experts < 0 || g->local_experts > c.E) return fail(MOE_ERR_INVALID_ARG, "local_experts outside [0, E]");
  memset(peers, 0, sizeof(*peers));
  for (int p = 0; p < c.P; ++p) {
    if (!g->windows[p] || (reinterpret_cast<uintptr_t>(g->windows[p]) & 255) != 0)
      return fail(MOE_ERR_INVALID_ARG, "every window must be non-NULL and 256-byte aligned");
    peers->base[p] = static_cast<char*>(g->windows[p]);
  }
  return MOE_OK;
}

moe_status check_ep_ws(const moe_config& c, const moe_ep_group* g, void* ws, size_t ws_bytes, bool fp8 = false,
                       bool mx = false) {
  if (!ws || ws_bytes < carve_ep(c, g->capacity, nullptr, fp8, mx).total)
    return fail(MOE_ERR_WORKSPACE, "EP workspace too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  return MOE_OK;
}

bool handle_complete(const moe_ep_handle* h) { return h && h->dest && h->owner_n_e && h->owner_off; }

moe_status ep_notify_impl(const moe_config& c, const moe_ep_group& g, const EpPeers& peers,
                          const int32_t* ids, int32_t* status, const EpWs& w, cudaStream_t st) {
  moe_status s = cuda_status(launch_layout(one_owner(c), nullptr, ids, w.loc, status, w.lay_ws, st), "local layout");
  if (s != MOE_OK) return s;
  return cuda_status(
      launch_ep_push_counts(peers, ep_offsets(c, g.capacity), w.loc.n_e, c.E, c.P, g.rank, st),
      "count exchange");
}

moe_status ep_layout_impl(const moe_config& c, const moe_ep_group& g, const EpPeers& peers,
                          const int32_t* owner, const int32_t* ids, const moe_ep_handle& hd, int32_t* status,
                          const EpWs& w, cudaStream_t st) {
  return cuda_status(launch_ep_layout(c, peers, ep_offsets(c, g.capacity), g.rank, g.capacity, g.local_experts,
                                      owner, ids, w.loc, hd.dest, hd.owner_n_e, hd.owner_off, status, st),
                     "EP layout");
}

// The owner's expert GEMMs over groups [g0, g0+G): groups [0, local_experts) are the
// owned experts over the received rows (A_routed = capacity, no row map: row r's gate is
// gate[r], and with FP8 its token scale is scale[r]); the S shared groups run over the
// rank's own N tokens.  Outputs go to the window's output rows.  FP8: FC1 on e4m3 rows,
// per-row quantisation of the h rows of the range, FC2 on e4m3 h.
struct EpFfn {
  bool fp8;
  const void* x;  // bf16 tokens, or e4m3 codes with x_scale (FP8) / x_sf (MX)
  const float* x_scale;
  const void* w13;
  const float* w13_scale;
  const void* w2;
  const float* w2_scale;
  // MX (block-scaled e4m3): E8M0 scale rows beside the codes; the received rows' scales
  // follow their codes in the window's receive region
  bool mx = false;
  const uint8_t* x_sf = nullptr;
  const uint8_t* w13_sf = nullptr;
  const uint8_t* w2_sf = nullptr;
};

// The MX form of ep_gemms: FC1 on the received codes and their scale rows (the shared
// groups on this rank's own x codes) with h quantised to MX in its epilogue, then FC2.
moe_status ep_gemms_mx(const moe_config& c, const moe_ep_group& g, char* win, const EpOffsets& off, const EpFfn& f,
                       const moe_ep_handle& hd, const EpWs& w, cudaStream_t st, int g0, int G) {
  moe_config co = c;
  co.E = g.local_experts;
  moe_layout L;
  memset(&L, 0, sizeof(L));
  L.n_e = hd.owner_n_e;
  L.expert_off = hd.owner_off;
  const int S = c.N > 0 ? c.n_shared : 0;
  const long long cap = g.capacity;
  const long long rows = cap + (long long)S * c.N;
  GemmArgs g1 = fc1_args(co, L, win + off.x_recv, S > 0 ? f.x : nullptr, f.w13, w.h);
  g1.g0 = g0;
  g1.G = G;
  g1.A_routed = g.capacity;
  g1.max_ctas = shared_cap(co, g0);
  g1.a0_sf = reinterpret_cast<const uint8_t*>(win + off.x_recv) + cap * c.d;  // after the codes
  g1.a1_sf = f.x_sf;
  g1.b_sf = f.w13_sf;
  g1.a0_rows = cap;
  g1.a1_rows = c.N > 0 ? c.N : 1;
  g1.out = nullptr;  // h quantised by the epilogue, not kept in bf16
  g1.q_out = w.h_q;
  g1.q_sf = w.h_sf;
  cudaError_t e = launch_tc_gemm_mx(g1, st);
  if (e != cudaSuccess) return cuda_status(e, "EP FC1 grouped GEMM (mx)");
  GemmArgs g2 = fc2_args(co, L, w.h_q, f.w2, reinterpret_cast<const float*>(win + off.gate), win + off.out_recv);
  g2.g0 = g0;
  g2.G = G;
  g2.A_routed = g.capacity;
  g2.max_ctas = shared_cap(co, g0);
  g2.a0_sf = w.h_sf;
  g2.b_sf = f.w2_sf;
  g2.a0_rows = rows;
  g2.a1_rows = rows;
  return cuda_status(launch_tc_gemm_mx(g2, st), "EP FC2 grouped GEMM (mx)");
}

moe_status ep_gemms(const moe_config& c, const moe_ep_group& g, char* win, const EpOffsets& off, const EpFfn& f,
                    const moe_ep_handle& hd, const EpWs& w, cudaStream_t st, int g0, int G) {
  if (G <= 0) return MOE_OK;
  if (f.mx) return ep_gemms_mx(c, g, win, off, f, hd, w, st, g0, G);
  moe_config co = c;
  co.E = g.local_experts;
  moe_layout L;
  memset(&L, 0, sizeof(L));
  L.n_e = hd.owner_n_e;
  L.expert_off = hd.owner_off;
  const int S = c.N > 0 ? c.n_shared : 0;  // the shared experts have no rows without tokens
  const long long cap = g.capacity;
  // pair tiles pay for wide rows when a group can exceed 128 rows
  moe_config dec = c;
  dec.N = g.capacity > c.N ? g.capacity : c.N;
  GemmArgs g1 = fc1_args(co, L, win + off.x_recv, S > 0 ? f.x : nullptr, f.w13, w.h);
  g1.g0 = g0;
  g1.G = G;
  g1.A_routed = g.capacity;
  g1.max_ctas = shared_cap(co, g0);
  if (f.fp8) {
    g1.fp8 = 1;
    g1.k = c.k;
    g1.a_scale = f.x_scale;
    g1.a_scale_rows = reinterpret_cast<const float*>(win + off.scale);
    g1.b_scale = f.w13_scale;
  }
  cudaError_t e = c.dtype == MOE_BF16 ? tc_grouped(g1, dec, g.capacity, c.N, st) : launch_simt_gemm(g1, st);
  if (e != cudaSuccess) return cuda_status(e, "EP FC1 grouped GEMM");
  const long long rows = cap + (long long)S * c.N;
  if (f.fp8) {  // h rows of this range: the routed rows [0, capacity), then N per shared group
    const int Lx = g.local_experts;
    const long long r0 = g0 < Lx ? 0 : cap + (long long)(g0 - Lx) * c.N;
    const long long r1 = g0 + G <= Lx ? cap : cap + (long long)(g0 + G - Lx) * c.N;
    e = launch_quantize_rows(static_cast<const uint16_t*>(w.h) + r0 * c.I, r1 - r0, c.I,
                             static_cast<uint8_t*>(w.h_q) + r0 * c.I, w.h_scale + r0, st);
    if (e != cudaSuccess) return cuda_status(e, "h quantisation");
  }
  GemmArgs g2 = fc2_args(co, L, f.fp8 ? w.h_q : w.h, f.w2, reinterpret_cast<const float*>(win + off.gate),
                         win + off.out_recv);
  g2.g0 = g0;
  g2.G = G;
  g2.A_routed = g.capacity;
  g2.max_ctas = shared_cap(co, g0);
  if (f.fp8) {
    g2.fp8 = 1;
    g2.k = c.k;
    g2.a_scale = w.h_scale;
    g2.b_scale = f.w2_scale;
  }
  e = c.dtype == MOE_BF16 ? tc_grouped(g2, dec, (int)rows, 0, st) : launch_simt_gemm(g2, st);
  return cuda_status(e, "EP FC2 grouped GEMM");
}

// wait for every source's dispatch, the expert GEMMs of groups [0, G), "done" to every source
moe_status ep_ffn_impl(const moe_config& c, const moe_ep_group& g, const EpPeers& peers, const EpFfn& f,
                       const moe_ep_handle& hd, int32_t* status, const EpWs& w, cudaStream_t st, int G) {
  const EpOffsets off = ep_offsets(c, g.capacity);
  char* win = peers.base[g.rank];
  cudaError_t e = launch_ep_wait(win, off, off.disp_flag, c.P, status, st);
  if (e != cudaSuccess) return cuda_status(e, "dispatch wait");
  moe_status s = ep_gemms(c, g, win, off, f, hd, w, st, 0, G);
  if (s != MOE_OK) return s;
  return cuda_status(launch_ep_signal(peers, off, off.done_flag, c.P, g.rank, st), "FFN done signal");
}

int ep_groups(const moe_config& c, const moe_ep_group& g) { return g.local_experts + (c.N > 0 ? c.n_shared : 0); }

// One rank's layer.  With a side stream (and shared experts), the shared experts' GEMMs
// run there from right after the router, beside the count exchange, the dispatch, the
// wait for the other ranks' rows and the routed GEMMs; the combine waits for them.
moe_status ep_forward(const moe_config& c, const moe_ep_group& g, const EpPeers& peers, const void* x,
                      const void* w_gate, const float* bias, const int32_t* owner, const EpFfn& fin, void* y,
                      const moe_ep_handle* handle_out, int32_t* status, const EpWs& w, cudaStream_t st,
                      cudaStream_t side) {
  const moe_ep_handle& hd = handle_out ? *handle_out : w.hd;
  const EpOffsets off = ep_offsets(c, g.capacity);
  EpFfn f = fin;
  moe_status s = MOE_OK;
  if (c.N > 0) {
    if ((s = route_impl(c, x, w_gate, bias, w.logits, w.ids, w.w, st)) != MOE_OK) return s;
    if (f.mx) {
      s = cuda_status(launch_quantize_mx(x, c.N, c.d, w.x_q, w.x_sf, st), "x quantisation (mx)");
      if (s != MOE_OK) return s;
      f.x = w.x_q;
      f.x_sf = w.x_sf;
    } else if (f.fp8) {
      s = cuda_status(launch_quantize_rows(x, c.N, c.d, w.x_q, w.x_scale, st), "x quantisation");
      if (s != MOE_OK) return s;
      f.x = w.x_q;
      f.x_scale = w.x_scale;
    } else {
      f.x = x;
    }
  }
  const bool overlap = side && side != st && c.N > 0 && c.n_shared > 0;
  cudaEvent_t fork = nullptr, join = nullptr;
  if (overlap) {
    cudaError_t e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
    if (e == cudaSuccess) {
      s = ep_gemms(c, g, peers.base[g.rank], off, f, hd, w, side, g.local_experts, c.n_shared);
      e = cudaEventRecord(join, side);
    }
    if (e != cudaSuccess && s == MOE_OK) s = cuda_status(e, "fork");
  }
  const int G = overlap ? g.local_experts : ep_groups(c, g);
  if (s == MOE_OK) s = ep_notify_impl(c, g, peers, w.ids, status, w, st);
  if (s == MOE_OK) s = ep_layout_impl(c, g, peers, owner, w.ids, hd, status, w, st);
  if (s == MOE_OK)
    s = cuda_status(launch_ep_dispatch(c, peers, off, g.rank, g.capacity, f.x, hd.dest, w.w,
                                       f.fp8 && !f.mx ? f.x_scale : nullptr,
                                       c.d * (f.fp8 || f.mx ? 1 : elem_bytes(c)), st, f.mx ? f.x_sf : nullptr,
                                       c.d / 32),
                    "EP dispatch");
  if (s == MOE_OK) s = ep_ffn_impl(c, g, peers, f, hd, status, w, st, G);
  if (overlap) {
    if (join) cudaStreamWaitEvent(st, join, 0);  // join even after an error
    if (fork) cudaEventDestroy(fork);
    if (join) cudaEventDestroy(join);
  }
  if (s != MOE_OK) return s;
  return cuda_status(launch_ep_combine(c, peers, off, g.rank, g.capacity, hd.dest, y, status, st), "EP combine");
}

}  // namespace

namespace moe {
// Bounds-checked build: the caller's device word failed checks are recorded into.
static int32_t* g_check_word = nullptr;
int* check_word() { return g_check_word; }

// The error recorder for entry points defined in other files of this library (the text
// moe_last_error returns).
moe_status record_error(moe_status s, const char* what) { return fail(s, what); }
moe_status record_cuda_error(cudaError_t e, const char* where) { return cuda_status(e, where); }
}  // namespace moe

extern "C" {

int32_t moe_version(void) { return 101; }

int32_t moe_checks_enabled(void) { return kChecks ? 1 : 0; }

moe_status moe_checks_register(int32_t* dev_word) {
  g_check_word = dev_word;
  return MOE_OK;
}

const char* moe_status_string(int32_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported size";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_BAD_INDEX: return "expert id or owner out of range (device)";
    case MOE_ERR_TIMEOUT: return "bounded wait timed out (device)";
    default: return "unknown status";
  }
}

const char* moe_last_error(void) { return g_last_error; }

moe_status moe_check_config(const moe_config* cfg) { return check_config(cfg); }

size_t moe_layout_workspace_bytes(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return layout_scratch(*cfg);
}

size_t moe_workspace_bytes(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return carve_forward(*cfg, nullptr).total;
}

moe_status moe_route(const moe_config* cfg, const void* x, const void* w_gate, const float* bias, float* logits,
                     int32_t* topk_ids, float* topk_w, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_router(*cfg)) != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!x || !w_gate || !logits || !topk_ids || !topk_w) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return route_impl(*cfg, x, w_gate, bias, logits, topk_ids, topk_w, (cudaStream_t)stream);
}

moe_status moe_dispatch_layout(const moe_config* cfg, const int32_t* expert_owner, const int32_t* topk_ids,
                               const moe_layout* out, int32_t* dev_status, void* ws, size_t ws_bytes,
                               moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_owner(*cfg, expert_owner)) != MOE_OK) return s;
  if (!layout_complete(out) || (cfg->N > 0 && !topk_ids)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!ws || ws_bytes < layout_scratch(*cfg)) return fail(MOE_ERR_WORKSPACE, "layout workspace too small");
  return cuda_status(launch_layout(*cfg, expert_owner, topk_ids, *out, dev_status, ws, (cudaStream_t)stream),
                     "layout");
}

moe_status moe_permute(const moe_config* cfg, const moe_layout* layout, const void* x, void* x_perm,
                       moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout->tok2row || !x || !x_perm) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_permute(*cfg, *layout, x, x_perm, (cudaStream_t)stream), "permute");
}

moe_status moe_permute_staged(const moe_config* cfg, const moe_layout* layout, const void* x, void* send_buf,
                              void* x_perm, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout->tok2send || !layout->send2row || !x || !send_buf || !x_perm)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_permute_staged(*cfg, *layout, x, send_buf, x_perm, (cudaStream_t)stream),
                     "permute (staged)");
}

moe_status moe_grouped_ffn(const moe_config* cfg, const moe_layout* layout, const void* x_perm, const void* x,
                           const void* w13, const void* w2, const float* topk_w, void* h_ws, void* out,
                           moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout->n_e || !layout->expert_off || !layout->row2tok || !x_perm || !w13 || !w2 || !h_ws ||
      !out || (cfg->n_shared > 0 && !x))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return ffn_impl(*cfg, *layout, x_perm, x, w13, w2, topk_w, h_ws, out, (cudaStream_t)stream);
}

static bool group_range(const moe_config& c, int32_t groups, int* g0, int* G) {
  switch (groups) {
    case MOE_GROUPS_ALL: *g0 = 0; *G = c.E + c.n_shared; return true;
    case MOE_GROUPS_ROUTED: *g0 = 0; *G = c.E; return true;
    case MOE_GROUPS_SHARED: *g0 = c.E; *G = c.n_shared; return true;
    default: return false;
  }
}

moe_status moe_expert_fc1(const moe_config* cfg, const moe_layout* layout, const void* x_perm, const void* x,
                          const void* w13, void* h_ws, int32_t groups, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  int g0, G;
  if (!group_range(*cfg, groups, &g0, &G)) return fail(MOE_ERR_INVALID_ARG, "groups out of range");
  if (cfg->N == 0) return MOE_OK;
  const bool routed = groups != MOE_GROUPS_SHARED, shared = groups != MOE_GROUPS_ROUTED && cfg->n_shared > 0;
  if (!w13 || !h_ws || (routed && (!layout || !layout->n_e || !layout->expert_off || !x_perm)) || (shared && !x))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  moe_layout none;
  memset(&none, 0, sizeof(none));
  return fc1_impl(*cfg, routed ? *layout : none, x_perm, x, w13, h_ws, (cudaStream_t)stream, g0, G);
}

moe_status moe_expert_fc2(const moe_config* cfg, const moe_layout* layout, const void* h_ws, const void* w2,
                          const float* topk_w, void* out, int32_t groups, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  int g0, G;
  if (!group_range(*cfg, groups, &g0, &G)) return fail(MOE_ERR_INVALID_ARG, "groups out of range");
  if (cfg->N == 0) return MOE_OK;
  const bool routed = groups != MOE_GROUPS_SHARED;
  if (!h_ws || !w2 || !out || (routed && (!layout || !layout->n_e || !layout->expert_off || !layout->row2tok)))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  moe_layout none;
  memset(&none, 0, sizeof(none));
  return fc2_impl(*cfg, routed ? *layout : none, h_ws, w2, topk_w, out, (cudaStream_t)stream, g0, G);
}

moe_status moe_routed_ffn(const moe_config* cfg, const moe_layout* layout, const void* x_perm, const void* w13,
                          const void* w2, const float* topk_w, void* h_ws, void* out, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout->n_e || !layout->expert_off || !layout->row2tok || !x_perm || !w13 || !w2 || !h_ws ||
      !out)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return ffn_impl(*cfg, *layout, x_perm, nullptr, w13, w2, topk_w, h_ws, out, (cudaStream_t)stream, 0, cfg->E);
}

moe_status moe_shared_ffn(const moe_config* cfg, const void* x, const void* w13, const void* w2, void* h_ws,
                          void* out, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0 || cfg->n_shared == 0) return MOE_OK;
  if (!x || !w13 || !w2 || !h_ws || !out) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  moe_layout none;
  memset(&none, 0, sizeof(none));
  return ffn_impl(*cfg, none, nullptr, x, w13, w2, nullptr, h_ws, out, (cudaStream_t)stream, cfg->E,
                  cfg->n_shared);
}

moe_status moe_combine(const moe_config* cfg, const moe_layout* layout, const void* out, const float* topk_w,
                       void* y, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout->tok2row || !out || !y) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_combine(*cfg, *layout, out, topk_w, y, (cudaStream_t)stream), "combine");
}

moe_status moe_combine_staged(const moe_config* cfg, const moe_layout* layout, const void* out,
                              const float* topk_w, void* ret_buf, void* y, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout->tok2send || !layout->send2row || !out || !ret_buf || !y)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_combine_staged(*cfg, *layout, out, topk_w, ret_buf, y, (cudaStream_t)stream),
                     "combine (staged)");
}

moe_status moe_layer_forward(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                             const int32_t* expert_owner, const void* w13, const void* w2, void* y,
                             const moe_layout* layout_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_router(*cfg)) != MOE_OK) return s;
  if ((s = check_owner(*cfg, expert_owner)) != MOE_OK) return s;
  const moe_config& c = *cfg;
  FwdWs w = carve_forward(c, nullptr);
  if (!ws || ws_bytes < w.total) return fail(MOE_ERR_WORKSPACE, "forward workspace too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (layout_out && !layout_complete(layout_out)) return fail(MOE_ERR_INVALID_ARG, "incomplete layout_out");
  if (c.N > 0 && (!x || !w_gate || !w13 || !w2 || !y)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  w = carve_forward(c, static_cast<char*>(ws));
  const moe_layout& L = layout_out ? *layout_out : w.lay;
  cudaStream_t st = (cudaStream_t)stream;
  if (c.N > 0 && (s = route_impl(c, x, w_gate, bias, w.logits, w.ids, w.w, st)) != MOE_OK) return s;
  if ((s = cuda_status(launch_layout(c, expert_owner, w.ids, L, dev_status, w.lay_ws, st), "layout")) != MOE_OK)
    return s;
  if (c.N == 0) return MOE_OK;
  if ((s = cuda_status(launch_permute(c, L, x, w.x_perm, st), "permute")) != MOE_OK) return s;
  if ((s = ffn_impl(c, L, w.x_perm, x, w13, w2, w.w, w.h, w.out, st)) != MOE_OK) return s;
  return cuda_status(launch_combine(c, L, w.out, nullptr, y, st), "combine");
}

moe_status moe_layer_forward_overlapped(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                                        const int32_t* expert_owner, const void* w13, const void* w2, void* y,
                                        const moe_layout* layout_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                                        moe_stream_t stream, moe_stream_t side_stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_router(*cfg)) != MOE_OK) return s;
  if ((s = check_owner(*cfg, expert_owner)) != MOE_OK) return s;
  const moe_config& c = *cfg;
  if (c.n_shared == 0 || c.N == 0 || side_stream == stream)
    return moe_layer_forward(cfg, x, w_gate, bias, expert_owner, w13, w2, y, layout_out, dev_status, ws, ws_bytes,
                             stream);
  FwdWs w = carve_forward(c, nullptr);
  if (!ws || ws_bytes < w.total) return fail(MOE_ERR_WORKSPACE, "forward workspace too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (layout_out && !layout_complete(layout_out)) return fail(MOE_ERR_INVALID_ARG, "incomplete layout_out");
  if (!x || !w_gate || !w13 || !w2 || !y) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  w = carve_forward(c, static_cast<char*>(ws));
  const moe_layout& L = layout_out ? *layout_out : w.lay;
  cudaStream_t st = (cudaStream_t)stream, side = (cudaStream_t)side_stream;
  if ((s = route_impl(c, x, w_gate, bias, w.logits, w.ids, w.w, st)) != MOE_OK) return s;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaError_t e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventRecord(fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
  if (e != cudaSuccess) {
    if (fork) cudaEventDestroy(fork);
    if (join) cudaEventDestroy(join);
    return cuda_status(e, "fork");
  }
  // side stream: shared experts (they read only x)
  moe_layout none;
  memset(&none, 0, sizeof(none));
  s = ffn_impl(c, none, nullptr, x, w13, w2, nullptr, w.h, w.out, side, c.E, c.n_shared);
  e = cudaEventRecord(join, side);
  // main stream: layout, permute, routed experts
  if (s == MOE_OK)
    s = cuda_status(launch_layout(c, expert_owner, w.ids, L, dev_status, w.lay_ws, st), "layout");
  if (s == MOE_OK) s = cuda_status(launch_permute(c, L, x, w.x_perm, st), "permute");
  if (s == MOE_OK) s = ffn_impl(c, L, w.x_perm, x, w13, w2, w.w, w.h, w.out, st, 0, c.E);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, join, 0);  // join even after an error
  cudaEventDestroy(fork);
  cudaEventDestroy(join);
  if (s != MOE_OK) return s;
  if (e != cudaSuccess) return cuda_status(e, "join");
  return cuda_status(launch_combine(c, L, w.out, nullptr, y, st), "combine");
}

}  // extern "C"

namespace {

// ------------------------------------------------------------------ chunked pipeline
// The tokens in n_chunks contiguous chunks, each a layer of its own after one router
// launch over all of them ([EP-DeepEP] §7: T = T_warm + sum over chunks of max(T_disp,
// T_exp, T_comb) + T_drain).  Chunk c's layout and permute run on `stream` beside chunk
// c-1's expert FFN on `side_stream`; chunk c-1's combine follows on `stream`.
constexpr int kMaxChunks = 16;

struct ChunkPlan {
  int n_chunks, per;  // tokens per chunk (the last one may hold fewer)
  moe_config cc[kMaxChunks];
  size_t off[kMaxChunks];  // workspace offset of each chunk's buffers
  size_t route_bytes, total;
};

ChunkPlan plan_chunks(const moe_config& c, int n_chunks) {
  ChunkPlan pl;
  memset(&pl, 0, sizeof(pl));
  pl.n_chunks = n_chunks;
  pl.per = (c.N + n_chunks - 1) / n_chunks;
  // routing of all tokens: logits, ids, gates
  const size_t A = (size_t)c.N * c.k;
  pl.route_bytes = align256((size_t)c.N * c.E * 4) + 2 * align256(A * 4 ? A * 4 : 1);
  size_t off = pl.route_bytes;
  for (int i = 0; i < n_chunks; ++i) {
    pl.cc[i] = c;
    const int t0 = i * pl.per;
    pl.cc[i].N = t0 >= c.N ? 0 : (c.N - t0 < pl.per ? c.N - t0 : pl.per);
    pl.off[i] = off;
    off += carve_forward(pl.cc[i], nullptr).total;
  }
  pl.total = off;
  return pl;
}

}  // namespace

extern "C" {

size_t moe_workspace_bytes_chunked(const moe_config* cfg, int32_t n_chunks) {
  if (check_config(cfg) != MOE_OK || n_chunks < 1 || n_chunks > kMaxChunks) return 0;
  return plan_chunks(*cfg, n_chunks).total;
}

moe_status moe_layer_forward_chunked(const moe_config* cfg, int32_t n_chunks, const void* x, const void* w_gate,
                                     const float* bias, const int32_t* expert_owner, const void* w13, const void* w2,
                                     void* y, int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream,
                                     moe_stream_t side_stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_router(*cfg)) != MOE_OK) return s;
  if ((s = check_owner(*cfg, expert_owner)) != MOE_OK) return s;
  if (n_chunks < 1 || n_chunks > kMaxChunks) return fail(MOE_ERR_INVALID_ARG, "n_chunks must be in [1, 16]");
  const moe_config& c = *cfg;
  const ChunkPlan pl = plan_chunks(c, n_chunks);
  if (!ws || ws_bytes < pl.total) return fail(MOE_ERR_WORKSPACE, "chunked forward workspace too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (c.N == 0) return MOE_OK;
  if (!x || !w_gate || !w13 || !w2 || !y) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  cudaStream_t st = (cudaStream_t)stream, side = (cudaStream_t)side_stream;
  char* base = static_cast<char*>(ws);
  const size_t A = (size_t)c.N * c.k;
  float* logits = reinterpret_cast<float*>(base);
  int32_t* ids = reinterpret_cast<int32_t*>(base + align256((size_t)c.N * c.E * 4));
  float* gates = reinterpret_cast<float*>(reinterpret_cast<char*>(ids) + align256(A * 4));
  if ((s = route_impl(c, x, w_gate, bias, logits, ids, gates, st)) != MOE_OK) return s;
  const size_t xrow = (size_t)c.d * elem_bytes(c);
  cudaEvent_t ev[2 * kMaxChunks];
  int n_ev = 0;
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 2 * n_chunks && e == cudaSuccess; ++i) {
    e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
    if (e == cudaSuccess) ++n_ev;
  }
  FwdWs w[kMaxChunks];
  const char* xs[kMaxChunks];
  auto combine_chunk = [&](int i) -> moe_status {  // on `stream`, after chunk i's FFN
    if (pl.cc[i].N == 0) return MOE_OK;
    cudaError_t ee = cudaStreamWaitEvent(st, ev[n_chunks + i], 0);
    if (ee != cudaSuccess) return cuda_status(ee, "chunk join");
    return cuda_status(launch_combine(pl.cc[i], w[i].lay, w[i].out, nullptr,
                                      static_cast<char*>(y) + (size_t)i * pl.per * xrow, st),
                       "combine");
  };
  s = e == cudaSuccess ? MOE_OK : cuda_status(e, "chunk events");
  for (int i = 0; i < n_chunks && s == MOE_OK; ++i) {
    const moe_config& cc = pl.cc[i];
    w[i] = carve_forward(cc, base + pl.off[i]);
    xs[i] = static_cast<const char*>(x) + (size_t)i * pl.per * xrow;
    if (cc.N > 0) {
      // stream: this chunk's layout and permute (beside the FFN of the chunk before)
      const int32_t* ids_i = ids + (size_t)i * pl.per * c.k;
      s = cuda_status(launch_layout(cc, expert_owner, ids_i, w[i].lay, dev_status, w[i].lay_ws, st), "layout");
      if (s == MOE_OK) s = cuda_status(launch_permute(cc, w[i].lay, xs[i], w[i].x_perm, st), "permute");
      if (s == MOE_OK) s = cuda_status(cudaEventRecord(ev[i], st), "chunk fork");
      // side stream: its experts (routed rows, then the shared experts over its tokens)
      if (s == MOE_OK) s = cuda_status(cudaStreamWaitEvent(side, ev[i], 0), "chunk fork");
      if (s == MOE_OK)
        s = ffn_impl(cc, w[i].lay, w[i].x_perm, xs[i], w13, w2, gates + (size_t)i * pl.per * c.k, w[i].h,
                     w[i].out, side);
    }
    if (s == MOE_OK) s = cuda_status(cudaEventRecord(ev[n_chunks + i], side), "chunk done");
    // stream: the combine of the chunk before, now that this chunk's movement is queued
    if (s == MOE_OK && i > 0) s = combine_chunk(i - 1);
  }
  if (s == MOE_OK) s = combine_chunk(n_chunks - 1);
  // whatever happened, `stream` orders after all the side stream's work
  if (n_ev == 2 * n_chunks && cudaEventRecord(ev[0], side) == cudaSuccess) cudaStreamWaitEvent(st, ev[0], 0);
  for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
  return s;
}

size_t moe_eplb_workspace_bytes(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return eplb_ws_bytes(*cfg);
}

moe_status moe_eplb_plan(int32_t E, int32_t R, int32_t P, const int64_t* load, int32_t* copies,
                         int32_t* replica_off, int32_t* replica_slots, int32_t* slot_expert, int32_t* slot_owner,
                         int64_t* owner_load) {
  if (E < 1 || R < 0 || P < 1) return fail(MOE_ERR_INVALID_ARG, "need E >= 1, R >= 0, P >= 1");
  if ((E + R) % P != 0) return fail(MOE_ERR_INVALID_ARG, "E + R must be a multiple of P");
  if (E + R > kMaxSlots) return fail(MOE_ERR_UNSUPPORTED, "E + R <= 512");
  if (!load || !copies || !replica_off || !replica_slots || !slot_expert || !slot_owner || !owner_load)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  for (int e = 0; e < E; ++e)
    if (load[e] < 0 || load[e] > (1LL << 40)) return fail(MOE_ERR_INVALID_ARG, "load out of range [0, 2^40]");
  return eplb_plan(E, R, P, load, copies, replica_off, replica_slots, slot_expert, slot_owner, owner_load);
}

moe_status moe_eplb_assign(const moe_config* cfg, const int32_t* topk_ids, const int32_t* replica_off,
                           const int32_t* replica_slots, int32_t n_slots, int32_t* phys_ids, int32_t* dev_status,
                           void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (n_slots < cfg->E || n_slots > kMaxSlots) return fail(MOE_ERR_INVALID_ARG, "need E <= n_slots <= 512");
  if (!replica_off || !replica_slots || (cfg->N > 0 && (!topk_ids || !phys_ids)))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!ws || ws_bytes < eplb_ws_bytes(*cfg)) return fail(MOE_ERR_WORKSPACE, "EPLB workspace too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  return cuda_status(launch_eplb_assign(*cfg, topk_ids, replica_off, replica_slots, n_slots, phys_ids, dev_status,
                                        ws, (cudaStream_t)stream),
                     "eplb assign");
}

moe_status moe_eplb_place_weights(const int32_t* slot_expert, int32_t n_slots, int32_t E, int32_t n_shared,
                                  size_t expert_bytes, const void* w_logical, void* w_physical, moe_stream_t stream) {
  if (n_slots < 1 || n_slots > kMaxSlots || E < 1 || n_shared < 0 || n_shared > kMaxShared)
    return fail(MOE_ERR_INVALID_ARG, "need 1 <= n_slots <= 512, E >= 1, 0 <= n_shared <= 8");
  if (!slot_expert || !w_logical || !w_physical) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  for (int i = 0; i < n_slots; ++i)
    if (slot_expert[i] < 0 || slot_expert[i] >= E) return fail(MOE_ERR_INVALID_ARG, "slot_expert out of [0, E)");
  const char* src = static_cast<const char*>(w_logical);
  char* dst = static_cast<char*>(w_physical);
  cudaStream_t st = (cudaStream_t)stream;
  for (int i = 0; i < n_slots; ++i) {
    cudaError_t e = cudaMemcpyAsync(dst + (size_t)i * expert_bytes, src + (size_t)slot_expert[i] * expert_bytes,
                                    expert_bytes, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_status(e, "eplb place weights");
  }
  if (n_shared > 0) {
    cudaError_t e = cudaMemcpyAsync(dst + (size_t)n_slots * expert_bytes, src + (size_t)E * expert_bytes,
                                    (size_t)n_shared * expert_bytes, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_status(e, "eplb place weights");
  }
  return MOE_OK;
}

moe_status moe_quantize_fp8(const void* src, int64_t rows, int32_t cols, void* dst, float* scale,
                            moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 8 != 0) return fail(MOE_ERR_INVALID_ARG, "need rows >= 0, cols % 8 == 0");
  if (rows > 0 && (!src || !dst || !scale)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_quantize_rows(src, rows, cols, dst, scale, (cudaStream_t)stream), "fp8 quantisation");
}

moe_status moe_permute_fp8(const moe_config* cfg, const moe_layout* layout, const void* x_q, void* x_q_perm,
                           moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (cfg->d % 16 != 0) return fail(MOE_ERR_UNSUPPORTED, "fp8 rows need d % 16 == 0");
  if (!layout || !layout->tok2row || !x_q || !x_q_perm) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_permute_bytes(*cfg, *layout, x_q, x_q_perm, cfg->d, (cudaStream_t)stream),
                     "permute (fp8)");
}

static moe_status check_fp8(const moe_config* cfg) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "the FP8 path takes a bf16 configuration");
  if (cfg->d % 16 != 0 || cfg->I % 16 != 0) return fail(MOE_ERR_UNSUPPORTED, "fp8 rows need d, I % 16 == 0");
  return MOE_OK;
}

moe_status moe_grouped_ffn_fp8(const moe_config* cfg, const moe_layout* layout, const void* x_q_perm,
                               const void* x_q, const float* x_scale, const void* w13_q, const float* w13_scale,
                               const void* w2_q, const float* w2_scale, const float* topk_w, void* h, void* h_q,
                               float* h_scale, void* out, moe_stream_t stream) {
  moe_status s = check_fp8(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout_complete(layout) || !x_q_perm || !x_scale || !w13_q || !w13_scale || !w2_q || !w2_scale ||
      !h || !h_q || !h_scale || !out || (cfg->n_shared > 0 && !x_q))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  Fp8Ffn f{x_q_perm, x_q, x_scale, w13_q, w13_scale, w2_q, w2_scale, topk_w, h, h_q, h_scale, out};
  return ffn_fp8_impl(*cfg, *layout, f, (cudaStream_t)stream);
}

size_t moe_workspace_bytes_fp8(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return carve_forward(*cfg, nullptr, true).total;
}

static moe_status forward_fp8(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                              const int32_t* expert_owner, const void* w13_q, const float* w13_scale,
                              const void* w2_q, const float* w2_scale, void* y, const moe_layout* layout_out,
                              int32_t* dev_status, void* ws, size_t ws_bytes, cudaStream_t st, cudaStream_t side) {
  moe_status s = check_fp8(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_router(*cfg)) != MOE_OK) return s;
  if ((s = check_owner(*cfg, expert_owner)) != MOE_OK) return s;
  const moe_config& c = *cfg;
  FwdWs w = carve_forward(c, nullptr, true);
  if (!ws || ws_bytes < w.total) return fail(MOE_ERR_WORKSPACE, "forward workspace too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (layout_out && !layout_complete(layout_out)) return fail(MOE_ERR_INVALID_ARG, "incomplete layout_out");
  if (c.N > 0 && (!x || !w_gate || !w13_q || !w13_scale || !w2_q || !w2_scale || !y))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  w = carve_forward(c, static_cast<char*>(ws), true);
  const moe_layout& L = layout_out ? *layout_out : w.lay;
  if (c.N > 0 && (s = route_impl(c, x, w_gate, bias, w.logits, w.ids, w.w, st)) != MOE_OK) return s;
  if (c.N > 0 && (s = cuda_status(launch_quantize_rows(x, c.N, c.d, w.x_q, w.x_scale, st), "x quantisation")) !=
                     MOE_OK)
    return s;
  Fp8Ffn f{w.x_perm, w.x_q, w.x_scale, w13_q, w13_scale, w2_q, w2_scale, w.w, w.h, w.h_q, w.h_scale, w.out};
  const bool overlap = side != nullptr && side != st && c.n_shared > 0 && c.N > 0;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaError_t e = cudaSuccess;
  if (overlap) {  // the shared experts read only x_q: they run on the side stream
    e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
    if (e != cudaSuccess) {
      if (fork) cudaEventDestroy(fork);
      if (join) cudaEventDestroy(join);
      return cuda_status(e, "fork");
    }
    s = ffn_fp8_impl(c, L, f, side, c.E, c.n_shared);
    e = cudaEventRecord(join, side);
  }
  if (s == MOE_OK)
    s = cuda_status(launch_layout(c, expert_owner, w.ids, L, dev_status, w.lay_ws, st), "layout");
  if (s == MOE_OK && c.N > 0)
    s = cuda_status(launch_permute_bytes(c, L, w.x_q, w.x_perm, c.d, st), "permute (fp8)");
  if (s == MOE_OK && c.N > 0) s = overlap ? ffn_fp8_impl(c, L, f, st, 0, c.E) : ffn_fp8_impl(c, L, f, st);
  if (overlap) {
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, join, 0);  // join even after an error
    cudaEventDestroy(fork);
    cudaEventDestroy(join);
  }
  if (s != MOE_OK) return s;
  if (e != cudaSuccess) return cuda_status(e, "join");
  if (c.N == 0) return MOE_OK;
  return cuda_status(launch_combine(c, L, w.out, nullptr, y, st), "combine");
}

moe_status moe_layer_forward_fp8(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                                 const int32_t* expert_owner, const void* w13_q, const float* w13_scale,
                                 const void* w2_q, const float* w2_scale, void* y, const moe_layout* layout_out,
                                 int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return forward_fp8(cfg, x, w_gate, bias, expert_owner, w13_q, w13_scale, w2_q, w2_scale, y, layout_out,
                     dev_status, ws, ws_bytes, (cudaStream_t)stream, nullptr);
}

moe_status moe_layer_forward_fp8_overlapped(const moe_config* cfg, const void* x, const void* w_gate,
                                            const float* bias, const int32_t* expert_owner, const void* w13_q,
                                            const float* w13_scale, const void* w2_q, const float* w2_scale, void* y,
                                            const moe_layout* layout_out, int32_t* dev_status, void* ws,
                                            size_t ws_bytes, moe_stream_t stream, moe_stream_t side_stream) {
  return forward_fp8(cfg, x, w_gate, bias, expert_owner, w13_q, w13_scale, w2_q, w2_scale, y, layout_out,
                     dev_status, ws, ws_bytes, (cudaStream_t)stream, (cudaStream_t)side_stream);
}

moe_status moe_quantize_mx(const void* src, int64_t rows, int32_t cols, void* dst, uint8_t* sf,
                           moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0) return fail(MOE_ERR_INVALID_ARG, "need rows >= 0, cols % 32 == 0");
  if (rows > 0 && (!src || !dst || !sf)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (rows > 0 && ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) != 0)
    return fail(MOE_ERR_INVALID_ARG, "src and dst must be 16-byte aligned");
  return cuda_status(launch_quantize_mx(src, rows, cols, dst, sf, (cudaStream_t)stream), "mx quantisation");
}

static moe_status check_mx(const moe_config* cfg) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (cfg->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "the MX path takes a bf16 configuration");
  if (cfg->d % 512 != 0 || cfg->I % 128 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "the MX path needs d % 512 == 0 and I % 128 == 0");
  return MOE_OK;
}

moe_status moe_permute_mx(const moe_config* cfg, const moe_layout* layout, const void* x_q, const uint8_t* x_sf,
                          void* x_q_perm, uint8_t* x_sf_perm, moe_stream_t stream) {
  moe_status s = check_mx(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout->tok2row || !x_q || !x_sf || !x_q_perm || !x_sf_perm)
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  const cudaStream_t st = (cudaStream_t)stream;
  s = cuda_status(launch_permute_bytes(*cfg, *layout, x_q, x_q_perm, cfg->d, st), "permute (mx codes)");
  if (s != MOE_OK) return s;
  return cuda_status(launch_permute_bytes(*cfg, *layout, x_sf, x_sf_perm, cfg->d / 32, st), "permute (mx scales)");
}

moe_status moe_grouped_ffn_mx(const moe_config* cfg, const moe_layout* layout, const void* x_q_perm,
                              const uint8_t* x_sf_perm, const void* x_q, const uint8_t* x_sf, const void* w13_q,
                              const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf, const float* topk_w,
                              void* h, void* h_q, uint8_t* h_sf, void* out, moe_stream_t stream) {
  moe_status s = check_mx(cfg);
  if (s != MOE_OK) return s;
  if (cfg->N == 0) return MOE_OK;
  if (!layout || !layout_complete(layout) || !x_q_perm || !x_sf_perm || !w13_q || !w13_sf || !w2_q || !w2_sf ||
      !h || !h_q || !h_sf || !out || (cfg->n_shared > 0 && (!x_q || !x_sf)))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  MxFfn f{x_q_perm, x_sf_perm, x_q, x_sf, w13_q, w13_sf, w2_q, w2_sf, topk_w, h, h_q, h_sf, out};
  return ffn_mx_impl(*cfg, *layout, f, (cudaStream_t)stream);
}

size_t moe_workspace_bytes_mx(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return carve_forward(*cfg, nullptr, true, true).total;
}

static moe_status forward_mx(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                             const int32_t* expert_owner, const void* w13_q, const uint8_t* w13_sf, const void* w2_q,
                             const uint8_t* w2_sf, void* y, const moe_layout* layout_out, int32_t* dev_status,
                             void* ws, size_t ws_bytes, cudaStream_t st, cudaStream_t side) {
  moe_status s = check_mx(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_router(*cfg)) != MOE_OK) return s;
  if ((s = check_owner(*cfg, expert_owner)) != MOE_OK) return s;
  const moe_config& c = *cfg;
  FwdWs w = carve_forward(c, nullptr, true, true);
  if (!ws || ws_bytes < w.total) return fail(MOE_ERR_WORKSPACE, "forward workspace too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (layout_out && !layout_complete(layout_out)) return fail(MOE_ERR_INVALID_ARG, "incomplete layout_out");
  if (c.N > 0 && (!x || !w_gate || !w13_q || !w13_sf || !w2_q || !w2_sf || !y))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (c.N == 0) return MOE_OK;
  w = carve_forward(c, static_cast<char*>(ws), true, true);
  const moe_layout& L = layout_out ? *layout_out : w.lay;
  if ((s = route_impl(c, x, w_gate, bias, w.logits, w.ids, w.w, st)) != MOE_OK) return s;
  if ((s = cuda_status(launch_quantize_mx(x, c.N, c.d, w.x_q, w.x_sf, st), "x quantisation (mx)")) != MOE_OK)
    return s;
  // h is quantised by FC1's epilogue and not kept in bf16
  MxFfn f{w.x_perm, w.x_sf_perm, w.x_q, w.x_sf, w13_q, w13_sf, w2_q, w2_sf, w.w, nullptr, w.h_q, w.h_sf, w.out};
  const bool overlap = side != nullptr && side != st && c.n_shared > 0;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaError_t e = cudaSuccess;
  if (overlap) {  // the shared experts read only x's codes and scales: they run on the side stream
    e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side, fork, 0);
    if (e != cudaSuccess) {
      if (fork) cudaEventDestroy(fork);
      if (join) cudaEventDestroy(join);
      return cuda_status(e, "fork");
    }
    s = ffn_mx_impl(c, L, f, side, c.E, c.n_shared);
    e = cudaEventRecord(join, side);
  }
  if (s == MOE_OK) s = cuda_status(launch_layout(c, expert_owner, w.ids, L, dev_status, w.lay_ws, st), "layout");
  if (s == MOE_OK) s = cuda_status(launch_permute_bytes(c, L, w.x_q, w.x_perm, c.d, st), "permute (mx codes)");
  if (s == MOE_OK)
    s = cuda_status(launch_permute_bytes(c, L, w.x_sf, w.x_sf_perm, c.d / 32, st), "permute (mx scales)");
  if (s == MOE_OK) s = overlap ? ffn_mx_impl(c, L, f, st, 0, c.E) : ffn_mx_impl(c, L, f, st);
  if (overlap) {
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, join, 0);  // join even after an error
    cudaEventDestroy(fork);
    cudaEventDestroy(join);
  }
  if (s != MOE_OK) return s;
  if (e != cudaSuccess) return cuda_status(e, "join");
  return cuda_status(launch_combine(c, L, w.out, nullptr, y, st), "combine");
}

moe_status moe_layer_forward_mx(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                                const int32_t* expert_owner, const void* w13_q, const uint8_t* w13_sf,
                                const void* w2_q, const uint8_t* w2_sf, void* y, const moe_layout* layout_out,
                                int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return forward_mx(cfg, x, w_gate, bias, expert_owner, w13_q, w13_sf, w2_q, w2_sf, y, layout_out, dev_status, ws,
                    ws_bytes, (cudaStream_t)stream, nullptr);
}

moe_status moe_layer_forward_mx_overlapped(const moe_config* cfg, const void* x, const void* w_gate,
                                           const float* bias, const int32_t* expert_owner, const void* w13_q,
                                           const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf, void* y,
                                           const moe_layout* layout_out, int32_t* dev_status, void* ws,
                                           size_t ws_bytes, moe_stream_t stream, moe_stream_t side_stream) {
  return forward_mx(cfg, x, w_gate, bias, expert_owner, w13_q, w13_sf, w2_q, w2_sf, y, layout_out, dev_status, ws,
                    ws_bytes, (cudaStream_t)stream, (cudaStream_t)side_stream);
}

size_t moe_ep_window_bytes(const moe_config* cfg, int32_t capacity) {
  if (check_config(cfg) != MOE_OK || capacity < 1) return 0;
  return ep_offsets(*cfg, capacity).total;
}

size_t moe_ep_workspace_bytes(const moe_config* cfg, int32_t capacity) {
  if (check_config(cfg) != MOE_OK || capacity < 1) return 0;
  return carve_ep(*cfg, capacity, nullptr).total;
}

moe_status moe_ep_window_layout(const moe_config* cfg, int32_t capacity, size_t* offsets) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (capacity < 1 || !offsets) return fail(MOE_ERR_INVALID_ARG, "capacity < 1 or NULL offsets");
  const EpOffsets o = ep_offsets(*cfg, capacity);
  const size_t v[11] = {o.cnt_flag, o.disp_flag, o.done_flag, o.step,   o.disp_ctr, o.err_step,
                        o.cnt_tab,  o.gate,      o.scale,     o.x_recv, o.out_recv};
  memcpy(offsets, v, sizeof(v));
  return MOE_OK;
}

typedef CUresult (*GetAddressRange)(CUdeviceptr*, size_t*, CUdeviceptr);

moe_status moe_ep_ipc_handle(const void* window, void* handle, size_t* offset) {
  if (!window || !handle || !offset) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return fail(MOE_ERR_CUDA, "cuMemGetAddressRange unavailable");
  CUdeviceptr base = 0;
  size_t size = 0;
  if (reinterpret_cast<GetAddressRange>(fn)(&base, &size, reinterpret_cast<CUdeviceptr>(window)) != CUDA_SUCCESS)
    return fail(MOE_ERR_INVALID_ARG, "window is not device memory");
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return cuda_status(e, "cudaIpcGetMemHandle");
  static_assert(sizeof(h) == 64, "CUDA IPC handles are 64 bytes");
  memcpy(handle, &h, sizeof(h));
  *offset = reinterpret_cast<CUdeviceptr>(window) - base;
  return MOE_OK;
}

moe_status moe_ep_ipc_open(const void* handle, size_t offset, void** window) {
  if (!handle || !window) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_status(e, "cudaIpcOpenMemHandle");
  *window = static_cast<char*>(base) + offset;
  return MOE_OK;
}

moe_status moe_ep_ipc_close(void* window, size_t offset) {
  if (!window) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(cudaIpcCloseMemHandle(static_cast<char*>(window) - offset), "cudaIpcCloseMemHandle");
}

moe_status moe_ep_notify(const moe_config* cfg, const moe_ep_group* grp, const int32_t* topk_ids,
                         int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream) {
  EpPeers peers;
  moe_status s = check_ep(cfg, grp, &peers);
  if (s != MOE_OK) return s;
  if ((s = check_ep_ws(*cfg, grp, ws, ws_bytes)) != MOE_OK) return s;
  if (cfg->N > 0 && !topk_ids) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return ep_notify_impl(*cfg, *grp, peers, topk_ids, dev_status, carve_ep(*cfg, grp->capacity, (char*)ws),
                        (cudaStream_t)stream);
}

moe_status moe_ep_layout(const moe_config* cfg, const moe_ep_group* grp, const int32_t* expert_owner,
                         const int32_t* topk_ids, const moe_ep_handle* handle, int32_t* dev_status, void* ws,
                         size_t ws_bytes, moe_stream_t stream) {
  EpPeers peers;
  moe_status s = check_ep(cfg, grp, &peers);
  if (s != MOE_OK) return s;
  if ((s = check_owner(*cfg, expert_owner)) != MOE_OK) return s;
  if ((s = check_ep_ws(*cfg, grp, ws, ws_bytes)) != MOE_OK) return s;
  if (!handle_complete(handle) || (cfg->N > 0 && !topk_ids)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return ep_layout_impl(*cfg, *grp, peers, expert_owner, topk_ids, *handle, dev_status,
                        carve_ep(*cfg, grp->capacity, (char*)ws), (cudaStream_t)stream);
}

moe_status moe_ep_dispatch(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                           const float* topk_w, const moe_ep_handle* handle, moe_stream_t stream) {
  EpPeers peers;
  moe_status s = check_ep(cfg, grp, &peers);
  if (s != MOE_OK) return s;
  if (!handle_complete(handle) || (cfg->N > 0 && (!x || !topk_w))) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_ep_dispatch(*cfg, peers, ep_offsets(*cfg, grp->capacity), grp->rank, grp->capacity, x,
                                        handle->dest, topk_w, nullptr, cfg->d * elem_bytes(*cfg),
                                        (cudaStream_t)stream),
                     "EP dispatch");
}

moe_status moe_ep_expert_ffn(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                             const void* w13, const void* w2, const moe_ep_handle* handle, int32_t* dev_status,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
  EpPeers peers;
  moe_status s = check_ep(cfg, grp, &peers);
  if (s != MOE_OK) return s;
  if ((s = check_ep_ws(*cfg, grp, ws, ws_bytes)) != MOE_OK) return s;
  const bool any = grp->local_experts > 0 || (cfg->N > 0 && cfg->n_shared > 0);
  if (!handle_complete(handle) || (any && (!w13 || !w2)) || (cfg->N > 0 && cfg->n_shared > 0 && !x))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  const EpFfn f = {false, x, nullptr, w13, nullptr, w2, nullptr};
  return ep_ffn_impl(*cfg, *grp, peers, f, *handle, dev_status, carve_ep(*cfg, grp->capacity, (char*)ws),
                     (cudaStream_t)stream, ep_groups(*cfg, *grp));
}

moe_status moe_ep_combine(const moe_config* cfg, const moe_ep_group* grp, const moe_ep_handle* handle,
                          void* y, int32_t* dev_status, moe_stream_t stream) {
  EpPeers peers;
  moe_status s = check_ep(cfg, grp, &peers);
  if (s != MOE_OK) return s;
  if (!handle_complete(handle) || (cfg->N > 0 && !y)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_ep_combine(*cfg, peers, ep_offsets(*cfg, grp->capacity), grp->rank, grp->capacity,
                                       handle->dest, y, dev_status, (cudaStream_t)stream),
                     "EP combine");
}

static moe_status ep_layer(const moe_config* cfg, const moe_ep_group* grp, const void* x, const void* w_gate,
                           const float* bias, const int32_t* expert_owner, const EpFfn& f, void* y,
                           const moe_ep_handle* handle_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                           moe_stream_t stream, moe_stream_t side) {
  moe_status s = f.mx ? check_mx(cfg) : (f.fp8 ? check_fp8(cfg) : check_config(cfg));
  if (s != MOE_OK) return s;
  EpPeers peers;
  if ((s = check_ep(cfg, grp, &peers)) != MOE_OK) return s;
  if ((s = check_router(*cfg)) != MOE_OK) return s;
  if ((s = check_owner(*cfg, expert_owner)) != MOE_OK) return s;
  if ((s = check_ep_ws(*cfg, grp, ws, ws_bytes, f.fp8, f.mx)) != MOE_OK) return s;
  if (handle_out && !handle_complete(handle_out)) return fail(MOE_ERR_INVALID_ARG, "incomplete handle_out");
  const moe_config& c = *cfg;
  const bool any = grp->local_experts > 0 || (c.N > 0 && c.n_shared > 0);
  if ((c.N > 0 && (!x || !w_gate || !y)) || (any && (!f.w13 || !f.w2)) ||
      (any && f.fp8 && (!f.w13_scale || !f.w2_scale)) || (any && f.mx && (!f.w13_sf || !f.w2_sf)))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return ep_forward(c, *grp, peers, x, w_gate, bias, expert_owner, f, y, handle_out, dev_status,
                    carve_ep(c, grp->capacity, static_cast<char*>(ws), f.fp8, f.mx), (cudaStream_t)stream,
                    (cudaStream_t)side);
}

moe_status moe_ep_layer_forward(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                                const void* w_gate, const float* bias, const int32_t* expert_owner, const void* w13,
                                const void* w2, void* y, const moe_ep_handle* handle_out, int32_t* dev_status,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
  const EpFfn f = {false, nullptr, nullptr, w13, nullptr, w2, nullptr};
  return ep_layer(cfg, grp, x, w_gate, bias, expert_owner, f, y, handle_out, dev_status, ws, ws_bytes, stream,
                  nullptr);
}

moe_status moe_ep_layer_forward_overlapped(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                                           const void* w_gate, const float* bias, const int32_t* expert_owner,
                                           const void* w13, const void* w2, void* y, const moe_ep_handle* handle_out,
                                           int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream,
                                           moe_stream_t side_stream) {
  const EpFfn f = {false, nullptr, nullptr, w13, nullptr, w2, nullptr};
  return ep_layer(cfg, grp, x, w_gate, bias, expert_owner, f, y, handle_out, dev_status, ws, ws_bytes, stream,
                  side_stream);
}

size_t moe_ep_workspace_bytes_fp8(const moe_config* cfg, int32_t capacity) {
  if (check_fp8(cfg) != MOE_OK || capacity < 1) return 0;
  return carve_ep(*cfg, capacity, nullptr, true).total;
}

moe_status moe_ep_dispatch_fp8(const moe_config* cfg, const moe_ep_group* grp, const void* x_q, const float* x_scale,
                               const float* topk_w, const moe_ep_handle* handle, moe_stream_t stream) {
  moe_status s = check_fp8(cfg);
  if (s != MOE_OK) return s;
  EpPeers peers;
  if ((s = check_ep(cfg, grp, &peers)) != MOE_OK) return s;
  if (!handle_complete(handle) || (cfg->N > 0 && (!x_q || !x_scale || !topk_w)))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_ep_dispatch(*cfg, peers, ep_offsets(*cfg, grp->capacity), grp->rank, grp->capacity, x_q,
                                        handle->dest, topk_w, x_scale, cfg->d, (cudaStream_t)stream),
                     "EP dispatch (fp8)");
}

moe_status moe_ep_expert_ffn_fp8(const moe_config* cfg, const moe_ep_group* grp, const void* x_q, const float* x_scale,
                                 const void* w13_q, const float* w13_scale, const void* w2_q, const float* w2_scale,
                                 const moe_ep_handle* handle, int32_t* dev_status, void* ws, size_t ws_bytes,
                                 moe_stream_t stream) {
  moe_status s = check_fp8(cfg);
  if (s != MOE_OK) return s;
  EpPeers peers;
  if ((s = check_ep(cfg, grp, &peers)) != MOE_OK) return s;
  if ((s = check_ep_ws(*cfg, grp, ws, ws_bytes, true)) != MOE_OK) return s;
  const bool any = grp->local_experts > 0 || (cfg->N > 0 && cfg->n_shared > 0);
  if (!handle_complete(handle) || (any && (!w13_q || !w13_scale || !w2_q || !w2_scale)) ||
      (cfg->N > 0 && cfg->n_shared > 0 && (!x_q || !x_scale)))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  const EpFfn f = {true, x_q, x_scale, w13_q, w13_scale, w2_q, w2_scale};
  return ep_ffn_impl(*cfg, *grp, peers, f, *handle, dev_status, carve_ep(*cfg, grp->capacity, (char*)ws, true),
                     (cudaStream_t)stream, ep_groups(*cfg, *grp));
}

moe_status moe_ep_layer_forward_fp8(const moe_config* cfg, const moe_ep_group* grp, const void* x, const void* w_gate,
                                    const float* bias, const int32_t* expert_owner, const void* w13_q,
                                    const float* w13_scale, const void* w2_q, const float* w2_scale, void* y,
                                    const moe_ep_handle* handle_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  const EpFfn f = {true, nullptr, nullptr, w13_q, w13_scale, w2_q, w2_scale};
  return ep_layer(cfg, grp, x, w_gate, bias, expert_owner, f, y, handle_out, dev_status, ws, ws_bytes, stream,
                  nullptr);
}

moe_status moe_ep_layer_forward_fp8_overlapped(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                                               const void* w_gate, const float* bias, const int32_t* expert_owner,
                                               const void* w13_q, const float* w13_scale, const void* w2_q,
                                               const float* w2_scale, void* y, const moe_ep_handle* handle_out,
                                               int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream,
                                               moe_stream_t side_stream) {
  const EpFfn f = {true, nullptr, nullptr, w13_q, w13_scale, w2_q, w2_scale};
  return ep_layer(cfg, grp, x, w_gate, bias, expert_owner, f, y, handle_out, dev_status, ws, ws_bytes, stream,
                  side_stream);
}

size_t moe_ep_workspace_bytes_mx(const moe_config* cfg, int32_t capacity) {
  if (check_mx(cfg) != MOE_OK || capacity < 1) return 0;
  return carve_ep(*cfg, capacity, nullptr, false, true).total;
}

moe_status moe_ep_dispatch_mx(const moe_config* cfg, const moe_ep_group* grp, const void* x_q, const uint8_t* x_sf,
                              const float* topk_w, const moe_ep_handle* handle, moe_stream_t stream) {
  moe_status s = check_mx(cfg);
  if (s != MOE_OK) return s;
  EpPeers peers;
  if ((s = check_ep(cfg, grp, &peers)) != MOE_OK) return s;
  if (!handle_complete(handle) || (cfg->N > 0 && (!x_q || !x_sf || !topk_w)))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  return cuda_status(launch_ep_dispatch(*cfg, peers, ep_offsets(*cfg, grp->capacity), grp->rank, grp->capacity, x_q,
                                        handle->dest, topk_w, nullptr, cfg->d, (cudaStream_t)stream, x_sf,
                                        cfg->d / 32),
                     "EP dispatch (mx)");
}

moe_status moe_ep_expert_ffn_mx(const moe_config* cfg, const moe_ep_group* grp, const void* x_q, const uint8_t* x_sf,
                                const void* w13_q, const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf,
                                const moe_ep_handle* handle, int32_t* dev_status, void* ws, size_t ws_bytes,
                                moe_stream_t stream) {
  moe_status s = check_mx(cfg);
  if (s != MOE_OK) return s;
  EpPeers peers;
  if ((s = check_ep(cfg, grp, &peers)) != MOE_OK) return s;
  if ((s = check_ep_ws(*cfg, grp, ws, ws_bytes, false, true)) != MOE_OK) return s;
  const bool any = grp->local_experts > 0 || (cfg->N > 0 && cfg->n_shared > 0);
  if (!handle_complete(handle) || (any && (!w13_q || !w13_sf || !w2_q || !w2_sf)) ||
      (cfg->N > 0 && cfg->n_shared > 0 && (!x_q || !x_sf)))
    return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  EpFfn f = {false, x_q, nullptr, w13_q, nullptr, w2_q, nullptr};
  f.mx = true;
  f.x_sf = x_sf;
  f.w13_sf = w13_sf;
  f.w2_sf = w2_sf;
  return ep_ffn_impl(*cfg, *grp, peers, f, *handle, dev_status,
                     carve_ep(*cfg, grp->capacity, (char*)ws, false, true), (cudaStream_t)stream,
                     ep_groups(*cfg, *grp));
}

static EpFfn mx_weights(const void* w13_q, const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf) {
  EpFfn f = {false, nullptr, nullptr, w13_q, nullptr, w2_q, nullptr};
  f.mx = true;
  f.w13_sf = w13_sf;
  f.w2_sf = w2_sf;
  return f;
}

moe_status moe_ep_layer_forward_mx(const moe_config* cfg, const moe_ep_group* grp, const void* x, const void* w_gate,
                                   const float* bias, const int32_t* expert_owner, const void* w13_q,
                                   const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf, void* y,
                                   const moe_ep_handle* handle_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                                   moe_stream_t stream) {
  return ep_layer(cfg, grp, x, w_gate, bias, expert_owner, mx_weights(w13_q, w13_sf, w2_q, w2_sf), y, handle_out,
                  dev_status, ws, ws_bytes, stream, nullptr);
}

moe_status moe_ep_layer_forward_mx_overlapped(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                                              const void* w_gate, const float* bias, const int32_t* expert_owner,
                                              const void* w13_q, const uint8_t* w13_sf, const void* w2_q,
                                              const uint8_t* w2_sf, void* y, const moe_ep_handle* handle_out,
                                              int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream,
                                              moe_stream_t side_stream) {
  return ep_layer(cfg, grp, x, w_gate, bias, expert_owner, mx_weights(w13_q, w13_sf, w2_q, w2_sf), y, handle_out,
                  dev_status, ws, ws_bytes, stream, side_stream);
}

moe_status moe_capacity_rows(const moe_config* cfg, double factor, int32_t* capacity) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (!capacity) return fail(MOE_ERR_INVALID_ARG, "capacity is NULL");
  if (!(factor >= 0.0) || !isfinite(factor)) return fail(MOE_ERR_INVALID_ARG, "factor must be finite and >= 0");
  // the uniform share N*k/E times the factor, rounded up (evaluated left to right in double)
  const double c = ceil(factor * (double)cfg->N * (double)cfg->k / (double)cfg->E);
  if (c > 2147483647.0) return fail(MOE_ERR_UNSUPPORTED, "capacity exceeds int32");
  *capacity = (int32_t)c;
  return MOE_OK;
}

moe_status moe_capacity_drop(const moe_config* cfg, const int32_t* topk_ids, int32_t capacity, int32_t* kept_ids,
                             int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (capacity < 0) return fail(MOE_ERR_INVALID_ARG, "capacity must be >= 0");
  if (cfg->N > 0 && (!topk_ids || !kept_ids)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer");
  if (!ws || ws_bytes < eplb_ws_bytes(*cfg)) return fail(MOE_ERR_WORKSPACE, "capacity workspace too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  return cuda_status(launch_capacity_keep(*cfg, topk_ids, capacity, kept_ids, dev_status, ws, (cudaStream_t)stream),
                     "capacity");
}

}  // extern "C"
