// Internal declarations shared by the translation units of libmoe.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "moe.h"

namespace moe {

constexpr int kMaxE = 256;        // routed experts a router scores
constexpr int kMaxSlots = 512;    // experts (or physical expert slots) the layout and expert GEMMs take
constexpr int kMaxK = 8;          // top-k
constexpr int kMaxP = 32;         // virtual owners
constexpr int kMaxGroups = 32;    // expert groups
constexpr int kMaxTopkGroups = 8; // groups kept per token
constexpr int kMaxShared = 8;     // shared experts
constexpr int kLayoutChunk = 1024;  // assignments per counting chunk
constexpr int kTileRows = 128;      // rows per block in tile_off

// ---- moe_abi.cu : the text moe_last_error returns, for entry points in other files
moe_status record_error(moe_status s, const char* what);
moe_status record_cuda_error(cudaError_t e, const char* where);
// the device word a bounds-checked build records failed checks into (NULL: none registered)
int* check_word();

// ---- layout.cu
size_t layout_ws_bytes(int A, int E, int P, int nchunks);
cudaError_t launch_layout(const moe_config& cfg, const int32_t* owner, const int32_t* ids, const moe_layout& L,
                          int32_t* status, void* ws, cudaStream_t st);

// ---- route.cu : top-k selection and gates from fp32 logits
// gate_bias: NULL, or the router bias to subtract from the selection keys before gating
cudaError_t launch_topk(const moe_config& cfg, const float* logits, const float* gate_bias, int32_t* ids, float* w,
                        cudaStream_t st);

// ---- movement.cu : permute / combine and their two-hop (staged) forms
cudaError_t launch_permute(const moe_config& cfg, const moe_layout& L, const void* x, void* x_perm,
                           cudaStream_t st);
cudaError_t launch_permute_staged(const moe_config& cfg, const moe_layout& L, const void* x, void* send_buf,
                                  void* x_perm, cudaStream_t st);
cudaError_t launch_combine(const moe_config& cfg, const moe_layout& L, const void* out, const float* topk_w,
                           void* y, cudaStream_t st);
cudaError_t launch_combine_staged(const moe_config& cfg, const moe_layout& L, const void* out,
                                  const float* topk_w, void* ret_buf, void* y, cudaStream_t st);

// ---- GEMM family: a "group" is a block of rows multiplied by one weight matrix.
// Groups 0..E-1 are routed experts (rows [expert_off[g], +n_e[g]) of A map 0); groups
// E..E+S-1 are shared experts over N rows (from A map 1 when shared_from_map1, else
// from A map 0 starting at row A_routed + s*N).  The router is one shared group.
enum GemmMode { MODE_ROUTER = 0, MODE_FC1 = 1, MODE_FC2 = 2 };

struct GemmArgs {
  int mode;
  int G;             // groups in this launch: global groups g0 .. g0+G-1
  int g0;            // first global group (routed experts are 0..E-1, shared E..E+S-1)
  int E;             // routed groups
  int N;             // rows of a shared group
  int A_routed;      // rows of all routed groups (= N*k for the FFN, 0 for the router)
  int K;             // reduction length
  int n_out;         // valid output columns (E, I or d)
  int I;             // FC1: row offset of W_up inside W13
  int shared_from_map1;
  const int32_t* n_e;
  const int32_t* expert_off;
  const int32_t* row2tok;
  const float* gate_w;  // FC2: routed row r is scaled by gate_w[row2tok[r]], or gate_w[r] when
                        // row2tok is NULL (NULL gate_w: no scale)
  const float* bias;    // router: added to every logit (NULL: none)
  void* out;
  long long ldo;        // output row stride in elements
  int* status;
  // raw operand pointers (SIMT path; the tensor-core path reads through tensor maps)
  const void* a0;
  const void* a1;
  const void* b;
  long long b_rows;     // rows of one weight matrix (2I, d or E)
  int max_ctas;         // cap on the persistent grid (0 = one CTA per SM)
  // FP8 (e4m3) operands: accumulator x a_scale(row) x b_scale(weight row)
  int fp8;
  int k;                // top-k (FC1: routed row -> token = row2tok / k)
  const float* a_scale; // FC1: per token [N]; FC2: per h row [A + S*N]
  const float* b_scale; // per weight row [groups, b_rows]
  const float* a_scale_rows;  // FC1: when set, routed row r's scale is a_scale_rows[r] (no row map)
  int* check;           // bounds-checked build: where failed checks are recorded (NULL: nowhere)
  // block-scaled (MX) e4m3 operands: E8M0 scale bytes, row-major [rows, K/32]
  const uint8_t* a0_sf;  // rows of A map 0
  const uint8_t* a1_sf;  // rows of A map 1 (FC1: the tokens, for the shared experts)
  const uint8_t* b_sf;   // [groups, b_rows, K/32]
  long long a0_rows, a1_rows;  // rows of the A tensors (the last row is read for rows past them)
  // MX FC1: the epilogue also writes h MX-quantised (after its bf16 rounding): codes
  // [rows, n_out] and E8M0 scale bytes [rows, n_out/32] (NULL: not written); out may then
  // be NULL (h not stored in bf16)
  void* q_out;
  uint8_t* q_sf;
};

#ifdef __CUDACC__
// FP8 FC1: the scale of a routed row's token (row -> assignment -> token); in the
// bounds-checked build an assignment outside [0, A_routed) is recorded and scales by 0.
__device__ __forceinline__ float token_scale(const GemmArgs& p, long long orow) {
  const int a = p.row2tok[orow];
  if (kChecks && (a < 0 || a >= p.A_routed)) {
    if (p.check) atomicCAS(p.check, 0, MOE_ERR_BAD_INDEX);
    return 0.0f;
  }
  return p.a_scale[a / p.k];
}
#endif

// Rows a launch covers, for grid sizing: routed rows if any routed group is in range,
// plus N rows per shared group in range.
inline long long launch_rows(const GemmArgs& g) {
  const int routed = (g.g0 < g.E) ? ((g.g0 + g.G < g.E ? g.g0 + g.G : g.E) - g.g0) : 0;
  return (routed > 0 ? (long long)g.A_routed : 0LL) + (long long)(g.G - routed) * g.N;
}

// tensor-core (tcgen05) path, bf16 operands, fp32 accumulation: one CTA per tile
cudaError_t launch_tc_gemm(const GemmArgs& g, int a0_rows, int a1_rows, cudaStream_t st);
// the same over CTA pairs (cta_group::2): every row of a group in one pass over its weights
cudaError_t launch_tc_gemm_pair(const GemmArgs& g, int a0_rows, int a1_rows, cudaStream_t st);
// block-scaled (MX) e4m3 operands with E8M0 scales per 32 K values (FC1 / FC2 only)
cudaError_t launch_tc_gemm_mx(const GemmArgs& g, cudaStream_t st);
// CUDA-core path, fp32 operands (the fp32 configurations)
cudaError_t launch_simt_gemm(const GemmArgs& g, cudaStream_t st);

// rows of row_bytes bytes (the FP8 dispatch payload moves d bytes per row)
cudaError_t launch_permute_bytes(const moe_config& c, const moe_layout& L, const void* x, void* x_perm,
                                 int row_bytes, cudaStream_t st);
// FP8 (fp8.cu): per-row e4m3 quantisation of bf16 rows, scale = amax / 448
cudaError_t launch_quantize_rows(const void* src, long long rows, int cols, void* dst, float* scale,
                                 cudaStream_t st);
// MX (fp8.cu): e4m3 codes and one E8M0 scale byte per 32 values of a bf16 row; cols % 32 == 0
cudaError_t launch_quantize_mx(const void* src, long long rows, int cols, void* dst, uint8_t* sf, cudaStream_t st);

// redundant expert slots (eplb.cu)
size_t eplb_ws_bytes(const moe_config& c);
cudaError_t launch_eplb_assign(const moe_config& c, const int32_t* ids, const int32_t* replica_off,
                               const int32_t* replica_slots, int n_slots, int32_t* phys, int32_t* status, void* ws,
                               cudaStream_t st);
cudaError_t launch_capacity_keep(const moe_config& c, const int32_t* ids, int capacity, int32_t* kept,
                                 int32_t* status, void* ws, cudaStream_t st);
moe_status eplb_plan(int E, int R, int P, const int64_t* load, int32_t* copies, int32_t* replica_off,
                     int32_t* replica_slots, int32_t* slot_expert, int32_t* slot_owner, int64_t* owner_load);

// expert parallelism over peer memory (ep.cu).  A window is the buffer every rank
// allocates with the same size; its parts sit at the same offsets on every rank.
struct EpOffsets {
  size_t cnt_flag, disp_flag, done_flag;  // [kMaxP] u64 epochs, indexed by the signalling rank
  size_t step;                            // u64: this rank's steps so far (= the running step's epoch)
  size_t disp_ctr;                        // u32: this rank's dispatch CTAs finished in the running launch
  size_t err_step;                        // u64: the last step in which a wait of this rank failed
  size_t cnt_tab;                         // [P, E] int32: row i = source i's expert counts
  size_t gate;                            // [capacity] fp32: gate of each received row
  size_t scale;                           // [capacity] fp32: FP8 dispatch: token scale of each received row
  size_t x_recv;                          // [capacity, d]: received rows, expert-major
  size_t out_recv;                        // [capacity + S*N, d]: FC2 rows (routed, then shared)
  size_t total;
};
struct EpPeers {
  char* base[kMaxP];  // every rank's window as mapped in this process
};
EpOffsets ep_offsets(const moe_config& c, int capacity);
cudaError_t launch_ep_push_counts(const EpPeers& peers, const EpOffsets& off, const int32_t* n_loc, int E, int P,
                                  int me, cudaStream_t st);
cudaError_t launch_ep_layout(const moe_config& c, const EpPeers& peers, const EpOffsets& off, int me, int capacity,
                             int local_experts, const int32_t* owner, const int32_t* ids, const moe_layout& loc,
                             int32_t* dest, int32_t* own_n_e, int32_t* own_off, int* status, cudaStream_t st);
// rows of row_bytes bytes (d * elem for bf16 / fp32, d for e4m3 codes); x_scale (FP8): each
// token's scale, stored beside each of its received rows (NULL: none); x2 (MX): each token's
// scale row of row_bytes2 bytes (at most 512), stored in the receive region after the
// capacity rows of codes (NULL: none)
cudaError_t launch_ep_dispatch(const moe_config& c, const EpPeers& peers, const EpOffsets& off, int me,
                               int capacity, const void* x, const int32_t* dest, const float* topk_w,
                               const float* x_scale, int row_bytes, cudaStream_t st, const void* x2 = nullptr,
                               int row_bytes2 = 0);
cudaError_t launch_ep_wait(const char* own, const EpOffsets& off, size_t flag_off, int n, int* status,
                           cudaStream_t st);
cudaError_t launch_ep_signal(const EpPeers& peers, const EpOffsets& off, size_t flag_off, int P, int me,
                             cudaStream_t st);
cudaError_t launch_ep_combine(const moe_config& c, const EpPeers& peers, const EpOffsets& off, int me, int capacity,
                              const int32_t* dest, void* y, int* status, cudaStream_t st);

int sm_count();
// TMA maps for bf16 K-major operands; box_k (64, 32 or 16) selects the 128/64/32-byte swizzle
bool make_map_a(CUtensorMap* m, const void* base, long long rows, long long K, int box_k = 64, bool u8 = false,
                int box_rows = 128);
bool make_map_b(CUtensorMap* m, const void* base, long long G, long long R, long long K, int box_rows,
                int box_k = 64, bool u8 = false);

}  // namespace moe
