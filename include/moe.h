/*
 * moe.h — C ABI of libmoe: one Mixture-of-Experts layer's token movement and expert
 * compute on one NVIDIA B200 (sm_100a).
 *
 * The layer (router -> top-k -> dispatch layout -> permute -> grouped SwiGLU experts ->
 * combine) follows these web pages, cited by title and section:
 *   [EP-DeepEP] ep_deepep explainer (papers-3lj.pages.dev): §2 y_t = sum_{e in I_t}
 *               g_{t,e} Expert_e(x_t) and n_e; §3 dispatch/combine; §5 interface: input
 *               = token layout + routing info, output = an owner-local computable
 *               layout, completion and buffer lifetime explicit; §6 the three maps.
 *   [DSMoE]     "深入浅出 DeepSeek MoE：EP 与 FSDP 经典二次开发实战指南": naive 5-step
 *               forward; EP as a distributed transpose; DeepEP dispatch -> handle ->
 *               combine(handle) split (Automodel excerpt).
 *   [DeepEP]    DeepEP notes (lizn-zn.github.io) §2-3: all-to-all transpose, counts first.
 *   [WideEP]    "Wide EP：当 MoE Expert Parallel 横跨几十张 GPU": count matrix C_ij,
 *               receive load R_r, group-limited routing, E_local placement.
 *   [MoE-IV]    "MoE我们喜欢你（四）：DeepEP 与 GroupedGEMM 如何拆解通信和计算瓶颈" §4:
 *               permute -> a2a -> grouped_gemm -> a2a -> unpermute_and_weighted_sum.
 *
 * Conventions for every call
 *   - All array arguments are DEVICE pointers to row-major, contiguous memory, 16-byte
 *     aligned, allocated and owned by the caller.  The library allocates nothing, keeps
 *     no state between calls, and never synchronises with the host.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Host-detectable errors (bad sizes, NULL pointers, small workspace) return a
 *     non-zero moe_status immediately and launch nothing.
 *   - Device-detected errors (an expert id outside [0, E) other than -1, which marks a
 *     dropped assignment (moe_capacity_drop), or a wait that timed out) are
 *     written to *dev_status (an int32 the caller zeroes and reads after synchronising);
 *     the first error wins.  dev_status may be NULL, in which case they go unreported.
 *   - Sizes: A = N * k assignments, a = t * k + slot indexes them.  E % P == 0 unless an
 *     explicit expert_owner table is given.  k <= 8, E >= k, P <= 32,
 *     n_groups <= 32 with E % n_groups == 0, topk_groups <= 8.  The router (moe_route
 *     and the fused forwards) takes E <= 256; the layout, movement and expert calls take
 *     E <= 512 (e.g. E + R physical expert slots, see moe_eplb_*).
 *     bf16: d % 8 == 0, I % 8 == 0.   f32: d % 4 == 0, I % 4 == 0.
 *   - dtype applies to activations, weights and expert outputs; every reduction
 *     accumulates in fp32.  Router logits and gate weights are fp32.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* NULL pointer, negative or inconsistent size */
  MOE_ERR_UNSUPPORTED = 2, /* valid request outside the sizes this library supports */
  MOE_ERR_WORKSPACE = 3,   /* workspace smaller than the matching *_workspace_bytes() */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed (launch, tensor map) */
  MOE_ERR_BAD_INDEX = 5,   /* device: an expert id outside [0, E) (other than -1) was seen */
  MOE_ERR_TIMEOUT = 6      /* device: a bounded wait gave up */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score;
/* MOE_BIAS_LOGITS: z = x W_g^T + b feeds both the selection and the gates.
 * MOE_BIAS_SELECTION: a correction bias ([MoE-IV] §4.2 "correction_bias"): the selection
 * uses z + b, the gate weights use the unbiased z of the chosen experts. */
typedef enum { MOE_BIAS_LOGITS = 0, MOE_BIAS_SELECTION = 1 } moe_bias_mode;

/* Shape and routing rule of one layer. */
typedef struct {
  int32_t N;           /* tokens */
  int32_t d;           /* hidden size */
  int32_t E;           /* routed experts */
  int32_t k;           /* experts per token (top-k) */
  int32_t I;           /* expert intermediate size (SwiGLU) */
  int32_t n_shared;    /* S: shared experts, always active, added with weight 1 */
  int32_t P;           /* virtual expert-owner ranks (EP size) */
  int32_t n_groups;    /* expert groups for group-limited routing; 1 = plain top-k */
  int32_t topk_groups; /* groups kept per token (1 when n_groups == 1) */
  int32_t score;       /* moe_score: softmax over E, or per-expert sigmoid */
  int32_t renormalize; /* 1: gates renormalised to sum 1 over the chosen k */
  int32_t dtype;       /* moe_dtype */
  int32_t bias_mode;   /* moe_bias_mode: how the router bias (when given) is used */
} moe_config;

/*
 * The dispatch layout ("handle"): caller-owned device arrays, all int32.
 *   n_e[E]          tokens per expert                         ([EP-DeepEP] §2)
 *   expert_off[E+1] first row of expert e in the expert-contiguous buffer; experts are
 *                   ordered by (owner, expert id); expert_off[E] = A
 *   C[P*P]          C[i*P+j] = assignments from source rank i to owner j ([WideEP])
 *   send_off[P*P]   start of block (i, j) in the send buffer (ordered by source, then owner)
 *   recv_off[P+1]   start of owner j's rows; recv_off[j+1]-recv_off[j] = R_j = sum_i C_ij
 *   tok2send[A]     assignment a -> send slot                 ([EP-DeepEP] §6, map 1)
 *   send2row[A]     send slot -> expert-contiguous row         ([EP-DeepEP] §6, map 2)
 *   ret2tok[A]      return row (= send slot of the combine all-to-all) -> assignment a
 *                                                             ([EP-DeepEP] §6, map 3)
 *   tok2row[A]      a -> row (= send2row[tok2send[a]])
 *   row2tok[A]      row -> a (inverse of tok2row)
 *   tile_off[E+S+1] prefix of ceil(rows/128) over routed experts (id order) then the S
 *                   shared groups of N rows
 * Source rank of token t is t / ceil(N/P).  Inside an expert, rows ascend in a.
 */
typedef struct {
  int32_t* n_e;
  int32_t* expert_off;
  int32_t* C;
  int32_t* send_off;
  int32_t* recv_off;
  int32_t* tok2send;
  int32_t* send2row;
  int32_t* ret2tok;
  int32_t* tok2row;
  int32_t* row2tok;
  int32_t* tile_off;
} moe_layout;

/* Library version (major*10000 + minor*100 + patch) and a text for a status code. */
int32_t moe_version(void);
const char* moe_status_string(int32_t status);

/* Host-side description of the last error returned on this thread ("" if none). */
const char* moe_last_error(void);

/*
 * Bounds-checked build (no counterpart in the pages; it stands in for a race / bounds
 * sanitizer).  The same sources compiled with
 * -DMOE_CHECKS give libmoe_checked.so, whose kernels check every index they read from a
 * caller-visible map or table before using it: token -> row maps (tok2row, send2row,
 * tok2send) in the permute and combine, row -> assignment (row2tok) in the FC2 gate and
 * the FP8 token scales, each group's rows (n_e, expert_off) in the grouped GEMMs, and the
 * expert-parallel destinations (dest).  A value outside its range is skipped (no read or
 * write through it) and MOE_ERR_BAD_INDEX is recorded in the registered device word with
 * an atomic compare-and-swap (the first error is kept).  Nothing traps.  The ids given to
 * the layout are checked in every build (moe_dispatch_layout's dev_status).
 *   moe_checks_enabled: 1 in the checked build, 0 otherwise.
 *   moe_checks_register: the caller's device int32 the checked kernels record into, for
 *     every later call on any thread (NULL: record nowhere); the normal build accepts
 *     and ignores it.  Launches nothing.
 */
int32_t moe_checks_enabled(void);
moe_status moe_checks_register(int32_t* dev_word);

/* Validate a configuration on the host (the same checks every call makes). */
moe_status moe_check_config(const moe_config* cfg);

/* Bytes of scratch moe_dispatch_layout needs (ws argument). */
size_t moe_layout_workspace_bytes(const moe_config* cfg);

/* Bytes of scratch moe_layer_forward needs: logits, ids, gates, layout, layout scratch,
 * permuted rows [A, d], SwiGLU activations [A+S*N, I] and expert outputs [A+S*N, d]. */
size_t moe_workspace_bytes(const moe_config* cfg);

/*
 * Router and top-k selection ([DSMoE] naive forward steps 1-2; [EP-DeepEP] §2;
 * [WideEP] "Group-limited routing"; renormalisation as named in [MoE-IV] §4.2).
 *   x        [N, d]  dtype      w_gate [E, d] dtype (one row per expert)
 *   bias     [E] fp32 or NULL   added to the logits (see moe_bias_mode)
 *   logits   [N, E] fp32, required: written with z = x W_g^T (+ b); the selection
 *            reads back exactly these fp32 values
 *   topk_ids [N, k] int32: slot 0 = largest logit; ties go to the lower expert index.
 *            With n_groups > 1 a token first keeps the topk_groups groups with the
 *            largest group max (ties to the lower group), then takes its top-k there.
 *   topk_w   [N, k] fp32 gate weights:
 *            softmax: exp(z_e - m) / sum_{all E} exp(z - m), or over the chosen k when
 *            renormalize; sigmoid: 1/(1+exp(-z_e)), divided by their sum when renormalize.
 *            With MOE_BIAS_SELECTION, z here is the unbiased x W_g^T (logits holds z + b).
 */
moe_status moe_route(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                     float* logits, int32_t* topk_ids, float* topk_w, moe_stream_t stream);

/*
 * Dispatch layout from the top-k ids ([EP-DeepEP] §3 and §6; [WideEP] C_ij, R_r;
 * [DeepEP] §3 "counts first"; [DSMoE] VeOmni preprocess).  Pure integer work, bit-exact
 * and deterministic; nothing is copied to the host.
 *   expert_owner [E] int32 or NULL (NULL = owner e / (E/P)); each owner's experts keep
 *                id order and its rows are contiguous
 *   topk_ids     [N, k] int32; -1 marks a dropped assignment (no row, see
 *                moe_capacity_drop); other ids outside [0, E) set *dev_status = MOE_ERR_BAD_INDEX
 *                and are treated as expert 0 (no out-of-bounds write happens)
 *   out          the layout arrays (all must be non-NULL)
 *   ws, ws_bytes scratch of at least moe_layout_workspace_bytes(cfg)
 */
moe_status moe_dispatch_layout(const moe_config* cfg, const int32_t* expert_owner, const int32_t* topk_ids,
                               const moe_layout* out, int32_t* dev_status, void* ws, size_t ws_bytes,
                               moe_stream_t stream);

/*
 * moe_dispatch_layout for callers that cannot allocate GPU memory (no counterpart in
 * the pages: it exists for deployment, not for the method).  A plugin inside a runtime
 * that owns all device buffers, a serving loop that must not call cudaMalloc (which
 * synchronises the device), or a service with a memory budget fixed at start-up may
 * have no workspace to pass.  This call computes exactly what moe_dispatch_layout
 * computes, with the same kernels, but takes no ws argument: the scratch is a 2 MiB
 * array compiled into the library, which every GPU that loads the library holds until
 * the process exits.  It allocates nothing and calls no allocating routine.
 *   Limit: moe_layout_workspace_bytes(cfg) <= 2 MiB (about N*k <= 131072 assignments
 *          with E <= 256, P <= 32); larger configurations return MOE_ERR_UNSUPPORTED.
 *   Set-up: the first call on each device looks up the array's device address
 *          (cudaGetSymbolAddress, with that device current) and caches it; make that
 *          first call before any stream capture.  The cache is tied to the device's
 *          context: after a device reset (cudaDeviceReset, or anything else that
 *          destroys the primary context) the array is reloaded at another address and
 *          the next call looks it up again, so that call, too, should come before any
 *          capture.  The scratch contents do not survive a reset.
 *   Sharing: all calls on a device use the same array, so calls that overlap on the GPU
 *          (different streams, or different host threads) race and corrupt each other's
 *          results; serialise them.  Contents left by an earlier call are harmless:
 *          every scratch word is written before it is read within a call.
 * Arguments, layout and device-side errors are those of moe_dispatch_layout.
 */
moe_status moe_dispatch_layout_noalloc(const moe_config* cfg, const int32_t* expert_owner, const int32_t* topk_ids,
                                       const moe_layout* out, int32_t* dev_status, moe_stream_t stream);

/*
 * Permute ([MoE-IV] §4 permute_by_expert; [DSMoE] token_pre_all2all): the dispatch
 * all-to-all and the expert sort composed into one gather, x_perm[tok2row[a]] = x[a/k].
 * Each token row is read once and written k times.
 *   x [N, d] dtype  ->  x_perm [A, d] dtype (expert-contiguous, owner-major)
 */
moe_status moe_permute(const moe_config* cfg, const moe_layout* layout, const void* x, void* x_perm,
                       moe_stream_t stream);

/*
 * The same movement in two explicit hops, for inspection of the virtual all-to-all
 * ([DeepEP] §2 transpose figure; [EP-DeepEP] §3): send_buf[tok2send[a]] = x[a/k]
 * (each source buckets by owner), then x_perm[send2row[s]] = send_buf[s] (transpose to
 * the owners and expert-local sort).  Bit-identical to moe_permute.
 *   send_buf [A, d] dtype scratch owned by the caller.
 */
moe_status moe_permute_staged(const moe_config* cfg, const moe_layout* layout, const void* x, void* send_buf,
                              void* x_perm, moe_stream_t stream);

/*
 * Grouped SwiGLU experts ([MoE-IV] §4.1 "FC1, activation, FC2"; [EP-DeepEP] §2
 * Expert_e):  for each expert e with n_e > 0 and its rows X_e of x_perm,
 *   H_e = SiLU(X_e W_gate_e^T) * (X_e W_up_e^T),   O_e = H_e W_down_e^T  (x gate if topk_w)
 * and for each shared expert s the same over all N rows of x.
 *   x_perm [A, d], x [N, d] (read only when n_shared > 0)
 *   w13 [E+S, 2I, d]: rows [0, I) = W_gate, rows [I, 2I) = W_up; shared experts last
 *   w2  [E+S, d, I]
 *   topk_w [N, k] fp32 or NULL: when given, routed output row r is scaled by
 *          topk_w[row2tok[r]] before rounding (the combine's gate, applied here)
 *   h_ws [A + S*N, I] dtype scratch (the SwiGLU activations)
 *   out  [A + S*N, d] dtype: routed rows [0, A) in expert-contiguous order, then shared
 *        expert s's N rows at A + s*N, in token order
 * Each routed row's numbers depend only on that row and its expert: rows past an
 * expert's end are computed in no other expert's tile result.
 */
moe_status moe_grouped_ffn(const moe_config* cfg, const moe_layout* layout, const void* x_perm, const void* x,
                           const void* w13, const void* w2, const float* topk_w, void* h_ws, void* out,
                           moe_stream_t stream);

/* Which expert groups an FFN call covers. */
typedef enum { MOE_GROUPS_ALL = 0, MOE_GROUPS_ROUTED = 1, MOE_GROUPS_SHARED = 2 } moe_group_set;

/*
 * The two halves of moe_grouped_ffn, for callers that schedule them separately:
 *   moe_expert_fc1: h_ws = SiLU(X W_gate^T) * (X W_up^T) for every group in `groups`
 *                   (routed rows of x_perm; each shared expert over the N rows of x)
 *   moe_expert_fc2: out = (h_ws W_down^T), routed rows scaled by topk_w[row2tok[r]] when
 *                   topk_w is non-NULL
 * `groups` is a moe_group_set.  Shapes, layouts and errors as for moe_grouped_ffn; with
 * MOE_GROUPS_SHARED the layout may be NULL and, as in moe_shared_ffn, 16 SMs are left free.
 */
moe_status moe_expert_fc1(const moe_config* cfg, const moe_layout* layout, const void* x_perm, const void* x,
                          const void* w13, void* h_ws, int32_t groups, moe_stream_t stream);
moe_status moe_expert_fc2(const moe_config* cfg, const moe_layout* layout, const void* h_ws, const void* w2,
                          const float* topk_w, void* out, int32_t groups, moe_stream_t stream);

/*
 * moe_grouped_ffn split by expert kind, so that the shared experts (which need only x)
 * can run concurrently with the routing and dispatch of the routed ones:
 *   moe_routed_ffn: FC1 + SwiGLU and FC2 (x topk_w when non-NULL) for the routed experts,
 *                   rows [0, A) of h_ws and out
 *   moe_shared_ffn: the same for the S shared experts over all N rows of x, rows
 *                   [A, A + S*N) of h_ws and out (no layout is needed); it leaves 16 SMs
 *                   free for the routing kernels meant to run beside it
 * Together they write exactly what moe_grouped_ffn writes.
 */
moe_status moe_routed_ffn(const moe_config* cfg, const moe_layout* layout, const void* x_perm, const void* w13,
                          const void* w2, const float* topk_w, void* h_ws, void* out, moe_stream_t stream);
moe_status moe_shared_ffn(const moe_config* cfg, const void* x, const void* w13, const void* w2, void* h_ws,
                          void* out, moe_stream_t stream);

/*
 * Combine ([EP-DeepEP] §2-3; [DSMoE] combine = gate-weighted sum at the source;
 * [MoE-IV] §4 unpermute_and_weighted_sum): the combine all-to-all composed with the
 * unpermute and the weighted sum,
 *   y_t = sum_{slot<k} g_{t,slot} * out[tok2row[t*k+slot]] + sum_{s<S} out[A + s*N + t]
 * accumulated in fp32 in that fixed order and rounded once to dtype.
 *   topk_w [N, k] fp32, or NULL when moe_grouped_ffn already applied the gates
 *   y [N, d] dtype, token order
 */
moe_status moe_combine(const moe_config* cfg, const moe_layout* layout, const void* out, const float* topk_w,
                       void* y, moe_stream_t stream);

/*
 * The combine in two explicit hops: ret_buf[s] = out[send2row[s]] (reverse transpose,
 * the owners send rows back in send-slot order), then
 * y_t = sum_slot g * ret_buf[tok2send[t*k+slot]] + shared rows.  Bit-identical to
 * moe_combine.   ret_buf [A, d] dtype scratch owned by the caller.
 */
moe_status moe_combine_staged(const moe_config* cfg, const moe_layout* layout, const void* out,
                              const float* topk_w, void* ret_buf, void* y, moe_stream_t stream);

/*
 * The whole layer on one stream: moe_route -> moe_dispatch_layout -> moe_permute ->
 * moe_grouped_ffn (gates applied in the down-projection epilogue) -> moe_combine.
 * No host synchronisation, no allocation; capturable in a CUDA graph.
 *   layout_out  NULL, or caller arrays that receive the layout (otherwise it lives in ws)
 *   ws          at least moe_workspace_bytes(cfg) bytes, 256-byte aligned
 */
moe_status moe_layer_forward(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                             const int32_t* expert_owner, const void* w13, const void* w2, void* y,
                             const moe_layout* layout_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * Self-test of the failure path (no counterpart in the pages).  Launches one thread that
 * waits, with the library's bounded-wait routine and a limit of `limit_ns` nanoseconds
 * (1 .. 1e10), on an mbarrier that nothing will ever arrive on.  The wait gives up, the
 * kernel writes MOE_ERR_TIMEOUT to *dev_status and returns; the context stays usable.
 * Every wait in the library's kernels behaves this way (limit 2 s).
 */
moe_status moe_selftest_bounded_wait(int32_t* dev_status, uint64_t limit_ns, moe_stream_t stream);

/*
 * moe_layer_forward with the shared experts overlapped (the pages' overlap lever:
 * [EP-DeepEP] §7 pipelining; [WideEP] dual-batch overlap; [MoE-IV] §4.2 overlap): the
 * router runs on `stream`; then the shared experts run on `side_stream` while the
 * layout, permute and routed experts run on `stream`; `stream` waits for `side_stream`
 * before the combine.  Same result as moe_layer_forward, bit for bit.  Two events are
 * created and destroyed per call (no device memory is allocated).  With n_shared == 0 or
 * side_stream == stream this is moe_layer_forward.  When the call returns, `stream`
 * orders after all the work; `side_stream` may be reused immediately.
 */
moe_status moe_layer_forward_overlapped(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                                        const int32_t* expert_owner, const void* w13, const void* w2, void* y,
                                        const moe_layout* layout_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                                        moe_stream_t stream, moe_stream_t side_stream);

/*
 * The layer as a pipeline over token chunks ([EP-DeepEP] §7, pipelined overlap: the layer
 * time approaches T_warm + sum over chunks of max(T_disp, T_exp, T_comb) + T_drain).  The
 * N tokens are split into n_chunks contiguous chunks of ceil(N / n_chunks) tokens (the last
 * may hold fewer, and chunks past the end hold none).  One router launch covers all tokens;
 * then each chunk is a layer of its own: its layout (its own counts, offsets and maps over
 * its tokens) and permute on `stream`, its expert FFN (routed, then shared experts) on
 * `side_stream`, and its combine on `stream` again, so that chunk c's layout and permute
 * and chunk c-2's combine run beside chunk c-1's experts.  Each token's output rows are
 * computed exactly as in moe_layer_forward (the same kernels, the same k order), so y is
 * the same.  On one GPU the experts' weights are streamed once per chunk; the form pays
 * off where the movement is long against the experts (the all-to-all of an EP layer).
 *   n_chunks        1 .. 16
 *   ws, ws_bytes    at least moe_workspace_bytes_chunked(cfg, n_chunks), 256-byte aligned
 *   stream, side_stream  two different streams; when the call returns, `stream` orders
 *                   after all the work and `side_stream` may be reused immediately
 * Errors as moe_layer_forward; n_chunks outside [1, 16] -> MOE_ERR_INVALID_ARG.
 */
size_t moe_workspace_bytes_chunked(const moe_config* cfg, int32_t n_chunks);
moe_status moe_layer_forward_chunked(const moe_config* cfg, int32_t n_chunks, const void* x, const void* w_gate,
                                     const float* bias, const int32_t* expert_owner, const void* w13, const void* w2,
                                     void* y, int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream,
                                     moe_stream_t side_stream);

/*
 * Redundant expert slots, EPLB ([WideEP] "为什么要把 EP 做宽": E logical experts plus R
 * copies make E + R physical experts, (E + R) / P per owner; "DeepSeek-V3/R1 的两个具体
 * 布局": 256 + 32 = 288 slots; "Expert 副本在 Wide EP 中还有整除作用": hot experts are
 * copied and a logical expert's assignments are spread over its copies; "三种负载必须同时
 * 平衡": the balancer minimises the largest expert / receive load).  The router's choice
 * is kept; only which copy serves an assignment changes.  Use:
 *   1. moe_eplb_plan on the host, from per-expert loads (e.g. n_e of earlier batches);
 *   2. moe_eplb_place_weights once per plan: W13 / W2 of the E + R slots (+ shared);
 *   3. per batch: moe_route (E logical experts) -> moe_eplb_assign -> the layout, permute,
 *      expert and combine calls with a config whose E is E + R (slot s is owned by
 *      s / ((E + R) / P), so expert_owner may be NULL), the physical weights and the same
 *      topk_w.  The output equals the layer without copies.
 */

/*
 * Plan (host only; all pointers are HOST memory; no GPU work).  Steps, since the pages
 * give the goal but no algorithm:
 *   copies: every expert keeps one copy; each of the R extra copies in turn goes to the
 *           expert with the largest load per copy, load_e / copies_e (ties: lower id),
 *           which minimises max_e load_e / copies_e;
 *   placement: copy c of expert e carries load_e / copies_e rounded down, plus one when
 *           c < load_e mod copies_e (the rows moe_eplb_assign gives it); copies are
 *           placed in descending load order (ties: lower expert, lower copy) on the
 *           owner with free room that holds no copy of the same expert if there is one,
 *           then the least loaded owner, then the lower owner;
 *   slots:  owner j holds slots [j (E+R)/P, (j+1) (E+R)/P) in (expert, copy) order.
 *   load          [E] int64, 0 .. 2^40
 *   copies        [E] out: copies per expert (sum E + R)
 *   replica_off   [E+1] out: copies of expert e are replica_slots[replica_off[e] ..)
 *   replica_slots [E+R] out: slot of copy c of expert e at replica_off[e] + c
 *   slot_expert   [E+R] out: logical expert of each slot
 *   slot_owner    [E+R] out: owner of each slot
 *   owner_load    [P] out: planned rows per owner
 * Errors: (E + R) % P != 0 or a NULL pointer -> MOE_ERR_INVALID_ARG; E + R > 512 ->
 * MOE_ERR_UNSUPPORTED.
 */
moe_status moe_eplb_plan(int32_t E, int32_t R, int32_t P, const int64_t* load, int32_t* copies,
                         int32_t* replica_off, int32_t* replica_slots, int32_t* slot_expert, int32_t* slot_owner,
                         int64_t* owner_load);

/*
 * Capacity factor with dropping ([EP-DeepEP] §4: a capacity factor caps the assignments an
 * expert receives per round and the excess may be dropped): the q-th assignment of expert
 * e in ascending a = t*k + slot is kept when q < capacity, else dropped.  kept_ids [N, k]
 * = topk_ids with the dropped ones set to -1 (a -1 in topk_ids stays -1).  The usual
 * capacity is ceil(factor * N * k / E).  A dropped assignment takes no row and no send
 * slot: moe_dispatch_layout gives it tok2row = tok2send = -1, counts only the kept ones
 * (expert_off[E] = recv_off[P] = the rows in use, A_kept), and marks the unused tails
 * [A_kept, A) of row2tok, send2row and ret2tok with -1; the permute skips it and the
 * combine adds nothing for it (the other gates are not renormalised).  Routed rows of the
 * FFN buffers are [0, A_kept); shared experts' rows still start at A = N*k.
 *   ws, ws_bytes: at least moe_eplb_workspace_bytes(cfg), 256-byte aligned.
 * Device errors: ids outside [0, E) other than -1 -> MOE_ERR_BAD_INDEX (counted as 0).
 */
moe_status moe_capacity_drop(const moe_config* cfg, const int32_t* topk_ids, int32_t capacity, int32_t* kept_ids,
                             int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The capacity of a capacity factor ([EP-DeepEP] §4: an expert's share of one round's
 * assignments, N*k/E, times the factor): *capacity = ceil(factor * N * k / E), evaluated
 * in double precision left to right (host only, launches nothing).
 * Errors: factor not finite or < 0, or capacity NULL -> MOE_ERR_INVALID_ARG; a result
 * above INT32_MAX -> MOE_ERR_UNSUPPORTED; an invalid cfg as moe_check_config.
 */
moe_status moe_capacity_rows(const moe_config* cfg, double factor, int32_t* capacity);

/* Bytes of scratch moe_eplb_assign and moe_capacity_drop need (a one-owner dispatch
 * layout of the logical ids). */
size_t moe_eplb_workspace_bytes(const moe_config* cfg);

/*
 * Replica assignment (device): the q-th assignment of logical expert e, in ascending
 * a = t*k + slot, goes to copy q mod copies_e: phys_ids[a] = replica_slots[replica_off[e]
 * + q mod (replica_off[e+1] - replica_off[e])].  Copies of e thus get n_e / copies_e rows
 * to within one.  q comes from a dispatch layout of the logical ids with one owner,
 * computed in the workspace.
 *   cfg            the LOGICAL configuration (E experts)
 *   topk_ids       [N, k] int32 logical ids
 *   replica_off    [E+1], replica_slots [n_slots] int32 device copies of the plan
 *   n_slots        E + R (E <= n_slots <= 512)
 *   phys_ids       [N, k] int32 out: slot ids in [0, n_slots)
 *   ws, ws_bytes   scratch of at least moe_eplb_workspace_bytes(cfg), 256-byte aligned
 * Device errors (MOE_ERR_BAD_INDEX in *dev_status): an id outside [0, E) (counted as
 * expert 0), an expert without copies or a slot outside [0, n_slots) (slot 0 written).
 */
moe_status moe_eplb_assign(const moe_config* cfg, const int32_t* topk_ids, const int32_t* replica_off,
                           const int32_t* replica_slots, int32_t n_slots, int32_t* phys_ids, int32_t* dev_status,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Weights of the physical slots: w_physical[s] = w_logical[slot_expert[s]] for the
 * n_slots slots, then the n_shared shared experts w_logical[E ..] after them.  One
 * device-to-device copy per slot (plus one for the shared experts) on `stream`; a
 * placement step, run once per plan.
 *   slot_expert  [n_slots] HOST int32 in [0, E)
 *   expert_bytes bytes of one expert's matrix (2*I*d*b for W13, d*I*b for W2)
 *   w_logical    [E + n_shared] matrices, w_physical [n_slots + n_shared] matrices (device)
 */
moe_status moe_eplb_place_weights(const int32_t* slot_expert, int32_t n_slots, int32_t E, int32_t n_shared,
                                  size_t expert_bytes, const void* w_logical, void* w_physical, moe_stream_t stream);

/*
 * FP8 (e4m3) expert path ([MoE-IV] FP8 dispatch payloads and FP8 grouped GEMMs;
 * [WideEP] FP8 weights and dispatch; [EP-DeepEP] §7 low-precision dispatch with the
 * combine in higher precision).  The pages fix neither format nor scaling; this library
 * uses e4m3 without infinities (largest finite 448) and one fp32 scale per row of every
 * operand: s = amax(|row|) / 448 (fp32 division; 1 for an all-zero row), code = round to
 * nearest even of x / s (fp32 division), saturating at +-448.  A GEMM on e4m3 rows
 * computes (sum_k qa qb) * s_a(row) * s_b(weight row) with fp32 accumulation.  The
 * configuration stays bf16 (dtype = MOE_BF16): x, y, h, expert outputs and the combine are
 * bf16 / fp32 as in the bf16 path; d % 16 == 0 and I % 16 == 0.
 */

/* Per-row quantisation: src [rows, cols] bf16 -> dst [rows, cols] e4m3 codes (one byte
 * each), scale [rows] fp32.  cols % 8 == 0.  Used for weights (once), x and h (per step). */
moe_status moe_quantize_fp8(const void* src, int64_t rows, int32_t cols, void* dst, float* scale,
                            moe_stream_t stream);

/* FP8 dispatch payload: x_q_perm[tok2row[a]] = x_q[a / k], rows of d bytes (the permute
 * of moe_permute on e4m3 rows; the token scales stay in token order). */
moe_status moe_permute_fp8(const moe_config* cfg, const moe_layout* layout, const void* x_q, void* x_q_perm,
                           moe_stream_t stream);

/*
 * FP8 grouped SwiGLU FFN, routed and shared experts:
 *   h   = SiLU(Xq Wq_gate^T * s) * (Xq Wq_up^T * s)     (bf16 [A + S*N, I])
 *   h_q, h_scale = moe_quantize_fp8(h)                  (e4m3 [A + S*N, I], fp32 [A + S*N])
 *   out = (h_q W2q^T) * h_scale(row) * w2_scale(col) * gate(row)  (bf16 [A + S*N, d])
 *   x_q_perm [A, d] e4m3 (moe_permute_fp8), x_q [N, d] e4m3 (shared experts' rows),
 *   x_scale [N] per token; w13_q [E+S, 2I, d] e4m3, w13_scale [E+S, 2I]; w2_q [E+S, d, I]
 *   e4m3, w2_scale [E+S, d]; topk_w as in moe_grouped_ffn (NULL: no gate scale).
 */
moe_status moe_grouped_ffn_fp8(const moe_config* cfg, const moe_layout* layout, const void* x_q_perm,
                               const void* x_q, const float* x_scale, const void* w13_q, const float* w13_scale,
                               const void* w2_q, const float* w2_scale, const float* topk_w, void* h, void* h_q,
                               float* h_scale, void* out, moe_stream_t stream);

/* Bytes of scratch moe_layer_forward_fp8 needs. */
size_t moe_workspace_bytes_fp8(const moe_config* cfg);

/* The whole layer with the FP8 expert path, one stream: moe_route -> moe_dispatch_layout
 * -> moe_quantize_fp8(x) -> moe_permute_fp8 -> moe_grouped_ffn_fp8 -> moe_combine.  The
 * weights come quantised (moe_quantize_fp8 of W13 and W2 rows, once). */
moe_status moe_layer_forward_fp8(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                                 const int32_t* expert_owner, const void* w13_q, const float* w13_scale,
                                 const void* w2_q, const float* w2_scale, void* y, const moe_layout* layout_out,
                                 int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward_fp8 with the shared experts overlapped: after the router and the
 * quantisation of x on `stream`, the shared experts' FP8 FFN runs on `side_stream` while
 * the layout, the FP8 permute and the routed FP8 FFN run on `stream`; `stream` waits for
 * `side_stream` before the combine.  Same result as moe_layer_forward_fp8, bit for bit;
 * two events are created and destroyed per call.  With n_shared == 0 or side_stream ==
 * stream this is moe_layer_forward_fp8. */
moe_status moe_layer_forward_fp8_overlapped(const moe_config* cfg, const void* x, const void* w_gate,
                                            const float* bias, const int32_t* expert_owner, const void* w13_q,
                                            const float* w13_scale, const void* w2_q, const float* w2_scale, void* y,
                                            const moe_layout* layout_out, int32_t* dev_status, void* ws,
                                            size_t ws_bytes, moe_stream_t stream, moe_stream_t side_stream);

/*
 * Block-scaled (MX) e4m3 expert path ([MoE-IV] names MXFP8 as the low-precision expert
 * compute; the format read as the published microscaling format for FP8 elements).
 * Every 32 consecutive values of a row along the reduction dimension share one power-of-
 * two scale X = 2^e, stored as one E8M0 byte (e + 127; 255 is never written):
 * e = floor(log2(amax of the 32 values)) - 8, clamped to [-127, 127] (-127 for an
 * all-zero block); code = e4m3 round-to-nearest-even of v / X, saturating at +-448.
 * Scale bytes are row-major [rows, cols / 32] beside the codes [rows, cols].  A GEMM on
 * MX operands computes sum_k (qa_k Xa(k/32)) (qb_k Xb(k/32)) with fp32 accumulation; the
 * scales are applied by the tensor cores (tcgen05 kind::mxf8f6f4.block_scale).  The
 * configuration stays bf16 (dtype = MOE_BF16) and needs d % 512 == 0, I % 128 == 0; x, y,
 * h, the expert outputs and the combine are bf16 / fp32 as in the bf16 path.  Buffers are
 * device memory, 16-byte aligned, owned by the caller.
 */

/* MX quantisation: src [rows, cols] bf16 -> dst [rows, cols] e4m3 codes, sf [rows, cols/32]
 * E8M0 bytes.  cols % 32 == 0.  Used for the weights (once), x and h (per step). */
moe_status moe_quantize_mx(const void* src, int64_t rows, int32_t cols, void* dst, uint8_t* sf,
                           moe_stream_t stream);

/* MX dispatch payload: x_q_perm[tok2row[a]] = x_q[a / k] (d bytes) and x_sf_perm[tok2row[a]]
 * = x_sf[a / k] (d / 32 bytes): the permute of moe_permute on codes and scale rows. */
moe_status moe_permute_mx(const moe_config* cfg, const moe_layout* layout, const void* x_q, const uint8_t* x_sf,
                          void* x_q_perm, uint8_t* x_sf_perm, moe_stream_t stream);

/*
 * MX grouped SwiGLU FFN, routed and shared experts:
 *   h = SiLU(X W_gate^T) * (X W_up^T) on MX operands         (bf16 [A + S*N, I])
 *   h_q, h_sf = the MX quantisation of h (as moe_quantize_mx; done by FC1's epilogue)
 *                                                           (e4m3 [A + S*N, I], E8M0 [A + S*N, I/32])
 *   out = (h W2^T on MX operands) * gate(row)               (bf16 [A + S*N, d])
 *   x_q_perm [A, d] + x_sf_perm [A, d/32] (moe_permute_mx); x_q [N, d] + x_sf [N, d/32]
 *   (the shared experts' rows; NULL when n_shared == 0); w13_q [E+S, 2I, d] + w13_sf
 *   [E+S, 2I, d/32]; w2_q [E+S, d, I] + w2_sf [E+S, d, I/32]; topk_w as in moe_grouped_ffn.
 */
moe_status moe_grouped_ffn_mx(const moe_config* cfg, const moe_layout* layout, const void* x_q_perm,
                              const uint8_t* x_sf_perm, const void* x_q, const uint8_t* x_sf, const void* w13_q,
                              const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf, const float* topk_w,
                              void* h, void* h_q, uint8_t* h_sf, void* out, moe_stream_t stream);

/* Bytes of scratch moe_layer_forward_mx needs (0 for an invalid configuration). */
size_t moe_workspace_bytes_mx(const moe_config* cfg);

/* The whole layer with the MX expert path, one stream: moe_route -> moe_dispatch_layout ->
 * moe_quantize_mx(x) -> moe_permute_mx -> moe_grouped_ffn_mx -> moe_combine.  The weights
 * come quantised (moe_quantize_mx of W13 and W2, once).  ws: 256-byte aligned, of
 * moe_workspace_bytes_mx bytes. */
moe_status moe_layer_forward_mx(const moe_config* cfg, const void* x, const void* w_gate, const float* bias,
                                const int32_t* expert_owner, const void* w13_q, const uint8_t* w13_sf,
                                const void* w2_q, const uint8_t* w2_sf, void* y, const moe_layout* layout_out,
                                int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward_mx with the shared experts overlapped: after the router and the MX
 * quantisation of x on `stream`, the shared experts' MX FFN runs on `side_stream` while
 * the layout, the MX permute and the routed MX FFN run on `stream`; `stream` waits for
 * `side_stream` before the combine.  Same result as moe_layer_forward_mx, bit for bit; two
 * events are created and destroyed per call.  With n_shared == 0 or side_stream == stream
 * this is moe_layer_forward_mx. */
moe_status moe_layer_forward_mx_overlapped(const moe_config* cfg, const void* x, const void* w_gate,
                                           const float* bias, const int32_t* expert_owner, const void* w13_q,
                                           const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf, void* y,
                                           const moe_layout* layout_out, int32_t* dev_status, void* ws,
                                           size_t ws_bytes, moe_stream_t stream, moe_stream_t side_stream);

/* ============================================================================
 * Expert parallelism across GPUs ([EP-DeepEP] §2-3: every rank is a source of tokens
 * and the owner of some experts; dispatch sends each assignment to the owner of its
 * expert, combine returns the outputs to the source; [DeepEP] §2-3: counts are exchanged
 * first, then the all-to-all runs as a transpose; [WideEP]: the count matrix C_ij and
 * the receive load R_j).  One rank per GPU, P = cfg->P ranks, rank r owns the experts
 * with expert_owner[e] == r (or e / (E/P) when expert_owner is NULL), in ascending id.
 *
 * cfg describes THIS rank's batch: cfg->N is the rank's own tokens (its source shard);
 * E, k, d, I, S and the routing rule are the layer's.  Rank r's receive rows are exactly
 * rows [recv_off[r], recv_off[r+1]) of the one-GPU moe_dispatch_layout whose virtual
 * sources are the ranks (the ranks' batches concatenated in rank order): expert-major in
 * ascending id, inside an expert by source rank, then by assignment a.
 *
 * The window.  Every rank allocates one device buffer of moe_ep_window_bytes(cfg,
 * capacity) bytes, zeroes it, and maps every other rank's window into its address space
 * (moe_ep_ipc_handle on the owner's side, moe_ep_ipc_open on the others'), all before
 * any rank's first step.  It holds the step flags, the count table [P, E], the gate and
 * the row of each received assignment (capacity rows) and the expert output rows
 * (capacity routed rows, then S*N shared rows).  capacity = receive rows per owner, the
 * same on every rank; at most the layer's total assignments are ever needed.  When the
 * routing sends more than capacity rows to an owner, the rows beyond it are dropped and
 * MOE_ERR_WORKSPACE is written to *dev_status on every rank.
 *
 * Steps: every rank counts its layer steps in its own window (moe_ep_notify's kernel
 * increments the count; the later calls of the step read it on the device), so the
 * step number is never a call argument and a CUDA graph that captures a step replays
 * correctly.  Every rank must run the same sequence of steps.  Each wait compares a flag
 * with the step number; flags only grow, so nothing is reset between steps.  Every wait
 * is bounded (2 s); on timeout MOE_ERR_TIMEOUT is written to *dev_status and the waiting
 * kernel skips its work, so outputs of that step are undefined but no access leaves its
 * buffer.
 *
 * One step on rank r, in this order on one stream:
 *   moe_ep_notify      the local layout of r's assignments (moe_dispatch_layout with one
 *                      owner); r's per-expert counts stored into row r of every rank's
 *                      count table (peer stores); flag
 *   moe_ep_layout      waits for all P count rows; the destination (owner, row) of each of
 *                      r's assignments and the rows r receives per owned expert
 *   moe_ep_dispatch    each token row read once and stored straight into its owners'
 *                      receive rows (peer stores over NVLink) with its gate; flag
 *   moe_ep_expert_ffn  waits for all P sources; grouped SwiGLU over the received rows
 *                      (FC2 scales each row by its gate) and the shared experts over r's
 *                      own tokens; flag to every source
 *   moe_ep_combine     waits for all P owners; y_t = sum over slots of the owners' output
 *                      rows (peer loads) + the shared rows, fp32, one rounding
 * A step never waits on a later step of another rank, and a rank's next step writes
 * another rank's window only after that rank's previous step has finished with the
 * buffer it writes, so one window serves every step.  moe_ep_layer_forward runs the
 * router and the five calls in this order.  The calls of one step take the same ws.
 *
 * Errors (host, before any launch): grp or grp->windows NULL, rank outside [0, P),
 * local_experts outside [0, E], a window that is NULL or not 256-byte aligned, a NULL
 * array the call needs -> MOE_ERR_INVALID_ARG; capacity < 1, capacity * P >= 2^31 or
 * capacity + S*N >= 2^30 -> MOE_ERR_UNSUPPORTED; ws smaller than the matching
 * moe_ep_workspace_bytes*() -> MOE_ERR_WORKSPACE; plus the moe_config checks.  On the
 * device (*dev_status): an expert id outside [0, E) other than -1 or an owner outside
 * [0, P) -> MOE_ERR_BAD_INDEX; a rank owning another number of experts than
 * local_experts -> MOE_ERR_INVALID_ARG; a routing that overflows capacity ->
 * MOE_ERR_WORKSPACE; a wait that ran out -> MOE_ERR_TIMEOUT.
 * ========================================================================== */

typedef struct {
  int32_t rank;          /* this rank, 0 <= rank < cfg->P */
  int32_t capacity;      /* receive rows per owner (the same on every rank), >= 0 */
  int32_t local_experts; /* experts this rank owns (the routed rows of its w13 / w2) */
  void* const* windows;  /* HOST array [P] of device pointers: each rank's window as mapped in
                            this process; windows[rank] is this rank's own */
} moe_ep_group;

/* This rank's part of the EP layout: caller-owned device arrays, all int32.
 *   dest[N*k]                  owner * capacity + row of each local assignment a in its
 *                              owner's receive rows; -1 = no row (dropped, or beyond capacity)
 *   owner_n_e[local_experts]   rows received per owned expert (ascending expert id)
 *   owner_off[local_experts+1] first receive row of each owned expert; the last entry =
 *                              rows received (at most capacity) */
typedef struct {
  int32_t* dest;
  int32_t* owner_n_e;
  int32_t* owner_off;
} moe_ep_handle;

/* Bytes of one rank's window (0 on an invalid configuration). */
size_t moe_ep_window_bytes(const moe_config* cfg, int32_t capacity);
/* Byte offsets of the window's parts (the same on every rank; a rank's own N only sizes
 * the shared rows at the end): offsets[0..10] = count flags [32] u64, dispatch flags [32]
 * u64, done flags [32] u64 (each indexed by the signalling rank), step counter u64,
 * dispatch counter u32, failed-step word u64 (the last step in which a wait of this rank
 * gave up), count table [P, E] int32, gates [capacity] fp32, token scales [capacity] fp32
 * (FP8 dispatch), received rows [capacity, d] (of d bytes each for the FP8 dispatch; the
 * MX dispatch puts its [capacity, d/32] scale rows right after its capacity code rows),
 * output rows [capacity + S*N, d].  (ABI version 101 added the failed-step word.) */
moe_status moe_ep_window_layout(const moe_config* cfg, int32_t capacity, size_t* offsets);
/* Bytes of scratch the EP calls of one step need (ws; the same ws for all calls of a step
 * and for moe_ep_layer_forward, which also keeps the router outputs and the handle there). */
size_t moe_ep_workspace_bytes(const moe_config* cfg, int32_t capacity);

/* Window mapping (setup, off the hot path).  moe_ep_ipc_handle writes the 64-byte CUDA IPC
 * handle of the allocation that holds `window` to handle[64] and the window's byte offset
 * inside it to *offset; another process passes both to moe_ep_ipc_open, which maps the
 * allocation (peer access enabled lazily) and returns the window's address there;
 * moe_ep_ipc_close(window, offset) unmaps it. */
moe_status moe_ep_ipc_handle(const void* window, void* handle, size_t* offset);
moe_status moe_ep_ipc_open(const void* handle, size_t offset, void** window);
moe_status moe_ep_ipc_close(void* window, size_t offset);

/* Step 1: local layout + count exchange.  topk_ids [N, k] (-1 = dropped). */
moe_status moe_ep_notify(const moe_config* cfg, const moe_ep_group* grp, const int32_t* topk_ids, int32_t* dev_status, void* ws, size_t ws_bytes,
                         moe_stream_t stream);
/* Step 2: destinations.  expert_owner [E] or NULL; fills *handle. */
moe_status moe_ep_layout(const moe_config* cfg, const moe_ep_group* grp, const int32_t* expert_owner, const int32_t* topk_ids, const moe_ep_handle* handle,
                         int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream);
/* Step 3: dispatch.  x [N, d] dtype, topk_w [N, k] fp32 (the gates FC2 applies). */
moe_status moe_ep_dispatch(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                           const float* topk_w, const moe_ep_handle* handle, moe_stream_t stream);
/* Step 4: this owner's experts.  x [N, d] (the shared experts' rows); w13 [local_experts + S,
 * 2I, d] and w2 [local_experts + S, d, I]: the owned experts in ascending id, then the
 * shared experts (the layout of moe_grouped_ffn's weights restricted to this owner). */
moe_status moe_ep_expert_ffn(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                             const void* w13, const void* w2, const moe_ep_handle* handle, int32_t* dev_status,
                             void* ws, size_t ws_bytes, moe_stream_t stream);
/* Step 5: combine into y [N, d] dtype, in token order. */
moe_status moe_ep_combine(const moe_config* cfg, const moe_ep_group* grp, const moe_ep_handle* handle, void* y, int32_t* dev_status, moe_stream_t stream);
/* The layer on this rank: moe_route on its N tokens, then steps 1-5.  handle_out (NULL ok)
 * receives the EP layout instead of the workspace. */
moe_status moe_ep_layer_forward(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                                const void* w_gate, const float* bias, const int32_t* expert_owner,
                                const void* w13, const void* w2, void* y, const moe_ep_handle* handle_out,
                                int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_ep_layer_forward with the shared experts overlapped ([MoE-IV] §4 and [EP-DeepEP]
 * §7: hide the dispatch behind independent compute): after the router on `stream`, the
 * shared experts' GEMMs over this rank's own tokens run on `side_stream` while the count
 * exchange, the dispatch, the wait for the other ranks' rows and the routed GEMMs run on
 * `stream`; `stream` waits for `side_stream` before the combine.  Same y, bit for bit; two
 * events are created and destroyed per call.  With n_shared == 0, N == 0 or side_stream
 * == stream this is moe_ep_layer_forward. */
moe_status moe_ep_layer_forward_overlapped(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                                           const void* w_gate, const float* bias, const int32_t* expert_owner,
                                           const void* w13, const void* w2, void* y, const moe_ep_handle* handle_out,
                                           int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream,
                                           moe_stream_t side_stream);

/* The EP layer with the FP8 expert path (FP8 dispatch, bf16 combine: the e4m3 payload is
 * d bytes per row instead of 2d, so half the NVLink bytes of the dispatch; conventions of
 * moe_quantize_fp8 / moe_grouped_ffn_fp8).  dtype = MOE_BF16, d % 16 == 0, I % 16 == 0.
 *   moe_ep_dispatch_fp8: as moe_ep_dispatch, rows of e4m3 codes x_q [N, d] with each
 *     token's scale x_scale [N] stored beside each of its received rows.
 *   moe_ep_expert_ffn_fp8: as moe_ep_expert_ffn on e4m3 operands: x_q, x_scale are this
 *     rank's own quantised tokens (the shared experts' rows); w13_q [local_experts + S, 2I,
 *     d] e4m3 with w13_scale [local_experts + S, 2I], w2_q [local_experts + S, d, I] e4m3
 *     with w2_scale [local_experts + S, d]; h is quantised per row between FC1 and FC2.
 *   moe_ep_layer_forward_fp8: moe_route, moe_quantize_fp8(x), then the five EP steps with
 *     the two above.  ws of moe_ep_workspace_bytes_fp8 bytes. */
size_t moe_ep_workspace_bytes_fp8(const moe_config* cfg, int32_t capacity);
moe_status moe_ep_dispatch_fp8(const moe_config* cfg, const moe_ep_group* grp, const void* x_q, const float* x_scale,
                               const float* topk_w, const moe_ep_handle* handle, moe_stream_t stream);
moe_status moe_ep_expert_ffn_fp8(const moe_config* cfg, const moe_ep_group* grp, const void* x_q, const float* x_scale,
                                 const void* w13_q, const float* w13_scale, const void* w2_q, const float* w2_scale,
                                 const moe_ep_handle* handle, int32_t* dev_status, void* ws, size_t ws_bytes,
                                 moe_stream_t stream);
moe_status moe_ep_layer_forward_fp8(const moe_config* cfg, const moe_ep_group* grp, const void* x, const void* w_gate,
                                    const float* bias, const int32_t* expert_owner, const void* w13_q,
                                    const float* w13_scale, const void* w2_q, const float* w2_scale, void* y,
                                    const moe_ep_handle* handle_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);
/* moe_ep_layer_forward_fp8 with the shared experts on side_stream (as
 * moe_ep_layer_forward_overlapped; bit for bit the same y). */
moe_status moe_ep_layer_forward_fp8_overlapped(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                                               const void* w_gate, const float* bias, const int32_t* expert_owner,
                                               const void* w13_q, const float* w13_scale, const void* w2_q,
                                               const float* w2_scale, void* y, const moe_ep_handle* handle_out,
                                               int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream,
                                               moe_stream_t side_stream);

/* The EP layer with the MXFP8 expert path (MX dispatch, bf16 combine: the e4m3 code rows
 * travel with their E8M0 scale rows, which land in the window's receive region after the
 * capacity rows of codes, [capacity, d/32] bytes; see moe_quantize_mx / moe_grouped_ffn_mx).
 * dtype = MOE_BF16, d % 512 == 0, I % 128 == 0.
 *   moe_ep_dispatch_mx: as moe_ep_dispatch, code rows x_q [N, d] and scale rows x_sf
 *     [N, d/32] of this rank's tokens.
 *   moe_ep_expert_ffn_mx: as moe_ep_expert_ffn on MX operands: x_q, x_sf are this rank's
 *     tokens (the shared experts' rows); w13_q [local+S, 2I, d] + w13_sf [local+S, 2I, d/32],
 *     w2_q [local+S, d, I] + w2_sf [local+S, d, I/32].
 *   moe_ep_layer_forward_mx(_overlapped): moe_route, moe_quantize_mx(x), then the five EP
 *     steps with the two above (shared experts on side_stream in the overlapped form).
 *     ws of moe_ep_workspace_bytes_mx bytes. */
size_t moe_ep_workspace_bytes_mx(const moe_config* cfg, int32_t capacity);
moe_status moe_ep_dispatch_mx(const moe_config* cfg, const moe_ep_group* grp, const void* x_q, const uint8_t* x_sf,
                              const float* topk_w, const moe_ep_handle* handle, moe_stream_t stream);
moe_status moe_ep_expert_ffn_mx(const moe_config* cfg, const moe_ep_group* grp, const void* x_q, const uint8_t* x_sf,
                                const void* w13_q, const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf,
                                const moe_ep_handle* handle, int32_t* dev_status, void* ws, size_t ws_bytes,
                                moe_stream_t stream);
moe_status moe_ep_layer_forward_mx(const moe_config* cfg, const moe_ep_group* grp, const void* x, const void* w_gate,
                                   const float* bias, const int32_t* expert_owner, const void* w13_q,
                                   const uint8_t* w13_sf, const void* w2_q, const uint8_t* w2_sf, void* y,
                                   const moe_ep_handle* handle_out, int32_t* dev_status, void* ws, size_t ws_bytes,
                                   moe_stream_t stream);
moe_status moe_ep_layer_forward_mx_overlapped(const moe_config* cfg, const moe_ep_group* grp, const void* x,
                                              const void* w_gate, const float* bias, const int32_t* expert_owner,
                                              const void* w13_q, const uint8_t* w13_sf, const void* w2_q,
                                              const uint8_t* w2_sf, void* y, const moe_ep_handle* handle_out,
                                              int32_t* dev_status, void* ws, size_t ws_bytes, moe_stream_t stream,
                                              moe_stream_t side_stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
