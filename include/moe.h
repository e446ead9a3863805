/*

 * The token-direction codes (XT_Q, HT_Q, GT_Q, YT_Q, a [C,R] matrix) are stored in
 * 128 x 128 tiles: the tile of features [128 fb, 128 fb + 128) and tokens [128 tb,
 * 128 tb + 128) is 16384 contiguous bytes at offset (tb * C/128 + fb) * 16384, row-major
 * inside (128 feature rows of 128 token bytes); their scales are the UMMA layout of [C,R]. * moe.h -- C ABI of the B200 (sm_100a) Mixture-of-Experts layer hot path.
 *
 * The method is the one described in "Cursor's MoK achieves 2.37x performance boost on
 * NVIDIA GB300 NVL72" (kucoin news flash article): a single MoE layer that routes tokens
 * to experts, lays them out contiguously per expert, runs the expert SwiGLU FFNs as a
 * grouped GEMM on MXFP8 operands and combines the results back into token order with the
 * routing weights, plus the matching backward pass.  On one GPU the article's dispatch
 * and combine communications become on-device permutations.
 *
 * Conventions for every entry point
 *   - Pointers are caller-owned DEVICE memory unless stated otherwise; row-major and
 *     contiguous.  bf16 tensors are passed as uint16_t bit patterns.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream), never allocates device memory, never synchronises and never copies
 *     routing counts to the host (buffers are sized for the worst case instead).
 *   - Host-side argument checks return an error before anything is launched.  Errors
 *     found on the device (an index out of bounds, a bounded wait that ran out) are
 *     latched into a status word inside the workspace and read back with
 *     moe_get_device_status(); device code never traps.
 *   - Shapes: d % 256 == 0, f % 256 == 0, 1 <= k <= min(E, 32), 1 <= E <= 1024, T >= 0,
 *     T*k + 127*E + 127 < 2^31 (the padded row count fits int32).  Pointers must be
 *     16-byte aligned; workspaces 256-byte aligned, and the first 256 bytes of a
 *     workspace must be zero when it is first used (they hold the latched device status).
 *
 * Notation: T tokens, d hidden size, f expert intermediate size, E experts, k experts per
 * token, A = T*k assignments with id a = t*k + j (j = rank of the expert among the
 * token's k choices), R = moe_padded_rows(): rows of the expert-contiguous operand
 * buffers, in which expert e's segment starts at pad_offsets[e] (a multiple of 128).
 *
 * MX layouts.  MXFP8 = E4M3 bytes plus one E8M0 scale byte per 32 consecutive elements
 * along the GEMM reduction axis K (OCP MX v1.0).  "Canonical" scales of a [rows, K]
 * matrix are [rows, K/32] bytes.  The "UMMA" scale layout (the one the tcgen05
 * block-scaled MMA consumes) stores the scales of a [rows, K] matrix (rows a multiple of
 * 128, K a multiple of 128) in 512-byte chunks, one per (128-row block rb, 128-column
 * group kg), chunk index rb*(K/128) + kg; inside a chunk the scale of row r and 32-block
 * kb sits at byte (r%32)*16 + ((r%128)/32)*4 + (kb%4).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum */
  MOE_ERR_UNSUPPORTED_SHAPE = 2, /* outside the shape rules above */
  MOE_ERR_MISALIGNED = 3,        /* pointer not 16-byte (workspace: 256-byte) aligned */
  MOE_ERR_WORKSPACE_TOO_SMALL = 4,
  MOE_ERR_CUDA = 5,              /* a CUDA runtime call failed (launch, attribute, ...) */
  MOE_ERR_DEVICE_TIMEOUT = 6,    /* latched: a bounded device-side wait ran out */
  MOE_ERR_DEVICE_BOUNDS = 7,     /* latched: a device-side index check failed */
  MOE_ERR_NO_DEVICE = 8          /* no usable sm_100 device */
} moe_status;

typedef enum { MOE_SCORE_SOFTMAX_TOPK = 0, MOE_SCORE_SIGMOID_RENORM = 1 } moe_score_fn;

typedef enum {
  MOE_OP_ROUTE = 0,
  MOE_OP_FORWARD = 1,
  MOE_OP_BACKWARD = 2,
  MOE_OP_FORWARD_BF16 = 3, /* moe_forward_bf16 */
  MOE_OP_ROUTER = 4        /* moe_router_logits, moe_router_grads */
} moe_op;

typedef struct {
  int64_t T;         /* tokens */
  int32_t d, f, E, k;
  int32_t score_fn;  /* moe_score_fn */
} moe_dims;

/* Expert weights in the layouts the grouped GEMMs read (written by moe_prepare_weights;
 * sizes from moe_weights_bytes).  All MX; scales in the UMMA layout of the stated matrix. */
typedef struct {
  uint8_t *wgu_q;   /* [E*2f, d] E4M3: per expert, 128-row blocks alternate W_gate^T block j,
                       W_up^T block j (rows = output features, K = d)                       */
  uint8_t *wgu_s;   /* UMMA scales of the [E*2f, d] matrix                                 */
  uint8_t *wd_q;    /* [E*d, f]: W_down^T per expert (rows = output features, K = f)       */
  uint8_t *wd_s;    /* UMMA scales of the [E*d, f] matrix                                  */
  uint8_t *wdT_q;   /* backward, nullable: [E*f, d] = W_down as stored, K = d              */
  uint8_t *wdT_s;
  uint8_t *wguT_q;  /* backward, nullable: [E*d, 2f] = [W_gate | W_up], K = 2f             */
  uint8_t *wguT_s;
} moe_weights;

/* Forward state kept for the backward pass (all device buffers, caller-owned).  With no
 * tokens (T == 0) the token-sized arrays topk_idx, topk_w, perm and inv_perm hold nothing
 * and may be NULL. */
typedef struct {
  int32_t *topk_idx;     /* [T,k]  expert of assignment a                                */
  float   *topk_w;       /* [T,k]  combine weight                                       */
  int32_t *counts;       /* [E]                                                         */
  int32_t *offsets;      /* [E+1]  exclusive prefix sum of counts, offsets[E] = A       */
  int32_t *perm;         /* [A]    position -> assignment id (expert-contiguous)        */
  int32_t *inv_perm;     /* [A]    assignment id -> position                            */
  int32_t *pad_offsets;  /* [E+1]  padded segment starts, multiples of 128              */
  uint8_t *xq;           /* [R,d]  MX codes of x, permuted (row pad_offsets[e]+r)         */
  uint8_t *xs;           /* UMMA scales of the [R,d] matrix                             */
  uint8_t *hq;           /* [R,f]  MX codes of silu(g)*u                                */
  uint8_t *hs;           /* UMMA scales of the [R,f] matrix                             */
  uint16_t *gu;          /* [R,2f] bf16 SwiGLU pre-activations: g in [0,f), u in [f,2f) */
} moe_saved;

/* ---- sizes (pure host arithmetic, no CUDA call) -------------------------------------- */
int64_t moe_padded_rows(const moe_dims* dims);
/* Bytes of the UMMA scale layout of a [rows, K] matrix (rows rounded up to 128). */
int64_t moe_umma_scale_bytes(int64_t rows, int64_t K);
/* Bytes of moe_weights field `field` (0 wgu_q, 1 wgu_s, 2 wd_q, 3 wd_s, 4 wdT_q, 5 wdT_s,
 * 6 wguT_q, 7 wguT_s); -1 on bad arguments. */
int64_t moe_weights_bytes(const moe_dims* dims, int32_t field);
/* Bytes of moe_saved field `field` in struct order (0 topk_idx ... 11 gu); -1 on error. */
int64_t moe_saved_bytes(const moe_dims* dims, int32_t field);
/* Workspace bytes for an operation (moe_op); 0 on bad arguments. */
size_t moe_workspace_bytes(const moe_dims* dims, int32_t op);
/* Inspection of intermediate results (tests, debugging): the byte offset inside an
 * operation's workspace of one internal buffer, -1 if that operation has no such buffer.
 * The contents are those of the last call that used the workspace, once it has completed
 * on its stream; the layouts are the ones stated per buffer.  R = moe_padded_rows().
 * "Scaled fp16" [rows, C]: fp16 values q and, separately, one byte b per 32 consecutive
 * values of a row ([rows, C/32]); the value is q * 2^(b - 127). */
typedef enum {
  MOE_WS_MTILE = 0,   /* every op: [E+1] int32, 128-row tiles per expert, prefix-summed     */
  MOE_WS_Y = 1,       /* forward: [R,d] expert outputs y, scaled fp16 values (padded order) */
  MOE_WS_DOUT_Q = 2,  /* backward: [R,d] MX codes of dOut gathered to expert order          */
  MOE_WS_DOUT_S = 3,  /*   their UMMA scales                                                */
  MOE_WS_G = 4,       /* backward: [R,f] fp32 G = dOut^ . W_down'^T                          */
  MOE_WS_DGU_Q = 5,   /* backward: [R,2f] MX codes of [dg | du] (along 2f)                   */
  MOE_WS_DGU_S = 6,
  MOE_WS_DXA = 7,     /* backward: [R,d] per-assignment input gradients, scaled fp16 values  */
  MOE_WS_XT_Q = 8,    /* backward: [d,R] token-direction MX of x^ (UMMA scales of [d,R])     */
  MOE_WS_XT_S = 9,
  MOE_WS_HT_Q = 10,   /* backward: [f,R] token-direction MX of h^                            */
  MOE_WS_HT_S = 11,
  MOE_WS_GT_Q = 12,   /* backward: [2f,R] token-direction MX of [dg|du]^                      */
  MOE_WS_GT_S = 13,
  MOE_WS_YT_Q = 14,   /* backward: [d,R] token-direction MX of w * dOut^                      */
  MOE_WS_YT_S = 15,
  MOE_WS_COUNTS = 16, /* forward without a saved struct: [E] int32 tokens per expert        */
  MOE_WS_Y_S = 17,    /* forward: [R,d/32] scale bytes of MOE_WS_Y                           */
  MOE_WS_DXA_S = 19   /* backward: [R,d/32] scale bytes of MOE_WS_DXA                        */
} moe_ws_buffer;
int64_t moe_workspace_offset(const moe_dims* dims, int32_t op, int32_t buffer);

/* Tile-scheduler wave rule: the smallest token count M for which the tile_m x tile_n
 * output tiles of an M x n_cols GEMM fill `waves` full waves on `num_sms` SMs:
 * M = ceil(waves * num_sms * tile_m * tile_n / n_cols).  Article §02: a minibatch should
 * make at least two full waves; 2368 tokens at hidden 7168 / expert intermediate 2048
 * (gate/up GEMM, n_cols = 2*2048, 148 SMs, 128 x 256 tiles).  -1 on bad arguments. */
int64_t moe_min_tokens_for_waves(int32_t num_sms, int32_t waves, int32_t tile_m,
                                 int32_t tile_n, int64_t n_cols);

const char* moe_status_string(moe_status s);

/* ---- routing and layout ---------------------------------------------------------------
 * Article lead and §01 (router picks experts per token; count tokens per expert, decide
 * placement, keep each expert's tokens contiguous).
 * logits [T,E] fp32 -> topk_idx [T,k] (top-k by logit, ties to the lower expert index,
 * slot j = rank; a NaN logit ranks as -inf, so every index is a valid expert),
 * topk_w [T,k] (softmax over the k selected logits, or sigmoid scores renormalised over
 * the k selected), counts [E], offsets [E+1], perm [A] (stable:
 * ascending token inside each expert), inv_perm [A].  Indices are exact; weights fp32.
 * pad_offsets [E+1] (nullable): padded segment starts.  ws: moe_workspace_bytes(ROUTE). */
moe_status moe_route_layout(const moe_dims* dims, const float* logits, int32_t* topk_idx,
                            float* topk_w, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* inv_perm, int32_t* pad_offsets, void* ws,
                            size_t ws_bytes, void* stream);

/* ---- routing and layout without a workspace ---------------------------------------
 * No counterpart in the article: an addition for callers that cannot allocate device
 * memory themselves (a plugin whose host framework owns every device allocation, an
 * embedded runtime with a fixed memory budget, or a latency-critical path where
 * cudaMalloc's implicit device synchronisation is not acceptable).  Same inputs, outputs
 * and results as moe_route_layout, but the scratch lives in a fixed 8 MiB array inside
 * the library (held by every GPU that loads the library until the process exits);
 * nothing is allocated and no workspace is passed.
 *  - The shape rules, pointer checks and device check are those of moe_route_layout.
 *    Problems whose scratch exceeds 8 MiB return MOE_ERR_UNSUPPORTED_SHAPE before any
 *    launch.  The scratch is 256 + 8*nt*E + 4*T*k + 4*(E+1) bytes (each term rounded up
 *    to 256) with nt = ceil(T/64): e.g. E = 256, k = 8 fits T <= 131024.
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress; it allocates nothing), so a device reset is picked up; make
 *    the first call on a device before any stream capture.
 *  - Every call shares the one array: calls whose executions overlap on the GPU race on
 *    it and give wrong results.  Each call clears the parts that must start at zero.
 *  - status (device int32, zeroed by the caller; required when T > 0): device-side
 *    errors are latched there (first error wins) instead of in a workspace. */
moe_status moe_route_layout_noalloc(const moe_dims* dims, const float* logits,
                                    int32_t* topk_idx, float* topk_w, int32_t* counts,
                                    int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                                    int32_t* pad_offsets, int32_t* status, void* stream);

/* ---- MXFP8 quantiser ------------------------------------------------------------------
 * Article §02 (MXFP8 activations fused into dispatch, grouped GEMM and SwiGLU); format:
 * OCP MX v1.0 (s = floor(log2 amax) - 8 clamped to [-127,127], E4M3 round-to-nearest-even
 * with saturation to 448; an all-zero block gets scale byte 0).
 * in [rows, K] bf16 with row stride ld (elements) -> q [rows, K] E4M3, scales:
 * scale_layout 0 = canonical [rows, K/32]; 1 = UMMA layout (K % 128 == 0; the buffer
 * must hold moe_umma_scale_bytes(rows, K); entries of rows >= rows are not written).
 * K % 32 == 0. */
moe_status mxfp8_quantize(const uint16_t* in, int64_t rows, int64_t K, int64_t ld,
                          uint8_t* q, uint8_t* scales, int32_t scale_layout, void* stream);

/* ---- weight preparation (setup, not part of the timed layer) ---------------------------
 * W_gate, W_up [E,d,f] and W_down [E,f,d] bf16 (x @ W convention) -> the MX layouts of
 * moe_weights.  with_backward_copies != 0 also fills wdT_* and wguT_*. */
moe_status moe_prepare_weights(const moe_dims* dims, const uint16_t* w_gate,
                               const uint16_t* w_up, const uint16_t* w_down,
                               int32_t with_backward_copies, const moe_weights* out,
                               void* stream);

/* ---- forward --------------------------------------------------------------------------
 * Article §02/§03: route -> layout -> pull dispatch with fused MXFP8 quantisation ->
 * grouped GEMM gate/up with SwiGLU and MXFP8 requantisation in the epilogue -> grouped
 * GEMM down -> push combine / final weighted merge.
 * x [T,d] bf16, logits [T,E] fp32 -> out [T,d] bf16, out_t = sum_j w[t,j] * y_{t*k+j}.
 * saved: nullable (inference); when given, every field must be non-null and is filled
 * for moe_backward.  ws: moe_workspace_bytes(FORWARD). */
moe_status moe_forward(const moe_dims* dims, const moe_weights* w, const uint16_t* x,
                       const float* logits, uint16_t* out, const moe_saved* saved,
                       void* ws, size_t ws_bytes, void* stream);

/* ---- the layer's BF16 variant ----------------------------------------------------------
 * Article §03 (MoE-layer results are reported with BF16 as well as MXFP8 operands).  The
 * same layer with bf16 operands throughout and no MX quantisation: g = x Wg, u = x Wu,
 * h = bf16(silu(g) * u) (round to nearest even), y = h Wd, out_t = sum_j w[t,j] y_{t*k+j}
 * (fp32 accumulation, bf16 output), on the 5th-generation tensor cores with
 * tcgen05.mma kind::f16.
 *
 * moe_prepare_weights_bf16: W_gate, W_up [E,d,f], W_down [E,f,d] bf16 (x @ W convention) ->
 * wgu_t [E*2f, d] bf16 (per expert, 128-row blocks alternate W_gate^T block j and W_up^T
 * block j, as the MX layout) and wd_t [E*d, f] (W_down^T per expert); 2*E*2f*d and
 * 2*E*d*f bytes.  Setup, not part of the layer's step.
 * moe_forward_bf16: x [T,d] bf16, logits [T,E] fp32 -> out [T,d] bf16; routing as
 * moe_route_layout; ws: moe_workspace_bytes(MOE_OP_FORWARD_BF16). */
moe_status moe_prepare_weights_bf16(const moe_dims* dims, const uint16_t* w_gate,
                                    const uint16_t* w_up, const uint16_t* w_down,
                                    uint16_t* wgu_t, uint16_t* wd_t, void* stream);
moe_status moe_forward_bf16(const moe_dims* dims, const uint16_t* wgu_t, const uint16_t* wd_t,
                            const uint16_t* x, const float* logits, uint16_t* out, void* ws,
                            size_t ws_bytes, void* stream);

/* ---- backward -------------------------------------------------------------------------
 * Article §01/§02 (backward = pull reverse-combine + push reverse-dispatch).
 * dout [T,d] bf16 + saved -> dx [T,d] bf16, dw_route [T,k] fp32 (d loss / d topk_w),
 * dWg, dWu [E,d,f] bf16, dWd [E,f,d] bf16.  Needs the backward weight copies.
 * Every backward GEMM operand is MX-quantised along that GEMM's K (the weight gradients
 * along each expert's tokens); accumulation fp32.  For d >= 6144 the SwiGLU backward of
 * an expert's full 128-row tiles runs in the epilogue of the dgrad GEMM of the down
 * projection (its K = d is then long enough to hide that work); below that width, and for
 * every expert's partial last tile, it runs in its own kernel.  The results are the same
 * either way.  ws: moe_workspace_bytes(BACKWARD). */
moe_status moe_backward(const moe_dims* dims, const moe_weights* w, const moe_saved* saved,
                        const uint16_t* dout, uint16_t* dx, float* dw_route, uint16_t* dWg,
                        uint16_t* dWu, uint16_t* dWd, void* ws, size_t ws_bytes,
                        void* stream);

/* ---- router backward -------------------------------------------------------------------
 * Article lead and §01 (the router picks each token's experts at every training step, so
 * training needs the gradient that reaches the router).  d(loss)/d(logits) [T,E] fp32 from
 * d(loss)/d(combine weights) dw_route [T,k] (the output of moe_backward), the logits [T,E]
 * and the selected experts topk_idx [T,k] of the forward.  The selection is piecewise
 * constant, so the E - k unselected logits of a token get exactly 0; the k selected ones
 * get the chain rule of the score function (softmax over the selected logits:
 * w_i (dw_i - sum_j w_j dw_j); sigmoid renormalised: s_i (1 - s_i)(dw_i - sum_j w_j dw_j)/S
 * with S = sum_j s_j), the weights recomputed from the logits as moe_route_layout forms
 * them.  dims->d and dims->f only have to satisfy the shape rules.  status (nullable,
 * device int32): an expert id outside [0, E) latches MOE_ERR_DEVICE_BOUNDS there and leaves
 * that token's row unwritten. */
moe_status moe_router_backward(const moe_dims* dims, const float* logits,
                               const int32_t* topk_idx, const float* dw_route, float* dlogits,
                               int32_t* status, void* stream);

/* ---- router GEMM in front of the routing step ------------------------------------------
 * Article lead and §01 (at every step a router decides which experts each token goes to;
 * the pages give no formula: read as a bias-free linear layer whose outputs are the
 * logits moe_route_layout ranks).
 *   logits[t, e] = sum_i x[t, i] * wr[e, i]
 * x [T,d] bf16 and wr [E,d] bf16 (one row per expert: a linear layer's weight layout),
 * row-major; logits [T,E] fp32.  Runs on the tensor cores (tcgen05.mma kind::f16, fp32
 * accumulation) as a one-group grouped GEMM; W_r is first copied into the workspace padded
 * to whole 256-expert tiles.  Needs E % 8 == 0 (besides the moe_dims rules); workspace of
 * moe_workspace_bytes(dims, MOE_OP_ROUTER) bytes, 256-byte aligned, caller-owned, no
 * zeroing needed; device status latched at its offset 0.  All pointers device memory,
 * 16-byte aligned; nothing is allocated, nothing synchronised. */
moe_status moe_router_logits(const moe_dims* dims, const uint16_t* x, const uint16_t* wr,
                             float* logits, void* ws, size_t ws_bytes, void* stream);

/* ---- router GEMM backward ----------------------------------------------------------------
 * Article lead and §01 (training differentiates through the router).  From the logits'
 * gradient G [T,E] fp32 (e.g. moe_router_backward's output):
 *   dx_r[t, i] = sum_e bf16(G[t, e]) * wr[e, i]     [T,d] fp32: the router's share of dx
 *   dwr[e, i]  = sum_t bf16(G[t, e]) * x[t, i]      [E,d] fp32
 * bf16(.) rounds to nearest, ties to even: both products run on the tensor cores with bf16
 * operands and fp32 accumulation, like the forward.  The operand copies it needs (bf16(G)
 * and its transpose, W_r^T, x^T, zero-padded to whole tiles) live in the workspace
 * (MOE_OP_ROUTER size).  T == 0 writes dwr = 0.  Same rules as moe_router_logits. */
moe_status moe_router_grads(const moe_dims* dims, const float* dlogits, const uint16_t* x,
                            const uint16_t* wr, float* dx_r, float* dwr, void* ws,
                            size_t ws_bytes, void* stream);

/* ---- expert parallelism over NVLink ------------------------------------------------------
 * Article §01 and §02: G GPUs ("ranks") each own E/G experts (rank r: experts
 * [r*E/G, (r+1)*E/G)) and route their own tokens; the owner of an expert pulls the rows it
 * needs from the tokens' GPUs by source and offset into its own memory (pull dispatch),
 * runs its grouped GEMMs, and pushes each output row back to its token's GPU (push
 * combine), where the weighted merge runs.  Peers are reached through a device array of
 * moe_ep_peer entries, one per rank, read and written by these kernels with plain loads
 * and stores: on a multi-GPU node the entries hold peer mappings of the other GPUs'
 * buffers (CUDA IPC or symmetric memory, NVLink traffic); with one GPU, buffers of several
 * ranks on that GPU.  A step has three phases; every rank starts a phase only once every
 * rank has finished the previous one (a barrier between phases, e.g. a stream-ordered
 * NCCL all-reduce of one word; with one GPU, stream order):
 *   1. moe_ep_prepare  (each rank)  route + layout of its tokens, MX quantisation of x
 *   2. moe_ep_experts  (each rank)  pull its experts' rows from every rank, gate/up +
 *                                   SwiGLU + MX requant, down, push the rows back
 *   3. moe_ep_combine  (each rank)  out[t] = sum_j w[t,j] * y[t*k + j]
 * The result equals moe_forward on each rank's tokens: the same operands and per-row
 * arithmetic, only the rows' placement in the GEMM tiles differs. */
typedef struct {
  int64_t T;               /* tokens of this rank */
  const int32_t* counts;   /* [E] rows per expert (moe_ep_prepare) */
  const int32_t* offsets;  /* [E+1] exclusive prefix of counts */
  const int32_t* perm;     /* [T*k] position -> assignment id a = t*k + j */
  const uint8_t* xq;       /* [T, d] E4M3 codes of the rank's tokens, along d */
  const uint8_t* xs;       /* [T, d/32] their E8M0 scale bytes, row-major */
  uint16_t* y;             /* [T*k, d] expert outputs pushed back (scaled fp16 values) */
  uint8_t* ys;             /* [T*k, d/32] their scale bytes (common to 32 columns) */
} moe_ep_peer;

/* Phase 1: dims->T = this rank's tokens, dims->E = all experts.  moe_route_layout's outputs
 * plus xq [T,d], xs [T,d/32] (row-major scales).  ws: moe_workspace_bytes(ROUTE). */
moe_status moe_ep_prepare(const moe_dims* dims, const uint16_t* x, const float* logits,
                          int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                          int32_t* perm, int32_t* inv_perm, uint8_t* xq, uint8_t* xs,
                          void* ws, size_t ws_bytes, void* stream);
/* Workspace of moe_ep_experts: dims->T = the tokens of ALL ranks together (the receive
 * buffer holds the worst case, sum_s T_s * min(k, E/G) rows plus tile padding, so no
 * count ever goes to the host); 0 on bad arguments (E % world != 0, world outside 1..64). */
size_t moe_ep_workspace_bytes(const moe_dims* dims, int32_t world);
/* Phase 2 on rank `rank`: dims as for moe_ep_workspace_bytes; peers [world] device array;
 * w: this rank's E/G experts, prepared by moe_prepare_weights with dims.E = E/G (expert
 * r*E/G + i of the layer is its expert i).  Received rows are laid out expert by expert,
 * source rank by source rank, in each source's segment order.  A count or index found out
 * of range latches MOE_ERR_DEVICE_BOUNDS (status at the workspace's offset 0) and the rank
 * then receives nothing. */
moe_status moe_ep_experts(const moe_dims* dims, int32_t rank, int32_t world,
                          const moe_ep_peer* peers, const moe_weights* w, void* ws,
                          size_t ws_bytes, void* stream);
/* Phase 3: dims->T = this rank's tokens; y, ys: this rank's moe_ep_peer.y / .ys, filled by
 * every owner's push; out [T,d] bf16.  status: nullable device int32 (bounds latch). */
moe_status moe_ep_combine(const moe_dims* dims, const float* topk_w, const uint16_t* y,
                          const uint8_t* ys, uint16_t* out, int32_t* status, void* stream);

/* ---- grouped block-scaled GEMM (the engine of the expert FFN, exposed for direct use)
 * For each group g and each row r in [128*mtile_prefix[g], 128*mtile_prefix[g+1]):
 *   D[r, n] = sum_k A[r,k] * B[g*N + n, k],  n < N,  fp32 accumulation, fp32 output
 * with A [R,K] / B [G*N,K] MX (UMMA scales).  mtile_prefix [G+1] is device memory
 * (128-row tiles per group, prefix-summed); rows_valid [G] (nullable) gives the valid
 * rows of each group: a group's last tile then runs only as wide as its valid rows, and
 * rows past rows_valid[g] inside the group's tiles receive unspecified values.
 * N % 256 == 0, K % 128 == 0, R = 128*mtile_prefix[G] at most rows_a; d_out [rows_a, N]
 * fp32, 16-byte aligned with N*4 a multiple of 16. */
moe_status moe_grouped_gemm_mx(int32_t G, int64_t rows_a, int32_t N, int32_t K,
                               const int32_t* mtile_prefix, const int32_t* rows_valid,
                               const uint8_t* a_q, const uint8_t* a_s, const uint8_t* b_q,
                               const uint8_t* b_s, float* d_out, void* ws, size_t ws_bytes,
                               void* stream);

/* ---- failure-detection test hook -------------------------------------------------------
 * Article §02 (device-local counters signal that a minibatch of dispatched rows is ready;
 * the grouped GEMM waits on them).  For tests of the bounded wait only: from the next
 * moe_forward / moe_backward on, the dispatch never publishes minibatch `minibatch` (its
 * rows are still written); the GEMM's wait for it gives up after its time limit (2 s),
 * latches MOE_ERR_DEVICE_TIMEOUT in the workspace and the CTAs leave cleanly, so the
 * results of that call are garbage but the context stays usable.  A negative value turns
 * the hook off (the default). */
moe_status moe_debug_withhold_ready(int32_t minibatch);

/* ---- grouped bf16 GEMM (the engine of the BF16 variant, exposed for direct use) --------
 * As moe_grouped_gemm_mx with bf16 operands A [rows_a, K] and B [G*N, K] (row-major, K
 * contiguous) and no scales: D[r, n] = sum_k A[r,k] * B[g*N + n, k], fp32 accumulation and
 * output.  N % 256 == 0, K % 64 == 0, rows_a % 128 == 0; ws >= 256 bytes. */
moe_status moe_grouped_gemm_bf16(int32_t G, int64_t rows_a, int32_t N, int32_t K,
                                 const int32_t* mtile_prefix, const int32_t* rows_valid,
                                 const uint16_t* a, const uint16_t* b, float* d_out, void* ws,
                                 size_t ws_bytes, void* stream);

/* ---- per-stage timing (measurement support) ------------------------------------------
 * Stage ids of moe_forward / moe_backward launches. */
typedef enum {
  MOE_STAGE_ROUTE = 0,      /* routing, layout, perm/inv scatter                       */
  MOE_STAGE_PERMUTE = 1,    /* pull dispatch with MXFP8 quantisation                    */
  MOE_STAGE_GATEUP = 2,     /* grouped GEMM gate/up + SwiGLU + requantisation            */
  MOE_STAGE_DOWN = 3,       /* grouped GEMM down                                        */
  MOE_STAGE_COMBINE = 4,    /* weighted combine / un-permute                            */
  MOE_STAGE_BWD_DOUT = 5,   /* backward: dOut quantisation + gather                     */
  MOE_STAGE_BWD_DGRAD_DOWN = 6,
  MOE_STAGE_BWD_DGRAD_GATEUP = 7,
  MOE_STAGE_BWD_DX = 8,
  MOE_STAGE_BWD_TRANSPOSE = 9,
  MOE_STAGE_BWD_WGRAD = 10,
  MOE_STAGE_BWD_SWIGLU = 11, /* d(router weights) + SwiGLU backward + MX of dg|du       */
  MOE_STAGE_EP_PULL = 12,   /* expert parallelism: receive layout + pull dispatch         */
  MOE_STAGE_EP_PUSH = 13,   /* expert parallelism: push of the expert outputs             */
  MOE_NUM_STAGES = 14
} moe_stage;

/* When enabled, every stage launched by moe_forward / moe_backward / moe_ep_experts /
 * moe_ep_combine is bracketed by CUDA
 * events on the launch stream (host-side bookkeeping only; not for use during graph
 * capture).  The events serialise the stages (the gate/up GEMM then starts after the dispatch
 * has finished instead of as its CTAs retire).  moe_profile_collect synchronises on the recorded events, writes the summed
 * milliseconds and the number of bracketed launches per stage id, and clears the record. */
moe_status moe_profile_enable(int32_t on);
moe_status moe_profile_collect(double* ms_per_stage, int32_t* launches_per_stage,
                               int32_t n_stages);

/* ---- device status ------------------------------------------------------------------
 * Synchronises `stream`, returns the status latched in the workspace (MOE_OK if none)
 * in *code and clears it. */
moe_status moe_get_device_status(void* ws, void* stream, int32_t* code);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
