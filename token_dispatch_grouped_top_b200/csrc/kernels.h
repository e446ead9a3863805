// Launch interfaces of the MoE-layer kernels (host <-> device plumbing, no torch types).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Host-side checks shared by the entry points (api.cu): the shape rules of moe.h (no
// CUDA call), and the current device's SM count (MOE_ERR_NO_DEVICE unless sm_100).
moe_status check_dims(const moe_dims* D);
moe_status device_sms(int* num_sms);

struct RouteParams {
  const float* logits;
  int64_t T;
  int E, k, score_fn;
  int num_tiles;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* rank;          // [A] rank of each assignment among its tile's rows of the expert
  int32_t* counts;        // [E]
  int32_t* offsets;       // [E+1]
  int32_t* mtile_prefix;  // [E+1] 128-row tiles per expert, prefix-summed
  int32_t* pad_offsets;   // [E+1] nullable
  uint32_t* tile_counter;
  uint32_t* done_counter;
  int32_t* agg;           // [num_tiles, E] each tile's count per expert
  int32_t* tile_start;    // [num_tiles, E] each tile's first rank inside each expert
  int32_t* status;
};

cudaError_t launch_route_layout(const RouteParams& P, int32_t* perm, int32_t* inv, int num_sms,
                                cudaStream_t stream);
int route_num_tiles(int64_t T);

// Row quantiser: rows of a bf16 matrix -> E4M3 + scales (canonical or UMMA layout).
struct QuantRowsParams {
  const uint16_t* src;
  int64_t src_ld;        // elements
  int64_t rows;
  int64_t K;             // elements per row to quantise (multiple of 32)
  uint8_t* dst;          // row r written at dst + r*dst_ld + dst_col0
  int64_t dst_ld;
  int64_t dst_col0;
  uint8_t* scales;
  int layout;            // 0 canonical [rows, K/32] (dst_col0 must be 0), 1 UMMA
  int64_t kgroups;       // UMMA: (total K of the destination matrix) / 128
};
cudaError_t launch_quant_rows(const QuantRowsParams& P, int num_sms, cudaStream_t stream);

// Column quantiser for weights: W [G][K][ncols] bf16, column n of group g quantised along K
// and written as row rowmap(g, n) of a [*, K] E4M3 matrix with UMMA scales.
struct QuantColsParams {
  const uint16_t* src;
  int G, K, ncols;
  uint8_t* dst;
  uint8_t* scales;
  int64_t kgroups;       // K / 128
  int map_mode;          // 0: row = g*ncols + n; 1: gate/up interleave (see moe.h) with
  int interleave_half;   //    half (0 gate, 1 up): row = g*2*ncols + (n/128)*256 + half*128 + n%128
};
cudaError_t launch_quant_cols(const QuantColsParams& P, cudaStream_t stream);

// Pull gather of per-token MX rows: q_out[pad_offsets[e] + r] = q_tok[perm[offsets[e]+r]/k],
// scales from the canonical per-token layout [T, d/32] into the UMMA layout of [R, d]
// (s_tok nullable: rows only).
struct GatherParams {
  // ready (nullable): after writing a row, its minibatch counter ready[row / ready_rows] is
  // decremented (release); withhold >= 0 skips that minibatch's decrements (a test hook
  // that makes a consumer's bounded wait run out).
  int32_t* ready;
  int ready_rows;
  int withhold;
  int64_t row_bytes;     // bytes per row: d (MX codes) or 2d (bf16 rows, s_tok == nullptr)
  const uint8_t* q_tok;
  const uint8_t* s_tok;
  int64_t T;
  int d, E, k;
  const int32_t* offsets;
  const int32_t* mtile_prefix;
  int prefix_shift;
  const int32_t* perm;
  uint8_t* q_out;
  uint8_t* s_out;
  int32_t* status;
};
cudaError_t launch_gather_rows(const GatherParams& P, int num_sms, cudaStream_t stream);

// Push combine: out[t] = sum_j w[t,j] * Y[pad_offsets[e] + inv[a] - offsets[e]], bf16.
// topk_w == nullptr: unit weights (the backward's reverse dispatch, dX = sum_j dXa).
struct CombineParams {
  const uint16_t* y;     // [R, d] scaled fp16 values (common.cuh)
  const uint8_t* ys;     // [R, d/32] their scale bytes
  const float* topk_w;
  const int32_t* topk_idx;
  const int32_t* inv;
  const int32_t* offsets;
  const int32_t* mtile_prefix;
  int prefix_shift;
  int64_t T;
  int d, E, k;
  uint16_t* out;
  int32_t* status;
  // direct_rows != 0: the row of assignment a = t*k + j is a itself (Y in assignment order,
  // as the expert-parallel push combine delivers it); topk_idx, inv, offsets and
  // mtile_prefix are then unused.
  int direct_rows;
};
cudaError_t launch_combine(const CombineParams& P, int num_sms, cudaStream_t stream);

// Token-direction quantiser for the weight gradients: a [R, C] operand in the padded
// expert-contiguous row order is quantised along its rows (tokens) in blocks of 32 inside
// each expert segment (rows past the segment's count read as zero) and stored transposed,
// [C, R] E4M3 with the UMMA scales of the [C, R] matrix.  Only columns [0, pad_offsets[E])
// of the output are written: no expert's K range reaches past them.
enum TransposeSrc : int {
  TSRC_MX = 0,       // MX codes [R, C] + UMMA scales (kgroups C/128): dequantised exactly
  TSRC_MX_W = 1,     // the same, each row times the combine weight of its assignment
};
struct TransposeQuantParams {
  int src;
  const uint8_t* q;            // [R, C] codes (read through tm_src: 128 x 128 box, no swizzle)
  const uint8_t* s;            // their UMMA scales
  const int32_t* perm;
  const int32_t* offsets;
  const float* topk_w;
  int k;
  const int32_t* pad_offsets;  // [E+1]
  const int32_t* counts;       // [E]
  int E;
  int64_t R;
  int C;
  uint8_t* dst_q;              // [C, R] (written through tm_dst: 128 x 128 box, 128B swizzle)
  uint8_t* dst_s;
  int32_t* status;
};
cudaError_t launch_transpose_quant(const CUtensorMap& tm_src, const CUtensorMap& tm_dst,
                                   const TransposeQuantParams& P, int num_sms,
                                   cudaStream_t stream);

// SwiGLU backward + d(router weights) per assignment row, from G = dout^ . Wd'^T.
struct SwigluBwdParams {
  const float* G;           // [R, f] fp32, padded expert order
  const uint16_t* gu;       // [R, 2f] saved bf16 g | u
  const uint8_t* h_q;       // [R, f] forward h codes + UMMA scales
  const uint8_t* h_s;
  const int32_t* perm;
  const int32_t* offsets;
  const int32_t* pad_offsets;
  const float* topk_w;
  int64_t A;
  int E, f;
  float* dw_route;          // [A]
  uint8_t* dgu_q;           // [R, 2f] MX codes of dg | du + UMMA scales
  uint8_t* dgu_s;
  // nullable: rows of full 128-row tiles were done by the GEMM epilogue (DGRAD_SWIGLU);
  // their d(combine weight) is the sum of these [R, f/128] partials, in block order
  const float* dw_part;
};
cudaError_t launch_swiglu_bwd(const SwigluBwdParams& P, int num_sms, cudaStream_t stream);

// Weight transpose for the BF16 variant: W [G][K][ncols] bf16 -> row rowmap(g, n) of a
// [*, K] bf16 matrix (map_mode as QuantColsParams: 0 plain, 1 gate/up interleave).
struct TransposeBf16Params {
  const uint16_t* src;
  int G, K, ncols;
  uint16_t* dst;
  int map_mode;
  int interleave_half;
};
cudaError_t launch_transpose_bf16(const TransposeBf16Params& P, cudaStream_t stream);

// Router backward: dlogits [T, E] (zero except the k selected experts of each token).
struct RouterBwdParams {
  const float* logits;     // [T, E]
  const int32_t* topk_idx; // [T, k]
  const float* dw_route;   // [T, k]
  int64_t T;
  int E, k, score_fn;
  float* dlogits;          // [T, E]
  int32_t* status;         // nullable
};
cudaError_t launch_router_bwd(const RouterBwdParams& P, int num_sms, cudaStream_t stream);

// Grouped block-scaled GEMM.
enum GemmMode : int {
  GEMM_GATEUP_SWIGLU = 1,  // SwiGLU + MX requant of h, optional bf16 g/u save
  GEMM_WGRAD_BF16 = 3,     // variable K per group (the group's token segment), bf16 out
  GEMM_STORE_F32_TMA = 4,  // D fp32 [rows, N] through shared memory + TMA stores (down
                           // projection, both dgrads, the generic entry point); writes whole
                           // 128-row tiles (rows past a group's count get unused values)
  // BF16 variant of the layer (kind::f16, bf16 operands, no scale factors; K counted in
  // bytes, 2 per element):
  GEMM_GATEUP_BF16 = 5,    // SwiGLU, h rounded to bf16 [rows, f]
  GEMM_STORE_F32_BF16 = 6, // as STORE_F32_TMA
  // the dgrad of the down projection with the SwiGLU backward in its epilogue: full
  // 128-row tiles turn G into [dg | du] (MX along f) and partial sums of <G, h^> without
  // storing G; an expert's last, partial tile stores G (fp32, as STORE_F32_TMA) for the
  // SwiGLU-backward kernel
  GEMM_DGRAD_SWIGLU = 7,
};

struct GemmParams {
  int G;
  int N;                 // output columns per group (multiple of 256)
  int K;                 // reduction length (multiple of 128); WGRAD: total K of A and B;
                         // the BF16 modes: in bytes (2 x elements)
  int M;                 // WGRAD: output rows per group (multiple of 128)
  int f;                 // GATEUP / DGRAD: expert intermediate size
  const int32_t* mtile_prefix;  // [G+1] (shifted right by prefix_shift when loaded)
  int prefix_shift;
  const int32_t* rows_valid;    // [G] nullable
  const uint8_t* sfa;    // UMMA scales of A
  const uint8_t* sfb;    // UMMA scales of B
  uint8_t* hq;           // GATEUP: [rows, f]
  uint8_t* hs;           // GATEUP: UMMA scales of [rows, f]
  uint16_t* gu;          // GATEUP: nullable [rows, 2f] bf16 save of g | u
  uint16_t* h16;         // GATEUP_BF16: [rows, f] bf16 h
  // STORE_F32 modes: nullable.  When given, D is stored as scaled fp16 (common.cuh) --
  // fp16 values through tmC0 (box 64 x 32, 128-byte swizzle; swapped tails through tmC1,
  // box 32 x 32, no swizzle) and one scale byte per 32 columns here, [rows, N/32].
  uint8_t* out_scales;
  // WGRAD: D[g] rows m < M, cols n < N -> (n < split ? out_a : out_b)[g][m][n mod split]
  uint16_t* out_a;
  uint16_t* out_b;
  int split;
  int32_t* status;
  // Tile scheduling.  Tiles are handed out in order by an atomic counter (zero before the
  // launch), so a CTA that starts late (its SM still busy with a concurrent kernel) takes
  // fewer tiles.  ready (nullable): count-down counters of valid rows still to be written
  // per minibatch of ready_rows padded rows (variable-M modes); a tile's A rows are loaded
  // once its minibatch's counter is zero.  order (nullable, WGRAD): the order in which the
  // groups' tiles are handed out (longest first).
  uint32_t* tile_ctr;
  const int32_t* ready;
  int ready_rows;
  const int32_t* order;
  // STORE_F32 modes: output columns n >= n_valid are not stored (0: all N).  Lets a group
  // width that is not a multiple of 256 (the router's E experts) run on whole N tiles of
  // a zero-padded B.
  int n_valid;
  // DGRAD_SWIGLU: the forward's saved g | u (gu), h codes and scales (hq, hs), the layout
  // (perm, offsets) and routing weights; outputs [dg | du] codes + UMMA scales and, per
  // row and 128-feature block, the partial sum of G * h^ ([rows, f/128] fp32).
  const int32_t* perm;
  const int32_t* offsets;
  const float* topk_w;
  uint8_t* dgu_q;
  uint8_t* dgu_s;
  float* dw_part;
};
// tmC0 / tmC1: output tensor maps of the TMA-store modes (STORE_F32_TMA: fp32 [rows, N],
// box 32 x 32; WGRAD: bf16 out_a / out_b, box 64 cols x 32 rows); ignored otherwise.
// pdl: launched as a programmatic dependent of the previous kernel in the stream, which
// must publish the rows this GEMM reads through P.ready.
cudaError_t launch_grouped_gemm(int mode, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const CUtensorMap& tmC0, const CUtensorMap& tmC1,
                                const GemmParams& P, int num_sms, cudaStream_t stream,
                                bool pdl = false);

// Scheduling tables, one CTA: ready[b] = valid rows of expert segments inside padded rows
// [b*ready_rows, (b+1)*ready_rows) for b < n_ready (count-down counters for a producer
// kernel to decrement); order (nullable) = experts sorted by descending count (ties: lower
// index first).
struct SchedInitParams {
  const int32_t* counts;
  const int32_t* pad_offsets;   // [E+1] (multiples of 128)
  int E;
  int32_t* ready;
  int n_ready;
  int ready_rows;
  int32_t* order;
};
cudaError_t launch_sched_init(const SchedInitParams& P, cudaStream_t stream);

// Expert parallelism: the owner rank's receive layout, pull dispatch and push of
// the expert outputs, over the peers' buffers (moe_ep_peer table in device memory).
struct EpParams {
  const moe_ep_peer* peers;  // [world]
  int world, rank, E_loc, k, d;
  int64_t R_cap;             // rows of the receive buffers (multiple of 128)
  int32_t* recv_counts;      // [E_loc]
  int32_t* recv_off;         // [E_loc+1] exclusive prefix (unpadded)
  int32_t* mtile;            // [E_loc+1] 128-row tile prefix of the padded segments
  int32_t* src_base;         // [world * E_loc]: first row of source s inside expert el
  int64_t* origin;           // [R_cap]: (source rank << 32) | assignment id, per padded row
  uint8_t* xq;               // [R_cap, d] received codes
  uint8_t* xs;               // UMMA scales of [R_cap, d]
  const uint16_t* y;         // [R_cap, d] expert outputs (scaled fp16) to push
  const uint8_t* ys;         // [R_cap, d/32]
  int32_t* status;
};
cudaError_t launch_ep_layout(const EpParams& P, cudaStream_t stream);
cudaError_t launch_ep_pull(const EpParams& P, int num_sms, cudaStream_t stream);
cudaError_t launch_ep_push(const EpParams& P, int num_sms, cudaStream_t stream);

// Router GEMM (logits = x . W_r^T) and its backward on the grouped GEMM engine (one group):
// the one-group tile lists and the zero-padded bf16 operand copies.
struct RouterSetupParams {
  int n;               // GEMMs (<= 3)
  int64_t rows[3];     // A rows of each GEMM
  int32_t* prefix;     // [2n]: {0, ceil(rows/128)} per GEMM
  int32_t* valid;      // [n]: rows per GEMM
  uint32_t* ctr;       // [n]: tile counters, zeroed
};
cudaError_t launch_router_setup(const RouterSetupParams& P, cudaStream_t stream);
// dst [dst_rows, dst_cols] bf16 = src[r][c] (r < R, c < C; src row pitch ld elements),
// zero elsewhere; fp32 sources are rounded to bf16 (nearest, ties to even).
cudaError_t launch_pad_copy_bf16(const uint16_t* src, int64_t R, int64_t C, int64_t ld,
                                 uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                 cudaStream_t stream);
cudaError_t launch_pad_copy_f32_bf16(const float* src, int64_t R, int64_t C, int64_t ld,
                                     uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                     cudaStream_t stream);
// dst [dst_rows >= C, dst_cols >= R] bf16 = transpose of src [R, C] (row pitch ld), zero
// outside; fp32 sources rounded to bf16 as above.
cudaError_t launch_transpose_pad_bf16(const uint16_t* src, int64_t R, int64_t C, int64_t ld,
                                      uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                      cudaStream_t stream);
cudaError_t launch_transpose_pad_f32_bf16(const float* src, int64_t R, int64_t C, int64_t ld,
                                          uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                          cudaStream_t stream);

}  // namespace moe
