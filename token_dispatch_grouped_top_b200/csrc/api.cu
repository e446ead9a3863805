// C ABI of the MoE layer (include/moe.h): argument checks, workspace carving, TMA
// descriptors and the launch sequence of each entry point.  Host code only.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/moe.h"
#include "kernels.h"

using namespace moe;

namespace moe {

// ---------------------------------------------------------------------------------------
// argument checks (pure host logic, no CUDA call)
// ---------------------------------------------------------------------------------------
moe_status check_dims(const moe_dims* D) {
  if (!D) return MOE_ERR_INVALID_ARG;
  if (D->T < 0 || D->d <= 0 || D->f <= 0 || D->E <= 0 || D->k <= 0) return MOE_ERR_INVALID_ARG;
  if (D->score_fn != MOE_SCORE_SOFTMAX_TOPK && D->score_fn != MOE_SCORE_SIGMOID_RENORM)
    return MOE_ERR_INVALID_ARG;
  if (D->E > 1024 || D->k > D->E || D->k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (D->d % 256 || D->f % 256) return MOE_ERR_UNSUPPORTED_SHAPE;
  // row indices of the padded expert-contiguous buffers (and their offsets) are int32
  if (D->T * D->k + static_cast<int64_t>(D->E) * 127 + 127 >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// ---------------------------------------------------------------------------------------
// device properties
// ---------------------------------------------------------------------------------------
moe_status device_sms(int* num_sms) {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_NO_DEVICE;
  if (dev < 64 && cache[dev] > 0) {
    *num_sms = cache[dev];
    return MOE_OK;
  }
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_NO_DEVICE;
  if (major != 10) return MOE_ERR_NO_DEVICE;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_NO_DEVICE;
  if (dev < 64) cache[dev] = sms;
  *num_sms = sms;
  return MOE_OK;
}

}  // namespace moe

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

constexpr int64_t kAlign = 256;
inline int64_t align_up(int64_t x, int64_t a = kAlign) { return (x + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D byte matrix [rows, cols] (cols contiguous), box [box_rows, 128 bytes], 128-byte swizzle.
moe_status make_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows,
                     bool swizzle = true) {
  auto fn = encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Output map for the TMA-store epilogues: [rows, cols] of fp32 or bf16, box of 128 bytes
// (32 fp32 or 64 bf16 columns) x 32 rows, 128-byte swizzle.
moe_status make_out_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols,
                         bool bf16) {
  auto fn = encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  const int64_t esz = bf16 ? 2 : 4;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * esz)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Output maps of a scaled-fp16 result [rows, cols]: box 64 columns x 32 rows with
// 128-byte swizzle (the regular tiles) and box 32 x 32 unswizzled (swapped last tiles).
moe_status make_f16s_tmaps(CUtensorMap* m64, CUtensorMap* m32, const void* base, int64_t rows,
                           int64_t cols) {
  auto fn = encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
  cuuint32_t estr[2] = {1u, 1u};
  cuuint32_t box64[2] = {64u, 32u};
  cuuint32_t box32[2] = {32u, 32u};
  CUresult r = fn(m64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box64, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return MOE_ERR_CUDA;
  r = fn(m32, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box32,
         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

inline moe_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ---------------------------------------------------------------------------------------
// optional per-stage timing: when enabled, every stage launch of moe_forward/moe_backward
// is bracketed by CUDA events on the launch stream; moe_profile_collect() sums them.
// ---------------------------------------------------------------------------------------
struct StageMark {
  int stage;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<StageMark> g_prof_marks;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct StageScope {
  int stage;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  StageScope(int s, cudaStream_t stream) : stage(s), st(stream) {
    std::lock_guard<std::mutex> g(g_prof_mu);
    if (!g_prof_on) return;
    a = prof_event();
    cudaEventRecord(a, st);
  }
  ~StageScope() {
    if (!a) return;
    std::lock_guard<std::mutex> g(g_prof_mu);
    cudaEvent_t b = prof_event();
    cudaEventRecord(b, st);
    g_prof_marks.push_back({stage, a, b});
  }
};
#define MOE_TRY(x)                     \
  do {                                 \
    moe_status _s = (x);               \
    if (_s != MOE_OK) return _s;       \
  } while (0)

// ---------------------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------------------
struct Carve {
  int64_t off = 0;
  int64_t take(int64_t bytes) {
    const int64_t o = off;
    off = align_up(off + bytes);
    return o;
  }
};

// Tile counters of the grouped GEMM launches, in the workspace header (zeroed per call).
constexpr int kFuseSwigluMinD = 6144;  // d from which the dgrad GEMM runs the SwiGLU backward
enum : int64_t { kCtrFwdGateUp = 72, kCtrFwdDown = 76, kCtrBwdDgradDown = 72,
                 kCtrBwdDgradGateUp = 76, kCtrBwdWgrad0 = 80, kCtrBwdWgrad1 = 84,
                 kCtrGeneric = 72 };

struct WsLayout {
  // header: [0] status word; [64] routing tile counter; [68] routing done counter;
  // [72, 96) grouped-GEMM tile counters
  int64_t zero_begin = 64, zero_bytes = 0;
  int64_t agg = 0, tstart = 0, rank = 0, mtile = 0, ready = 0, order = 0;
  int64_t idx = 0, w = 0, counts = 0, offsets = 0, perm = 0, inv = 0, pad = 0;
  int64_t xq = 0, xs = 0, hq = 0, hs = 0, y = 0, ys = 0;
  int64_t tq = 0, ts = 0;  // per-token MX copy of x (forward) or dout (backward)
  // backward
  int64_t dq = 0, ds = 0, dgu_q = 0, dgu_s = 0, dxa = 0, dxas = 0, gbuf = 0, dwpart = 0;
  int64_t xt_q = 0, xt_s = 0, ht_q = 0, ht_s = 0, gt_q = 0, gt_s = 0, yt_q = 0, yt_s = 0;
  int64_t total = 0;
};

int64_t padded_rows(const moe_dims* D) {
  const int64_t A = D->T * D->k;
  return align_up(A + static_cast<int64_t>(D->E) * 127, 128);
}

// Readiness minibatch of a token-row GEMM with n_cols output columns: the article's rule
// that a minibatch should fill at least two full waves of 128 x 256 tiles on the SMs
// (moe_min_tokens_for_waves), rounded up to whole 128-row tiles.
int ready_rows(int num_sms, int64_t n_cols) {
  const int64_t m = moe_min_tokens_for_waves(num_sms, 2, 128, 256, n_cols);
  return static_cast<int>(align_up(m > 0 ? m : 128, 128));
}

// Test hook (moe_debug_withhold_ready): a minibatch whose readiness is never published.
std::atomic<int> g_withhold{-1};

WsLayout ws_layout(const moe_dims* D, int op) {
  WsLayout L;
  const int64_t A = D->T * D->k, E = D->E, R = padded_rows(D);
  const int64_t nt = route_num_tiles(D->T);
  Carve c;
  c.take(128);  // status word + counters
  L.zero_bytes = 128 - L.zero_begin;
  L.agg = c.take(4 * nt * E);
  L.tstart = c.take(4 * nt * E);
  L.rank = c.take(4 * A);
  L.mtile = c.take(4 * (E + 1));
  L.ready = c.take(4 * (R / 128 + 1));
  L.order = c.take(4 * E);
  if (op >= MOE_OP_FORWARD) {
    L.tq = c.take(D->T * D->d);
    L.ts = c.take(D->T * (D->d / 32));
  }
  if (op == MOE_OP_FORWARD_BF16) {
    L.idx = c.take(4 * A);
    L.w = c.take(4 * A);
    L.counts = c.take(4 * E);
    L.offsets = c.take(4 * (E + 1));
    L.perm = c.take(4 * A);
    L.inv = c.take(4 * A);
    L.pad = c.take(4 * (E + 1));
    L.xq = c.take(2 * R * D->d);   // bf16 rows of x in padded expert order
    L.hq = c.take(2 * R * D->f);   // bf16 h
    L.y = c.take(2 * R * D->d);    // scaled fp16 expert outputs
    L.ys = c.take(R * (D->d / 32));
    L.total = c.off;
    return L;
  }
  if (op == MOE_OP_BACKWARD) {
    const int64_t d = D->d, f = D->f;
    L.dq = c.take(R * d);
    L.ds = c.take(moe_umma_scale_bytes(R, d));
    L.dgu_q = c.take(R * 2 * f);
    L.dgu_s = c.take(moe_umma_scale_bytes(R, 2 * f));
    L.dxa = c.take(2 * R * d);     // scaled fp16
    L.dxas = c.take(R * (d / 32));
    L.gbuf = c.take(4 * R * f);    // fp32: it feeds the MX requantisation of [dg|du]
    L.dwpart = c.take(4 * R * (f / 128));  // partial sums of <G, h^> per 128 features
    L.xt_q = c.take(d * R);
    L.xt_s = c.take(moe_umma_scale_bytes(d, R));
    L.ht_q = c.take(f * R);
    L.ht_s = c.take(moe_umma_scale_bytes(f, R));
    L.gt_q = c.take(2 * f * R);
    L.gt_s = c.take(moe_umma_scale_bytes(2 * f, R));
    L.yt_q = c.take(d * R);
    L.yt_s = c.take(moe_umma_scale_bytes(d, R));
    L.total = c.off;
    return L;
  }
  if (op >= MOE_OP_FORWARD) {
    L.idx = c.take(4 * A);
    L.w = c.take(4 * A);
    L.counts = c.take(4 * E);
    L.offsets = c.take(4 * (E + 1));
    L.perm = c.take(4 * A);
    L.inv = c.take(4 * A);
    L.pad = c.take(4 * (E + 1));
    L.xq = c.take(R * D->d);
    L.xs = c.take(moe_umma_scale_bytes(R, D->d));
    L.hq = c.take(R * D->f);
    L.hs = c.take(moe_umma_scale_bytes(R, D->f));
    L.y = c.take(2 * R * D->d);    // scaled fp16 expert outputs
    L.ys = c.take(R * (D->d / 32));
  }
  L.total = c.off;
  return L;
}

template <class T>
inline T* at(void* ws, int64_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// Workspace of the router GEMM calls (MOE_OP_ROUTER): a 256-byte header (status word at 0,
// three tile counters at 64, the one-group tile prefixes at 128 and valid rows at 160),
// then the zero-padded bf16 operand copies:
//   wr_pad [NE, d]     W_r with its rows padded to whole 256-row N tiles (forward B)
//   dlog   [Tp128, Ep] bf16(G), rows to whole 128-row tiles, K (experts) to 64   (dx A)
//   dlogT  [Ep128, Tp] bf16(G)^T, rows (experts) to 128, K (tokens) to 64        (dW A)
//   wrT    [d, Ep]     W_r^T, K (experts) padded to 64                           (dx B)
//   xT     [d, Tp]     x^T, K (tokens) padded to 64                              (dW B)
struct RouterWsLayout {
  int64_t NE, Ep, Tp, Tp128, Ep128;
  int64_t wr_pad, dlog, dlogT, wrT, xT, total;
};
constexpr int64_t kRouterCtr = 64, kRouterPrefix = 128, kRouterValid = 160;

RouterWsLayout router_ws_layout(const moe_dims* D) {
  auto up = [](int64_t v, int64_t m) { return (v + m - 1) / m * m; };
  RouterWsLayout L;
  const int64_t T = std::max<int64_t>(D->T, 1), E = D->E, d = D->d;
  L.NE = up(E, 256);
  L.Ep = up(E, 64);
  L.Tp = up(T, 64);
  L.Tp128 = up(T, 128);
  L.Ep128 = up(E, 128);
  int64_t off = 256;
  auto take = [&](int64_t bytes) {
    const int64_t o = off;
    off += up(bytes, 256);
    return o;
  };
  L.wr_pad = take(L.NE * d * 2);
  L.dlog = take(L.Tp128 * L.Ep * 2);
  L.dlogT = take(L.Ep128 * L.Tp * 2);
  L.wrT = take(d * L.Ep * 2);
  L.xT = take(d * L.Tp * 2);
  L.total = off;
  return L;
}

// Workspace of moe_ep_experts on one rank: a 256-byte header (status at 0, tile counters at
// 72 and 76), the receive layout, then the receive buffers for the worst case of
// R_cap = sum_s T_s * min(k, E_loc) rows plus each segment's tile padding:
//   recv_counts [E_loc], recv_off [E_loc+1], mtile [E_loc+1], src_base [world*E_loc] int32
//   origin [R_cap] int64, xq [R_cap,d] + UMMA scales, hq [R_cap,f] + UMMA scales,
//   y [R_cap,d] scaled fp16 + [R_cap,d/32] scale bytes
struct EpWsLayout {
  int64_t E_loc, R_cap;
  int64_t recv_counts, recv_off, mtile, src_base, origin, xq, xs, hq, hs, y, ys, total;
};

bool ep_ws_layout(const moe_dims* D, int32_t world, EpWsLayout* out) {
  if (check_dims(D) != MOE_OK || world < 1 || world > 64 || D->E % world) return false;
  auto up = [](int64_t v, int64_t m) { return (v + m - 1) / m * m; };
  EpWsLayout L;
  L.E_loc = D->E / world;
  const int64_t per_tok = std::min<int64_t>(D->k, L.E_loc);
  L.R_cap = std::max<int64_t>(up(D->T * per_tok + L.E_loc * 127, 128), 128);
  if (L.R_cap >= (int64_t(1) << 31)) return false;  // row indices are int32
  const int64_t d = D->d, f = D->f;
  int64_t off = 256;
  auto take = [&](int64_t bytes) {
    const int64_t o = off;
    off += up(bytes, 256);
    return o;
  };
  L.recv_counts = take(4 * L.E_loc);
  L.recv_off = take(4 * (L.E_loc + 1));
  L.mtile = take(4 * (L.E_loc + 1));
  L.src_base = take(4 * static_cast<int64_t>(world) * L.E_loc);
  L.origin = take(8 * L.R_cap);
  L.xq = take(L.R_cap * d);
  L.xs = take(L.R_cap * d / 32);
  L.hq = take(L.R_cap * f);
  L.hs = take(L.R_cap * f / 32);
  L.y = take(2 * L.R_cap * d);
  L.ys = take(L.R_cap * d / 32);
  L.total = off;
  *out = L;
  return true;
}

moe_status router_checks(const moe_dims* D, const void* const* ptrs, int n, void* ws,
                         size_t ws_bytes) {
  MOE_TRY(check_dims(D));
  if (D->E % 8) return MOE_ERR_UNSUPPORTED_SHAPE;  // row pitches of [*, E] in 16-byte units
  if (!ws) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (!ptrs[i]) return MOE_ERR_INVALID_ARG;
    if (!aligned16(ptrs[i])) return MOE_ERR_MISALIGNED;
  }
  if (!aligned256(ws)) return MOE_ERR_MISALIGNED;
  if (ws_bytes < static_cast<size_t>(router_ws_layout(D).total))
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

moe_status run_route(const moe_dims* D, const float* logits, int32_t* idx, float* w,
                     int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* pad,
                     void* ws, const WsLayout& L, int num_sms, cudaStream_t st) {
  const int nt = route_num_tiles(D->T);
  MOE_TRY(cuda_ok(cudaMemsetAsync(at<uint8_t>(ws, L.zero_begin), 0, L.zero_bytes, st)));
  RouteParams P;
  P.logits = logits;
  P.T = D->T;
  P.E = D->E;
  P.k = D->k;
  P.score_fn = D->score_fn;
  P.num_tiles = nt;
  P.topk_idx = idx;
  P.topk_w = w;
  P.rank = at<int32_t>(ws, L.rank);
  P.counts = counts;
  P.offsets = offsets;
  P.mtile_prefix = at<int32_t>(ws, L.mtile);
  P.pad_offsets = pad;
  P.tile_counter = at<uint32_t>(ws, 64);
  P.done_counter = at<uint32_t>(ws, 68);
  P.agg = at<int32_t>(ws, L.agg);
  P.tile_start = at<int32_t>(ws, L.tstart);
  P.status = at<int32_t>(ws, 0);
  return cuda_ok(launch_route_layout(P, perm, inv, num_sms, st));
}

// Routing outputs for an empty batch: all counts and offsets are zero.
moe_status route_empty(const moe_dims* D, int32_t* counts, int32_t* offsets, int32_t* mtile,
                       int32_t* pad, cudaStream_t st) {
  MOE_TRY(cuda_ok(cudaMemsetAsync(counts, 0, 4 * D->E, st)));
  MOE_TRY(cuda_ok(cudaMemsetAsync(offsets, 0, 4 * (D->E + 1), st)));
  if (mtile) MOE_TRY(cuda_ok(cudaMemsetAsync(mtile, 0, 4 * (D->E + 1), st)));
  if (pad) MOE_TRY(cuda_ok(cudaMemsetAsync(pad, 0, 4 * (D->E + 1), st)));
  return MOE_OK;
}

// Pull dispatch: quantise every token row once (MXFP8 along d, canonical scales), then
// each expert row pulls its token's codes and scales by index into the padded layout.
moe_status dispatch_pull(const moe_dims* D, const uint16_t* src, const int32_t* offsets,
                         const int32_t* prefix, int prefix_shift, const int32_t* perm,
                         uint8_t* tok_q, uint8_t* tok_s, uint8_t* out_q, uint8_t* out_s,
                         int32_t* status, int sms, cudaStream_t st, int32_t* ready = nullptr,
                         int ready_rows_ = 0) {
  QuantRowsParams Q;
  Q.src = src;
  Q.src_ld = D->d;
  Q.rows = D->T;
  Q.K = D->d;
  Q.dst = tok_q;
  Q.dst_ld = D->d;
  Q.dst_col0 = 0;
  Q.scales = tok_s;
  Q.layout = 0;
  Q.kgroups = D->d / 128;
  MOE_TRY(cuda_ok(launch_quant_rows(Q, sms, st)));
  GatherParams G;
  G.ready = ready;
  G.ready_rows = ready_rows_;
  G.withhold = g_withhold.load();
  G.row_bytes = D->d;
  G.q_tok = tok_q;
  G.s_tok = tok_s;
  G.T = D->T;
  G.d = D->d;
  G.E = D->E;
  G.k = D->k;
  G.offsets = offsets;
  G.mtile_prefix = prefix;
  G.prefix_shift = prefix_shift;
  G.perm = perm;
  G.q_out = out_q;
  G.s_out = out_s;
  G.status = status;
  return cuda_ok(launch_gather_rows(G, sms, st));
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_MISALIGNED: return "misaligned pointer";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "device-side index out of bounds";
    case MOE_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

int64_t moe_padded_rows(const moe_dims* dims) {
  if (check_dims(dims) != MOE_OK) return -1;
  return padded_rows(dims);
}

int64_t moe_umma_scale_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 128) return -1;
  return align_up(rows, 128) * (K / 32);
}

int64_t moe_weights_bytes(const moe_dims* D, int32_t field) {
  if (check_dims(D) != MOE_OK) return -1;
  const int64_t E = D->E, d = D->d, f = D->f;
  switch (field) {
    case 0: return E * 2 * f * d;
    case 1: return moe_umma_scale_bytes(E * 2 * f, d);
    case 2: return E * d * f;
    case 3: return moe_umma_scale_bytes(E * d, f);
    case 4: return E * f * d;
    case 5: return moe_umma_scale_bytes(E * f, d);
    case 6: return E * d * 2 * f;
    case 7: return moe_umma_scale_bytes(E * d, 2 * f);
    default: return -1;
  }
}

int64_t moe_saved_bytes(const moe_dims* D, int32_t field) {
  if (check_dims(D) != MOE_OK) return -1;
  const int64_t A = D->T * D->k, E = D->E, R = padded_rows(D);
  switch (field) {
    case 0: case 1: case 4: case 5: return 4 * A;
    case 2: return 4 * E;
    case 3: case 6: return 4 * (E + 1);
    case 7: return R * D->d;
    case 8: return moe_umma_scale_bytes(R, D->d);
    case 9: return R * D->f;
    case 10: return moe_umma_scale_bytes(R, D->f);
    case 11: return R * 2 * D->f * 2;
    default: return -1;
  }
}

size_t moe_workspace_bytes(const moe_dims* dims, int32_t op) {
  if (check_dims(dims) != MOE_OK || op < MOE_OP_ROUTE || op > MOE_OP_ROUTER) return 0;
  if (op == MOE_OP_ROUTER) return static_cast<size_t>(router_ws_layout(dims).total);
  return static_cast<size_t>(ws_layout(dims, op).total);
}

int64_t moe_workspace_offset(const moe_dims* D, int32_t op, int32_t buffer) {
  if (check_dims(D) != MOE_OK || op < MOE_OP_ROUTE || op > MOE_OP_FORWARD_BF16) return -1;
  const WsLayout L = ws_layout(D, op);
  if (buffer == MOE_WS_MTILE) return L.mtile;
  if ((op == MOE_OP_FORWARD || op == MOE_OP_FORWARD_BF16) && buffer == MOE_WS_Y) return L.y;
  if ((op == MOE_OP_FORWARD || op == MOE_OP_FORWARD_BF16) && buffer == MOE_WS_Y_S) return L.ys;
  if ((op == MOE_OP_FORWARD || op == MOE_OP_FORWARD_BF16) && buffer == MOE_WS_COUNTS)
    return L.counts;
  if (op != MOE_OP_BACKWARD) return -1;
  switch (buffer) {
    case MOE_WS_DOUT_Q: return L.dq;
    case MOE_WS_DOUT_S: return L.ds;
    case MOE_WS_G: return L.gbuf;
    case MOE_WS_DXA_S: return L.dxas;
    case MOE_WS_DGU_Q: return L.dgu_q;
    case MOE_WS_DGU_S: return L.dgu_s;
    case MOE_WS_DXA: return L.dxa;
    case MOE_WS_XT_Q: return L.xt_q;
    case MOE_WS_XT_S: return L.xt_s;
    case MOE_WS_HT_Q: return L.ht_q;
    case MOE_WS_HT_S: return L.ht_s;
    case MOE_WS_GT_Q: return L.gt_q;
    case MOE_WS_GT_S: return L.gt_s;
    case MOE_WS_YT_Q: return L.yt_q;
    case MOE_WS_YT_S: return L.yt_s;
    default: return -1;
  }
}

int64_t moe_min_tokens_for_waves(int32_t num_sms, int32_t waves, int32_t tile_m, int32_t tile_n,
                                 int64_t n_cols) {
  if (num_sms <= 0 || waves <= 0 || tile_m <= 0 || tile_n <= 0 || n_cols <= 0) return -1;
  // tokens * (n_cols / tile_n) / tile_m tiles >= waves * num_sms
  const int64_t num = static_cast<int64_t>(waves) * num_sms * tile_m * tile_n;
  return (num + n_cols - 1) / n_cols;
}

moe_status moe_route_layout(const moe_dims* D, const float* logits, int32_t* topk_idx,
                            float* topk_w, int32_t* counts, int32_t* offsets, int32_t* perm,
                            int32_t* inv_perm, int32_t* pad_offsets, void* ws, size_t ws_bytes,
                            void* stream) {
  MOE_TRY(check_dims(D));
  if (!ws || !counts || !offsets || (D->T > 0 && (!logits || !topk_idx || !topk_w || !perm ||
                                                  !inv_perm)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned256(ws)) return MOE_ERR_MISALIGNED;
  {
    const void* ptrs[] = {logits, topk_idx, topk_w, counts, offsets, perm, inv_perm, pad_offsets};
    for (const void* p : ptrs)
      if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  const WsLayout L = ws_layout(D, MOE_OP_ROUTE);
  if (ws_bytes < static_cast<size_t>(L.total)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D->T == 0) return route_empty(D, counts, offsets, at<int32_t>(ws, L.mtile), pad_offsets, st);
  return run_route(D, logits, topk_idx, topk_w, counts, offsets, perm, inv_perm, pad_offsets, ws,
                   L, sms, st);
}

moe_status mxfp8_quantize(const uint16_t* in, int64_t rows, int64_t K, int64_t ld, uint8_t* q,
                          uint8_t* scales, int32_t scale_layout, void* stream) {
  if (rows < 0 || K <= 0 || ld < K || (scale_layout != 0 && scale_layout != 1))
    return MOE_ERR_INVALID_ARG;
  if (K % 32 || (scale_layout == 1 && K % 128) || ld % 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!in || !q || !scales) return MOE_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(q) || !aligned16(scales)) return MOE_ERR_MISALIGNED;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  QuantRowsParams P;
  P.src = in;
  P.src_ld = ld;
  P.rows = rows;
  P.K = K;
  P.dst = q;
  P.dst_ld = K;
  P.dst_col0 = 0;
  P.scales = scales;
  P.layout = scale_layout;
  P.kgroups = K / 128;
  return cuda_ok(launch_quant_rows(P, sms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_prepare_weights(const moe_dims* D, const uint16_t* wg, const uint16_t* wu,
                               const uint16_t* wd, int32_t with_bwd, const moe_weights* out,
                               void* stream) {
  MOE_TRY(check_dims(D));
  if (!wg || !wu || !wd || !out || !out->wgu_q || !out->wgu_s || !out->wd_q || !out->wd_s)
    return MOE_ERR_INVALID_ARG;
  if (with_bwd && (!out->wdT_q || !out->wdT_s || !out->wguT_q || !out->wguT_s))
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {wg, wu, wd, out->wgu_q, out->wgu_s, out->wd_q, out->wd_s};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int E = D->E, d = D->d, f = D->f;
  // gate / up: column n of W[e] ([d, f]) along d -> interleaved rows of the [E*2f, d] matrix
  for (int half = 0; half < 2; ++half) {
    QuantColsParams P;
    P.src = half == 0 ? wg : wu;
    P.G = E;
    P.K = d;
    P.ncols = f;
    P.dst = out->wgu_q;
    P.scales = out->wgu_s;
    P.kgroups = d / 128;
    P.map_mode = 1;
    P.interleave_half = half;
    MOE_TRY(cuda_ok(launch_quant_cols(P, st)));
  }
  {  // down: column n of W_down[e] ([f, d]) along f -> row e*d + n of the [E*d, f] matrix
    QuantColsParams P;
    P.src = wd;
    P.G = E;
    P.K = f;
    P.ncols = d;
    P.dst = out->wd_q;
    P.scales = out->wd_s;
    P.kgroups = f / 128;
    P.map_mode = 0;
    P.interleave_half = 0;
    MOE_TRY(cuda_ok(launch_quant_cols(P, st)));
  }
  if (with_bwd) {
    // W_down as stored: rows [E*f] along d
    QuantRowsParams P;
    P.src = wd;
    P.src_ld = d;
    P.rows = static_cast<int64_t>(E) * f;
    P.K = d;
    P.dst = out->wdT_q;
    P.dst_ld = d;
    P.dst_col0 = 0;
    P.scales = out->wdT_s;
    P.layout = 1;
    P.kgroups = d / 128;
    MOE_TRY(cuda_ok(launch_quant_rows(P, sms, st)));
    // [W_gate | W_up] rows [E*d] along 2f
    for (int half = 0; half < 2; ++half) {
      QuantRowsParams Q;
      Q.src = half == 0 ? wg : wu;
      Q.src_ld = f;
      Q.rows = static_cast<int64_t>(E) * d;
      Q.K = f;
      Q.dst = out->wguT_q;
      Q.dst_ld = 2 * f;
      Q.dst_col0 = half * f;
      Q.scales = out->wguT_s;
      Q.layout = 1;
      Q.kgroups = 2 * f / 128;
      MOE_TRY(cuda_ok(launch_quant_rows(Q, sms, st)));
    }
  }
  return MOE_OK;
}

moe_status moe_grouped_gemm_mx(int32_t G, int64_t rows_a, int32_t N, int32_t K,
                               const int32_t* mtile_prefix, const int32_t* rows_valid,
                               const uint8_t* a_q, const uint8_t* a_s, const uint8_t* b_q,
                               const uint8_t* b_s, float* d_out, void* ws, size_t ws_bytes,
                               void* stream) {
  if (G <= 0 || G > 1024 || rows_a < 0 || N <= 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (N % 256 || K % 128 || rows_a % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!mtile_prefix || !a_q || !a_s || !b_q || !b_s || !d_out || !ws) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < 256) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const void* ptrs[] = {a_q, a_s, b_q, b_s, d_out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  if (!aligned256(ws)) return MOE_ERR_MISALIGNED;
  if (rows_a == 0) return MOE_OK;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  CUtensorMap ta, tb;
  MOE_TRY(make_tmap(&ta, a_q, rows_a, K, 128));
  MOE_TRY(make_tmap(&tb, b_q, static_cast<int64_t>(G) * N, K, 256));
  GemmParams P = {};
  P.G = G;
  P.N = N;
  P.K = K;
  P.mtile_prefix = mtile_prefix;
  P.rows_valid = rows_valid;
  P.sfa = a_s;
  P.sfb = b_s;
  P.status = at<int32_t>(ws, 0);
  P.tile_ctr = at<uint32_t>(ws, kCtrGeneric);
  MOE_TRY(cuda_ok(cudaMemsetAsync(P.tile_ctr, 0, 4, static_cast<cudaStream_t>(stream))));
  CUtensorMap tc;
  MOE_TRY(make_out_tmap(&tc, d_out, rows_a, N, false));
  return cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_TMA, ta, tb, tc, tc, P, sms,
                                     static_cast<cudaStream_t>(stream)));
}

moe_status moe_grouped_gemm_bf16(int32_t G, int64_t rows_a, int32_t N, int32_t K,
                                 const int32_t* mtile_prefix, const int32_t* rows_valid,
                                 const uint16_t* a, const uint16_t* b, float* d_out, void* ws,
                                 size_t ws_bytes, void* stream) {
  if (G <= 0 || G > 1024 || rows_a < 0 || N <= 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (N % 256 || K % 64 || rows_a % 128) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!mtile_prefix || !a || !b || !d_out || !ws) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < 256) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const void* ptrs[] = {a, b, d_out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  if (!aligned256(ws)) return MOE_ERR_MISALIGNED;
  if (rows_a == 0) return MOE_OK;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap ta, tb, tc;
  MOE_TRY(make_tmap(&ta, a, rows_a, 2 * static_cast<int64_t>(K), 128));
  MOE_TRY(make_tmap(&tb, b, static_cast<int64_t>(G) * N, 2 * static_cast<int64_t>(K), 256));
  MOE_TRY(make_out_tmap(&tc, d_out, rows_a, N, false));
  GemmParams P = {};
  P.G = G;
  P.N = N;
  P.K = 2 * K;
  P.mtile_prefix = mtile_prefix;
  P.rows_valid = rows_valid;
  P.status = at<int32_t>(ws, 0);
  P.tile_ctr = at<uint32_t>(ws, kCtrGeneric);
  MOE_TRY(cuda_ok(cudaMemsetAsync(P.tile_ctr, 0, 4, st)));
  return cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_BF16, ta, tb, tc, tc, P, sms, st));
}

moe_status moe_prepare_weights_bf16(const moe_dims* D, const uint16_t* wg, const uint16_t* wu,
                                    const uint16_t* wd, uint16_t* wgu_t, uint16_t* wd_t,
                                    void* stream) {
  MOE_TRY(check_dims(D));
  if (!wg || !wu || !wd || !wgu_t || !wd_t) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {wg, wu, wd, wgu_t, wd_t};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int half = 0; half < 2; ++half) {  // gate / up: column n of W[e] -> interleaved row
    TransposeBf16Params P;
    P.src = half == 0 ? wg : wu;
    P.G = D->E;
    P.K = D->d;
    P.ncols = D->f;
    P.dst = wgu_t;
    P.map_mode = 1;
    P.interleave_half = half;
    MOE_TRY(cuda_ok(launch_transpose_bf16(P, st)));
  }
  TransposeBf16Params P;  // down: column n of W_down[e] -> row e*d + n
  P.src = wd;
  P.G = D->E;
  P.K = D->f;
  P.ncols = D->d;
  P.dst = wd_t;
  P.map_mode = 0;
  P.interleave_half = 0;
  return cuda_ok(launch_transpose_bf16(P, st));
}

moe_status moe_forward_bf16(const moe_dims* D, const uint16_t* wgu_t, const uint16_t* wd_t,
                            const uint16_t* x, const float* logits, uint16_t* out, void* ws,
                            size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(D));
  if (!wgu_t || !wd_t || !ws || (D->T > 0 && (!x || !logits || !out)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned256(ws)) return MOE_ERR_MISALIGNED;
  {
    const void* ptrs[] = {wgu_t, wd_t, x, logits, out};
    for (const void* p : ptrs)
      if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  const WsLayout L = ws_layout(D, MOE_OP_FORWARD_BF16);
  if (ws_bytes < static_cast<size_t>(L.total)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* w = at<float>(ws, L.w);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  int32_t* pad = at<int32_t>(ws, L.pad);
  int32_t* mtile = at<int32_t>(ws, L.mtile);
  uint16_t* xp = at<uint16_t>(ws, L.xq);
  uint16_t* h16 = at<uint16_t>(ws, L.hq);
  uint16_t* y = at<uint16_t>(ws, L.y);
  uint8_t* ys = at<uint8_t>(ws, L.ys);
  int32_t* status = at<int32_t>(ws, 0);
  if (D->T == 0) return route_empty(D, counts, offsets, mtile, pad, st);
  {
    StageScope sc(MOE_STAGE_ROUTE, st);
    MOE_TRY(run_route(D, logits, idx, w, counts, offsets, perm, inv, pad, ws, L, sms, st));
  }
  const int64_t R = padded_rows(D);
  const int mb = ready_rows(sms, 2 * static_cast<int64_t>(D->f));
  int32_t* ready = at<int32_t>(ws, L.ready);
  {  // pull dispatch of the bf16 rows, published minibatch by minibatch
    StageScope sc(MOE_STAGE_PERMUTE, st);
    SchedInitParams SI;
    SI.counts = counts;
    SI.pad_offsets = pad;
    SI.E = D->E;
    SI.ready = ready;
    SI.ready_rows = mb;
    SI.n_ready = static_cast<int>((R + mb - 1) / mb);
    SI.order = nullptr;
    MOE_TRY(cuda_ok(launch_sched_init(SI, st)));
    GatherParams G;
    G.ready = ready;
    G.ready_rows = mb;
    G.withhold = g_withhold.load();
      G.row_bytes = 2 * static_cast<int64_t>(D->d);
    G.q_tok = reinterpret_cast<const uint8_t*>(x);
    G.s_tok = nullptr;
    G.T = D->T;
    G.d = D->d;
    G.E = D->E;
    G.k = D->k;
    G.offsets = offsets;
    G.mtile_prefix = mtile;
    G.prefix_shift = 0;
    G.perm = perm;
    G.q_out = reinterpret_cast<uint8_t*>(xp);
    G.s_out = nullptr;
    G.status = status;
    MOE_TRY(cuda_ok(launch_gather_rows(G, sms, st)));
  }
  {
    StageScope sc(MOE_STAGE_GATEUP, st);
    CUtensorMap ta, tb;
    MOE_TRY(make_tmap(&ta, xp, R, 2 * static_cast<int64_t>(D->d), 128));
    MOE_TRY(make_tmap(&tb, wgu_t, static_cast<int64_t>(D->E) * 2 * D->f,
                      2 * static_cast<int64_t>(D->d), 256));
    GemmParams P = {};
    P.G = D->E;
    P.N = 2 * D->f;
    P.K = 2 * D->d;
    P.f = D->f;
    P.mtile_prefix = mtile;
    P.rows_valid = counts;
    P.h16 = h16;
    P.status = status;
    P.tile_ctr = at<uint32_t>(ws, kCtrFwdGateUp);
    P.ready = ready;
    P.ready_rows = mb;
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_GATEUP_BF16, ta, tb, ta, tb, P, sms, st, true)));
  }
  {
    StageScope sc(MOE_STAGE_DOWN, st);
    CUtensorMap ta, tb, ty;
    MOE_TRY(make_tmap(&ta, h16, R, 2 * static_cast<int64_t>(D->f), 128));
    MOE_TRY(make_tmap(&tb, wd_t, static_cast<int64_t>(D->E) * D->d,
                      2 * static_cast<int64_t>(D->f), 256));
    CUtensorMap ty32;
    MOE_TRY(make_f16s_tmaps(&ty, &ty32, y, R, D->d));
    GemmParams P = {};
    P.G = D->E;
    P.N = D->d;
    P.K = 2 * D->f;
    P.mtile_prefix = mtile;
    P.rows_valid = counts;
    P.status = status;
    P.tile_ctr = at<uint32_t>(ws, kCtrFwdDown);
    P.out_scales = ys;
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_BF16, ta, tb, ty, ty32, P, sms, st)));
  }
  {
    StageScope sc(MOE_STAGE_COMBINE, st);
    CombineParams P = {};
    P.y = y;
    P.ys = ys;
    P.topk_w = w;
    P.topk_idx = idx;
    P.inv = inv;
    P.offsets = offsets;
    P.mtile_prefix = mtile;
    P.prefix_shift = 0;
    P.T = D->T;
    P.d = D->d;
    P.E = D->E;
    P.k = D->k;
    P.out = out;
    P.status = status;
    MOE_TRY(cuda_ok(launch_combine(P, sms, st)));
  }
  return MOE_OK;
}

moe_status moe_forward(const moe_dims* D, const moe_weights* W, const uint16_t* x,
                       const float* logits, uint16_t* out, const moe_saved* saved, void* ws,
                       size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(D));
  if (!W || !ws || (D->T > 0 && (!x || !logits || !out))) return MOE_ERR_INVALID_ARG;
  if (!W->wgu_q || !W->wgu_s || !W->wd_q || !W->wd_s) return MOE_ERR_INVALID_ARG;
  // the token-sized arrays (T*k entries) may be null when there are no tokens
  if (saved && ((D->T > 0 && (!saved->topk_idx || !saved->topk_w || !saved->perm ||
                              !saved->inv_perm)) ||
                !saved->counts || !saved->offsets || !saved->pad_offsets || !saved->xq ||
                !saved->xs || !saved->hq || !saved->hs || !saved->gu))
    return MOE_ERR_INVALID_ARG;
  if (!aligned256(ws)) return MOE_ERR_MISALIGNED;
  {
    const void* ptrs[] = {x, logits, out, W->wgu_q, W->wgu_s, W->wd_q, W->wd_s};
    for (const void* p : ptrs)
      if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
    if (saved) {
      const void* sp[] = {saved->xq, saved->xs, saved->hq, saved->hs, saved->gu};
      for (const void* p : sp)
        if (!aligned16(p)) return MOE_ERR_MISALIGNED;
    }
  }
  const WsLayout L = ws_layout(D, MOE_OP_FORWARD);
  if (ws_bytes < static_cast<size_t>(L.total)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  int32_t* idx = saved ? saved->topk_idx : at<int32_t>(ws, L.idx);
  float* w = saved ? saved->topk_w : at<float>(ws, L.w);
  int32_t* counts = saved ? saved->counts : at<int32_t>(ws, L.counts);
  int32_t* offsets = saved ? saved->offsets : at<int32_t>(ws, L.offsets);
  int32_t* perm = saved ? saved->perm : at<int32_t>(ws, L.perm);
  int32_t* inv = saved ? saved->inv_perm : at<int32_t>(ws, L.inv);
  int32_t* pad = saved ? saved->pad_offsets : at<int32_t>(ws, L.pad);
  uint8_t* xq = saved ? saved->xq : at<uint8_t>(ws, L.xq);
  uint8_t* xs = saved ? saved->xs : at<uint8_t>(ws, L.xs);
  uint8_t* hq = saved ? saved->hq : at<uint8_t>(ws, L.hq);
  uint8_t* hs = saved ? saved->hs : at<uint8_t>(ws, L.hs);
  uint16_t* gu = saved ? saved->gu : nullptr;
  int32_t* mtile = at<int32_t>(ws, L.mtile);
  uint16_t* y = at<uint16_t>(ws, L.y);
  uint8_t* ys = at<uint8_t>(ws, L.ys);
  int32_t* status = at<int32_t>(ws, 0);

  if (D->T == 0) return route_empty(D, counts, offsets, mtile, pad, st);
  {
    StageScope sc(MOE_STAGE_ROUTE, st);
    MOE_TRY(run_route(D, logits, idx, w, counts, offsets, perm, inv, pad, ws, L, sms, st));
  }

  const int64_t R = padded_rows(D);
  const int mb = ready_rows(sms, 2 * static_cast<int64_t>(D->f));
  int32_t* ready = at<int32_t>(ws, L.ready);
  {
    StageScope sc(MOE_STAGE_PERMUTE, st);
    SchedInitParams SI;
    SI.counts = counts;
    SI.pad_offsets = pad;
    SI.E = D->E;
    SI.ready = ready;
    SI.ready_rows = mb;
    SI.n_ready = static_cast<int>((R + mb - 1) / mb);
    SI.order = nullptr;
    MOE_TRY(cuda_ok(launch_sched_init(SI, st)));
    MOE_TRY(dispatch_pull(D, x, offsets, mtile, 0, perm, at<uint8_t>(ws, L.tq),
                          at<uint8_t>(ws, L.ts), xq, xs, status, sms, st, ready, mb));
  }
  {
    StageScope sc(MOE_STAGE_GATEUP, st);
    CUtensorMap ta, tb;
    MOE_TRY(make_tmap(&ta, xq, R, D->d, 128));
    MOE_TRY(make_tmap(&tb, W->wgu_q, static_cast<int64_t>(D->E) * 2 * D->f, D->d, 256));
    GemmParams P = {};
    P.G = D->E;
    P.N = 2 * D->f;
    P.K = D->d;
    P.f = D->f;
    P.mtile_prefix = mtile;
    P.rows_valid = counts;
    P.sfa = xs;
    P.sfb = W->wgu_s;
    P.hq = hq;
    P.hs = hs;
    P.gu = gu;
    P.status = status;
    P.tile_ctr = at<uint32_t>(ws, kCtrFwdGateUp);
    P.ready = ready;
    P.ready_rows = mb;
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_GATEUP_SWIGLU, ta, tb, ta, tb, P, sms, st, true)));
  }
  {
    StageScope sc(MOE_STAGE_DOWN, st);
    CUtensorMap ta, tb;
    MOE_TRY(make_tmap(&ta, hq, R, D->f, 128));
    MOE_TRY(make_tmap(&tb, W->wd_q, static_cast<int64_t>(D->E) * D->d, D->f, 256));
    GemmParams P = {};
    P.G = D->E;
    P.N = D->d;
    P.K = D->f;
    P.mtile_prefix = mtile;
    P.rows_valid = counts;
    P.sfa = hs;
    P.sfb = W->wd_s;
    P.status = status;
    P.tile_ctr = at<uint32_t>(ws, kCtrFwdDown);
    P.out_scales = ys;
    CUtensorMap ty, ty32;
    MOE_TRY(make_f16s_tmaps(&ty, &ty32, y, R, D->d));
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_TMA, ta, tb, ty, ty32, P, sms, st)));
  }
  {
    StageScope sc(MOE_STAGE_COMBINE, st);
    CombineParams P = {};
    P.y = y;
    P.ys = ys;
    P.topk_w = w;
    P.topk_idx = idx;
    P.inv = inv;
    P.offsets = offsets;
    P.mtile_prefix = mtile;
    P.prefix_shift = 0;
    P.T = D->T;
    P.d = D->d;
    P.E = D->E;
    P.k = D->k;
    P.out = out;
    P.status = status;
    MOE_TRY(cuda_ok(launch_combine(P, sms, st)));
  }
  return MOE_OK;
}

moe_status moe_backward(const moe_dims* D, const moe_weights* W, const moe_saved* S,
                        const uint16_t* dout, uint16_t* dx, float* dw_route, uint16_t* dWg,
                        uint16_t* dWu, uint16_t* dWd, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(D));
  if (!W || !S || !ws || !dWg || !dWu || !dWd) return MOE_ERR_INVALID_ARG;
  if (!W->wdT_q || !W->wdT_s || !W->wguT_q || !W->wguT_s) return MOE_ERR_INVALID_ARG;
  if ((D->T > 0 && (!S->topk_idx || !S->topk_w || !S->perm || !S->inv_perm)) ||
      !S->counts || !S->offsets || !S->pad_offsets || !S->xq || !S->xs || !S->hq || !S->hs ||
      !S->gu)
    return MOE_ERR_INVALID_ARG;
  if (D->T > 0 && (!dout || !dx || !dw_route)) return MOE_ERR_INVALID_ARG;
  if (!aligned256(ws)) return MOE_ERR_MISALIGNED;
  {
    const void* ptrs[] = {dout, dx, dWg, dWu, dWd, W->wdT_q, W->wdT_s, W->wguT_q, W->wguT_s,
                          S->xq, S->xs, S->hq, S->hs, S->gu};
    for (const void* p : ptrs)
      if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  const WsLayout L = ws_layout(D, MOE_OP_BACKWARD);
  if (ws_bytes < static_cast<size_t>(L.total)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t R = padded_rows(D);
  const int E = D->E, d = D->d, f = D->f;
  int32_t* status = at<int32_t>(ws, 0);
  uint8_t* dq = at<uint8_t>(ws, L.dq);
  uint8_t* dsc = at<uint8_t>(ws, L.ds);
  uint8_t* dgu_q = at<uint8_t>(ws, L.dgu_q);
  uint8_t* dgu_s = at<uint8_t>(ws, L.dgu_s);
  uint16_t* dxa = at<uint16_t>(ws, L.dxa);
  uint8_t* dxas = at<uint8_t>(ws, L.dxas);
  float* gbuf = at<float>(ws, L.gbuf);

  // grouped-GEMM tile counters start at zero
  MOE_TRY(cuda_ok(cudaMemsetAsync(at<uint8_t>(ws, 64), 0, 64, st)));
  const int mb = ready_rows(sms, f);
  int32_t* ready = at<int32_t>(ws, L.ready);
  int32_t* order = at<int32_t>(ws, L.order);
  if (D->T > 0) {
    {  // pull reverse-combine: dOut rows gathered into expert order, MXFP8 along d
      StageScope sc(MOE_STAGE_BWD_DOUT, st);
      SchedInitParams SI;
      SI.counts = S->counts;
      SI.pad_offsets = S->pad_offsets;
      SI.E = E;
      SI.ready = ready;
      SI.ready_rows = mb;
      SI.n_ready = static_cast<int>((R + mb - 1) / mb);
      SI.order = order;  // the weight gradients' longest-first expert order
      MOE_TRY(cuda_ok(launch_sched_init(SI, st)));
      MOE_TRY(dispatch_pull(D, dout, S->offsets, S->pad_offsets, 7, S->perm,
                            at<uint8_t>(ws, L.tq), at<uint8_t>(ws, L.ts), dq, dsc, status, sms,
                            st, ready, mb));
    }
    // The SwiGLU backward in the dgrad epilogue costs ~30-40K cycles per 128 x 256 tile; it
    // hides under a tile's MMAs only when K = d is long (measured: 56 K blocks at d = 7168,
    // -0.15 ms per step; 16 at d = 2048, +0.06 ms), so the fusion is used from this width.
    const bool fuse_swiglu = d >= kFuseSwigluMinD;
    {  // G = dout^ . Wd'^T (fp32, padded expert order)
      StageScope sc(MOE_STAGE_BWD_DGRAD_DOWN, st);
      CUtensorMap ta, tb, tg;
      MOE_TRY(make_tmap(&ta, dq, R, d, 128));
      MOE_TRY(make_tmap(&tb, W->wdT_q, static_cast<int64_t>(E) * f, d, 256));
      MOE_TRY(make_out_tmap(&tg, gbuf, R, f, false));
      GemmParams P = {};
      P.G = E;
      P.N = f;
      P.K = d;
      P.mtile_prefix = S->pad_offsets;
      P.prefix_shift = 7;
      P.rows_valid = S->counts;
      P.sfa = dsc;
      P.sfb = W->wdT_s;
      P.status = status;
      P.tile_ctr = at<uint32_t>(ws, kCtrBwdDgradDown);
      P.ready = ready;
      P.ready_rows = mb;
      // d >= kFuseSwigluMinD: the SwiGLU backward in the epilogue of full tiles (G never
      // stored for them); partial tiles, and every tile below that width, store G
      P.f = f;
      P.gu = S->gu;
      P.hq = S->hq;
      P.hs = S->hs;
      P.perm = S->perm;
      P.offsets = S->offsets;
      P.topk_w = S->topk_w;
      P.dgu_q = dgu_q;
      P.dgu_s = dgu_s;
      P.dw_part = at<float>(ws, L.dwpart);
      MOE_TRY(cuda_ok(launch_grouped_gemm(fuse_swiglu ? GEMM_DGRAD_SWIGLU : GEMM_STORE_F32_TMA,
                                          ta, tb, tg, tg, P, sms, st, true)));
    }
    {  // d(router weights), SwiGLU backward, [dg|du] -> MXFP8 along f
      StageScope sc(MOE_STAGE_BWD_SWIGLU, st);
      SwigluBwdParams P = {};
      P.G = gbuf;
      P.gu = S->gu;
      P.h_q = S->hq;
      P.h_s = S->hs;
      P.perm = S->perm;
      P.offsets = S->offsets;
      P.pad_offsets = S->pad_offsets;
      P.topk_w = S->topk_w;
      P.A = D->T * D->k;
      P.E = E;
      P.f = f;
      P.dw_route = dw_route;
      P.dgu_q = dgu_q;
      P.dgu_s = dgu_s;
      P.dw_part = fuse_swiglu ? at<float>(ws, L.dwpart) : nullptr;
      MOE_TRY(cuda_ok(launch_swiglu_bwd(P, sms, st)));
    }
    {  // dXa = [dg|du]^ . [Wg|Wu]'^T
      StageScope sc(MOE_STAGE_BWD_DGRAD_GATEUP, st);
      CUtensorMap ta, tb;
      MOE_TRY(make_tmap(&ta, dgu_q, R, 2 * f, 128));
      MOE_TRY(make_tmap(&tb, W->wguT_q, static_cast<int64_t>(E) * d, 2 * f, 256));
      GemmParams P = {};
      P.G = E;
      P.N = d;
      P.K = 2 * f;
      P.mtile_prefix = S->pad_offsets;
      P.prefix_shift = 7;
      P.rows_valid = S->counts;
      P.sfa = dgu_s;
      P.sfb = W->wguT_s;
      P.status = status;
      P.tile_ctr = at<uint32_t>(ws, kCtrBwdDgradGateUp);
      P.out_scales = dxas;
      CUtensorMap tx, tx32;
      MOE_TRY(make_f16s_tmaps(&tx, &tx32, dxa, R, d));
      MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_TMA, ta, tb, tx, tx32, P, sms, st)));
    }
    {  // push reverse-dispatch: dX[t] = sum_j dXa[row of (t, j)]
      StageScope sc(MOE_STAGE_BWD_DX, st);
      CombineParams P = {};
      P.y = dxa;
      P.ys = dxas;
      P.topk_w = nullptr;
      P.topk_idx = S->topk_idx;
      P.inv = S->inv_perm;
      P.offsets = S->offsets;
      P.mtile_prefix = S->pad_offsets;
      P.prefix_shift = 7;
      P.T = D->T;
      P.d = d;
      P.E = E;
      P.k = D->k;
      P.out = dx;
      P.status = status;
      MOE_TRY(cuda_ok(launch_combine(P, sms, st)));
    }
  }
  uint8_t* xt_q = at<uint8_t>(ws, L.xt_q);
  uint8_t* xt_s = at<uint8_t>(ws, L.xt_s);
  uint8_t* ht_q = at<uint8_t>(ws, L.ht_q);
  uint8_t* ht_s = at<uint8_t>(ws, L.ht_s);
  uint8_t* gt_q = at<uint8_t>(ws, L.gt_q);
  uint8_t* gt_s = at<uint8_t>(ws, L.gt_s);
  uint8_t* yt_q = at<uint8_t>(ws, L.yt_q);
  uint8_t* yt_s = at<uint8_t>(ws, L.yt_s);
  if (D->T > 0) {  // token-direction MX operands of the weight gradients
    StageScope sc(MOE_STAGE_BWD_TRANSPOSE, st);
    TransposeQuantParams P = {};
    P.perm = S->perm;
    P.offsets = S->offsets;
    P.topk_w = S->topk_w;
    P.k = D->k;
    P.pad_offsets = S->pad_offsets;
    P.counts = S->counts;
    P.E = E;
    P.R = R;
    P.status = status;
    auto run = [&](int src, const uint8_t* q, const uint8_t* s, int C, uint8_t* dq_out,
                   uint8_t* ds_out) -> moe_status {
      P.src = src;
      P.q = q;
      P.s = s;
      P.C = C;
      P.dst_q = dq_out;
      P.dst_s = ds_out;
      CUtensorMap tsrc, tdst;
      MOE_TRY(make_tmap(&tsrc, q, R, C, 32, false));  // 32-row boxes
      MOE_TRY(make_tmap(&tdst, dq_out, R * C / 128, 128, 128, true));  // 128 x 128 tiles
      return cuda_ok(launch_transpose_quant(tsrc, tdst, P, sms, st));
    };
    MOE_TRY(run(TSRC_MX, S->xq, S->xs, d, xt_q, xt_s));         // x^ -> X~^T [d, R]
    MOE_TRY(run(TSRC_MX, S->hq, S->hs, f, ht_q, ht_s));         // h^ -> H~^T [f, R]
    MOE_TRY(run(TSRC_MX, dgu_q, dgu_s, 2 * f, gt_q, gt_s));     // [dg|du]^ -> DGU~^T [2f, R]
    MOE_TRY(run(TSRC_MX_W, dq, dsc, d, yt_q, yt_s));            // w * dout^ -> DY~^T [d, R]
  } else {
    // no tokens: every expert's K range is empty; the prefix below is all zeros
  }
  {  // weight gradients, K = each expert's token segment
    StageScope sc(MOE_STAGE_BWD_WGRAD, st);
    const int32_t* prefix = S->pad_offsets;
    if (D->T == 0) MOE_TRY(cuda_ok(cudaMemsetAsync(S->pad_offsets, 0, 4 * (E + 1), st)));
    const int64_t Kt = std::max<int64_t>(R, 128);
    CUtensorMap ta, tb;
    MOE_TRY(make_tmap(&ta, xt_q, Kt * d / 128, 128, 128));  // tiled (see the requantisation)
    MOE_TRY(make_tmap(&tb, gt_q, Kt * 2 * f / 128, 128, 256));
    GemmParams P = {};
    P.G = E;
    P.M = d;
    P.N = 2 * f;
    P.K = static_cast<int>(Kt);
    P.mtile_prefix = prefix;
    P.prefix_shift = 7;
    P.sfa = xt_s;
    P.sfb = gt_s;
    P.out_a = dWg;
    P.out_b = dWu;
    P.split = f;
    P.status = status;
    P.tile_ctr = at<uint32_t>(ws, kCtrBwdWgrad0);
    P.order = D->T > 0 ? order : nullptr;
    CUtensorMap tg, tu;
    MOE_TRY(make_out_tmap(&tg, dWg, static_cast<int64_t>(E) * d, f, true));
    MOE_TRY(make_out_tmap(&tu, dWu, static_cast<int64_t>(E) * d, f, true));
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_WGRAD_BF16, ta, tb, tg, tu, P, sms, st)));
    MOE_TRY(make_tmap(&ta, ht_q, Kt * f / 128, 128, 128));
    MOE_TRY(make_tmap(&tb, yt_q, Kt * d / 128, 128, 256));
    P.M = f;
    P.N = d;
    P.sfa = ht_s;
    P.sfb = yt_s;
    P.out_a = dWd;
    P.out_b = nullptr;
    P.split = d;
    P.tile_ctr = at<uint32_t>(ws, kCtrBwdWgrad1);
    CUtensorMap tdw;
    MOE_TRY(make_out_tmap(&tdw, dWd, static_cast<int64_t>(E) * f, d, true));
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_WGRAD_BF16, ta, tb, tdw, tdw, P, sms, st)));
  }
  return MOE_OK;
}

moe_status moe_router_backward(const moe_dims* D, const float* logits, const int32_t* topk_idx,
                               const float* dw_route, float* dlogits, int32_t* status,
                               void* stream) {
  MOE_TRY(check_dims(D));
  if (D->T == 0) return MOE_OK;
  if (!logits || !topk_idx || !dw_route || !dlogits) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {logits, topk_idx, dw_route, dlogits, status};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  RouterBwdParams P;
  P.logits = logits;
  P.topk_idx = topk_idx;
  P.dw_route = dw_route;
  P.T = D->T;
  P.E = D->E;
  P.k = D->k;
  P.score_fn = D->score_fn;
  P.dlogits = dlogits;
  P.status = status;
  return cuda_ok(launch_router_bwd(P, sms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_router_logits(const moe_dims* D, const uint16_t* x, const uint16_t* wr,
                             float* logits, void* ws, size_t ws_bytes, void* stream) {
  const void* ptrs[] = {wr, x, logits};
  MOE_TRY(router_checks(D, ptrs, D && D->T > 0 ? 3 : 1, ws, ws_bytes));
  if (D->T == 0) return MOE_OK;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const RouterWsLayout L = router_ws_layout(D);
  const int64_t T = D->T, d = D->d, E = D->E;
  RouterSetupParams S = {};
  S.n = 1;
  S.rows[0] = T;
  S.prefix = at<int32_t>(ws, kRouterPrefix);
  S.valid = at<int32_t>(ws, kRouterValid);
  S.ctr = at<uint32_t>(ws, kRouterCtr);
  MOE_TRY(cuda_ok(launch_router_setup(S, st)));
  uint16_t* wr_pad = at<uint16_t>(ws, L.wr_pad);
  MOE_TRY(cuda_ok(launch_pad_copy_bf16(wr, E, d, d, wr_pad, L.NE, d, st)));
  CUtensorMap ta, tb, tc;
  MOE_TRY(make_tmap(&ta, x, T, 2 * d, 128));
  MOE_TRY(make_tmap(&tb, wr_pad, L.NE, 2 * d, 256));
  MOE_TRY(make_out_tmap(&tc, logits, T, E, false));
  GemmParams P = {};
  P.G = 1;
  P.N = static_cast<int>(L.NE);
  P.K = static_cast<int>(2 * d);
  P.mtile_prefix = S.prefix;
  P.rows_valid = S.valid;
  P.status = at<int32_t>(ws, 0);
  P.tile_ctr = S.ctr;
  P.n_valid = static_cast<int>(E);
  return cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_BF16, ta, tb, tc, tc, P, sms, st));
}

moe_status moe_router_grads(const moe_dims* D, const float* dlogits, const uint16_t* x,
                            const uint16_t* wr, float* dx_r, float* dwr, void* ws,
                            size_t ws_bytes, void* stream) {
  const void* ptrs[] = {wr, dwr, dlogits, x, dx_r};
  MOE_TRY(router_checks(D, ptrs, D && D->T > 0 ? 5 : 2, ws, ws_bytes));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t T = D->T, d = D->d, E = D->E;
  if (T == 0)  // no tokens: the weight gradient is zero
    return cuda_ok(cudaMemsetAsync(dwr, 0, static_cast<size_t>(E * d * 4), st));
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  const RouterWsLayout L = router_ws_layout(D);
  RouterSetupParams S = {};
  S.n = 2;
  S.rows[0] = T;  // dx_r = bf16(G) . W_r: token rows
  S.rows[1] = E;  // dW_r = bf16(G)^T . x: expert rows
  S.prefix = at<int32_t>(ws, kRouterPrefix);
  S.valid = at<int32_t>(ws, kRouterValid);
  S.ctr = at<uint32_t>(ws, kRouterCtr);
  MOE_TRY(cuda_ok(launch_router_setup(S, st)));
  uint16_t* dlog = at<uint16_t>(ws, L.dlog);
  uint16_t* dlogT = at<uint16_t>(ws, L.dlogT);
  uint16_t* wrT = at<uint16_t>(ws, L.wrT);
  uint16_t* xT = at<uint16_t>(ws, L.xT);
  MOE_TRY(cuda_ok(launch_pad_copy_f32_bf16(dlogits, T, E, E, dlog, L.Tp128, L.Ep, st)));
  MOE_TRY(cuda_ok(launch_transpose_pad_f32_bf16(dlogits, T, E, E, dlogT, L.Ep128, L.Tp, st)));
  MOE_TRY(cuda_ok(launch_transpose_pad_bf16(wr, E, d, d, wrT, d, L.Ep, st)));
  MOE_TRY(cuda_ok(launch_transpose_pad_bf16(x, T, d, d, xT, d, L.Tp, st)));
  {
    CUtensorMap ta, tb, tc;
    MOE_TRY(make_tmap(&ta, dlog, L.Tp128, 2 * L.Ep, 128));
    MOE_TRY(make_tmap(&tb, wrT, d, 2 * L.Ep, 256));
    MOE_TRY(make_out_tmap(&tc, dx_r, T, d, false));
    GemmParams P = {};
    P.G = 1;
    P.N = static_cast<int>(d);
    P.K = static_cast<int>(2 * L.Ep);
    P.mtile_prefix = S.prefix;
    P.rows_valid = S.valid;
    P.status = at<int32_t>(ws, 0);
    P.tile_ctr = S.ctr;
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_BF16, ta, tb, tc, tc, P, sms, st)));
  }
  CUtensorMap ta, tb, tc;
  MOE_TRY(make_tmap(&ta, dlogT, L.Ep128, 2 * L.Tp, 128));
  MOE_TRY(make_tmap(&tb, xT, d, 2 * L.Tp, 256));
  MOE_TRY(make_out_tmap(&tc, dwr, E, d, false));
  GemmParams P = {};
  P.G = 1;
  P.N = static_cast<int>(d);
  P.K = static_cast<int>(2 * L.Tp);
  P.mtile_prefix = S.prefix + 2;
  P.rows_valid = S.valid + 1;
  P.status = at<int32_t>(ws, 0);
  P.tile_ctr = S.ctr + 1;
  return cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_BF16, ta, tb, tc, tc, P, sms, st));
}

moe_status moe_ep_prepare(const moe_dims* D, const uint16_t* x, const float* logits,
                          int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                          int32_t* perm, int32_t* inv_perm, uint8_t* xq, uint8_t* xs, void* ws,
                          size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(D));
  if (D->T > 0 && (!x || !xq || !xs)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(moe_route_layout(D, logits, topk_idx, topk_w, counts, offsets, perm, inv_perm, nullptr,
                           ws, ws_bytes, stream));
  if (D->T == 0) return MOE_OK;
  return mxfp8_quantize(x, D->T, D->d, D->d, xq, xs, 0, stream);
}

size_t moe_ep_workspace_bytes(const moe_dims* D, int32_t world) {
  EpWsLayout L;
  return ep_ws_layout(D, world, &L) ? static_cast<size_t>(L.total) : 0;
}

moe_status moe_ep_experts(const moe_dims* D, int32_t rank, int32_t world,
                          const moe_ep_peer* peers, const moe_weights* W, void* ws,
                          size_t ws_bytes, void* stream) {
  MOE_TRY(check_dims(D));
  if (world < 1 || world > 64 || D->E % world) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (rank < 0 || rank >= world || !peers || !W || !ws) return MOE_ERR_INVALID_ARG;
  if (!W->wgu_q || !W->wgu_s || !W->wd_q || !W->wd_s) return MOE_ERR_INVALID_ARG;
  {
    const void* ptrs[] = {peers, W->wgu_q, W->wgu_s, W->wd_q, W->wd_s};
    for (const void* p : ptrs)
      if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  if (!aligned256(ws)) return MOE_ERR_MISALIGNED;
  EpWsLayout L;
  if (!ep_ws_layout(D, world, &L)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < static_cast<size_t>(L.total)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t d = D->d, f = D->f;
  const int E_loc = static_cast<int>(L.E_loc);
  int32_t* status = at<int32_t>(ws, 0);
  MOE_TRY(cuda_ok(cudaMemsetAsync(at<uint8_t>(ws, 64), 0, 64, st)));  // tile counters
  EpParams P = {};
  P.peers = peers;
  P.world = world;
  P.rank = rank;
  P.E_loc = E_loc;
  P.k = D->k;
  P.d = static_cast<int>(d);
  P.R_cap = L.R_cap;
  P.recv_counts = at<int32_t>(ws, L.recv_counts);
  P.recv_off = at<int32_t>(ws, L.recv_off);
  P.mtile = at<int32_t>(ws, L.mtile);
  P.src_base = at<int32_t>(ws, L.src_base);
  P.origin = at<int64_t>(ws, L.origin);
  P.xq = at<uint8_t>(ws, L.xq);
  P.xs = at<uint8_t>(ws, L.xs);
  P.y = at<uint16_t>(ws, L.y);
  P.ys = at<uint8_t>(ws, L.ys);
  P.status = status;
  {
    StageScope sc(MOE_STAGE_EP_PULL, st);
    MOE_TRY(cuda_ok(launch_ep_layout(P, st)));
    MOE_TRY(cuda_ok(launch_ep_pull(P, sms, st)));
  }
  uint8_t* hq = at<uint8_t>(ws, L.hq);
  uint8_t* hs = at<uint8_t>(ws, L.hs);
  {  // gate/up + SwiGLU + MX requantisation of h, over the received rows of E_loc experts
    StageScope sc(MOE_STAGE_GATEUP, st);
    CUtensorMap ta, tb;
    MOE_TRY(make_tmap(&ta, P.xq, L.R_cap, d, 128));
    MOE_TRY(make_tmap(&tb, W->wgu_q, L.E_loc * 2 * f, d, 256));
    GemmParams G = {};
    G.G = E_loc;
    G.N = static_cast<int>(2 * f);
    G.K = static_cast<int>(d);
    G.f = static_cast<int>(f);
    G.mtile_prefix = P.mtile;
    G.rows_valid = P.recv_counts;
    G.sfa = P.xs;
    G.sfb = W->wgu_s;
    G.hq = hq;
    G.hs = hs;
    G.status = status;
    G.tile_ctr = at<uint32_t>(ws, kCtrFwdGateUp);
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_GATEUP_SWIGLU, ta, tb, ta, tb, G, sms, st)));
  }
  {  // down: y as scaled fp16
    StageScope sc(MOE_STAGE_DOWN, st);
    CUtensorMap ta, tb, ty, ty32;
    MOE_TRY(make_tmap(&ta, hq, L.R_cap, f, 128));
    MOE_TRY(make_tmap(&tb, W->wd_q, L.E_loc * d, f, 256));
    MOE_TRY(make_f16s_tmaps(&ty, &ty32, at<uint16_t>(ws, L.y), L.R_cap, d));
    GemmParams G = {};
    G.G = E_loc;
    G.N = static_cast<int>(d);
    G.K = static_cast<int>(f);
    G.mtile_prefix = P.mtile;
    G.rows_valid = P.recv_counts;
    G.sfa = hs;
    G.sfb = W->wd_s;
    G.status = status;
    G.tile_ctr = at<uint32_t>(ws, kCtrFwdDown);
    G.out_scales = at<uint8_t>(ws, L.ys);
    MOE_TRY(cuda_ok(launch_grouped_gemm(GEMM_STORE_F32_TMA, ta, tb, ty, ty32, G, sms, st)));
  }
  StageScope sc(MOE_STAGE_EP_PUSH, st);
  return cuda_ok(launch_ep_push(P, sms, st));
}

moe_status moe_ep_combine(const moe_dims* D, const float* topk_w, const uint16_t* y,
                          const uint8_t* ys, uint16_t* out, int32_t* status, void* stream) {
  MOE_TRY(check_dims(D));
  if (D->T == 0) return MOE_OK;
  if (!topk_w || !y || !ys || !out) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {topk_w, y, ys, out, status};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  int sms = 0;
  MOE_TRY(device_sms(&sms));
  CombineParams P = {};
  P.y = y;
  P.ys = ys;
  P.topk_w = topk_w;
  P.T = D->T;
  P.d = D->d;
  P.E = D->E;
  P.k = D->k;
  P.out = out;
  P.status = status;
  P.direct_rows = 1;
  StageScope sc(MOE_STAGE_COMBINE, static_cast<cudaStream_t>(stream));
  return cuda_ok(launch_combine(P, sms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_debug_withhold_ready(int32_t minibatch) {
  g_withhold.store(minibatch < 0 ? -1 : minibatch);
  return MOE_OK;
}

moe_status moe_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof_on = on != 0;
  return MOE_OK;
}

moe_status moe_profile_collect(double* ms_per_stage, int32_t* launches_per_stage,
                               int32_t n_stages) {
  if (!ms_per_stage || !launches_per_stage || n_stages <= 0) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(g_prof_mu);
  for (int i = 0; i < n_stages; ++i) {
    ms_per_stage[i] = 0.0;
    launches_per_stage[i] = 0;
  }
  moe_status rc = MOE_OK;
  for (const StageMark& m : g_prof_marks) {
    float ms = 0.f;
    if (cudaEventSynchronize(m.b) != cudaSuccess ||
        cudaEventElapsedTime(&ms, m.a, m.b) != cudaSuccess)
      rc = MOE_ERR_CUDA;
    if (m.stage >= 0 && m.stage < n_stages) {
      ms_per_stage[m.stage] += ms;
      launches_per_stage[m.stage] += 1;
    }
    g_prof_pool.push_back(m.a);
    g_prof_pool.push_back(m.b);
  }
  g_prof_marks.clear();
  return rc;
}

moe_status moe_get_device_status(void* ws, void* stream, int32_t* code) {
  if (!ws || !code) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  MOE_TRY(cuda_ok(cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st)));
  MOE_TRY(cuda_ok(cudaStreamSynchronize(st)));
  *code = v;
  if (v != 0) MOE_TRY(cuda_ok(cudaMemsetAsync(ws, 0, sizeof(int32_t), st)));
  return MOE_OK;
}

}  // extern "C"
