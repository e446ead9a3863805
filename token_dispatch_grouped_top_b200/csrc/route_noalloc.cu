// moe_route_layout_noalloc: routing + layout without any caller-provided workspace.
//
// Some callers cannot allocate device memory themselves: a plugin whose host framework
// owns every device allocation, an embedded runtime with a fixed memory budget, or a
// latency-critical request path where cudaMalloc's implicit device synchronisation is
// not acceptable.  For them this entry point keeps its scratch (the per-tile count
// vectors and first ranks, the per-assignment ranks, the tile counters) in a file-scope
// __device__ array of fixed size instead of a workspace.  It runs the same kernels as
// moe_route_layout.
//
// Properties the caller must know:
//  - The array (kScratchBytes) is part of the library image: every GPU that loads the
//    library holds it until the process exits.
//  - Problems whose scratch exceeds kScratchBytes are rejected (MOE_ERR_UNSUPPORTED_SHAPE)
//    before anything is launched.
//  - Every call looks the array's device address up for the current device
//    (cudaGetSymbolAddress: no allocation, no synchronisation), so a context that was torn
//    down and re-created (cudaDeviceReset) is picked up; make the first call on a device
//    before any stream capture, since that lookup may load the library's module.
//  - All calls share the one array.  Each call clears the parts that must start at zero
//    (the tile counters); calls whose executions overlap on the GPU (different
//    streams, or different host threads) race on the array and give wrong results.
//  - The same shape rules and device check as moe_route_layout apply; device-side errors
//    are latched into the caller's status word, which is therefore required.
//  - No cudaMalloc, cudaFree or allocating library routine is called.
#include <cuda_runtime.h>

#include "../../include/moe.h"
#include "kernels.h"

namespace {

constexpr int64_t kScratchBytes = int64_t(8) << 20;  // 8 MiB

static __device__ __align__(256) uint8_t g_route_scratch[kScratchBytes];

constexpr int64_t kA = 256;
inline int64_t up(int64_t x) { return (x + kA - 1) / kA * kA; }

struct ScratchLayout {
  int64_t counters, agg, tstart, rank, mtile, total, zero_bytes;
};

// header: [0, 8) tile + done counters, then the count vectors
ScratchLayout scratch_layout(const moe_dims* D) {
  ScratchLayout L;
  const int64_t nt = moe::route_num_tiles(D->T), E = D->E, A = D->T * D->k;
  L.counters = 0;
  L.zero_bytes = 8;
  L.agg = kA;
  L.tstart = up(L.agg + 4 * nt * E);
  L.rank = up(L.tstart + 4 * nt * E);
  L.mtile = up(L.rank + 4 * A);
  L.total = up(L.mtile + 4 * (E + 1));
  return L;
}

// device address of the array for the current device (looked up on every call)
uint8_t* scratch_ptr(moe_status* st) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
    *st = MOE_ERR_CUDA;
    return nullptr;
  }
  *st = MOE_OK;
  return static_cast<uint8_t*>(p);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" moe_status moe_route_layout_noalloc(const moe_dims* D, const float* logits,
                                               int32_t* topk_idx, float* topk_w, int32_t* counts,
                                               int32_t* offsets, int32_t* perm, int32_t* inv_perm,
                                               int32_t* pad_offsets, int32_t* status,
                                               void* stream) {
  const moe_status dim_ok = moe::check_dims(D);
  if (dim_ok != MOE_OK) return dim_ok;
  const ScratchLayout L = scratch_layout(D);
  if (L.total > kScratchBytes) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!counts || !offsets || (D->T > 0 && (!logits || !topk_idx || !topk_w || !perm ||
                                           !inv_perm || !status)))
    return MOE_ERR_INVALID_ARG;
  {
    const void* ptrs[] = {logits, topk_idx, topk_w, counts, offsets, perm, inv_perm,
                          pad_offsets, status};
    for (const void* p : ptrs)
      if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  int sms = 0;
  const moe_status dev_ok = moe::device_sms(&sms);
  if (dev_ok != MOE_OK) return dev_ok;
  moe_status st = MOE_OK;
  uint8_t* base = scratch_ptr(&st);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* mtile = reinterpret_cast<int32_t*>(base + L.mtile);
  if (D->T == 0) {
    if (cudaMemsetAsync(counts, 0, 4 * D->E, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, 4 * (D->E + 1), s) != cudaSuccess ||
        (pad_offsets && cudaMemsetAsync(pad_offsets, 0, 4 * (D->E + 1), s) != cudaSuccess))
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  // the counters must start at zero; everything else is written before read
  if (cudaMemsetAsync(base, 0, L.zero_bytes, s) != cudaSuccess) return MOE_ERR_CUDA;
  moe::RouteParams P;
  P.logits = logits;
  P.T = D->T;
  P.E = D->E;
  P.k = D->k;
  P.score_fn = D->score_fn;
  P.num_tiles = moe::route_num_tiles(D->T);
  P.topk_idx = topk_idx;
  P.topk_w = topk_w;
  P.rank = reinterpret_cast<int32_t*>(base + L.rank);
  P.counts = counts;
  P.offsets = offsets;
  P.mtile_prefix = mtile;
  P.pad_offsets = pad_offsets;
  P.tile_counter = reinterpret_cast<uint32_t*>(base + L.counters);
  P.done_counter = reinterpret_cast<uint32_t*>(base + L.counters + 4);
  P.agg = reinterpret_cast<int32_t*>(base + L.agg);
  P.tile_start = reinterpret_cast<int32_t*>(base + L.tstart);
  P.status = status;
  return moe::launch_route_layout(P, perm, inv_perm, sms, s) == cudaSuccess ? MOE_OK
                                                                            : MOE_ERR_CUDA;
}
