// Expert parallelism: the article's dispatch and combine between GPUs.
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72":
//   §01 -- the expert owner needs to know how many rows each GPU sends it and where they
//          go before the grouped GEMM can run on them contiguously;
//   §02 -- pull dispatch: the consumer fetches the rows it needs by source and offset into
//          its own memory; push combine: the outputs go back to the tokens' GPUs, where the
//          weighted merge runs.
//
// Rank `rank` owns experts [rank * E_loc, (rank + 1) * E_loc).  Its received rows are laid
// out expert by expert (each segment padded to whole 128-row tiles, as the single-GPU
// layer's), inside an expert source rank by source rank, inside a source in that source's
// segment order (ascending token).  The peers' counts, offsets, permutations and per-token
// MX rows are read, and the expert outputs written back, through the moe_ep_peer table:
// plain loads and stores that reach the other GPUs' memory over NVLink when the table holds
// peer mappings.  No TMA touches peer memory here (no multicast anywhere).
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kEpLayoutThreads = 1024;  // one thread per local expert (E_loc <= 1024)
constexpr int kMaxE = 1024;             // experts of a layer (moe_dims rule)

// Exclusive prefix sum over the block (kEpLayoutThreads values), total returned to all.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t* buf,
                                                        int64_t* total) {
  const int tid = threadIdx.x;
  buf[tid] = v;
  __syncthreads();
  for (int off = 1; off < kEpLayoutThreads; off <<= 1) {
    const int64_t add = tid >= off ? buf[tid - off] : 0;
    __syncthreads();
    buf[tid] += add;
    __syncthreads();
  }
  const int64_t incl = buf[tid];
  *total = buf[kEpLayoutThreads - 1];
  __syncthreads();  // buf is reused by the next scan
  return incl - v;
}

// The receive layout: per local expert el, the rows of each source rank (the sources'
// counts of expert rank * E_loc + el, read from their memory), their prefix and the padded
// tile prefix.  A negative count, a source count above its T * k, or a total beyond the
// receive buffer latches MOE_ERR_DEVICE_BOUNDS and leaves every count zero (the rank then
// receives nothing and its GEMMs have no tiles).
__global__ void __launch_bounds__(kEpLayoutThreads) ep_layout_kernel(EpParams P) {
  __shared__ int64_t buf[kEpLayoutThreads];
  __shared__ int s_bad;
  const int el = threadIdx.x;
  if (el == 0) s_bad = 0;
  __syncthreads();
  int64_t cnt = 0;
  if (el < P.E_loc) {
    const int e = P.rank * P.E_loc + el;
    for (int s = 0; s < P.world; ++s) {
      const int64_t c = P.peers[s].counts[e];
      if (c < 0 || c > P.peers[s].T * P.k) s_bad = 1;
      P.src_base[s * P.E_loc + el] = static_cast<int32_t>(cnt < (1LL << 31) ? cnt : 0);
      cnt += c < 0 ? 0 : c;
    }
  }
  const int64_t tiles = (cnt + 127) / 128;
  int64_t total_rows = 0, total_tiles = 0;
  const int64_t off = block_exclusive_scan(cnt, buf, &total_rows);
  const int64_t toff = block_exclusive_scan(tiles, buf, &total_tiles);
  const bool bad = s_bad != 0 || total_tiles * 128 > P.R_cap;
  if (bad && el == 0) latch(P.status, MOE_ERR_DEVICE_BOUNDS);
  if (el < P.E_loc) {
    P.recv_counts[el] = bad ? 0 : static_cast<int32_t>(cnt);
    P.recv_off[el] = bad ? 0 : static_cast<int32_t>(off);
    P.mtile[el] = bad ? 0 : static_cast<int32_t>(toff);
  }
  if (el == 0) {
    P.recv_off[P.E_loc] = bad ? 0 : static_cast<int32_t>(total_rows);
    P.mtile[P.E_loc] = bad ? 0 : static_cast<int32_t>(total_tiles);
  }
}

cudaError_t launch_ep_layout(const EpParams& P, cudaStream_t stream) {
  if (P.E_loc < 1 || P.E_loc > kEpLayoutThreads || P.world < 1) return cudaErrorInvalidValue;
  ep_layout_kernel<<<1, kEpLayoutThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

// Received row q (0 <= q < recv_off[E_loc]) -> its local expert el (binary search over the
// shared prefix), source rank s and the index i inside that source's segment.
struct EpRow {
  int el, s;
  int64_t r, i;  // row inside the expert's segment, row inside the source's part
};
__device__ __forceinline__ EpRow ep_row(const EpParams& P, const int* s_off, int64_t q) {
  EpRow w;
  int lo = 0, hi = P.E_loc;  // s_off[lo] <= q < s_off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_off[mid] <= q) lo = mid; else hi = mid;
  }
  w.el = lo;
  w.r = q - s_off[lo];
  int s = 0;
  while (s + 1 < P.world && P.src_base[(s + 1) * P.E_loc + lo] <= w.r) ++s;
  w.s = s;
  w.i = w.r - P.src_base[s * P.E_loc + lo];
  return w;
}

// Pull dispatch: one warp per received row fetches its token's MX codes (d bytes, 16-byte
// loads) and scale bytes from the source rank's per-token copy and writes them at the
// row's padded position, the scales re-laid into the UMMA layout; the row's origin
// (source, assignment) is kept for the push.
__global__ void __launch_bounds__(256) ep_pull_kernel(EpParams P) {
  __shared__ int s_off[kMaxE + 1];
  __shared__ int s_mt[kMaxE + 1];
  for (int i = threadIdx.x; i <= P.E_loc; i += blockDim.x) {
    s_off[i] = P.recv_off[i];
    s_mt[i] = P.mtile[i];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t total = s_off[P.E_loc];
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int d = P.d;
  const int64_t kg = d >> 7;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
       q < total; q += warps) {
    const EpRow w = ep_row(P, s_off, q);
    const moe_ep_peer& src = P.peers[w.s];
    const int e = P.rank * P.E_loc + w.el;
    const int a = src.perm[src.offsets[e] + w.i];
    const int64_t t = a / P.k;
    const int64_t p = static_cast<int64_t>(s_mt[w.el]) * 128 + w.r;
    if (a < 0 || t >= src.T || p >= P.R_cap) {
      if (lane == 0) latch(P.status, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    const uint4* qs = reinterpret_cast<const uint4*>(src.xq + t * d);
    uint4* qd = reinterpret_cast<uint4*>(P.xq + p * d);
    for (int i = lane; i < (d >> 4); i += 32) qd[i] = qs[i];
    const uint32_t* ss = reinterpret_cast<const uint32_t*>(src.xs + t * (d >> 5));
    for (int g = lane; g < kg; g += 32)
      *reinterpret_cast<uint32_t*>(P.xs + umma_scale_offset(p, 4 * g, kg)) = ss[g];
    if (lane == 0) P.origin[p] = (static_cast<int64_t>(w.s) << 32) | static_cast<uint32_t>(a);
  }
}

// Push combine: one warp per received row writes its expert output (scaled fp16 values and
// their scale bytes) into the source rank's buffer at the row of its assignment.
__global__ void __launch_bounds__(256) ep_push_kernel(EpParams P) {
  __shared__ int s_off[kMaxE + 1];
  __shared__ int s_mt[kMaxE + 1];
  for (int i = threadIdx.x; i <= P.E_loc; i += blockDim.x) {
    s_off[i] = P.recv_off[i];
    s_mt[i] = P.mtile[i];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t total = s_off[P.E_loc];
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int d = P.d;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
       q < total; q += warps) {
    int lo = 0, hi = P.E_loc;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_off[mid] <= q) lo = mid; else hi = mid;
    }
    const int64_t p = static_cast<int64_t>(s_mt[lo]) * 128 + (q - s_off[lo]);
    if (p >= P.R_cap) continue;  // the pull latched this already
    const int64_t o = P.origin[p];
    const int s = static_cast<int>(o >> 32);
    const int64_t a = static_cast<uint32_t>(o);
    if (s < 0 || s >= P.world) continue;
    const moe_ep_peer& dst = P.peers[s];
    if (a >= dst.T * P.k) {
      if (lane == 0) latch(P.status, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    const uint4* ys = reinterpret_cast<const uint4*>(P.y + p * d);
    uint4* yd = reinterpret_cast<uint4*>(dst.y + a * d);
    for (int i = lane; i < (d >> 3); i += 32) yd[i] = ys[i];
    const uint32_t* ss = reinterpret_cast<const uint32_t*>(P.ys + p * (d >> 5));
    uint32_t* sd = reinterpret_cast<uint32_t*>(dst.ys + a * (d >> 5));
    for (int g = lane; g < (d >> 7); g += 32) sd[g] = ss[g];
  }
}

static int ep_grid(int num_sms) { return 8 * num_sms; }

cudaError_t launch_ep_pull(const EpParams& P, int num_sms, cudaStream_t stream) {
  if (P.E_loc < 1 || P.E_loc > kMaxE) return cudaErrorInvalidValue;
  ep_pull_kernel<<<ep_grid(num_sms), 256, 0, stream>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_ep_push(const EpParams& P, int num_sms, cudaStream_t stream) {
  if (P.E_loc < 1 || P.E_loc > kMaxE) return cudaErrorInvalidValue;
  ep_push_kernel<<<ep_grid(num_sms), 256, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace moe
