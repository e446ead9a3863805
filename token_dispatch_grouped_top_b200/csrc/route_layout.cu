// Top-k routing and the per-expert layout.
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72":
//   lead / §01 -- the router picks a few experts per token at every step; before the
//   tokens can move, the system counts each expert's tokens, decides where every token is
//   placed and keeps one expert's tokens contiguous, all without a CPU round trip (§02).
//
// Two launches:
//   route_rank_kernel   one CTA of 32 warps per tile of 64 tokens, two tokens per warp.
//                       Top-k on integer ranking keys (one per logit, ordered as the
//                       values): each of the k rounds is a warp max of the keys and a warp
//                       min of the indices holding it (hardware warp reductions; ties go
//                       to the lower expert index), then routing weights, deterministic
//                       ranks inside the tile (ballot masks, no order-dependent atomics)
//                       and the tile's count vector over the experts.  The tile that
//                       finishes last scans the count vectors over the tiles, giving every
//                       tile its first rank inside each expert, and turns the totals into
//                       counts, offsets and the padded tile prefix.
//   scatter_kernel      pos = offsets[e] + tile_start[tile, e] + rank in the tile;
//                       perm[pos] = a; inv[a] = pos.
// The result is the stable counting sort: inside an expert, ascending token.
#include <limits.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRouteTile = 64;       // tokens per CTA
constexpr int kRouteThreads = 1024;  // one thread per expert in the count phases
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kTokPerWarp = kRouteTile / kRouteWarps;
constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;
constexpr int kKeyGone = INT_MIN;    // key of an expert already selected (below every logit)
static_assert(kMaxE <= kRouteThreads, "one thread per expert");
static_assert(kRouteTile == 2 * 32, "two 32-token rank groups per tile");

// Ranking key of a logit: a signed integer ordered as the value.  A NaN logit ranks as
// -inf and -0 as +0, so equal values (including both zeros) get equal keys and the tie
// rule decides between them.  key_value inverts the map for the kept (canonical) value.
__device__ __forceinline__ int rank_key(float v) {
  if (v != v) v = -INFINITY;
  if (v == 0.f) v = 0.f;
  const int b = __float_as_int(v);
  return b >= 0 ? b : b ^ 0x7fffffff;
}
__device__ __forceinline__ float key_value(int key) {
  return __int_as_float(key >= 0 ? key : key ^ 0x7fffffff);
}

// Inclusive scan of two values over the block's warps in warp order (kRouteThreads
// threads); returns the exclusive prefix of each through cex / mex.
__device__ __forceinline__ void block_excl_scan2(int c, int m, int& cex, int& mex, int* s_wc,
                                                 int* s_wm, int lane, int warp) {
  int cs = c, ms = m;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int tc = __shfl_up_sync(kFull, cs, off), tm = __shfl_up_sync(kFull, ms, off);
    if (lane >= off) {
      cs += tc;
      ms += tm;
    }
  }
  if (lane == 31) {
    s_wc[warp] = cs;
    s_wm[warp] = ms;
  }
  __syncthreads();
  if (warp == 0) {
    int a = s_wc[lane], bm = s_wm[lane];
    const int a0 = a, b0 = bm;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int ta = __shfl_up_sync(kFull, a, off), tb = __shfl_up_sync(kFull, bm, off);
      if (lane >= off) {
        a += ta;
        bm += tb;
      }
    }
    s_wc[lane] = a - a0;  // exclusive prefix over the preceding warps
    s_wm[lane] = bm - b0;
  }
  __syncthreads();
  cex = s_wc[warp] + cs - c;
  mex = s_wm[warp] + ms - m;
}

template <int NPL>
__global__ void __launch_bounds__(kRouteThreads, 1) route_rank_kernel(RouteParams P) {
  __shared__ int s_idx[kRouteTile][kMaxK];
  __shared__ int s_rank[kRouteTile][kMaxK];
  __shared__ uint32_t s_mask[2][kMaxE];
  __shared__ int s_cnt[2][kMaxE];  // per 32-token group count, then exclusive group prefix
  __shared__ int s_red[kRouteThreads];
  __shared__ int s_wc[kRouteWarps], s_wm[kRouteWarps];
  __shared__ int s_bid, s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = P.E, k = P.k;

  if (tid == 0) s_bid = static_cast<int>(atomicAdd(P.tile_counter, 1u));
  for (int e = tid; e < E; e += kRouteThreads) {
    s_mask[0][e] = s_mask[1][e] = 0u;
    s_cnt[0][e] = s_cnt[1][e] = 0;
  }
  __syncthreads();
  launch_dependents();  // the scatter launches now and waits for this grid's completion
  const int b = s_bid;
  const int64_t t0 = static_cast<int64_t>(b) * kRouteTile;

  // ---- 1. top-k per token: a warp selects for its kTPW tokens at once (independent
  //         chains interleave), k rounds of warp max (key) + warp min (index) -----------
  constexpr int kTPW = NPL <= 8 ? kTokPerWarp : 1;
#pragma unroll 1
  for (int tl0 = warp * kTokPerWarp; tl0 < warp * kTokPerWarp + kTokPerWarp; tl0 += kTPW) {
    int kv[kTPW][NPL];
    int sel_key[kTPW], sel_e[kTPW];
#pragma unroll
    for (int u = 0; u < kTPW; ++u) {
      const int64_t t = t0 + tl0 + u;
      const bool tv = t < P.T;
      const float* row = P.logits + (tv ? t : 0) * E;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        kv[u][i] = (tv && e < E) ? rank_key(__ldg(row + e)) : (e < E ? rank_key(-INFINITY)
                                                                    : kKeyGone);
      }
      sel_key[u] = 0;
      sel_e[u] = 0;
    }
    for (int j = 0; j < k; ++j) {
#pragma unroll
      for (int u = 0; u < kTPW; ++u) {
        int lm = kv[u][0];
#pragma unroll
        for (int i = 1; i < NPL; ++i) lm = max(lm, kv[u][i]);
        const int m = __reduce_max_sync(kFull, lm);
        int li = NPL;  // this lane's first slot holding the maximum
#pragma unroll
        for (int i = NPL - 1; i >= 0; --i) li = kv[u][i] == m ? i : li;
        int be = __reduce_min_sync(kFull, li < NPL ? (li << 5) | lane : 0x7fffffff);
        if (be < 0 || be >= E) {  // cannot happen while fewer than E are taken; never index with it
          if (lane == 0) latch(P.status, MOE_ERR_DEVICE_BOUNDS);
          be = 0;
        }
        const bool mine = (be & 31) == lane;
        const int bi = be >> 5;
#pragma unroll
        for (int i = 0; i < NPL; ++i) kv[u][i] = (mine && bi == i) ? kKeyGone : kv[u][i];
        if (lane == j) {
          sel_key[u] = m;
          sel_e[u] = be;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kTPW; ++u) {
      const int tl = tl0 + u;
      const int64_t t = t0 + tl;
      const float sel_v = key_value(sel_key[u]);
      float score;
      if (P.score_fn == MOE_SCORE_SOFTMAX_TOPK) {
        const float m = __shfl_sync(kFull, sel_v, 0);  // slot 0 holds the largest logit
        score = (lane < k) ? expf(sel_v - m) : 0.f;
      } else {
        score = (lane < k) ? 1.f / (1.f + expf(-sel_v)) : 0.f;
      }
      float sum = score;
#pragma unroll
      for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
      if (t < P.T && lane < k) {
        P.topk_idx[t * k + lane] = sel_e[u];
        P.topk_w[t * k + lane] = score / sum;
        s_idx[tl][lane] = sel_e[u];
      }
    }
  }
  __syncthreads();

  // ---- 2. deterministic ranks inside each 32-token group (token = lane) --------------
  // One warp per (group, slot).  s_mask[g][e]: the lanes of group g that chose expert e
  // (in any slot: a token chooses an expert once).  Lanes choosing the same expert in a
  // slot are grouped first, so each expert's word takes one atomic per slot instead of
  // one per lane (hot experts are chosen by most lanes of a group: per-lane atomics on
  // one word serialise).
  const uint32_t below = (1u << lane) - 1u;
  for (int p = warp; p < 2 * k; p += kRouteWarps) {
    const int g = p & 1, j = p >> 1, tl = 32 * g + lane;
    const bool valid = t0 + tl < P.T;
    const int e = valid ? s_idx[tl][j] : -1 - lane;  // invalid lanes match nobody
    const uint32_t same = __match_any_sync(kFull, e);
    if (valid && (same & below) == 0u) atomicOr(&s_mask[g][e], same);
  }
  __syncthreads();
  for (int p = warp; p < 2 * k; p += kRouteWarps) {
    const int g = p & 1, j = p >> 1, tl = 32 * g + lane;
    if (t0 + tl < P.T) {
      const int e = s_idx[tl][j];
      const uint32_t m = s_mask[g][e];
      s_rank[tl][j] = __popc(m & below);
      if ((m & below) == 0u) s_cnt[g][e] = __popc(m);  // the group's first lane choosing e
    }
  }
  __syncthreads();

  // ---- 3. tile histogram; tile-local ranks (thread e owns expert e) -----------------
  const bool owner = tid < E;
  const int64_t rowE = static_cast<int64_t>(E);
  if (owner) {
    const int c0 = s_cnt[0][tid], c1 = s_cnt[1][tid];
    s_cnt[0][tid] = 0;
    s_cnt[1][tid] = c0;
    P.agg[b * rowE + tid] = c0 + c1;
  }
  __syncthreads();
  for (int i = tid; i < kRouteTile * k; i += kRouteThreads) {
    const int tl = i / k, j = i - tl * k;
    const int64_t t = t0 + tl;
    if (t >= P.T) continue;
    const int e = s_idx[tl][j];
    P.rank[t * k + j] = s_cnt[tl >> 5][e] + s_rank[tl][j];
  }

  // ---- 4. the last tile to finish scans the count vectors -----------------------------
  // Publication: the block's stores, a block barrier, then one thread's fence and atomic
  // (cumulative over the stores the barrier ordered before it); the last tile's thread
  // fences again after its atomic, before the block reads the other tiles' vectors.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(P.done_counter, 1u) == static_cast<uint32_t>(P.num_tiles - 1);
    __threadfence();
  }
  __syncthreads();
  if (!s_last) return;

  // Per expert, the exclusive prefix of the tiles' counts = each tile's first rank inside
  // the expert (tile_start).  ng thread groups split the tiles into contiguous runs: a
  // first pass sums each run, the runs' sums give every run its base, a second pass
  // writes the prefixes; all loads of a batch are in flight at once.
  const int nt = P.num_tiles;
  const int ng = kRouteThreads / E;
  const int grp = tid / E, ge = tid - grp * E;
  const int run_len = (nt + ng - 1) / ng;
  const int r0 = grp < ng ? min(grp * run_len, nt) : 0;
  const int r1 = grp < ng ? min(r0 + run_len, nt) : 0;
  int run_sum = 0;
  for (int t = r0; t < r1; t += 16) {
    int v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = t + u < r1 ? __ldcg(P.agg + (t + u) * rowE + ge) : 0;
#pragma unroll
    for (int u = 0; u < 16; ++u) run_sum += v[u];
  }
  s_red[tid] = run_sum;
  __syncthreads();
  int base = 0, total = 0;
  if (grp < ng) {
    for (int q = 0; q < ng; ++q) {
      const int r = s_red[q * E + ge];
      base += q < grp ? r : 0;
      total += r;
    }
  }
  for (int t = r0; t < r1; t += 16) {
    int v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = t + u < r1 ? __ldcg(P.agg + (t + u) * rowE + ge) : 0;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (t + u < r1) P.tile_start[(t + u) * rowE + ge] = base;
      base += v[u];
    }
  }

  // ---- 5. counts, offsets and the padded tile prefix (thread e < E is in group 0) ---
  const int c = owner ? total : 0;
  const int m = (c + 127) >> 7;
  int cex, mex;
  block_excl_scan2(c, m, cex, mex, s_wc, s_wm, lane, warp);
  if (owner) {
    P.counts[tid] = c;
    P.offsets[tid] = cex;
    P.mtile_prefix[tid] = mex;
    if (P.pad_offsets) P.pad_offsets[tid] = mex * 128;
    if (tid == E - 1) {
      P.offsets[E] = cex + c;
      P.mtile_prefix[E] = mex + m;
      if (P.pad_offsets) P.pad_offsets[E] = (mex + m) * 128;
    }
  }
}

__global__ void scatter_kernel(const int32_t* __restrict__ topk_idx,
                               const int32_t* __restrict__ rank,
                               const int32_t* __restrict__ tile_start,
                               const int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                               int32_t* __restrict__ inv, int64_t A, int E, int k,
                               int32_t* status) {
  wait_prior_grid();  // launched as a programmatic dependent of route_rank_kernel
  for (int64_t a = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; a < A;
       a += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = topk_idx[a];
    if (e < 0 || e >= E) {
      latch(status, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    const int64_t tile = a / k / kRouteTile;
    const int64_t pos = static_cast<int64_t>(offsets[e]) + tile_start[tile * E + e] + rank[a];
    if (pos < 0 || pos >= A) {
      latch(status, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    perm[pos] = static_cast<int32_t>(a);
    inv[a] = static_cast<int32_t>(pos);
  }
}

cudaError_t launch_route_layout(const RouteParams& P, int32_t* perm, int32_t* inv,
                                int num_sms, cudaStream_t stream) {
  const int grid = P.num_tiles;
  const int ept = (P.E + 31) / 32;
  if (ept <= 1)
    route_rank_kernel<1><<<grid, kRouteThreads, 0, stream>>>(P);
  else if (ept <= 2)
    route_rank_kernel<2><<<grid, kRouteThreads, 0, stream>>>(P);
  else if (ept <= 4)
    route_rank_kernel<4><<<grid, kRouteThreads, 0, stream>>>(P);
  else if (ept <= 8)
    route_rank_kernel<8><<<grid, kRouteThreads, 0, stream>>>(P);
  else if (ept <= 16)
    route_rank_kernel<16><<<grid, kRouteThreads, 0, stream>>>(P);
  else
    route_rank_kernel<32><<<grid, kRouteThreads, 0, stream>>>(P);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t A = P.T * P.k;
  const int64_t blocks = (A + 255) / 256;
  const int sgrid = static_cast<int>(blocks < 8 * num_sms ? blocks : 8 * num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sgrid));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, scatter_kernel, static_cast<const int32_t*>(P.topk_idx),
                            static_cast<const int32_t*>(P.rank),
                            static_cast<const int32_t*>(P.tile_start),
                            static_cast<const int32_t*>(P.offsets), perm, inv, A, P.E, P.k,
                            P.status);
}

int route_num_tiles(int64_t T) { return static_cast<int>((T + kRouteTile - 1) / kRouteTile); }

}  // namespace moe
