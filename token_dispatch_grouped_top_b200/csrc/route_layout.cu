// S1 + S2: top-k routing and the per-expert layout.
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72":
//   lead / §01 -- the router picks a few experts per token at every step; before the
//   tokens can move, the system counts each expert's tokens, decides where every token is
//   placed and keeps one expert's tokens contiguous, all without a CPU round trip (§02).
//
// Two launches:
//   route_rank_kernel   one CTA per tile of 64 tokens.  Warp-per-token top-k (ties to the
//                       lower expert index), routing weights, a block histogram over the
//                       experts with deterministic in-tile ranks (ballot masks, no
//                       order-dependent atomics), and a decoupled-lookback scan of the
//                       per-tile expert-count vectors that gives every tile its starting
//                       rank inside each expert (32 predecessors inspected per step).
//                       The tile that finishes last turns the totals into counts,
//                       offsets and the padded tile prefix.
//   scatter_kernel      pos = offsets[e] + rank; perm[pos] = a; inv[a] = pos.
// The result is the stable counting sort: inside an expert, ascending token.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kRouteTile = 64;     // tokens per CTA
constexpr int kRouteThreads = 256;
constexpr int kMaxE = 1024;
constexpr int kMaxK = 32;

enum : uint32_t { FLAG_NONE = 0, FLAG_AGG = 1, FLAG_PREFIX = 2 };

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <int NPL>
__global__ void __launch_bounds__(kRouteThreads) route_rank_kernel(RouteParams P) {
  __shared__ int s_idx[kRouteTile][kMaxK];
  __shared__ int s_rank[kRouteTile][kMaxK];
  __shared__ uint32_t s_mask[2][kMaxE];
  __shared__ int s_cnt[2][kMaxE];  // per 32-token group count, then exclusive group prefix
  __shared__ int s_excl[kMaxE];    // exclusive prefix over preceding tiles
  __shared__ int s_part[kRouteThreads];
  __shared__ int s_bid, s_flag, s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = P.E, k = P.k;

  if (tid == 0) s_bid = static_cast<int>(atomicAdd(P.tile_counter, 1u));
  for (int e = tid; e < E; e += kRouteThreads) {
    s_mask[0][e] = s_mask[1][e] = 0u;
    s_cnt[0][e] = s_cnt[1][e] = 0;
  }
  __syncthreads();
  const int b = s_bid;
  const int64_t t0 = static_cast<int64_t>(b) * kRouteTile;

  // ---- 1. top-k per token: each warp selects for kTPW tokens at once (independent
  //         shuffle chains interleave), k rounds of a warp-wide (value, -index) argmax ----
  constexpr int kTPW = 4;
  for (int tl0 = warp * kTPW; tl0 < kRouteTile; tl0 += (kRouteThreads / 32) * kTPW) {
    float v[kTPW][NPL];
    uint32_t removed[kTPW];
    float sel_v[kTPW];
    int sel_e[kTPW];
#pragma unroll
    for (int u = 0; u < kTPW; ++u) {
      const int64_t t = t0 + tl0 + u;
      const bool tv = t < P.T;
      const float* row = P.logits + (tv ? t : 0) * E;
      removed[u] = 0;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        // A NaN logit ranks as -inf: the comparisons below then always find k valid
        // experts (ties, -inf included, go to the lower index).
        const float lv = (tv && e < E) ? row[e] : -INFINITY;
        v[u][i] = lv != lv ? -INFINITY : lv;
        if (e >= E) removed[u] |= 1u << i;
      }
      sel_v[u] = 0.f;
      sel_e[u] = 0;
    }
    for (int j = 0; j < k; ++j) {
      float bv[kTPW];
      int be[kTPW];
#pragma unroll
      for (int u = 0; u < kTPW; ++u) {
        bv[u] = -INFINITY;
        be[u] = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          const int e = lane + 32 * i;
          if (!((removed[u] >> i) & 1u) && (v[u][i] > bv[u] || (v[u][i] == bv[u] && e < be[u]))) {
            bv[u] = v[u][i];
            be[u] = e;
          }
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) {
#pragma unroll
        for (int u = 0; u < kTPW; ++u) {
          const float ov = __shfl_xor_sync(kFull, bv[u], off);
          const int oe = __shfl_xor_sync(kFull, be[u], off);
          if (ov > bv[u] || (ov == bv[u] && oe < be[u])) {
            bv[u] = ov;
            be[u] = oe;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kTPW; ++u) {
        if (be[u] < 0 || be[u] >= E) {  // cannot happen with finite or -inf keys; never index with it
          if (lane == 0) latch(P.status, MOE_ERR_DEVICE_BOUNDS);
          be[u] = 0;
        }
        if ((be[u] & 31) == lane) removed[u] |= 1u << (be[u] >> 5);
        if (lane == j) {
          sel_v[u] = bv[u];
          sel_e[u] = be[u];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kTPW; ++u) {
      const int tl = tl0 + u;
      const int64_t t = t0 + tl;
      float score;
      if (P.score_fn == MOE_SCORE_SOFTMAX_TOPK) {
        const float m = __shfl_sync(kFull, sel_v[u], 0);  // slot 0 holds the largest logit
        score = (lane < k) ? expf(sel_v[u] - m) : 0.f;
      } else {
        score = (lane < k) ? 1.f / (1.f + expf(-sel_v[u])) : 0.f;
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
  if (warp < kRouteTile / 32) {
    const int g = warp, tl = 32 * g + lane;
    const bool valid = t0 + tl < P.T;
    // lanes choosing the same expert in slot j are grouped first, so each expert's word
    // takes one atomic per slot instead of one per lane (hot experts are chosen by most
    // lanes of a group: per-lane atomics on one word serialise)
    for (int j = 0; j < k; ++j) {
      const int e = valid ? s_idx[tl][j] : -1 - lane;  // invalid lanes match nobody
      const uint32_t same = __match_any_sync(kFull, e);
      if (valid && (same & ((1u << lane) - 1u)) == 0u) atomicOr(&s_mask[g][e], same);
    }
    __syncwarp();
    if (valid) {
      const uint32_t below = (1u << lane) - 1u;
      for (int j = 0; j < k; ++j) {
        const int e = s_idx[tl][j];
        const uint32_t m = s_mask[g][e];
        s_rank[tl][j] = __popc(m & below);
        if ((m & below) == 0u) s_cnt[g][e] = __popc(m);
      }
    }
  }
  __syncthreads();

  // ---- 3. tile histogram, group prefix ----------------------------------------------
  constexpr int kPer = kMaxE / kRouteThreads;
  int hist[kPer], excl[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int e = tid + kRouteThreads * r;
    hist[r] = 0;
    excl[r] = 0;
    if (e < E) {
      const int c0 = s_cnt[0][e], c1 = s_cnt[1][e];
      s_cnt[0][e] = 0;
      s_cnt[1][e] = c0;
      hist[r] = c0 + c1;
    }
  }

  // ---- 4. decoupled lookback over the tiles' count vectors --------------------------
  const int64_t rowE = static_cast<int64_t>(E);
  if (b == 0) {
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int e = tid + kRouteThreads * r;
      if (e < E) P.incl[e] = hist[r];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release(&P.flags[0], FLAG_PREFIX);
  } else {
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int e = tid + kRouteThreads * r;
      if (e < E) P.agg[b * rowE + e] = hist[r];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release(&P.flags[b], FLAG_AGG);
    // Windowed lookback: warp 0 reads the flags of the next 32 predecessors at once; the
    // block adds their aggregates down to (and including) the nearest inclusive prefix.
    int hi = b - 1;  // highest predecessor not yet added
    bool failed = false;
    while (hi >= 0) {
      if (warp == 0) {
        const int p = hi - lane;
        uint32_t f = FLAG_NONE;
        if (p >= 0) {
          f = ld_acquire(&P.flags[p]);
          if (f == FLAG_NONE) {
            const uint64_t start = globaltimer_ns();
            while ((f = ld_acquire(&P.flags[p])) == FLAG_NONE) {
              if (globaltimer_ns() - start > kWaitLimitNs) break;
              __nanosleep(32);
            }
          }
        }
        const uint32_t pref = __ballot_sync(kFull, p >= 0 && f == FLAG_PREFIX);
        const uint32_t present = __ballot_sync(kFull, p >= 0);
        const uint32_t missing = __ballot_sync(kFull, p >= 0 && f == FLAG_NONE);
        if (lane == 0) {
          s_flag = missing ? -1 : (pref ? __ffs(pref) : -__popc(present) - 2);
        }
      }
      __syncthreads();
      const int code = s_flag;
      if (code == -1) {  // a bounded wait ran out: latch, publish garbage, carry on
        failed = true;
        break;
      }
      const bool found = code > 0;
      const int n = found ? code : -(code + 2);  // predecessors hi, hi-1, ..., hi-n+1
      // The window's count vectors are read with all loads in flight at once (16 per
      // batch): summing them one L2 round trip at a time made this loop the routing
      // kernel's critical path.
      for (int i0 = 0; i0 < n; i0 += 16) {
#pragma unroll
        for (int r = 0; r < kPer; ++r) {
          const int e = tid + kRouteThreads * r;
          if (e < E) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const int i = i0 + u;
              const int* src = (found && i == n - 1 ? P.incl : P.agg) + (hi - i) * rowE;
              v[u] = i < n ? __ldcg(src + e) : 0;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) excl[r] += v[u];
          }
        }
      }
      __syncthreads();  // s_flag is rewritten in the next window
      if (found) break;
      hi -= n;
    }
    if (failed && tid == 0) latch(P.status, MOE_ERR_DEVICE_TIMEOUT);
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int e = tid + kRouteThreads * r;
      if (e < E) P.incl[b * rowE + e] = excl[r] + hist[r];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release(&P.flags[b], FLAG_PREFIX);
  }
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int e = tid + kRouteThreads * r;
    if (e < E) s_excl[e] = excl[r];
  }
  __syncthreads();

  // ---- 5. rank of every assignment inside its expert --------------------------------
  for (int i = tid; i < kRouteTile * k; i += kRouteThreads) {
    const int tl = i / k, j = i - tl * k;
    const int64_t t = t0 + tl;
    if (t >= P.T) continue;
    const int e = s_idx[tl][j];
    P.rank[t * k + j] = s_excl[e] + s_cnt[tl >> 5][e] + s_rank[tl][j];
  }

  // ---- 6. the last tile to finish writes counts, offsets and the tile prefix ---------
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(P.done_counter, 1u) == static_cast<uint32_t>(P.num_tiles - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int* tot = P.incl + static_cast<int64_t>(P.num_tiles - 1) * rowE;
  int c[kPer], m[kPer], csum = 0, msum = 0;
#pragma unroll
  for (int r = 0; r < kPer; ++r) {  // thread owns experts kPer*tid .. kPer*tid+kPer-1
    const int e = kPer * tid + r;
    c[r] = (e < E) ? __ldcg(tot + e) : 0;
    m[r] = (c[r] + 127) >> 7;
    csum += c[r];
    msum += m[r];
  }
  // block exclusive scan of (csum, msum) packed as two passes over s_part
  int cex = 0, mex = 0;
  for (int pass = 0; pass < 2; ++pass) {
    s_part[tid] = pass == 0 ? csum : msum;
    __syncthreads();
    for (int off = 1; off < kRouteThreads; off <<= 1) {
      const int add = tid >= off ? s_part[tid - off] : 0;
      __syncthreads();
      s_part[tid] += add;
      __syncthreads();
    }
    const int inc = s_part[tid];
    (pass == 0 ? cex : mex) = inc - (pass == 0 ? csum : msum);
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int e = kPer * tid + r;
    if (e < E) {
      P.counts[e] = c[r];
      P.offsets[e] = cex;
      P.mtile_prefix[e] = mex;
      if (P.pad_offsets) P.pad_offsets[e] = mex * 128;
    }
    cex += c[r];
    mex += m[r];
  }
  if (tid == kRouteThreads - 1) {
    P.offsets[E] = cex;
    P.mtile_prefix[E] = mex;
    if (P.pad_offsets) P.pad_offsets[E] = mex * 128;
  }
}

__global__ void scatter_kernel(const int32_t* __restrict__ topk_idx,
                               const int32_t* __restrict__ rank,
                               const int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                               int32_t* __restrict__ inv, int64_t A, int E, int32_t* status) {
  for (int64_t a = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; a < A;
       a += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = topk_idx[a];
    if (e < 0 || e >= E) {
      latch(status, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    const int64_t pos = static_cast<int64_t>(offsets[e]) + rank[a];
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
  scatter_kernel<<<sgrid, 256, 0, stream>>>(P.topk_idx, P.rank, P.offsets, perm, inv, A, P.E,
                                            P.status);
  return cudaGetLastError();
}

int route_num_tiles(int64_t T) { return static_cast<int>((T + kRouteTile - 1) / kRouteTile); }

}  // namespace moe
