// MXFP8 quantisation kernels, the pull-dispatch gather and the push combine.
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72":
//   §02 -- pull dispatch: the consumer fetches the rows it needs by source and offset and
//          lays them out by expert; MXFP8 activations travel through dispatch: each token
//          is quantised once (the copy stays in L2) and every expert row pulls its token's
//          codes, so the bf16 rows are read from HBM once instead of k times;
//   §02/§03 -- push combine returns each expert result to its token's slot, followed by
//          the final weighted merge.
// All kernels here are HBM-bound: 16-byte vector loads, one warp per row, grids sized in
// multiples of the SM count.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kMaxE = 1024;

__device__ __forceinline__ void unpack_bf16x8(const uint4& r, float (&v)[8]) {
  v[0] = bf16_bits_to_f32(r.x & 0xFFFFu);
  v[1] = bf16_bits_to_f32(r.x >> 16);
  v[2] = bf16_bits_to_f32(r.y & 0xFFFFu);
  v[3] = bf16_bits_to_f32(r.y >> 16);
  v[4] = bf16_bits_to_f32(r.z & 0xFFFFu);
  v[5] = bf16_bits_to_f32(r.z >> 16);
  v[6] = bf16_bits_to_f32(r.w & 0xFFFFu);
  v[7] = bf16_bits_to_f32(r.w >> 16);
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// One warp quantises K bf16 values of one row (K % 32 == 0).  Lane l handles 8 values per
// 256-column step; four lanes share a 32-element block.  kUnroll steps are loaded before
// any of them is converted, so each lane keeps several 16-byte loads in flight.  Scales go
// to the canonical layout (row stride K/32, first block kb0) or to the UMMA layout
// (kgroups = K_total/128; kb0 % 4 == 0 required).
constexpr int kUnroll = 4;

__device__ __forceinline__ void quant_step(const uint4& raw, bool in, int64_t col,
                                           uint8_t* __restrict__ dst,
                                           uint8_t* __restrict__ scales, int64_t row, int64_t kb0,
                                           int layout, int64_t canon_stride, int64_t kgroups,
                                           int lane) {
  float v[8];
  unpack_bf16x8(raw, v);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
  const int s = mx_scale_exp(amax);
  const float inv = mx_inv_scale(s);
  uint2 packed;
  packed.x = pack_e4m3x4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
  packed.y = pack_e4m3x4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
  if (in) *reinterpret_cast<uint2*>(dst + col) = packed;
  const uint32_t sb = static_cast<uint32_t>(s + 127);
  const int64_t kb = kb0 + (col >> 5);
  if (layout == 0) {
    if (in && (lane & 3) == 0) scales[row * canon_stride + kb] = static_cast<uint8_t>(sb);
  } else {
    const uint32_t b1 = __shfl_down_sync(kFull, sb, 4);
    const uint32_t b2 = __shfl_down_sync(kFull, sb, 8);
    const uint32_t b3 = __shfl_down_sync(kFull, sb, 12);
    if (in && (lane & 15) == 0)
      *reinterpret_cast<uint32_t*>(scales + umma_scale_offset(row, kb, kgroups)) =
          sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
  }
}

__device__ __forceinline__ void warp_quant_row(const uint16_t* __restrict__ src, int64_t K,
                                               uint8_t* __restrict__ dst,
                                               uint8_t* __restrict__ scales, int64_t row,
                                               int64_t kb0, int layout, int64_t canon_stride,
                                               int64_t kgroups, int lane) {
  for (int64_t c0 = 0; c0 < K; c0 += 256 * kUnroll) {
    uint4 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t col = c0 + 256 * u + lane * 8;
      raw[u] = col < K ? ld_nc_v4(src + col) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t col = c0 + 256 * u + lane * 8;
      if (c0 + 256 * u < K)  // warp-uniform: whole 256-column step inside or outside
        quant_step(raw[u], col < K, col, dst, scales, row, kb0, layout, canon_stride, kgroups,
                   lane);
    }
  }
}

__global__ void __launch_bounds__(256) quant_rows_kernel(QuantRowsParams P) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t kb0 = P.dst_col0 >> 5;
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
       r < P.rows; r += warps) {
    warp_quant_row(P.src + r * P.src_ld, P.K, P.dst + r * P.dst_ld + P.dst_col0, P.scales, r,
                   kb0, P.layout, P.K >> 5, P.kgroups, lane);
  }
}

cudaError_t launch_quant_rows(const QuantRowsParams& P, int num_sms, cudaStream_t stream) {
  if (P.rows <= 0) return cudaSuccess;
  const int64_t blocks = (P.rows + 7) / 8;
  const int grid = static_cast<int>(blocks < 16LL * num_sms ? blocks : 16LL * num_sms);
  quant_rows_kernel<<<grid, 256, 0, stream>>>(P);
  return cudaGetLastError();
}

// Weights: thread per (group, 32-block along K, column); columns fastest so that the
// strided column reads of a warp are coalesced.
__global__ void __launch_bounds__(256) quant_cols_kernel(QuantColsParams P) {
  const int64_t nkb = P.K >> 5;
  const int64_t total = static_cast<int64_t>(P.G) * nkb * P.ncols;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx % P.ncols;
    const int64_t rest = idx / P.ncols;
    const int64_t kb = rest % nkb;
    const int64_t g = rest / nkb;
    const uint16_t* col = P.src + (g * P.K + kb * 32) * P.ncols + n;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = bf16_bits_to_f32(col[static_cast<int64_t>(i) * P.ncols]);
    uint32_t q[8];
    const uint32_t sb = mx_quant_block32(v, q);
    int64_t row;
    if (P.map_mode == 0)
      row = g * P.ncols + n;
    else
      row = g * 2 * P.ncols + (n >> 7) * 256 + P.interleave_half * 128 + (n & 127);
    uint4* dst = reinterpret_cast<uint4*>(P.dst + row * P.K + kb * 32);
    dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
    dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
    P.scales[umma_scale_offset(row, kb, P.kgroups)] = static_cast<uint8_t>(sb);
  }
}

cudaError_t launch_quant_cols(const QuantColsParams& P, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(P.G) * (P.K >> 5) * P.ncols;
  if (total <= 0) return cudaSuccess;
  const int64_t blocks = (total + 255) / 256;
  const int grid = static_cast<int>(blocks < 65536 ? blocks : 65536);
  quant_cols_kernel<<<grid, 256, 0, stream>>>(P);
  return cudaGetLastError();
}

// Weighted combine, one CTA per token: out[t] = sum_j w[t,j] * Y[row of assignment (t, j)] (j
// ascending, fp32; Y read as scaled fp16, each value times its block scale), rounded to
// bf16.  With unit weights this is the backward's push reverse-dispatch, dX[t] = sum_j
// dXa[row of (t, j)].  The CTA reads each of the token's k rows as one contiguous stretch
// (thread i takes 16-byte chunks i, i + 256, ...), so every DRAM access is a long run of a
// single row rather than k short pieces of different rows.
constexpr int kCombineThreads = 256;
constexpr int kCombineChunks = 2;  // 16-byte chunks per thread per column block (64 registers: 4 CTAs per SM)

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineParams P) {
  __shared__ int s_off[kMaxE + 1];
  __shared__ int s_mt[kMaxE + 1];
  __shared__ int64_t s_row[32];
  __shared__ float s_w[32];
  __shared__ int s_bad;
  if (!P.direct_rows) {
    for (int i = threadIdx.x; i <= P.E; i += blockDim.x) {
      s_off[i] = P.offsets[i];
      s_mt[i] = P.mtile_prefix[i] >> P.prefix_shift;
    }
  }
  __syncthreads();
  const int tid = threadIdx.x;
  const int k = P.k;
  const int64_t R = P.direct_rows ? P.T * k : static_cast<int64_t>(s_mt[P.E]) * 128;
  const int64_t nsb = P.d >> 5;  // scale bytes per row
  for (int64_t t = blockIdx.x; t < P.T; t += gridDim.x) {
    if (tid == 0) s_bad = 0;
    __syncthreads();
    if (tid < k) {
      const int64_t a = t * k + tid;
      int64_t row = -1;
      if (P.direct_rows) {
        row = a;
      } else {
        const int e = P.topk_idx[a];
        if (e >= 0 && e < P.E) row = static_cast<int64_t>(s_mt[e]) * 128 + (P.inv[a] - s_off[e]);
      }
      if (row < 0 || row >= R) {
        s_bad = 1;
        row = 0;
      }
      s_row[tid] = row;
      s_w[tid] = P.topk_w ? P.topk_w[a] : 1.f;
    }
    __syncthreads();
    if (s_bad) {
      if (tid == 0) latch(P.status, MOE_ERR_DEVICE_BOUNDS);
      __syncthreads();  // s_row / s_bad are rewritten for the next token
      continue;
    }
    for (int64_t cb = 0; cb < P.d; cb += 8 * kCombineThreads * kCombineChunks) {
      float acc[kCombineChunks][8];
#pragma unroll
      for (int c = 0; c < kCombineChunks; ++c)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[c][i] = 0.f;
#pragma unroll 2  // two rows' loads in flight
      for (int j = 0; j < k; ++j) {  // j ascending: the sum order is fixed
        const int64_t row = s_row[j];
        const float w = s_w[j];
        const uint16_t* yr = P.y + row * P.d;
        const uint8_t* sr = P.ys + row * nsb;
        uint4 q[kCombineChunks];
        float ws[kCombineChunks];
#pragma unroll
        for (int c = 0; c < kCombineChunks; ++c) {
          const int64_t col = cb + 8 * (tid + kCombineThreads * c);
          if (col < P.d) {
            q[c] = __ldg(reinterpret_cast<const uint4*>(yr + col));
            ws[c] = w * f16s_scale_value(__ldg(sr + (col >> 5)));
          }
        }
#pragma unroll
        for (int c = 0; c < kCombineChunks; ++c) {
          const int64_t col = cb + 8 * (tid + kCombineThreads * c);
          if (col < P.d) {
            const uint32_t wv[4] = {q[c].x, q[c].y, q[c].z, q[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[c][2 * i] += ws[c] * f16_bits_to_f32(wv[i]);
              acc[c][2 * i + 1] += ws[c] * f16_bits_to_f32(wv[i] >> 16);
            }
          }
        }
      }
#pragma unroll
      for (int c = 0; c < kCombineChunks; ++c) {
        const int64_t col = cb + 8 * (tid + kCombineThreads * c);
        if (col < P.d) {
          uint4 o;
          o.x = pack_bf16x2(acc[c][0], acc[c][1]);
          o.y = pack_bf16x2(acc[c][2], acc[c][3]);
          o.z = pack_bf16x2(acc[c][4], acc[c][5]);
          o.w = pack_bf16x2(acc[c][6], acc[c][7]);
          *reinterpret_cast<uint4*>(P.out + t * P.d + col) = o;
        }
      }
    }
    __syncthreads();  // s_row / s_w are rewritten for the next token
  }
}

cudaError_t launch_combine(const CombineParams& P, int num_sms, cudaStream_t stream) {
  if (P.T <= 0) return cudaSuccess;
  const int grid = static_cast<int>(P.T < 8LL * num_sms ? P.T : 8LL * num_sms);
  combine_kernel<<<grid, kCombineThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

// Dispatch, second half: the pull gather.  Each expert row fetches the MX codes and scales of its
// token by index from the per-token quantised copy (x quantised once per token, small
// enough to stay in L2) and writes them to its padded position: the codes with bulk copies
// through shared memory (the copy engine moves the bytes; one thread per warp issues
// them), the scales re-laid into the UMMA layout one 4-byte K-group word at a time.
// The layer's BF16 variant pulls the bf16 rows of x the same way (no scales).
constexpr int kGatherChunk = 64;    // rows per CTA step; readiness is published per chunk
constexpr int kGatherWarps = 8;
constexpr int kGatherPiece = 4096;  // bytes per bulk copy; a row is one or more pieces

// Per warp two piece buffers: the bulk load of the next piece runs while the current one is
// stored (a 7 KB MX row is two pieces, a bf16 row of the BF16 variant four).
struct GatherSmem {
  uint8_t buf[kGatherWarps][2][kGatherPiece];
  uint64_t bar[kGatherWarps][2];
  int64_t rt[kGatherWarps][kGatherChunk / kGatherWarps];  // each row's token (-1: none)
  int64_t rp[kGatherWarps][kGatherChunk / kGatherWarps];  // and padded position
  int s_off[kMaxE + 1];
  int s_mt[kMaxE + 1];
  int s_b[kGatherChunk];  // minibatch of each row of the chunk (-1: none)
  int abort_flag;
};
constexpr size_t kGatherSmemBytes = sizeof(GatherSmem) + 128;

__global__ void __launch_bounds__(kGatherWarps * 32, 3) gather_rows_kernel(GatherParams P) {
  extern __shared__ uint8_t g_raw[];
  GatherSmem& S = *reinterpret_cast<GatherSmem*>(
      g_raw + ((128u - (smem_u32(g_raw) & 127u)) & 127u));
  // the consumer GEMM (launched as a programmatic dependent) may start now: it waits for
  // each minibatch of rows through the readiness counters, not for this grid to finish
  launch_dependents();
  for (int i = threadIdx.x; i <= P.E; i += blockDim.x) {
    S.s_off[i] = P.offsets[i];
    S.s_mt[i] = P.mtile_prefix[i] >> P.prefix_shift;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) S.abort_flag = 0;
  if (lane == 0) {
    mbar_init(smem_u32(&S.bar[warp][0]), 1);
    mbar_init(smem_u32(&S.bar[warp][1]), 1);
    fence_barrier_init();
  }
  __syncthreads();
  const int64_t A = P.T * P.k;
  const int64_t R = static_cast<int64_t>(S.s_mt[P.E]) * 128;
  const int d = P.d;
  const int64_t kg = d >> 7;
  const int64_t rb = P.row_bytes;
  const int64_t nchunks = (A + kGatherChunk - 1) / kGatherChunk;
  uint32_t ph = 0;  // lane 0: parity of each buffer's next load
  // Chunks of consecutive positions in expert order, one per CTA step, so the rows of the
  // first experts (the ones the GEMM starts with) are published first.
  for (int64_t chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    // The warp's rows warp, warp + 8, ... of the chunk: lane j < 8 resolves row j's
    // expert (binary search), token and padded position at once.
    int64_t my_t = -1, my_p = 0;  // -1: no row (past A, or a failed bounds check)
    if (lane < kGatherChunk / kGatherWarps) {
      const int64_t q = chunk * kGatherChunk + warp + kGatherWarps * lane;
      if (q < A) {
        int lo = 0, hi = P.E;  // s_off[lo] <= q < s_off[hi]
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (S.s_off[mid] <= q) lo = mid; else hi = mid;
        }
        const int a = P.perm[q];
        const int64_t t = a / P.k;
        const int64_t p = static_cast<int64_t>(S.s_mt[lo]) * 128 + (q - S.s_off[lo]);
        if (a < 0 || t >= P.T || p >= R) {
          latch(P.status, MOE_ERR_DEVICE_BOUNDS);
        } else {
          my_t = t;
          my_p = p;
        }
      }
    }
    if (lane < kGatherChunk / kGatherWarps) {
      S.rt[warp][lane] = my_t;
      S.rp[warp][lane] = my_p;
    }
    __syncwarp();
    const int64_t* tj = S.rt[warp];
    const int64_t* pj = S.rp[warp];
    // scale words (UMMA layout, one 4-byte word per 128-column group) and readiness rows
#pragma unroll 1
    for (int j = 0; j < kGatherChunk / kGatherWarps; ++j) {
      const int64_t t = tj[j], p = pj[j];
      int b = -1;
      if (t >= 0) {
        if (P.s_tok) {
          const uint32_t* ssrc = reinterpret_cast<const uint32_t*>(P.s_tok + t * (d >> 5));
          for (int g = lane; g < kg; g += 32)
            *reinterpret_cast<uint32_t*>(P.s_out + umma_scale_offset(p, 4 * g, kg)) = ssrc[g];
        }
        if (P.ready) b = static_cast<int>(p / P.ready_rows);
      }
      if (P.ready && lane == 0) S.s_b[warp + kGatherWarps * j] = b;
    }
    // the codes: lane 0 copies the warp's rows piece by piece with bulk copies, through
    // shared memory (load of the next piece in flight while the current one is stored)
    if (lane == 0) {
      constexpr int NJ = kGatherChunk / kGatherWarps;
      int lj = 0, sj = 0;
      int64_t loff = 0, soff = 0;
      int lb = 0, sbf = 0;
      while (lj < NJ && tj[lj] < 0) ++lj;
      sj = lj;
      uint32_t armed = 0;
      auto issue_load = [&]() {
        const uint32_t bytes = static_cast<uint32_t>(rb - loff < kGatherPiece ? rb - loff : kGatherPiece);
        const uint32_t bar = smem_u32(&S.bar[warp][lb]);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(smem_u32(S.buf[warp][lb]), P.q_tok + tj[lj] * rb + loff, bytes, bar);
        armed |= 1u << lb;
        loff += kGatherPiece;
        if (loff >= rb) {
          loff = 0;
          do ++lj; while (lj < NJ && tj[lj] < 0);
        }
        lb ^= 1;
      };
      if (lj < NJ) issue_load();
      while (sj < NJ) {
        if (lj < NJ) {
          bulk_wait_read<0>();  // the buffer's previous store has read it
          issue_load();
        }
        if (!mbar_wait(smem_u32(&S.bar[warp][sbf]), (ph >> sbf) & 1u, &S.abort_flag, P.status))
          break;
        ph ^= 1u << sbf;
        armed &= ~(1u << sbf);
        const uint32_t bytes = static_cast<uint32_t>(rb - soff < kGatherPiece ? rb - soff : kGatherPiece);
        bulk_store(P.q_out + pj[sj] * rb + soff, smem_u32(S.buf[warp][sbf]), bytes);
        bulk_commit();
        soff += kGatherPiece;
        if (soff >= rb) {
          soff = 0;
          do ++sj; while (sj < NJ && tj[sj] < 0);
        }
        sbf ^= 1;
      }
      // after an abort, let the loads still in flight land before the buffers are reused
      for (int bq = 0; bq < 2; ++bq)
        if ((armed >> bq) & 1u) {
          mbar_drain(smem_u32(&S.bar[warp][bq]), (ph >> bq) & 1u);
          ph ^= 1u << bq;
        }
      bulk_wait_all();            // the rows are in global memory before they are published
      fence_proxy_async_global();  // (written through the async proxy)
    }
    __syncwarp();  // the warp's row table is rewritten by the next chunk
    if (P.ready) {
      // Publish the chunk: every thread's stores are made visible device-wide, then one
      // thread lowers the minibatch counters by the chunk's rows (release; the consumer
      // acquires the counter before its TMA loads read the rows).
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) {
        int cur = -1, n = 0;
        for (int r = 0; r <= kGatherChunk; ++r) {
          const int b = r < kGatherChunk ? S.s_b[r] : -1;
          if (b != cur) {
            if (cur >= 0 && cur != P.withhold) red_release_add(P.ready + cur, -n);
            cur = b;
            n = 0;
          }
          ++n;
        }
      }
      __syncthreads();  // s_b is rewritten by the next chunk
    }
  }
}

cudaError_t launch_gather_rows(const GatherParams& P, int num_sms, cudaStream_t stream) {
  const int64_t A = P.T * P.k;
  if (A <= 0) return cudaSuccess;
  const int64_t blocks = (A + kGatherChunk - 1) / kGatherChunk;
  if (P.row_bytes % 16 || P.row_bytes <= 0) return cudaErrorInvalidValue;  // bulk copies
  // All SMs, three CTAs each (the piece buffers take 72 KB of shared memory per CTA): the
  // whole grid is resident at once, so the consumer GEMM, a programmatic dependent,
  // launches at once and takes each SM as its dispatch CTAs finish.  Running the dispatch
  // on a quarter of the SMs beside the GEMM from the start was measured slower.
  const int grid = static_cast<int>(blocks < 3LL * num_sms ? blocks : 3LL * num_sms);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gather_rows_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kGatherSmemBytes));
    if (e != cudaSuccess) return e;
    // the largest shared-memory carveout on the SMs this kernel lands on, so that a GEMM
    // CTA takes an SM without a reconfiguration once the dispatch CTAs there finish
    e = cudaFuncSetAttribute(gather_rows_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             static_cast<int>(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  gather_rows_kernel<<<grid, kGatherWarps * 32, kGatherSmemBytes, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace moe

namespace moe {

// Weights of the BF16 variant: a 32 x 32 tile of W[g] ([K, ncols], x @ W convention) goes
// through shared memory so that both the reads (along ncols) and the writes (along K of
// the output rows) are coalesced.  Setup only, not part of the layer's step.
__global__ void __launch_bounds__(256) transpose_bf16_kernel(TransposeBf16Params P) {
  __shared__ uint16_t tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const int64_t tiles_n = P.ncols / 32, tiles_k = P.K / 32;
  const int64_t total = static_cast<int64_t>(P.G) * tiles_k * tiles_n;
  for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
    const int64_t tn = t % tiles_n, rest = t / tiles_n;
    const int64_t tk = rest % tiles_k, g = rest / tiles_k;
    const uint16_t* src = P.src + (g * P.K + tk * 32) * P.ncols + tn * 32;
    for (int r = ty; r < 32; r += 8) tile[r][tx] = src[static_cast<int64_t>(r) * P.ncols + tx];
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {  // output row = column n of W, its K entries
      const int64_t n = tn * 32 + r;
      const int64_t row = P.map_mode == 0
                              ? g * P.ncols + n
                              : g * 2 * P.ncols + (n >> 7) * 256 + P.interleave_half * 128 +
                                    (n & 127);
      P.dst[row * P.K + tk * 32 + tx] = tile[tx][r];
    }
    __syncthreads();
  }
}

cudaError_t launch_transpose_bf16(const TransposeBf16Params& P, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(P.G) * (P.K / 32) * (P.ncols / 32);
  if (total <= 0) return cudaSuccess;
  const int grid = static_cast<int>(total < 65536 ? total : 65536);
  transpose_bf16_kernel<<<grid, 256, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace moe
