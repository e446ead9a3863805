// S4 / S5 / S7: persistent grouped GEMM on the 5th-generation tensor cores with MXFP8
// block scaling (tcgen05.mma kind::mxf8f6f4, E8M0 scales, fp32 accumulation in TMEM).
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72":
//   §01 -- the grouped GEMM needs each expert's tokens contiguous, else it reorders again;
//   §02 -- expert FFN = grouped GEMM with SwiGLU; MXFP8 activations fused into the grouped
//          GEMM and SwiGLU; work per expert is cut into tiles handed to the SMs in waves.
//
// Problem: for group g (an expert) with rows [128*prefix[g], 128*prefix[g+1]) of A,
//   D[r, n] = sum_k A[r, k] * B[g*N + n, k]      (A, B K-major E4M3, UMMA scales)
// Tile 128 x 256 x 128 (rows x cols x K per stage), 4-stage TMA pipeline.
//
// Warp roles (320 threads, one CTA per SM, persistent over a static round-robin tile list
// that is derived on the device from the per-expert tile prefix -- no host round trip):
//   warp 0      TMA producer: A tile 16 KB + B tile 32 KB via cp.async.bulk.tensor (128-byte
//               swizzle), scale chunks (512 B for A, 2 x 512 B for B) via cp.async.bulk.
//   warp 1      TMEM owner; lane 0 issues tcgen05.cp (scales -> TMEM) and tcgen05.mma.
//   warps 2..9  epilogue: TMEM -> registers (tcgen05.ld), release the accumulator at once,
//               then the mode's math and stores.  Warp w reads TMEM lanes 32*(w%4).. and
//               column half (w-2)/4.
// Tile order inside an expert is N-major (all M tiles of one weight tile back to back) so
// that a weight tile is read from HBM once and re-read by the neighbouring CTAs from L2.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int BM = 128, BN = 256, BK = 128, STAGES = 4;
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;
constexpr uint32_t kSfCol = 256;  // + 16 * stage: A scales 4 columns, B scales 8 columns
constexpr uint32_t kABytes = BM * BK, kBBytes = BN * BK;
constexpr uint32_t kTxBytes = kABytes + kBBytes + 512 + 1024;
constexpr int kMaxG = 1024;

struct GemmSmem {
  uint8_t a[STAGES][kABytes];
  uint8_t b[STAGES][kBBytes];
  uint8_t sfa[STAGES][512];
  uint8_t sfb[STAGES][1024];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full;
  uint64_t tmem_empty;
  uint32_t tmem_base;
  int abort_flag;
  int prefix[kMaxG + 1];
  int valid[kMaxG];
};
constexpr size_t kGemmSmemBytes = sizeof(GemmSmem) + 1024;

struct TileInfo {
  int g, i, j;
  int64_t a_row0, b_row0;
};

__device__ __forceinline__ TileInfo decode_tile(int tile, const int* prefix, int G, int NT, int N) {
  int lo = 0, hi = G;  // prefix[lo]*NT <= tile < prefix[hi]*NT
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] * NT <= tile) lo = mid; else hi = mid;
  }
  TileInfo t;
  t.g = lo;
  const int mt = prefix[lo + 1] - prefix[lo];
  const int local = tile - prefix[lo] * NT;
  t.j = local / mt;
  t.i = local - t.j * mt;
  t.a_row0 = static_cast<int64_t>(prefix[lo] + t.i) * BM;
  t.b_row0 = static_cast<int64_t>(lo) * N + static_cast<int64_t>(t.j) * BN;
  return t;
}

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  GemmSmem& S = *reinterpret_cast<GemmSmem*>(smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = P.G, N = P.N, NT = P.N / BN;
  const int nk = P.K / BK;
  const int64_t kgroups = P.K / 128;

  for (int i = tid; i <= G; i += kGemmThreads) S.prefix[i] = P.mtile_prefix[i];
  for (int i = tid; i < G; i += kGemmThreads)
    S.valid[i] = P.rows_valid ? P.rows_valid[i] : 0x7fffffff;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&S.full[s]), 1);
      mbar_init(smem_u32(&S.empty[s]), 1);
    }
    mbar_init(smem_u32(&S.tmem_full), 1);
    mbar_init(smem_u32(&S.tmem_empty), kEpiWarps);
    S.abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;
  const int total = S.prefix[G] * NT;
  volatile int* abort_flag = &S.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        const TileInfo ti = decode_tile(tile, S.prefix, G, NT, N);
        const int64_t rbA = ti.a_row0 >> 7, rbB = ti.b_row0 >> 7;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(&S.empty[stage]), phase ^ 1u, abort_flag, P.status)) break;
          const uint32_t fb = smem_u32(&S.full[stage]);
          mbar_arrive_expect_tx(fb, kTxBytes);
          tma_load_2d(smem_u32(S.a[stage]), &tmA, fb, kb * BK, static_cast<int32_t>(ti.a_row0));
          tma_load_2d(smem_u32(S.b[stage]), &tmB, fb, kb * BK, static_cast<int32_t>(ti.b_row0));
          bulk_load(smem_u32(S.sfa[stage]), P.sfa + ((rbA * kgroups + kb) << 9), 512, fb);
          bulk_load(smem_u32(S.sfb[stage]), P.sfb + ((rbB * kgroups + kb) << 9), 512, fb);
          bulk_load(smem_u32(S.sfb[stage]) + 512, P.sfb + (((rbB + 1) * kgroups + kb) << 9), 512,
                    fb);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      const uint32_t idesc = idesc_mxf8_e4m3(BM, BN);
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        if (!mbar_wait(smem_u32(&S.tmem_empty), acc_phase ^ 1u, abort_flag, P.status)) break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(&S.full[stage]), phase, abort_flag, P.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf = tbase + kSfCol + 16u * stage;
          tmem_cp_scales(sf, sdesc_scale_chunk(smem_u32(S.sfa[stage])));
          tmem_cp_scales(sf + 4, sdesc_scale_chunk(smem_u32(S.sfb[stage])));
          tmem_cp_scales(sf + 8, sdesc_scale_chunk(smem_u32(S.sfb[stage]) + 512));
          const uint32_t a0 = smem_u32(S.a[stage]), b0 = smem_u32(S.b[stage]);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint32_t id = idesc | (static_cast<uint32_t>(kk) << 29) |
                                (static_cast<uint32_t>(kk) << 4);
            mma_mxf8(tbase + kAccCol, sdesc_k_sw128(a0 + 32u * kk), sdesc_k_sw128(b0 + 32u * kk),
                     id, (kb | kk) != 0 ? 1u : 0u, sf, sf + 4);
          }
          mma_commit(smem_u32(&S.empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&S.tmem_full));
        acc_phase ^= 1u;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;   // column half
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileInfo ti = decode_tile(tile, S.prefix, G, NT, N);
      if (!mbar_wait(smem_u32(&S.tmem_full), acc_phase, abort_flag, P.status)) break;
      tc_fence_after();
      const uint32_t taddr = tbase + kAccCol + (static_cast<uint32_t>(32 * q) << 16);
      float v0[32], v1[32], v2[32], v3[32];
      if (MODE == GEMM_GATEUP_SWIGLU) {
        tmem_ld32(taddr + 64 * h, v0);         // gate features 64h .. 64h+31
        tmem_ld32(taddr + 64 * h + 32, v1);    // gate features 64h+32 .. 64h+63
        tmem_ld32(taddr + 128 + 64 * h, v2);   // up, same features
        tmem_ld32(taddr + 128 + 64 * h + 32, v3);
      } else {
        tmem_ld32(taddr + 128 * h, v0);
        tmem_ld32(taddr + 128 * h + 32, v1);
        tmem_ld32(taddr + 128 * h + 64, v2);
        tmem_ld32(taddr + 128 * h + 96, v3);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.tmem_empty));
      acc_phase ^= 1u;

      const int m = 32 * q + lane;
      if (ti.i * BM + m >= S.valid[ti.g]) continue;
      const int64_t row = ti.a_row0 + m;
      if (MODE == GEMM_GATEUP_SWIGLU) {
        const int f = P.f;
        const int fb = BN / 2 * ti.j + 64 * h;  // first feature of this thread's 64
        if (P.gu) {
          uint4* gdst = reinterpret_cast<uint4*>(P.gu + row * 2 * f + fb);
          uint4* udst = reinterpret_cast<uint4*>(P.gu + row * 2 * f + f + fb);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float* g = c < 4 ? v0 + 8 * c : v1 + 8 * (c - 4);
            const float* u = c < 4 ? v2 + 8 * c : v3 + 8 * (c - 4);
            gdst[c] = make_uint4(f32_to_bf16_bits(g[0]) | (f32_to_bf16_bits(g[1]) << 16),
                                 f32_to_bf16_bits(g[2]) | (f32_to_bf16_bits(g[3]) << 16),
                                 f32_to_bf16_bits(g[4]) | (f32_to_bf16_bits(g[5]) << 16),
                                 f32_to_bf16_bits(g[6]) | (f32_to_bf16_bits(g[7]) << 16));
            udst[c] = make_uint4(f32_to_bf16_bits(u[0]) | (f32_to_bf16_bits(u[1]) << 16),
                                 f32_to_bf16_bits(u[2]) | (f32_to_bf16_bits(u[3]) << 16),
                                 f32_to_bf16_bits(u[4]) | (f32_to_bf16_bits(u[5]) << 16),
                                 f32_to_bf16_bits(u[6]) | (f32_to_bf16_bits(u[7]) << 16));
          }
        }
        // h = silu(g) * u, in place over the gate registers
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          v0[c] = v0[c] / (1.f + expf(-v0[c])) * v2[c];
          v1[c] = v1[c] / (1.f + expf(-v1[c])) * v3[c];
        }
        uint32_t q0[8], q1[8];
        const uint32_t s0 = mx_quant_block32(v0, q0);
        const uint32_t s1 = mx_quant_block32(v1, q1);
        uint4* hdst = reinterpret_cast<uint4*>(P.hq + row * f + fb);
        hdst[0] = make_uint4(q0[0], q0[1], q0[2], q0[3]);
        hdst[1] = make_uint4(q0[4], q0[5], q0[6], q0[7]);
        hdst[2] = make_uint4(q1[0], q1[1], q1[2], q1[3]);
        hdst[3] = make_uint4(q1[4], q1[5], q1[6], q1[7]);
        *reinterpret_cast<uint16_t*>(P.hs + umma_scale_offset(row, fb >> 5, f >> 7)) =
            static_cast<uint16_t>(s0 | (s1 << 8));
      } else {
        float4* dst = reinterpret_cast<float4*>(P.out_f32 + row * P.ld_out +
                                                static_cast<int64_t>(ti.j) * BN + 128 * h);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          dst[c] = make_float4(v0[4 * c], v0[4 * c + 1], v0[4 * c + 2], v0[4 * c + 3]);
          dst[8 + c] = make_float4(v1[4 * c], v1[4 * c + 1], v1[4 * c + 2], v1[4 * c + 3]);
          dst[16 + c] = make_float4(v2[4 * c], v2[4 * c + 1], v2[4 * c + 2], v2[4 * c + 3]);
          dst[24 + c] = make_float4(v3[4 * c], v3[4 * c + 1], v3[4 * c + 2], v3[4 * c + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

template <int MODE>
static cudaError_t launch_mode(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& P,
                               int num_sms, cudaStream_t stream) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kGemmSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  grouped_gemm_kernel<MODE><<<num_sms, kGemmThreads, kGemmSmemBytes, stream>>>(tmA, tmB, P);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(int mode, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const GemmParams& P, int num_sms, cudaStream_t stream) {
  switch (mode) {
    case GEMM_STORE_F32:
      return launch_mode<GEMM_STORE_F32>(tmA, tmB, P, num_sms, stream);
    case GEMM_GATEUP_SWIGLU:
      return launch_mode<GEMM_GATEUP_SWIGLU>(tmA, tmB, P, num_sms, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace moe
