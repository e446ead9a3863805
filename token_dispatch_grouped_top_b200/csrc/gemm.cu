// Expert FFN and its tile scheduling: persistent grouped GEMM on the 5th-generation tensor
// cores with MXFP8 block scaling (tcgen05.mma kind::mxf8f6f4, E8M0 scales, fp32
// accumulation in TMEM).
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72":
//   §01 -- the grouped GEMM needs each expert's tokens contiguous, else it reorders again;
//   §02 -- expert FFN = grouped GEMM with SwiGLU; MXFP8 activations fused into the grouped
//          GEMM and SwiGLU; work per expert is cut into tiles handed to the SMs in waves.
//
// Problem: for group g (an expert) with rows [128*prefix[g], 128*prefix[g+1]) of A,
//   D[r, n] = sum_k A[r, k] * B[g*N + n, k]      (A, B K-major E4M3, UMMA scales)
// Tile 128 x 256 x 128 (rows x cols x K per stage), 4-stage TMA pipeline (3 stages in the
// TMA-store modes, whose output staging buffers take 64 KB of shared memory).
//
// Warp roles (320 threads, one CTA per SM, persistent; tiles come from a device-side list
// derived from the per-expert tile prefix -- no host round trip -- handed out one at a
// time by an atomic counter and passed from the producer to the other roles through a
// small ring in shared memory):
//   warp 0      TMA producer: A tile 16 KB + B tile 32 KB via cp.async.bulk.tensor (128-byte
//               swizzle), scale chunks (512 B for A, 2 x 512 B for B) via cp.async.bulk.
//   warp 1      TMEM owner; lane 0 issues tcgen05.cp (scales -> TMEM) and tcgen05.mma.
//   warps 2..9  epilogue: TMEM -> registers (tcgen05.ld), release the accumulator at once,
//               then the mode's math and stores.  Warp w reads TMEM lanes 32*(w%4).. and
//               column half (w-2)/4.
// Tile order inside an expert is N-major (all M tiles of one weight tile back to back) so
// that a weight tile is read from HBM once and re-read by the neighbouring CTAs from L2.
// Experts go in index order, the order in which the dispatch writes their rows: with a
// readiness table (article §02: device-local counters signal that a minibatch of rows is
// ready; a minibatch holds two full waves of tiles) the producer loads a tile's rows as
// soon as their minibatch is complete, so this GEMM runs while the dispatch still writes
// later experts.  The weight gradients, whose tile cost grows with the expert's token
// count, hand out the experts longest first.
//
// Modes (epilogues):
//   STORE_F32_TMA  D in fp32 through shared memory and TMA stores (the down projection
//                  and both dgrad GEMMs of the backward).
//   GATEUP_SWIGLU  h = silu(g) * u on paired gate/up columns, MXFP8 requantisation of h
//                  along f (the input of the down GEMM), optional bf16 save of g and u.
//   WGRAD_BF16     weight gradients: the reduction runs over one expert's (padded) token
//                  segment, so K varies per group and M, N are fixed; bf16 output, an
//                  expert without tokens gets an all-zero gradient.
#include "common.cuh"
#include "kernels.h"
#include "tile_store.cuh"

namespace moe {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;
constexpr uint32_t kSfCol = 256;  // + 16 * stage: A scales 4 columns, B scales 8 columns
constexpr uint32_t kABytes = BM * BK, kBBytes = BN * BK;
constexpr uint32_t kTxBytes = kABytes + kBBytes + 512 + 1024;
constexpr int kMaxG = 1024;
constexpr int kRing = 8;  // tiles in flight between the producer and the other roles

// Modes that store their output with TMA need staging space: 3 pipeline stages instead of 4.
template <int MODE>
struct ModeCfg {
  // operand kind: MXFP8 with block scales, or bf16 (the layer's BF16 variant, kind::f16)
  static constexpr bool kBf16 = MODE == GEMM_GATEUP_BF16 || MODE == GEMM_STORE_F32_BF16;
  static constexpr bool kGateUp = MODE == GEMM_GATEUP_SWIGLU || MODE == GEMM_GATEUP_BF16;
  static constexpr bool kStoreF32 = MODE == GEMM_STORE_F32_TMA || MODE == GEMM_STORE_F32_BF16 ||
                                    MODE == GEMM_DGRAD_SWIGLU;
  // full tiles of the dgrad of the down projection run the SwiGLU backward in the epilogue
  static constexpr bool kSwigluBwd = MODE == GEMM_DGRAD_SWIGLU;
  static constexpr uint32_t kTx = kBf16 ? kABytes + kBBytes : kTxBytes;
  static constexpr bool kTmaStore = kStoreF32 || MODE == GEMM_WGRAD_BF16;
  static constexpr int kStages = kTmaStore ? 3 : 4;
  static constexpr int kStageBufs = kTmaStore ? 2 : 0;  // per epilogue warp, 4 KB each
  // A tile with fewer than 128 valid rows (an expert's last tile) runs with the operands
  // swapped: the two 128-row halves of the B tile are the M side of two MMAs and the
  // valid A rows, rounded up to 16, the N side -- the tensor work shrinks with the rows.
  // Measured: a gain for the fp32 / scaled-fp16 output GEMMs.  The gate/up GEMM keeps
  // full tiles: its swapped form (SwiGLU lane-local, the MX block maximum across the
  // warp, one token's codes per warp store) made the epilogue of the tail tiles the
  // bottleneck (2.26 -> 2.57 ms at the DeepSeek-V3 shape).
  static constexpr bool kSwapTail = kStoreF32;
};

template <int ST, int NSTG>
struct GemmSmemT {
  uint8_t a[ST][kABytes];
  uint8_t b[ST][kBBytes];
  // epilogue staging: 32 rows x 128 bytes, 128-byte swizzle (unused without TMA stores)
  uint8_t stg[NSTG ? kEpiWarps * NSTG : 1][NSTG ? 4096 : 16];
  uint8_t sfa[ST][512];
  uint8_t sfb[ST][1024];
  uint64_t full[ST];
  uint64_t empty[ST];
  uint64_t tmem_full;
  uint64_t tmem_empty;
  uint64_t tmem_empty_hi;  // WGRAD: columns 128..255 drained (tmem_empty: 0..127)
  uint64_t ring_full[kRing];
  uint64_t ring_empty[kRing];
  uint64_t mma_drain;      // the MMA issuer's last commit, awaited before the CTA exits
  int ring[kRing];         // tile ids (-1: no more tiles)
  uint32_t tmem_base;
  int abort_flag;
  int prefix[kMaxG + 1];
  int valid[kMaxG];
};
template <int MODE>
using SmemOf = GemmSmemT<ModeCfg<MODE>::kStages, ModeCfg<MODE>::kStageBufs>;
template <int MODE>
constexpr size_t smem_bytes() { return sizeof(SmemOf<MODE>) + 1024; }
static_assert(smem_bytes<GEMM_STORE_F32_TMA>() <= 232448, "shared memory budget (227 KB)");
static_assert(smem_bytes<GEMM_GATEUP_SWIGLU>() <= 232448, "shared memory budget (227 KB)");
static_assert(smem_bytes<GEMM_WGRAD_BF16>() <= 232448, "shared memory budget (227 KB)");

struct TileInfo {
  int g, i, j;
  int kb0, nk;  // first K block and number of K blocks
  int rows;     // valid A rows in this tile (variable-M modes), 1..128
  int64_t a_row0, b_row0;
};

// Variable-M groups (forward, dgrad): group g owns 128-row tiles [prefix[g], prefix[g+1]).
__device__ __forceinline__ TileInfo decode_tile_var_m(int tile, const int* prefix,
                                                      const int* valid, int G, int NT, int N,
                                                      int nk) {
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
  t.kb0 = 0;
  t.nk = nk;
  const int left = valid[lo] - t.i * BM;
  t.rows = left < BM ? left : BM;
  t.a_row0 = static_cast<int64_t>(prefix[lo] + t.i) * BM;
  t.b_row0 = static_cast<int64_t>(lo) * N + static_cast<int64_t>(t.j) * BN;
  return t;
}

// Variable-K groups (wgrad): group g reduces over K blocks [prefix[g], prefix[g+1]); every
// group has the same MT x NT tiles, handed out group by group in `order` (if given).
__device__ __forceinline__ TileInfo decode_tile_var_k(int tile, const int* prefix, int MT, int NT,
                                                      const int32_t* order) {
  TileInfo t;
  const int per = MT * NT;
  t.g = tile / per;
  const int slot = t.g;
  if (order) t.g = __ldg(order + slot);
  const int local = tile - slot * per;
  t.i = local / NT;
  t.j = local - t.i * NT;
  t.kb0 = prefix[t.g];
  t.nk = prefix[t.g + 1] - prefix[t.g];
  t.rows = BM;
  t.a_row0 = static_cast<int64_t>(t.i) * BM;
  t.b_row0 = static_cast<int64_t>(t.j) * BN;
  return t;
}

template <int MODE>
__device__ __forceinline__ TileInfo decode_tile(int tile, const int* prefix, const int* valid,
                                                const GemmParams& P) {
  if (MODE == GEMM_WGRAD_BF16)
    return decode_tile_var_k(tile, prefix, P.M / BM, P.N / BN, P.order);
  return decode_tile_var_m(tile, prefix, valid, P.G, P.N / BN, P.N, P.K / BK);
}

// Swapped last tile of an fp32-output GEMM: the accumulator chunk v holds, for this lane's
// output column (feature xc + lane), 32 consecutive tokens tb..tb+31.  Stored as 32 rows of
// the output through shared memory and a TMA store: fp32 (box 32 x 32, 128-byte swizzle,
// tm32f) or scaled fp16 (box 32 x 32 unswizzled, tm16; a token's 32 features are this
// warp's lanes, so each block's maximum is taken across the lanes -- the bit patterns of
// non-negative floats order as the values).  stg: this warp's two staging buffers.
__device__ __forceinline__ void store_swapped_chunk(const float (&v)[32], int tb, int32_t xc,
                                                    int32_t y0, int rows, uint8_t (*stg)[4096],
                                                    int& stg_buf, const GemmParams& P,
                                                    const CUtensorMap* tm32f,
                                                    const CUtensorMap* tm16, int lane) {
  if (tb >= rows) return;  // warp-uniform
  if (P.n_valid && xc >= P.n_valid) return;  // columns past the group's width
  uint8_t* buf = stg[stg_buf];
  if (lane == 0) bulk_wait_read<1>();
  __syncwarp();
  if (P.out_scales) {
    uint32_t my_sb = 0;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const uint32_t am = __reduce_max_sync(kFull, __float_as_uint(fabsf(v[r])));
      const int sx = f16s_scale_exp(__uint_as_float(am));
      if (lane == r) my_sb = static_cast<uint32_t>(sx + 127);
      *reinterpret_cast<__half*>(buf + r * 64 + lane * 2) = __float2half_rn(v[r] * mx_inv_scale(sx));
    }
    P.out_scales[static_cast<int64_t>(y0 + tb + lane) * (P.N >> 5) + (xc >> 5)] =
        static_cast<uint8_t>(my_sb);
  } else {
#pragma unroll
    for (int r = 0; r < 32; ++r)  // token r of the chunk, feature = lane
      *reinterpret_cast<float*>(buf + r * 128 + ((((lane >> 2) ^ (r & 7))) << 4) +
                                ((lane & 3) << 2)) = v[r];
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(P.out_scales ? tm16 : tm32f, smem_u32(buf), xc, y0 + tb);
    bulk_commit();
  }
  stg_buf ^= 1;
}

// (sigmoid_fast, common.cuh: the epilogues evaluate it once per output element, and the IEEE
// exp + division sequence kept the transcendental pipe busy for as long as the MMA main loop
// of a short-K tile.)

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmC0,
                        const __grid_constant__ CUtensorMap tmC1, const GemmParams P) {
  constexpr int STAGES = ModeCfg<MODE>::kStages;
  using GemmSmem = SmemOf<MODE>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  GemmSmem& S = *reinterpret_cast<GemmSmem*>(smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = P.G, NT = P.N / BN;
  const int64_t kgroups = P.K / 128;

  for (int i = tid; i <= G; i += kGemmThreads) S.prefix[i] = P.mtile_prefix[i] >> P.prefix_shift;
  for (int i = tid; i < G; i += kGemmThreads)
    S.valid[i] = P.rows_valid ? P.rows_valid[i] : 0x7fffffff;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&S.full[s]), 1);
      mbar_init(smem_u32(&S.empty[s]), 1);
    }
    mbar_init(smem_u32(&S.tmem_full), 1);
    mbar_init(smem_u32(&S.tmem_empty), kEpiWarps);
    mbar_init(smem_u32(&S.tmem_empty_hi), kEpiWarps);
    for (int r = 0; r < kRing; ++r) {
      mbar_init(smem_u32(&S.ring_full[r]), 1);
      mbar_init(smem_u32(&S.ring_empty[r]), 1 + kEpiWarps);
    }
    mbar_init(smem_u32(&S.mma_drain), 1);
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
  const int total = MODE == GEMM_WGRAD_BF16 ? G * (P.M / BM) * NT : S.prefix[G] * NT;
  volatile int* abort_flag = &S.abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0, rs = 0, ready_b = -1;
      uint32_t phase = 0, rph = 0;
      uint32_t armed = 0, armed_par = 0;  // stages with a load issued, and that phase's parity
      for (;;) {
        const int tile = static_cast<int>(atomicAdd(P.tile_ctr, 1u));
        if (!mbar_wait(smem_u32(&S.ring_empty[rs]), rph ^ 1u, abort_flag, P.status)) break;
        S.ring[rs] = tile < total ? tile : -1;
        mbar_arrive(smem_u32(&S.ring_full[rs]));
        if (++rs == kRing) {
          rs = 0;
          rph ^= 1u;
        }
        if (tile >= total) break;
        const TileInfo ti = decode_tile<MODE>(tile, S.prefix, S.valid, P);
        if (MODE != GEMM_WGRAD_BF16 && P.ready) {
          // the tile's rows are loaded once the dispatch has published their minibatch
          const int b = static_cast<int>(ti.a_row0 / P.ready_rows);
          if (b > ready_b) {
            if (!wait_counter_zero(P.ready + b, abort_flag, P.status)) break;
            fence_proxy_async_global();
            ready_b = b;
          }
        }
        const int64_t rbA = ti.a_row0 >> 7, rbB = ti.b_row0 >> 7;
        bool ok = true;
        for (int kb = ti.kb0; kb < ti.kb0 + ti.nk; ++kb) {
          if (!mbar_wait(smem_u32(&S.empty[stage]), phase ^ 1u, abort_flag, P.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&S.full[stage]);
          mbar_arrive_expect_tx(fb, ModeCfg<MODE>::kTx);
          if (MODE == GEMM_WGRAD_BF16) {
            // token-direction operands in 128 x 128 tiles: feature block fb of token block kb
            // is the 128 rows from (kb * features / 128 + fb) * 128; the B box of 256 rows
            // spans feature blocks 2j and 2j + 1 of the same token block
            tma_load_2d(smem_u32(S.a[stage]), &tmA, fb, 0,
                        static_cast<int32_t>((kb * (P.M >> 7) + (ti.a_row0 >> 7)) * 128));
            tma_load_2d(smem_u32(S.b[stage]), &tmB, fb, 0,
                        static_cast<int32_t>((kb * (P.N >> 7) + (ti.b_row0 >> 7)) * 128));
          } else {
            tma_load_2d(smem_u32(S.a[stage]), &tmA, fb, kb * BK, static_cast<int32_t>(ti.a_row0));
            tma_load_2d(smem_u32(S.b[stage]), &tmB, fb, kb * BK, static_cast<int32_t>(ti.b_row0));
          }
          if (!ModeCfg<MODE>::kBf16) {
            bulk_load(smem_u32(S.sfa[stage]), P.sfa + ((rbA * kgroups + kb) << 9), 512, fb);
            bulk_load(smem_u32(S.sfb[stage]), P.sfb + ((rbB * kgroups + kb) << 9), 512, fb);
            bulk_load(smem_u32(S.sfb[stage]) + 512, P.sfb + (((rbB + 1) * kgroups + kb) << 9),
                      512, fb);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // Leave only once every load this thread issued has landed in shared memory (on the
      // normal path the MMAs consumed them all; after an abort some may still be in flight).
      for (int st = 0; st < STAGES; ++st)
        if ((armed >> st) & 1u) mbar_drain(smem_u32(&S.full[st]), (armed_par >> st) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, rs = 0;
      uint32_t phase = 0, acc_phase = 0, rph = 0;
      bool issued = false;
      const uint32_t idesc = idesc_mxf8_e4m3(BM, BN);
      for (;;) {
        if (!mbar_wait(smem_u32(&S.ring_full[rs]), rph, abort_flag, P.status)) break;
        const int tile = S.ring[rs];
        mbar_arrive(smem_u32(&S.ring_empty[rs]));
        if (++rs == kRing) {
          rs = 0;
          rph ^= 1u;
        }
        if (tile < 0) break;
        const TileInfo tinfo = decode_tile<MODE>(tile, S.prefix, S.valid, P);
        const int nk = tinfo.nk;
        if (nk == 0) continue;  // empty expert (wgrad): the epilogue writes zeros
        issued = true;
        const bool swapped = ModeCfg<MODE>::kSwapTail && tinfo.rows < BM;
        const uint32_t idesc_sw = idesc_mxf8_e4m3(BM, (tinfo.rows + 15) & ~15);
        if (!mbar_wait(smem_u32(&S.tmem_empty), acc_phase ^ 1u, abort_flag, P.status)) break;
        tc_fence_after();
        bool ok = true;
        if (MODE == GEMM_WGRAD_BF16) {
          // Two N = 128 MMAs per K step, columns 0..127 first: the epilogue releases that
          // half before it drains columns 128..255, so the next tile starts earlier.
          const uint32_t idesc_h = idesc_mxf8_e4m3(BM, BN / 2);
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
              const uint32_t id = idesc_h | (static_cast<uint32_t>(kk) << 29) |
                                  (static_cast<uint32_t>(kk) << 4);
              mma_mxf8(tbase + kAccCol, sdesc_k_sw128(a0 + 32u * kk),
                       sdesc_k_sw128(b0 + 32u * kk), id, (kb | kk) != 0 ? 1u : 0u, sf, sf + 4);
            }
            if (kb == 0) {
              if (!mbar_wait(smem_u32(&S.tmem_empty_hi), acc_phase ^ 1u, abort_flag, P.status)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk) {
              const uint32_t id = idesc_h | (static_cast<uint32_t>(kk) << 29) |
                                  (static_cast<uint32_t>(kk) << 4);
              mma_mxf8(tbase + kAccCol + BN / 2, sdesc_k_sw128(a0 + 32u * kk),
                       sdesc_k_sw128(b0 + 128u * 128u + 32u * kk), id, (kb | kk) != 0 ? 1u : 0u,
                       sf, sf + 8);
            }
            mma_commit(smem_u32(&S.empty[stage]));
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        } else {
          for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(smem_u32(&S.full[stage]), phase, abort_flag, P.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(S.a[stage]), b0 = smem_u32(S.b[stage]);
            if (ModeCfg<MODE>::kBf16) {
              // bf16 operands: 4 MMAs of K = 16 elements (32 bytes) per 128-byte stage
              const uint32_t id = swapped ? idesc_f16_bf16(BM, (tinfo.rows + 15) & ~15)
                                          : idesc_f16_bf16(BM, BN);
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk) {
                const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
                if (swapped) {
                  const uint64_t bt = sdesc_k_sw128(a0 + 32u * kk);
                  mma_bf16(tbase + kAccCol, sdesc_k_sw128(b0 + 32u * kk), bt, id, acc);
                  mma_bf16(tbase + kAccCol + 128, sdesc_k_sw128(b0 + 128u * 128u + 32u * kk), bt,
                           id, acc);
                } else {
                  mma_bf16(tbase + kAccCol, sdesc_k_sw128(a0 + 32u * kk),
                           sdesc_k_sw128(b0 + 32u * kk), id, acc);
                }
              }
              mma_commit(smem_u32(&S.empty[stage]));
              if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
              }
              continue;
            }
            const uint32_t sf = tbase + kSfCol + 16u * stage;
            tmem_cp_scales(sf, sdesc_scale_chunk(smem_u32(S.sfa[stage])));
            tmem_cp_scales(sf + 4, sdesc_scale_chunk(smem_u32(S.sfb[stage])));
            tmem_cp_scales(sf + 8, sdesc_scale_chunk(smem_u32(S.sfb[stage]) + 512));
            if (swapped) {
              // D0[w, t] = sum_k B[w, k] A[t, k] for weight rows w < 128, D1 for rows 128..255
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk) {
                const uint32_t id = idesc_sw | (static_cast<uint32_t>(kk) << 29) |
                                    (static_cast<uint32_t>(kk) << 4);
                const uint64_t bt = sdesc_k_sw128(a0 + 32u * kk);
                mma_mxf8(tbase + kAccCol, sdesc_k_sw128(b0 + 32u * kk), bt, id,
                         (kb | kk) != 0 ? 1u : 0u, sf + 4, sf);
                mma_mxf8(tbase + kAccCol + 128, sdesc_k_sw128(b0 + 128u * 128u + 32u * kk), bt, id,
                         (kb | kk) != 0 ? 1u : 0u, sf + 8, sf);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk) {
                const uint32_t id = idesc | (static_cast<uint32_t>(kk) << 29) |
                                    (static_cast<uint32_t>(kk) << 4);
                mma_mxf8(tbase + kAccCol, sdesc_k_sw128(a0 + 32u * kk),
                         sdesc_k_sw128(b0 + 32u * kk), id, (kb | kk) != 0 ? 1u : 0u, sf, sf + 4);
              }
            }
            mma_commit(smem_u32(&S.empty[stage]));
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&S.tmem_full));
        acc_phase ^= 1u;
      }
      // every MMA and scale copy issued here has completed before the CTA moves on
      if (issued) {
        mma_commit(smem_u32(&S.mma_drain));
        mbar_drain(smem_u32(&S.mma_drain), 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;   // column half
    uint32_t acc_phase = 0, rph = 0;
    int stg_buf = 0, rs = 0;
    for (;;) {
      if (!mbar_wait(smem_u32(&S.ring_full[rs]), rph, abort_flag, P.status)) break;
      const int tile = S.ring[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.ring_empty[rs]));
      if (++rs == kRing) {
        rs = 0;
        rph ^= 1u;
      }
      if (tile < 0) break;
      const TileInfo ti = decode_tile<MODE>(tile, S.prefix, S.valid, P);
      if (MODE == GEMM_WGRAD_BF16 && ti.nk == 0) {
        const int64_t m = ti.a_row0 + 32 * q + lane;
        const int n0 = ti.j * BN + 128 * h;
        const bool first = n0 < P.split;
        const int ld = first ? P.split : P.N - P.split;
        uint16_t* base = (first ? P.out_a : P.out_b) +
                         (static_cast<int64_t>(ti.g) * P.M + m) * ld + (first ? n0 : n0 - P.split);
        uint4* dst = reinterpret_cast<uint4*>(base);
#pragma unroll
        for (int c = 0; c < 16; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      if (!mbar_wait(smem_u32(&S.tmem_full), acc_phase, abort_flag, P.status)) break;
      tc_fence_after();
      const uint32_t taddr = tbase + kAccCol + (static_cast<uint32_t>(32 * q) << 16);
      if (MODE == GEMM_WGRAD_BF16) {
        // columns 64h..64h+63 of each 128-column half; the lower half is released first
        float v0[32], v1[32], v2[32], v3[32];
        tmem_ld32(taddr + 64 * h, v0);
        tmem_ld32(taddr + 64 * h + 32, v1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S.tmem_empty));
        tmem_ld32(taddr + 128 + 64 * h, v2);
        tmem_ld32(taddr + 128 + 64 * h + 32, v3);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S.tmem_empty_hi));
        acc_phase ^= 1u;
        const int32_t y = static_cast<int32_t>(ti.g * P.M + ti.a_row0 + 32 * q);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int n0 = ti.j * BN + 128 * half + 64 * h;  // 64 bf16 columns = one chunk
          const bool first = n0 < P.split;
          const float* va = half == 0 ? v0 : v2;
          const float* vb = half == 0 ? v1 : v3;
          uint4 r16[8];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            r16[c] = pack_bf16x8(va + 8 * c);
            r16[4 + c] = pack_bf16x8(vb + 8 * c);
          }
          stage_and_store(S.stg[2 * (warp - 2) + stg_buf], r16, first ? &tmC0 : &tmC1,
                          first ? n0 : n0 - P.split, y, lane);
          stg_buf ^= 1;
        }
        continue;
      }
      if (ModeCfg<MODE>::kSwapTail && ti.rows < BM) {
        // transposed accumulators: lane = weight row (feature), column = token
        const int tok0 = 64 * h;
        float d0a[32], d0b[32], d1a[32], d1b[32];
        tmem_ld32(taddr + tok0, d0a);
        tmem_ld32(taddr + tok0 + 32, d0b);
        tmem_ld32(taddr + 128 + tok0, d1a);
        tmem_ld32(taddr + 128 + tok0 + 32, d1b);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S.tmem_empty));
        acc_phase ^= 1u;
        if constexpr (ModeCfg<MODE>::kStoreF32) {
          const int32_t y0 = static_cast<int32_t>(ti.a_row0);
          const int32_t x0 = ti.j * BN + 32 * q;
          // one call per 32-token chunk, each with its own register array (indexed with
          // compile-time offsets only, so the arrays stay in registers)
          uint8_t(*stg)[4096] = &S.stg[2 * (warp - 2)];
          store_swapped_chunk(d0a, tok0, x0, y0, ti.rows, stg, stg_buf, P, &tmC0, &tmC1, lane);
          store_swapped_chunk(d0b, tok0 + 32, x0, y0, ti.rows, stg, stg_buf, P, &tmC0, &tmC1,
                              lane);
          store_swapped_chunk(d1a, tok0, x0 + 128, y0, ti.rows, stg, stg_buf, P, &tmC0, &tmC1,
                              lane);
          store_swapped_chunk(d1b, tok0 + 32, x0 + 128, y0, ti.rows, stg, stg_buf, P, &tmC0,
                              &tmC1, lane);
        }
        continue;
      }
      float v0[32], v1[32], v2[32], v3[32];
      if (ModeCfg<MODE>::kGateUp) {
        tmem_ld32(taddr + 64 * h, v0);         // gate features 64h .. 64h+31
        tmem_ld32(taddr + 64 * h + 32, v1);    // gate features 64h+32 .. 64h+63
        tmem_ld32(taddr + 128 + 64 * h, v2);   // up, same features
        tmem_ld32(taddr + 128 + 64 * h + 32, v3);
      } else if constexpr (ModeCfg<MODE>::kSwigluBwd) {
        // columns 64..127 first go to this warp's staging buffers (8 KB: [64 columns][32
        // rows], lane-contiguous), so that only 64 accumulator registers are live at a time;
        // an earlier (swapped) tile's TMA store may still be reading those buffers
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        float* stash = reinterpret_cast<float*>(S.stg[2 * (warp - 2)]);
        tmem_ld32(taddr + 128 * h + 64, v2);
        tmem_ld32(taddr + 128 * h + 96, v3);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          stash[i * 32 + lane] = v2[i];
          stash[(32 + i) * 32 + lane] = v3[i];
        }
        tmem_ld32(taddr + 128 * h, v0);
        tmem_ld32(taddr + 128 * h + 32, v1);
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
      if constexpr (ModeCfg<MODE>::kSwigluBwd) {
        // A full tile (an expert's partial last tile runs swapped and stores G): for this
        // row's 128 features, d(combine weight) partial <G, h^>, then dg, du from the saved
        // g | u, each 32-feature block requantised (MX along 2f) where the SwiGLU-backward
        // kernel would have stored it.
        const int64_t row = ti.a_row0 + m;
        const int f = P.N;
        const int64_t pos = P.offsets[ti.g] + (row - static_cast<int64_t>(S.prefix[ti.g]) * BM);
        const float w = P.topk_w[P.perm[pos]];
        const int nb = ti.j * BN + 128 * h;  // first feature of this thread's 128
        const uint16_t* grow = P.gu + row * 2 * f;
        const uint8_t* hrow = P.hq + row * f;
        const int64_t kgh = f >> 7, kg2 = (2 * f) >> 7;
        const float* stash = reinterpret_cast<const float*>(S.stg[2 * (warp - 2)]);
        float dwp = 0.f;
        uint32_t sbg = 0, sbu = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float G[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            G[i] = c == 0 ? v0[i] : c == 1 ? v1[i] : stash[((c - 2) * 32 + i) * 32 + lane];
          const int fb = nb + 32 * c;
          uint4 gq[4], uq[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            gq[i] = __ldg(reinterpret_cast<const uint4*>(grow + fb) + i);
            uq[i] = __ldg(reinterpret_cast<const uint4*>(grow + f + fb) + i);
          }
          const uint4 h0 = __ldg(reinterpret_cast<const uint4*>(hrow + fb));
          const uint4 h1 = __ldg(reinterpret_cast<const uint4*>(hrow + fb) + 1);
          const float hsc = e8m0_to_f32(P.hs[umma_scale_offset(row, fb >> 5, kgh)]);
          const uint32_t gw[16] = {gq[0].x, gq[0].y, gq[0].z, gq[0].w, gq[1].x, gq[1].y,
                                   gq[1].z, gq[1].w, gq[2].x, gq[2].y, gq[2].z, gq[2].w,
                                   gq[3].x, gq[3].y, gq[3].z, gq[3].w};
          const uint32_t uw[16] = {uq[0].x, uq[0].y, uq[0].z, uq[0].w, uq[1].x, uq[1].y,
                                   uq[1].z, uq[1].w, uq[2].x, uq[2].y, uq[2].z, uq[2].w,
                                   uq[3].x, uq[3].y, uq[3].z, uq[3].w};
          const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
          // pass 1: <G, h^> and the block maxima of dg and du; pass 2 recomputes dg, du (the
          // same instructions: the same values) and quantises them four at a time, so no
          // block array is held in registers
          float amg = 0.f, amu = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint32_t code = (hw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
            dwp = fmaf(G[i], e4m3_to_f32(code) * hsc, dwp);
            const float gb = bf16_bits_to_f32((gw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
            const float ub = bf16_bits_to_f32((uw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
            float dg, du;
            swiglu_bwd_elem(G[i], w, gb, ub, dg, du);
            amg = fmaxf(amg, fabsf(dg));
            amu = fmaxf(amu, fabsf(du));
          }
          const int sg = mx_scale_exp(amg), su = mx_scale_exp(amu);
          const float ig = mx_inv_scale(sg), iu = mx_inv_scale(su);
          sbg |= static_cast<uint32_t>(sg + 127) << (8 * c);
          sbu |= static_cast<uint32_t>(su + 127) << (8 * c);
          uint32_t qg[8], qu[8];
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            float dg[4], du[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 4 * i4 + e;
              const float gb = bf16_bits_to_f32((gw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
              const float ub = bf16_bits_to_f32((uw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
              swiglu_bwd_elem(G[i], w, gb, ub, dg[e], du[e]);
            }
            qg[i4] = pack_e4m3x4(dg[0] * ig, dg[1] * ig, dg[2] * ig, dg[3] * ig);
            qu[i4] = pack_e4m3x4(du[0] * iu, du[1] * iu, du[2] * iu, du[3] * iu);
          }
          uint4* dst = reinterpret_cast<uint4*>(P.dgu_q + row * 2 * f + fb);
          dst[0] = make_uint4(qg[0], qg[1], qg[2], qg[3]);
          dst[1] = make_uint4(qg[4], qg[5], qg[6], qg[7]);
          dst = reinterpret_cast<uint4*>(P.dgu_q + row * 2 * f + f + fb);
          dst[0] = make_uint4(qu[0], qu[1], qu[2], qu[3]);
          dst[1] = make_uint4(qu[4], qu[5], qu[6], qu[7]);
        }
        *reinterpret_cast<uint32_t*>(P.dgu_s + umma_scale_offset(row, nb >> 5, kg2)) = sbg;
        *reinterpret_cast<uint32_t*>(P.dgu_s + umma_scale_offset(row, (f + nb) >> 5, kg2)) = sbu;
        P.dw_part[row * (f >> 7) + (nb >> 7)] = dwp;
        continue;
      }
      if (ModeCfg<MODE>::kStoreF32) {
        // fp32 rows of 128 columns: four 32-column chunks; whole 32-row boxes are written
        const int32_t x0 = ti.j * BN + 128 * h;
        const int32_t y = static_cast<int32_t>(ti.a_row0 + 32 * q);
        if (P.out_scales) {
          // scaled fp16: each 32-column block of this row gets its own power-of-two scale;
          // two blocks make one staged 128-byte row (64 fp16 columns)
          uint32_t sb = 0;
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            uint4 r16[8];
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
              const int c = 2 * c2 + hb;
              const float* vc = c == 0 ? v0 : c == 1 ? v1 : c == 2 ? v2 : v3;
              float amax = 0.f;
#pragma unroll
              for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(vc[i]));
              const int sx = f16s_scale_exp(amax);
              const float inv = mx_inv_scale(sx);
              sb |= static_cast<uint32_t>(sx + 127) << (8 * c);
#pragma unroll
              for (int jj = 0; jj < 4; ++jj)
                r16[4 * hb + jj] = make_uint4(
                    pack_f16x2(vc[8 * jj] * inv, vc[8 * jj + 1] * inv),
                    pack_f16x2(vc[8 * jj + 2] * inv, vc[8 * jj + 3] * inv),
                    pack_f16x2(vc[8 * jj + 4] * inv, vc[8 * jj + 5] * inv),
                    pack_f16x2(vc[8 * jj + 6] * inv, vc[8 * jj + 7] * inv));
            }
            stage_and_store(S.stg[2 * (warp - 2) + stg_buf], r16, &tmC0, x0 + 64 * c2, y, lane);
            stg_buf ^= 1;
          }
          *reinterpret_cast<uint32_t*>(P.out_scales + (ti.a_row0 + m) * (P.N >> 5) + (x0 >> 5)) =
              sb;
          continue;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (P.n_valid && x0 + 32 * c >= P.n_valid) break;  // columns past the group's width
          const float* vc = c == 0 ? v0 : c == 1 ? v1 : c == 2 ? v2 : v3;
          uint4 r16[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            r16[j] = make_uint4(__float_as_uint(vc[4 * j]), __float_as_uint(vc[4 * j + 1]),
                                __float_as_uint(vc[4 * j + 2]), __float_as_uint(vc[4 * j + 3]));
          stage_and_store(S.stg[2 * (warp - 2) + stg_buf], r16, &tmC0, x0 + 32 * c, y, lane);
          stg_buf ^= 1;
        }
        continue;
      }
      if (ti.i * BM + m >= S.valid[ti.g]) continue;
      const int64_t row = ti.a_row0 + m;
      if (ModeCfg<MODE>::kGateUp) {
        const int f = P.f;
        const int fb = BN / 2 * ti.j + 64 * h;  // first feature of this thread's 64
        if (P.gu) {
          uint4* gdst = reinterpret_cast<uint4*>(P.gu + row * 2 * f + fb);
          uint4* udst = reinterpret_cast<uint4*>(P.gu + row * 2 * f + f + fb);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float* g = c < 4 ? v0 + 8 * c : v1 + 8 * (c - 4);
            const float* u = c < 4 ? v2 + 8 * c : v3 + 8 * (c - 4);
            gdst[c] = pack_bf16x8(g);
            udst[c] = pack_bf16x8(u);
          }
        }
        // h = silu(g) * u, in place over the gate registers
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          v0[c] = v0[c] * sigmoid_fast(v0[c]) * v2[c];
          v1[c] = v1[c] * sigmoid_fast(v1[c]) * v3[c];
        }
        if (ModeCfg<MODE>::kBf16) {  // the BF16 variant: h rounded to bf16 (RNE)
          uint4* hdst = reinterpret_cast<uint4*>(P.h16 + row * f + fb);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            hdst[c] = pack_bf16x8(v0 + 8 * c);
            hdst[4 + c] = pack_bf16x8(v1 + 8 * c);
          }
          continue;
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
      }
    }
  }

  if (ModeCfg<MODE>::kTmaStore && warp >= 2 && lane == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

template <int MODE>
static cudaError_t launch_mode(const CUtensorMap& tmA, const CUtensorMap& tmB,
                               const CUtensorMap& tmC0, const CUtensorMap& tmC1,
                               const GemmParams& P, int num_sms, cudaStream_t stream, bool pdl) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_bytes<MODE>()));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = smem_bytes<MODE>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<MODE>, tmA, tmB, tmC0, tmC1, P);
}

cudaError_t launch_grouped_gemm(int mode, const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const CUtensorMap& tmC0, const CUtensorMap& tmC1,
                                const GemmParams& P, int num_sms, cudaStream_t stream, bool pdl) {
  if (!P.tile_ctr) return cudaErrorInvalidValue;
  switch (mode) {
    case GEMM_GATEUP_SWIGLU:
      return launch_mode<GEMM_GATEUP_SWIGLU>(tmA, tmB, tmC0, tmC1, P, num_sms, stream, pdl);
    case GEMM_WGRAD_BF16:
      return launch_mode<GEMM_WGRAD_BF16>(tmA, tmB, tmC0, tmC1, P, num_sms, stream, pdl);
    case GEMM_STORE_F32_TMA:
      return launch_mode<GEMM_STORE_F32_TMA>(tmA, tmB, tmC0, tmC1, P, num_sms, stream, pdl);
    case GEMM_GATEUP_BF16:
      return launch_mode<GEMM_GATEUP_BF16>(tmA, tmB, tmC0, tmC1, P, num_sms, stream, pdl);
    case GEMM_STORE_F32_BF16:
      return launch_mode<GEMM_STORE_F32_BF16>(tmA, tmB, tmC0, tmC1, P, num_sms, stream, pdl);
    case GEMM_DGRAD_SWIGLU:
      return launch_mode<GEMM_DGRAD_SWIGLU>(tmA, tmB, tmC0, tmC1, P, num_sms, stream, pdl);
    default:
      return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------------------
// scheduling tables (one CTA): minibatch readiness counters and the longest-first order
// ---------------------------------------------------------------------------------------
constexpr int kSchedThreads = 256;

__global__ void __launch_bounds__(kSchedThreads) sched_init_kernel(SchedInitParams P) {
  __shared__ int s_cnt[kMaxG];
  __shared__ int s_pad[kMaxG + 1];
  const int tid = threadIdx.x, E = P.E;
  for (int e = tid; e < E; e += kSchedThreads) s_cnt[e] = P.counts[e];
  for (int e = tid; e <= E; e += kSchedThreads) s_pad[e] = P.pad_offsets[e];
  for (int b = tid; b < P.n_ready; b += kSchedThreads) P.ready[b] = 0;
  __syncthreads();
  // valid rows of every expert segment, added to each minibatch the segment overlaps
  for (int e = tid; e < E; e += kSchedThreads) {
    const int lo = s_pad[e], hi = s_pad[e] + s_cnt[e];
    for (int b = lo / P.ready_rows; b < P.n_ready && b * P.ready_rows < hi; ++b) {
      const int a0 = max(lo, b * P.ready_rows), a1 = min(hi, (b + 1) * P.ready_rows);
      if (a1 > a0) atomicAdd(P.ready + b, a1 - a0);
    }
  }
  if (!P.order) return;
  // order[rank(e)] = e with rank = experts before e in (count descending, index ascending)
  for (int e = tid; e < E; e += kSchedThreads) {
    const int c = s_cnt[e];
    int rank = 0;
    for (int f = 0; f < E; ++f) rank += (s_cnt[f] > c) || (s_cnt[f] == c && f < e);
    P.order[rank] = e;
  }
}

cudaError_t launch_sched_init(const SchedInitParams& P, cudaStream_t stream) {
  if (P.E <= 0 || P.E > kMaxG || P.ready_rows <= 0) return cudaErrorInvalidValue;
  sched_init_kernel<<<1, kSchedThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace moe
