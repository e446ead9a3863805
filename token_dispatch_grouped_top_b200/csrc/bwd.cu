// Backward support kernel: token-direction MXFP8 quantisation of the weight-gradient operands.
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72", §01/§02:
// training adds a backward pass with two reverse communications (pull reverse-combine of
// the output gradient, push reverse-dispatch of the input gradient); the weight gradients
// of each expert reduce over that expert's tokens.  A block-scaled GEMM needs its operands
// quantised along the reduction axis, which for the weight gradients is the token axis.
// Each operand is the token-direction requantisation of an MX operand the data path
// already holds (x^, h^, dout^ scaled by the row's combine weight, [dg|du]^):
// blocks of 32 consecutive tokens inside one expert's segment (segments start on 128-row
// boundaries, so a block never straddles two experts; rows past the segment's count are
// zeros).  The result is stored transposed, K-major for the GEMM, in 128 x 128 tiles: the
// tile of features [128 fb, +128) and tokens [128 tb, +128) is one contiguous 16 KB block
// (row = feature, 128 token bytes per row) at block index tb * (C / 128) + fb, so each
// tile leaves as one sequential 16 KB write and the GEMM loads its 128- and 256-row boxes
// (one or two adjacent feature blocks of a token block) from contiguous memory.
//
// TMA-staged 128 x 128 tiles: see transpose_quant_kernel.  C % 128 == 0 (d, f, 2f all are).
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kTqThreads = 256;
constexpr int kTqCtasPerSm = 3;
constexpr uint32_t kTqTile = 128 * 128;  // bytes of codes per 128 x 128 tile
constexpr int kTqMaxE = 1024;

// Per-CTA shared memory: two tiles in flight each way.
struct TqSmem {
  uint8_t in[2][kTqTile];    // source codes, 128-byte rows (TMA, no swizzle)
  uint8_t out[2][kTqTile];   // transposed codes, 128-byte swizzle (TMA store layout)
  uint8_t sin[2][512];       // the source's UMMA scale chunk of the tile
  uint8_t sout[2][512];      // the output's UMMA scale chunk of the tile
  float mul[4][128];         // 2^s(row, 32-column block) x weight of the row
  uint64_t full[2];
  int abort_flag;
  int pad[kTqMaxE + 1];
};
constexpr size_t kTqSmemBytes = sizeof(TqSmem) + 1024;


// Two fp32 products in one packed instruction (each lane rounded to nearest even, as the
// scalar multiply): (a0, a1) *= (b0, b1).
__device__ __forceinline__ void mul2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "mul.rn.f32x2 z, x, y;\n\tmov.b64 {%0, %1}, z;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}

// One thread: column c of the tile, 32-row block b: decode 32 codes down the column,
// scale them (rows at or past `lim` are zero), requantise along the rows, write the
// 32 output bytes into row c of the swizzled output tile and the scale byte into the
// output chunk.  The row multipliers come four at a time (one 16-byte shared load) and
// both multiplications run on packed pairs.
template <bool kRagged>
__device__ __forceinline__ void tq_column_block(const uint8_t* col, const float* mul, int b,
                                                int lim, uint8_t* orow, int c, uint8_t* sout) {
  float v[32];
#pragma unroll
  for (int r4 = 0; r4 < 32; r4 += 4) {
    const float4 m = *reinterpret_cast<const float4*>(mul + 32 * b + r4);
#pragma unroll
    for (int h = 0; h < 4; h += 2) {  // rows r, r+1: one hardware E4M3x2 -> f16x2 decode
      const int r = r4 + h, rr = 32 * b + r;
      const uint32_t pair = static_cast<uint32_t>(col[rr * 128]) |
                            (static_cast<uint32_t>(col[(rr + 1) * 128]) << 8);
      uint32_t h2;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(pair)));
      v[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
      v[r + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
      mul2(v[r], v[r + 1], h ? m.z : m.x, h ? m.w : m.y);
      if (kRagged) {
        if (r >= lim) v[r] = 0.f;
        if (r + 1 >= lim) v[r + 1] = 0.f;
      }
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int s = mx_scale_exp(amax);
  const float inv = mx_inv_scale(s);
#pragma unroll
  for (int i = 0; i < 32; i += 2) mul2(v[i], v[i + 1], inv, inv);
  uint32_t qw[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    qw[i] = cvt_e4m3x2(v[4 * i], v[4 * i + 1]) | (cvt_e4m3x2(v[4 * i + 2], v[4 * i + 3]) << 16);
  *reinterpret_cast<uint4*>(orow + (((2 * b) ^ (c & 7)) << 4)) =
      make_uint4(qw[0], qw[1], qw[2], qw[3]);
  *reinterpret_cast<uint4*>(orow + (((2 * b + 1) ^ (c & 7)) << 4)) =
      make_uint4(qw[4], qw[5], qw[6], qw[7]);
  sout[(c & 31) * 16 + (c >> 5) * 4 + b] = static_cast<uint8_t>(s + 127);
}

// A 32-row block entirely past the segment's valid rows: zero codes, scale byte 0 (the
// all-zero block's scale 2^-127), as the requantisation of zeros gives.
__device__ __forceinline__ void tq_zero_block(int b, uint8_t* orow, int c, uint8_t* sout) {
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  *reinterpret_cast<uint4*>(orow + (((2 * b) ^ (c & 7)) << 4)) = z;
  *reinterpret_cast<uint4*>(orow + (((2 * b + 1) ^ (c & 7)) << 4)) = z;
  sout[(c & 31) * 16 + (c >> 5) * 4 + b] = 0;
}

// Persistent: each CTA walks 128 x 128 tiles (column block fastest) of the rows that
// belong to some expert segment (rows [0, pad_offsets[E]); the rest of the R-row buffer is
// never read by the weight-gradient GEMM).  Thread 0 keeps the next tile's codes (TMA, the
// 32-row boxes that hold valid rows) and scale chunk (512 B) in flight while all threads
// work on the current one;
// the transposed tile (16 contiguous KB) and its scale chunk leave through TMA / bulk
// stores.  Thread (c, h) handles column c for the
// 32-row blocks h and h + 2.
__global__ void __launch_bounds__(kTqThreads) transpose_quant_kernel(
    const __grid_constant__ CUtensorMap tm_src, const __grid_constant__ CUtensorMap tm_dst,
    const TransposeQuantParams P) {
  extern __shared__ uint8_t tq_raw[];
  const uint32_t raw_addr = smem_u32(tq_raw);
  TqSmem& S = *reinterpret_cast<TqSmem*>(tq_raw + ((1024u - (raw_addr & 1023u)) & 1023u));
  const int tid = threadIdx.x;
  for (int i = tid; i <= P.E; i += kTqThreads) S.pad[i] = P.pad_offsets[i];
  if (tid == 0) {
    mbar_init(smem_u32(&S.full[0]), 1);
    mbar_init(smem_u32(&S.full[1]), 1);
    S.abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_src);
    prefetch_tmap(&tm_dst);
  }
  __syncthreads();
  const int ncb = P.C >> 7;
  const int ntiles = (S.pad[P.E] >> 7) * ncb;
  const int64_t kg_src = P.C >> 7, kg_dst = P.R >> 7;
  // valid rows of the 128-row block starting at padded row p0: its expert's segment starts
  // on a 128-row boundary, so the block lies in one segment and holds 1..128 valid rows
  auto valid_rows = [&](int64_t p0) {
    int lo = 0, hi = P.E;  // pad[lo] <= p0 < pad[hi]: the expert owning these rows
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (S.pad[mid] <= p0) lo = mid; else hi = mid;
    }
    const int64_t rel = p0 - S.pad[lo];
    int nv = static_cast<int>(P.counts[lo] - rel);
    nv = nv < 0 ? 0 : (nv > 128 ? 128 : nv);
    return make_int2(lo, nv);
  };
  // only the 32-row boxes holding valid rows are loaded (the rest of the buffer is padding)
  auto issue = [&](int tile, int buf) {
    const int rb = tile / ncb, cb = tile - rb * ncb;
    const int nv = valid_rows(static_cast<int64_t>(rb) * 128).y;
    const int nbox = nv > 0 ? (nv + 31) >> 5 : 1;
    const uint32_t fb = smem_u32(&S.full[buf]);
    mbar_arrive_expect_tx(fb, static_cast<uint32_t>(nbox) * 4096u + 512u);
    for (int i = 0; i < nbox; ++i)
      tma_load_2d(smem_u32(S.in[buf]) + 4096u * i, &tm_src, fb, cb * 128, rb * 128 + 32 * i);
    bulk_load(smem_u32(S.sin[buf]), P.s + ((static_cast<int64_t>(rb) * kg_src + cb) << 9), 512,
              fb);
  };
  if (tid == 0 && static_cast<int>(blockIdx.x) < ntiles) issue(blockIdx.x, 0);
  const int c = tid & 127, hb = tid >> 7;
  int it = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    const int buf = it & 1;
    if (tid == 0) {
      const int next = tile + gridDim.x;
      if (next < ntiles) issue(next, buf ^ 1);  // buf ^ 1 was released at the last barrier
      bulk_wait_read<1>();  // the stores issued from out[buf] two tiles ago have read it
    }
    const int rb = tile / ncb, cb = tile - rb * ncb;
    const int64_t p0 = static_cast<int64_t>(rb) * 128;
    const int2 ev = valid_rows(p0);
    const int lo = ev.x, nv = ev.y;
    const int64_t rel = p0 - S.pad[lo];
    float w = 0.f;
    if (tid < 128 && tid < nv)
      w = P.src == TSRC_MX_W ? P.topk_w[P.perm[P.offsets[lo] + rel + tid]] : 1.f;
    const bool ok = mbar_wait(smem_u32(&S.full[buf]), (it >> 1) & 1, &S.abort_flag, P.status);
    if (tid < 128) {
      const uint32_t sw = *reinterpret_cast<const uint32_t*>(S.sin[buf] + (tid & 31) * 16 +
                                                             (tid >> 5) * 4);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t e = (sw >> (8 * q)) & 0xFFu;
        S.mul[q][tid] = tid < nv ? e8m0_to_f32(e) * w : 0.f;
      }
    }
    if (__syncthreads_or(!ok)) break;
    const uint8_t* col = S.in[buf] + c;
    const float* mul = S.mul[c >> 5];
    uint8_t* orow = S.out[buf] + c * 128;
#pragma unroll 1
    for (int bb = 0; bb < 2; ++bb) {
      const int b = hb + 2 * bb;
      const int lim = nv - 32 * b;
      if (lim >= 32)
        tq_column_block<false>(col, mul, b, lim, orow, c, S.sout[buf]);
      else if (lim > 0)
        tq_column_block<true>(col, mul, b, lim, orow, c, S.sout[buf]);
      else
        tq_zero_block(b, orow, c, S.sout[buf]);  // a block of padding rows only (never loaded)
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tma_store_2d(&tm_dst, smem_u32(S.out[buf]), 0, (rb * ncb + cb) * 128);  // one 16 KB tile
      bulk_store(P.dst_s + ((static_cast<int64_t>(cb) * kg_dst + rb) << 9), smem_u32(S.sout[buf]),
                 512);
      bulk_commit();
    }
  }
  if (tid == 0) bulk_wait_all();
}

cudaError_t launch_transpose_quant(const CUtensorMap& tm_src, const CUtensorMap& tm_dst,
                                   const TransposeQuantParams& P, int num_sms,
                                   cudaStream_t stream) {
  if (P.R <= 0 || P.C <= 0) return cudaSuccess;
  if (P.E > kTqMaxE) return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(transpose_quant_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(kTqSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[dev] = true;
  }
  const int64_t max_tiles = (P.R / 128) * (P.C / 128);
  const int64_t grid = std::min<int64_t>(max_tiles, static_cast<int64_t>(num_sms) * kTqCtasPerSm);
  transpose_quant_kernel<<<static_cast<unsigned>(grid), kTqThreads, kTqSmemBytes, stream>>>(
      tm_src, tm_dst, P);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// SwiGLU backward and d(router weights), one warp per assignment row, after the dgrad GEMM
// of the down projection.  Rows of full 128-row tiles were done in that GEMM's epilogue
// (dw_part given): here only their d(w) is summed from its partials.  For the rest (an
// expert's last, partial tile) the GEMM wrote G = dout^ . Wd'^T (fp32, padded order; it is
// kept in fp32 because dg, du are requantised from it, where a coarser G would move values
// across E4M3 rounding boundaries):
//   dw_route[a] = <G, h^>,  dh = w * G,  dg = dh * u * s * (1 + g (1 - s)),
//   du = dh * g * s,  s = sigmoid(g)  (g, u: the saved bf16 pre-activations),
// then [dg | du] quantised to MXFP8 along f (the operand of the dX GEMM).  Lane l covers 8
// consecutive features per 256-feature step; four lanes share a 32-feature MX block.
// ---------------------------------------------------------------------------------------
constexpr int kSbMaxE = 1024;


__device__ __forceinline__ void quant8_store(const float (&v)[8], int lane, uint8_t* q_dst,
                                             uint8_t* s_base, int64_t row, int64_t kb,
                                             int64_t kgroups) {
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
  *reinterpret_cast<uint2*>(q_dst) = packed;
  const uint32_t sb = static_cast<uint32_t>(s + 127);
  const uint32_t b1 = __shfl_down_sync(kFull, sb, 4);
  const uint32_t b2 = __shfl_down_sync(kFull, sb, 8);
  const uint32_t b3 = __shfl_down_sync(kFull, sb, 12);
  if ((lane & 15) == 0)
    *reinterpret_cast<uint32_t*>(s_base + umma_scale_offset(row, kb, kgroups)) =
        sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
}

__global__ void __launch_bounds__(256) swiglu_bwd_kernel(SwigluBwdParams P) {
  __shared__ int s_off[kSbMaxE + 1];
  __shared__ int s_pad[kSbMaxE + 1];
  for (int i = threadIdx.x; i <= P.E; i += blockDim.x) {
    s_off[i] = P.offsets[i];
    s_pad[i] = P.pad_offsets[i];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int f = P.f;
  const int64_t kg2 = (2 * f) >> 7;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5); q < P.A;
       q += warps) {
    int lo = 0, hi = P.E;  // s_off[lo] <= q < s_off[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_off[mid] <= q) lo = mid; else hi = mid;
    }
    const int64_t row = s_pad[lo] + (q - s_off[lo]);
    const int a = P.perm[q];
    if (P.dw_part) {
      // a row of a full 128-row tile: the dgrad GEMM's epilogue wrote its [dg | du] and the
      // partial sums of <G, h^> per 128 features; their sum, in block order, is d(w)
      const int64_t rel = q - s_off[lo], cnt = s_off[lo + 1] - s_off[lo];
      if ((rel / 128 + 1) * 128 <= cnt) {
        // all partials loaded at once (lanes), summed by a fixed shuffle tree
        const float* part = P.dw_part + row * (f >> 7);
        float acc = 0.f;
        for (int nb = lane; nb < (f >> 7); nb += 32) acc += part[nb];
#pragma unroll
        for (int off = 16; off; off >>= 1) acc += __shfl_down_sync(kFull, acc, off);
        if (lane == 0) P.dw_route[a] = acc;
        continue;
      }
    }
    const float w = P.topk_w[a];
    const float* Grow = P.G + row * f;
    const uint16_t* grow = P.gu + row * 2 * f;
    const uint8_t* hrow = P.h_q + row * f;
    float dwp = 0.f;
    for (int c0 = 0; c0 < f; c0 += 256) {
      const int fi = c0 + lane * 8;
      const float4 G0 = *reinterpret_cast<const float4*>(Grow + fi);
      const float4 G1 = *reinterpret_cast<const float4*>(Grow + fi + 4);
      const uint4 gq = *reinterpret_cast<const uint4*>(grow + fi);
      const uint4 uq = *reinterpret_cast<const uint4*>(grow + f + fi);
      const uint2 hq = *reinterpret_cast<const uint2*>(hrow + fi);
      const uint32_t hsb = P.h_s[umma_scale_offset(row, fi >> 5, f >> 7)];
      const float hsc = hsb ? __uint_as_float(hsb << 23) : __uint_as_float(0x00400000u);
      const float Gv[8] = {G0.x, G0.y, G0.z, G0.w, G1.x, G1.y, G1.z, G1.w};
      const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
      const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
      const uint32_t hw[2] = {hq.x, hq.y};
      float dg[8], du[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t code = (hw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        dwp = fmaf(Gv[i], e4m3_to_f32(code) * hsc, dwp);
        const float gb = bf16_bits_to_f32((gw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
        const float ub = bf16_bits_to_f32((uw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
        swiglu_bwd_elem(Gv[i], w, gb, ub, dg[i], du[i]);
      }
      quant8_store(dg, lane, P.dgu_q + row * 2 * f + fi, P.dgu_s, row, fi >> 5, kg2);
      quant8_store(du, lane, P.dgu_q + row * 2 * f + f + fi, P.dgu_s, row, (f + fi) >> 5, kg2);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) dwp += __shfl_xor_sync(kFull, dwp, off);
    if (lane == 0) P.dw_route[a] = dwp;
  }
}

cudaError_t launch_swiglu_bwd(const SwigluBwdParams& P, int num_sms, cudaStream_t stream) {
  if (P.A <= 0) return cudaSuccess;
  const int64_t blocks = (P.A + 7) / 8;
  const int grid = static_cast<int>(blocks < 16LL * num_sms ? blocks : 16LL * num_sms);
  swiglu_bwd_kernel<<<grid, 256, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace moe
