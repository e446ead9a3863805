// S8 support kernel: token-direction MXFP8 quantisation of the weight-gradient operands.
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
// zeros).  The result is stored transposed ([C, R], K-major for the GEMM).
//
// Shared-memory staged: see transpose_quant_kernel.  C % 128 == 0 (d, f, 2f all are).
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ float e4m3_to_f32_t(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
  const float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20))
                    : static_cast<float>(m) * 0.001953125f;
  return (c & 0x80u) ? -v : v;
}

__device__ __forceinline__ float e8m0_to_f32_t(uint32_t b) {
  return b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

constexpr int kTqThreads = 256;
constexpr int kTqRows = 128;     // rows (tokens) per block: four 32-row quantisation blocks
constexpr int kTqCols = 128;     // columns per block
constexpr int kTqPitch = kTqCols + 16;
constexpr int kTqMaxE = 1024;

// Block = 128 rows x 128 columns.  Codes are staged in shared memory with coalesced
// 16-byte loads (8 threads per 128-byte row) and each row's four scales of these columns
// arrive as one 32-bit word; then thread (column c, half hb) walks down column c for two
// 32-row blocks, dequantises (times the row's combine weight for w * dout^), requantises
// along the rows and writes 32 bytes of the transposed output.
__global__ void __launch_bounds__(kTqThreads) transpose_quant_kernel(TransposeQuantParams P) {
  __shared__ __align__(16) uint8_t s_codes[kTqRows][kTqPitch];
  __shared__ float s_mul[kTqCols / 32][kTqRows];  // 2^s of (row, 32-column block) x weight
  __shared__ int s_pad[kTqMaxE + 1];
  const int64_t p0 = static_cast<int64_t>(blockIdx.y) * kTqRows;  // first row of the block
  const int c0 = blockIdx.x * kTqCols;                              // first column
  const int tid = threadIdx.x;
  for (int i = tid; i <= P.E; i += kTqThreads) s_pad[i] = P.pad_offsets[i];
  __syncthreads();
  // expert of the 128-row block (segments start on 128-row boundaries) and valid rows
  int lo = 0, hi = P.E;  // s_pad[lo] <= p0 < s_pad[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_pad[mid] <= p0) lo = mid; else hi = mid;
  }
  const int64_t rel = p0 - s_pad[lo];
  int nv_blk = static_cast<int>(P.counts[lo] - rel);
  if (p0 >= s_pad[P.E]) nv_blk = 0;
  nv_blk = nv_blk < 0 ? 0 : (nv_blk > kTqRows ? kTqRows : nv_blk);
  if (tid < kTqRows) {
    float w = 0.f;
    uint32_t sw = 0;
    if (tid < nv_blk) {
      w = P.src == TSRC_MX_W ? P.topk_w[P.perm[P.offsets[lo] + rel + tid]] : 1.f;
      sw = *reinterpret_cast<const uint32_t*>(P.s + umma_scale_offset(p0 + tid, c0 >> 5,
                                                                       P.C >> 7));
    }
#pragma unroll
    for (int cb = 0; cb < kTqCols / 32; ++cb)
      s_mul[cb][tid] = e8m0_to_f32_t((sw >> (8 * cb)) & 0xFFu) * w;
  }
  // codes: 128 rows x 128 bytes, 8 threads per row, 16 bytes each
#pragma unroll
  for (int it = 0; it < (kTqRows * kTqCols / 16) / kTqThreads; ++it) {
    const int idx = it * kTqThreads + tid;
    const int r = idx >> 3, ch = idx & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < nv_blk)
      v = *reinterpret_cast<const uint4*>(P.q + (p0 + r) * P.C + c0 + ch * 16);
    *reinterpret_cast<uint4*>(&s_codes[r][ch * 16]) = v;
  }
  __syncthreads();
  const int c = tid & (kTqCols - 1);  // column within the block
  const int hb = tid >> 7;            // 32-row blocks hb and hb + 2
  const float* mul = s_mul[c >> 5];
#pragma unroll 1
  for (int bb = 0; bb < 2; ++bb) {
    const int b = hb + 2 * bb;
    float v[32];
#pragma unroll
    for (int r = 0; r < 32; r += 2) {  // rows r, r+1: one hardware E4M3x2 -> f16x2 decode
      const int rr = 32 * b + r;
      const uint32_t pair = static_cast<uint32_t>(s_codes[rr][c]) |
                            (static_cast<uint32_t>(s_codes[rr + 1][c]) << 8);
      uint32_t h2;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(pair)));
      // rows past the segment's count have multiplier 0 (and zero codes)
      v[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu))) * mul[rr];
      v[r + 1] =
          __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16))) * mul[rr + 1];
    }
    uint32_t qw[8];
    const uint32_t sb = mx_quant_block32(v, qw);
    const int64_t pb = p0 + 32 * b;
    uint4* dst = reinterpret_cast<uint4*>(P.dst_q + static_cast<int64_t>(c0 + c) * P.R + pb);
    dst[0] = make_uint4(qw[0], qw[1], qw[2], qw[3]);
    dst[1] = make_uint4(qw[4], qw[5], qw[6], qw[7]);
    P.dst_s[umma_scale_offset(c0 + c, pb >> 5, P.R >> 7)] = static_cast<uint8_t>(sb);
  }
}

cudaError_t launch_transpose_quant(const TransposeQuantParams& P, cudaStream_t stream) {
  if (P.R <= 0 || P.C <= 0) return cudaSuccess;
  dim3 grid(P.C / kTqCols, static_cast<unsigned>(P.R / kTqRows));
  transpose_quant_kernel<<<grid, kTqThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// SwiGLU backward and d(router weights), one warp per assignment row, after the dgrad GEMM
// of the down projection has written G = dout^ . Wd'^T (fp32, padded expert order):
//   dw_route[a] = <G, h^>,  dh = w * G,  dg = dh * u * s * (1 + g (1 - s)),
//   du = dh * g * s,  s = sigmoid(g)  (g, u: the saved bf16 pre-activations),
// then [dg | du] quantised to MXFP8 along f (the operand of the dX GEMM).  Lane l covers 8
// consecutive features per 256-feature step; four lanes share a 32-feature MX block.
// ---------------------------------------------------------------------------------------
constexpr int kSbMaxE = 1024;

__device__ __forceinline__ float sigmoid_fast_b(float x) { return __frcp_rn(1.f + __expf(-x)); }

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
        dwp = fmaf(Gv[i], e4m3_to_f32_t(code) * hsc, dwp);
        const float gb = bf16_bits_to_f32((gw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
        const float ub = bf16_bits_to_f32((uw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
        const float dh = w * Gv[i];
        const float sg = sigmoid_fast_b(gb);
        dg[i] = dh * ub * sg * (1.f + gb * (1.f - sg));
        du[i] = dh * gb * sg;
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
