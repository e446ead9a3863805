// S8 support kernel: token-direction MXFP8 quantisation of the weight-gradient operands.
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72", §01/§02:
// training adds a backward pass with two reverse communications (pull reverse-combine of
// the output gradient, push reverse-dispatch of the input gradient); the weight gradients
// of each expert reduce over that expert's tokens.  A block-scaled GEMM needs its operands
// quantised along the reduction axis, which for the weight gradients is the token axis:
// blocks of 32 consecutive tokens inside one expert's segment (segments start on 128-row
// boundaries, so a block never straddles two experts; rows past the segment's count are
// zeros).  The result is stored transposed ([C, R], K-major for the GEMM).
//
// One thread per (32-token block, column): 32 strided reads (coalesced across the warp's
// consecutive columns), one scale, 32 contiguous output bytes.
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

__global__ void __launch_bounds__(kTqThreads) transpose_quant_kernel(TransposeQuantParams P) {
  __shared__ int s_row_t[32];
  __shared__ float s_row_w[32];
  __shared__ int s_nvalid;
  const int64_t p0 = static_cast<int64_t>(blockIdx.y) * 32;  // first row of the block
  const int c = blockIdx.x * kTqThreads + threadIdx.x;        // column
  if (threadIdx.x == 0) {
    int lo = 0, hi = P.E;  // segment containing p0: pad[lo] <= p0 < pad[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (P.pad_offsets[mid] <= p0) lo = mid; else hi = mid;
    }
    const int64_t rel = p0 - P.pad_offsets[lo];
    int nv = static_cast<int>(P.counts[lo] - rel);
    nv = nv < 0 ? 0 : (nv > 32 ? 32 : nv);
    if (p0 >= P.pad_offsets[P.E]) nv = 0;
    s_nvalid = nv;
    if (P.src == TSRC_DY) {
      for (int r = 0; r < nv; ++r) {
        const int a = P.perm[P.offsets[lo] + rel + r];
        s_row_t[r] = a / P.k;
        s_row_w[r] = P.topk_w[a];
      }
    }
  }
  __syncthreads();
  if (c >= P.C) return;
  const int nv = s_nvalid;
  float v[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    float x = 0.f;
    if (r < nv) {
      const int64_t row = p0 + r;
      if (P.src == TSRC_MX) {
        const uint32_t code = P.q[row * P.C + c];
        const uint32_t sb = P.s[umma_scale_offset(row, c >> 5, P.C >> 7)];
        x = e4m3_to_f32_t(code) * e8m0_to_f32_t(sb);
      } else if (P.src == TSRC_BF16) {
        x = bf16_bits_to_f32(P.bf[row * P.ld + c]);
      } else {
        const float dy = s_row_w[r] * bf16_bits_to_f32(P.bf[static_cast<int64_t>(s_row_t[r]) *
                                                             P.ld + c]);
        x = bf16_bits_to_f32(f32_to_bf16_bits(dy));  // dy is materialised in bf16
      }
    }
    v[r] = x;
  }
  uint32_t qw[8];
  const uint32_t sb = mx_quant_block32(v, qw);
  uint4* dst = reinterpret_cast<uint4*>(P.dst_q + static_cast<int64_t>(c) * P.R + p0);
  dst[0] = make_uint4(qw[0], qw[1], qw[2], qw[3]);
  dst[1] = make_uint4(qw[4], qw[5], qw[6], qw[7]);
  P.dst_s[umma_scale_offset(c, p0 >> 5, P.R >> 7)] = static_cast<uint8_t>(sb);
}

cudaError_t launch_transpose_quant(const TransposeQuantParams& P, cudaStream_t stream) {
  if (P.R <= 0 || P.C <= 0) return cudaSuccess;
  dim3 grid((P.C + kTqThreads - 1) / kTqThreads, static_cast<unsigned>(P.R / 32));
  transpose_quant_kernel<<<grid, kTqThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace moe
