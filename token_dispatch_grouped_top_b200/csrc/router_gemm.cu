// The router GEMM in front of the routing step (logits = x . W_r^T, fp32) and its
// backward (dx_r = bf16(G) . W_r, dW_r = bf16(G)^T . x), run on the grouped GEMM engine's
// bf16 mode (tcgen05.mma kind::f16, fp32 accumulation in TMEM) as one-group problems.
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72", lead and
// §01: the router decides at every step which experts each token goes to, so training also
// differentiates through it.  The pages give no formula for it; it is read as a bias-free
// linear layer whose outputs are the logits the routing step ranks.
//
// This file holds what the GEMMs need around them: the tile lists of a one-group problem
// (its tile prefix, valid rows and a zeroed tile counter, written on the device so a call
// never copies from the host), and zero-padded bf16 copies of the operands, so that every
// TMA box the GEMM loads lies inside its tensor: W_r padded to whole 256-row N tiles, the
// logits' gradient rounded to bf16 and padded to whole 64-element K blocks, and the
// transposes the weight gradient reduces over (G^T and x^T, K = tokens).
#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ uint16_t to_bf16_bits(uint16_t v) { return v; }
__device__ __forceinline__ uint16_t to_bf16_bits(float v) {
  return static_cast<uint16_t>(pack_bf16x2(v, 0.f) & 0xFFFFu);  // nearest, ties to even
}

__global__ void router_setup_kernel(RouterSetupParams P) {
  const int i = threadIdx.x;
  if (i < P.n) {
    P.prefix[2 * i] = 0;
    const int64_t rows = i == 0 ? P.rows[0] : i == 1 ? P.rows[1] : P.rows[2];
    P.prefix[2 * i + 1] = static_cast<int32_t>((rows + 127) / 128);
    P.valid[i] = static_cast<int32_t>(rows);
    P.ctr[i] = 0u;
  }
}

cudaError_t launch_router_setup(const RouterSetupParams& P, cudaStream_t stream) {
  if (P.n < 1 || P.n > 3) return cudaErrorInvalidValue;
  router_setup_kernel<<<1, 32, 0, stream>>>(P);
  return cudaGetLastError();
}

// dst[r][c] = (r < R && c < C) ? bf16(src[r * ld + c]) : 0 over dst [dst_rows, dst_cols].
template <typename SrcT>
__global__ void __launch_bounds__(256) pad_copy_kernel(const SrcT* __restrict__ src, int64_t R,
                                                       int64_t C, int64_t ld, uint16_t* dst,
                                                       int64_t dst_rows, int64_t dst_cols) {
  const int64_t n = dst_rows * dst_cols;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / dst_cols, c = i - r * dst_cols;
    dst[i] = (r < R && c < C) ? to_bf16_bits(src[r * ld + c]) : static_cast<uint16_t>(0);
  }
}

// 64 x 64 tiles through shared memory: dst[c][r] = (r < R && c < C) ? bf16(src[r][c]) : 0.
// Block (bx, by) covers source rows 64 bx.. (destination columns) and source columns 64 by..
// (destination rows); both global passes walk 64 consecutive elements per row.
template <typename SrcT>
__global__ void __launch_bounds__(256) transpose_pad_kernel(const SrcT* __restrict__ src,
                                                            int64_t R, int64_t C, int64_t ld,
                                                            uint16_t* dst, int64_t dst_rows,
                                                            int64_t dst_cols) {
  __shared__ uint16_t tile[64][66];  // [source row][source column], padded rows
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int64_t c0 = static_cast<int64_t>(blockIdx.y) * 64;
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int rr = i >> 6, cc = i & 63;
    const int64_t r = r0 + rr, c = c0 + cc;
    tile[rr][cc] = (r < R && c < C) ? to_bf16_bits(src[r * ld + c]) : static_cast<uint16_t>(0);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 64 * 64; i += 256) {
    const int cr = i >> 6, rc = i & 63;
    const int64_t dr = c0 + cr, dc = r0 + rc;
    if (dr < dst_rows && dc < dst_cols) dst[dr * dst_cols + dc] = tile[rc][cr];
  }
}

template <typename SrcT>
static cudaError_t pad_copy(const SrcT* src, int64_t R, int64_t C, int64_t ld, uint16_t* dst,
                            int64_t dst_rows, int64_t dst_cols, cudaStream_t stream) {
  if (dst_rows < R || dst_cols < C || ld < C) return cudaErrorInvalidValue;
  const int64_t n = dst_rows * dst_cols;
  if (n == 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  pad_copy_kernel<SrcT><<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(
      src, R, C, ld, dst, dst_rows, dst_cols);
  return cudaGetLastError();
}

template <typename SrcT>
static cudaError_t transpose_pad(const SrcT* src, int64_t R, int64_t C, int64_t ld,
                                 uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                 cudaStream_t stream) {
  if (dst_rows < C || dst_cols < R || ld < C) return cudaErrorInvalidValue;
  const int64_t bx = (dst_cols + 63) / 64, by = (dst_rows + 63) / 64;
  if (bx == 0 || by == 0) return cudaSuccess;
  if (bx > 0x7fffffffLL || by > 65535) return cudaErrorInvalidValue;
  transpose_pad_kernel<SrcT><<<dim3(static_cast<unsigned>(bx), static_cast<unsigned>(by)), 256,
                               0, stream>>>(src, R, C, ld, dst, dst_rows, dst_cols);
  return cudaGetLastError();
}

cudaError_t launch_pad_copy_bf16(const uint16_t* src, int64_t R, int64_t C, int64_t ld,
                                 uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                 cudaStream_t stream) {
  return pad_copy(src, R, C, ld, dst, dst_rows, dst_cols, stream);
}
cudaError_t launch_pad_copy_f32_bf16(const float* src, int64_t R, int64_t C, int64_t ld,
                                     uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                     cudaStream_t stream) {
  return pad_copy(src, R, C, ld, dst, dst_rows, dst_cols, stream);
}
cudaError_t launch_transpose_pad_bf16(const uint16_t* src, int64_t R, int64_t C, int64_t ld,
                                      uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                      cudaStream_t stream) {
  return transpose_pad(src, R, C, ld, dst, dst_rows, dst_cols, stream);
}
cudaError_t launch_transpose_pad_f32_bf16(const float* src, int64_t R, int64_t C, int64_t ld,
                                          uint16_t* dst, int64_t dst_rows, int64_t dst_cols,
                                          cudaStream_t stream) {
  return transpose_pad(src, R, C, ld, dst, dst_rows, dst_cols, stream);
}

}  // namespace moe
