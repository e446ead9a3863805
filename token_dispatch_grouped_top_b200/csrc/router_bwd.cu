// Router backward: d(loss)/d(logits) from d(loss)/d(combine weights).
//
// Article "Cursor's MoK achieves 2.37x performance boost on NVIDIA GB300 NVL72", lead and
// §01: the router decides at every training step which experts each token goes to, so
// training needs the gradient that reaches the router's logits through the combine
// weights.  The top-k selection is piecewise constant in the logits: only the k selected
// logits of a token receive a gradient, the other E - k get exactly zero.  Through the
// weights it is the chain rule of the two score functions:
//   softmax over the k selected logits:  dl_i = w_i (dw_i - sum_j w_j dw_j)
//   sigmoid scores renormalised:         dl_i = s_i (1 - s_i) (dw_i - sum_j w_j dw_j) / S,
//                                        s_i = sigmoid(l_i), S = sum_j s_j, w_i = s_i / S
// The weights are recomputed from the logits exactly as the routing kernel forms them
// (a NaN logit counts as -inf).
//
// One warp per token, lane j < k holds slot j; the row of E outputs is written as zeros
// with 16-byte stores, then the k selected entries.  HBM-bound: 4*E bytes written and
// 12*k bytes read per token.
#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void __launch_bounds__(256) router_bwd_kernel(RouterBwdParams P) {
  const int lane = threadIdx.x & 31;
  const int E = P.E, k = P.k;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
       t < P.T; t += warps) {
    int e = 0;
    float l = -INFINITY, dw = 0.f;
    bool bad = false;
    if (lane < k) {
      e = P.topk_idx[t * k + lane];
      if (e < 0 || e >= E) {
        bad = true;
        e = 0;
      }
      const float raw = P.logits[t * E + e];
      l = raw != raw ? -INFINITY : raw;
      dw = P.dw_route[t * k + lane];
    }
    if (__any_sync(kFull, bad)) {
      if (lane == 0) latch(P.status, MOE_ERR_DEVICE_BOUNDS);
      continue;
    }
    float score, grad;
    if (P.score_fn == MOE_SCORE_SOFTMAX_TOPK) {
      float m = l;  // the largest selected logit
#pragma unroll
      for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
      score = lane < k ? expf(l - m) : 0.f;
    } else {
      score = lane < k ? 1.f / (1.f + expf(-l)) : 0.f;
    }
    float S = score;
#pragma unroll
    for (int off = 16; off; off >>= 1) S += __shfl_xor_sync(kFull, S, off);
    const float w = score / S;
    float wdw = lane < k ? w * dw : 0.f;
#pragma unroll
    for (int off = 16; off; off >>= 1) wdw += __shfl_xor_sync(kFull, wdw, off);
    const float centred = dw - wdw;
    if (P.score_fn == MOE_SCORE_SOFTMAX_TOPK)
      grad = w * centred;
    else
      grad = centred / S * score * (1.f - score);
    float* row = P.dlogits + t * E;
    if ((E & 3) == 0) {
      for (int c = lane * 4; c < E; c += 128)
        *reinterpret_cast<float4*>(row + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      for (int c = lane; c < E; c += 32) row[c] = 0.f;
    }
    __syncwarp();
    if (lane < k) row[e] = grad;
  }
}

cudaError_t launch_router_bwd(const RouterBwdParams& P, int num_sms, cudaStream_t stream) {
  if (P.T <= 0) return cudaSuccess;
  const int64_t blocks = (P.T + 7) / 8;
  const int grid = static_cast<int>(blocks < 16LL * num_sms ? blocks : 16LL * num_sms);
  router_bwd_kernel<<<grid, 256, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace moe
