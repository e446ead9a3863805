// Epilogue helpers shared by the grouped GEMM kernels: bf16 packing and the staged TMA
// store of 32-row x 128-byte output chunks.
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ uint4 pack_bf16x8(const float* v) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                    pack_bf16x2(v[6], v[7]));
}

// Stage one 32-row x 128-byte chunk (row = lane) in shared memory with the 128-byte swizzle
// the output tensor map uses, then one lane stores it with TMA.  Two buffers per warp:
// before a buffer is rewritten, the store issued from it two chunks ago must have read it.
__device__ __forceinline__ void stage_and_store(uint8_t* buf, const uint4 (&row16)[8],
                                                const CUtensorMap* tmap, int32_t x, int32_t y,
                                                int lane) {
  if (lane == 0) bulk_wait_read<1>();
  __syncwarp();
  uint8_t* r = buf + lane * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<uint4*>(r + ((j ^ (lane & 7)) << 4)) = row16[j];
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmap, smem_u32(buf), x, y);
    bulk_commit();
  }
}

}  // namespace moe
