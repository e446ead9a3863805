// Device helpers shared by the kernels of the MoE layer: status latching, bounded waits,
// inline PTX for mbarriers, TMA, and the 5th-generation tensor core (tcgen05 / TMEM), and
// the MXFP8 (E4M3 + E8M0) block quantiser.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr uint32_t kFull = 0xffffffffu;

// ----------------------------------------------------------------------------------------
// device status: the first error wins and stays latched until the host reads it
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void latch(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// A device-side wait gives up after this long and latches MOE_ERR_DEVICE_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// ----------------------------------------------------------------------------------------
// shared memory / mbarrier
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity has completed.  Bounded: after
// kWaitLimitNs (or once another role raised *abort) it latches a timeout, raises *abort
// and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        latch(status, MOE_ERR_DEVICE_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

// Waits for the phase with the given parity without giving up when another role aborts
// (used on the way out, to let this thread's own asynchronous copies or MMAs land before
// the CTA exits); still bounded by kWaitLimitNs.
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ----------------------------------------------------------------------------------------
// device-wide signalling between kernels that run at the same time
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ int32_t ld_acquire_s32(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(int32_t* p, int32_t v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Orders this thread's earlier generic-proxy view of global memory (e.g. data another
// kernel published behind an acquire) before its later async-proxy (TMA) reads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Programmatic dependent launch: let the next kernel in the stream start launching now.
__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Programmatic dependent launch: wait until the previous kernel in the stream has
// completed and its memory operations are visible.
__device__ __forceinline__ void wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Bounded wait until a count-down counter published by another kernel reaches zero.
__device__ __forceinline__ bool wait_counter_zero(const int32_t* ctr, volatile int* abort,
                                                  int32_t* status) {
  if (ld_acquire_s32(ctr) <= 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    __nanosleep(128);
    if (ld_acquire_s32(ctr) <= 0) return true;
    if ((i & 15u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        latch(status, MOE_ERR_DEVICE_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t smem_dst, const void* tmap, uint32_t bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t smem_dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Untiled bulk copy shared -> global (bulk-group completion; 16-byte aligned, size a
// multiple of 16).
__device__ __forceinline__ void bulk_store(void* dst, uint32_t smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_src), "r"(bytes)
               : "memory");
}

// TMA tensor store shared -> global (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t smem_src, int32_t x,
                                             int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(smem_src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ----------------------------------------------------------------------------------------
// tcgen05 / TMEM
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_result),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major operand tile written by TMA with 128-byte
// swizzle: rows of 128 bytes, 8-row swizzle atoms stacked every 1024 bytes.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address  [0,14)
  d |= static_cast<uint64_t>(1) << 16;                   // leading offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;           // stride offset   [32,46)
  d |= static_cast<uint64_t>(1) << 46;                   // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                   // 128-byte swizzle
  return d;
}

// Descriptor of a 32-row x 16-byte scale chunk (no swizzle, rows packed every 16 bytes,
// 8-row core matrices every 128 bytes) -- the source of tcgen05.cp .32x128b.
__device__ __forceinline__ uint64_t sdesc_scale_chunk(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(128 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Instruction descriptor, kind::mxf8f6f4 with block scaling: A and B E4M3 (format 0),
// both K-major, scale type E8M0, D fp32, shape M x N.  The scale-factor byte selectors
// (bits 29-30 for A, 4-5 for B) are or-ed in per MMA.
__host__ __device__ constexpr uint32_t idesc_mxf8_e4m3(int M, int N) {
  return (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate, uint32_t sfa_tmem,
                                         uint32_t sfb_tmem) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor, kind::f16 with A and B bf16 (format 1), both K-major, D fp32
// (format 1), shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// D (+)= A . B^T with bf16 operands in shared memory (K = 16 elements = 32 bytes per MMA).
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// Copy a 32-row x 128-bit scale chunk from shared memory into TMEM, replicated into the
// four 32-lane quarters.
__device__ __forceinline__ void tmem_cp_scales(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ----------------------------------------------------------------------------------------
// MXFP8 quantisation (OCP MX v1.0: s = floor(log2 amax) - 8, clamped to [-127, 127];
// elements x * 2^-s rounded to E4M3 with round-to-nearest-even and saturation)
// ----------------------------------------------------------------------------------------

// Block scale exponent from the block's absolute maximum.  The exponent field of amax is
// floor(log2 amax) for normal values; zero and subnormal amax give -127, which clamps to
// the same s = -127 as the exact rule.
__device__ __forceinline__ int mx_scale_exp(float amax) {
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
  return max(min(e - 8, 127), -127);
}

// 2^-s as an fp32 (always a normal number for s in [-127, 119]).
__device__ __forceinline__ float mx_inv_scale(int s) {
  return __uint_as_float(static_cast<uint32_t>(127 - s) << 23);
}

// Two fp32 -> two E4M3 bytes (lo in bits 0-7), RNE, saturate to +-448.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  return cvt_e4m3x2(a, b) | (cvt_e4m3x2(c, d) << 16);
}

// Quantise one 32-element block held by a single thread.  Writes 8 packed words.
__device__ __forceinline__ uint32_t mx_quant_block32(const float (&v)[32], uint32_t (&q)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int s = mx_scale_exp(amax);
  const float inv = mx_inv_scale(s);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    q[i] = pack_e4m3x4(v[4 * i] * inv, v[4 * i + 1] * inv, v[4 * i + 2] * inv, v[4 * i + 3] * inv);
  return static_cast<uint32_t>(s + 127);
}

// E4M3 code -> its value (exact in fp32); E8M0 byte -> 2^(b - 127) (byte 0: 2^-127).
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
  const float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20))
                    : static_cast<float>(m) * 0.001953125f;
  return (c & 0x80u) ? -v : v;
}

__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
  return b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

// sigmoid(x) = 1 / (1 + e^-x) with the fast exponential and a rounded reciprocal (relative
// error ~1e-6; large |x|: e^-x -> 0 or inf gives exactly 1 or 0).
__device__ __forceinline__ float sigmoid_fast(float x) { return __frcp_rn(1.f + __expf(-x)); }

// SwiGLU backward of one element, h = silu(g) * u: with dh = w * G,
// dg = dh * u * s * (1 + g (1 - s)), du = dh * g * s, s = sigmoid(g).
__device__ __forceinline__ void swiglu_bwd_elem(float G, float w, float g, float u, float& dg,
                                                float& du) {
  const float dh = w * G;
  const float s = sigmoid_fast(g);
  dg = dh * u * s * (1.f + g * (1.f - s));
  du = dh * g * s;
}

// Byte offset of the scale of (row r, 32-block kb) in the UMMA scale layout of a matrix
// with `kgroups` = K/128 column groups.
__host__ __device__ __forceinline__ int64_t umma_scale_offset(int64_t r, int64_t kb,
                                                              int64_t kgroups) {
  return (((r >> 7) * kgroups + (kb >> 2)) << 9) + ((r & 31) << 4) + (((r & 127) >> 5) << 2) +
         (kb & 3);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// ----------------------------------------------------------------------------------------
// Scaled fp16 ("F16S"), the storage of the fp32 intermediates that one kernel writes and
// the next one reads back (expert outputs y, the dgrad results G and dXa): 32 consecutive
// values share a power-of-two scale 2^s, stored as the byte s + 127, and each value is the
// fp16 (round to nearest even) of v * 2^-s.  s = floor(log2 amax) - 14 puts the block's
// largest magnitude in [2^14, 2^15), below the fp16 maximum; each value keeps 11
// significant bits (relative error <= 2^-12 of its binade), where fp32 would cost twice
// the bytes.
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ int f16s_scale_exp(float amax) {
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
  return max(min(e - 14, 113), -127);  // 2^-s stays a normal fp32 number
}

// Two fp32 -> two fp16 (lo in bits 0-15), round to nearest even.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^s from its stored byte s + 127 (byte 0: 2^-127, a subnormal fp32 number).
__device__ __forceinline__ float f16s_scale_value(uint32_t b) {
  return b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

// fp16 bits -> fp32 (exact).
__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}

// Two fp32 -> two bf16 (lo in bits 0-15), round to nearest even, one instruction.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace moe
