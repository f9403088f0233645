// common.cuh -- device helpers shared by the pkv kernels (sm_100a).
//
// Holds no quantization or attention arithmetic of its own beyond the integer -> float code
// conversion; the method's steps live in store_impl.cuh, decode_kernel.cuh and copy_impl.cuh.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pkv.h"

namespace pkv {

// First error wins: only a zero slot is overwritten.
__device__ __forceinline__ void record_error(int32_t* dev_error, int32_t code) {
  if (dev_error != nullptr) atomicCAS(dev_error, 0, code);
}

// atomicInc with no ordering of its own (a split-unit ticket taken after a separate release
// fence; the warp that gets the last ticket fences again before reading the partials).
__device__ __forceinline__ uint32_t atomic_inc_relaxed_gpu(uint32_t* addr, uint32_t wrap) {
  uint32_t old;
  asm volatile("atom.relaxed.gpu.global.inc.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(wrap) : "memory");
  return old;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// ---- integer code -> float conversion without I2F -------------------------------------------
// IEEE-754 binary32 with exponent field 150 (bit pattern 0x4B000000 | m, m < 2^23) is exactly
// 2^23 + m. Placing a biased byte in the low mantissa bits and subtracting the bias as a float
// therefore yields the integer exactly (the "magic number" conversion of integer fields through
// the float bit layout; see e.g. Kim et al., "Who Says Elephants Can't Run", 2022).
constexpr float kMagic = 8388608.0f;  // 2^23

// byte i of w (as unsigned, 0..255) placed into the mantissa: returns 2^23 + byte
__device__ __forceinline__ float byte_to_magic(uint32_t w, int i) {
  // result bytes: [w.byte_i, 0x00, 0x00, 0x4B] taken from {w, 0x4B000000}
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7650u + (uint32_t)i));
}

// 4 signed int8 codes packed in w -> 4 exact floats (c0 is the lowest byte)
__device__ __forceinline__ void s8x4_to_f32(uint32_t w, float& f0, float& f1, float& f2, float& f3) {
  const uint32_t u = w ^ 0x80808080u;  // c + 128 in 0..255
  const float bias = kMagic + 128.0f;
  f0 = byte_to_magic(u, 0) - bias;
  f1 = byte_to_magic(u, 1) - bias;
  f2 = byte_to_magic(u, 2) - bias;
  f3 = byte_to_magic(u, 3) - bias;
}

// Packed forms for the sm_100 paired fp32 pipe (__fadd2_rn / __ffma2_rn): one FADD2 removes the
// bias from two codes. `neg_bias` = -(2^23 + bias) in both lanes.
__device__ __forceinline__ void s8x4_to_f32x2(uint32_t w, float2& lo, float2& hi) {
  const uint32_t u = w ^ 0x80808080u;  // c + 128 in 0..255
  const float2 neg_bias = make_float2(-(kMagic + 128.0f), -(kMagic + 128.0f));
  lo = __fadd2_rn(make_float2(byte_to_magic(u, 0), byte_to_magic(u, 1)), neg_bias);
  hi = __fadd2_rn(make_float2(byte_to_magic(u, 2), byte_to_magic(u, 3)), neg_bias);
}

// 8 unsigned 4-bit codes (nibble k = dim k) -> 4 float2 of (code - zp), dims in order.
__device__ __forceinline__ void u4x8_to_f32x2(uint32_t w, float2 neg_bias, float2 f[4]) {
  const uint32_t even = w & 0x0F0F0F0Fu;        // nibbles 0,2,4,6 in bytes 0..3
  const uint32_t odd = (w >> 4) & 0x0F0F0F0Fu;  // nibbles 1,3,5,7
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f[i] = __fadd2_rn(make_float2(byte_to_magic(even, i), byte_to_magic(odd, i)), neg_bias);
}

// 8 unsigned 4-bit codes packed in w (nibble k = dim k, low nibble first) -> (code - zp) exact.
// bias = 2^23 + zp.
__device__ __forceinline__ void u4x8_to_f32(uint32_t w, float bias, float f[8]) {
  const uint32_t even = w & 0x0F0F0F0Fu;         // nibbles 0,2,4,6 in bytes 0..3
  const uint32_t odd = (w >> 4) & 0x0F0F0F0Fu;   // nibbles 1,3,5,7
  f[0] = byte_to_magic(even, 0) - bias;
  f[1] = byte_to_magic(odd, 0) - bias;
  f[2] = byte_to_magic(even, 1) - bias;
  f[3] = byte_to_magic(odd, 1) - bias;
  f[4] = byte_to_magic(even, 2) - bias;
  f[5] = byte_to_magic(odd, 2) - bias;
  f[6] = byte_to_magic(even, 3) - bias;
  f[7] = byte_to_magic(odd, 3) - bias;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- mbarrier + bulk asynchronous copy (global -> shared) -----------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// 1-D bulk copy; dst, src 16-byte aligned, bytes a multiple of 16. Completion is signalled on
// `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Tiled tensor copies (TMA) of one box into shared memory, completing on `bar` as transaction
// bytes. `map` is a tensor map in kernel parameter space; x (the innermost coordinate) is 0 at
// every call site, so the box starts on a 16-byte boundary.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// One bounded probe of the barrier phase; true once phase `parity` has completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait with an iteration cap. Returns false if the cap was reached (the caller reports
// PKV_DEVERR_TIMEOUT and stops issuing work). Each try_wait already suspends for a
// hardware-chosen interval, so the cap bounds the wait to well under a few seconds.
constexpr uint32_t kMaxWaitIters = 1u << 22;
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kMaxWaitIters; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
  }
  return false;
}

}  // namespace pkv
