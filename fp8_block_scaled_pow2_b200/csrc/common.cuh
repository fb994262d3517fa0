// Shared device helpers of the MoE kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_fp8_pow2.h"

namespace moe {

// ---------------------------------------------------------------------------
// Device error word: the first non-zero status recorded by any kernel since
// the last moe_get_device_error().
// ---------------------------------------------------------------------------
__device__ int g_device_error = 0;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_error, 0, code); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// Power-of-two FP8 scale rule.  k = ceil(log2(amax / 448)), the divide in
// float32 round-to-nearest-even, the ceiling taken exactly from the bits of
// the quotient (normal and subnormal), clamped to [-127, 127]; k = 0 when
// amax == 0.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int pow2_scale_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  const float r = __fdiv_rn(amax, 448.0f);
  const uint32_t b = __float_as_uint(r);
  const int e = (int)((b >> 23) & 0xFFu);
  const uint32_t m = b & 0x7FFFFFu;
  int k;
  if (e == 0) {
    k = (m <= 1u) ? -149 : (32 - __clz((int)(m - 1u))) - 149;   // r = m * 2^-149
  } else {
    k = e - 127 + (m != 0u ? 1 : 0);
  }
  return max(-127, min(127, k));
}

// 2^e as a float for e in [-149, 127], built from the bit pattern (exact).
// Programmatic dependent launch (every kernel of this library is launched
// with programmatic stream serialization): pdl_trigger lets the next kernel
// on the stream be scheduled now, so its launch and local set-up overlap this
// kernel; pdl_wait blocks until the previous kernel on the stream has
// completed and its writes are visible.  Every kernel calls pdl_wait before
// its first read or write of global memory.  Both are no-ops for a kernel
// launched without the attribute.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float exp2_int(int e) {
  if (e >= -126) return __uint_as_float((uint32_t)(e + 127) << 23);
  return __uint_as_float(1u << (e + 149));
}

// Two floats -> two E4M3 bytes (round to nearest even, saturate to +-448);
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  return e4m3x2(a, b) | (e4m3x2(c, d) << 16);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Max over a warp of non-negative floats (their bit patterns order like ints).
__device__ __forceinline__ float warp_max_nonneg(float v) {
  return __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(v)));
}

// SwiGLU with symmetric clamp of gate and up.  silu uses the hardware
// exponential and the approximate divide: on the clamped range |g| <= 10 the
// documented bounds are 2 + floor(1.173 |g|) <= 13 ulp for __expf and 2 ulp
// for __fdividef (its denominator stays below 2^126), so h is within about
// 16 ulp of the correctly rounded float32 value.  Both the fused epilogue and
// the standalone kernel call this function, so they agree bit for bit.
__device__ __forceinline__ float swiglu_clamped(float g, float u, float limit) {
  g = fminf(fmaxf(g, -limit), limit);
  u = fminf(fmaxf(u, -limit), limit);
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace moe
