// Weight repacks of the companion path (streaming, HBM-bound).
//
// MXFP4 -> NVFP4: "DeepSeek-V4-Pro-0813-nvfp4-DSpark" walkthrough, 阶段三 and
// its storage table: E2M1 nibbles move unchanged, each E8M0 scale per 32
// becomes E4M3 scales per 16 (the page: scale bytes double).  An E8M0 scale
// 2^e is written as two E4M3 codes of 2^(e - G); G is chosen per matrix so
// every exponent fits E4M3's exact powers of two 2^-9 .. 2^8.
//
// MXFP4 -> symmetric INT4 group 128: "DeepSeek-V4-Flash-0731-W4AFP8-mt",
// 量化方式 / 权重约定: signed INT4 two per int8, float32 scale_inv [N, K/128].
#pragma once

#include "common.cuh"

namespace moe {

// Pass 1: one block per matrix; min / max block exponent -> G; 2^G stored
// in out_global[m] (float32, possibly subnormal).
__global__ void __launch_bounds__(256) nvfp4_global_kernel(const uint8_t* __restrict__ e8m0, int64_t per_mat,
                                                           float* __restrict__ out_global) {
  const int64_t m = blockIdx.x;
  const uint8_t* s = e8m0 + m * per_mat;
  int lo = 255, hi = 0, nan = 0;
  for (int64_t i = threadIdx.x; i < per_mat; i += blockDim.x) {
    const int b = __ldg(s + i);
    nan |= (b == 255);
    lo = min(lo, b);
    hi = max(hi, b);
  }
  lo = __reduce_min_sync(0xFFFFFFFFu, lo);
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  nan = __reduce_or_sync(0xFFFFFFFFu, nan);
  __shared__ int s_lo[8], s_hi[8], s_nan[8];
  const int wid = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) { s_lo[wid] = lo; s_hi[wid] = hi; s_nan[wid] = nan; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) {
      lo = min(lo, s_lo[i]);
      hi = max(hi, s_hi[i]);
      nan |= s_nan[i];
    }
    lo = min(lo, s_lo[0]);
    hi = max(hi, s_hi[0]);
    nan |= s_nan[0];
    int G = 0;
    if (nan) {
      record_error(MOE_ERR_NAN_SCALE);
    } else {
      const int elo = lo - 127, ehi = hi - 127;
      if (elo >= -9 && ehi <= 8) G = 0;
      else if (ehi - elo <= 17) G = ehi - 8;
      else record_error(MOE_ERR_RANGE);
    }
    out_global[m] = exp2_int(G);
  }
}

__device__ __forceinline__ int exponent_of_pow2(float v) {
  const uint32_t b = __float_as_uint(v);
  const int e = (int)(b >> 23) & 0xFF;
  return e ? e - 127 : (31 - __clz((int)b)) - 149;
}

// E4M3 code of 2^j for j in [-9, 8] (normal for j >= -6, subnormal below).
__device__ __forceinline__ uint32_t e4m3_pow2_code(int j) {
  return j >= -6 ? (uint32_t)(j + 7) << 3 : 1u << (j + 9);
}

// Pass 2: grid-stride over scale bytes (4 at a time) and, when not aliased,
// over the nibble bytes (16 at a time).
__global__ void __launch_bounds__(256) nvfp4_convert_kernel(const uint8_t* __restrict__ e8m0, int64_t n_scale,
                                                            int64_t per_mat, const float* __restrict__ glob,
                                                            uint8_t* __restrict__ out_e4m3,
                                                            const uint4* __restrict__ fp4, uint4* __restrict__ out_fp4,
                                                            int64_t n_fp4_16) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t i = tid; i < n_scale; i += stride) {
    const int64_t m = i / per_mat;
    const int G = exponent_of_pow2(__ldg(glob + m));
    int j = (int)__ldg(e8m0 + i) - 127 - G;
    j = max(-9, min(8, j));                          // only out of range after a recorded error
    const uint32_t c = e4m3_pow2_code(j);
    reinterpret_cast<uint16_t*>(out_e4m3)[i] = (uint16_t)(c | (c << 8));
  }
  if (out_fp4 != nullptr)
    for (int64_t i = tid; i < n_fp4_16; i += stride) out_fp4[i] = __ldg(fp4 + i);
}

// INT4 group-128: one thread per (row, group of 128): 64 nibble bytes and 4
// scale bytes in, 64 bytes and one float32 out.
__global__ void __launch_bounds__(256) int4g128_kernel(const uint4* __restrict__ fp4, const uint32_t* __restrict__ e8m0,
                                                       int64_t n_groups, uint4* __restrict__ out,
                                                       float* __restrict__ scale_inv) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= n_groups) return;
  const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  uint4 in[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) in[i] = __ldg(fp4 + g * 4 + i);
  const uint32_t sb = __ldg(e8m0 + g);
  // exact float32 block maxima
  float amax = 0.0f;
  bool bad = false;
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    const int b = (sb >> (8 * blk)) & 0xFF;
    if (b == 255) { bad = true; continue; }
    const uint32_t* words = reinterpret_cast<const uint32_t*>(&in[blk]);
    uint32_t mc = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int n = 0; n < 8; ++n) mc = max(mc, (words[w] >> (4 * n)) & 7u);
    const float bm = __fmul_rn(kE2M1[mc], exp2_int(b - 127));
    if (isinf(bm)) record_error(MOE_ERR_RANGE);
    amax = fmaxf(amax, bm);
  }
  if (bad) { record_error(MOE_ERR_NAN_SCALE); return; }
  const float sinv = amax > 0.0f ? __fdiv_rn(amax, 7.0f) : 1.0f;
  scale_inv[g] = sinv;
  uint4 res[4];
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    const int b = (sb >> (8 * blk)) & 0xFF;
    const float sc = exp2_int(b - 127);
    // quantised magnitude of each of the 8 E2M1 magnitudes in this block
    uint32_t qm = 0;                                   // 8 x 4-bit table
#pragma unroll
    for (int c = 1; c < 8; ++c) {
      const float x = __fmul_rn(kE2M1[c], sc);
      const float q = fminf(rintf(__fdiv_rn(x, sinv)), 7.0f);
      qm |= (uint32_t)q << (4 * c);
    }
    const uint32_t* words = reinterpret_cast<const uint32_t*>(&in[blk]);
    uint32_t* ow = reinterpret_cast<uint32_t*>(&res[blk]);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t o = 0;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const uint32_t nib = (words[w] >> (4 * n)) & 0xFu;
        const uint32_t mag = (qm >> (4 * (nib & 7u))) & 0xFu;
        const uint32_t q = (nib & 8u) ? ((16u - mag) & 0xFu) : mag;   // two's complement
        o |= q << (4 * n);
      }
      ow[w] = o;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) out[g * 4 + i] = res[i];
}

}  // namespace moe
