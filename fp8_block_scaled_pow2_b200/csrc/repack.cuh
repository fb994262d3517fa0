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
//
// MXFP4 -> FP8 E4M3 with a [128, 128] block scale: "DeepSeek-V4-Pro-0813-
// nvfp4-DSpark" walkthrough (the lossless MXFP4 seed: nibbles split from the
// int8, values looked up, scale rewritten per 128 block) and the
// "DeepSeek-V4-Flash-SI" model card's weight block size [128, 128].
#pragma once

#include <climits>

#include "common.cuh"

namespace moe {

// Pass 1: one block per matrix; min / max block exponent -> G; 2^G stored
// in out_global[m] (float32, possibly subnormal).
__global__ void __launch_bounds__(256) nvfp4_global_kernel(const uint8_t* __restrict__ e8m0, int64_t per_mat,
                                                           float* __restrict__ out_global) {
  pdl_trigger();
  pdl_wait();
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
  pdl_trigger();
  pdl_wait();
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

// Vector forms of the two NVFP4 passes, used when the scale arrays are
// 16-byte aligned and a matrix holds a multiple of 16 scales.
// Pass 1: min / max of the bytes 16 at a time (255 is the largest byte, so a
// NaN scale shows as max == 255).
__global__ void __launch_bounds__(512) nvfp4_global_vec_kernel(const uint4* __restrict__ e8m0, int64_t per_mat16,
                                                               float* __restrict__ out_global) {
  pdl_trigger();
  pdl_wait();
  const int64_t m = blockIdx.x;
  const uint4* s = e8m0 + m * per_mat16;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int64_t i = threadIdx.x; i < per_mat16; i += blockDim.x) {
    const uint4 v = __ldg(s + i);
    lo = __vminu4(lo, __vminu4(__vminu4(v.x, v.y), __vminu4(v.z, v.w)));
    hi = __vmaxu4(hi, __vmaxu4(__vmaxu4(v.x, v.y), __vmaxu4(v.z, v.w)));
  }
  lo = __vminu4(lo, lo >> 16);
  lo = min(lo & 0xFFu, (lo >> 8) & 0xFFu);
  hi = __vmaxu4(hi, hi >> 16);
  hi = max(hi & 0xFFu, (hi >> 8) & 0xFFu);
  int l = __reduce_min_sync(0xFFFFFFFFu, (int)lo);
  int h = __reduce_max_sync(0xFFFFFFFFu, (int)hi);
  __shared__ int s_lo[16], s_hi[16];
  const int wid = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) { s_lo[wid] = l; s_hi[wid] = h; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) {
      l = min(l, s_lo[i]);
      h = max(h, s_hi[i]);
    }
    int G = 0;
    if (h == 255) {
      record_error(MOE_ERR_NAN_SCALE);
    } else {
      const int elo = l - 127, ehi = h - 127;
      if (elo >= -9 && ehi <= 8) G = 0;
      else if (ehi - elo <= 17) G = ehi - 8;
      else record_error(MOE_ERR_RANGE);
    }
    out_global[m] = exp2_int(G);
  }
}

// Two copies of the E4M3 code of byte b's 2^(b - 127 - G), as a 16-bit pair.
__device__ __forceinline__ uint32_t nvfp4_scale_pair(uint32_t b, int G) {
  int j = (int)b - 127 - G;
  j = max(-9, min(8, j));                            // only out of range after a recorded error
  const uint32_t c = e4m3_pow2_code(j);
  return c | (c << 8);
}

// Pass 2: 16 scale bytes per thread -> 32 output bytes; the nibble copy
// (when not aliased) in a second grid-stride loop, 16 bytes at a time.
__global__ void __launch_bounds__(256) nvfp4_convert_vec_kernel(const uint4* __restrict__ e8m0, int64_t n16,
                                                                int64_t per_mat16, const float* __restrict__ glob,
                                                                uint4* __restrict__ out_e4m3,
                                                                const uint4* __restrict__ fp4,
                                                                uint4* __restrict__ out_fp4, int64_t n_fp4_16) {
  pdl_trigger();
  pdl_wait();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t i = tid; i < n16; i += stride) {
    const int G = exponent_of_pow2(__ldg(glob + i / per_mat16));
    const uint4 v = __ldg(e8m0 + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = nvfp4_scale_pair(w[k] & 0xFFu, G) | (nvfp4_scale_pair((w[k] >> 8) & 0xFFu, G) << 16);
      o[2 * k + 1] = nvfp4_scale_pair((w[k] >> 16) & 0xFFu, G) | (nvfp4_scale_pair(w[k] >> 24, G) << 16);
    }
    out_e4m3[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    out_e4m3[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
  if (out_fp4 != nullptr)
    for (int64_t i = tid; i < n_fp4_16; i += stride) out_fp4[i] = __ldg(fp4 + i);
}

// Largest magnitude code (0..7) among the 32 E2M1 nibbles of v, by a three-
// step binary search: some nibble m reaches t exactly when m + 8 - t sets the
// nibble's bit 3 (the sums stay below 16, so no carry crosses nibbles); the
// first step (m >= 4) is bit 2 itself.
__device__ __forceinline__ uint32_t max_magnitude_code(const uint4 v) {
  const uint32_t m0 = v.x & 0x77777777u, m1 = v.y & 0x77777777u;
  const uint32_t m2 = v.z & 0x77777777u, m3 = v.w & 0x77777777u;
  auto any_ge = [&](uint32_t t) {
    const uint32_t k = (8u - t) * 0x11111111u;
    return (((m0 + k) | (m1 + k) | (m2 + k) | (m3 + k)) & 0x88888888u) != 0u;
  };
  uint32_t mc = ((m0 | m1 | m2 | m3) & 0x44444444u) != 0u ? 4u : 0u;
  mc += any_ge(mc + 2u) ? 2u : 0u;
  mc += any_ge(mc + 1u) ? 1u : 0u;
  return mc;
}

// INT4 group-128: one thread per 32-element block (one 16-byte chunk of
// nibbles and its E8M0 byte), four consecutive threads per 128-group, so the
// loads and stores of a warp are contiguous; blocks of 256 threads walk the
// matrix grid-stride.  The group maximum is reduced over the four threads by
// shuffles.
//
// Codes from a table.  The group maximum is amax = A * 2^F with A = 1 or 1.5
// (every E2M1 value is 1 or 1.5 times a power of two), so while amax is a
// normal float32 (F >= -96 here), scale_inv = fl(amax / 7) = 2^F * fl(A / 7),
// and the quotient of a code of value v in a block of exponent e is
// fl(v 2^e / scale_inv) = 2^(e - F) * fl(v / fl(A / 7)): exact power-of-two
// scalings of the IEEE results, until the quotient is far below 0.5 (e - F <
// -8), where every code rounds to 0.  A block with a nonzero code has e - F
// <= 1.  So the eight codes of a block depend only on (A, e - F): each block
// of threads first computes those 2 x 10 tables with the same IEEE divides,
// multiplies and round-to-nearest-even the per-element rule uses (and an
// all-zero table for e - F < -8), then every 32-element block looks its table
// up instead of dividing.  Groups with a maximum below 2^-96 take the direct
// path: two IEEE divisions per block (2^e / s and 3 * 2^e / s, scaled by
// powers of two).
__device__ __forceinline__ float e2m1_magnitude(uint32_t m) {     // code 0..7 -> 0, .5, 1, 1.5, 2, 3, 4, 6
  const uint32_t bits = m >= 2u ? ((((m >> 1) + 126u) << 23) | ((m & 1u) << 22)) : (m ? 126u << 23 : 0u);
  return __uint_as_float(bits);
}

// Byte tables over the magnitude code from the eight codes c[0..7] (c[0] = 0):
// t.x, t.y = q (codes 0..3, 4..7), t.z, t.w = (16 - q) & 15, the two's
// complement nibble of -q (q <= 7, so the byte-wise subtraction never borrows).
__device__ __forceinline__ uint4 int4_code_tables(const uint32_t (&c)[8]) {
  const uint32_t p0 = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
  const uint32_t p1 = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
  return make_uint4(p0, p1, (0x10101010u - p0) & 0x0F0F0F0Fu, (0x10101010u - p1) & 0x0F0F0F0Fu);
}

// PTX prmt in its default mode: selector nibble i picks byte (nibble & 7) of
// {b, a} (a = bytes 0..3); when the nibble's bit 3 is set the result byte is
// instead that byte's sign bit replicated (0x00 or 0xFF).  (__byte_perm reads
// only the low 3 bits of each selector nibble.)
__device__ __forceinline__ uint32_t prmt_sign(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// 16 bytes of E2M1 nibbles -> 16 bytes of INT4 nibbles through the tables t.
// Each E2M1 nibble (bit 3 sign, bits 0-2 magnitude m) is its own selector:
// with sign 0 the lookup in t.x/t.y copies q(m) and the lookup in t.z/t.w
// (selector ^ 8, sign mode) gives 0x00 (table bytes are below 0x80); with
// sign 1 it is the other way round, so OR-ing the two lookups yields the INT4
// code of either sign, one byte per element.  Two such bytes are then merged
// into one output byte (element 2i in the low nibble).
__device__ __forceinline__ uint4 int4_remap(const uint4 in, const uint4 t) {
  const uint32_t words[4] = {in.x, in.y, in.z, in.w};
  uint32_t ow[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const uint32_t v = words[w], vn = v ^ 0x88888888u;
    const uint32_t a = prmt_sign(t.x, t.y, v) | prmt_sign(t.z, t.w, vn);               // elements 0..3
    const uint32_t b = prmt_sign(t.x, t.y, v >> 16) | prmt_sign(t.z, t.w, vn >> 16);   // elements 4..7
    const uint32_t x = a | (a >> 4), y = b | (b >> 4);   // bytes 0 and 2: two codes each
    ow[w] = __byte_perm(x, y, 0x6420u);
  }
  return make_uint4(ow[0], ow[1], ow[2], ow[3]);
}

constexpr int kInt4TableD = 10;       // tables for e - F = -8 .. 1 (index 1 .. 10), index 0 all zero

__global__ void __launch_bounds__(256) int4g128_kernel(const uint4* __restrict__ fp4,
                                                       const uint8_t* __restrict__ e8m0, int64_t n_blocks,
                                                       uint4* __restrict__ out, float* __restrict__ scale_inv) {
  __shared__ uint4 s_tab[2][kInt4TableD + 1];
  __shared__ float s_sa[2];
  pdl_trigger();
  // the tables read no global memory: built before waiting for the previous kernel
  if (threadIdx.x < 2 * (kInt4TableD + 1)) {
    const int ai = threadIdx.x / (kInt4TableD + 1), di = threadIdx.x % (kInt4TableD + 1);
    const float sa = __fdiv_rn(ai ? 1.5f : 1.0f, 7.0f);
    uint32_t c[8];
    c[0] = 0u;
#pragma unroll
    for (uint32_t m = 1; m < 8; ++m) {
      const float quot = __fmul_rn(__fdiv_rn(e2m1_magnitude(m), sa), exp2_int(di - 9));
      c[m] = di == 0 ? 0u : (uint32_t)rintf(fminf(quot, 7.0f));
    }
    s_tab[ai][di] = int4_code_tables(c);
    if (di == 0) s_sa[ai] = sa;
  }
  __syncthreads();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // warp-uniform loop: every lane takes part in the group shuffles.  The next
  // block's bytes are loaded before this one is worked on, so two loads per
  // thread are in flight.
  int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  uint4 in_next = make_uint4(0u, 0u, 0u, 0u);
  int b_next = 0;
  if (base + lane < n_blocks) {
    in_next = __ldg(fp4 + base + lane);
    b_next = (int)__ldg(e8m0 + base + lane);
  }
  for (; base < n_blocks; base += stride) {
    const int64_t blk = base + lane;
    const bool live = blk < n_blocks;
    const uint4 in = in_next;
    const int b = b_next;
    if (blk + stride < n_blocks) {
      in_next = __ldg(fp4 + blk + stride);
      b_next = (int)__ldg(e8m0 + blk + stride);
    }
    const uint32_t mc = max_magnitude_code(in);     // largest magnitude code of the block
    const float sc = exp2_int(b - 127);
    float bm = __fmul_rn(e2m1_magnitude(mc), sc);
    const bool nan = b == 255;
    if (live && !nan && isinf(bm)) record_error(MOE_ERR_RANGE);
    if (nan) bm = 0.0f;
    float amax = fmaxf(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
    // a NaN scale anywhere in the group (its four lanes) skips the group
    const bool gnan = ((__ballot_sync(0xFFFFFFFFu, nan) >> (lane & 28)) & 0xFu) != 0u;
    if (!live) continue;
    if (gnan) {
      if (nan) record_error(MOE_ERR_NAN_SCALE);
      continue;
    }
    const uint32_t ab = __float_as_uint(amax);
    const int F = (int)((ab >> 23) & 0xFFu) - 127;
    uint4 t;
    float sinv;
    if (amax > 0.0f && F >= -96 && F <= 127) {
      const int ai = (int)((ab >> 22) & 1u);             // mantissa of the maximum: 1 or 1.5
      sinv = __fmul_rn(s_sa[ai], exp2_int(F));
      const int d = (b - 127) - F;
      t = s_tab[ai][d < -8 ? 0 : min(d, 1) + 9];
    } else {
      sinv = amax > 0.0f ? __fdiv_rn(amax, 7.0f) : 1.0f;
      // the seven quotients of this block: magnitudes 1, 2, 4, 6 times d1 / 2 and
      // 1.5, 3, 6 times d3 / 3, each an exact power-of-two scaling
      const float d1 = __fdiv_rn(sc, sinv);
      const float d3 = __fdiv_rn(__fmul_rn(3.0f, sc), sinv);
      const float qv[8] = {0.0f, 0.5f * d1, d1, 0.5f * d3, 2.0f * d1, d3, 4.0f * d1, 2.0f * d3};
      uint32_t c[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) c[m] = (uint32_t)rintf(fminf(qv[m], 7.0f));
      t = int4_code_tables(c);
    }
    if ((lane & 3) == 0) scale_inv[blk >> 2] = sinv;
    out[blk] = int4_remap(in, t);
  }
}

// FP8 cast: one block of 128 threads per (matrix, 128-row block, 128-column
// block).  The block's 512 16-byte chunks of nibbles (one 32-element
// sub-block each) are handed out so that four consecutive threads read one
// row's 64 bytes and write its 128 E4M3 bytes (a warp covers 8 rows per pass,
// 4 passes).  The block scale is 2^s with s = ceil(log2(amax / 448)) (the
// activation rule) for the exact block maximum, clamped to [-127, 127]; for an
// MXFP4 maximum {1, 1.5} * 2^E this is E - 8.  Maxima are compared as the
// order-preserving key 2 * E + [mantissa 1.5], so values beyond float32 (6 *
// 2^127) still order correctly.  Element codes: E4M3 round to nearest even of
// E2M1 * 2^d, d = e - s, from an 8-entry table per sub-block (four paired
// conversions) applied with byte permutes; the sign bit is copied.  A present
// code c is exact iff d >= -9 - lsb(c) (its lowest set bit must stay at or
// above E4M3's 2^-9); otherwise MOE_ERR_RANGE is recorded and the rounded
// code is kept.  An E8M0 NaN records MOE_ERR_NAN_SCALE and skips the block.
__global__ void __launch_bounds__(128) fp8_block128_kernel(const uint8_t* __restrict__ fp4,
                                                           const uint8_t* __restrict__ e8m0, int N, int K,
                                                           uint8_t* __restrict__ out,
                                                           float* __restrict__ scale_inv) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_key[4];
  __shared__ int s_nan[4];
  const int KB = K / 128, NB = N / 128;
  const int64_t blk = blockIdx.x;
  const int kb = (int)(blk % KB);
  const int64_t t = blk / KB;
  const int nb = (int)(t % NB);
  const int64_t mat = t / NB;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int j = tid & 3;                       // sub-block (32 columns) of this thread's chunks
  const int64_t row0 = mat * N + (int64_t)nb * 128;
  // pass p: row (p * 32 + tid / 4), sub-block j
  uint4 in[4];
  int b[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int64_t row = row0 + p * 32 + (tid >> 2);
    in[p] = __ldg(reinterpret_cast<const uint4*>(fp4 + row * (K / 2) + (int64_t)kb * 64) + j);
    b[p] = (int)__ldg(e8m0 + row * (K / 32) + (int64_t)kb * 4 + j);
  }
  // E2M1 magnitude code c = 1..7 (0.5, 1, 1.5, 2, 3, 4, 6): floor(log2) = (c >> 1) - 1,
  // mantissa bit = c & 1 for c >= 2 (0 for c = 1)
  int key = INT_MIN;
  int nan = 0;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    nan |= b[p] == 255;
    const int mc = (int)max_magnitude_code(in[p]);
    if (mc > 0) key = max(key, 2 * (b[p] - 127 + (mc >> 1) - 1) + ((mc >> 1) != 0 ? (mc & 1) : 0));
  }
  key = __reduce_max_sync(0xFFFFFFFFu, key);
  nan = __reduce_or_sync(0xFFFFFFFFu, nan);
  if (lane == 0) { s_key[wid] = key; s_nan[wid] = nan; }
  __syncthreads();
  key = max(max(s_key[0], s_key[1]), max(s_key[2], s_key[3]));
  nan = s_nan[0] | s_nan[1] | s_nan[2] | s_nan[3];
  if (nan) {
    if (tid == 0) record_error(MOE_ERR_NAN_SCALE);
    return;
  }
  const int s = key == INT_MIN ? 0 : max(-127, min(127, (key >> 1) - 8));   // key >> 1 = floor(key / 2) = E
  if (tid == 0) scale_inv[(mat * NB + nb) * KB + kb] = exp2_int(s);
  const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  bool inexact = false;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int d = b[p] - 127 - s;
    // values below 2^-10 round to 0 in E4M3 whatever their float32 form, so
    // the scale factor is clamped into float32's range
    const float sc = exp2_int(max(d, -149));
    const uint32_t t0 = e4m3x4(0.0f, kE2M1[1] * sc, kE2M1[2] * sc, kE2M1[3] * sc);
    const uint32_t t1 = e4m3x4(kE2M1[4] * sc, kE2M1[5] * sc, kE2M1[6] * sc, kE2M1[7] * sc);
    const uint32_t w[4] = {in[p].x, in[p].y, in[p].z, in[p].w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // a byte permute reads the low 3 bits of the four selector nibbles of
        // its low 16 bits: the nibbles pick the magnitude codes, and in
        // w >> 3 the selector is odd exactly for a set sign bit (odd table
        // bytes are 0x80)
        const uint32_t sel = w[k] >> (16 * h);
        const uint32_t sgn = __byte_perm(0x80008000u, 0x80008000u, sel >> 3);
        o[2 * k + h] = __byte_perm(t0, t1, sel) | sgn;
      }
    }
    const int64_t row = row0 + p * 32 + (tid >> 2);
    uint4* dst = reinterpret_cast<uint4*>(out + row * K + (int64_t)kb * 128 + j * 32);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    if (d < -8) {
      // exact iff every present nonzero code c has d >= -9 - lsb(c)
      const int kMin[8] = {INT_MIN, -8, -9, -8, -10, -9, -11, -10};
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int n = 0; n < 8; ++n) inexact |= d < kMin[(w[k] >> (4 * n)) & 7u];
    }
  }
  if (inexact) record_error(MOE_ERR_RANGE);
}

// MXFP4 -> PTPC-FP8 weights ("DeepSeek-V4.1-Flash-Quark-PTPC-FP8"
// walkthrough, 核心参数: per output channel, static, symmetric, half_even):
// one block of 256 threads per row of K elements; w = exact float32
// dequantisation; scale = amax / 448 (float32 IEEE divide, 1 for a zero row);
// q = E4M3(w / scale) with a float32 IEEE divide.  A float32 overflow of w
// records MOE_ERR_RANGE; an E8M0 NaN records MOE_ERR_NAN_SCALE and skips the
// row.  K % 32 == 0.
__global__ void __launch_bounds__(256) fp8_per_channel_kernel(const uint8_t* __restrict__ fp4,
                                                              const uint8_t* __restrict__ e8m0, int K,
                                                              uint8_t* __restrict__ out, float* __restrict__ scale) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_max[8];
  __shared__ int s_bad[8];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  // thread t owns 8-element chunks t, t + 256, ...: 4 bytes of nibbles each
  auto load8 = [&](int c8, float (&v)[8], int& bad) {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(fp4 + row * (K / 2)) + c8);
    const int b = __ldg(e8m0 + row * (K / 32) + c8 / 4);
    bad |= b == 255;
    const float sc = exp2_int(b - 127);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t nib = (w >> (4 * j)) & 0xFu;
      const float mag = __fmul_rn(kE2M1[nib & 7u], sc);
      v[j] = (nib & 8u) ? -mag : mag;
    }
  };
  float m = 0.0f;
  int bad = 0;
  for (int c8 = tid; c8 < K / 8; c8 += blockDim.x) {
    float v[8];
    load8(c8, v, bad);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
  }
  m = warp_max_nonneg(m);
  bad = __reduce_or_sync(0xFFFFFFFFu, bad);
  if (lane == 0) { s_max[wid] = m; s_bad[wid] = bad; }
  __syncthreads();
  m = s_max[0];
  bad = s_bad[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) {
    m = fmaxf(m, s_max[w]);
    bad |= s_bad[w];
  }
  if (bad) {
    if (tid == 0) record_error(MOE_ERR_NAN_SCALE);
    return;
  }
  if (isinf(m)) {
    if (tid == 0) record_error(MOE_ERR_RANGE);
    return;
  }
  const float sc = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
  if (tid == 0) scale[row] = sc;
  for (int c8 = tid; c8 < K / 8; c8 += blockDim.x) {
    float v[8];
    int unused = 0;
    load8(c8, v, unused);
    const uint32_t lo = e4m3x4(__fdiv_rn(v[0], sc), __fdiv_rn(v[1], sc), __fdiv_rn(v[2], sc), __fdiv_rn(v[3], sc));
    const uint32_t hi = e4m3x4(__fdiv_rn(v[4], sc), __fdiv_rn(v[5], sc), __fdiv_rn(v[6], sc), __fdiv_rn(v[7], sc));
    reinterpret_cast<uint2*>(out + row * K)[c8] = make_uint2(lo, hi);
  }
}

}  // namespace moe
