// Bandwidth-bound kernels of the expert path: activation quantisation (a1),
// standalone SwiGLU + requantisation (a5), routing (a2), grouping (a3) and
// the weighted combine (a7).  All are one pass over their data with 8-16
// byte accesses per thread.
#pragma once

#include "common.cuh"

namespace moe {

// ------------------------------- a1 ---------------------------------------
// Each half-warp quantises one (row, 128-column) group: a lane owns 8
// consecutive columns (16 bytes of bf16 in, 8 bytes of E4M3 out).  A warp
// takes kQuantSlots pairs of groups and issues all their loads before using
// any, so each SM keeps enough bytes in flight to stream at the copy rate.
// "DeepSeek-V4-Flash-SI", 低精度计算: FP8 E4M3 per 128 elements with a
// power-of-two scale.
constexpr int kQuantSlots = 4;
constexpr int kQuantGroupsPerBlock = 8 * 2 * kQuantSlots;     // 8 warps of 256 threads

__global__ void __launch_bounds__(256) quant_act_kernel(const uint4* __restrict__ x, int64_t n_groups,
                                                        uint2* __restrict__ xq, uint8_t* __restrict__ sx) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int hl = lane & 15;                          // lane within the half-warp
  // group of slot s: first + 2 s + (lane >> 4)
  const int64_t first = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * (2 * kQuantSlots);
  uint4 wv[kQuantSlots];
#pragma unroll
  for (int s = 0; s < kQuantSlots; ++s) {
    const int64_t grp = first + 2 * s + (lane >> 4);
    wv[s] = grp < n_groups ? __ldg(x + grp * 16 + hl) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int s = 0; s < kQuantSlots; ++s) {
    const int64_t grp = first + 2 * s + (lane >> 4);
    const uint32_t u[4] = {wv[s].x, wv[s].y, wv[s].z, wv[s].w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf16_lo(u[i]);
      f[2 * i + 1] = bf16_hi(u[i]);
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    // maximum over the half-warp (offsets below 16 stay within it)
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int k = pow2_scale_exponent(m);
    const float sc = exp2_int(-k);
    if (grp < n_groups) {
      xq[grp * 16 + hl] = make_uint2(e4m3x4(__fmul_rn(f[0], sc), __fmul_rn(f[1], sc), __fmul_rn(f[2], sc),
                                            __fmul_rn(f[3], sc)),
                                     e4m3x4(__fmul_rn(f[4], sc), __fmul_rn(f[5], sc), __fmul_rn(f[6], sc),
                                            __fmul_rn(f[7], sc)));
      if (hl == 0) sx[grp] = (uint8_t)(k + 127);
    }
  }
}

// ------------------------------- a5 ---------------------------------------
// One warp per (row, 128 columns of h); gate at column c, up at column I + c.
__global__ void __launch_bounds__(256) swiglu_quant_kernel(const float4* __restrict__ gu, int rows, int I,
                                                           float limit, uint32_t* __restrict__ hq,
                                                           uint8_t* __restrict__ sh) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int gpr = I / 128;
  const int64_t grp = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (grp >= (int64_t)rows * gpr) return;
  const int64_t row = grp / gpr;
  const int gi = (int)(grp % gpr);
  const int64_t q4 = (row * 2 * I + gi * 128) / 4 + lane;     // float4 index of the gate
  const float4 g = __ldg(gu + q4);
  const float4 u = __ldg(gu + q4 + I / 4);
  const float h0 = swiglu_clamped(g.x, u.x, limit), h1 = swiglu_clamped(g.y, u.y, limit);
  const float h2 = swiglu_clamped(g.z, u.z, limit), h3 = swiglu_clamped(g.w, u.w, limit);
  const float m = warp_max_nonneg(fmaxf(fmaxf(fabsf(h0), fabsf(h1)), fmaxf(fabsf(h2), fabsf(h3))));
  const int k = pow2_scale_exponent(m);
  const float s = exp2_int(-k);
  hq[(row * I + gi * 128) / 4 + lane] =
      e4m3x4(__fmul_rn(h0, s), __fmul_rn(h1, s), __fmul_rn(h2, s), __fmul_rn(h3, s));
  if (lane == 0) sh[row * gpr + gi] = (uint8_t)(k + 127);
}

// ------------------------------- a2 ---------------------------------------
// One warp per token.  Lane l holds logits of experts l, l+32, ...; k rounds
// of a warp arg-max on (value desc, index asc).  "DeepSeek-V4-Flash-SI",
// 架构特性: sqrtsoftplus scores, top-k, routing scale 1.5.
__device__ __forceinline__ float softplus_f(float z) { return z > 20.0f ? z : log1pf(expf(z)); }

template <int V>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                         int k, float route_scale, int route_norm,
                                                         int32_t* __restrict__ idx, float* __restrict__ w) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + (int64_t)t * E;
  float v[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(row + e) : 0.0f;
  }
  uint32_t taken = 0;
  int sel_e[16];
  float sel_v[16];
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
      const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j == r) { sel_e[j] = be; sel_v[j] = bv; }
  }
  // every lane computes all k scores in slot order (identical on all lanes)
  float s_sel = 0.0f, sum = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j < k) {
      const float s = sqrtf(softplus_f(sel_v[j]));
      sum += s;
      if (j == lane) s_sel = s;
    }
  }
  if (lane < k) {
    int e_sel = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j == lane) e_sel = sel_e[j];
    idx[(int64_t)t * k + lane] = e_sel;
    w[(int64_t)t * k + lane] = route_norm ? route_scale * __fdiv_rn(s_sel, sum) : route_scale * s_sel;
  }
}

// ---------------------------- hash routing --------------------------------
// "DeepSeek-V4-Flash-SI", 架构特性: the first layers route by hash, chosen
// deterministically from the token ID.  The experts of token t are the k
// entries of its row in a caller-supplied table (tid2eid[token_ids[t]]); the
// weights follow the scored layers' rule at those experts: sqrtsoftplus of
// the gate logits, normalised in slot order and scaled.  One thread per
// token.  An out-of-range token id or table entry records MOE_ERR_INVALID;
// the token's row (bad id) or that slot (bad entry) gets idx -1 and weight 0.
__global__ void __launch_bounds__(256) route_hash_kernel(const int32_t* __restrict__ token_ids, int T,
                                                         const int32_t* __restrict__ tid2eid, int vocab,
                                                         const float* __restrict__ logits, int E, int k,
                                                         float route_scale, int route_norm,
                                                         int32_t* __restrict__ idx, float* __restrict__ w) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const int id = __ldg(token_ids + t);
  int32_t* irow = idx + (int64_t)t * k;
  float* wrow = w + (int64_t)t * k;
  if (id < 0 || id >= vocab) {
    record_error(MOE_ERR_INVALID);
    for (int j = 0; j < k; ++j) { irow[j] = -1; wrow[j] = 0.0f; }
    return;
  }
  const int32_t* trow = tid2eid + (int64_t)id * k;
  const float* lrow = logits + (int64_t)t * E;
  int e_sel[16];
  float s_sel[16];
  float sum = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    e_sel[j] = -1;
    s_sel[j] = 0.0f;
    if (j < k) {
      const int e = __ldg(trow + j);
      if (e >= 0 && e < E) {
        e_sel[j] = e;
        s_sel[j] = sqrtf(softplus_f(__ldg(lrow + e)));
        sum += s_sel[j];
      } else {
        record_error(MOE_ERR_INVALID);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j < k) {
      irow[j] = e_sel[j];
      wrow[j] = e_sel[j] < 0 ? 0.0f : (route_norm ? route_scale * __fdiv_rn(s_sel[j], sum) : route_scale * s_sel[j]);
    }
  }
}

// ------------------------- per-token FP8 (PTPC) ----------------------------
// PTPC-FP8 ("DeepSeek-V4.1-Flash-Quark-PTPC-FP8" walkthrough, 核心参数):
// per-row (per-token) dynamic scale = amax / 448 (float32 IEEE divide, 1 for
// a zero row); q = E4M3(x / scale), float32 IEEE divide, nearest even,
// saturating.  One block of 256 threads per row; cols % 8 == 0.
template <bool F32_IN>
__global__ void __launch_bounds__(256) quant_fp8_per_row_kernel(const void* __restrict__ x, int cols,
                                                                uint8_t* __restrict__ q, float* __restrict__ scale) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_max[8];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  auto load8 = [&](int c8, float (&v)[8]) {
    if constexpr (F32_IN) {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(x) + row * cols) + 2 * c8;
      const float4 a = __ldg(src), b = __ldg(src + 1);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + row * cols) + c8);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = bf16_lo(u[j]);
        v[2 * j + 1] = bf16_hi(u[j]);
      }
    }
  };
  float m = 0.0f;
  for (int c8 = tid; c8 < cols / 8; c8 += blockDim.x) {
    float v[8];
    load8(c8, v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
  }
  m = warp_max_nonneg(m);
  if (lane == 0) s_max[wid] = m;
  __syncthreads();
  m = s_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, s_max[w]);
  const float sc = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
  if (tid == 0) scale[row] = sc;
  for (int c8 = tid; c8 < cols / 8; c8 += blockDim.x) {
    float v[8];
    load8(c8, v);
    const uint32_t lo = e4m3x4(__fdiv_rn(v[0], sc), __fdiv_rn(v[1], sc), __fdiv_rn(v[2], sc), __fdiv_rn(v[3], sc));
    const uint32_t hi = e4m3x4(__fdiv_rn(v[4], sc), __fdiv_rn(v[5], sc), __fdiv_rn(v[6], sc), __fdiv_rn(v[7], sc));
    reinterpret_cast<uint2*>(q + row * cols)[c8] = make_uint2(lo, hi);
  }
}

// Per-row float32 scales of the grouped rows: row r takes the scale of its
// source token (perm[r] / k for a routed pair, perm[r] - T*k for a shared
// row).  Rows past offsets[E + 1] (pairs the grouping rejected) are skipped.
__global__ void __launch_bounds__(256) gather_row_scales_kernel(const int32_t* __restrict__ perm, int T, int k,
                                                                const int32_t* __restrict__ offsets, int E,
                                                                const float* __restrict__ src,
                                                                float* __restrict__ dst) {
  pdl_trigger();
  pdl_wait();
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int P = T * k;
  if (r >= offsets[E + 1] || r >= (int64_t)P + T) return;
  const int p = perm[r];
  if (p < 0 || p >= P + T) {
    record_error(MOE_ERR_INVALID);
    dst[r] = 0.0f;
    return;
  }
  dst[r] = src[p < P ? p / k : p - P];
}

// ------------------------------- a3 ---------------------------------------
// Grouping in deterministic passes:
//   count:   per chunk of kChunk pairs, a histogram over experts
//   scan:    per expert the running sum over chunks, then offsets
//   scatter: per chunk, the pairs are staged in shared memory and one warp
//            walks them in order; __match_any_sync gives each pair its rank
//            among equal experts -> stable rows
//   gather:  one warp per output row copies the FP8 row and its scales
// When all pairs fit in one chunk (decode), one block does count, scan and
// scatter (permute_small_kernel).  A pair with an expert id outside [0, E)
// is flagged (MOE_ERR_INVALID), gets no row, and its inv entry is -1.
constexpr int kChunk = 2048;

__global__ void __launch_bounds__(256) permute_count_kernel(const int32_t* __restrict__ idx, int P, int E,
                                                            int32_t* __restrict__ chunk_hist) {
  pdl_trigger();
  pdl_wait();
  __shared__ int hist[1024];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * kChunk;
  for (int p = p0 + threadIdx.x; p < min(P, p0 + kChunk); p += blockDim.x) {
    const int e = __ldg(idx + p);
    if (e < 0 || e >= E) record_error(MOE_ERR_INVALID);
    else atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(int64_t)blockIdx.x * E + e] = hist[e];
}

__global__ void __launch_bounds__(1024) permute_scan_kernel(int32_t* __restrict__ chunk_hist, int n_chunks,
                                                            int E, int T, int has_shared,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets) {
  pdl_trigger();
  pdl_wait();
  __shared__ int warp_sums[32];
  const int e = threadIdx.x;          // E + 1 <= 1024 groups
  int c = 0;
  if (e < E) {
    for (int ch = 0; ch < n_chunks; ++ch) {
      const int h = chunk_hist[(int64_t)ch * E + e];
      chunk_hist[(int64_t)ch * E + e] = c;
      c += h;
    }
  } else if (e == E) {
    c = has_shared ? T : 0;
  }
  // exclusive scan of c over threads
  const int lane = e & 31, wid = e >> 5;
  int x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const int excl = (wid ? warp_sums[wid - 1] : 0) + x - c;
  if (e <= E) {
    counts[e] = c;
    offsets[e] = excl;
    if (e == E) offsets[E + 1] = excl + c;
  }
}

// Stable placement of the pairs sidx[0, n) (ids p0 + i) by one warp: ctr[e]
// holds the next row of expert e and advances as the warp walks the pairs.
__device__ __forceinline__ void scatter_walk(const int* sidx, int n, int p0, int* ctr, int32_t* __restrict__ perm,
                                             int32_t* __restrict__ inv) {
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const int e = (i < n) ? sidx[i] : -2;
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int pos = (e >= 0) ? ctr[e] + rank : 0;
    __syncwarp();
    if (e >= 0 && (__ffs(peers) - 1) == lane) ctr[e] += __popc(peers);
    __syncwarp();
    if (e >= 0) {
      perm[pos] = p0 + i;
      inv[p0 + i] = pos;
    } else if (e == -1) {
      inv[p0 + i] = -1;
    }
  }
}

// One block of 256 threads per chunk: stage the chunk's expert ids and the
// chunk's first row per expert in shared memory, then one warp places them.
__global__ void __launch_bounds__(256) permute_scatter_kernel(const int32_t* __restrict__ idx, int P, int E,
                                                              const int32_t* __restrict__ chunk_hist,
                                                              const int32_t* __restrict__ offsets,
                                                              int32_t* __restrict__ perm,
                                                              int32_t* __restrict__ inv) {
  pdl_trigger();
  pdl_wait();
  __shared__ int ctr[1024];
  __shared__ int sidx[kChunk];
  const int p0 = blockIdx.x * kChunk;
  const int n = min(P, p0 + kChunk) - p0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) ctr[e] = offsets[e] + chunk_hist[(int64_t)blockIdx.x * E + e];
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = __ldg(idx + p0 + i);
    sidx[i] = (e >= 0 && e < E) ? e : -1;         // invalid ids were flagged by the count pass
  }
  __syncthreads();
  if (threadIdx.x < 32) scatter_walk(sidx, n, p0, ctr, perm, inv);
}

// All pairs in one chunk (P <= kChunk): count, scan and scatter in one block of
// 1024 threads.  Group E (the shared expert) has has_shared ? T : 0 rows.
__global__ void __launch_bounds__(1024) permute_small_kernel(const int32_t* __restrict__ idx, int P, int E, int T,
                                                             int has_shared, int32_t* __restrict__ counts,
                                                             int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ perm,
                                                             int32_t* __restrict__ inv) {
  pdl_trigger();
  pdl_wait();
  __shared__ int hist[1024];
  __shared__ int sidx[kChunk];
  __shared__ int warp_sums[32];
  const int tid = threadIdx.x;
  hist[tid] = 0;
  __syncthreads();
  for (int i = tid; i < P; i += blockDim.x) {
    int e = __ldg(idx + i);
    if (e < 0 || e >= E) {
      record_error(MOE_ERR_INVALID);
      e = -1;
    } else {
      atomicAdd(&hist[e], 1);
    }
    sidx[i] = e;
  }
  __syncthreads();
  // exclusive scan of the group sizes (thread e: group e, e <= E < 1024)
  const int c = tid < E ? hist[tid] : (tid == E && has_shared ? T : 0);
  const int lane = tid & 31, wid = tid >> 5;
  int x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int sum = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, sum, o);
      if (lane >= o) sum += y;
    }
    warp_sums[lane] = sum;
  }
  __syncthreads();
  const int excl = (wid ? warp_sums[wid - 1] : 0) + x - c;
  if (tid <= E) {
    counts[tid] = c;
    offsets[tid] = excl;
    if (tid == E) offsets[E + 1] = excl + c;
  }
  __syncthreads();                  // every thread has read hist[tid]
  if (tid < E) hist[tid] = excl;    // reused as the running row of each expert
  __syncthreads();
  if (tid < 32) scatter_walk(sidx, P, 0, hist, perm, inv);
}

// One warp per row.  H % 128 == 0, rows 16-byte aligned.
__global__ void __launch_bounds__(256) permute_gather_kernel(const uint4* __restrict__ xq,
                                                             const uint8_t* __restrict__ sx, int H, int T,
                                                             int k, const int32_t* __restrict__ offsets,
                                                             int E, int32_t* __restrict__ perm,
                                                             uint4* __restrict__ xq_perm,
                                                             uint8_t* __restrict__ sx_perm) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int R = offsets[E + 1];
  if (r >= R) return;
  const int shared0 = offsets[E];
  const int P = T * k;
  int t;
  if (r >= shared0) {
    t = (int)(r - shared0);
    if (lane == 0) perm[r] = P + t;
  } else {
    t = perm[r] / k;
  }
  const int n16 = H / 16;
  const uint4* src = xq + (int64_t)t * n16;
  uint4* dst = xq_perm + r * n16;
  for (int i = lane; i < n16; i += 32) dst[i] = __ldg(src + i);
  const int ns = H / 128;
  for (int i = lane; i < ns; i += 32) sx_perm[r * ns + i] = __ldg(sx + (int64_t)t * ns + i);
}

// ------------------------------- a7 ---------------------------------------
// Block (token t, 512-column slice): each thread sums two 4-column chunks 256
// chunks apart, issuing the row loads of up to 8 slots of both before
// accumulating them (float32, slot order, then the shared expert's row; one
// bf16 rounding), so a thread keeps up to 18 16-byte loads in flight.  The
// token's slot indices and weights are read by every thread (through L1).
constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const float4* __restrict__ o,
                                                                  const int32_t* __restrict__ inv,
                                                                  const float* __restrict__ w, int T, int k, int H,
                                                                  int has_shared, const int32_t* __restrict__ offsets,
                                                                  int E, uint2* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const int64_t t = blockIdx.x;
  const int h4 = H / 4;
  const int c0 = blockIdx.y * 2 * kCombineThreads + threadIdx.x;
  const int c1 = c0 + kCombineThreads;
  const bool has0 = c0 < h4, has1 = c1 < h4;
  if (!has0) return;
  const int32_t* it = inv + t * k;
  const float* wt = w + t * k;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 a0 = zero, a1 = zero;
  for (int jb = 0; jb < k; jb += 8) {
    int r[8];
    float wj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = jb + j < k;
      r[j] = in ? __ldg(it + jb + j) : -1;       // -1 also: a pair the grouping rejected
      wj[j] = in ? __ldg(wt + jb + j) : 0.f;
    }
    float4 v0[8], v1[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v0[j] = r[j] >= 0 ? __ldg(o + (int64_t)r[j] * h4 + c0) : zero;
      v1[j] = (r[j] >= 0 && has1) ? __ldg(o + (int64_t)r[j] * h4 + c1) : zero;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (r[j] < 0) continue;
      a0.x = fmaf(wj[j], v0[j].x, a0.x);
      a0.y = fmaf(wj[j], v0[j].y, a0.y);
      a0.z = fmaf(wj[j], v0[j].z, a0.z);
      a0.w = fmaf(wj[j], v0[j].w, a0.w);
      a1.x = fmaf(wj[j], v1[j].x, a1.x);
      a1.y = fmaf(wj[j], v1[j].y, a1.y);
      a1.z = fmaf(wj[j], v1[j].z, a1.z);
      a1.w = fmaf(wj[j], v1[j].w, a1.w);
    }
  }
  if (has_shared) {
    const int64_t rs = (int64_t)__ldg(offsets + E) + t;
    const float4 v = __ldg(o + rs * h4 + c0);
    const float4 u = has1 ? __ldg(o + rs * h4 + c1) : zero;
    a0.x += v.x;
    a0.y += v.y;
    a0.z += v.z;
    a0.w += v.w;
    a1.x += u.x;
    a1.y += u.y;
    a1.z += u.z;
    a1.w += u.w;
  }
  auto pack = [](const float4& a) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(a.z, a.w);
    return make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
  };
  y[t * h4 + c0] = pack(a0);
  if (has1) y[t * h4 + c1] = pack(a1);
}

}  // namespace moe
