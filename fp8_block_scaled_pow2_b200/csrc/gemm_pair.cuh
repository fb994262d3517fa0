// Grouped expert GEMM on SM pairs, token-major: FP8 E4M3 activations x MXFP4
// (E2M1 + E8M0/32) weights with tcgen05.mma.cta_group::2 kind::mxf8f6f4.
//
// For wide token tiles (prefill) the swap-AB kernel (gemm_mxfp4.cuh) is bound
// by shared-memory bandwidth, not by the tensor core: per 128-wide K step of a
// full 128-token tile pair its copies write ~49 KB and its MMAs read 64 KB of
// shared memory for 8 MFLOP.  Here two CTAs on the two SMs of a cluster share
// one MMA of M = 256 tokens x N = 256 weight rows x K = 32: each CTA holds 128
// token rows (A) and 128 weight rows (B: the gate tile on rank 0 and the up
// tile on rank 1 for w1/w3, two adjacent output blocks for w2), so per K step
// a CTA writes ~34 KB and its tensor core reads 32 KB for 8.4 MFLOP (the
// tensor work, 512 cycles, sets the pace).
//
// Work item: (256-token tile of a group, 256 weight rows = 128 features of
// gate + up, or 256 output columns).  Items are ordered as in the swap-AB
// kernel (group-major, then weight block, then token tile) and the clusters
// walk them persistently.
//
// Accumulator (each CTA's tensor memory): [128 token rows (lanes)] x [256
// columns]: columns 0-127 from rank 0's weight tile, 128-255 from rank 1's.
// For SwiGLU a token's gate and up values of feature j are columns j and
// 128 + j of the same lane, so the epilogue needs no exchange between CTAs.
//
// Roles per CTA (both CTAs alike except where noted; 320 threads):
//   warp 0      producer: this CTA's token rows, weight tile, both weight
//               scale blocks (the MMA reads the scales of all N from each
//               CTA) and its token scales; completion is counted on rank 0's
//               stage barrier, which rank 0's producer arms with the bytes
//               of both CTAs
//   warp 1      tensor-memory allocation (both CTAs, collective) and, on
//               rank 0, the MMA issuer: scale copies, 4 MMAs per K step, a
//               commit that frees the stage in both CTAs
//   warps 2..9  epilogue: tensor memory -> registers -> global; after its
//               loads each warp releases the accumulator on rank 0's barrier
// Every wait is bounded (kWaitTimeoutNs); a CTA that gives up raises its
// abort flag, and both CTAs meet at a cluster barrier before freeing tensor
// memory.
#pragma once

#include "common.cuh"
#include "sm100.cuh"
#include "gemm_mxfp4.cuh"

namespace moe {
namespace pair {

using namespace sm100;
using gemm::Item;
using gemm::kWBlock;

constexpr int BN = 256;                 // tokens per work item (128 per CTA)
constexpr int kThreads = 320;
constexpr int EPI_WARPS = 8;
constexpr int EPI_FIRST = 2;

struct Cfg {
  // ring slot of one CTA: [token rows][weight tile][weight scales x2][token scales]
  static constexpr int A_OFF = 0;                 // 128 token rows x 128 bytes (E4M3)
  static constexpr int B_OFF = 16384;             // 128 weight rows x 128 nibbles, unpacked to bytes
  static constexpr int SFB_OFF = 32768;           // scale blocks of weight rows 0-127 and 128-255
  static constexpr int SFA_OFF = SFB_OFF + 1024;  // this CTA's token scales (4 K steps)
  static constexpr int STAGE_RAW = SFA_OFF + 512;
  static constexpr int STAGE = (STAGE_RAW + 1023) / 1024 * 1024;
  // epilogue area: the SwiGLU row maxima (per half, double-buffered), or the
  // float32 / bf16 staging tiles (32 rows x 20 floats per warp) that turn each
  // warp's rows into row-contiguous stores
  static constexpr int RED_BYTES = 2 * 2 * 128 * 4;
  static constexpr int STG_ROW = 20;
  static constexpr int STG_BYTES = EPI_WARPS * 32 * STG_ROW * 4;
  static constexpr int EPI_BYTES = RED_BYTES > STG_BYTES ? RED_BYTES : STG_BYTES;
  static constexpr int RING_BUDGET = 227 * 1024 - (512 + EPI_BYTES + 1024);
  static constexpr int STAGES = RING_BUDGET / STAGE > 8 ? 8 : RING_BUDGET / STAGE;
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int EPI_OFF = BAR_OFF + 512;
  static constexpr int SMEM_ALLOC = EPI_OFF + EPI_BYTES + 1024;
  // tensor memory: accumulator 0-255, weight scales 256-263, token scales 264-267
  static constexpr int TMEM_COLS = 512;
  static constexpr int SFB_COL = 256;
  static constexpr int SFA_COL = 264;
  // bytes one CTA's copies deliver per K step, besides its token rows and
  // (every fourth step) its token scales: packed weight tile + two scale blocks
  static constexpr int TX_W = 8192 + 1024;
  static_assert(STAGES >= 4, "too few pipeline stages");
  static_assert(2 * STAGES + 4 <= 60, "barrier area overflow");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory overflow");
  static_assert(SMEM_ALLOC > 116 * 1024, "one CTA per SM");
};

// Token maps of the pair kernel: boxes of 16, 32, 64 and 128 rows (one CTA's
// share of the 256-row tile), and the token-scale blocks.
struct PairMaps {
  CUtensorMap tok[4];
  CUtensorMap tok_sf;    // [blocks][128 words] over the plan's interleaved token scales
};

// The plan, read from global memory (the items are long: decoding one costs
// little next to its K loop).
struct GlobalPlan {
  const int* prefix;
  const int* tstart;
  const int2* groups;
};

struct PairArgs {
  const int* header;
  const int* prefix;
  const int* tstart;
  const int2* groups;
  int G, N, K;
  void* out;
  uint8_t* out_scale;
  float limit;
};

// Rows of the 256-row tile in CTA `rank`'s half, and the box that covers them
// (-1: nothing to load).
__device__ __forceinline__ int half_rows(const Item& it, uint32_t rank) {
  return min(128, max(0, it.rows - 128 * (int)rank));
}
__device__ __forceinline__ int half_box(int rows) {
  if (rows <= 0) return -1;
  const int r = (rows + 15) & ~15;
  return r <= 16 ? 0 : (r <= 32 ? 1 : (r <= 64 ? 2 : 3));
}

template <int EPI>
__device__ __forceinline__ void pair_epilogue(const Item& it, uint32_t rank, uint32_t lane_addr, int q, int half,
                                              int lane, int fb, const PairArgs& args, float* red, float* stg,
                                              uint32_t acc_empty_remote) {
  const int lr = 128 * (int)rank + q * 32 + lane;       // row within the 256-row tile
  const bool valid = lr < it.rows;
  const size_t row = (size_t)it.row0 + lr;
  if constexpr (EPI == MOE_EPI_SWIGLU_QUANT) {
    // features 64*half .. +63: gate in columns j, up in columns 128 + j
    uint32_t g[64], u[64];
#pragma unroll
    for (int c = 0; c < 64; c += 16) {
      tmem_ld16(lane_addr + half * 64 + c, *reinterpret_cast<uint32_t(*)[16]>(g + c));
      tmem_ld16(lane_addr + 128 + half * 64 + c, *reinterpret_cast<uint32_t(*)[16]>(u + c));
    }
    tmem_wait_ld_n<64>(g);
    tmem_wait_ld_n<64>(u);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(acc_empty_remote);
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const float h = swiglu_clamped(__uint_as_float(g[j]), __uint_as_float(u[j]), args.limit);
      g[j] = __float_as_uint(h);
      m = fmaxf(m, fabsf(h));
    }
    red[half * 128 + q * 32 + lane] = m;
    named_bar_sync(1, 32 * EPI_WARPS);
    const float amax = fmaxf(red[q * 32 + lane], red[128 + q * 32 + lane]);
    const int k = pow2_scale_exponent(amax);
    const float sk = exp2_int(-k);
    if (valid) {
      const int I = args.N / 2;
      uint8_t* hq = reinterpret_cast<uint8_t*>(args.out) + row * I + fb * 128 + half * 64;
#pragma unroll
      for (int c = 0; c < 64; c += 16) {
        uint32_t w[4];
#pragma unroll
        for (int v = 0; v < 4; ++v)
          w[v] = e4m3x4(__fmul_rn(__uint_as_float(g[c + 4 * v]), sk), __fmul_rn(__uint_as_float(g[c + 4 * v + 1]), sk),
                        __fmul_rn(__uint_as_float(g[c + 4 * v + 2]), sk),
                        __fmul_rn(__uint_as_float(g[c + 4 * v + 3]), sk));
        *reinterpret_cast<uint4*>(hq + c) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (half == 0) args.out_scale[row * (I / 128) + fb] = (uint8_t)(k + 127);
    }
  } else {
    // output columns fb * 256 + 128 * half .. +127: all loaded and the
    // accumulator released, then stored through this warp's staging tile in
    // chunks of 16 columns: a store instruction writes 64 contiguous bytes of
    // each of two rows (lanes 0-15 and 16-31) instead of 16 bytes of 32 rows
    uint32_t v[128];
#pragma unroll
    for (int c = 0; c < 128; c += 16)
      tmem_ld16(lane_addr + half * 128 + c, *reinterpret_cast<uint32_t(*)[16]>(v + c));
    tmem_wait_ld_n<128>(v);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(acc_empty_remote);
    const int rr = lane >> 4, k = lane & 15;               // read-back: row pair offset, column
    const size_t col0 = (size_t)fb * 256 + half * 128;
#pragma unroll
    for (int c = 0; c < 128; c += 16) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        reinterpret_cast<float4*>(stg + lane * Cfg::STG_ROW)[i] =
            make_float4(__uint_as_float(v[c + 4 * i]), __uint_as_float(v[c + 4 * i + 1]),
                        __uint_as_float(v[c + 4 * i + 2]), __uint_as_float(v[c + 4 * i + 3]));
      __syncwarp();
#pragma unroll 4
      for (int r = 0; r < 32; r += 2) {
        const int lr_r = 128 * (int)rank + q * 32 + r + rr;
        const float x = stg[(r + rr) * Cfg::STG_ROW + k];
        if (lr_r < it.rows) {
          const size_t o = ((size_t)it.row0 + lr_r) * args.N + col0 + c + k;
          if constexpr (EPI == MOE_EPI_STORE_F32) reinterpret_cast<float*>(args.out)[o] = x;
          else reinterpret_cast<__nv_bfloat16*>(args.out)[o] = __float2bfloat16_rn(x);
        }
      }
      __syncwarp();
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ PairMaps tmT,
                     const __grid_constant__ CUtensorMap tmS, const PairArgs args) {
  using C = Cfg;
  // SwiGLU reads gate and up from the two weight tiles (paired weight order)
  constexpr bool PAIRED_ORDER = EPI == MOE_EPI_SWIGLU_QUANT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);    // [STAGES], used on rank 0
  uint64_t* empty = full + C::STAGES;                                  // [STAGES]
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;                                  // used on rank 0
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_area = reinterpret_cast<float*>(smem + C::EPI_OFF);
  const GlobalPlan plan{args.prefix, args.tstart, args.groups};

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int n_clusters = gridDim.x / 2;
  const int cluster = blockIdx.x / 2;
  const int G = args.G, N = args.N, K = args.K;
  const int KT = K / 128, KG = (KT + 3) / 4;
  const int n_fb = N / 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * EPI_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmW);
#pragma unroll
    for (int i = 0; i < 4; ++i) prefetch_tensormap(&tmT.tok[i]);
    prefetch_tensormap(&tmT.tok_sf);
    prefetch_tensormap(&tmS);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_wait();
  const int n_items = args.header[0];
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    const uint32_t full0 = cluster_addr(full, 0);     // rank 0's stage barriers
    uint32_t stage = 0, phase = 0;
    for (int item = cluster; item < n_items; item += n_clusters) {
      const Item it = gemm::decode_item(item, plan, G, n_fb, BN);
      const int fb = it.ft;
      const int box_mine = half_box(half_rows(it, rank));
      const int box0 = half_box(half_rows(it, 0)), box1 = half_box(half_rows(it, 1));
      const uint32_t tok_bytes = (box0 < 0 ? 0 : gemm::token_box_rows(box0, 128) * 128) +
                                 (box1 < 0 ? 0 : gemm::token_box_rows(box1, 128) * 128);
      const int p0 = (it.g * n_fb + fb) * KT;                 // paired order: pair of K step kt is p0 + kt
      const int rb = it.g * (N / 128) + 2 * fb;               // plain order: row blocks rb, rb + 1
      bool ok = true;
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        if (elect_one()) {
          uint8_t* st = smem + stage * C::STAGE;
          const uint32_t bar = full0 + stage * 8;
          const bool new_group = (kt & 3) == 0;
          if (rank == 0)
            mbar_arrive_expect_tx(&full[stage], 2 * C::TX_W + tok_bytes + (new_group ? 2 * 512 : 0));
          if (PAIRED_ORDER) {
            tma_load_4d_pair(st + C::B_OFF, &tmW, 0, 0, (int)rank, p0 + kt, bar);
            tma_load_3d_pair(st + C::SFB_OFF, &tmS, 0, 0, p0 + kt, bar);
          } else {
            tma_load_4d_pair(st + C::B_OFF, &tmW, 0, 0, kt, rb + (int)rank, bar);
            tma_load_3d_pair(st + C::SFB_OFF, &tmS, 0, kt, rb, bar);
          }
          if (box_mine >= 0)
            tma_load_2d_pair(st + C::A_OFF, &tmT.tok[box_mine], kt * 128, it.row0 + 128 * (int)rank, bar);
          if (new_group) tma_load_2d_pair(st + C::SFA_OFF, &tmT.tok_sf, 0, (it.t * KG + (kt >> 2)) * 2 + (int)rank, bar);
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (rank 0) --------------------
    if (rank == 0) {
      const uint32_t ring0 = smem_u32(smem);
      const uint32_t sfb_t = tmem + C::SFB_COL, sfa_t = tmem + C::SFA_COL;
      const uint32_t idesc = idesc_mxf8f6f4(0u /*E4M3*/, 5u /*E2M1*/, 256, 256);
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      for (int item = cluster; item < n_items; item += n_clusters) {
        if (!mbar_wait_warp(acc_empty, acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = ring0 + stage * C::STAGE;
          const uint64_t da = sdesc_kmajor_sw128(st + C::A_OFF);
          const uint64_t db = sdesc_kmajor_sw128(st + C::B_OFF);
          const uint32_t asel = (uint32_t)(kt & 3);
          if (elect_one()) {
            tmem_cp_32x128b_warpx4_pair(sfb_t, sdesc_sf(st + C::SFB_OFF));
            tmem_cp_32x128b_warpx4_pair(sfb_t + 4, sdesc_sf(st + C::SFB_OFF + 512));
            if (asel == 0) tmem_cp_32x128b_warpx4_pair(sfa_t, sdesc_sf(st + C::SFA_OFF));
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
              mma_mxf8f6f4_pair(tmem, da + 2 * kb, db + 2 * kb, idesc_with_sf_ids(idesc, asel, (uint32_t)kb),
                                sfa_t | (asel << 30), sfb_t | ((uint32_t)kb << 30), (kt | kb) != 0);
            tc_commit_pair(&empty[stage], 3);
          }
          __syncwarp();
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair(acc_full, 3);
        __syncwarp();
        acc_phase ^= 1u;
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int e = warp - EPI_FIRST;
    const int q = warp & 3;                 // tensor-memory lane quadrant of this warp
    const int half = e >> 2;                // which half of the columns
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t acc_empty0 = cluster_addr(acc_empty, 0);
    uint32_t acc_phase = 0, rb = 0;
    for (int item = cluster; item < n_items; item += n_clusters) {
      const Item it = gemm::decode_item(item, plan, G, n_fb, BN);
      bool ok = mbar_wait(acc_full, acc_phase, abort_flag);
      // the SwiGLU epilogue's warps meet at a named barrier: they continue or
      // stop together, never one without the others
      if (EPI == MOE_EPI_SWIGLU_QUANT) ok = named_bar_and(1, 32 * EPI_WARPS, ok);
      if (!ok) break;
      tc_fence_after();
      pair_epilogue<EPI>(it, rank, lane_addr, q, half, lane, it.ft, args, epi_area + rb * 256,
                         epi_area + e * 32 * C::STG_ROW, acc_empty0);
      acc_phase ^= 1u;
      rb ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();          // no CTA frees tensor memory or exits while its peer still works
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

}  // namespace pair
}  // namespace moe
