// Grouped expert GEMM: FP8 E4M3 activations x MXFP4 (E2M1 + E8M0/32) weights
// on the Blackwell block-scaled tensor cores (tcgen05.mma kind::mxf8f6f4).
//
// Formats follow the "DeepSeek-V4-Flash-SI" model card (低精度计算): expert
// weights FP4 E2M1 with an E8M0 scale per 32 elements, activations FP8 E4M3
// with a power-of-two scale per 128 elements.  The per-128 activation scale
// is an E8M0 value, so it enters the MMA as four identical per-32 scales.
//
// Mapping ("swap AB"): the weight tile is the MMA's M = 128 operand (A) and
// the token tile its N operand (B), so small token counts per expert (decode)
// still fill the 128-row tensor-core datapath; the accumulator lives in tensor
// memory as [128 weight rows (lanes)] x [BN tokens (columns)].
//
// Work decomposition: tokens of each expert (group) are cut into tiles of BN
// rows; a work item is (token tile, 128-row weight tile).  For the w1/w3
// projection (DUAL) one item holds the gate tile and the up tile of the same
// 128 output features so the SwiGLU epilogue has both in one thread.  Items
// are ordered group-major, then weight tile, then token tile, so CTAs running
// at the same time stream the same weight tile from L2.
//
// CTA roles (persistent kernel, one CTA per SM, 6 warps):
//   warp 0        TMA producer: weight tiles (FP4 unpacked to bytes in shared
//                 memory by the 16U4_ALIGN16B tensor-map type), token tile, and
//                 the pre-interleaved scale-factor blocks (1-D bulk copies)
//   warp 1        TMEM owner and MMA issuer (one thread): scale factors
//                 shared -> TMEM (tcgen05.cp), 4 MMAs of K = 32 per stage
//   warps 2..5    epilogue: TMEM -> registers -> global (float32 / bf16 /
//                 SwiGLU + per-128 FP8 requantisation)
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace moe {
namespace gemm {

using namespace sm100;

constexpr int kThreads = 192;

template <int BN, bool DUAL>
struct Cfg {
  static constexpr int NA = (BN + 127) / 128;            // 128-row scale blocks of the token tile
  static constexpr int NUM_A = DUAL ? 2 : 1;
  static constexpr int A_BYTES = 128 * 128;              // one FP4 weight tile in shared memory
  static constexpr int A_TX = 128 * 128 / 2;             // bytes the tensor copy moves for it
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SF_BYTES = 512;
  static constexpr int A0_OFF = 0;
  static constexpr int A1_OFF = A_BYTES;
  static constexpr int B_OFF = NUM_A * A_BYTES;
  static constexpr int SFA_OFF = B_OFF + B_BYTES;
  static constexpr int SFB_OFF = SFA_OFF + NUM_A * SF_BYTES;
  static constexpr int STAGE_RAW = SFB_OFF + NA * SF_BYTES;
  static constexpr int STAGE = (STAGE_RAW + 1023) / 1024 * 1024;
  static constexpr int STAGES_FIT = (200 * 1024) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int TX = NUM_A * A_TX + B_BYTES + NUM_A * SF_BYTES + NA * SF_BYTES;
  // tensor-memory columns
  static constexpr int D0_COL = 0;
  static constexpr int D1_COL = BN;
  static constexpr int SFA_COL = NUM_A * BN;             // 4 columns per weight tile
  static constexpr int SFB_COL = SFA_COL + 4 * NUM_A;    // 4 columns per 128 tokens
  static constexpr int TMEM_USED = SFB_COL + 4 * NA;
  static constexpr int TMEM_COLS = 512;
  // shared memory after the stages
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int RED_OFF = BAR_OFF + 256;
  static constexpr int SMEM_USED = RED_OFF + 4 * 16 * 4;
  static constexpr int SMEM_ALLOC = SMEM_USED + 1024;     // slack for 1024-byte alignment
  static_assert(TMEM_USED <= TMEM_COLS, "tensor memory overflow");
  static_assert(STAGES >= 2, "too few pipeline stages");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory overflow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "bad token tile");
};

// ----------------------- plan (work decomposition) -------------------------
// Workspace layout, all offsets 256-byte aligned:
//   header   int32[4]: n_items, n_tiles, n_ft, BN
//   prefix   int32[G+1]: first work item of each group
//   tstart   int32[G]:   first token tile of each group
//   tiles    int2[max_tiles]: (first row, rows) of each token tile
//   a_sf     uint8[max_tiles * KT * NA * 512]: per-tile interleaved activation scales
struct WsLayout {
  size_t header, prefix, tstart, tiles, a_sf, total;
  int max_tiles;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline WsLayout ws_layout(int a_rows, int G, int K, int BN) {
  WsLayout L;
  L.max_tiles = ceil_div(a_rows, BN) + G;
  const int KT = K / 128, NA = ceil_div(BN, 128);
  L.header = 0;
  L.prefix = align256(16);
  L.tstart = L.prefix + align256(4 * (size_t)(G + 1));
  L.tiles = L.tstart + align256(4 * (size_t)G);
  L.a_sf = L.tiles + align256(8 * (size_t)L.max_tiles);
  L.total = L.a_sf + align256((size_t)L.max_tiles * KT * NA * 512);
  return L;
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ inline int block_exclusive_scan_1024(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const int base = wid ? warp_sums[wid - 1] : 0;
  *total = warp_sums[31];
  __syncthreads();
  return base + x - v;
}

// One block of 1024 threads; thread g handles group g (G <= 1024).
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ offsets, int G, int BN,
                                                    int n_ft, int* __restrict__ header,
                                                    int* __restrict__ prefix, int* __restrict__ tstart,
                                                    int2* __restrict__ tiles) {
  const int g = threadIdx.x;
  int rows = 0, r0 = 0;
  if (g < G) {
    r0 = offsets[g];
    rows = offsets[g + 1] - r0;
    if (rows < 0 || (g == 0 && r0 != 0)) {
      record_error(MOE_ERR_INVALID);
      rows = 0;
    }
  }
  const int nt = ceil_div(rows, BN);
  int n_tiles, n_items;
  const int t0 = block_exclusive_scan_1024(nt, &n_tiles);
  const int i0 = block_exclusive_scan_1024(nt * n_ft, &n_items);
  if (g < G) {
    tstart[g] = t0;
    prefix[g] = i0;
    for (int j = 0; j < nt; ++j) tiles[t0 + j] = make_int2(r0 + j * BN, min(BN, rows - j * BN));
  }
  if (g == 0) {
    prefix[G] = n_items;
    header[0] = n_items;
    header[1] = n_tiles;
    header[2] = n_ft;
    header[3] = BN;
  }
}

// Interleave the per-128 activation scales of each token tile into the
// tensor-memory scale order: for token n of a 128-row block, the 32-bit word
// at byte (n % 32) * 16 + (n / 32) * 4 holds its scale four times (one per
// 32-element sub-block of the 128-wide K step).  Rows past the tile are 0.
__global__ void __launch_bounds__(128) tile_act_scales_kernel(const uint8_t* __restrict__ sx, int KT,
                                                              const int* __restrict__ header,
                                                              const int2* __restrict__ tiles, int NA,
                                                              uint8_t* __restrict__ a_sf) {
  const int t = blockIdx.x, kt = blockIdx.y;
  if (t >= header[1]) return;
  const int2 tr = tiles[t];
  const int n = threadIdx.x;
  for (int a = 0; a < NA; ++a) {
    const int r = a * 128 + n;
    uint32_t b = (r < tr.y) ? (uint32_t)sx[(size_t)(tr.x + r) * KT + kt] : 0u;
    uint8_t* blk = a_sf + ((size_t)(t * KT + kt) * NA + a) * 512;
    *reinterpret_cast<uint32_t*>(blk + (n & 31) * 16 + (n >> 5) * 4) = b * 0x01010101u;
  }
}

struct Item {
  int g, ft, t, row0, rows;
};

__device__ __forceinline__ Item decode_item(int item, const int* __restrict__ prefix,
                                            const int* __restrict__ tstart,
                                            const int2* __restrict__ tiles, int G, int n_ft) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= item) lo = mid; else hi = mid - 1;
  }
  Item it;
  it.g = lo;
  const int base = __ldg(prefix + lo);
  const int nt = (__ldg(prefix + lo + 1) - base) / n_ft;
  const int local = item - base;
  it.ft = local / nt;
  it.t = __ldg(tstart + lo) + local % nt;
  const int2 tr = __ldg(tiles + it.t);
  it.row0 = tr.x;
  it.rows = tr.y;
  return it;
}

struct GemmArgs {
  const uint8_t* w_sf;     // prepared weight scales [G, N/128, KT, 512]
  const uint8_t* a_sf;     // per-tile activation scales
  const int* header;
  const int* prefix;
  const int* tstart;
  const int2* tiles;
  int G, N, K;
  void* out;
  uint8_t* out_scale;
  float limit;
};

template <int BN, bool DUAL, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_mxfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmArgs args) {
  using C = Cfg<BN, DUAL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(smem + C::RED_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = args.G, N = args.N, K = args.K;
  const int KT = K / 128;
  const int n_ft = DUAL ? N / 256 : N / 128;
  const int n_items = args.header[0];

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 128);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const Item it = decode_item(item, args.prefix, args.tstart, args.tiles, G, n_ft);
        const int rb_per_g = N / 128;
        const int rb0 = it.g * rb_per_g + it.ft;
        const int rb1 = rb0 + rb_per_g / 2;
        const uint8_t* sfa0 = args.w_sf + (size_t)rb0 * KT * 512;
        const uint8_t* sfa1 = args.w_sf + (size_t)rb1 * KT * 512;
        const uint8_t* sfb = args.a_sf + (size_t)it.t * KT * C::NA * 512;
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* st = smem + stage * C::STAGE;
          mbar_arrive_expect_tx(&full[stage], C::TX);
          tma_load_2d(st + C::A0_OFF, &tmA, kt * 128, rb0 * 128, &full[stage]);
          if (DUAL) tma_load_2d(st + C::A1_OFF, &tmA, kt * 128, rb1 * 128, &full[stage]);
          tma_load_2d(st + C::B_OFF, &tmB, kt * 128, it.row0, &full[stage]);
          bulk_load(st + C::SFA_OFF, sfa0 + (size_t)kt * 512, 512, &full[stage]);
          if (DUAL) bulk_load(st + C::SFA_OFF + 512, sfa1 + (size_t)kt * 512, 512, &full[stage]);
          bulk_load(st + C::SFB_OFF, sfb + (size_t)kt * C::NA * 512, C::NA * 512, &full[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const Item it = decode_item(item, args.prefix, args.tstart, args.tiles, G, n_ft);
        const int n_mma = max(16, (it.rows + 15) & ~15);
        const uint32_t idesc = idesc_mxf8f6f4(5u /*E2M1*/, 0u /*E4M3*/, 128, n_mma);
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag)) break;
        acc_phase ^= 1u;
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + stage * C::STAGE);
          tmem_cp_32x128b_warpx4(tmem + C::SFA_COL, sdesc_sf(st + C::SFA_OFF));
          if (DUAL) tmem_cp_32x128b_warpx4(tmem + C::SFA_COL + 4, sdesc_sf(st + C::SFA_OFF + 512));
#pragma unroll
          for (int a = 0; a < C::NA; ++a)
            tmem_cp_32x128b_warpx4(tmem + C::SFB_COL + 4 * a, sdesc_sf(st + C::SFB_OFF + 512 * a));
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint32_t id = idesc_with_sf_ids(idesc, kb, kb);
            const uint64_t bdesc = sdesc_kmajor_sw128(st + C::B_OFF + kb * 32);
            const uint32_t acc = (kt | kb) != 0;
            mma_mxf8f6f4(tmem + C::D0_COL, sdesc_kmajor_sw128(st + C::A0_OFF + kb * 32), bdesc, id,
                         (tmem + C::SFA_COL) | ((uint32_t)kb << 30),
                         (tmem + C::SFB_COL) | ((uint32_t)kb << 30), acc);
            if (DUAL)
              mma_mxf8f6f4(tmem + C::D1_COL, sdesc_kmajor_sw128(st + C::A1_OFF + kb * 32), bdesc, id,
                           (tmem + C::SFA_COL + 4) | ((uint32_t)kb << 30),
                           (tmem + C::SFB_COL) | ((uint32_t)kb << 30), acc);
          }
          tc_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int q = warp & 3;                 // TMEM sub-partition of this warp
    const int f = q * 32 + lane;            // weight row (output feature) within the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t acc_phase = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = decode_item(item, args.prefix, args.tstart, args.tiles, G, n_ft);
      if (!mbar_wait(acc_full, acc_phase, abort_flag)) break;
      acc_phase ^= 1u;
      tc_fence_after();
      for (int c0 = 0; c0 < it.rows; c0 += 16) {
        uint32_t r0[16];
        tmem_ld16(lane_addr + C::D0_COL + c0, r0);
        if constexpr (EPI == MOE_EPI_SWIGLU_QUANT) {
          uint32_t r1[16];
          tmem_ld16(lane_addr + C::D1_COL + c0, r1);
          tmem_wait_ld(r0, r1);
          const int I = N / 2;
          float h[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            h[j] = swiglu_clamped(__uint_as_float(r0[j]), __uint_as_float(r1[j]), args.limit);
            const float m = warp_max_nonneg(fabsf(h[j]));
            if (lane == 0) red[q * 16 + j] = m;
          }
          named_bar_sync(1, 128);
          uint8_t* hq = reinterpret_cast<uint8_t*>(args.out);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float amax = fmaxf(fmaxf(red[j], red[16 + j]), fmaxf(red[32 + j], red[48 + j]));
            const int k = pow2_scale_exponent(amax);
            const float s = exp2_int(-k);
            if (c0 + j < it.rows) {
              const size_t row = (size_t)(it.row0 + c0 + j);
              hq[row * I + it.ft * 128 + f] = (uint8_t)(e4m3x2(__fmul_rn(h[j], s), 0.0f) & 0xFFu);
              if (f == 0) args.out_scale[row * (I / 128) + it.ft] = (uint8_t)(k + 127);
            }
          }
          named_bar_sync(1, 128);
        } else {
          tmem_wait_ld(r0);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (c0 + j < it.rows) {
              const size_t o = (size_t)(it.row0 + c0 + j) * N + it.ft * 128 + f;
              if constexpr (EPI == MOE_EPI_STORE_F32)
                reinterpret_cast<float*>(args.out)[o] = __uint_as_float(r0[j]);
              else
                reinterpret_cast<__nv_bfloat16*>(args.out)[o] = __float2bfloat16_rn(__uint_as_float(r0[j]));
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Weight-scale interleave (load-time): [M, N, K/32] -> [M, N/128, K/128, 512].
__global__ void prepare_weight_scales_kernel(const uint8_t* __restrict__ src, int64_t n_blocks, int K,
                                             uint8_t* __restrict__ dst) {
  // one thread per (128-row block, 128-column step, row): 4 bytes
  const int KT = K / 128;
  const int64_t total = n_blocks * KT * 128;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int m = (int)(i & 127);
    const int64_t bk = i >> 7;               // (block, kt)
    const int kt = (int)(bk % KT);
    const int64_t blk = bk / KT;
    const int64_t row = blk * 128 + m;
    const uint32_t v = *reinterpret_cast<const uint32_t*>(src + row * (K / 32) + kt * 4);
    *reinterpret_cast<uint32_t*>(dst + bk * 512 + (m & 31) * 16 + (m >> 5) * 4) = v;
  }
}

}  // namespace gemm
}  // namespace moe
