// Grouped expert GEMM in PTPC-FP8 ("DeepSeek-V4.1-Flash-Quark-PTPC-FP8"
// walkthrough, 核心参数): FP8 E4M3 weights with one float32 scale per output
// channel (static), FP8 E4M3 activations with one float32 scale per token
// (dynamic).  For every group g and row r in [offsets[g], offsets[g+1]):
//   acc[r, n] = (sum_k a[r, k] * w[g, n, k]) * a_scale[r] * w_scale[g, n]
//
// Both scales are constant along K, so no per-step scaling is needed: the
// tensor core (tcgen05.mma kind::f8f6f4, E4M3 x E4M3, no scale factors)
// accumulates the whole K range of a tile in tensor memory, and the epilogue
// applies the two scales once.
//
// Same swap-AB tiling as the MXFP4 GEMM: a tile is 128 weight rows (output
// channels) x BN token rows; with DUAL (the SwiGLU epilogue) a tile holds the
// gate rows [ft*128, ft*128+128) and the matching up rows N/2 further, so
// one accumulator pair gives both halves of h for 128 channels.
// Warps: 0 TMA producer, 1 TMEM owner + MMA issuer (gate, or the only tile),
// 2..9 epilogue (two warps per tensor-memory lane quadrant, each on half of
// the token columns), 10 MMA issuer of the up tile (DUAL): one warp issuing
// MMAs is bound by its own issue latency, so the two tiles of a pair are
// issued from two warps.
// Tensor memory holds two accumulators (the epilogue of one tile overlaps the
// main loop of the next).
#pragma once

#include "gemm_mxfp4.cuh"

namespace moe {
namespace ptpc {

using namespace sm100;
using gemm::Item;
using gemm::decode_item;

constexpr int kEpiWarps = 8;
constexpr int kThreads = (3 + kEpiWarps) * 32;

__host__ __device__ constexpr int tmem_cols_for(int used) {
  return used <= 32 ? 32 : used <= 64 ? 64 : used <= 128 ? 128 : used <= 256 ? 256 : 512;
}

template <int BN, bool DUAL>
struct Cfg {
  static constexpr int NUM_A = DUAL ? 2 : 1;
  static constexpr int A_BYTES = 128 * 128;            // one E4M3 weight tile per K step
  static constexpr int B_BYTES = BN * 128;             // token rows x 128 K bytes
  static constexpr int B_OFF = NUM_A * A_BYTES;
  static constexpr int STAGE = (B_OFF + B_BYTES + 1023) / 1024 * 1024;
  static constexpr int BAR_BYTES = 256;
  static constexpr int RING_BUDGET = 227 * 1024 - (BAR_BYTES + gemm::kPlanSmemBytes + 1024);
  static constexpr int STAGES_FIT = RING_BUDGET / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int TX = NUM_A * A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = NUM_A * BN;          // gate | up accumulators of one tile
  static constexpr int TMEM_COLS = tmem_cols_for(2 * ACC_COLS);
  static constexpr int CW = BN / 2;                    // token columns per epilogue warp
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int PLAN_OFF = BAR_OFF + BAR_BYTES;
  static constexpr int SMEM_ALLOC = PLAN_OFF + gemm::kPlanSmemBytes + 1024;
  static_assert(STAGES >= 2, "too few stages");
  static_assert(2 * ACC_COLS <= 512, "tensor memory overflow");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory overflow");
  static_assert(BN % 16 == 0 && BN <= 128, "token tile");
};

struct Args {
  const float* w_scale;    // [G, N] per-channel weight scales
  const float* a_scale;    // [a_rows] per-row activation scales
  const int* header;
  const int* prefix;
  const int* tstart;
  const int2* groups;
  int G, N, K;
  void* out;               // float32 / bfloat16 [a_rows, N], or float32 h [a_rows, N/2]
  float limit;
};

template <int BN, bool DUAL, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_ptpc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const Args args) {
  using C = Cfg<BN, DUAL>;
  static_assert(DUAL == (EPI == MOE_EPI_SWIGLU_F32), "the SwiGLU epilogue reads gate/up tile pairs");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;       // [2]
  uint64_t* acc_empty = acc_full + 2;           // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  gemm::SmemPlan plan(smem + C::PLAN_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = args.G, N = args.N, K = args.K;
  const int KT = K / 128;
  const int n_ft = DUAL ? N / 256 : N / 128;
  const int rb_per_g = N / 128;
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::NUM_A);            // one commit per issuer
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], C::NUM_A);
      mbar_init(&acc_empty[b], 32 * kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  // the set-up above is local; the plan and the operands come from earlier kernels
  pdl_wait();
  const int n_items = args.header[0];
  plan.load(args.prefix, args.tstart, args.groups, G);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    uint32_t stage = 0, phase = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = decode_item(item, plan, G, n_ft, BN);
      const int rb0 = it.g * rb_per_g + it.ft;           // gate (or only) weight rows
      const int rb1 = rb0 + rb_per_g / 2;                 // up rows (DUAL)
      bool ok = true;
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        if (elect_one()) {
          uint8_t* st = smem + stage * C::STAGE;
          mbar_arrive_expect_tx(&full[stage], C::TX);
          tma_load_2d(st, &tmA, kt * 128, rb0 * 128, &full[stage]);
          if (DUAL) tma_load_2d(st + C::A_BYTES, &tmA, kt * 128, rb1 * 128, &full[stage]);
          tma_load_2d(st + C::B_OFF, &tmB, kt * 128, it.row0, &full[stage]);
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == 1 || warp == kThreads / 32 - 1) {
    // ------------------------------ MMA issuers ---------------------------
    // issuer 0 (warp 1): tile 0; issuer 1 (last warp): tile 1 of a pair
    const int iss = warp == 1 ? 0 : 1;
    if (iss < C::NUM_A) {
      const uint32_t ring0 = smem_u32(smem);
      uint32_t stage = 0, phase = 0, ab = 0, acc_bits = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const Item it = decode_item(item, plan, G, n_ft, BN);
        const int n_mma = max(16, (it.rows + 15) & ~15);
        const uint32_t idesc = idesc_f8f6f4(0u /*E4M3*/, 0u /*E4M3*/, 128, n_mma);
        if (!mbar_wait_warp(&acc_empty[ab], ((acc_bits >> ab) & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + ab * C::ACC_COLS + iss * BN;
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = ring0 + stage * C::STAGE;
          const uint64_t da = sdesc_kmajor_sw128(st + iss * C::A_BYTES);
          const uint64_t db = sdesc_kmajor_sw128(st + C::B_OFF);
          if (elect_one()) {
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
              mma_f8f6f4(d, da + 2 * kb, db + 2 * kb, idesc, (kt > 0 || kb > 0) ? 1u : 0u);
            tc_commit(&empty[stage]);
          }
          __syncwarp();
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) tc_commit(&acc_full[ab]);
        __syncwarp();
        acc_bits ^= 1u << ab;
        ab ^= 1u;
      }
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int e = warp - 2;
    const int q = warp & 3;                 // tensor-memory lane quadrant of this warp
    const int c_first = (e >> 2) * C::CW;   // first token column of this warp
    const int f = q * 32 + lane;            // output channel within the 128-row tile
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t ab = 0, acc_bits = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = decode_item(item, plan, G, n_ft, BN);
      const float sw0 = __ldg(args.w_scale + (size_t)(it.g * rb_per_g + it.ft) * 128 + f);
      const float sw1 = DUAL ? __ldg(args.w_scale + (size_t)(it.g * rb_per_g + rb_per_g / 2 + it.ft) * 128 + f)
                             : 0.0f;
      if (!mbar_wait(&acc_full[ab], (acc_bits >> ab) & 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t base = lane_addr + ab * C::ACC_COLS + c_first;
#pragma unroll
      for (int c0 = 0; c0 < C::CW; c0 += 8) {
        if (c_first + c0 < it.rows) {       // warp-uniform
          uint32_t g8[8], u8[8];
          tmem_ld8(base + c0, g8);
          if (DUAL) tmem_ld8(base + BN + c0, u8);
          tmem_wait_ld_n<8>(g8);
          if (DUAL) tmem_wait_ld_n<8>(u8);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int c = c_first + c0 + j;
            if (c < it.rows) {
              const float ta = __ldg(args.a_scale + it.row0 + c);
              const float g = __fmul_rn(__fmul_rn(__uint_as_float(g8[j]), ta), sw0);
              if constexpr (EPI == MOE_EPI_SWIGLU_F32) {
                const float u = __fmul_rn(__fmul_rn(__uint_as_float(u8[j]), ta), sw1);
                const int I = N / 2;
                reinterpret_cast<float*>(args.out)[(size_t)(it.row0 + c) * I + it.ft * 128 + f] =
                    swiglu_clamped(g, u, args.limit);
              } else if constexpr (EPI == MOE_EPI_STORE_F32) {
                reinterpret_cast<float*>(args.out)[(size_t)(it.row0 + c) * N + it.ft * 128 + f] = g;
              } else {
                reinterpret_cast<__nv_bfloat16*>(args.out)[(size_t)(it.row0 + c) * N + it.ft * 128 + f] =
                    __float2bfloat16_rn(g);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
      acc_bits ^= 1u << ab;
      ab ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace ptpc
}  // namespace moe
