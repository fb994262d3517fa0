// Grouped expert GEMM with W4AFP8 weights: symmetric INT4, group 128, float32
// weight_scale_inv [N, K/128] ("DeepSeek-V4-Flash-0731-W4AFP8-mt" model card,
// 量化方式 / 权重约定), times FP8 E4M3 activations with per-128 power-of-two
// scales (dynamic, e4m3).
//
// The weight scale is an arbitrary float32 per (row, 128-column group), so it
// cannot ride in the MMA's E8M0 scale slots.  Each 128-wide K step is one
// weight group:
//   * converter warps transcode the INT4 tile to E4M3 in shared memory in the
//     128-byte-swizzled K-major layout the tensor core reads;
//   * the MMA (kind::mxf8f6f4, E4M3 x E4M3, per-128 activation scales)
//     writes the group's partial sum into one of two tensor-memory buffers;
//   * promotion warps multiply each partial by the row's scale_inv and add it
//     into float32 registers, then run the same epilogues as the MXFP4 GEMM.
// Two transcodes:
//   * narrow token tiles (BN <= 32, decode), where the transcode is the
//     critical path: each code n becomes u = n + 8 (0..15) by flipping its top
//     bit, and the byte u is the E4M3 encoding of u * 2^-9 (0..7 subnormal,
//     8..15 with exponent field 1): a mask, an exclusive or and a byte
//     interleave, five operations per eight weights.  The weight scale slots
//     hold 2^9, so the MMA sums x * u; the promotion subtracts 8 * (the token
//     row's scaled activation sum over the step, computed once per call by
//     the plan kernel).  sum(x * u) - 8 * sum(x) = sum(x * n) exactly; in
//     float32 the rounding is relative to sum(|x| * u) rather than
//     sum(|x * n|);
//   * wider tiles (prefill), bound by the operand ring rather than the
//     transcode: byte-permute table lookups of the exact E4M3 codes of
//     -8..7, unit weight scales, no correction.
// Warps: 0 TMA producer, 1 TMEM owner + MMA issuer, then CONV_WARPS
// converters (8 for narrow token tiles, where transcoding is the critical
// path, else 4), then 4 promotion + epilogue warps, then an L2 prefetcher
// that runs pf_steps K steps ahead of the producer (weight tile, token tile,
// and once per item the tile's weight-scale rows and activation sums).
//
// W8 = true is the same GEMM for FP8 E4M3 weights with a float32 scale_inv
// per [128, 128] block (the FP8 shared expert: "DeepSeek-V4-Pro-0813-nvfp4-
// DSpark" walkthrough, only-experts section; "DeepSeek-V4-Flash-SI" model
// card, weight block size [128, 128]): the producer copies the E4M3 tiles
// straight into the MMA layout (128-byte swizzle), there are no converters,
// and the promotion multiplies by the tile's block scale.
#pragma once

#include "gemm_mxfp4.cuh"

namespace moe {
namespace w4a {

using namespace sm100;
using gemm::Item;
using gemm::decode_item;

// INT4 token tiles of at most 32 rows use the offset codes (and the plan
// kernel's activation sums)
__host__ __device__ constexpr bool offset_codes(int bn) { return bn <= 32; }

template <int BN, bool DUAL, bool W8 = false>
struct Cfg {
  static constexpr bool OFFS = !W8 && offset_codes(BN);
  static constexpr int CONV_WARPS = W8 ? 0 : (BN <= 32 ? 8 : 4);
  static constexpr int PROMO_FIRST = 2 + CONV_WARPS;      // first promotion warp
  // promotion warps: 4 (one per tensor-memory lane quadrant, every token column
  // in each thread), or 8 for the 96-row tiles with gate and up (two per
  // quadrant, each on half of the token columns: 2 x 48 accumulators a thread)
  static constexpr int PROMO_WARPS = (W8 && DUAL && BN > 64) ? 8 : 4;
  static constexpr int HALVES = PROMO_WARPS / 4;
  static constexpr int CB = BN / HALVES;                   // token columns per promotion thread
  static constexpr int PF_WARP = PROMO_FIRST + PROMO_WARPS;  // L2 prefetcher
  static constexpr int THREADS = (PF_WARP + 1) * 32;
  static constexpr int CONV_THREADS = CONV_WARPS * 32;
  static constexpr int NA = (BN + 127) / 128;
  static constexpr int NUM_A = DUAL ? 2 : 1;
  static constexpr int RAW_BYTES = W8 ? 0 : 128 * 64;   // INT4 tile as loaded (64 B per row)
  static constexpr int A_BYTES = 128 * 128;           // E4M3 tile for the MMA
  static constexpr int B_BYTES = BN * 128;
  static constexpr int A_OFF = 0;                      // NUM_A E4M3 tiles (1024-aligned)
  static constexpr int B_OFF = NUM_A * A_BYTES;
  static constexpr int RAW_OFF = B_OFF + B_BYTES;      // NUM_A raw tiles
  static constexpr int SFB_OFF = RAW_OFF + NUM_A * RAW_BYTES;
  static constexpr int STAGE_RAW = SFB_OFF + NA * 512;
  static constexpr int STAGE = (STAGE_RAW + 1023) / 1024 * 1024;
  static constexpr int STAGES_FIT = (196 * 1024) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static constexpr int TX = NUM_A * (W8 ? A_BYTES : RAW_BYTES) + B_BYTES;   // + NA * 512 every 4th K step
  // TMEM: two partial buffers of NUM_A * BN columns, then scale factors
  static constexpr int P_COLS = NUM_A * BN;
  static constexpr int SFA_COL = 2 * P_COLS;
  static constexpr int SFB_COL = SFA_COL + 4;
  static constexpr int TMEM_USED = SFB_COL + 4 * NA;
  static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
  static constexpr int SFA_SMEM_OFF = STAGES * STAGE;  // 512 bytes of unit scales
  static constexpr int BAR_OFF = SFA_SMEM_OFF + 512;
  static constexpr int RED_OFF = BAR_OFF + 512;
  static constexpr int CORR_OFF = RED_OFF + 5 * BN * 4;      // after [4][BN] maxima + [BN] scales
  static constexpr int PLAN_OFF = CORR_OFF + 2 * BN * 4;     // after [2][BN] offset terms
  static constexpr int SMEM_USED = PLAN_OFF + gemm::kPlanSmemBytes;
  static constexpr int SMEM_ALLOC = SMEM_USED + 1024;
  static_assert(TMEM_USED <= 512, "tensor memory overflow");
  static_assert(STAGES >= 2, "too few stages");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory overflow");
  static_assert(!DUAL || CB <= 64, "register accumulators: 64 columns a thread with gate and up");
  static_assert(CB <= 128, "register accumulators: 128 columns a thread");
  static_assert(CB % 16 == 0 || BN <= 16, "promotion loads: whole 16-column slices");
  static_assert(!(OFFS && HALVES > 1), "offset codes use one set of promotion warps");
};

// Four INT4 (two's complement nibbles, element 0 in the low nibble) from
// bit s of w -> four E4M3 bytes, by byte-permute table lookups.  A byte
// permute reads the low 3 bits of each selector nibble of the low 16 bits.
__device__ __forceinline__ uint32_t int4x4_to_e4m3x4(uint32_t w, int s) {
  // codes of 0..7 and of -8..-1
  const uint32_t P0 = 0x44403800u, P1 = 0x4E4C4A48u;
  const uint32_t N0 = 0xCACCCED0u, N1 = 0xB8C0C4C8u;
  const uint32_t h = w >> s;
  const uint32_t pos = __byte_perm(P0, P1, h);
  const uint32_t neg = __byte_perm(N0, N1, h);
  // selector nibble i of h >> 3 is odd exactly when element i is negative
  // (its sign bit, plus higher bits times 2): odd table bytes are 0xFF
  const uint32_t mask = __byte_perm(0xFF00FF00u, 0xFF00FF00u, h >> 3);
  return (pos & ~mask) | (neg & mask);
}

// Eight INT4 (two's complement nibbles, element 0 in the low nibble) ->
// eight E4M3 bytes of (n + 8) * 2^-9: lo4 holds elements 0..3, hi4 4..7.
__device__ __forceinline__ void int4x8_to_e4m3_offset(uint32_t w, uint32_t& lo4, uint32_t& hi4) {
  const uint32_t ev = (w & 0x0F0F0F0Fu) ^ 0x08080808u;            // elements 0, 2, 4, 6
  const uint32_t od = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;     // elements 1, 3, 5, 7
  lo4 = __byte_perm(ev, od, 0x5140u);
  hi4 = __byte_perm(ev, od, 0x7362u);
}

struct W4Args {
  const float* w_sinv;     // [G, N, K/128] (INT4) or [G, N/128, K/128] (FP8)
  const uint8_t* a_sf;     // per-tile activation scales (as in the MXFP4 GEMM)
  const float* a_corr;     // offset codes: [a_rows][K/128] terms from the plan kernel
  const int* header;
  const int* prefix;
  const int* tstart;
  const int2* groups;
  int G, N, K;
  void* out;
  uint8_t* out_scale;
  float limit;
  int pf_steps;            // K steps the L2 prefetcher runs ahead of the producer (0: off)
};

// ROWS (with W8): E4M3 weights with the INT4 layout's per-row scales
// [G, N, K/128] -- the E4M3 copy of INT4 weights that transcode_int4_kernel
// writes once per call for wide token tiles.
template <int BN, bool DUAL, int EPI, bool W8 = false, bool ROWS = false>
__global__ void __launch_bounds__(Cfg<BN, DUAL, W8>::THREADS, 1)
    gemm_w4afp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const W4Args args) {
  using C = Cfg<BN, DUAL, W8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* conv = full + C::STAGES;
  uint64_t* empty = conv + C::STAGES;
  uint64_t* pfull = empty + C::STAGES;      // [2]
  uint64_t* pempty = pfull + 2;             // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* produced = reinterpret_cast<volatile int*>(tmem_slot + 2);   // K steps issued so far
  float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
  gemm::SmemPlan plan(smem + C::PLAN_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = args.G, N = args.N, K = args.K;
  const int KT = K / 128;
  const int n_ft = DUAL ? N / 256 : N / 128;
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&conv[s], C::CONV_THREADS > 0 ? C::CONV_THREADS : 1);   // unused with FP8 weights
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], 32 * C::PROMO_WARPS);
    }
    *abort_flag = 0;
    *produced = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  // weight scale slots for every row and sub-block: 2^9 (E8M0 136) for the
  // offset codes stored as u * 2^-9, else 2^0 (E8M0 127)
  if (threadIdx.x < 128)
    reinterpret_cast<uint32_t*>(smem + C::SFA_SMEM_OFF)[threadIdx.x] = C::OFFS ? 0x88888888u : 0x7F7F7F7Fu;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
    // The whole warp walks the items; one elected lane issues the copies.
    const int rb_per_g = N / 128;
    uint32_t stage = 0, phase = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = decode_item(item, plan, G, n_ft, BN);
      const int rb0 = it.g * rb_per_g + it.ft;
      const int rb1 = rb0 + rb_per_g / 2;
      const uint8_t* sfb = args.a_sf + (size_t)it.t * ((KT + 3) / 4) * C::NA * 512;
      bool ok = true;
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        if (elect_one()) {
          uint8_t* st = smem + stage * C::STAGE;
          const bool new_group = (kt & 3) == 0;
          mbar_arrive_expect_tx(&full[stage], C::TX + (new_group ? C::NA * 512 : 0));
          if constexpr (W8) {
            tma_load_2d(st + C::A_OFF, &tmA, kt * 128, rb0 * 128, &full[stage]);
            if (DUAL) tma_load_2d(st + C::A_OFF + C::A_BYTES, &tmA, kt * 128, rb1 * 128, &full[stage]);
          } else {
            tma_load_2d(st + C::RAW_OFF, &tmA, kt * 64, rb0 * 128, &full[stage]);
            if (DUAL) tma_load_2d(st + C::RAW_OFF + C::RAW_BYTES, &tmA, kt * 64, rb1 * 128, &full[stage]);
          }
          tma_load_2d(st + C::B_OFF, &tmB, kt * 128, it.row0, &full[stage]);
          if (new_group) bulk_load(st + C::SFB_OFF, sfb + (size_t)(kt >> 2) * C::NA * 512, C::NA * 512, &full[stage]);
          *produced = *produced + 1;
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == C::PF_WARP) {
    // ------------------------------ L2 prefetcher --------------------------
    // A hint only: gives up quietly when the CTA aborts or after the wait bound.
    if (args.pf_steps > 0 && lane == 0) {
      const int rb_per_g = N / 128;
      const uint64_t t0 = globaltimer_ns();
      int pf = 0;
      bool go = true;
      for (int item = blockIdx.x; item < n_items && go; item += gridDim.x) {
        const Item it = decode_item(item, plan, G, n_ft, BN);
        const int rb0 = it.g * rb_per_g + it.ft;
        const int rb1 = rb0 + rb_per_g / 2;
        for (int kt = 0; kt < KT && go; ++kt) {
          while (pf >= *produced + args.pf_steps) {
            if (*abort_flag || globaltimer_ns() - t0 > kWaitTimeoutNs) { go = false; break; }
            __nanosleep(128);
          }
          if (!go) break;
          if (kt == 0) {
            // the per-row weight scales of the tile(s) and the token rows'
            // activation sums, once per item (16-byte aligned ranges only)
            if constexpr (!(W8 && !ROWS)) {
              const float* s0 = args.w_sinv + (size_t)rb0 * 128 * KT;
              const uint32_t bytes = 128u * KT * 4u;
              if ((reinterpret_cast<uintptr_t>(s0) & 15u) == 0) bulk_prefetch(s0, bytes);
              if (DUAL) {
                const float* s1 = args.w_sinv + (size_t)rb1 * 128 * KT;
                if ((reinterpret_cast<uintptr_t>(s1) & 15u) == 0) bulk_prefetch(s1, bytes);
              }
            }
            if (C::OFFS && args.a_corr != nullptr) {
              const float* c0 = args.a_corr + (size_t)it.row0 * KT;
              const uint32_t bytes = (uint32_t)(it.rows * KT * 4) & ~15u;
              if ((reinterpret_cast<uintptr_t>(c0) & 15u) == 0 && bytes > 0) bulk_prefetch(c0, bytes);
            }
          }
          if constexpr (W8) {
            tma_prefetch_2d(&tmA, kt * 128, rb0 * 128);
            if (DUAL) tma_prefetch_2d(&tmA, kt * 128, rb1 * 128);
          } else {
            tma_prefetch_2d(&tmA, kt * 64, rb0 * 128);
            if (DUAL) tma_prefetch_2d(&tmA, kt * 64, rb1 * 128);
          }
          tma_prefetch_2d(&tmB, kt * 128, it.row0);
          ++pf;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ----------------------------
    // The whole warp runs the loop and waits; one elected lane issues.
    const uint32_t sfa_smem = smem_u32(smem + C::SFA_SMEM_OFF);
    if (elect_one()) tmem_cp_32x128b_warpx4(tmem + C::SFA_COL, sdesc_sf(sfa_smem));
    __syncwarp();
    uint32_t stage = 0, phase = 0;
    uint32_t pb = 0, pbits = 0;            // bit b: phase of partial buffer b
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = decode_item(item, plan, G, n_ft, BN);
      const int n_mma = max(16, (it.rows + 15) & ~15);
      const uint32_t idesc = idesc_mxf8f6f4(0u /*E4M3*/, 0u /*E4M3*/, 128, n_mma);
      bool ok = true;
      for (int kt = 0; kt < KT && ok; ++kt) {
        if (!mbar_wait_warp(&pempty[pb], ((pbits >> pb) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        // FP8 weights are MMA-ready when they land; INT4 after the converters
        if (!mbar_wait_warp(W8 ? &full[stage] : &conv[stage], phase, abort_flag)) { ok = false; break; }
        tc_fence_after();     // orders the MMA after the promotion warps' release of the partial buffer
        const uint32_t st = smem_u32(smem + stage * C::STAGE);
        const uint32_t dcol = tmem + pb * C::P_COLS;
        const uint32_t kb_b = (uint32_t)(kt & 3);
        if (elect_one()) {
          if ((kt & 3) == 0) {
#pragma unroll
            for (int a = 0; a < C::NA; ++a)
              tmem_cp_32x128b_warpx4(tmem + C::SFB_COL + 4 * a, sdesc_sf(st + C::SFB_OFF + 512 * a));
          }
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint32_t id = idesc_with_sf_ids(idesc, kb, kb_b);
            const uint64_t bdesc = sdesc_kmajor_sw128(st + C::B_OFF + kb * 32);
            const uint32_t sfa = (tmem + C::SFA_COL) | ((uint32_t)kb << 30);
            const uint32_t sfb = (tmem + C::SFB_COL) | (kb_b << 30);
            mma_mxf8f6f4(dcol, sdesc_kmajor_sw128(st + C::A_OFF + kb * 32), bdesc, id, sfa, sfb, kb != 0);
            if (DUAL)
              mma_mxf8f6f4(dcol + BN, sdesc_kmajor_sw128(st + C::A_OFF + C::A_BYTES + kb * 32), bdesc, id, sfa,
                           sfb, kb != 0);
          }
          tc_commit(&empty[stage]);
          tc_commit(&pfull[pb]);
        }
        __syncwarp();
        pbits ^= 1u << pb;
        pb ^= 1u;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (!W8 && warp < C::PROMO_FIRST) {
    // ------------------------------ converters ----------------------------
    // thread layout: converter warp w (0..CONV_WARPS-1), lane l -> 16-byte
    // input chunk (l & 3) of rows w*8 + (l >> 2) + 8*CONV_WARPS*j;
    // conflict-free reads of the raw tile and conflict-free writes into the
    // 128-byte swizzle.
    const int w = warp - 2;
    const int chunk = lane & 3;
    uint32_t stage = 0, phase = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      bool ok = true;
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
        uint8_t* st = smem + stage * C::STAGE;
#pragma unroll
        for (int a = 0; a < C::NUM_A; ++a) {
          const uint8_t* raw = st + C::RAW_OFF + a * C::RAW_BYTES;
          uint8_t* dst = st + C::A_OFF + a * C::A_BYTES;
#pragma unroll
          for (int j = 0; j < 128 / (8 * (C::CONV_WARPS > 0 ? C::CONV_WARPS : 1)); ++j) {
            const int r = w * 8 + (lane >> 2) + 8 * C::CONV_WARPS * j;
            const uint4 in = *reinterpret_cast<const uint4*>(raw + r * 64 + chunk * 16);
            uint4 o0, o1;
            if constexpr (C::OFFS) {
              int4x8_to_e4m3_offset(in.x, o0.x, o0.y);
              int4x8_to_e4m3_offset(in.y, o0.z, o0.w);
              int4x8_to_e4m3_offset(in.z, o1.x, o1.y);
              int4x8_to_e4m3_offset(in.w, o1.z, o1.w);
            } else {
              o0.x = int4x4_to_e4m3x4(in.x, 0);
              o0.y = int4x4_to_e4m3x4(in.x, 16);
              o0.z = int4x4_to_e4m3x4(in.y, 0);
              o0.w = int4x4_to_e4m3x4(in.y, 16);
              o1.x = int4x4_to_e4m3x4(in.z, 0);
              o1.y = int4x4_to_e4m3x4(in.z, 16);
              o1.z = int4x4_to_e4m3x4(in.w, 0);
              o1.w = int4x4_to_e4m3x4(in.w, 16);
            }
            const int c0 = 2 * chunk, c1 = 2 * chunk + 1;
            *reinterpret_cast<uint4*>(dst + r * 128 + ((c0 ^ (r & 7)) << 4)) = o0;
            *reinterpret_cast<uint4*>(dst + r * 128 + ((c1 ^ (r & 7)) << 4)) = o1;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&conv[stage]);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else {
    // --------------------------- promotion + epilogue ---------------------
    const int q = warp & 3;
    const int f = q * 32 + lane;
    const int half = (warp - C::PROMO_FIRST) >> 2;     // token-column half (0 with 4 promotion warps)
    const int col0 = half * C::CB;
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t pb = 0, pbits = 0;
    // offset-term slot, alternating per K step across items: the barrier of
    // step s + 1 separates the reads of step s from the writes of step s + 2
    uint32_t cslot = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = decode_item(item, plan, G, n_ft, BN);
      const int rb_per_g = N / 128;
      // scale_inv of this thread's weight row per K step: [G, N, K/128] (INT4
      // and its E4M3 copy, per row) or [G, N/128, K/128] (FP8, one value per
      // 128-row block)
      constexpr bool BLOCK_SCALE = W8 && !ROWS;
      const float* s0 = args.w_sinv + (BLOCK_SCALE ? (size_t)(it.g * rb_per_g + it.ft) * KT
                                                   : ((size_t)(it.g * rb_per_g + it.ft) * 128 + f) * KT);
      const float* s1 = args.w_sinv + (BLOCK_SCALE ? (size_t)(it.g * rb_per_g + rb_per_g / 2 + it.ft) * KT
                                                   : ((size_t)(it.g * rb_per_g + rb_per_g / 2 + it.ft) * 128 + f) * KT);
      constexpr int CB = C::CB;
      float acc0[CB], acc1[DUAL ? CB : 1];
#pragma unroll
      for (int c = 0; c < CB; ++c) acc0[c] = 0.0f;
#pragma unroll
      for (int c = 0; c < (DUAL ? CB : 1); ++c) acc1[c] = 0.0f;
      const int my_cols = max(0, min(CB, it.rows - col0));      // valid token columns of this thread
      const int nchunks = (my_cols + 15) >> 4;
      bool ok = true;
      float sc0 = __ldg(s0), sc1 = DUAL ? __ldg(s1) : 0.0f;
      // offset codes: thread f < rows fetches token column f's term of each
      // K step; the 128 promotion threads swap them through shared memory
      const bool has_c = C::OFFS && f < it.rows;
      const float* cf = has_c ? args.a_corr + (size_t)(it.row0 + f) * KT : nullptr;
      float cv = has_c ? __ldg(cf) : 0.0f;
      for (int kt = 0; kt < KT; ++kt) {
        const float nx0 = (kt + 1 < KT) ? __ldg(s0 + kt + 1) : 0.0f;
        const float nx1 = (DUAL && kt + 1 < KT) ? __ldg(s1 + kt + 1) : 0.0f;
        const float* cs = reinterpret_cast<const float*>(smem + C::CORR_OFF) + cslot * BN;
        if constexpr (C::OFFS) {
          const float nc = (has_c && kt + 1 < KT) ? __ldg(cf + kt + 1) : 0.0f;
          if (f < BN) reinterpret_cast<float*>(smem + C::CORR_OFF)[cslot * BN + f] = cv;
          cv = nc;
          cslot ^= 1u;
          // the barrier publishes the terms and makes the give-up decision the
          // same in all 128 threads (the epilogue has more barriers)
          const bool got = mbar_wait(&pfull[pb], (pbits >> pb) & 1u, abort_flag);
          if (!named_bar_and(1, 128, got)) { ok = false; break; }
        } else {
          if (!mbar_wait(&pfull[pb], (pbits >> pb) & 1u, abort_flag)) { ok = false; break; }
        }
        tc_fence_after();
        const uint32_t base = lane_addr + pb * C::P_COLS + col0;
#pragma unroll
        for (int ch = 0; ch < (CB + 15) / 16; ++ch) {
          if (ch < nchunks) {
            uint32_t r0[16];
            tmem_ld16(base + ch * 16, r0);
            if constexpr (DUAL) {
              uint32_t r1[16];
              tmem_ld16(base + BN + ch * 16, r1);
              tmem_wait_ld(r0, r1);
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float c = C::OFFS ? cs[col0 + ch * 16 + j] : 0.0f;
                acc0[ch * 16 + j] = fmaf(sc0, __uint_as_float(r0[j]) - c, acc0[ch * 16 + j]);
                acc1[ch * 16 + j] = fmaf(sc1, __uint_as_float(r1[j]) - c, acc1[ch * 16 + j]);
              }
            } else {
              tmem_wait_ld(r0);
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float c = C::OFFS ? cs[col0 + ch * 16 + j] : 0.0f;
                acc0[ch * 16 + j] = fmaf(sc0, __uint_as_float(r0[j]) - c, acc0[ch * 16 + j]);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&pempty[pb]);
        pbits ^= 1u << pb;
        pb ^= 1u;
        sc0 = nx0;
        sc1 = nx1;
      }
      if (!ok) break;
      // ---- epilogue from registers ----
      if constexpr (EPI == MOE_EPI_SWIGLU_QUANT) {
        const int I = N / 2;
        uint8_t* hq = reinterpret_cast<uint8_t*>(args.out);
        float* h = acc0;                    // h replaces the gate accumulators
        // this half's [4 warps][CB] column maxima, then its [CB] scales
        float* rr = red + half * 4 * CB;
        float* sk = red + 4 * BN + half * CB;
#pragma unroll
        for (int c = 0; c < CB; ++c) {
          h[c] = swiglu_clamped(acc0[c], acc1[DUAL ? c : 0], args.limit);
          const float m = warp_max_nonneg(fabsf(h[c]));
          if (lane == 0) rr[q * CB + c] = m;
        }
        named_bar_sync(1 + half, 128);
        // one thread per token column turns the column maximum into the scale
        if (f < my_cols) {
          const int c = f;
          const float amax = fmaxf(fmaxf(rr[c], rr[CB + c]), fmaxf(rr[2 * CB + c], rr[3 * CB + c]));
          const int k = pow2_scale_exponent(amax);
          sk[c] = exp2_int(-k);
          args.out_scale[(size_t)(it.row0 + col0 + c) * (I / 128) + it.ft] = (uint8_t)(k + 127);
        }
        named_bar_sync(1 + half, 128);
        uint8_t* hq_f = hq + (size_t)(it.row0 + col0) * I + it.ft * 128 + f;
#pragma unroll
        for (int c = 0; c < CB; ++c) {
          if (c < my_cols) hq_f[(size_t)c * I] = (uint8_t)(e4m3x2(__fmul_rn(h[c], sk[c]), 0.0f) & 0xFFu);
        }
        named_bar_sync(1 + half, 128);
      } else {
#pragma unroll
        for (int c = 0; c < CB; ++c) {
          if (c < my_cols) {
            const size_t o = (size_t)(it.row0 + col0 + c) * N + it.ft * 128 + f;
            if constexpr (EPI == MOE_EPI_STORE_F32)
              reinterpret_cast<float*>(args.out)[o] = acc0[c];
            else
              reinterpret_cast<__nv_bfloat16*>(args.out)[o] = __float2bfloat16_rn(acc0[c]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// INT4 [G, N, K/2] -> E4M3 [G, N, K] (the exact codes of -8..7), once per
// call, for the wide-token-tile path: the GEMM then streams E4M3 tiles with
// TMA instead of transcoding every weight tile once per token tile.  Grid
// (chunks of 256 x 16 input bytes, G); groups without rows (offsets[g + 1] <=
// offsets[g]) are skipped, their copy is never read.  Offsets are only read
// here; the plan kernel validates them.
__global__ void __launch_bounds__(256) transcode_int4_kernel(const uint4* __restrict__ q,
                                                             const int32_t* __restrict__ offsets,
                                                             int64_t chunks_per_group, uint4* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int g = blockIdx.y;
  if (__ldg(offsets + g + 1) <= __ldg(offsets + g)) return;
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= chunks_per_group) return;
  const int64_t i = (int64_t)g * chunks_per_group + c;
  const uint4 in = __ldg(q + i);
  uint4 o0, o1;
  o0.x = int4x4_to_e4m3x4(in.x, 0);
  o0.y = int4x4_to_e4m3x4(in.x, 16);
  o0.z = int4x4_to_e4m3x4(in.y, 0);
  o0.w = int4x4_to_e4m3x4(in.y, 16);
  o1.x = int4x4_to_e4m3x4(in.z, 0);
  o1.y = int4x4_to_e4m3x4(in.z, 16);
  o1.z = int4x4_to_e4m3x4(in.w, 0);
  o1.w = int4x4_to_e4m3x4(in.w, 16);
  out[2 * i] = o0;
  out[2 * i + 1] = o1;
}

}  // namespace w4a
}  // namespace moe
