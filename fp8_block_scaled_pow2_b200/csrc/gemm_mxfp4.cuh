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
// rows; a work item is (token tile, weight tile pair).  A pair (PAIR) is two
// 128-row weight tiles that share the token tile: for the w1/w3 projection
// the gate tile and the up tile of the same 128 output features (paired
// weight order), so the SwiGLU epilogue has both in one thread; otherwise two
// adjacent 128-row blocks of the output (plain order).  Without PAIR (N not a
// multiple of 256) an item is one weight tile.  Items are ordered
// group-major, then weight tile, then token tile, so CTAs running at the same
// time stream the same weight tiles from L2.
//
// CTA roles (persistent kernel, one CTA per SM, 12 warps):
//   warp 0        TMA producer: weight tiles (FP4 unpacked to one nibble per
//                 byte in shared memory by the 16U4_ALIGN16B tensor-map type),
//                 their pre-interleaved scale blocks, the token tile and the
//                 token scales
//   warp 1        TMEM owner and MMA issuer 0: scale factors shared -> TMEM
//                 (tcgen05.cp), 4 MMAs of K = 32 per 128-wide K step
//   warp 10       MMA issuer 1 (tile 1 of a pair, or alternate K steps of a
//                 single tile; see Cfg::ISSUERS)
//   warps 2..9    epilogue: TMEM -> registers -> global (float32 / bf16 /
//                 SwiGLU + per-128 FP8 requantisation)
//   warp 11       L2 prefetcher on decode-sized token tiles (see GemmArgs::pf_steps)
// The producer and issuer loops run converged on their whole warp and one
// elected lane issues the copies and tensor-core instructions.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace moe {
namespace gemm {

using namespace sm100;

constexpr int kThreads = 384;                   // 12 warps: producer, 2 MMA issuers, 8 workers, L2 prefetcher
constexpr int kIssuer1Warp = 10;
constexpr int kPrefetchWarp = 11;

// Prepared weights (moe_prepare_weights): one 8704-byte block per (128-row
// block, 128-wide K step): 128 rows x 64 bytes of packed E2M1 nibbles, then
// the 512-byte scale block in tensor-memory order.  For the SwiGLU projection
// the gate block and the matching up block of each K step are adjacent.
constexpr int kWBlock = 8192 + 512;

// Groups per call (one plan thread per group) and the shared-memory copy of
// the plan: prefix [G + 1], tstart [G], groups [G].
constexpr int kMaxGroups = 1024;
constexpr int kPlanSmemBytes = 16 * (kMaxGroups + 4);

// Pipeline: per 128-wide K step one 4-D TMA copy writes the item's weight
// tiles (both tiles of a pair: its box holds two prepared blocks) straight
// into the unpacked one-nibble-per-byte layout the MMA reads (16U4_ALIGN16B),
// one TMA copy over a view of the prepared blocks' scale parts brings their
// 512-byte scale blocks, a 2-D TMA copy the token tile, and every fourth step
// a bulk copy the token scales: 3.25 copy instructions per K step.
//
// Shared memory bandwidth is what the pipeline spends: per K step of a full
// tile pair the tensor core reads 64 KB (8 MMAs x (4 KB of weights + 4 KB of
// tokens)) and the copies write ~49 KB.  The token tile is therefore copied
// with the smallest of four boxes (16, 32, 64 or BN rows) that covers the
// item's rows: a ragged tile of 20 tokens writes 4 KB per step, not 16 KB.
//
// Tensor maps of the prepared weights (built by the host):
//   tmA  [pairs][2][128 rows][128 nibbles] in paired order (box: one pair),
//        [row blocks][K steps][128 rows][128 nibbles] in plain order (box: the
//        item's one or two row blocks at one K step);
//   tmS  the same views of the scale blocks as 128 32-bit words each.
template <int BN, bool PAIR>
struct Cfg {
  static constexpr int NA = (BN + 127) / 128;            // 128-row scale blocks of the token tile
  static constexpr int NUM_A = PAIR ? 2 : 1;
  static constexpr int A_BYTES = 128 * 128;              // one MMA-ready FP4 weight tile
  static constexpr int A_PACKED = 128 * 64;              // the same tile packed (global layout)
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SF_BYTES = 512;
  // ring slot: [unpacked weight tiles][token tile][weight scales][token scales]
  static constexpr int A0_OFF = 0;
  static constexpr int B_OFF = NUM_A * A_BYTES;
  static constexpr int SFA_OFF = B_OFF + B_BYTES;          // weight scales of tile a: SFA_OFF + a * SF_BYTES
  static constexpr int SFB_OFF = SFA_OFF + NUM_A * SF_BYTES;
  static constexpr int STAGE_RAW = SFB_OFF + NA * SF_BYTES;
  static constexpr int STAGE = (STAGE_RAW + 1023) / 1024 * 1024;
  // the ring takes the shared memory the rest of the kernel leaves (227 KB
  // per CTA; barriers, SwiGLU reduction, plan and alignment slack)
  static constexpr int CW0 = BN / 2;                     // epilogue columns per warp, see CW
  static constexpr int RED_BYTES = 2 * 4 * CW0 * 4 + 2 * CW0 * 4;   // SwiGLU maxima + column scales
  static constexpr int RING_BUDGET = 227 * 1024 - (512 + RED_BYTES + kPlanSmemBytes + 1024);
  static constexpr int STAGES_FIT = RING_BUDGET / STAGE;
  static constexpr int STAGES = STAGES_FIT > 16 ? 16 : STAGES_FIT;
  // transaction bytes of a step (the TMA counts the packed weight bytes);
  // steps that also load token scales add NA * 512
  // (plus the token tile's box and, every fourth step, the token scales)
  static constexpr int TX_W = NUM_A * (A_PACKED + SF_BYTES);
  // MMA issue: one warp issuing block-scaled MMAs is bound by its own issue
  // latency (about 60 cycles per instruction, the tensor work of N = 128),
  // so two warps issue.  With a tile pair issuer 0 computes tile 0 and
  // issuer 1 tile 1; with one tile they take alternate K steps into two
  // partial accumulators the epilogue adds.
  // tensor-memory columns: ACC_BUFS accumulators of 2 * BN columns, then one
  // scale set (weight + token scales) per issuer
  static constexpr int ISSUERS = 2;
  static constexpr int ACC_COLS = 2 * BN;
  static constexpr int SF_SET = 4 + 4 * NA;
  static constexpr int SF_COLS = 2 * SF_SET;
  static constexpr int ACC_BUFS = (2 * ACC_COLS + SF_COLS <= 512) ? 2 : 1;
  static constexpr int SF_COL = ACC_BUFS * ACC_COLS;      // issuer i: SF_COL + i * SF_SET
  static constexpr int TMEM_USED = SF_COL + SF_COLS;
  static constexpr int CONSUMERS = PAIR ? ISSUERS : 1;    // issuers reading each ring stage
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : (TMEM_USED <= 256 ? 256 : 512);
  // epilogue warps: each owns 32 weight rows (its TMEM sub-partition) and
  // BN / (EPI_WARPS / 4) token columns
  static constexpr int EPI_WARPS = 8;
  static constexpr int EPI_FIRST = 2;
  static constexpr int CW = BN / (EPI_WARPS / 4);
  static_assert(CW == CW0, "ring budget assumes 8 epilogue warps");
  // shared memory after the ring
  static constexpr int BAR_OFF = STAGES * STAGE;
  static constexpr int RED_OFF = BAR_OFF + 512;
  static constexpr int PLAN_OFF = RED_OFF + RED_BYTES;            // SmemPlan (kPlanSmemBytes)
  static constexpr int SMEM_USED = PLAN_OFF + kPlanSmemBytes;
  static constexpr int SMEM_ALLOC = SMEM_USED + 1024;     // slack for 1024-byte alignment
  static_assert(TMEM_USED <= 512, "tensor memory overflow");
  static_assert(STAGES >= 2, "too few pipeline stages");
  static_assert(2 * STAGES + 4 + 2 <= 64, "barrier area overflow");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory overflow");
  static_assert(SMEM_ALLOC > 116 * 1024, "one CTA per SM keeps tensor-memory allocation uncontended");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 128, "bad token tile");
  // epilogue loads of 16 (or, for CW = 8, 8) columns start on a multiple of
  // their width: each warp's column slice starts at a multiple of CW
  static_assert(CW == 8 || CW % 16 == 0, "epilogue column slices must be whole 16-column loads");
};

// Token-tile tensor maps whose boxes hold 16, 32, 64 and BN rows (capped at
// BN); an item copies with the smallest box that covers its MMA width.
struct TokenMaps {
  CUtensorMap m[4];
};
__host__ __device__ __forceinline__ int token_box_rows(int i, int BN) { return (16 << i) < BN ? (16 << i) : BN; }
__device__ __forceinline__ int token_box_index(int n_mma) {
  return n_mma <= 16 ? 0 : (n_mma <= 32 ? 1 : (n_mma <= 64 ? 2 : 3));
}

// ----------------------- plan (work decomposition) -------------------------
// Workspace layout, all offsets 256-byte aligned:
//   header   int32[4]: n_items, n_tiles, n_ft, BN
//   prefix   int32[G+1]: first work item of each group
//   tstart   int32[G]:   first token tile of each group
//   groups   int2[G]:    (first row, rows) of each group, rows 0 for an invalid plan
//   a_sf     uint8[max_tiles * KG * NA * 512]: per-tile activation scales, interleaved
//            for tensor memory, four 128-wide K steps per 512-byte block (KG = ceil(KT/4))
struct WsLayout {
  size_t header, prefix, tstart, groups, a_sf, a_corr, total;
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
  L.groups = L.tstart + align256(4 * (size_t)G);
  L.a_sf = L.groups + align256(8 * (size_t)G);
  L.a_corr = L.a_sf + align256((size_t)L.max_tiles * ((KT + 3) / 4) * NA * 512);
  L.total = L.a_corr + align256(4 * (size_t)a_rows * KT);
  return L;
}

// Sum of sixteen E4M3 values (bytes of v, any order) in float32; each pair is
// converted exactly to half precision first.
__device__ __forceinline__ float sum_e4m3x16(const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> (16 * h)), __NV_E4M3);
      const float2 f = __half22float2(__half2(r));
      s += f.x + f.y;
    }
  }
  return s;
}

constexpr int kPrepThreads = 128;
constexpr int kPrepPerThread = (kMaxGroups + kPrepThreads) / kPrepThreads;   // covers G + 1 entries

// Plan and token scales of one GEMM call in one launch; one block per token
// tile (grid = the tile bound ceil(a_rows / BN) + G).  Every block loads the
// group offsets and scans the tile counts itself (G <= 1024: 9 entries per
// thread), finds its tile, and interleaves that tile's per-128 activation
// scales into the tensor-memory scale order: for token n of a 128-row block,
// the 32-bit word at byte (n % 32) * 16 + (n / 32) * 4 of block (tile, g)
// holds its scales of the K steps 4g .. 4g+3, one per byte (the MMA of K step
// kt selects byte kt % 4); rows past the tile and K steps past K are 0.
// Block 0 writes the plan.  Unless the offsets are nondecreasing from
// offsets[0] >= 0 to offsets[G] <= a_rows, the plan has no work and
// MOE_ERR_INVALID is recorded, so no tile ever addresses rows outside the
// operands or the workspace.  (offsets[0] > 0 lets a caller run a subset of
// groups, e.g. one group of a larger grouping.)
//
// split_tile > 0 splits every group between two kernels, each with its own
// plan: part 0 takes the group's first floor(rows / split_tile) * split_tile
// rows (whole tiles of the SM-pair kernel), part 1 the remaining rows.  A
// group's entry in `groups` then holds the (first row, rows) of its part.
//
// With a_corr (the INT4 weight GEMM on narrow token tiles), each block also
// writes, for every row r of its tile and K step kt, a_corr[r * KT + kt] =
// 8 * 2^(sx - 127) * (sum of the row's 128 E4M3 values in that step): the GEMM
// multiplies the activations by the weights offset by +8 (codes 0..15) and
// subtracts this term.
__global__ void __launch_bounds__(kPrepThreads) gemm_prep_kernel(const int32_t* __restrict__ offsets, int G,
                                                                 int a_rows, int BN, int n_ft,
                                                                 const uint8_t* __restrict__ sx, int KT,
                                                                 int* __restrict__ header, int* __restrict__ prefix,
                                                                 int* __restrict__ tstart, int2* __restrict__ groups,
                                                                 uint8_t* __restrict__ a_sf,
                                                                 const uint8_t* __restrict__ aq,
                                                                 float* __restrict__ a_corr, int split_tile,
                                                                 int split_part) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_off[kMaxGroups + 1];
  __shared__ int s_t0[kMaxGroups + 1];      // first tile of each group; s_t0[G] = tiles in all
  __shared__ int s_skip[kMaxGroups];        // rows of the group before this plan's part
  __shared__ int s_warp[kPrepThreads / 32];
  const int tid = threadIdx.x;
  for (int g = tid; g <= G; g += kPrepThreads) s_off[g] = offsets[g];
  __syncthreads();
  bool bad = false;
  for (int g = tid; g < G; g += kPrepThreads)
    bad |= s_off[g + 1] < s_off[g] || (g == 0 && s_off[0] < 0) || (g == G - 1 && s_off[G] > a_rows);
  bad = __syncthreads_or(bad);
  // exclusive scan of the tile counts; thread tid owns groups [tid*P, tid*P + P)
  const int g0 = tid * kPrepPerThread;
  int nt[kPrepPerThread];
  int local = 0;
#pragma unroll
  for (int i = 0; i < kPrepPerThread; ++i) {
    const int g = g0 + i;
    int rows = (!bad && g < G) ? s_off[g + 1] - s_off[g] : 0;
    int skip = 0;
    if (split_tile > 0) {
      const int whole = rows / split_tile * split_tile;
      if (split_part == 0) rows = whole;
      else { skip = whole; rows -= whole; }
    }
    if (g < G) s_skip[g] = skip;
    nt[i] = ceil_div(rows, BN);
    local += nt[i];
  }
  const int lane = tid & 31, wid = tid >> 5;
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[wid] = x;
  __syncthreads();
  int base = x - local;
  for (int w = 0; w < wid; ++w) base += s_warp[w];
#pragma unroll
  for (int i = 0; i < kPrepPerThread; ++i) {
    const int g = g0 + i;
    if (g <= G) s_t0[g] = base;
    base += nt[i];
  }
  __syncthreads();
  const int n_tiles = s_t0[G];
  if (blockIdx.x == 0) {
    if (bad && tid == 0) record_error(MOE_ERR_INVALID);
    for (int g = tid; g < G; g += kPrepThreads) {
      tstart[g] = s_t0[g];
      prefix[g] = s_t0[g] * n_ft;
      int rows = s_off[g + 1] - s_off[g];
      if (split_tile > 0) rows = split_part == 0 ? rows / split_tile * split_tile : rows - s_skip[g];
      groups[g] = bad ? make_int2(0, 0) : make_int2(s_off[g] + s_skip[g], rows);
    }
    if (tid == 0) {
      prefix[G] = n_tiles * n_ft;
      header[0] = n_tiles * n_ft;
      header[1] = n_tiles;
      header[2] = n_ft;
      header[3] = BN;
    }
  }
  const int t = blockIdx.x;
  if (t >= n_tiles || sx == nullptr) return;     // sx == nullptr: the plan only
  // the group of tile t: the last g with s_t0[g] <= t (empty groups share
  // their successor's first tile and sort before it)
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_t0[mid] <= t) lo = mid; else hi = mid - 1;
  }
  const int row0 = s_off[lo] + s_skip[lo] + (t - s_t0[lo]) * BN;
  const int g_end = (split_tile > 0 && split_part == 0) ? s_off[lo] + (s_off[lo + 1] - s_off[lo]) / split_tile * split_tile
                                                        : s_off[lo + 1];
  const int rows = min(BN, g_end - row0);
  const int KG = (KT + 3) / 4, NA = ceil_div(BN, 128);
  for (int kg = 0; kg < KG; ++kg) {
    for (int a = 0; a < NA; ++a) {
      const int n = tid;
      const int r = a * 128 + n;
      uint32_t w = 0;
      if (r < rows) {
        const uint8_t* src = sx + (size_t)(row0 + r) * KT;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (4 * kg + j < KT) w |= (uint32_t)src[4 * kg + j] << (8 * j);
      }
      uint8_t* blk = a_sf + ((size_t)(t * KG + kg) * NA + a) * 512;
      *reinterpret_cast<uint32_t*>(blk + (n & 31) * 16 + (n >> 5) * 4) = w;
    }
  }
  if (a_corr == nullptr) return;
  // eight threads per (row, K step), 16 bytes each; the loop count is uniform
  // over the block so that the shuffles see full warps
  const int sub = tid & 7, n_pairs = rows * KT;
  for (int p0 = 0; p0 < n_pairs; p0 += kPrepThreads / 8) {
    const int p = p0 + (tid >> 3);
    const int r = p / KT, kt = p - r * KT;
    float s = 0.0f;
    if (p < n_pairs) {
      const uint4 v = *reinterpret_cast<const uint4*>(aq + ((size_t)(row0 + r) * KT + kt) * 128 + sub * 16);
      s = sum_e4m3x16(v);
    }
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 2);
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 4);
    if (p < n_pairs && sub == 0) {
      const size_t o = (size_t)(row0 + r) * KT + kt;
      a_corr[o] = 8.0f * s * exp2_int((int)sx[o] - 127);
    }
  }
}

struct Item {
  int g, ft, t, row0, rows;
};

// The plan of one GEMM call, copied to shared memory at kernel start so that
// decoding a work item reads no global memory.
struct SmemPlan {
  int* prefix;     // [G + 1]
  int* tstart;     // [G]
  int2* groups;    // [G]
  __device__ explicit SmemPlan(uint8_t* base)
      : prefix(reinterpret_cast<int*>(base)),
        tstart(reinterpret_cast<int*>(base + 4 * (kMaxGroups + 4))),
        groups(reinterpret_cast<int2*>(base + 8 * (kMaxGroups + 4))) {}
  // all threads of the block; the caller synchronises before use
  __device__ void load(const int* g_prefix, const int* g_tstart, const int2* g_groups, int G) {
    for (int g = threadIdx.x; g <= G; g += blockDim.x) {
      prefix[g] = g_prefix[g];
      if (g < G) {
        tstart[g] = g_tstart[g];
        groups[g] = g_groups[g];
      }
    }
  }
};

// Work item -> (group, weight tile, token tile).  Items are group-major, then
// weight tile, then token tile.  Plan: SmemPlan, or any struct with the same
// three arrays (prefix, tstart, groups).
template <class Plan>
__device__ __forceinline__ Item decode_item(int item, const Plan& plan, int G, int n_ft, int BN) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (plan.prefix[mid] <= item) lo = mid; else hi = mid - 1;
  }
  Item it;
  it.g = lo;
  const int base = plan.prefix[lo];
  const int nt = (plan.prefix[lo + 1] - base) / n_ft;
  const int local = item - base;
  it.ft = local / nt;
  const int tl = local - it.ft * nt;
  it.t = plan.tstart[lo] + tl;
  const int2 gr = plan.groups[lo];
  it.row0 = gr.x + tl * BN;
  it.rows = min(BN, gr.y - tl * BN);
  return it;
}

struct GemmArgs {
  const uint8_t* w;        // prepared weights (nibbles + scales), see kWBlock
  const uint8_t* a_sf;     // per-tile activation scales
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

// Epilogue of one work item for one epilogue warp: copy the warp's slice of
// the accumulator (32 weight rows x CW token columns) to registers, release
// the TMEM buffer (the next item's MMAs may start), then finish from registers:
// float32 / bf16 stores, or SwiGLU + per-128 power-of-two FP8 requantisation
// with the group maximum reduced across the four warps of a column slice.
template <int BN, bool PAIR, int EPI, int CW>
__device__ __forceinline__ void epilogue_item(const Item& it, uint32_t src, int f, int q, int half, int lane,
                                              int N, int KT, const GemmArgs& args, float* red,
                                              uint64_t* acc_empty_bar) {
  const int c_base = half * CW;
  const int my_cols = max(0, min(CW, it.rows - c_base));     // valid columns of this warp
  // PAIR: v0 / v1 = tile 0 / tile 1 (gate / up for SwiGLU).  Otherwise v0 / v1
  // are the even / odd K-step partial sums (v1 holds nothing when there is a
  // single K step).
  const bool use_v1 = PAIR || KT > 1;
  uint32_t v0[CW];
  uint32_t v1[CW];
  // 16-column loads, and an 8-column load for a remainder (CW % 16 == 8)
#pragma unroll
  for (int c = 0; c < CW; c += (c + 16 <= CW ? 16 : 8)) {
    if (c < my_cols) {
      if (c + 16 <= CW) {
        tmem_ld16(src + c, *reinterpret_cast<uint32_t(*)[16]>(v0 + c));
        if (use_v1) tmem_ld16(src + BN + c, *reinterpret_cast<uint32_t(*)[16]>(v1 + c));
      } else {
        tmem_ld8(src + c, v0 + c);
        if (use_v1) tmem_ld8(src + BN + c, v1 + c);
      }
    }
  }
  tmem_wait_ld_n<CW>(v0);
  tmem_wait_ld_n<CW>(v1);
  tc_fence_before();
  mbar_arrive(acc_empty_bar);
  if constexpr (!PAIR) {
    if (use_v1) {
#pragma unroll
      for (int c = 0; c < CW; ++c) v0[c] = __float_as_uint(__uint_as_float(v0[c]) + __uint_as_float(v1[c]));
    }
  }

  if constexpr (EPI == MOE_EPI_SWIGLU_QUANT) {
    // The 128 features of a token column live in the four warps of this half
    // (one TMEM sub-partition each): per-warp maxima go through shared memory,
    // one thread per column turns the column maximum into the scale, and every
    // thread then quantises its 128 features x CW tokens with that scale.
    const int I = N / 2;
    float* rr = red + half * 4 * CW;             // [4 warps][CW] partial maxima
    float* sk = red + 2 * 4 * CW + half * CW;    // [CW] 2^-k per column
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      const float h = swiglu_clamped(__uint_as_float(v0[c]), __uint_as_float(v1[c]), args.limit);
      v0[c] = __float_as_uint(h);
      const float m = warp_max_nonneg(fabsf(h));
      if (lane == 0) rr[q * CW + c] = m;
    }
    named_bar_sync(1 + half, 128);
    if (f < my_cols) {
      const int c = f;
      const float amax = fmaxf(fmaxf(rr[c], rr[CW + c]), fmaxf(rr[2 * CW + c], rr[3 * CW + c]));
      const int k = pow2_scale_exponent(amax);
      sk[c] = exp2_int(-k);
      args.out_scale[(size_t)(it.row0 + c_base + c) * (I / 128) + it.ft] = (uint8_t)(k + 127);
    }
    named_bar_sync(1 + half, 128);
    uint8_t* hq = reinterpret_cast<uint8_t*>(args.out) + (size_t)(it.row0 + c_base) * I + it.ft * 128 + f;
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      if (c < my_cols)
        hq[(size_t)c * I] = (uint8_t)(e4m3x2(__fmul_rn(__uint_as_float(v0[c]), sk[c]), 0.0f) & 0xFFu);
    }
    named_bar_sync(1 + half, 128);
  } else {
    // output column block of tile 0 (tile 1 is the next block with PAIR)
    const int cb = PAIR ? 2 * it.ft : it.ft;
#pragma unroll
    for (int c = 0; c < CW; ++c) {
      if (c < my_cols) {
        const size_t o = (size_t)(it.row0 + c_base + c) * N + cb * 128 + f;
        if constexpr (EPI == MOE_EPI_STORE_F32) {
          reinterpret_cast<float*>(args.out)[o] = __uint_as_float(v0[c]);
          if (PAIR) reinterpret_cast<float*>(args.out)[o + 128] = __uint_as_float(v1[c]);
        } else {
          reinterpret_cast<__nv_bfloat16*>(args.out)[o] = __float2bfloat16_rn(__uint_as_float(v0[c]));
          if (PAIR) reinterpret_cast<__nv_bfloat16*>(args.out)[o + 128] = __float2bfloat16_rn(__uint_as_float(v1[c]));
        }
      }
    }
  }
}

// One MMA-issuing warp: the whole warp runs the loop and waits, one elected
// lane issues the scale copies, MMAs and commits.  Every value that does not
// change within an item is computed before its K loop; per-K-block operands
// are constant offsets of per-stage bases (a descriptor's start-address field
// is the byte address / 16, so +32 bytes is +2).
template <int BN, bool PAIR>
__device__ __forceinline__ void mma_issuer(const int iss, uint8_t* smem, const uint32_t tmem, uint64_t* full,
                                           uint64_t* empty, uint64_t* acc_full,
                                           uint64_t* acc_empty, volatile int* abort_flag, const SmemPlan& plan,
                                           const GemmArgs& args, const int n_items,
                                           const int KT, const int n_ft) {
  using C = Cfg<BN, PAIR>;
  const uint32_t ring0 = smem_u32(smem);
  const uint32_t sfa_t = tmem + C::SF_COL + iss * C::SF_SET;     // 4 columns per weight tile
  const uint32_t sfb_t = sfa_t + 4;
  uint32_t stage = 0, phase = 0, ab = 0, acc_bits = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const Item it = decode_item(item, plan, args.G, n_ft, BN);
    const int n_mma = max(16, (it.rows + 15) & ~15);
    const uint32_t idesc = idesc_mxf8f6f4(5u /*E2M1*/, 0u /*E4M3*/, 128, n_mma);
    uint32_t id_kb[4];
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) id_kb[kb] = idesc_with_sf_ids(idesc, kb, 0);
    if (!mbar_wait_warp(&acc_empty[ab], ((acc_bits >> ab) & 1u) ^ 1u, abort_flag)) return;
    tc_fence_after();
    const uint32_t d = tmem + ab * C::ACC_COLS + iss * BN;
    for (int kt = 0; kt < KT; ++kt) {
      const bool mine = PAIR || (kt & 1) == iss;
      if (mine) {
        if (!mbar_wait_warp(&full[stage], phase, abort_flag)) return;
        const uint32_t st = ring0 + stage * C::STAGE;
        const uint32_t a_base = st + (PAIR ? iss * C::A_BYTES : 0);
        const uint32_t bsel = (uint32_t)(kt & 3);
        const uint32_t sfb = sfb_t | (bsel << 30);
        const uint64_t da = sdesc_kmajor_sw128(a_base);
        const uint64_t db = sdesc_kmajor_sw128(st + C::B_OFF);
        // this issuer's first step of the item starts a fresh accumulator
        const uint32_t first = PAIR ? (kt != 0) : (kt > 1);
        if (elect_one()) {
          tmem_cp_32x128b_warpx4(sfa_t, sdesc_sf(st + C::SFA_OFF + (PAIR ? iss * C::SF_BYTES : 0)));
          if ((kt & 3) == (PAIR ? 0 : iss)) {
#pragma unroll
            for (int a = 0; a < C::NA; ++a) tmem_cp_32x128b_warpx4(sfb_t + 4 * a, sdesc_sf(st + C::SFB_OFF + 512 * a));
          }
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            mma_mxf8f6f4(d, da + 2 * kb, db + 2 * kb, id_kb[kb] | (bsel << 4), sfa_t | ((uint32_t)kb << 30), sfb,
                         kb ? 1u : first);
          }
          tc_commit(&empty[stage]);
        }
        __syncwarp();
      }
      if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
    }
    if (elect_one()) tc_commit(&acc_full[ab]);
    __syncwarp();
    acc_bits ^= 1u << ab;
    if (C::ACC_BUFS == 2) ab ^= 1u;
  }
}

template <int BN, bool PAIR, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_mxfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ TokenMaps tmB,
                      const __grid_constant__ CUtensorMap tmS, const GemmArgs args) {
  using C = Cfg<BN, PAIR>;
  // SwiGLU reads gate and up from the two tiles of a pair (paired weight order)
  constexpr bool PAIRED_ORDER = EPI == MOE_EPI_SWIGLU_QUANT;
  static_assert(!PAIRED_ORDER || PAIR, "the SwiGLU epilogue needs gate/up tile pairs");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;       // [ACC_BUFS]
  uint64_t* acc_empty = acc_full + 2;           // [ACC_BUFS]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* produced = reinterpret_cast<volatile int*>(tmem_slot + 2);   // K steps issued so far
  float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
  SmemPlan plan(smem + C::PLAN_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = args.G, N = args.N, K = args.K;
  const int KT = K / 128;
  const int n_ft = PAIR ? N / 256 : N / 128;
  const int rb_per_g = N / 128;
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::CONSUMERS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], C::ISSUERS);
      mbar_init(&acc_empty[b], 32 * C::EPI_WARPS);
    }
    *abort_flag = 0;
    *produced = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
#pragma unroll
    for (int i = 0; i < 4; ++i) prefetch_tensormap(&tmB.m[i]);
    prefetch_tensormap(&tmS);
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
    // The whole warp walks the items (its coordinates stay warp-uniform); one
    // elected lane issues each step's copies.
    uint32_t stage = 0, phase = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = decode_item(item, plan, G, n_ft, BN);
      // paired order: the gate and up blocks of K step kt are pair p0 + kt;
      // plain order: the item's first 128-row block is rb (its K steps are
      // contiguous), the second one rb + 1
      const int p0 = (it.g * n_ft + it.ft) * KT;
      const int rb = it.g * rb_per_g + (PAIR ? 2 * it.ft : it.ft);
      const uint8_t* sfb = args.a_sf + (size_t)it.t * ((KT + 3) / 4) * C::NA * 512;
      // token rows the MMAs read (the issuers' N) and the box that covers them
      const int box = token_box_index(max(16, (it.rows + 15) & ~15));
      const CUtensorMap* tm_tok = &tmB.m[box];
      const uint32_t tx = C::TX_W + token_box_rows(box, BN) * 128;
      bool ok = true;
      for (int kt = 0; kt < KT; ++kt) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        if (elect_one()) {
          uint8_t* st = smem + stage * C::STAGE;
          // token scales: one block per 4 K steps, read by each issuer at its
          // first step of the group (issuers alternate steps without PAIR)
          const bool new_group = PAIR ? (kt & 3) == 0 : (kt & 3) < 2;
          mbar_arrive_expect_tx(&full[stage], tx + (new_group ? C::NA * 512 : 0));
          if (PAIRED_ORDER) {
            tma_load_4d(st + C::A0_OFF, &tmA, 0, 0, 0, p0 + kt, &full[stage]);
            tma_load_3d(st + C::SFA_OFF, &tmS, 0, 0, p0 + kt, &full[stage]);
          } else {
            tma_load_4d(st + C::A0_OFF, &tmA, 0, 0, kt, rb, &full[stage]);
            tma_load_3d(st + C::SFA_OFF, &tmS, 0, kt, rb, &full[stage]);
          }
          tma_load_2d(st + C::B_OFF, tm_tok, kt * 128, it.row0, &full[stage]);
          if (new_group) bulk_load(st + C::SFB_OFF, sfb + (size_t)(kt >> 2) * C::NA * 512, C::NA * 512, &full[stage]);
          *produced = *produced + 1;
        }
        __syncwarp();
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == kPrefetchWarp) {
    // ------------------------------ L2 prefetcher --------------------------
    // Walks the producer's sequence of K steps pf_steps ahead of it and
    // prefetches each step's weight blocks and token tile into L2, so more of
    // the HBM stream is in flight than the shared-memory ring holds.  A hint
    // only: it gives up quietly when the CTA aborts or after the wait bound.
    if (args.pf_steps > 0 && lane == 0) {
      const uint64_t t0 = globaltimer_ns();
      int pf = 0;
      bool go = true;
      for (int item = blockIdx.x; item < n_items && go; item += gridDim.x) {
        const Item it = decode_item(item, plan, G, n_ft, BN);
        size_t blk0, kt_step, a_step;
        if (PAIRED_ORDER) {
          blk0 = (size_t)(it.g * n_ft + it.ft) * KT * 2;
          kt_step = 2;
          a_step = 1;
        } else {
          blk0 = (size_t)(it.g * rb_per_g + (PAIR ? 2 * it.ft : it.ft)) * KT;
          kt_step = 1;
          a_step = KT;
        }
        for (int kt = 0; kt < KT && go; ++kt) {
          while (pf >= *produced + args.pf_steps) {
            if (*abort_flag || globaltimer_ns() - t0 > kWaitTimeoutNs) { go = false; break; }
            __nanosleep(128);
          }
          if (!go) break;
          const size_t blk = blk0 + (size_t)kt * kt_step;
          if (PAIRED_ORDER) {
            bulk_prefetch(args.w + blk * kWBlock, 2 * kWBlock);
          } else {
#pragma unroll
            for (int a = 0; a < C::NUM_A; ++a) bulk_prefetch(args.w + (blk + (size_t)a * a_step) * kWBlock, kWBlock);
          }
          tma_prefetch_2d(&tmB.m[token_box_index(max(16, (it.rows + 15) & ~15))], kt * 128, it.row0);
          ++pf;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer 0 ---------------------------
    mma_issuer<BN, PAIR>(0, smem, tmem, full, empty, acc_full, acc_empty, abort_flag, plan, args,
                         n_items, KT, n_ft);
  } else if (warp == kIssuer1Warp) {
    // ------------------------------ MMA issuer 1 ---------------------------
    mma_issuer<BN, PAIR>(1, smem, tmem, full, empty, acc_full, acc_empty, abort_flag, plan, args,
                         n_items, KT, n_ft);
  } else {
    // ------------------------------ epilogue ------------------------------
    const int e = warp - C::EPI_FIRST;
    const int q = warp & 3;                 // TMEM sub-partition of this warp
    const int half = e >> 2;                // which token-column slice (8 epilogue warps)
    const int f = q * 32 + lane;            // weight row (output feature) within the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t ab = 0, acc_bits = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const Item it = decode_item(item, plan, G, n_ft, BN);
      bool ok = mbar_wait(&acc_full[ab], (acc_bits >> ab) & 1u, abort_flag);
      // the SwiGLU epilogue's four warps of a half meet at a named barrier:
      // they continue or stop together, never one without the others
      if (EPI == MOE_EPI_SWIGLU_QUANT) ok = named_bar_and(1 + half, 128, ok);
      if (!ok) break;
      tc_fence_after();
      epilogue_item<BN, PAIR, EPI, C::CW>(it, lane_addr + ab * C::ACC_COLS + half * C::CW, f, q, half, lane, N,
                                          KT, args, red, &acc_empty[ab]);
      acc_bits ^= 1u << ab;
      if (C::ACC_BUFS == 2) ab ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Weight preparation (load-time): MXFP4 [M, N, K/2] nibbles + [M, N, K/32]
// E8M0 -> 8704-byte blocks (kWBlock), one per (128-row block, 128-wide K step):
// rows of 64 packed bytes, then the scales in tensor-memory order (byte
// (m % 32) * 16 + (m / 32) * 4 + b: row m, 32-element sub-block b).  Block order
// plain [M, N/128, K/128]; paired (gate | up halves of a w1/w3 matrix)
// [M, N/256, K/128, 2].  One block of 128 threads per output block; thread m
// moves row m.
__global__ void __launch_bounds__(128) prepare_weights_kernel(const uint8_t* __restrict__ fp4,
                                                              const uint8_t* __restrict__ e8m0, int N, int K,
                                                              int paired, uint8_t* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int KT = K / 128, RB = N / 128;
  const int64_t ob = blockIdx.x;            // output block index
  int64_t mat, rb;
  int kt;
  if (paired) {
    const int h = (int)(ob & 1);
    const int64_t t = ob >> 1;              // (mat, ft, kt)
    kt = (int)(t % KT);
    const int64_t mf = t / KT;
    mat = mf / (RB / 2);
    rb = (mf % (RB / 2)) + h * (RB / 2);
  } else {
    kt = (int)(ob % KT);
    const int64_t mr = ob / KT;
    mat = mr / RB;
    rb = mr % RB;
  }
  const int m = threadIdx.x;
  const int64_t row = (mat * RB + rb) * 128 + m;
  const uint4* src = reinterpret_cast<const uint4*>(fp4 + row * (K / 2) + kt * 64);
  uint4* dst = reinterpret_cast<uint4*>(out + ob * kWBlock + m * 64);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = __ldg(src + i);
  const uint32_t v = *reinterpret_cast<const uint32_t*>(e8m0 + row * (K / 32) + kt * 4);
  *reinterpret_cast<uint32_t*>(out + ob * kWBlock + 8192 + (m & 31) * 16 + (m >> 5) * 4) = v;
}

}  // namespace gemm
}  // namespace moe
