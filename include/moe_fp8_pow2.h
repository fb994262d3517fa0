/*
 * moe_fp8_pow2.h -- C ABI of the B200 (sm_100a) routed-expert MoE FFN with
 * MXFP4 expert weights and FP8 E4M3 activations scaled by powers of two.
 *
 * Conventions (all entry points)
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *     the argument description says "host".  The library never frees caller
 *     memory and allocates nothing on these calls; scratch memory, where a
 *     call needs it, is passed in as `workspace` and sized by the matching
 *     *_workspace_size() query.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = legacy default stream) and returns an int status:
 *        MOE_OK (0)            launched
 *        MOE_ERR_INVALID (-1)  null pointer, bad shape, misaligned pointer
 *        MOE_ERR_UNSUPPORTED   configuration outside the compiled kernels
 *        MOE_ERR_NAN_SCALE     (device word only) an E8M0 byte 255 was met
 *        MOE_ERR_RANGE         (device word only) a value is not representable
 *        MOE_ERR_LAUNCH (-5)   the CUDA launch failed (cudaGetLastError)
 *        MOE_ERR_TIMEOUT (-6)  (device word only) a bounded device wait expired
 *     Problems that depend on tensor CONTENTS (NaN scales, range) cannot be
 *     seen at launch; kernels record them in a device error word that
 *     moe_get_device_error() returns (first error wins).  Outputs of a call
 *     that recorded a device error are unspecified.
 *   - Row-major layouts throughout; weights are [N, K] with K (the input
 *     dimension) contiguous, the orientation of torch.nn.functional.linear.
 *   - Packed FP4 / INT4: element 2i is the LOW nibble of byte i, 2i+1 the high.
 *   - No exceptions cross this boundary; calls on different streams may run
 *     concurrently when their buffers are disjoint.
 *   - Kernels are launched with programmatic dependent launch: each may be
 *     scheduled while the previous kernel on the stream runs, and waits for
 *     it before touching memory, so stream order is kept.  A caller kernel
 *     that follows on the same stream and is itself launched with
 *     programmatic stream serialization must wait for its predecessor
 *     (cudaGridDependencySynchronize) before reading these outputs.
 *
 * Sources (web pages describing the method; cited by title and section)
 *   [SI]    "DeepSeek-V4-Flash-SI" model card: 架构特性 (Mixture of Experts
 *           paragraph: 256 routed + 1 shared expert, top-6, sqrtsoftplus
 *           scoring, routing scale 1.5, SwiGLU clamp +-10) and 低精度计算
 *           (FP4 E2M1 experts with an F8_E8M0 scale per 32 elements; online
 *           FP8 E4M3 activations, one power-of-2 scale per 128 elements);
 *           模型训练 table (dynamic FP8 E4M3 activations, ue8m0 scale).
 *   [NVFP4] "DeepSeek-V4-Pro-0813-nvfp4-DSpark" walkthrough: 阶段三 and its
 *           MXFP4 vs NVFP4 storage table (same E2M1 nibbles, E4M3 scale per
 *           16, weight bits not recomputed, scale bytes doubled).
 *   [W4A]   "DeepSeek-V4-Flash-0731-W4AFP8-mt" model card: 量化方式 and
 *           权重约定 (FP4 -> signed INT4, group 128, two INT4 per int8,
 *           float32 weight_scale_inv [N, K/128], dynamic E4M3 activations).
 *   [PTPC]  "DeepSeek-V4.1-Flash-Quark-PTPC-FP8" walkthrough: 核心参数 (FP8
 *           E4M3 weights, per-channel static symmetric scales; activations
 *           per-token dynamic symmetric; round half to even).
 *
 * Step labels used below
 *   a1 activation quantisation    a2 routing          a3 grouping (permute)
 *   a4 gate/up GEMM               a5 SwiGLU + requant a6 down GEMM
 *   a7 weighted combine           a8 MXFP4 -> NVFP4   a9 MXFP4 -> INT4 g128
 *   a10 W4AFP8 GEMM               f1 MXFP4 -> FP8 [128, 128] blocks
 *   f2 hash routing               f3 FP8 block-scaled GEMM (shared expert)
 *   f4 PTPC-FP8 expert path
 */
#ifndef MOE_FP8_POW2_H
#define MOE_FP8_POW2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_INVALID (-1)
#define MOE_ERR_UNSUPPORTED (-2)
#define MOE_ERR_NAN_SCALE (-3)
#define MOE_ERR_RANGE (-4)
#define MOE_ERR_LAUNCH (-5)
#define MOE_ERR_TIMEOUT (-6)

/* Grouped-GEMM epilogues. */
#define MOE_EPI_STORE_F32 0    /* out: float32 [rows, N]                                   */
#define MOE_EPI_STORE_BF16 1   /* out: bfloat16 [rows, N]                                  */
#define MOE_EPI_SWIGLU_QUANT 2 /* out: E4M3 h [rows, N/2]; out_scale: E8M0 [rows, N/256] */
#define MOE_EPI_SWIGLU_F32 3   /* out: float32 h [rows, N/2] (PTPC GEMM only)               */

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int moe_version(void);

/*
 * Device error word: waits for `stream`, copies the word to *code (host) and
 * clears it.  Returns MOE_OK, or MOE_ERR_LAUNCH if the copy itself failed.
 */
int moe_get_device_error(int* code, void* stream);

/*
 * Failure-detection self-test (no counterpart on the source pages): launches
 * one thread that waits on a barrier nothing ever arrives at, using the same
 * bounded wait as the GEMM pipelines with a limit of timeout_ns (0 <
 * timeout_ns <= 2 s).  The wait gives up, the kernel records MOE_ERR_TIMEOUT
 * in the device error word and exits; the CUDA context stays usable.
 */
int moe_selftest_wait_timeout(int64_t timeout_ns, void* stream);

/*
 * a1 -- activation quantisation [SI 低精度计算, 模型训练].
 * For each row and each group of 128 columns: amax = max |x|;
 * k = ceil(log2(amax / 448)) with amax / 448 a float32 round-to-nearest-even
 * divide and the ceiling taken exactly; k clamped to [-127, 127]; k = 0 for
 * an all-zero group.  xq = E4M3(x * 2^-k) rounded to nearest even and
 * saturated to +-448; sx = k + 127 (E8M0).
 *   x   bfloat16 [rows, cols], 16-byte aligned; cols % 128 == 0
 *   xq  uint8 E4M3 [rows, cols], 8-byte aligned
 *   sx  uint8 E8M0 [rows, cols / 128]
 * rows == 0 is a no-op.  NaN/Inf inputs are a precondition violation.
 */
int moe_quantize_act_fp8(const void* x, int rows, int cols, uint8_t* xq, uint8_t* sx,
                         void* stream);

/*
 * a2 -- router [SI 架构特性]: idx[t, :] = the k largest logits of row t in
 * descending order, ties to the lower expert index; s_j = sqrt(softplus(z_j));
 * w[t, j] = route_scale * s_j / sum_j s_j   (route_norm != 0)
 *         = route_scale * s_j               (route_norm == 0).
 *   logits float32 [T, E]; 1 <= k <= min(E, 16); E <= 1024
 *   idx    int32 [T, k];  w float32 [T, k]
 * Indices are exact; weights use the device expf/log1pf/sqrtf (within a few
 * float32 ulps of the exact value).
 */
int moe_route_topk(const float* logits, int T, int E, int k, float route_scale,
                   int route_norm, int32_t* idx, float* w, void* stream);

/*
 * f2 -- hash routing of the first layers [SI 架构特性: the first 3 layers
 * choose experts by hash, deterministically from the token ID].  The page
 * gives no hash function; the choice is read as a lookup in a table of k
 * expert ids per vocabulary entry that the caller supplies (a checkpoint
 * carries it): idx[t, j] = tid2eid[token_ids[t], j], in table order.  The
 * weights take the scored layers' rule at those experts:
 * s_j = sqrt(softplus(logits[t, idx[t, j]])),
 * w[t, j] = route_scale * s_j / sum_j s_j   (route_norm != 0)
 *         = route_scale * s_j               (route_norm == 0),
 * the sum taken in slot order in float32 (device expf/log1pf/sqrtf, as
 * moe_route_topk).
 *   token_ids int32 [T];  tid2eid int32 [vocab, k] (expert ids in [0, E));
 *   logits float32 [T, E];  idx int32 [T, k];  w float32 [T, k];
 *   1 <= k <= 16
 * A token id outside [0, vocab) records MOE_ERR_INVALID in the device error
 * word and gives that token idx -1 and weight 0 in every slot; a table entry
 * outside [0, E) does the same for its slot only (moe_permute then gives
 * such a pair no row and moe_combine skips it).
 */
int moe_route_hash(const int32_t* token_ids, int T, const int32_t* tid2eid, int vocab, const float* logits,
                   int E, int k, float route_scale, int route_norm, int32_t* idx, float* w, void* stream);

/*
 * a3 -- grouping by expert.  Groups g = 0..E-1 are the routed experts,
 * group E the shared expert (one row per token when has_shared != 0, none
 * otherwise).  Within a routed group rows are in ascending pair id p = t*k+j;
 * shared rows follow in token order.
 *   idx      int32 [T, k] expert ids in [0, E)   (an out-of-range id: device
 *            error MOE_ERR_INVALID; that pair gets no row and inv = -1)
 *   xq, sx   outputs of moe_quantize_act_fp8 for H columns (H % 128 == 0)
 *   counts   int32 [E+1];  offsets int32 [E+2] (exclusive prefix of counts)
 *   perm     int32 [R], R = T*k + (has_shared ? T : 0): source id of row r,
 *            the pair id p for routed rows, T*k + t for the shared row of t
 *   inv      int32 [T*k]: row of pair p (-1 for a pair with an invalid id)
 *   xq_perm  uint8 [R, H] (16-byte aligned), sx_perm uint8 [R, H/128]:
 *            the rows of xq / sx of each row's source token
 *   workspace  device scratch of moe_permute_workspace_size(T, E, k) bytes,
 *            256-byte aligned; its contents on entry do not matter
 */
size_t moe_permute_workspace_size(int T, int E, int k);
int moe_permute(const int32_t* idx, int T, int E, int k, int has_shared,
                const uint8_t* xq, const uint8_t* sx, int H,
                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                uint8_t* xq_perm, uint8_t* sx_perm,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Grouping without caller scratch.  The source pages have no counterpart to
 * this call; it exists for callers that cannot allocate device memory: a host
 * runtime working from a fixed memory plan that hands the layer only its
 * input and output buffers, or a caller that is not allowed to call
 * cudaMalloc at this point.  Same arguments, outputs and results as
 * moe_permute, minus the workspace: the per-chunk expert counters live in a
 * file-scope device array of moe_permute_noalloc_max_counters() int32
 * (256 KiB), which every GPU that loads this library holds until the process
 * exits.  Requires ceil(T*k / 2048) * E <= that maximum, else it returns
 * MOE_ERR_UNSUPPORTED without launching anything.  It calls no cudaMalloc,
 * cudaFree or allocating library routine.
 *   - The first call on each device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress); make that first call before
 *     any stream capture on the device.  The address is cached with the CUDA
 *     context it was found in; a device reset (cudaDeviceReset) ends that
 *     context and invalidates the address, so the first call after a reset
 *     looks it up again (and should likewise precede any capture).
 *   - All calls share the one array and it keeps the last call's contents;
 *     nothing in it needs to start at zero (each call writes every counter it
 *     reads).  Calls whose executions overlap on the GPU (different streams,
 *     no ordering between them) race on the array and give wrong results.
 */
int64_t moe_permute_noalloc_max_counters(void);
int moe_permute_noalloc(const int32_t* idx, int T, int E, int k, int has_shared,
                        const uint8_t* xq, const uint8_t* sx, int H,
                        int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                        uint8_t* xq_perm, uint8_t* sx_perm, void* stream);

/*
 * Weight preparation (once per weight tensor, at load time): MXFP4 nibbles
 * [n_mats, N, K/2] and E8M0 scales [n_mats, N, K/32] -> blocks of 8704 bytes,
 * one per (128-row block, 128-wide K step): the block's 128 rows x 64 bytes of
 * packed nibbles (the source rows, unchanged), then its 512 scale bytes in the
 * order the block-scaled tensor-core MMA reads from tensor memory (byte
 * (m % 32) * 16 + (m / 32) * 4 + b holds row m's scale of 32-element sub-block
 * b).  Block order:
 *   paired == 0: [n_mats, N/128, K/128]                   (MOE_EPI_STORE_F32 / BF16)
 *   paired != 0: [n_mats, N/256, K/128, 2]: the block of the first half (gate,
 *                w1) and the matching block of the second half (up, w3) side by
 *                side; required by MOE_EPI_SWIGLU_QUANT; N % 256 == 0
 * N % 128 == 0, K % 128 == 0; fp4 16-byte aligned; `prepared` holds
 * moe_prepared_weights_size(n_mats, N, K) bytes (N*K/2 * 17/16 per matrix),
 * 32-byte aligned.  The values are unchanged (a relayout).
 */
size_t moe_prepared_weights_size(int64_t n_mats, int N, int K);
int moe_prepare_weights(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K, int paired,
                        uint8_t* prepared, void* stream);

/*
 * a4 / a5 / a6 -- grouped expert GEMM with MXFP4 weights [SI 低精度计算],
 * tcgen05 block-scaled MMA (kind::mxf8f6f4, E2M1 x E4M3, E8M0 scales) with
 * float32 accumulation.  For every group g and row r in
 * [offsets[g], offsets[g+1]):  acc[r, n] = sum_k a[r, k] * 2^(sa[r, k/128]-127)
 *                                          * w[g, n, k] * 2^(sw[g, n, k/32]-127)
 *   a_e4m3       uint8 [a_rows, K] (16-byte aligned), a_rows >= offsets[G]
 *   a_e8m0_128   uint8 [a_rows, K/128]
 *   offsets      int32 [G+1] device, non-decreasing, offsets[0] >= 0,
 *                offsets[G] <= a_rows (rows outside [offsets[0], offsets[G])
 *                are neither read nor written); otherwise the call does no
 *                work, leaves out untouched and records MOE_ERR_INVALID in the
 *                device error word (moe_get_device_error)
 *   w_prepared   output of moe_prepare_weights for the MXFP4 weights [G, N, K/2]
 *                and scales [G, N, K/32] (paired order for
 *                MOE_EPI_SWIGLU_QUANT, plain otherwise)
 *   N % 128 == 0 (N % 256 == 0 for SWIGLU_QUANT), K % 128 == 0
 *   epilogue  MOE_EPI_STORE_F32 / MOE_EPI_STORE_BF16: out = acc [a_rows, N]
 *             (rows past offsets[G] untouched);
 *             MOE_EPI_SWIGLU_QUANT [SI 架构特性]: columns [0, N/2) are the
 *             gate (w1) and [N/2, N) the up (w3) projection; with I = N/2,
 *             h = silu(clamp(g, +-limit)) * clamp(u, +-limit) in float32,
 *             then the a1 rule per 128 columns of h: out = E4M3 [a_rows, I],
 *             out_scale = E8M0 [a_rows, I/128]
 *   block_n   token rows per tile: 16, 32, 64 or 128 (one CTA per SM, the
 *             weight tile as the MMA's M operand), or 256 (SM pairs: clusters
 *             of two CTAs share one tcgen05.mma.cta_group::2 of 256 tokens x
 *             256 weight rows; needs N % 256 == 0, else MOE_ERR_UNSUPPORTED).
 *             0 = choose from a_rows and G; for SWIGLU_QUANT with at least
 *             192 rows per group on average, when the workspace holds both
 *             plans, each group's whole 256-row tiles run on SM pairs and its
 *             remaining rows on 128-row tiles (two kernel launches, disjoint
 *             output rows).
 *   workspace scratch of moe_gemm_workspace_size(a_rows, G, K, block_n) bytes;
 *             with block_n = 0 this covers the two plans of a split call
 */
size_t moe_gemm_workspace_size(int a_rows, int n_groups, int K, int block_n);

/*
 * One layer's configuration [SI 架构特性: top-k 6, routing scale 1.5, SwiGLU
 * clamp 10, one shared expert].  T tokens, hidden H, expert intermediate I,
 * E routed experts, topk experts per token.
 */
typedef struct {
  int T, H, I, E, topk;
  float route_scale;   /* 1.5 */
  float swiglu_limit;  /* 10.0 */
  int has_shared;      /* 1: the shared expert is group E and sees every token */
  int route_norm;      /* 1: routing weights normalised to sum 1 before the scale */
} MoeConfig;

#define MOE_PATH_MXFP4 0
#define MOE_PATH_W4AFP8 1
#define MOE_PATH_PTPC 2

/*
 * Scratch bytes of one layer step (host call, no CUDA call): one buffer of
 * this size, 256-byte aligned, can serve as the `workspace` of moe_permute
 * and of every grouped GEMM of the step (w1/w3 and w2, any block_n), since
 * they run in order on one stream; for MOE_PATH_W4AFP8 it includes the E4M3
 * weight copy of moe_w4afp8_workspace_size.  path: MOE_PATH_MXFP4, MOE_PATH_W4AFP8 or
 * MOE_PATH_PTPC.  Returns 0 for a NULL or invalid configuration (T < 0,
 * H or I not a positive multiple of 128, E < 1, topk < 1 or > E, unknown
 * path).
 */
size_t moe_workspace_size(const MoeConfig* cfg, int path);
int moe_grouped_gemm_mxfp4(const uint8_t* a_e4m3, const uint8_t* a_e8m0_128, int a_rows,
                           const int32_t* offsets, int n_groups,
                           const uint8_t* w_prepared, int N, int K,
                           int epilogue, float swiglu_limit, int block_n,
                           void* out, uint8_t* out_scale,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * a10 -- grouped expert GEMM with W4AFP8 weights [W4A 量化方式 / 权重约定]:
 * symmetric INT4 weights (two's complement nibbles, element 2i low) with a
 * float32 dequantisation multiplier per (row, 128 columns), times the same
 * FP8 activations as moe_grouped_gemm_mxfp4:
 *   acc[r, n] = sum_g scale_inv[g', n, g] * sum_{k in group g}
 *               a[r, k] * 2^(sa[r, g]-127) * q[g', n, k]        (g' = r's group)
 * Each 128-wide group is one block-scaled MMA whose float32 partial is
 * scaled and summed in registers, groups in ascending order.  Token tiles of
 * at most 32 rows run the MMA on the offset codes q + 8 (exact E4M3 values
 * of (q + 8) * 2^-9, with weight scale slots 2^9) and subtract 8 x the row's
 * scaled activation sum over the group (computed once per call into the
 * workspace) from each partial: an exact identity, whose float32 rounding is
 * relative to sum |a| * 2^(sa-127) * (q + 8) per group rather than
 * sum |a * q|.  Wider tiles transcode q exactly to E4M3 (unit weight scale
 * slots).
 *   w_int4       int8 [G, N, K/2] (16-byte aligned); w_scale_inv float32 [G, N, K/128]
 *   other arguments, layouts and epilogues as moe_grouped_gemm_mxfp4;
 *   block_n: 16, 32, 64 or 96 (SWIGLU_QUANT; 96 needs the E4M3-copy workspace
 *   below, and with block_n = 0 is chosen instead of 64 when the workspace
 *   holds it) or up to 128 (STORE_F32 / STORE_BF16);  the FP8 block-scaled GEMM
 *   below takes 96 with SWIGLU_QUANT without a copy, chosen with block_n = 0
 *   when the workspace holds the plan of 96-row tiles;
 *   workspace: at least moe_gemm_workspace_size(a_rows, G, K, block_n) bytes.
 *   Token tiles of 64 rows or more, given the larger workspace that
 *   moe_w4afp8_workspace_size(a_rows, G, N, K, block_n) returns: the call
 *   first writes an E4M3 copy of the INT4 weights of every group that has
 *   rows (G * N * K bytes, after the plan) and the GEMM streams that copy,
 *   instead of transcoding each weight tile in shared memory once per token
 *   tile.  The arithmetic is the same (exact E4M3 codes of q, unit weight
 *   scale slots, the same promotion), so both give the same result.
 */
size_t moe_w4afp8_workspace_size(int a_rows, int n_groups, int N, int K, int block_n);
int moe_grouped_gemm_w4afp8(const uint8_t* a_e4m3, const uint8_t* a_e8m0_128, int a_rows,
                            const int32_t* offsets, int n_groups,
                            const int8_t* w_int4, const float* w_scale_inv, int N, int K,
                            int epilogue, float swiglu_limit, int block_n,
                            void* out, uint8_t* out_scale,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * f3 -- grouped GEMM with FP8 E4M3 weights and a float32 scale_inv per
 * [128, 128] block (the FP8 shared expert [NVFP4 只量化专家: shared experts
 * stay FP8; SI 模型训练: weight block size [128, 128]]).  For every group g:
 * acc[r, n] = sum over 128-wide K steps kt of scale_inv[g, n/128, kt] *
 * (sum_{k in kt} a[r, k] * 2^(sa[r, kt]-127) * w[g, n, k]); each step is one
 * block-scaled MMA with unit weight scales whose float32 partial is scaled
 * and summed in ascending kt.
 *   w_e4m3       uint8 [G, N, K] (16-byte aligned); w_scale_inv float32
 *                [G, N/128, K/128]
 *   other arguments, layouts and epilogues as moe_grouped_gemm_w4afp8.
 */
int moe_grouped_gemm_fp8_block128(const uint8_t* a_e4m3, const uint8_t* a_e8m0_128, int a_rows,
                                  const int32_t* offsets, int n_groups, const uint8_t* w_e4m3,
                                  const float* w_scale_inv, int N, int K, int epilogue, float swiglu_limit,
                                  int block_n, void* out, uint8_t* out_scale, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * f4 -- PTPC-FP8 per-token activation quantisation [PTPC 核心参数: activations
 * per-token, dynamic, symmetric, half_even].  Per row: amax = max |x|;
 * scale = amax / 448 (float32 IEEE divide; 1.0 when amax == 0);
 * q = E4M3(x / scale) with a float32 IEEE divide, nearest even, saturating
 * at +-448.  x holding NaN or inf gives unspecified codes for that row.
 *   x      bfloat16 (x_is_f32 == 0) or float32 [rows, cols], 16-byte aligned
 *   q      uint8 E4M3 [rows, cols] (8-byte aligned);  scale float32 [rows]
 *   cols % 8 == 0
 */
int moe_quantize_fp8_per_token(const void* x, int x_is_f32, int rows, int cols, uint8_t* q, float* scale,
                               void* stream);

/*
 * f4 -- per-row scales of the grouped rows: dst[r] = src[perm[r] / k] for a
 * routed row (perm[r] < T*k), src[perm[r] - T*k] for a shared-expert row,
 * for r < offsets[E+1]; rows past it are untouched.  perm and offsets are the
 * outputs of moe_permute; a perm entry outside [0, T*(k+1)) writes 0 and
 * records MOE_ERR_INVALID.
 *   perm int32 [T*(k+1)];  offsets int32 [E+2];  src float32 [T];
 *   dst float32 [T*(k+1)]
 */
int moe_gather_row_scales(const int32_t* perm, int T, int k, const int32_t* offsets, int E, const float* src,
                          float* dst, void* stream);

/*
 * f4 -- grouped GEMM in PTPC-FP8 [PTPC 核心参数]: E4M3 weights with one
 * float32 scale per output channel, E4M3 activations with one float32 scale
 * per row.  For every group g and row r in [offsets[g], offsets[g+1]):
 *   acc[r, n] = (sum_k a[r, k] * w[g, n, k]) * a_scale[r] * w_scale[g, n]
 * (the sum over all of K accumulated by the tensor cores in float32; then
 * two float32 multiplies, a_scale first).
 *   a_e4m3 uint8 [a_rows, K] (16-byte aligned);  a_scale float32 [a_rows]
 *   w_e4m3 uint8 [G, N, K] (16-byte aligned);  w_scale float32 [G, N]
 *   offsets as moe_grouped_gemm_mxfp4;  N % 128 == 0, K % 128 == 0
 *   epilogue MOE_EPI_STORE_F32 / MOE_EPI_STORE_BF16: out = acc [a_rows, N];
 *            MOE_EPI_SWIGLU_F32 (N % 256 == 0): columns [0, N/2) gate,
 *            [N/2, N) up; out = float32 h [a_rows, N/2],
 *            h = silu(clamp(g, +-limit)) * clamp(u, +-limit)
 *   block_n token rows per tile: 16, 32, 64 or 128 (0 = choose)
 *   workspace moe_gemm_workspace_size(a_rows, G, K, block_n) bytes
 */
int moe_grouped_gemm_fp8_ptpc(const uint8_t* a_e4m3, const float* a_scale, int a_rows, const int32_t* offsets,
                              int n_groups, const uint8_t* w_e4m3, const float* w_scale, int N, int K, int epilogue,
                              float swiglu_limit, int block_n, void* out, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * a5 standalone -- SwiGLU with clamp and per-128 power-of-two requantisation
 * [SI 架构特性 / 低精度计算], same arithmetic as MOE_EPI_SWIGLU_QUANT.
 *   gu  float32 [rows, 2I] (gate | up), 16-byte aligned; I % 128 == 0
 *   hq  uint8 E4M3 [rows, I];  sh uint8 E8M0 [rows, I/128]
 */
int moe_swiglu_clamp(const float* gu, int rows, int I, float limit, uint8_t* hq, uint8_t* sh,
                     void* stream);

/*
 * a7 -- combine [SI 架构特性]:
 *   y[t] = sum_{j<k} w[t, j] * o[inv[t*k+j]] + (has_shared ? o[offsets[E] + t] : 0)
 * accumulated in float32 in slot order, rounded once to bfloat16 (nearest even).
 *   o  float32 [R, H] (16-byte aligned), H % 4 == 0;  inv int32 [T*k]
 *      (a negative entry, a pair the grouping rejected, contributes nothing);
 *   w  float32 [T, k];  offsets int32 [E+2] (device);  y bfloat16 [T, H]
 */
int moe_combine(const float* o, const int32_t* inv, const float* w, int T, int k, int H,
                int has_shared, const int32_t* offsets, int E, void* y, void* stream);

/*
 * a8 -- MXFP4 -> NVFP4 [NVFP4 阶段三].  For each of n_mats matrices [N, K]:
 * nibbles are copied unchanged (out_fp4 may equal fp4: then nothing is
 * written there); every E8M0 scale 2^e (per 32) becomes two E4M3 scales
 * 2^(e - G) (per 16), with G = 0 when all exponents of the matrix lie in
 * [-9, 8], else G = max_e - 8 when max_e - min_e <= 17; out_global[m] = 2^G.
 * Device errors: MOE_ERR_NAN_SCALE (byte 255), MOE_ERR_RANGE (span > 17).
 *   fp4, out_fp4  uint8 [n_mats, N, K/2] (16-byte aligned);
 *   e8m0 [n_mats, N, K/32];  out_e4m3 [n_mats, N, K/16];  out_global float32 [n_mats]
 *   K % 32 == 0
 */
int repack_mxfp4_to_nvfp4(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K,
                          uint8_t* out_fp4, uint8_t* out_e4m3, float* out_global, void* stream);

/*
 * a9 -- MXFP4 -> symmetric INT4, group 128 [W4A 量化方式 / 权重约定].  Per row
 * and group of 128: x = exact float32 dequantisation; amax; scale_inv =
 * amax / 7 (float32 IEEE divide; 1.0 when amax == 0);
 * q = clamp(rint(x / scale_inv), -7, 7) (IEEE divide, ties to even);
 * two's complement nibbles, element 2i low.
 * Device errors: MOE_ERR_NAN_SCALE, MOE_ERR_RANGE (x overflows float32).
 *   fp4 uint8 [n_mats, N, K/2] (16-byte aligned); e8m0 [n_mats, N, K/32];
 *   out_int4 int8 [n_mats, N, K/2]; out_scale_inv float32 [n_mats, N, K/128];
 *   K % 128 == 0
 */
int repack_mxfp4_to_int4g128(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N,
                             int K, int8_t* out_int4, float* out_scale_inv, void* stream);

/*
 * f1 -- MXFP4 -> FP8 E4M3 with a [128, 128] block scale [NVFP4 关于 MXFP4 的无损
 * 种子: cast_e2m1fn_to_e4m3fn rewrites the scale per 128 block; SI 模型训练:
 * weight block size [128, 128]].  Per (128-row, 128-column) block of each
 * matrix: amax = exact block maximum; s = ceil(log2(amax / 448)) clamped to
 * [-127, 127] (0 when amax == 0), the a1 rule; out_scale_inv = 2^s (the
 * dequant multiplier: w = e4m3 * scale_inv); out = E4M3(w / 2^s), nearest
 * even, sign kept.  Exact unless a nonzero element falls below E4M3's 2^-9
 * (exponents spread by more than 14 inside a block); then the rounded codes
 * are written and MOE_ERR_RANGE is recorded.  A block with an E8M0 NaN
 * (byte 255) records MOE_ERR_NAN_SCALE and is not written.
 *   fp4 uint8 [n_mats, N, K/2] (16-byte aligned); e8m0 [n_mats, N, K/32]
 *   (4-byte aligned); out_e4m3 uint8 [n_mats, N, K] (16-byte aligned);
 *   out_scale_inv float32 [n_mats, N/128, K/128];  N % 128 == 0, K % 128 == 0
 */
int repack_mxfp4_to_fp8_block128(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K,
                                 uint8_t* out_e4m3, float* out_scale_inv, void* stream);

/*
 * f4 -- MXFP4 -> PTPC-FP8 weights [PTPC 核心参数: weights FP8 E4M3,
 * per-channel, static, symmetric, half_even].  Per output channel (row of
 * K elements): w = exact float32 dequantisation; amax; scale = amax / 448
 * (float32 IEEE divide; 1.0 when amax == 0); out = E4M3(w / scale), float32
 * IEEE divide, nearest even (|w / scale| <= 448 by construction).
 * Device errors: MOE_ERR_NAN_SCALE (row not written), MOE_ERR_RANGE (w
 * overflows float32; row not written).
 *   fp4 uint8 [n_mats, N, K/2] (4-byte aligned); e8m0 [n_mats, N, K/32];
 *   out_e4m3 uint8 [n_mats, N, K] (8-byte aligned); out_scale float32
 *   [n_mats, N];  K % 32 == 0
 */
int repack_mxfp4_to_fp8_per_channel(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K,
                                    uint8_t* out_e4m3, float* out_scale, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_FP8_POW2_H */
