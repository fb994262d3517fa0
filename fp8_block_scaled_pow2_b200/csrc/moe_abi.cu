// C-ABI entry points of libmoe: argument validation, tensor-map creation and
// kernel launches.  All kernels are compiled in this one translation unit so
// they share the device error word.
#include <cudaTypedefs.h>

#include <climits>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "elementwise.cuh"
#include "gemm_mxfp4.cuh"
#include "gemm_pair.cuh"
#include "gemm_w4afp8.cuh"
#include "gemm_ptpc.cuh"
#include "repack.cuh"

using namespace moe;

namespace {

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_LAUNCH;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tiled map, inner dimension first.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// Tiled map of any rank (inner dimension first); strides[i] is the byte
// stride of dimension i + 1.
bool make_map_nd(CUtensorMap* map, CUtensorMapDataType dt, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  return fn(map, dt, (cuuint32_t)rank, const_cast<void*>(base), d, st, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// Every kernel is launched with programmatic stream serialization: it may be
// scheduled while the previous kernel on the stream is still running, and
// waits for it (pdl_wait) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int pick_block_n(int a_rows, int G) {
  const double avg = (double)a_rows / (G > 0 ? G : 1);
  if (avg <= 12) return 16;
  if (avg <= 28) return 32;
  if (avg <= 56) return 64;
  return 128;
}

template <int BN, bool PAIR, int EPI>
int launch_gemm(const CUtensorMap& ta, const gemm::TokenMaps& tb, const CUtensorMap& ts, const gemm::GemmArgs& a,
                cudaStream_t st) {
  using C = gemm::Cfg<BN, PAIR>;
  auto k = gemm::gemm_mxfp4_kernel<BN, PAIR, EPI>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) != cudaSuccess)
    return MOE_ERR_LAUNCH;
  launch(k, dim3(sm_count()), dim3(gemm::kThreads), C::SMEM_ALLOC, st, ta, tb, ts, a);
  return launch_status();
}

template <bool PAIR, int EPI>
int launch_gemm_bn(int bn, const CUtensorMap& ta, const gemm::TokenMaps& tb, const CUtensorMap& ts,
                   const gemm::GemmArgs& a, cudaStream_t st) {
  switch (bn) {
    case 16: return launch_gemm<16, PAIR, EPI>(ta, tb, ts, a, st);
    case 32: return launch_gemm<32, PAIR, EPI>(ta, tb, ts, a, st);
    case 64: return launch_gemm<64, PAIR, EPI>(ta, tb, ts, a, st);
    case 128: return launch_gemm<128, PAIR, EPI>(ta, tb, ts, a, st);
    default: return MOE_ERR_UNSUPPORTED;
  }
}

// The pair kernel runs as clusters of two CTAs (one per SM); the grid is the
// number of clusters that can be resident at once, so every cluster of the
// persistent kernel starts immediately.
template <int EPI>
int launch_pair(const CUtensorMap& tw, const pair::PairMaps& tt, const CUtensorMap& ts, const pair::PairArgs& a,
                cudaStream_t st) {
  auto k = pair::gemm_pair_kernel<EPI>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, pair::Cfg::SMEM_ALLOC) != cudaSuccess)
    return MOE_ERR_LAUNCH;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count() / 2));
  cfg.blockDim = dim3(pair::kThreads);
  cfg.dynamicSmemBytes = pair::Cfg::SMEM_ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  static int cached_dev = -1, cached_clusters = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_LAUNCH;
  if (dev != cached_dev) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(k), &cfg) != cudaSuccess || n <= 0)
      return MOE_ERR_LAUNCH;
    cached_clusters = n;
    cached_dev = dev;
  }
  cfg.gridDim = dim3(2 * cached_clusters);
  if (cudaLaunchKernelEx(&cfg, k, tw, tt, ts, a) != cudaSuccess) return MOE_ERR_LAUNCH;
  return launch_status();
}

template <int BN, bool DUAL, int EPI, bool W8, bool ROWS = false>
int launch_w4a(const CUtensorMap& ta, const CUtensorMap& tb, const w4a::W4Args& a, cudaStream_t st) {
  using C = w4a::Cfg<BN, DUAL, W8>;
  auto k = w4a::gemm_w4afp8_kernel<BN, DUAL, EPI, W8, ROWS>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) != cudaSuccess)
    return MOE_ERR_LAUNCH;
  launch(k, dim3(sm_count()), dim3(C::THREADS), C::SMEM_ALLOC, st, ta, tb, a);
  return launch_status();
}

// Bytes of the E4M3 copy of INT4 weights [G, N, K/2] that the W4AFP8 GEMM
// writes into its workspace (after the plan) for token tiles of 64 rows or
// more.
size_t w4a_scratch_bytes(int G, int N, int K) { return gemm::align256((size_t)G * N * K); }

bool w4a_uses_scratch(int block_n) { return block_n >= 64; }

// Grouped GEMM whose weight scale is applied by promotion warps: INT4 group-128
// weights (W8 = false) or FP8 E4M3 weights with [128, 128] block scales (W8 =
// true).  INT4 on token tiles of 64 rows or more, when the workspace holds
// w4a_scratch_bytes after the plan: transcoded once per call to an E4M3 copy
// in the workspace, then streamed like FP8 weights with per-row scales;
// otherwise transcoded to E4M3 in shared memory, once per weight tile and
// token tile.
template <bool W8>
int promoted_gemm(const uint8_t* a_e4m3, const uint8_t* a_e8m0_128, int a_rows, const int32_t* offsets, int n_groups,
                  const void* w, const float* w_scale_inv, int N, int K, int epilogue, float swiglu_limit, int block_n,
                  void* out, uint8_t* out_scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (a_rows < 0 || n_groups < 1 || n_groups > 1024 || N <= 0 || K <= 0 || N % 128 || K % 128)
    return MOE_ERR_INVALID;
  if (epilogue < MOE_EPI_STORE_F32 || epilogue > MOE_EPI_SWIGLU_QUANT) return MOE_ERR_INVALID;
  const bool dual = epilogue == MOE_EPI_SWIGLU_QUANT;
  if (dual && N % 256) return MOE_ERR_INVALID;
  const bool auto_bn = block_n == 0;
  if (block_n == 0) block_n = std::min(pick_block_n(a_rows, n_groups), dual ? 64 : 128);
  // with gate and up an automatic choice takes 96-row tiles (eight promotion
  // warps) when the workspace holds their plan (and, for INT4, the E4M3 copy)
  if (dual && auto_bn && block_n == 64 &&
      workspace_bytes >= gemm::ws_layout(a_rows, n_groups, K, 96).total + (W8 ? 0 : w4a_scratch_bytes(n_groups, N, K)))
    block_n = 96;
  if (block_n != 16 && block_n != 32 && block_n != 64 && !(block_n == 128 && !dual) && !(block_n == 96 && dual))
    return MOE_ERR_UNSUPPORTED;
  if (a_rows == 0) return MOE_OK;
  if (!a_e4m3 || !a_e8m0_128 || !offsets || !w || !w_scale_inv || !out || !workspace) return MOE_ERR_INVALID;
  if (dual && !out_scale) return MOE_ERR_INVALID;
  if (!aligned(a_e4m3, 16) || !aligned(w, 16) || !aligned(w_scale_inv, 4) || !aligned(workspace, 256))
    return MOE_ERR_INVALID;
  const gemm::WsLayout L = gemm::ws_layout(a_rows, n_groups, K, block_n);
  if (workspace_bytes < L.total) return MOE_ERR_INVALID;
  const bool scratch = !W8 && w4a_uses_scratch(block_n) &&
                       workspace_bytes >= L.total + w4a_scratch_bytes(n_groups, N, K);
  if (!W8 && block_n == 96 && !scratch) return MOE_ERR_INVALID;     // INT4 96-row tiles stream the E4M3 copy
  uint8_t* e4m3_copy = scratch ? reinterpret_cast<uint8_t*>(workspace) + L.total : nullptr;
  CUtensorMap ta, tb;
  // INT4: raw [rows, K/2] tiles of 64 x 128 bytes; FP8 (and the E4M3 copy of
  // INT4): [rows, K] tiles of 128 x 128 bytes written straight into the
  // 128-byte-swizzled MMA layout
  if ((W8 || scratch) ? !make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, scratch ? e4m3_copy : w, (uint64_t)K,
                                  (uint64_t)n_groups * N, (uint64_t)K, 128, 128)
                      : !make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (uint64_t)K / 2, (uint64_t)n_groups * N,
                                  (uint64_t)K / 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return MOE_ERR_LAUNCH;
  if (!make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_e4m3, (uint64_t)K, (uint64_t)a_rows, (uint64_t)K, 128,
                (uint32_t)block_n))
    return MOE_ERR_LAUNCH;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  w4a::W4Args args;
  args.w_sinv = w_scale_inv;
  args.a_sf = ws + L.a_sf;
  args.header = reinterpret_cast<const int*>(ws + L.header);
  args.prefix = reinterpret_cast<const int*>(ws + L.prefix);
  args.tstart = reinterpret_cast<const int*>(ws + L.tstart);
  args.groups = reinterpret_cast<const int2*>(ws + L.groups);
  args.G = n_groups;
  args.N = N;
  args.K = K;
  args.out = out;
  args.out_scale = out_scale;
  args.limit = swiglu_limit;
  // INT4 weights on narrow token tiles: per (row, K step) activation sums for
  // the +8 weight offset
  float* a_corr = (!W8 && w4a::offset_codes(block_n)) ? reinterpret_cast<float*>(ws + L.a_corr) : nullptr;
  args.a_corr = a_corr;
  // the L2 prefetcher on decode-sized token tiles (0.5415 -> 0.5337 ms for
  // the 64-token w1/w3 GEMM; wider tiles are not latency bound)
  args.pf_steps = block_n <= 32 ? 4 : 0;
  cudaStream_t st = S(stream);
  const int n_ft = dual ? N / 256 : N / 128;
  launch(gemm::gemm_prep_kernel, dim3(L.max_tiles), dim3(gemm::kPrepThreads), 0, st, 
      offsets, n_groups, (int)a_rows, block_n, n_ft, a_e8m0_128, K / 128, reinterpret_cast<int*>(ws + L.header),
      reinterpret_cast<int*>(ws + L.prefix), reinterpret_cast<int*>(ws + L.tstart),
      reinterpret_cast<int2*>(ws + L.groups), ws + L.a_sf, a_e4m3, a_corr, 0, 0);
  if (launch_status() != MOE_OK) return MOE_ERR_LAUNCH;
  if (scratch) {
    const int64_t chunks = (int64_t)N * K / 32;     // 16 input bytes (32 INT4) per thread
    launch(w4a::transcode_int4_kernel, dim3((unsigned)((chunks + 255) / 256), (unsigned)n_groups), dim3(256), 0, st,
           reinterpret_cast<const uint4*>(w), offsets, chunks, reinterpret_cast<uint4*>(e4m3_copy));
    if (launch_status() != MOE_OK) return MOE_ERR_LAUNCH;
    if (dual)
      return block_n == 96 ? launch_w4a<96, true, MOE_EPI_SWIGLU_QUANT, true, true>(ta, tb, args, st)
                           : launch_w4a<64, true, MOE_EPI_SWIGLU_QUANT, true, true>(ta, tb, args, st);
    if (epilogue == MOE_EPI_STORE_F32)
      return block_n == 64 ? launch_w4a<64, false, MOE_EPI_STORE_F32, true, true>(ta, tb, args, st)
                           : launch_w4a<128, false, MOE_EPI_STORE_F32, true, true>(ta, tb, args, st);
    return block_n == 64 ? launch_w4a<64, false, MOE_EPI_STORE_BF16, true, true>(ta, tb, args, st)
                         : launch_w4a<128, false, MOE_EPI_STORE_BF16, true, true>(ta, tb, args, st);
  }
  if (dual) {
    switch (block_n) {
      case 16: return launch_w4a<16, true, MOE_EPI_SWIGLU_QUANT, W8>(ta, tb, args, st);
      case 32: return launch_w4a<32, true, MOE_EPI_SWIGLU_QUANT, W8>(ta, tb, args, st);
      case 96:
        if constexpr (W8) return launch_w4a<96, true, MOE_EPI_SWIGLU_QUANT, true>(ta, tb, args, st);
        return MOE_ERR_UNSUPPORTED;
      default: return launch_w4a<64, true, MOE_EPI_SWIGLU_QUANT, W8>(ta, tb, args, st);
    }
  }
  if (epilogue == MOE_EPI_STORE_F32) {
    switch (block_n) {
      case 16: return launch_w4a<16, false, MOE_EPI_STORE_F32, W8>(ta, tb, args, st);
      case 32: return launch_w4a<32, false, MOE_EPI_STORE_F32, W8>(ta, tb, args, st);
      case 64: return launch_w4a<64, false, MOE_EPI_STORE_F32, W8>(ta, tb, args, st);
      default: return launch_w4a<128, false, MOE_EPI_STORE_F32, W8>(ta, tb, args, st);
    }
  }
  switch (block_n) {
    case 16: return launch_w4a<16, false, MOE_EPI_STORE_BF16, W8>(ta, tb, args, st);
    case 32: return launch_w4a<32, false, MOE_EPI_STORE_BF16, W8>(ta, tb, args, st);
    case 64: return launch_w4a<64, false, MOE_EPI_STORE_BF16, W8>(ta, tb, args, st);
    default: return launch_w4a<128, false, MOE_EPI_STORE_BF16, W8>(ta, tb, args, st);
  }
}

template <int BN, bool DUAL, int EPI>
int launch_ptpc(const CUtensorMap& ta, const CUtensorMap& tb, const ptpc::Args& a, cudaStream_t st) {
  using C = ptpc::Cfg<BN, DUAL>;
  auto k = ptpc::gemm_ptpc_kernel<BN, DUAL, EPI>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) != cudaSuccess)
    return MOE_ERR_LAUNCH;
  launch(k, dim3(sm_count()), dim3(ptpc::kThreads), C::SMEM_ALLOC, st, ta, tb, a);
  return launch_status();
}

template <bool DUAL, int EPI>
int launch_ptpc_bn(int block_n, const CUtensorMap& ta, const CUtensorMap& tb, const ptpc::Args& a, cudaStream_t st) {
  switch (block_n) {
    case 16: return launch_ptpc<16, DUAL, EPI>(ta, tb, a, st);
    case 32: return launch_ptpc<32, DUAL, EPI>(ta, tb, a, st);
    case 64: return launch_ptpc<64, DUAL, EPI>(ta, tb, a, st);
    default: return launch_ptpc<128, DUAL, EPI>(ta, tb, a, st);
  }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that no
// one arrives at; the wait gives up after timeout_ns and records
// MOE_ERR_TIMEOUT in the device error word.
__global__ void wait_timeout_selftest_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  sm100::mbar_init(&bar, 1);
  abort_flag = 0;
  sm100::fence_mbar_init();
  __syncwarp();
  volatile int* ab = &abort_flag;
  if (sm100::mbar_wait(&bar, 0, ab, timeout_ns)) record_error(MOE_ERR_INVALID);   // cannot complete
}

}  // namespace

extern "C" {

int moe_selftest_wait_timeout(int64_t timeout_ns, void* stream) {
  if (timeout_ns <= 0 || timeout_ns > 2000000000LL) return MOE_ERR_INVALID;
  wait_timeout_selftest_kernel<<<1, 1, 0, S(stream)>>>((uint64_t)timeout_ns);
  return launch_status();
}

const char* moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_NAN_SCALE: return "E8M0 NaN scale (byte 255)";
    case MOE_ERR_RANGE: return "value not representable in the target format";
    case MOE_ERR_LAUNCH: return "CUDA launch or copy failed";
    case MOE_ERR_TIMEOUT: return "bounded device wait expired";
    default: return "unknown status";
  }
}

int moe_version(void) { return 200; }

int moe_get_device_error(int* code, void* stream) {
  if (!code) return MOE_ERR_INVALID;
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, S(stream)) !=
      cudaSuccess)
    return MOE_ERR_LAUNCH;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return MOE_ERR_LAUNCH;
  const int zero = 0;
  if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, S(stream)) !=
      cudaSuccess)
    return MOE_ERR_LAUNCH;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return MOE_ERR_LAUNCH;
  *code = v;
  return MOE_OK;
}

int moe_quantize_act_fp8(const void* x, int rows, int cols, uint8_t* xq, uint8_t* sx, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 128) return MOE_ERR_INVALID;
  if (rows == 0) return MOE_OK;
  if (!x || !xq || !sx || !aligned(x, 16) || !aligned(xq, 8)) return MOE_ERR_INVALID;
  const int64_t n_groups = (int64_t)rows * (cols / 128);
  launch(quant_act_kernel, dim3((unsigned)((n_groups + kQuantGroupsPerBlock - 1) / kQuantGroupsPerBlock)), dim3(256),
         0, S(stream), reinterpret_cast<const uint4*>(x), n_groups, reinterpret_cast<uint2*>(xq), sx);
  return launch_status();
}

int moe_route_topk(const float* logits, int T, int E, int k, float route_scale, int route_norm, int32_t* idx,
                   float* w, void* stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > 16 || k > E) return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (!logits || !idx || !w) return MOE_ERR_INVALID;
  const int V = (E + 31) / 32;
  const dim3 grid((T + 7) / 8);
  cudaStream_t st = S(stream);
  if (V <= 1) launch(route_topk_kernel<1>, dim3(grid), dim3(256), 0, st, logits, T, E, k, route_scale, route_norm, idx, w);
  else if (V <= 2) launch(route_topk_kernel<2>, dim3(grid), dim3(256), 0, st, logits, T, E, k, route_scale, route_norm, idx, w);
  else if (V <= 4) launch(route_topk_kernel<4>, dim3(grid), dim3(256), 0, st, logits, T, E, k, route_scale, route_norm, idx, w);
  else if (V <= 8) launch(route_topk_kernel<8>, dim3(grid), dim3(256), 0, st, logits, T, E, k, route_scale, route_norm, idx, w);
  else if (V <= 16) launch(route_topk_kernel<16>, dim3(grid), dim3(256), 0, st, logits, T, E, k, route_scale, route_norm, idx, w);
  else launch(route_topk_kernel<32>, dim3(grid), dim3(256), 0, st, logits, T, E, k, route_scale, route_norm, idx, w);
  return launch_status();
}

int moe_route_hash(const int32_t* token_ids, int T, const int32_t* tid2eid, int vocab, const float* logits, int E,
                   int k, float route_scale, int route_norm, int32_t* idx, float* w, void* stream) {
  if (T < 0 || vocab < 1 || E < 1 || k < 1 || k > 16) return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (!token_ids || !tid2eid || !logits || !idx || !w) return MOE_ERR_INVALID;
  launch(route_hash_kernel, dim3((T + 255) / 256), dim3(256), 0, S(stream), token_ids, T, tid2eid, vocab, logits, E,
         k, route_scale, route_norm, idx, w);
  return launch_status();
}

// The a3 passes on one stream (arguments already validated).  hist: per-chunk
// expert counters, unused when all pairs fit in one chunk.
static void launch_permute(const int32_t* idx, int T, int E, int k, int has_shared, const uint8_t* xq,
                           const uint8_t* sx, int H, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                           uint8_t* xq_perm, uint8_t* sx_perm, int32_t* hist, cudaStream_t st) {
  const int P = T * k;
  const int n_chunks = (P + kChunk - 1) / kChunk;
  if (n_chunks <= 1) {
    launch(permute_small_kernel, dim3(1), dim3(1024), 0, st, idx, P, E, T, has_shared ? 1 : 0, counts, offsets, perm, inv);
  } else {
    launch(permute_count_kernel, dim3(n_chunks), dim3(256), 0, st, idx, P, E, hist);
    launch(permute_scan_kernel, dim3(1), dim3(1024), 0, st, hist, n_chunks, E, T, has_shared ? 1 : 0, counts, offsets);
    launch(permute_scatter_kernel, dim3(n_chunks), dim3(256), 0, st, idx, P, E, hist, offsets, perm, inv);
  }
  const int64_t R = (int64_t)P + (has_shared ? T : 0);
  if (R > 0)
    launch(permute_gather_kernel, dim3((unsigned)((R + 7) / 8)), dim3(256), 0, st, 
        reinterpret_cast<const uint4*>(xq), sx, H, T, k, offsets, E, perm, reinterpret_cast<uint4*>(xq_perm),
        sx_perm);
}

size_t moe_permute_workspace_size(int T, int E, int k) {
  if (T <= 0 || E <= 0 || k <= 0) return 256;
  const int64_t P = (int64_t)T * k;
  const int64_t chunks = (P + kChunk - 1) / kChunk;
  return (size_t)((chunks * E * 4 + 255) / 256 * 256);
}

int moe_permute(const int32_t* idx, int T, int E, int k, int has_shared, const uint8_t* xq, const uint8_t* sx,
                int H, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv, uint8_t* xq_perm,
                uint8_t* sx_perm, void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 0 || E < 1 || E > 1023 || k < 1 || H <= 0 || H % 128) return MOE_ERR_INVALID;
  if (!counts || !offsets) return MOE_ERR_INVALID;
  if ((int64_t)T * k > (int64_t)1 << 30) return MOE_ERR_UNSUPPORTED;
  cudaStream_t st = S(stream);
  if (T > 0) {
    if (!idx || !xq || !sx || !perm || !inv || !xq_perm || !sx_perm || !workspace) return MOE_ERR_INVALID;
    if (!aligned(xq, 16) || !aligned(xq_perm, 16) || !aligned(workspace, 16)) return MOE_ERR_INVALID;
    if (workspace_bytes < moe_permute_workspace_size(T, E, k)) return MOE_ERR_INVALID;
  }
  int32_t* hist = reinterpret_cast<int32_t*>(workspace);
  launch_permute(idx, T, E, k, has_shared, xq, sx, H, counts, offsets, perm, inv, xq_perm, sx_perm, hist, st);
  return launch_status();
}

size_t moe_prepared_weights_size(int64_t n_mats, int N, int K) {
  if (n_mats < 0 || N <= 0 || K <= 0 || N % 128 || K % 128) return 0;
  return (size_t)n_mats * (N / 128) * (K / 128) * gemm::kWBlock;
}

int moe_prepare_weights(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K, int paired,
                        uint8_t* prepared, void* stream) {
  if (n_mats < 0 || N <= 0 || K <= 0 || N % 128 || K % 128 || (paired && N % 256)) return MOE_ERR_INVALID;
  if (n_mats == 0) return MOE_OK;
  if (!fp4 || !e8m0 || !prepared || !aligned(fp4, 16) || !aligned(e8m0, 4) || !aligned(prepared, 16))
    return MOE_ERR_INVALID;
  const int64_t blocks = n_mats * (N / 128) * (K / 128);
  if (blocks > 0x7FFFFFFFLL) return MOE_ERR_UNSUPPORTED;
  launch(gemm::prepare_weights_kernel, dim3((unsigned)blocks), dim3(128), 0, S(stream), fp4, e8m0, N, K, paired ? 1 : 0, prepared);
  return launch_status();
}

// Workspace of an automatic MXFP4 call that splits its groups between the
// 128-row swap-AB kernel and the SM-pair kernel: both plans, one after the other.
size_t split_workspace_size(int a_rows, int n_groups, int K) {
  return gemm::align256(gemm::ws_layout(a_rows, n_groups, K, 128).total) +
         gemm::ws_layout(a_rows, n_groups, K, pair::BN).total;
}

size_t moe_gemm_workspace_size(int a_rows, int n_groups, int K, int block_n) {
  if (a_rows < 0 || n_groups <= 0 || K <= 0) return 0;
  if (block_n == 0) {
    block_n = pick_block_n(a_rows, n_groups);
    if (block_n == 128) return split_workspace_size(a_rows, n_groups, K);
  }
  return gemm::ws_layout(a_rows, n_groups, K, block_n).total;
}

size_t moe_w4afp8_workspace_size(int a_rows, int n_groups, int N, int K, int block_n) {
  if (a_rows < 0 || n_groups <= 0 || N <= 0 || K <= 0) return 0;
  size_t plan = 0;
  if (block_n == 0) {
    // the call caps its own choice at 64 rows for the SwiGLU epilogue: cover
    // the plan of every tile width it may pick
    for (int bn : {16, 32, 64, 96, 128}) plan = std::max(plan, gemm::ws_layout(a_rows, n_groups, K, bn).total);
    block_n = pick_block_n(a_rows, n_groups);
  } else {
    plan = gemm::ws_layout(a_rows, n_groups, K, block_n).total;
  }
  return plan + (w4a_uses_scratch(block_n) ? w4a_scratch_bytes(n_groups, N, K) : 0);
}

size_t moe_workspace_size(const MoeConfig* cfg, int path) {
  if (!cfg || path < MOE_PATH_MXFP4 || path > MOE_PATH_PTPC) return 0;
  const MoeConfig& c = *cfg;
  if (c.T < 0 || c.H <= 0 || c.I <= 0 || c.H % 128 || c.I % 128 || c.E < 1 || c.topk < 1 || c.topk > c.E)
    return 0;
  const int64_t R = (int64_t)c.T * c.topk + (c.has_shared ? c.T : 0);
  if (R > (int64_t)INT32_MAX) return 0;
  const int G = c.E + (c.has_shared ? 1 : 0);
  size_t need = moe_permute_workspace_size(c.T, c.E, c.topk);
  for (int bn : {0, 16, 32, 64, 128, 256})
    for (int K : {c.H, c.I}) need = std::max(need, moe_gemm_workspace_size((int)R, G, K, bn));
  if (path == MOE_PATH_W4AFP8) {   // the E4M3 copy of the weights for wide token tiles
    need = std::max(need, moe_w4afp8_workspace_size((int)R, G, 2 * c.I, c.H, 0));
    need = std::max(need, moe_w4afp8_workspace_size((int)R, G, c.H, c.I, 0));
  }
  return (need + 255) / 256 * 256;
}

int moe_grouped_gemm_mxfp4(const uint8_t* a_e4m3, const uint8_t* a_e8m0_128, int a_rows, const int32_t* offsets,
                           int n_groups, const uint8_t* w_prepared, int N, int K, int epilogue, float swiglu_limit,
                           int block_n, void* out, uint8_t* out_scale, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (a_rows < 0 || n_groups < 1 || n_groups > 1024 || N <= 0 || K <= 0 || N % 128 || K % 128)
    return MOE_ERR_INVALID;
  if (epilogue < MOE_EPI_STORE_F32 || epilogue > MOE_EPI_SWIGLU_QUANT) return MOE_ERR_INVALID;
  if (epilogue == MOE_EPI_SWIGLU_QUANT && N % 256) return MOE_ERR_INVALID;
  if (block_n != 0 && block_n != 16 && block_n != 32 && block_n != 64 && block_n != 128 && block_n != 256)
    return MOE_ERR_UNSUPPORTED;
  if (block_n == pair::BN && N % 256) return MOE_ERR_UNSUPPORTED;
  if (a_rows == 0) return MOE_OK;
  if (!a_e4m3 || !a_e8m0_128 || !offsets || !w_prepared || !out || !workspace) return MOE_ERR_INVALID;
  if (epilogue == MOE_EPI_SWIGLU_QUANT && !out_scale) return MOE_ERR_INVALID;
  if (!aligned(a_e4m3, 16) || !aligned(w_prepared, 32) || !aligned(workspace, 256)) return MOE_ERR_INVALID;
  if (epilogue != MOE_EPI_SWIGLU_QUANT && !aligned(out, 16)) return MOE_ERR_INVALID;

  // Automatic choice: the tile width from the mean rows per group.  For the
  // SwiGLU projection with at least 192 rows per group on average (long
  // prefill) and a workspace that holds both plans, every group's whole
  // 256-row tiles go to the SM-pair kernel and its remaining rows (fewer than
  // 256) to the swap-AB kernel's 128-row tiles: long-prefill w1/w3 1.97 ->
  // 1.87 ms.  At 4096 tokens (111 rows per group) and for the float32 w2
  // projection the split measured 1-6 % slower, so those keep one kernel.
  bool split = false;
  if (block_n == 0) {
    block_n = pick_block_n(a_rows, n_groups);
    split = block_n == 128 && epilogue == MOE_EPI_SWIGLU_QUANT && a_rows >= 192 * n_groups &&
            workspace_bytes >= split_workspace_size(a_rows, n_groups, K);
  }
  const bool run_swap = block_n != pair::BN;          // the swap-AB kernel (tiles of block_n rows)
  const bool run_pair = block_n == pair::BN || split;
  const gemm::WsLayout L = gemm::ws_layout(a_rows, n_groups, K, run_swap ? block_n : pair::BN);
  if (workspace_bytes < L.total) return MOE_ERR_INVALID;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  // the pair kernel's plan: after the swap-AB plan when split
  const gemm::WsLayout LP = gemm::ws_layout(a_rows, n_groups, K, pair::BN);
  uint8_t* wsp = split ? ws + gemm::align256(L.total) : ws;

  // work items of the swap-AB kernel hold two 128-row weight tiles whenever N
  // allows (gate + up for SwiGLU, which requires N % 256 == 0)
  const bool pair_tiles = epilogue == MOE_EPI_SWIGLU_QUANT || N % 256 == 0;
  const int n_ft = pair_tiles ? N / 256 : N / 128;

  // Weight tiles and their scale blocks, as views of the prepared blocks
  // (kWBlock bytes each: 128 rows x 64 bytes of nibbles, then the 512-byte
  // scale block).  Paired order (SwiGLU): [pairs][2][...]; plain order: [row
  // blocks][K steps][...].  ta: the swap-AB kernel's box (both tiles of an
  // item), tw: one tile (each CTA of a pair loads its own), ts: the scale
  // blocks of both tiles.
  CUtensorMap ta, tw, ts;
  {
    const uint64_t KT = (uint64_t)K / 128, n_rb = (uint64_t)n_groups * (N / 128);
    const uint64_t wb = (uint64_t)gemm::kWBlock;
    const bool paired_order = epilogue == MOE_EPI_SWIGLU_QUANT;
    const uint64_t d2 = paired_order ? 2 : KT, d3 = paired_order ? n_rb * KT / 2 : n_rb;
    const uint64_t s2 = wb, s3 = paired_order ? 2 * wb : KT * wb;
    const uint32_t b2 = paired_order ? 2 : 1, b3 = (!paired_order && pair_tiles) ? 2 : 1;
    const uint64_t wdims[4] = {128, 128, d2, d3}, wstr[3] = {64, s2, s3};
    const uint32_t wbox[4] = {128, 128, b2, b3}, wbox1[4] = {128, 128, 1, 1};
    if (!make_map_nd(&ta, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w_prepared, 4, wdims, wstr, wbox,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_nd(&tw, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w_prepared, 4, wdims, wstr, wbox1,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return MOE_ERR_LAUNCH;
    // scale blocks as 128 32-bit words at byte 8192 of each prepared block
    const uint64_t sdims[3] = {128, d2, d3}, sstr[2] = {s2, s3};
    const uint32_t sbox[3] = {128, b2, b3};
    if (!make_map_nd(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT32, w_prepared + 8192, 3, sdims, sstr, sbox,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return MOE_ERR_LAUNCH;
  }

  cudaStream_t st = S(stream);
  if (run_swap) {
    // token tiles: boxes of 16, 32, 64 and block_n rows (capped at block_n)
    gemm::TokenMaps tb;
    for (int i = 0; i < 4; ++i)
      if (!make_map(&tb.m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, a_e4m3, (uint64_t)K, (uint64_t)a_rows, (uint64_t)K,
                    128, (uint32_t)gemm::token_box_rows(i, block_n)))
        return MOE_ERR_LAUNCH;
    gemm::GemmArgs args;
    args.w = w_prepared;
    args.a_sf = ws + L.a_sf;
    args.header = reinterpret_cast<const int*>(ws + L.header);
    args.prefix = reinterpret_cast<const int*>(ws + L.prefix);
    args.tstart = reinterpret_cast<const int*>(ws + L.tstart);
    args.groups = reinterpret_cast<const int2*>(ws + L.groups);
    args.G = n_groups;
    args.N = N;
    args.K = K;
    args.out = out;
    args.out_scale = out_scale;
    args.limit = swiglu_limit;
    // decode-sized token tiles stream the weights once: an L2 prefetch 4 K
    // steps ahead of the producer keeps more of that stream in flight (0.270
    // -> 0.260 ms for the 64-token w1/w3 GEMM); wider tiles are bound by
    // shared-memory traffic and lose 6-12 % to the extra L2 traffic
    args.pf_steps = block_n <= 32 ? 4 : 0;
    launch(gemm::gemm_prep_kernel, dim3(L.max_tiles), dim3(gemm::kPrepThreads), 0, st, offsets, n_groups,
           (int)a_rows, block_n, n_ft, a_e8m0_128, K / 128, reinterpret_cast<int*>(ws + L.header),
           reinterpret_cast<int*>(ws + L.prefix), reinterpret_cast<int*>(ws + L.tstart),
           reinterpret_cast<int2*>(ws + L.groups), ws + L.a_sf, nullptr, nullptr, split ? pair::BN : 0, 1);
    if (launch_status() != MOE_OK) return MOE_ERR_LAUNCH;
    int rc;
    switch (epilogue) {
      case MOE_EPI_STORE_F32:
        rc = pair_tiles ? launch_gemm_bn<true, MOE_EPI_STORE_F32>(block_n, ta, tb, ts, args, st)
                        : launch_gemm_bn<false, MOE_EPI_STORE_F32>(block_n, ta, tb, ts, args, st);
        break;
      case MOE_EPI_STORE_BF16:
        rc = pair_tiles ? launch_gemm_bn<true, MOE_EPI_STORE_BF16>(block_n, ta, tb, ts, args, st)
                        : launch_gemm_bn<false, MOE_EPI_STORE_BF16>(block_n, ta, tb, ts, args, st);
        break;
      default: rc = launch_gemm_bn<true, MOE_EPI_SWIGLU_QUANT>(block_n, ta, tb, ts, args, st);
    }
    if (rc != MOE_OK) return rc;
  }
  if (run_pair) {
    if (LP.total > workspace_bytes - (size_t)(wsp - ws)) return MOE_ERR_INVALID;
    pair::PairMaps tt;
    for (int i = 0; i < 4; ++i)
      if (!make_map(&tt.tok[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, a_e4m3, (uint64_t)K, (uint64_t)a_rows, (uint64_t)K,
                    128, (uint32_t)gemm::token_box_rows(i, 128)))
        return MOE_ERR_LAUNCH;
    // token scales: the plan's interleaved blocks (two 512-byte blocks per
    // tile and group of four K steps, one per CTA) as rows of 128 words
    const uint64_t n_sf = (uint64_t)LP.max_tiles * ((K / 128 + 3) / 4) * 2;
    if (!make_map(&tt.tok_sf, CU_TENSOR_MAP_DATA_TYPE_UINT32, wsp + LP.a_sf, 128, n_sf, 512, 128, 1,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return MOE_ERR_LAUNCH;
    pair::PairArgs pa;
    pa.header = reinterpret_cast<const int*>(wsp + LP.header);
    pa.prefix = reinterpret_cast<const int*>(wsp + LP.prefix);
    pa.tstart = reinterpret_cast<const int*>(wsp + LP.tstart);
    pa.groups = reinterpret_cast<const int2*>(wsp + LP.groups);
    pa.G = n_groups;
    pa.N = N;
    pa.K = K;
    pa.out = out;
    pa.out_scale = out_scale;
    pa.limit = swiglu_limit;
    launch(gemm::gemm_prep_kernel, dim3(LP.max_tiles), dim3(gemm::kPrepThreads), 0, st, offsets, n_groups,
           (int)a_rows, pair::BN, N / 256, a_e8m0_128, K / 128, reinterpret_cast<int*>(wsp + LP.header),
           reinterpret_cast<int*>(wsp + LP.prefix), reinterpret_cast<int*>(wsp + LP.tstart),
           reinterpret_cast<int2*>(wsp + LP.groups), wsp + LP.a_sf, nullptr, nullptr, split ? pair::BN : 0, 0);
    if (launch_status() != MOE_OK) return MOE_ERR_LAUNCH;
    switch (epilogue) {
      case MOE_EPI_STORE_F32: return launch_pair<MOE_EPI_STORE_F32>(tw, tt, ts, pa, st);
      case MOE_EPI_STORE_BF16: return launch_pair<MOE_EPI_STORE_BF16>(tw, tt, ts, pa, st);
      default: return launch_pair<MOE_EPI_SWIGLU_QUANT>(tw, tt, ts, pa, st);
    }
  }
  return MOE_OK;
}

int moe_grouped_gemm_w4afp8(const uint8_t* a_e4m3, const uint8_t* a_e8m0_128, int a_rows, const int32_t* offsets,
                            int n_groups, const int8_t* w_int4, const float* w_scale_inv, int N, int K,
                            int epilogue, float swiglu_limit, int block_n, void* out, uint8_t* out_scale,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return promoted_gemm<false>(a_e4m3, a_e8m0_128, a_rows, offsets, n_groups, w_int4, w_scale_inv, N, K, epilogue,
                              swiglu_limit, block_n, out, out_scale, workspace, workspace_bytes, stream);
}

int moe_grouped_gemm_fp8_block128(const uint8_t* a_e4m3, const uint8_t* a_e8m0_128, int a_rows,
                                  const int32_t* offsets, int n_groups, const uint8_t* w_e4m3,
                                  const float* w_scale_inv, int N, int K, int epilogue, float swiglu_limit,
                                  int block_n, void* out, uint8_t* out_scale, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return promoted_gemm<true>(a_e4m3, a_e8m0_128, a_rows, offsets, n_groups, w_e4m3, w_scale_inv, N, K, epilogue,
                             swiglu_limit, block_n, out, out_scale, workspace, workspace_bytes, stream);
}

int moe_grouped_gemm_fp8_ptpc(const uint8_t* a_e4m3, const float* a_scale, int a_rows, const int32_t* offsets,
                              int n_groups, const uint8_t* w_e4m3, const float* w_scale, int N, int K, int epilogue,
                              float swiglu_limit, int block_n, void* out, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (a_rows < 0 || n_groups < 1 || n_groups > 1024 || N <= 0 || K <= 0 || N % 128 || K % 128)
    return MOE_ERR_INVALID;
  if (epilogue != MOE_EPI_STORE_F32 && epilogue != MOE_EPI_STORE_BF16 && epilogue != MOE_EPI_SWIGLU_F32)
    return MOE_ERR_INVALID;
  const bool dual = epilogue == MOE_EPI_SWIGLU_F32;
  if (dual && N % 256) return MOE_ERR_INVALID;
  if (block_n == 0) block_n = pick_block_n(a_rows, n_groups);
  if (block_n != 16 && block_n != 32 && block_n != 64 && block_n != 128) return MOE_ERR_UNSUPPORTED;
  if (a_rows == 0) return MOE_OK;
  if (!a_e4m3 || !a_scale || !offsets || !w_e4m3 || !w_scale || !out || !workspace) return MOE_ERR_INVALID;
  if (!aligned(a_e4m3, 16) || !aligned(w_e4m3, 16) || !aligned(a_scale, 4) || !aligned(w_scale, 4) ||
      !aligned(workspace, 256))
    return MOE_ERR_INVALID;
  const gemm::WsLayout L = gemm::ws_layout(a_rows, n_groups, K, block_n);
  if (workspace_bytes < L.total) return MOE_ERR_INVALID;
  CUtensorMap ta, tb;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_e4m3, (uint64_t)K, (uint64_t)n_groups * N, (uint64_t)K, 128,
                128))
    return MOE_ERR_LAUNCH;
  if (!make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_e4m3, (uint64_t)K, (uint64_t)a_rows, (uint64_t)K, 128,
                (uint32_t)block_n))
    return MOE_ERR_LAUNCH;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  ptpc::Args args;
  args.w_scale = w_scale;
  args.a_scale = a_scale;
  args.header = reinterpret_cast<const int*>(ws + L.header);
  args.prefix = reinterpret_cast<const int*>(ws + L.prefix);
  args.tstart = reinterpret_cast<const int*>(ws + L.tstart);
  args.groups = reinterpret_cast<const int2*>(ws + L.groups);
  args.G = n_groups;
  args.N = N;
  args.K = K;
  args.out = out;
  args.limit = swiglu_limit;
  cudaStream_t st = S(stream);
  const int n_ft = dual ? N / 256 : N / 128;
  // the plan only: no per-tile activation scale blocks (sx == nullptr)
  launch(gemm::gemm_prep_kernel, dim3(L.max_tiles), dim3(gemm::kPrepThreads), 0, st, 
      offsets, n_groups, (int)a_rows, block_n, n_ft, nullptr, K / 128, reinterpret_cast<int*>(ws + L.header),
      reinterpret_cast<int*>(ws + L.prefix), reinterpret_cast<int*>(ws + L.tstart),
      reinterpret_cast<int2*>(ws + L.groups), ws + L.a_sf, nullptr, nullptr, 0, 0);
  if (launch_status() != MOE_OK) return MOE_ERR_LAUNCH;
  if (dual) return launch_ptpc_bn<true, MOE_EPI_SWIGLU_F32>(block_n, ta, tb, args, st);
  if (epilogue == MOE_EPI_STORE_F32) return launch_ptpc_bn<false, MOE_EPI_STORE_F32>(block_n, ta, tb, args, st);
  return launch_ptpc_bn<false, MOE_EPI_STORE_BF16>(block_n, ta, tb, args, st);
}

int moe_quantize_fp8_per_token(const void* x, int x_is_f32, int rows, int cols, uint8_t* q, float* scale,
                               void* stream) {
  if (rows < 0 || cols <= 0 || cols % 8) return MOE_ERR_INVALID;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !scale || !aligned(x, 16) || !aligned(q, 8) || !aligned(scale, 4)) return MOE_ERR_INVALID;
  if (x_is_f32)
    launch(quant_fp8_per_row_kernel<true>, dim3((unsigned)rows), dim3(256), 0, S(stream), x, cols, q, scale);
  else
    launch(quant_fp8_per_row_kernel<false>, dim3((unsigned)rows), dim3(256), 0, S(stream), x, cols, q, scale);
  return launch_status();
}

int moe_gather_row_scales(const int32_t* perm, int T, int k, const int32_t* offsets, int E, const float* src,
                          float* dst, void* stream) {
  if (T < 0 || k < 0 || E < 0) return MOE_ERR_INVALID;
  const int64_t max_rows = (int64_t)T * (k + 1);
  if (max_rows > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (max_rows == 0) return MOE_OK;
  if (!perm || !offsets || !src || !dst || !aligned(src, 4) || !aligned(dst, 4)) return MOE_ERR_INVALID;
  launch(gather_row_scales_kernel, dim3((unsigned)((max_rows + 255) / 256)), dim3(256), 0, S(stream), perm, T, k, offsets, E, src,
                                                                                        dst);
  return launch_status();
}

int moe_swiglu_clamp(const float* gu, int rows, int I, float limit, uint8_t* hq, uint8_t* sh, void* stream) {
  if (rows < 0 || I <= 0 || I % 128) return MOE_ERR_INVALID;
  if (rows == 0) return MOE_OK;
  if (!gu || !hq || !sh || !aligned(gu, 16) || !aligned(hq, 4)) return MOE_ERR_INVALID;
  const int64_t groups = (int64_t)rows * (I / 128);
  launch(swiglu_quant_kernel, dim3((unsigned)((groups + 7) / 8)), dim3(256), 0, S(stream), 
      reinterpret_cast<const float4*>(gu), rows, I, limit, reinterpret_cast<uint32_t*>(hq), sh);
  return launch_status();
}

int moe_combine(const float* o, const int32_t* inv, const float* w, int T, int k, int H, int has_shared,
                const int32_t* offsets, int E, void* y, void* stream) {
  if (T < 0 || k < 0 || H <= 0 || H % 4 || E < 0) return MOE_ERR_INVALID;
  if (T == 0) return MOE_OK;
  if (!o || !y || (k > 0 && (!inv || !w)) || (has_shared && !offsets)) return MOE_ERR_INVALID;
  if (!aligned(o, 16) || !aligned(y, 8)) return MOE_ERR_INVALID;
  // one block per (token, 512 columns): two 4-column chunks a thread
  const int slices = (H / 4 + 2 * kCombineThreads - 1) / (2 * kCombineThreads);
  launch(combine_kernel, dim3((unsigned)T, (unsigned)slices), dim3(kCombineThreads), 0, S(stream),
         reinterpret_cast<const float4*>(o), inv, w, T, k, H, has_shared ? 1 : 0, offsets, E,
         reinterpret_cast<uint2*>(y));
  return launch_status();
}

int repack_mxfp4_to_nvfp4(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K, uint8_t* out_fp4,
                          uint8_t* out_e4m3, float* out_global, void* stream) {
  if (n_mats < 0 || N <= 0 || K <= 0 || K % 32) return MOE_ERR_INVALID;
  if (n_mats == 0) return MOE_OK;
  if (!fp4 || !e8m0 || !out_fp4 || !out_e4m3 || !out_global) return MOE_ERR_INVALID;
  if (!aligned(fp4, 16) || !aligned(out_fp4, 16) || !aligned(out_e4m3, 2)) return MOE_ERR_INVALID;
  const int64_t per_mat = (int64_t)N * (K / 32);
  const int64_t n_scale = n_mats * per_mat;
  const int64_t fp4_bytes = n_mats * (int64_t)N * (K / 2);
  if (fp4_bytes % 16) return MOE_ERR_INVALID;
  cudaStream_t st = S(stream);
  const bool alias = out_fp4 == fp4;
  // 16 scale bytes at a time when the scale arrays allow it
  const bool vec = per_mat % 16 == 0 && aligned(e8m0, 16) && aligned(out_e4m3, 16);
  if (vec) {
    launch(nvfp4_global_vec_kernel, dim3((unsigned)n_mats), dim3(512), 0, st, reinterpret_cast<const uint4*>(e8m0), per_mat / 16,
                                                             out_global);
    const int64_t work = std::max<int64_t>(n_scale / 16, alias ? 0 : fp4_bytes / 16);
    const int64_t grid = std::min<int64_t>((work + 255) / 256, (int64_t)sm_count() * 16);
    launch(nvfp4_convert_vec_kernel, dim3((unsigned)std::max<int64_t>(grid, 1)), dim3(256), 0, st, 
        reinterpret_cast<const uint4*>(e8m0), n_scale / 16, per_mat / 16, out_global,
        reinterpret_cast<uint4*>(out_e4m3), reinterpret_cast<const uint4*>(fp4),
        alias ? nullptr : reinterpret_cast<uint4*>(out_fp4), fp4_bytes / 16);
  } else {
    launch(nvfp4_global_kernel, dim3((unsigned)n_mats), dim3(256), 0, st, e8m0, per_mat, out_global);
    const int64_t work = std::max<int64_t>(n_scale, alias ? 0 : fp4_bytes / 16);
    const int64_t grid = std::min<int64_t>((work + 255) / 256, (int64_t)sm_count() * 16);
    launch(nvfp4_convert_kernel, dim3((unsigned)std::max<int64_t>(grid, 1)), dim3(256), 0, st, 
        e8m0, n_scale, per_mat, out_global, out_e4m3, reinterpret_cast<const uint4*>(fp4),
        alias ? nullptr : reinterpret_cast<uint4*>(out_fp4), fp4_bytes / 16);
  }
  return launch_status();
}

int repack_mxfp4_to_int4g128(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K,
                             int8_t* out_int4, float* out_scale_inv, void* stream) {
  if (n_mats < 0 || N <= 0 || K <= 0 || K % 128) return MOE_ERR_INVALID;
  if (n_mats == 0) return MOE_OK;
  if (!fp4 || !e8m0 || !out_int4 || !out_scale_inv) return MOE_ERR_INVALID;
  if (!aligned(fp4, 16) || !aligned(out_int4, 16) || !aligned(e8m0, 4) || !aligned(out_scale_inv, 4))
    return MOE_ERR_INVALID;
  const int64_t blocks = n_mats * (int64_t)N * (K / 32);     // 32-element blocks, 4 per group
  // grid-stride: each block of threads builds its code tables once
  const int64_t grid = std::min<int64_t>((blocks + 255) / 256, (int64_t)sm_count() * 8);
  launch(int4g128_kernel, dim3((unsigned)grid), dim3(256), 0, S(stream), 
      reinterpret_cast<const uint4*>(fp4), e8m0, blocks, reinterpret_cast<uint4*>(out_int4), out_scale_inv);
  return launch_status();
}

int repack_mxfp4_to_fp8_block128(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K,
                                 uint8_t* out_e4m3, float* out_scale_inv, void* stream) {
  if (n_mats < 0 || N <= 0 || K <= 0 || N % 128 || K % 128) return MOE_ERR_INVALID;
  if (n_mats == 0) return MOE_OK;
  if (!fp4 || !e8m0 || !out_e4m3 || !out_scale_inv) return MOE_ERR_INVALID;
  if (!aligned(fp4, 16) || !aligned(out_e4m3, 16) || !aligned(e8m0, 4) || !aligned(out_scale_inv, 4))
    return MOE_ERR_INVALID;
  const int64_t blocks = n_mats * (int64_t)(N / 128) * (K / 128);
  if (blocks > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  launch(fp8_block128_kernel, dim3((unsigned)blocks), dim3(128), 0, S(stream), fp4, e8m0, N, K, out_e4m3, out_scale_inv);
  return launch_status();
}

int repack_mxfp4_to_fp8_per_channel(const uint8_t* fp4, const uint8_t* e8m0, int64_t n_mats, int N, int K,
                                    uint8_t* out_e4m3, float* out_scale, void* stream) {
  if (n_mats < 0 || N <= 0 || K <= 0 || K % 32) return MOE_ERR_INVALID;
  if (n_mats == 0) return MOE_OK;
  if (!fp4 || !e8m0 || !out_e4m3 || !out_scale) return MOE_ERR_INVALID;
  if (!aligned(fp4, 4) || !aligned(out_e4m3, 8) || !aligned(out_scale, 4)) return MOE_ERR_INVALID;
  const int64_t rows = n_mats * (int64_t)N;
  if (rows > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  launch(fp8_per_channel_kernel, dim3((unsigned)rows), dim3(256), 0, S(stream), fp4, e8m0, K, out_e4m3, out_scale);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Grouping without caller scratch.  The per-chunk expert histograms live in a
// fixed device array owned by this library instead of a caller workspace.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

constexpr int64_t kNoAllocScratchInts = 65536;   // 256 KiB: n_chunks * E int32 counters
static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocScratchInts];

// Device address of g_permute_scratch, looked up with the device current
// (the host-side symbol is not a device address) and cached per device
// together with the context it was found in: after a device reset the
// primary context, and with it the module and the array's address, is new,
// so a changed context triggers a fresh lookup.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

int32_t* permute_scratch_ptr(int* status) {
  static std::mutex mu;
  static int32_t* ptrs[128] = {};
  static CUcontext ctxs[128] = {};
  int dev = 0;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (!get_ctx || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
    *status = MOE_ERR_LAUNCH;
    return nullptr;
  }
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) {
    *status = MOE_ERR_LAUNCH;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev] || !ctx || ctxs[dev] != ctx) {
    // the lookup also makes the device's primary context current when no
    // context was yet (it allocates nothing)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p || get_ctx(&ctx) != CUDA_SUCCESS ||
        !ctx) {
      *status = MOE_ERR_LAUNCH;
      return nullptr;
    }
    ptrs[dev] = static_cast<int32_t*>(p);
    ctxs[dev] = ctx;
  }
  *status = MOE_OK;
  return ptrs[dev];
}

}  // namespace

extern "C" {

int64_t moe_permute_noalloc_max_counters(void) { return kNoAllocScratchInts; }

int moe_permute_noalloc(const int32_t* idx, int T, int E, int k, int has_shared, const uint8_t* xq,
                        const uint8_t* sx, int H, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                        uint8_t* xq_perm, uint8_t* sx_perm, void* stream) {
  if (T < 0 || E < 1 || E > 1023 || k < 1 || H <= 0 || H % 128) return MOE_ERR_INVALID;
  if (!counts || !offsets) return MOE_ERR_INVALID;
  if ((int64_t)T * k > (int64_t)1 << 30) return MOE_ERR_UNSUPPORTED;
  const int P = T * k;
  const int64_t n_chunks = (P + kChunk - 1) / kChunk;
  if (n_chunks * E > kNoAllocScratchInts) return MOE_ERR_UNSUPPORTED;   // beyond the fixed scratch
  if (T > 0) {
    if (!idx || !xq || !sx || !perm || !inv || !xq_perm || !sx_perm) return MOE_ERR_INVALID;
    if (!aligned(xq, 16) || !aligned(xq_perm, 16)) return MOE_ERR_INVALID;
  }
  int st_code = MOE_OK;
  int32_t* hist = permute_scratch_ptr(&st_code);
  if (!hist) return st_code;
  cudaStream_t st = S(stream);
  // every counter the scan reads is written by the count pass of this call,
  // so the scratch needs no clearing between calls
  launch_permute(idx, T, E, k, has_shared, xq, sx, H, counts, offsets, perm, inv, xq_perm, sx_perm, hist, st);
  return launch_status();
}

}  // extern "C"
