// mr.cu -- libmr.so: the extern "C" entry points declared in include/mr.h.
//
// Host code only validates arguments, builds TMA descriptors and launches the
// kernels of this directory on the caller's stream; every step of the routing
// path runs on the GPU.  Built as one translation unit for sm_100a.
#include <cudaTypedefs.h>

#include <atomic>
#include <type_traits>
#include <cstdlib>
#include <cstring>
#include <cmath>
#include <mutex>

#include "dispatch.cuh"
#include "ep.cuh"
#include "expert_gemm.cuh"
#include "mr_common.cuh"
#include "router_ffma.cuh"
#include "router_splitk.cuh"
#include "router_tc.cuh"
#include "route.cuh"
#include "combine.cuh"
#include "gather.cuh"

namespace {

constexpr int kMaxDevices = 64;

int g_num_sms[kMaxDevices];
int g_cc_major[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

// Properties of the current device, queried once per device.
bool device_info(int* sms, int* cc_major) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::call_once(g_dev_once[dev], [dev] {
    int v = 0;
    g_num_sms[dev] = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? v : 0;
    g_cc_major[dev] = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess ? v : 0;
  });
  *sms = g_num_sms[dev];
  *cc_major = g_cc_major[dev];
  return *sms > 0;
}

std::atomic<uint64_t> g_launches{0};

// Status of the launch just made (and count it).
int launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MR_OK : MR_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// ---- TMA descriptors -------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// Row-major bf16 matrix [rows, cols], box [box_rows, 32] (64-byte rows, 64-byte swizzle).
bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows, bool swizzle = true) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {32, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swizzle ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major fp32 matrix [rows, cols], box [box_rows, box_cols], swizzled rows.
bool make_map_f32(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows, uint32_t box_cols) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * sizeof(float)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      box_cols * 4 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- router -----------------------------------------------------------------

int validate_router(const void* x, int x_dtype, const float* W, int T, int d, int N_r,
                    int n_group, int topk_group, int k, float route_scale, int mask_mode,
                    int precision, const int32_t* idx_out, const float* w_out) {
  if (T < 0 || d <= 0 || N_r <= 0 || n_group <= 0 || k <= 0) return MR_ERR_INVALID_ARG;
  if (N_r % n_group != 0 || topk_group < 1 || topk_group > n_group || k > N_r)
    return MR_ERR_INVALID_ARG;
  if (n_group > 1 && N_r / n_group < 2) return MR_ERR_INVALID_ARG;
  if (mask_mode != MR_MASK_NEG_INF && mask_mode != MR_MASK_ZERO) return MR_ERR_INVALID_ARG;
  if (mask_mode == MR_MASK_NEG_INF && n_group > 1 && k > topk_group * (N_r / n_group))
    return MR_ERR_INVALID_ARG;
  if (x_dtype != MR_F32 && x_dtype != MR_BF16) return MR_ERR_INVALID_ARG;
  if (precision != MR_PREC_3XTF32 && precision != MR_PREC_TF32 && precision != MR_PREC_FFMA &&
      precision != MR_PREC_BF16X3)
    return MR_ERR_INVALID_ARG;
  if (!std::isfinite(route_scale)) return MR_ERR_INVALID_ARG;
  if ((long long)T * k >= (1LL << 31) || (long long)T * d >= (1LL << 40)) return MR_ERR_INVALID_ARG;
  if (T > 0 && (!x || !W || !idx_out || !w_out)) return MR_ERR_INVALID_ARG;
  if (N_r > 512 || n_group > 32 || k > 8) return MR_ERR_UNSUPPORTED;
  return MR_OK;
}

// Tensor-core path: rows of 16-byte multiples for TMA, experts per CTA a
// multiple of 16 (the MMA's N granularity for M = 128).
bool tc_shape_ok(const void* x, int x_dtype, const float* W, int d, int N_r) {
  const bool n_ok = N_r <= 256 ? (N_r % 16 == 0 && N_r >= 16) : (N_r % 32 == 0);
  return x_dtype == MR_F32 && d % 4 == 0 && n_ok && aligned16(x) && aligned16(W);
}

template <int NJ, bool XBF16, bool WBF16>
int launch_ffma_nj(const void* x, const void* W, const float* bias, int T, int d, int N_r,
                   int n_group, int topk_group, int k, float route_scale, int mask_mode,
                   int flags, int32_t* idx_out, float* w_out, float* logits_out,
                   cudaStream_t st) {
  const size_t smem = mr::ffma_smem_bytes(NJ);
  auto kern = mr::router_ffma_kernel<NJ, XBF16, WBF16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MR_ERR_CUDA;
  const unsigned grid = (unsigned)((T + mr::kFfmaTokens - 1) / mr::kFfmaTokens);
  kern<<<grid, mr::kFfmaThreads, smem, st>>>(x, W, bias, T, d, N_r, n_group, topk_group, k,
                                              route_scale, mask_mode, flags, idx_out, w_out,
                                              logits_out);
  return launch_status();
}

template <bool XBF16, bool WBF16 = false>
int launch_ffma(const void* x, const void* W, const float* bias, int T, int d, int N_r,
                int n_group, int topk_group, int k, float route_scale, int mask_mode, int flags,
                int32_t* idx_out, float* w_out, float* logits_out, cudaStream_t st) {
  const int nj = (N_r + 31) / 32;
#define MR_FFMA_CASE(NJV)                                                                       \
  if (nj <= NJV)                                                                              \
    return launch_ffma_nj<NJV, XBF16, WBF16>(x, W, bias, T, d, N_r, n_group, topk_group, k,   \
                                             route_scale, mask_mode, flags, idx_out, w_out,   \
                                             logits_out, st);
  MR_FFMA_CASE(1)
  MR_FFMA_CASE(2)
  MR_FFMA_CASE(4)
  MR_FFMA_CASE(8)
  MR_FFMA_CASE(12)
  MR_FFMA_CASE(16)
#undef MR_FFMA_CASE
  return MR_ERR_UNSUPPORTED;
}

// ---- small-batch (split-K) router ---------------------------------------

constexpr int kSplitKMaxT = 256;  // batches up to one MMA N of tokens

struct SplitKShape {
  int NT, TT, MT, KC, KS, CL;
  size_t ws_bytes;
};

// Clusters of kCluster split-K CTAs that fit on the device at once (a cluster
// must sit inside one GPC, so fewer than sms / kCluster may); 0 if unknown.
int splitk_max_clusters(size_t smem) {
  static std::mutex mu;
  static int cache_dev[16], cache_n[16];
  static size_t cache_smem[16];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache_dev[i] == dev && cache_smem[i] == smem) return cache_n[i];
  if (cudaFuncSetAttribute(mr::sk::router_splitk_gemm_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(mr::sk::kCluster);
  cfg.blockDim = dim3(mr::sk::kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = mr::sk::kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, mr::sk::router_splitk_gemm_kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  if (used < 16) {
    cache_dev[used] = dev;
    cache_smem[used] = smem;
    cache_n[used] = n;
    ++used;
  }
  return n;
}

// bm: W and x both bf16 (kind::f16 on the staged tiles).
SplitKShape splitk_shape(int T, int d, int N_r, int sms, bool x_bf16, bool bm = false) {
  SplitKShape k;
  k.NT = ((T + 15) / 16) * 16;
  if (k.NT > mr::sk::kMaxNT) k.NT = mr::sk::kMaxNT;
  k.TT = (T + k.NT - 1) / k.NT;
  k.MT = (N_r + mr::tc::BM - 1) / mr::tc::BM;
  k.KC = (d + mr::tc::BK - 1) / mr::tc::BK;
  int ks = sms / (k.MT * k.TT);
  if (ks < 1) ks = 1;
  if (ks > k.KC) ks = k.KC;
  // slices reduced in clusters of kCluster through distributed shared memory
  k.CL = 1;
  if (ks >= 2 * mr::sk::kCluster) {
    // as many clusters as fit at once (one wave), kCluster slices each
    const mr::sk::Plan pl = mr::sk::make_plan(k.NT, (k.KC + ks - 1) / ks, x_bf16, bm);
    int per_tile = ks / mr::sk::kCluster;
    const int fit = splitk_max_clusters(pl.total + 1024);
    if (fit > 0 && per_tile * k.MT * k.TT > fit) per_tile = fit / (k.MT * k.TT);
    if (per_tile >= 2) {
      ks = per_tile * mr::sk::kCluster;
      k.CL = mr::sk::kCluster;
    }
  }
  k.KS = ks;
  k.ws_bytes = (size_t)(k.KS / k.CL) * (size_t)T * (size_t)N_r * sizeof(float);
  return k;
}

bool splitk_applies(int T, int N_r) { return T > 0 && T <= kSplitKMaxT && N_r <= 512; }

template <int NJ>
int launch_reduce_nj(const float* part, int KS, int T, int N_r, const float* bias, int n_group,
                     int topk_group, int k, float route_scale, int mask_mode, int flags,
                     int32_t* idx_out, float* w_out, float* logits_out, cudaStream_t st) {
  // programmatic dependent of the GEMM: launched while the GEMM drains, it
  // waits (griddepcontrol.wait) for the GEMM's results before reading them
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)T);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, mr::sk::router_reduce_route_kernel<NJ>, part, KS,
                                           T, N_r, bias, n_group, topk_group, k, route_scale,
                                           mask_mode, flags, idx_out, w_out, logits_out);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MR_ERR_CUDA;
  }
  return MR_OK;
}

int launch_route(const mr::rt::Params& rp, cudaStream_t st);

// W fp32 (3xTF32, or one tf32 product without use3x), or W stored in bf16
// (wb16 non-null; x must be bf16: kind::f16 MMAs on the staged tiles).
int launch_splitk(const void* x, bool x_bf16, const float* W, const float* bias, int T, int d,
                  int N_r, int n_group, int topk_group, int k, float route_scale, int mask_mode,
                  int flags, bool use3x, int32_t* idx_out, float* w_out, float* logits_out,
                  void* ws, int sms, cudaStream_t st, const void* wb16 = nullptr) {
  const bool bm = wb16 != nullptr;
  const SplitKShape sh = splitk_shape(T, d, N_r, sms, x_bf16, bm);
  const mr::sk::Plan plan = mr::sk::make_plan(sh.NT, (sh.KC + sh.KS - 1) / sh.KS, x_bf16, bm);
  CUtensorMap mw, mx;
  if (bm) {
    if (!x_bf16) return MR_ERR_UNSUPPORTED;
    if (!make_map_bf16(&mw, wb16, (uint64_t)N_r, (uint64_t)d, mr::tc::BM) ||
        !make_map_bf16(&mx, x, (uint64_t)T, (uint64_t)d, sh.NT))
      return MR_ERR_CUDA;
  } else if (!make_map_f32(&mw, W, (uint64_t)N_r, (uint64_t)d, mr::tc::BM, mr::tc::BK)) {
    return MR_ERR_CUDA;
  } else if (x_bf16) {
    if (!make_map_bf16(&mx, x, (uint64_t)T, (uint64_t)d, sh.NT, /*swizzle=*/false))
      return MR_ERR_CUDA;
  } else if (!make_map_f32(&mx, static_cast<const float*>(x), (uint64_t)T, (uint64_t)d, sh.NT,
                           mr::tc::BK)) {
    return MR_ERR_CUDA;
  }
  mr::sk::Params P;
  P.T = T;
  P.d = d;
  P.N = N_r;
  P.NT = sh.NT;
  P.KS = sh.KS;
  P.CL = sh.CL;
  P.num_kc = sh.KC;
  P.use3x = use3x ? 1 : 0;
  P.x_bf16 = x_bf16 ? 1 : 0;
  P.bf16_mma = bm ? 1 : 0;
  P.part = static_cast<float*>(ws);
  const size_t smem = plan.total + 1024;
  if (cudaFuncSetAttribute(mr::sk::router_splitk_gemm_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MR_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sh.KS, (unsigned)sh.MT, (unsigned)sh.TT);
  cfg.blockDim = dim3(mr::sk::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)sh.CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, mr::sk::router_splitk_gemm_kernel, mw, mx, P);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return MR_ERR_CUDA;
  }
  if (launch_status() != MR_OK) return MR_ERR_CUDA;
  const int KSr = sh.KS / sh.CL;
  // Reduce and route: the routing kernel (one warp per token where the lane
  // layout fits) unless MR_ROUTE_KERNEL=0 pins the one-CTA-per-token kernel
  const char* rk_env = getenv("MR_ROUTE_KERNEL");
  const int lanes = (rk_env && rk_env[0] == '0')
                        ? 0
                        : mr::rt::lanes_per_token(T, N_r, n_group, k, sms,
                                                  getenv("MR_ROUTE_LANES")
                                                      ? atoi(getenv("MR_ROUTE_LANES"))
                                                      : 0);
  if (lanes > 0) {
    mr::rt::Params rp;
    rp.part = P.part;
    rp.KS = KSr;
    rp.T = T;
    rp.N = N_r;
    rp.P = lanes;
    rp.n_group = n_group;
    rp.topk_group = topk_group;
    rp.k = k;
    rp.mask_mode = mask_mode;
    rp.flags = flags;
    rp.route_scale = route_scale;
    rp.bias = bias;
    rp.idx_out = idx_out;
    rp.w_out = w_out;
    rp.logits_out = logits_out;
    return launch_route(rp, st);
  }
  const int nj = (N_r + 31) / 32;
#define MR_RED_CASE(NJV)                                                                      \
  if (nj <= NJV)                                                                              \
    return launch_reduce_nj<NJV>(P.part, KSr, T, N_r, bias, n_group, topk_group, k,            \
                                 route_scale, mask_mode, flags, idx_out, w_out, logits_out, st);
  MR_RED_CASE(2)
  MR_RED_CASE(4)
  MR_RED_CASE(8)
  MR_RED_CASE(12)
  MR_RED_CASE(16)
#undef MR_RED_CASE
  return MR_ERR_UNSUPPORTED;
}

// Routing kernel after the tensor-core router (part = its logits or K-split
// partial sums, P lanes per token): a programmatic dependent of the router.
template <int EL>
int launch_route_el(const mr::rt::Params& rp, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  const int tpb = mr::rt::kThreads / rp.P;
  cfg.gridDim = dim3((unsigned)((rp.T + tpb - 1) / tpb));
  cfg.blockDim = dim3(mr::rt::kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, mr::rt::route_kernel<EL>, rp);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MR_ERR_CUDA;
  }
  return MR_OK;
}

int launch_route(const mr::rt::Params& rp, cudaStream_t st) {
  switch (rp.N / rp.P) {
    case 8: return launch_route_el<8>(rp, st);
    case 12: return launch_route_el<12>(rp, st);
    case 16: return launch_route_el<16>(rp, st);
    case 24: return launch_route_el<24>(rp, st);
    case 32: return launch_route_el<32>(rp, st);
    default: return MR_ERR_UNSUPPORTED;
  }
}

// How CTAs share a 128-token tile of the fused router:
//  - ks = 2 or 4 (N_r <= 256): a cluster of ks CTAs splits the K loop of the
//    tile (partial sums meet through distributed shared memory), taken while
//    ks times the tile count still fits the SMs and every CTA keeps at least
//    eight K chunks: the DeepSeek-V3 prefill batch (32 tiles) runs on 128
//    CTAs instead of 32;
//  - CS = 2 splits the experts over a 2-CTA cluster: always when N_r > 256
//    (TMEM holds two accumulation buffers of at most 256 columns);
//  - otherwise one CTA per tile (the full 16384-token batch: 128 tiles).
// pair (bf16x3, N_r <= 256): two CTAs run one M = 256 MMA over consecutive
// tiles and each stages half of W.  It is only taken when pinned: on the
// full DeepSeek-V3 batch (T = 16384) it measured 5 us slower than one CTA
// per tile (188 vs 182 us).
// MR_TC_CLUSTER = 1, 2, P, K2 or K4 pins the choice (used by the tests to
// cover each).
struct TcShape {
  int CS;
  bool pair;
  int ks;
};

TcShape tc_shape(int T, int N_r, int sms, bool bf16x3, int num_kc) {
  if (N_r > 256) return {2, false, 1};
  const bool pair_ok = bf16x3 && N_r % 32 == 0;
  if (const char* env = getenv("MR_TC_CLUSTER")) {
    if (env[0] == '1') return {1, false, 1};
    if (env[0] == '2' && N_r % 32 == 0) return {2, false, 1};
    if ((env[0] == 'P' || env[0] == 'p') && pair_ok) return {1, true, 1};
    if ((env[0] == 'K' || env[0] == 'k') && (env[1] == '2' || env[1] == '4')) {
      const int ks = env[1] - '0';
      if (num_kc >= ks) return {1, false, ks};
    }
  }
  const int tiles = (T + mr::tc::BM - 1) / mr::tc::BM;
  int ks = 1;
  while (ks < 4 && 2 * ks * tiles <= sms && num_kc >= 8 * 2 * ks) ks *= 2;
  if (ks > 1) return {1, false, ks};
  if (N_r % 32 == 0 && 2 * tiles <= sms) return {2, false, 1};
  return {1, false, 1};
}

// W's residuals [N_r, d] fp32, precomputed into the workspace by the fused path.
size_t wlo_bytes(int d, int N_r) { return (size_t)N_r * (size_t)d * sizeof(float); }
// W's three bf16 planes [3, N_r, d] for bf16 activations.
size_t planes_bytes(int d, int N_r) { return 3 * (size_t)N_r * (size_t)d * 2; }
// The fused router's logits for the routing kernel, [ks][T][N_r] fp32, placed
// after the planes (or W's residuals, which are smaller) in the workspace.
size_t route_part_bytes(int T, int N_r, int ks) { return (size_t)ks * T * N_r * sizeof(float); }
size_t route_part_offset(int d, int N_r) { return (planes_bytes(d, N_r) + 255) / 256 * 256; }
// Whether the routing kernel routes after the GEMM (when the workspace and
// the shape allow): for K-split batches and for two CTAs splitting the
// experts, where it measured faster than the epilogue (DeepSeek-V3 prefill
// 85 -> 64 us, Kimi K2 prefill 150.5 -> 138 us); one CTA per tile keeps its
// epilogue (the full batch: 161 us against 165-169 us with the routing
// kernel).  MR_ROUTE_KERNEL=0 never, =1 for every shape (the tests and
// measurements pin both).
bool route_after_gemm(const TcShape& shp) {
  if (const char* env = getenv("MR_ROUTE_KERNEL")) {
    if (env[0] == '0') return false;
    if (env[0] == '1') return true;
  }
  return shp.ks > 1 || shp.CS > 1;
}
float* route_part(void* ws, size_t ws_bytes, int d, int N_r) {
  const size_t off = route_part_offset(d, N_r);
  return ws && aligned16(ws) && ws_bytes > off
             ? reinterpret_cast<float*>(static_cast<char*>(ws) + off)
             : nullptr;
}
size_t route_part_cap(void* ws, size_t ws_bytes, int d, int N_r) {
  return route_part(ws, ws_bytes, d, N_r) ? ws_bytes - route_part_offset(d, N_r) : 0;
}

// x fp32 with tf32 arithmetic (use3x: 3xTF32), or x bf16 with W as three
// bf16 planes (bf16x3, planes written into `ws` here), or x bf16 with W
// stored in bf16 (wbf16 non-null: one plane, W itself, no split).
int launch_tc(const void* x, const float* W, const float* bias, int T, int d, int N_r,
              int n_group, int topk_group, int k, float route_scale, int mask_mode, int flags,
              bool use3x, bool bf16x3, int32_t* idx_out, float* w_out, float* logits_out,
              float* wlo, void* ws, int sms, cudaStream_t st, const void* wbf16 = nullptr,
              float* part = nullptr, size_t part_cap = 0) {
  const int nplanes = wbf16 ? 1 : 3;
  const int num_kc = (d + mr::tc::BK - 1) / mr::tc::BK;
  TcShape shp = tc_shape(T, N_r, sms, bf16x3, num_kc);
  auto fits = [&](const TcShape& t) {
    const mr::tc::Plan p = mr::tc::make_plan(N_r / t.CS, bf16x3, t.pair, nplanes, n_group);
    const uint32_t xk = t.ks > 1 ? (uint32_t)mr::tc::BM * (N_r + 4) * 4 : 0;  // K-split partials
    return p.stages >= 2 && xk <= p.bar_off;
  };
  if (!fits(shp) && (shp.pair || shp.ks > 1)) shp = {1, false, 1};  // a pair's ring is half
  if (!fits(shp)) return MR_ERR_UNSUPPORTED;
  const int CS = shp.CS;
  const bool pair = shp.pair;
  const int NL = N_r / CS;
  const mr::tc::Plan plan = mr::tc::make_plan(NL, bf16x3, pair, nplanes, n_group);
  CUtensorMap mx, mw, mwlo;
  const bool use_wlo = !bf16x3 && use3x && wlo != nullptr;
  if (bf16x3) {
    const void* planes = wbf16;
    if (!wbf16) {
      const long n = (long)N_r * d;
      mr::tc::split_planes_kernel<<<(unsigned)std::min<long>((n / 8 + 255) / 256 + 1,
                                                             (long)sms * 8),
                                    256, 0, st>>>(W, static_cast<__nv_bfloat16*>(ws), n);
      if (launch_status() != MR_OK) return MR_ERR_CUDA;
      planes = ws;
    }
    if (!make_map_bf16(&mx, x, (uint64_t)T, (uint64_t)d, mr::tc::BM)) return MR_ERR_CUDA;
    if (!make_map_bf16(&mw, planes, (uint64_t)nplanes * N_r, (uint64_t)d, pair ? NL / 2 : NL))
      return MR_ERR_CUDA;
    mwlo = mw;
  } else {
    if (!make_map_f32(&mx, static_cast<const float*>(x), (uint64_t)T, (uint64_t)d, mr::tc::BM,
                      mr::tc::BK))
      return MR_ERR_CUDA;
    if (!make_map_f32(&mw, W, (uint64_t)N_r, (uint64_t)d, NL, mr::tc::BK)) return MR_ERR_CUDA;
  }
  if (use_wlo) {
    const long n4 = (long)N_r * d / 4;
    mr::tc::split_residual_kernel<<<(unsigned)std::min<long>((n4 + 255) / 256, (long)sms * 8), 256,
                                    0, st>>>(reinterpret_cast<const float4*>(W),
                                             reinterpret_cast<float4*>(wlo), n4);
    if (launch_status() != MR_OK) return MR_ERR_CUDA;
    if (!make_map_f32(&mwlo, wlo, (uint64_t)N_r, (uint64_t)d, NL, mr::tc::BK)) return MR_ERR_CUDA;
  } else if (!bf16x3) {
    mwlo = mw;
  }
  mr::tc::Params P;
  P.T = T;
  P.d = d;
  P.N = N_r;
  P.NL = NL;
  P.CS = CS;
  P.n_group = n_group;
  P.topk_group = topk_group;
  P.k = k;
  P.mask_mode = mask_mode;
  P.flags = flags;
  P.num_kc = (d + mr::tc::BK - 1) / mr::tc::BK;
  P.use3x = use3x ? 1 : 0;
  P.wlo = use_wlo ? 1 : 0;
  P.bf16x3 = bf16x3 ? 1 : 0;
  P.pair = pair ? 1 : 0;
  P.ksplit = shp.ks;
  P.route_scale = route_scale;
  P.bias = bias;
  P.idx_out = idx_out;
  P.w_out = w_out;
  P.logits_out = logits_out;
  // After the GEMM (route_after_gemm): when the workspace holds the logits
  // (the ks partial sums of a K split) and the shape fits the routing
  // kernel's layout, the CTAs write them and the routing kernel adds the
  // slices and routes (instead of the exchanges through distributed shared
  // memory and the epilogue); MR_ROUTE_LANES=8, 16 or 32 pins the lanes per
  // token (the tests use it).
  int lanes = 0;
  // (the rows are staged in the ring: [128][NL + 4] fp32 must fit in it)
  if (part && !pair && part_cap >= route_part_bytes(T, N_r, shp.ks) &&
      (size_t)mr::tc::BM * (NL + 4) * 4 <= (size_t)plan.bar_off &&
      route_after_gemm(shp)) {
    const char* pin = getenv("MR_ROUTE_LANES");
    lanes = mr::rt::lanes_per_token(T, N_r, n_group, k, sms, pin ? atoi(pin) : 0);
  }
  P.part = lanes ? part : nullptr;
  const size_t smem = plan.total + 1024;
  const bool sm = (flags & MR_SCORE_SOFTMAX) != 0;
  using mr::tc::router_tc_kernel;
  // the K-split instantiation (never with a pair) also writes the logits for
  // the routing kernel
  const bool ksk = shp.ks > 1 || lanes > 0;
  auto kern =
      nplanes == 1
          ? (pair ? (sm ? router_tc_kernel<true, true, 1> : router_tc_kernel<true, false, 1>)
                  : ksk ? (sm ? router_tc_kernel<false, true, 1, true>
                              : router_tc_kernel<false, false, 1, true>)
                        : (sm ? router_tc_kernel<false, true, 1> : router_tc_kernel<false, false, 1>))
          : (pair ? (sm ? router_tc_kernel<true, true, 3> : router_tc_kernel<true, false, 3>)
                  : ksk ? (sm ? router_tc_kernel<false, true, 3, true>
                              : router_tc_kernel<false, false, 3, true>)
                        : (sm ? router_tc_kernel<false, true, 3> : router_tc_kernel<false, false, 3>));
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MR_ERR_CUDA;
  unsigned tiles = (unsigned)((T + mr::tc::BM - 1) / mr::tc::BM);
  if (pair) tiles = (tiles + 1) / 2 * 2;  // a pair's second tile may be past T
  const unsigned cluster = (CS > 1 || pair) ? 2u : (unsigned)shp.ks;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles * CS * shp.ks);
  cfg.blockDim = dim3(mr::tc::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent of the preceding kernel (the W split): the router
  // CTAs set up while it runs, then wait for it (griddepcontrol.wait)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mx, mw, mwlo, P);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return MR_ERR_CUDA;
  }
  if (launch_status() != MR_OK) return MR_ERR_CUDA;
  if (!lanes) return MR_OK;
  mr::rt::Params rp;
  rp.part = part;
  rp.KS = shp.ks;
  rp.T = T;
  rp.N = N_r;
  rp.P = lanes;
  rp.n_group = n_group;
  rp.topk_group = topk_group;
  rp.k = k;
  rp.mask_mode = mask_mode;
  rp.flags = flags;
  rp.route_scale = route_scale;
  rp.bias = bias;
  rp.idx_out = idx_out;
  rp.w_out = w_out;
  rp.logits_out = logits_out;
  return launch_route(rp, st);
}

// ---- the plain router's split-K partials --------------------------------------
//
// mr_router_forward has no workspace argument, so its small-batch (split-K)
// path keeps the partial logits in a fixed array of the library's device image
// (every device that loads the library holds one copy until the process
// exits).  Host code may not use the symbol as a pointer: its device address
// is looked up per device, with that device current, and only a successful
// lookup is kept.  All calls on a device share the array; the library orders
// them across streams with one event per device (each use waits for the
// previous use's event and records its own), except inside stream capture,
// where it adds no dependency.
constexpr size_t kRouterScratchBytes = size_t(2) << 20;
static __device__ __align__(256) float g_router_scratch[kRouterScratchBytes / sizeof(float)];

std::atomic<float*> g_router_scratch_ptr[kMaxDevices];
std::mutex g_router_scratch_mu[kMaxDevices];
cudaEvent_t g_router_scratch_done[kMaxDevices];

float* router_scratch(int dev) {
  float* p = g_router_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_router_scratch_mu[dev]);
  p = g_router_scratch_ptr[dev].load(std::memory_order_relaxed);
  if (p) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_router_scratch) != cudaSuccess || !addr) {
    (void)cudaGetLastError();
    return nullptr;
  }
  p = static_cast<float*>(addr);
  g_router_scratch_ptr[dev].store(p, std::memory_order_release);
  return p;
}

// One use of the array on `s`: holds the device's lock, makes `s` wait for
// the previous use (outside stream capture), and records this use's event.
class RouterScratchUse {
 public:
  RouterScratchUse(int dev, cudaStream_t s) : dev_(dev), s_(s), lock_(g_router_scratch_mu[dev]) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) {
      (void)cudaGetLastError();
      cap = cudaStreamCaptureStatusActive;  // unknown: add no event
    }
    order_ = cap == cudaStreamCaptureStatusNone;
    if (!order_) return;
    if (!g_router_scratch_done[dev] &&
        cudaEventCreateWithFlags(&g_router_scratch_done[dev], cudaEventDisableTiming) !=
            cudaSuccess) {
      g_router_scratch_done[dev] = nullptr;
      ok_ = false;
      return;
    }
    ok_ = cudaStreamWaitEvent(s, g_router_scratch_done[dev], 0) == cudaSuccess;
  }
  bool ok() const { return ok_; }
  int done(int status) {
    if (order_ && cudaEventRecord(g_router_scratch_done[dev_], s_) != cudaSuccess)
      return MR_ERR_CUDA;
    return status;
  }

 private:
  int dev_;
  cudaStream_t s_;
  std::lock_guard<std::mutex> lock_;
  bool order_ = false, ok_ = true;
};

// Bounded-wait self test (see mr_selftest_bounded_wait).
__global__ void selftest_mbar_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_s;
  if (threadIdx.x == 0) {
    abort_s = 0;
    mr::tc::mbar_init(mr::tc::smem_u32(&bar), 1);  // nothing ever arrives
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mr::tc::mbar_wait(mr::tc::smem_u32(&bar), 0, &abort_s);  // gives up, raises the flag
  }
}

// Arrival counter of the grid-barrier self test: a word in the library's
// device image (no allocation); the kernel clears it before arriving.
__device__ int g_selftest_counter = 0;

__global__ void selftest_grid_barrier_kernel() {
  // only CTA 0 arrives; its target counts two CTAs
  if (threadIdx.x == 0) {
    atomicExch(&g_selftest_counter, 0);
    __threadfence();
  }
  __syncthreads();
  mr::disp_grid_barrier(&g_selftest_counter, 2);
}

}  // namespace

extern "C" {

int mr_selftest_bounded_wait(int which, mr_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (which == 0) {
    selftest_mbar_wait_kernel<<<1, 32, 0, s>>>();
    return launch_status();
  }
  if (which == 1) {
    selftest_grid_barrier_kernel<<<1, 32, 0, s>>>();
    return launch_status();
  }
  return MR_ERR_INVALID_ARG;
}


int mr_version(void) { return 100; }

const char* mr_status_string(int status) {
  switch (status) {
    case MR_OK: return "ok";
    case MR_ERR_INVALID_ARG: return "invalid argument";
    case MR_ERR_UNSUPPORTED: return "unsupported shape, option or device";
    case MR_ERR_CUDA: return "CUDA launch or query failed";
    case MR_ERR_DEVICE: return "device flag: expert id out of range or inconsistent counts";
    case MR_ERR_TIMEOUT: return "device flag: bounded wait timed out";
    case MR_ERR_OVERFLOW: return "device flag: rows past a receive buffer's capacity dropped";
    default: return "unknown status";
  }
}

size_t mr_router_workspace_size(int T, int d, int N_r) {
  if (T <= 0 || d <= 0 || N_r <= 0 || N_r > 512) return 0;
  size_t need = planes_bytes(d, N_r);  // >= W residuals (fp32 x, fused path)
  {
    // then, for a K-split batch, the partial sums for the routing kernel
    int sms = 0, cc = 0;
    if (!device_info(&sms, &cc)) return 0;
    const TcShape shp = tc_shape(T, N_r, sms, true, (d + mr::tc::BK - 1) / mr::tc::BK);
    if (route_after_gemm(shp))
      need = route_part_offset(d, N_r) + route_part_bytes(T, N_r, shp.ks);
  }
  if (splitk_applies(T, N_r)) {
    int sms = 0, cc = 0;
    if (!device_info(&sms, &cc)) return 0;
    need = std::max(need, std::max(splitk_shape(T, d, N_r, sms, false).ws_bytes,
                                   splitk_shape(T, d, N_r, sms, true).ws_bytes));
    need = std::max(need, splitk_shape(T, d, N_r, sms, true, true).ws_bytes);
  }
  return need;
}

int mr_router_forward_ex2(const void* x, int x_dtype, const float* W, const float* bias, int T,
                          int d, int N_r, int n_group, int topk_group, int k, float route_scale,
                          int mask_mode, int precision, int flags, int32_t* idx_out,
                          float* w_out, float* logits_out, void* workspace,
                          size_t workspace_bytes, mr_stream_t stream) {
  if (flags & ~(MR_SCORE_SOFTMAX | MR_GROUP_MAX | MR_NORM_NO_EPS)) return MR_ERR_INVALID_ARG;
  int st = validate_router(x, x_dtype, W, T, d, N_r, n_group, topk_group, k, route_scale,
                           mask_mode, precision, idx_out, w_out);
  if (st != MR_OK || T == 0) return st;
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (precision == MR_PREC_FFMA) {
    return x_dtype == MR_BF16
               ? launch_ffma<true>(x, W, bias, T, d, N_r, n_group, topk_group, k, route_scale,
                                   mask_mode, flags, idx_out, w_out, logits_out, s)
               : launch_ffma<false>(x, W, bias, T, d, N_r, n_group, topk_group, k, route_scale,
                                    mask_mode, flags, idx_out, w_out, logits_out, s);
  }
  // Small batches (decode): split-K over all SMs, fp32 W read directly, for
  // either row type (3xTF32; a bf16 row needs no residual).
  if (cc == 10 && workspace && aligned16(workspace) && splitk_applies(T, N_r) &&
      tc_shape_ok(x, MR_F32, W, d, N_r) && (x_dtype == MR_F32 || d % 8 == 0) &&
      !(precision == MR_PREC_BF16X3 && x_dtype != MR_BF16) &&
      workspace_bytes >= splitk_shape(T, d, N_r, sms, x_dtype == MR_BF16).ws_bytes)
    return launch_splitk(x, x_dtype == MR_BF16, W, bias, T, d, N_r, n_group, topk_group, k,
                         route_scale, mask_mode, flags, precision != MR_PREC_TF32, idx_out, w_out,
                         logits_out, workspace, sms, s);
  if (x_dtype == MR_BF16 || precision == MR_PREC_BF16X3) {
    // bf16 activations on tensor cores: W as three bf16 planes (workspace)
    if (x_dtype != MR_BF16 || precision == MR_PREC_TF32 || cc != 10 || d % 8 != 0 ||
        !tc_shape_ok(x, MR_F32, W, d, N_r) || !workspace || !aligned16(workspace) ||
        workspace_bytes < planes_bytes(d, N_r))
      return MR_ERR_UNSUPPORTED;
    return launch_tc(x, W, bias, T, d, N_r, n_group, topk_group, k, route_scale, mask_mode, flags,
                     true, true, idx_out, w_out, logits_out, nullptr, workspace, sms, s, nullptr,
                     route_part(workspace, workspace_bytes, d, N_r),
                     route_part_cap(workspace, workspace_bytes, d, N_r));
  }
  if (cc != 10 || !tc_shape_ok(x, x_dtype, W, d, N_r)) return MR_ERR_UNSUPPORTED;
  float* wlo = (workspace && aligned16(workspace) && workspace_bytes >= wlo_bytes(d, N_r))
                   ? static_cast<float*>(workspace)
                   : nullptr;
  return launch_tc(x, W, bias, T, d, N_r, n_group, topk_group, k, route_scale, mask_mode, flags,
                   precision == MR_PREC_3XTF32, false, idx_out, w_out, logits_out, wlo, nullptr,
                   sms, s, nullptr, route_part(workspace, workspace_bytes, d, N_r),
                   route_part_cap(workspace, workspace_bytes, d, N_r));
}

int mr_router_forward_ex(const void* x, int x_dtype, const float* W, const float* bias, int T,
                         int d, int N_r, int n_group, int topk_group, int k, float route_scale,
                         int mask_mode, int precision, int32_t* idx_out, float* w_out,
                         float* logits_out, void* workspace, size_t workspace_bytes,
                         mr_stream_t stream) {
  return mr_router_forward_ex2(x, x_dtype, W, bias, T, d, N_r, n_group, topk_group, k,
                               route_scale, mask_mode, precision, 0, idx_out, w_out, logits_out,
                               workspace, workspace_bytes, stream);
}

int mr_router_forward(const float* x, const float* W, const float* bias, int T, int d, int N_r,
                      int n_group, int topk_group, int k, float route_scale, int mask_mode,
                      int32_t* idx_out, float* w_out, mr_stream_t stream) {
  int st = validate_router(x, MR_F32, W, T, d, N_r, n_group, topk_group, k, route_scale,
                           mask_mode, MR_PREC_3XTF32, idx_out, w_out);
  if (st != MR_OK || T == 0) return st;
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  const bool tc = cc == 10 && tc_shape_ok(x, MR_F32, W, d, N_r);
  // Small batches (decode): the split-K path, its partial logits in the
  // library's own array (this entry point takes no workspace).
  if (tc && splitk_applies(T, N_r) &&
      splitk_shape(T, d, N_r, sms, false).ws_bytes <= kRouterScratchBytes) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MR_ERR_CUDA;
    float* scratch = router_scratch(dev);
    if (!scratch) return MR_ERR_CUDA;
    RouterScratchUse use(dev, s);
    if (!use.ok()) return MR_ERR_CUDA;
    st = launch_splitk(x, false, W, bias, T, d, N_r, n_group, topk_group, k, route_scale,
                       mask_mode, 0, true, idx_out, w_out, nullptr, scratch, sms, s);
    return use.done(st);
  }
  return mr_router_forward_ex(x, MR_F32, W, bias, T, d, N_r, n_group, topk_group, k, route_scale,
                              mask_mode, tc ? MR_PREC_3XTF32 : MR_PREC_FFMA, idx_out, w_out,
                              nullptr, nullptr, 0, stream);
}

size_t mr_router_forward_max_scratch(void) { return kRouterScratchBytes; }

int mr_router_forward_bf16w(const void* x, int x_dtype, const void* W_bf16, const float* bias,
                            int T, int d, int N_r, int n_group, int topk_group, int k,
                            float route_scale, int mask_mode, int flags, int32_t* idx_out,
                            float* w_out, float* logits_out, void* workspace,
                            size_t workspace_bytes, mr_stream_t stream) {
  if (flags & ~(MR_SCORE_SOFTMAX | MR_GROUP_MAX | MR_NORM_NO_EPS)) return MR_ERR_INVALID_ARG;
  int st = validate_router(x, x_dtype, static_cast<const float*>(W_bf16), T, d, N_r, n_group,
                           topk_group, k, route_scale, mask_mode, MR_PREC_3XTF32, idx_out, w_out);
  if (st != MR_OK || T == 0) return st;
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool n_ok = N_r <= 256 ? (N_r % 16 == 0 && N_r >= 16) : (N_r % 32 == 0);
  const bool tc = cc == 10 && x_dtype == MR_BF16 && d % 8 == 0 && n_ok && aligned16(x) &&
                  aligned16(W_bf16);
  if (tc && splitk_applies(T, N_r)) {
    const size_t need = splitk_shape(T, d, N_r, sms, true, true).ws_bytes;
    if (workspace && aligned16(workspace) && workspace_bytes >= need)
      return launch_splitk(x, true, nullptr, bias, T, d, N_r, n_group, topk_group, k,
                           route_scale, mask_mode, flags, false, idx_out, w_out, logits_out,
                           workspace, sms, s, W_bf16);
    if (!workspace && need <= kRouterScratchBytes) {
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MR_ERR_CUDA;
      float* scratch = router_scratch(dev);
      if (!scratch) return MR_ERR_CUDA;
      RouterScratchUse use(dev, s);
      if (!use.ok()) return MR_ERR_CUDA;
      st = launch_splitk(x, true, nullptr, bias, T, d, N_r, n_group, topk_group, k, route_scale,
                         mask_mode, flags, false, idx_out, w_out, logits_out, scratch, sms, s,
                         W_bf16);
      return use.done(st);
    }
  }
  if (tc)
    return launch_tc(x, nullptr, bias, T, d, N_r, n_group, topk_group, k, route_scale, mask_mode,
                     flags, true, true, idx_out, w_out, logits_out, nullptr, nullptr, sms, s,
                     W_bf16);
  return x_dtype == MR_BF16
             ? launch_ffma<true, true>(x, W_bf16, bias, T, d, N_r, n_group, topk_group, k,
                                       route_scale, mask_mode, flags, idx_out, w_out, logits_out,
                                       s)
             : launch_ffma<false, true>(x, W_bf16, bias, T, d, N_r, n_group, topk_group, k,
                                        route_scale, mask_mode, flags, idx_out, w_out,
                                        logits_out, s);
}

// ---- dispatch -----------------------------------------------------------------

// Chunk histograms of the three-kernel dispatch: [nchunks][N_r] int32.
size_t disp_hist_bytes(int T, int k, int N_r) {
  return (size_t)mr::disp_num_chunks((long)T * k) * (size_t)N_r * sizeof(int32_t);
}

size_t mr_dispatch_workspace_size(int T, int k, int N_r) {
  if (T <= 0 || k <= 0 || N_r <= 0) return 0;
  // fused kernel: barrier counter (16 bytes), chunk histograms, expert totals
  return 16 + disp_hist_bytes(T, k, N_r) + (size_t)N_r * sizeof(int32_t);
}

int mr_dispatch(const int32_t* idx, int T, int k, int N_r, int32_t* counts, int32_t* offsets,
                int32_t* perm, int32_t* inv_perm, void* workspace, size_t workspace_bytes,
                mr_stream_t stream) {
  if (T < 0 || k <= 0 || N_r <= 0) return MR_ERR_INVALID_ARG;
  if ((long long)T * k >= (1LL << 31)) return MR_ERR_INVALID_ARG;
  if (k > 32 || N_r > mr::kDispMaxExperts) return MR_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MR_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * N_r, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (N_r + 1), s) != cudaSuccess)
      return MR_ERR_CUDA;
    return MR_OK;
  }
  if (!idx || !perm || !workspace) return MR_ERR_INVALID_ARG;
  if (workspace_bytes < mr_dispatch_workspace_size(T, k, N_r)) return MR_ERR_INVALID_ARG;
  const long n = (long)T * k;
  const long nchunks = mr::disp_num_chunks(n);
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  // One cooperative launch when every chunk's CTA can be resident at once.
  const size_t fsmem = sizeof(int) * std::max(mr::kDispThreads, mr::kDispWarps * N_r);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mr::dispatch_fused_kernel,
                                                    mr::kDispThreads, fsmem) != cudaSuccess)
    per_sm = 0;
  if ((long)per_sm * sms >= nchunks) {
    mr::DispFusedWs wsd;
    wsd.barrier = static_cast<int*>(workspace);
    wsd.hist = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + 16);
    wsd.totals = wsd.hist + nchunks * N_r;
    if (cudaMemsetAsync(wsd.barrier, 0, sizeof(int), s) != cudaSuccess) return MR_ERR_CUDA;
    void* args[] = {const_cast<int32_t**>(&idx), const_cast<long*>(&n), &N_r, &wsd, &counts,
                    &offsets, &perm, &inv_perm};
    const cudaError_t e = cudaLaunchCooperativeKernel(
        reinterpret_cast<const void*>(mr::dispatch_fused_kernel), dim3((unsigned)nchunks),
        dim3(mr::kDispThreads), args, fsmem, s);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return MR_ERR_CUDA;
    }
    return MR_OK;
  }
  int32_t* hist = static_cast<int32_t*>(workspace);
  mr::dispatch_count_kernel<<<(unsigned)nchunks, mr::kDispThreads, sizeof(int) * N_r, s>>>(
      idx, n, N_r, hist);
  if (launch_status() != MR_OK) return MR_ERR_CUDA;
  mr::dispatch_scan_kernel<<<1, 1024, 0, s>>>(hist, nchunks, N_r, n, counts, offsets, perm);
  if (launch_status() != MR_OK) return MR_ERR_CUDA;
  const size_t smem = sizeof(int) * mr::kDispWarps * N_r;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(mr::dispatch_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MR_ERR_CUDA;
  mr::dispatch_scatter_kernel<<<(unsigned)nchunks, mr::kDispThreads, smem, s>>>(idx, n, N_r, hist,
                                                                                perm, inv_perm);
  return launch_status();
}

// ---- dispatch without allocation ---------------------------------------------
//
// Scratch of mr_dispatch_noalloc: a fixed array in the library's device image.
// Every device that loads the library holds one copy until the process exits.
// Host code may not use the symbol as a pointer; its device address is looked
// up once per device (with that device current) by noalloc_scratch().
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;
static __device__ __align__(256) int32_t g_dispatch_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

std::atomic<int32_t*> g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device.  Only a
// successful lookup is cached: after a failed one (nullptr returned, the
// error cleared) the next call on that device tries again.
int32_t* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  int32_t* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  p = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
  if (p) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_dispatch_scratch) != cudaSuccess || !addr) {
    (void)cudaGetLastError();
    return nullptr;
  }
  p = static_cast<int32_t*>(addr);
  g_noalloc_ptr[dev].store(p, std::memory_order_release);
  return p;
}

size_t mr_dispatch_noalloc_max_workspace(void) { return kNoAllocScratchBytes; }

int mr_dispatch_noalloc(const int32_t* idx, int T, int k, int N_r, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv_perm, mr_stream_t stream) {
  if (T < 0 || k <= 0 || N_r <= 0) return MR_ERR_INVALID_ARG;
  if ((long long)T * k >= (1LL << 31)) return MR_ERR_INVALID_ARG;
  if (k > 32 || N_r > mr::kDispMaxExperts) return MR_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MR_ERR_INVALID_ARG;
  if (disp_hist_bytes(T, k, N_r) > kNoAllocScratchBytes) return MR_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * N_r, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (N_r + 1), s) != cudaSuccess)
      return MR_ERR_CUDA;
    return MR_OK;
  }
  if (!idx || !perm) return MR_ERR_INVALID_ARG;
  int32_t* hist = noalloc_scratch();
  if (!hist) return MR_ERR_CUDA;
  // Same kernels as mr_dispatch.  The count kernel writes every histogram
  // entry the later kernels read, so the scratch needs no clearing.
  const long n = (long)T * k;
  const long nchunks = mr::disp_num_chunks(n);
  mr::dispatch_count_kernel<<<(unsigned)nchunks, mr::kDispThreads, sizeof(int) * N_r, s>>>(
      idx, n, N_r, hist);
  if (launch_status() != MR_OK) return MR_ERR_CUDA;
  mr::dispatch_scan_kernel<<<1, 1024, 0, s>>>(hist, nchunks, N_r, n, counts, offsets, perm);
  if (launch_status() != MR_OK) return MR_ERR_CUDA;
  const size_t smem = sizeof(int) * mr::kDispWarps * N_r;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(mr::dispatch_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MR_ERR_CUDA;
  mr::dispatch_scatter_kernel<<<(unsigned)nchunks, mr::kDispThreads, smem, s>>>(idx, n, N_r, hist,
                                                                                perm, inv_perm);
  return launch_status();
}

// ---- expert-parallel receive order ------------------------------------------

int mr_ep_recv_order(const int32_t* recv_counts, int ep, int E_loc, int R, int32_t* order,
                     int32_t* inv_order, int32_t* local_counts, int32_t* local_offsets,
                     mr_stream_t stream) {
  if (ep <= 0 || E_loc <= 0 || R < 0) return MR_ERR_INVALID_ARG;
  if ((long)ep * E_loc > mr::kEpMaxSegments) return MR_ERR_UNSUPPORTED;
  if (!recv_counts || !local_counts || !local_offsets || (R > 0 && !order))
    return MR_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)std::max<long>(1, ((long)R + mr::kEpRowsPerCta - 1) /
                                                        mr::kEpRowsPerCta);
  mr::ep_recv_order_kernel<<<grid, mr::kEpThreads, 0, s>>>(recv_counts, ep, E_loc, R, order,
                                                            inv_order, local_counts,
                                                            local_offsets);
  return launch_status();
}

// ---- expert layer with the row gather fused in -------------------------------

}  // extern "C"

namespace {

// Shared by the plain and the packed-weight entry points.
// wts/acc non-null: the combine epilogue (router weights by slot, the
// zeroed fp32 [T, n_out] accumulator) instead of writing `out`.
int launch_expert_gemm(const void* x, const int32_t* perm, const int32_t* offsets,
                       const void* W, bool packed, int T, int d, int k, int N_r, int n_out,
                       void* out, cudaStream_t s, const float* wts = nullptr,
                       float* acc = nullptr) {
  if (T < 0 || d <= 0 || k <= 0 || N_r <= 0 || n_out <= 0) return MR_ERR_INVALID_ARG;
  if ((long long)T * k >= (1LL << 31) || (long long)N_r * n_out >= (1LL << 31))
    return MR_ERR_INVALID_ARG;
  if (T == 0) return MR_OK;
  const bool combine = acc != nullptr;
  if (!x || !offsets || !W || (!combine && !out) || (combine && (!wts || !perm)))
    return MR_ERR_INVALID_ARG;
  const bool gather = perm != nullptr;  // NULL: x already holds the sorted rows
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  if (cc != 10 || d % 8 != 0 || n_out % 16 != 0 || N_r > mr::kDispMaxExperts ||
      !aligned16(x) || !aligned16(W) || (combine ? !aligned16(acc) : !aligned16(out)))
    return MR_ERR_UNSUPPORTED;
  auto enc = tensor_map_encoder();
  if (!enc) return MR_ERR_CUDA;
  // K chunk: 64 bf16 (128-byte rows) unless MR_EG_BK=32 pins 32 (64-byte
  // rows); the packed layout always has 64-column tiles
  const char* bk_env = getenv("MR_EG_BK");
  const int bke = (!packed && bk_env && bk_env[0] == '3') ? 32 : 64;
  const CUtensorMapSwizzle sw = bke == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const int NT = (n_out + mr::eg::kBN - 1) / mr::eg::kBN;
  const int KC64 = (d + 63) / 64;
  CUtensorMap mx, mw;
  {
    // token rows, one-row boxes: each tile::gather4 copy fetches four of them;
    // without perm, the [T*k, d] sorted rows in 128-row boxes
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)(gather ? T : (long)T * k)};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {(cuuint32_t)bke, gather ? 1u : (cuuint32_t)mr::tc::BM};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MR_ERR_CUDA;
  }
  {
    // nn.Linear layout [N_r * n_out, d], or the packed blocks as [rows, 64]
    const cuuint64_t cols = packed ? 64 : (cuuint64_t)d;
    const cuuint64_t rows =
        packed ? (cuuint64_t)N_r * NT * KC64 * mr::eg::kBN : (cuuint64_t)N_r * n_out;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)bke, (cuuint32_t)mr::eg::kBN};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MR_ERR_CUDA;
  }
  mr::eg::Params P;
  P.T = T;
  P.d = d;
  P.k = k;
  P.N_r = N_r;
  P.n_out = n_out;
  P.perm = perm;
  P.offsets = offsets;
  P.x = x;
  P.w_packed = packed ? static_cast<const __nv_bfloat16*>(W) : nullptr;
  P.out = static_cast<__nv_bfloat16*>(out);
  P.wts = wts;
  P.acc = acc;
  // gathered rows: copied by the four epilogue warps (cp.async, 64-wide K
  // chunks) unless MR_EG_GATHER=tma pins the TMA tile::gather4 copies
  const char* g_env = getenv("MR_EG_GATHER");
  const bool tma_gather = bke == 32 || (g_env && g_env[0] == 't');
  using namespace mr::eg;
  auto kern = combine ? (tma_gather
                            ? (packed ? expert_gemm_gather_kernel<64, true, kGatherTma, true>
                                      : (bke == 32
                                             ? expert_gemm_gather_kernel<32, false, kGatherTma, true>
                                             : expert_gemm_gather_kernel<64, false, kGatherTma, true>))
                            : (packed ? expert_gemm_gather_kernel<64, true, kGatherLsu, true>
                                      : expert_gemm_gather_kernel<64, false, kGatherLsu, true>))
            : !gather ? (packed ? expert_gemm_gather_kernel<64, true, kRowsSorted>
                                : (bke == 32 ? expert_gemm_gather_kernel<32, false, kRowsSorted>
                                             : expert_gemm_gather_kernel<64, false, kRowsSorted>))
            : tma_gather
                ? (packed ? expert_gemm_gather_kernel<64, true, kGatherTma>
                          : (bke == 32 ? expert_gemm_gather_kernel<32, false, kGatherTma>
                                       : expert_gemm_gather_kernel<64, false, kGatherTma>))
                : (packed ? expert_gemm_gather_kernel<64, true, kGatherLsu>
                          : expert_gemm_gather_kernel<64, false, kGatherLsu>);
  const size_t smem = bke == 32 ? mr::eg::EgPlan<32>::kSmemBytes : mr::eg::EgPlan<64>::kSmemBytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MR_ERR_CUDA;
  // at most ceil(T*k / 128) + N_r blocks of 128 sorted rows; surplus CTAs exit
  const unsigned gx = (unsigned)(((long)T * k + mr::tc::BM - 1) / mr::tc::BM + N_r);
  kern<<<dim3(gx, (unsigned)NT), mr::eg::kThreads, smem, s>>>(mx, mw, P);
  return launch_status();
}

}  // namespace

extern "C" {

int mr_expert_gemm_gather(const void* x, const int32_t* perm, const int32_t* offsets,
                          const void* W_exp, int T, int d, int k, int N_r, int n_out, void* out,
                          mr_stream_t stream) {
  return launch_expert_gemm(x, perm, offsets, W_exp, false, T, d, k, N_r, n_out, out,
                            reinterpret_cast<cudaStream_t>(stream));
}

size_t mr_expert_packed_bytes(int N_r, int n_out, int d) {
  if (N_r <= 0 || n_out <= 0 || d <= 0) return 0;
  return (size_t)N_r * ((n_out + 255) / 256) * ((d + 63) / 64) * 256 * 64 * 2;
}

int mr_expert_pack_weights(const void* W_exp, int N_r, int n_out, int d, void* W_packed,
                           size_t packed_bytes, mr_stream_t stream) {
  if (N_r <= 0 || n_out <= 0 || d <= 0 || !W_exp || !W_packed) return MR_ERR_INVALID_ARG;
  if (packed_bytes < mr_expert_packed_bytes(N_r, n_out, d)) return MR_ERR_INVALID_ARG;
  if (d % 8 != 0 || !aligned16(W_exp) || !aligned16(W_packed)) return MR_ERR_UNSUPPORTED;
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  const int NT = (n_out + 255) / 256, KC = (d + 63) / 64;
  const long n_vec = (long)(mr_expert_packed_bytes(N_r, n_out, d) / 16);
  const unsigned grid = (unsigned)std::min<long>((n_vec + 255) / 256, (long)sms * 16);
  mr::eg::expert_pack_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(W_exp), static_cast<uint4*>(W_packed), n_out, d, NT, KC, n_vec);
  return launch_status();
}

int mr_expert_gemm_gather_packed(const void* x, const int32_t* perm, const int32_t* offsets,
                                 const void* W_packed, int T, int d, int k, int N_r, int n_out,
                                 void* out, mr_stream_t stream) {
  return launch_expert_gemm(x, perm, offsets, W_packed, true, T, d, k, N_r, n_out, out,
                            reinterpret_cast<cudaStream_t>(stream));
}

int mr_expert_gemm_gather_combine(const void* x, const int32_t* perm, const int32_t* offsets,
                                  const void* W, int w_packed, const float* w,
                                  const void* shared, int T, int d, int k, int N_r, int n_out,
                                  float* acc, void* y, mr_stream_t stream) {
  if (T < 0 || d <= 0 || k <= 0 || N_r <= 0 || n_out <= 0 || (w_packed != 0 && w_packed != 1))
    return MR_ERR_INVALID_ARG;
  if ((long long)T * n_out >= (1LL << 40)) return MR_ERR_INVALID_ARG;
  if (T == 0) return MR_OK;
  if (!x || !perm || !offsets || !W || !w || !acc || !y) return MR_ERR_INVALID_ARG;
  if (n_out % 16 != 0 || !aligned16(acc) || !aligned16(y) || (shared && !aligned16(shared)))
    return MR_ERR_UNSUPPORTED;
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long n = (long)T * n_out;
  if (cudaMemsetAsync(acc, 0, (size_t)n * sizeof(float), s) != cudaSuccess) return MR_ERR_CUDA;
  const int rc = launch_expert_gemm(x, perm, offsets, W, w_packed != 0, T, d, k, N_r, n_out,
                                    nullptr, s, w, acc);
  if (rc != MR_OK) return rc;
  const long n8 = n / 8;
  const unsigned grid = (unsigned)std::min<long>((n8 + 255) / 256, (long)sms * 16);
  mr::eg::combine_acc_finalize_kernel<<<grid, 256, 0, s>>>(
      reinterpret_cast<const float4*>(acc), static_cast<const uint4*>(shared),
      static_cast<uint4*>(y), n8);
  return launch_status();
}

}  // extern "C"

namespace {

// The combine kernel for the row type: 32-byte vectors for bf16 rows when
// kVec32 and `vec32`, 16-byte vectors (bf16 or fp32) when `vec`, elements
// otherwise.  make_src(V* tag) builds the slot-row policy over the element or
// vector type V.
template <bool kVec32, typename MakeSrc>
int launch_combine(bool vec, bool vec32, bool bf16, unsigned grid, cudaStream_t s,
                   const float* w, const void* shared, void* y, long T, long d, int k,
                   MakeSrc make_src) {
  if constexpr (kVec32) {
    if (vec32 && bf16) {
      auto src = make_src(static_cast<mr::Vec32*>(nullptr));
      mr::combine_bf16_vec_kernel<<<grid, mr::kRowThreads, 0, s>>>(
          src, w, static_cast<const mr::Vec32*>(shared), static_cast<mr::Vec32*>(y), T, d / 16,
          k);
      return launch_status();
    }
  }
  if (vec && bf16) {
    auto src = make_src(static_cast<uint4*>(nullptr));
    mr::combine_bf16_vec_kernel<<<grid, mr::kRowThreads, 0, s>>>(
        src, w, static_cast<const uint4*>(shared), static_cast<uint4*>(y), T, d / 8, k);
  } else if (vec) {
    auto src = make_src(static_cast<float4*>(nullptr));
    mr::combine_f32_vec_kernel<<<grid, mr::kRowThreads, 0, s>>>(
        src, w, static_cast<const float4*>(shared), static_cast<float4*>(y), T, d / 4, k);
  } else if (bf16) {
    auto src = make_src(static_cast<uint16_t*>(nullptr));
    mr::combine_scalar_kernel<true><<<grid, mr::kRowThreads, 0, s>>>(src, w, shared, y, T, d, k);
  } else {
    auto src = make_src(static_cast<float*>(nullptr));
    mr::combine_scalar_kernel<false><<<grid, mr::kRowThreads, 0, s>>>(src, w, shared, y, T, d, k);
  }
  return launch_status();
}

}  // namespace

extern "C" {

// ---- gather / combine -------------------------------------------------------

int mr_gather_rows(const void* x, int dtype, int T, int d, int k, const int32_t* perm,
                   const int32_t* inv_perm, void* xs, mr_stream_t stream) {
  if (T < 0 || d <= 0 || k <= 0 || (dtype != MR_F32 && dtype != MR_BF16)) return MR_ERR_INVALID_ARG;
  if ((long long)T * k >= (1LL << 31)) return MR_ERR_INVALID_ARG;
  if (k > mr::kRowMaxK) return MR_ERR_UNSUPPORTED;
  if (T == 0) return MR_OK;
  if (!x || !xs || (!perm && !inv_perm)) return MR_ERR_INVALID_ARG;
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long esz = dtype == MR_BF16 ? 2 : 4;
  const long row_bytes = (long)d * esz;
  const bool vec = row_bytes % 16 == 0 && aligned16(x) && aligned16(xs);
  const bool vec32 = row_bytes % 32 == 0 && aligned32(x) && aligned32(xs);
  const long rows = (long)T * k;
  // one CTA per token: measured 353 us on the full DeepSeek-V3 batch against
  // 366 us for a grid-stride over 32 CTAs per SM
  const unsigned grid_t = (unsigned)std::min<long>(T, 1L << 30);
  const unsigned grid_r = (unsigned)std::min<long>(rows, (long)sms * 32);
  if (inv_perm) {
    if (vec32)
      mr::gather_inv_kernel<mr::Vec32><<<grid_t, mr::kRowThreads, 0, s>>>(
          static_cast<const mr::Vec32*>(x), T, row_bytes / 32, k,
          mr::SlotRowsLocal<mr::Vec32>{static_cast<mr::Vec32*>(xs), inv_perm});
    else if (vec)
      mr::gather_inv_kernel<uint4><<<grid_t, mr::kRowThreads, 0, s>>>(
          static_cast<const uint4*>(x), T, row_bytes / 16, k,
          mr::SlotRowsLocal<uint4>{static_cast<uint4*>(xs), inv_perm});
    else if (esz == 4)
      mr::gather_inv_kernel<uint32_t><<<grid_t, mr::kRowThreads, 0, s>>>(
          static_cast<const uint32_t*>(x), T, d, k,
          mr::SlotRowsLocal<uint32_t>{static_cast<uint32_t*>(xs), inv_perm});
    else
      mr::gather_inv_kernel<uint16_t><<<grid_t, mr::kRowThreads, 0, s>>>(
          static_cast<const uint16_t*>(x), T, d, k,
          mr::SlotRowsLocal<uint16_t>{static_cast<uint16_t*>(xs), inv_perm});
  } else {
    if (vec)
      mr::gather_perm_kernel<uint4><<<grid_r, mr::kRowThreads, 0, s>>>(
          static_cast<const uint4*>(x), rows, row_bytes / 16, k, perm, static_cast<uint4*>(xs));
    else if (esz == 4)
      mr::gather_perm_kernel<uint32_t><<<grid_r, mr::kRowThreads, 0, s>>>(
          static_cast<const uint32_t*>(x), rows, d, k, perm, static_cast<uint32_t*>(xs));
    else
      mr::gather_perm_kernel<uint16_t><<<grid_r, mr::kRowThreads, 0, s>>>(
          static_cast<const uint16_t*>(x), rows, d, k, perm, static_cast<uint16_t*>(xs));
  }
  return launch_status();
}

int mr_combine(const void* expert_out, int dtype, const float* w, const int32_t* inv_perm,
               const void* shared, void* y, int T, int d, int k, mr_stream_t stream) {
  if (T < 0 || d <= 0 || k <= 0 || (dtype != MR_F32 && dtype != MR_BF16)) return MR_ERR_INVALID_ARG;
  if ((long long)T * k >= (1LL << 31)) return MR_ERR_INVALID_ARG;
  if (k > mr::kRowMaxK) return MR_ERR_UNSUPPORTED;
  if (T == 0) return MR_OK;
  if (!expert_out || !w || !inv_perm || !y) return MR_ERR_INVALID_ARG;
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long esz = dtype == MR_BF16 ? 2 : 4;
  const long row_bytes = (long)d * esz;
  const bool vec = row_bytes % 16 == 0 && aligned16(expert_out) && aligned16(y) &&
                   (!shared || aligned16(shared));
  const bool vec32 = row_bytes % 32 == 0 && aligned32(expert_out) && aligned32(y) &&
                     (!shared || aligned32(shared));
  // grid-stride: 16 CTAs per SM with 32-byte vectors (360.5 us on the full
  // DeepSeek-V3 batch against 362.5 us with 64 and 364.5 us with 4 or 32 per
  // SM), 64 with 16-byte vectors (369 us; 372 us with 32 per SM)
  const long per_sm = vec32 && dtype == MR_BF16 ? 16 : 64;
  const unsigned grid = (unsigned)std::min<long>(T, (long)sms * per_sm);
  return launch_combine<true>(vec, vec32, dtype == MR_BF16, grid, s, w, shared, y, T, d, k,
                              [&](auto* tag) {
                                using V = std::remove_const_t<std::remove_pointer_t<decltype(tag)>>;
                                return mr::SlotRowsLocal<const V>{
                                    static_cast<const V*>(expert_out), inv_perm};
                              });
}

// ---- expert parallelism over peer memory ------------------------------------

int mr_ep_dispatch_p2p(const void* x, int dtype, int T, int d, int k, const int32_t* idx,
                       const int32_t* inv_perm, const int32_t* offsets,
                       const int32_t* counts_all, int ep, int rank, int N_r,
                       void* const* recv_bufs, int capacity, int32_t* dest,
                       int32_t* local_counts, int32_t* local_offsets, mr_stream_t stream) {
  if (T < 0 || d <= 0 || k <= 0 || (dtype != MR_F32 && dtype != MR_BF16)) return MR_ERR_INVALID_ARG;
  if ((long long)T * k >= (1LL << 31) || capacity < 0) return MR_ERR_INVALID_ARG;
  if (ep <= 0 || rank < 0 || rank >= ep || N_r <= 0 || N_r % ep != 0) return MR_ERR_INVALID_ARG;
  if (k > mr::kRowMaxK || ep > mr::kEpMaxRanks || N_r > mr::kEpMaxSegments)
    return MR_ERR_UNSUPPORTED;
  if (!counts_all || !recv_bufs || !local_counts || !local_offsets) return MR_ERR_INVALID_ARG;
  if (T > 0 && (!x || !idx || !inv_perm || !offsets || !dest)) return MR_ERR_INVALID_ARG;
  mr::EpPeers peers{};
  for (int r = 0; r < ep; ++r) {
    if (!recv_bufs[r]) return MR_ERR_INVALID_ARG;
    peers.p[r] = recv_bufs[r];
  }
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long n = (long)T * k;
  const unsigned grid_d =
      (unsigned)std::max<long>(1, (n + mr::kEpRowsPerCta - 1) / mr::kEpRowsPerCta);
  mr::ep_dest_kernel<<<grid_d, mr::kEpThreads, 0, s>>>(idx, inv_perm, offsets, counts_all, n, ep,
                                                        rank, N_r, capacity, dest, local_counts,
                                                        local_offsets);
  if (launch_status() != MR_OK) return MR_ERR_CUDA;
  if (T == 0) return MR_OK;
  const long esz = dtype == MR_BF16 ? 2 : 4;
  const long row_bytes = (long)d * esz;
  bool vec = row_bytes % 16 == 0 && aligned16(x);
  for (int r = 0; r < ep; ++r) vec = vec && aligned16(recv_bufs[r]);
  const unsigned grid_t = (unsigned)std::min<long>(T, 1L << 30);
  const int E_loc = N_r / ep;
  if (vec)
    mr::gather_inv_kernel<uint4><<<grid_t, mr::kRowThreads, 0, s>>>(
        static_cast<const uint4*>(x), T, row_bytes / 16, k,
        mr::SlotRowsPeer<uint4>{peers, idx, dest, E_loc, N_r, capacity});
  else if (esz == 4)
    mr::gather_inv_kernel<uint32_t><<<grid_t, mr::kRowThreads, 0, s>>>(
        static_cast<const uint32_t*>(x), T, d, k,
        mr::SlotRowsPeer<uint32_t>{peers, idx, dest, E_loc, N_r, capacity});
  else
    mr::gather_inv_kernel<uint16_t><<<grid_t, mr::kRowThreads, 0, s>>>(
        static_cast<const uint16_t*>(x), T, d, k,
        mr::SlotRowsPeer<uint16_t>{peers, idx, dest, E_loc, N_r, capacity});
  return launch_status();
}

int mr_ep_combine_p2p(const void* const* out_bufs, int dtype, int d, const float* w,
                      const int32_t* idx, const int32_t* dest, int ep, int N_r, int capacity,
                      const void* shared, void* y, int T, int k, mr_stream_t stream) {
  if (T < 0 || d <= 0 || k <= 0 || (dtype != MR_F32 && dtype != MR_BF16)) return MR_ERR_INVALID_ARG;
  if ((long long)T * k >= (1LL << 31) || capacity < 0) return MR_ERR_INVALID_ARG;
  if (ep <= 0 || N_r <= 0 || N_r % ep != 0) return MR_ERR_INVALID_ARG;
  if (k > mr::kRowMaxK || ep > mr::kEpMaxRanks) return MR_ERR_UNSUPPORTED;
  if (!out_bufs) return MR_ERR_INVALID_ARG;
  if (T == 0) return MR_OK;
  if (!w || !idx || !dest || !y) return MR_ERR_INVALID_ARG;
  mr::EpPeers peers{};
  for (int r = 0; r < ep; ++r) {
    if (!out_bufs[r]) return MR_ERR_INVALID_ARG;
    peers.p[r] = const_cast<void*>(out_bufs[r]);
  }
  int sms = 0, cc = 0;
  if (!device_info(&sms, &cc)) return MR_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long esz = dtype == MR_BF16 ? 2 : 4;
  bool vec = ((long)d * esz) % 16 == 0 && aligned16(y) && (!shared || aligned16(shared));
  for (int r = 0; r < ep; ++r) vec = vec && aligned16(out_bufs[r]);
  const unsigned grid = (unsigned)std::min<long>(T, (long)sms * 64);
  const int E_loc = N_r / ep;
  return launch_combine<false>(vec, false, dtype == MR_BF16, grid, s, w, shared, y, T, d, k,
                               [&](auto* tag) {
                                 using V = std::remove_const_t<std::remove_pointer_t<decltype(tag)>>;
                                 return mr::SlotRowsPeer<const V>{peers, idx, dest, E_loc, N_r,
                                                                  capacity};
                               });
}

// ---- peer buffers between processes -----------------------------------------

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(((mr_ipc_handle_t*)nullptr)->handle),
              "mr_ipc_handle_t.handle holds one CUDA IPC handle");

int mr_ipc_export(const void* dev_ptr, size_t bytes, mr_ipc_handle_t* out) {
  if (!dev_ptr || !out) return MR_ERR_INVALID_ARG;
  static PFN_cuMemGetAddressRange_v3020 range = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
  });
  if (!range) return MR_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return MR_ERR_INVALID_ARG;  // not device memory of this process
  const uint64_t off = reinterpret_cast<CUdeviceptr>(dev_ptr) - base;
  if (off + bytes > size) return MR_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
    cudaGetLastError();
    return MR_ERR_UNSUPPORTED;  // e.g. memory from the virtual memory API
  }
  memcpy(out->handle, &h, sizeof(h));
  out->offset = off;
  out->bytes = bytes;
  return MR_OK;
}

int mr_ipc_import(const mr_ipc_handle_t* h, void** base, void** ptr) {
  if (!h || !base || !ptr) return MR_ERR_INVALID_ARG;
  cudaIpcMemHandle_t ch;
  memcpy(&ch, h->handle, sizeof(ch));
  void* b = nullptr;
  if (cudaIpcOpenMemHandle(&b, ch, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    return MR_ERR_CUDA;
  }
  *base = b;
  *ptr = static_cast<char*>(b) + h->offset;
  return MR_OK;
}

int mr_ipc_close(void* base) {
  if (!base) return MR_ERR_INVALID_ARG;
  if (cudaIpcCloseMemHandle(base) != cudaSuccess) {
    cudaGetLastError();
    return MR_ERR_CUDA;
  }
  return MR_OK;
}

// ---- device error flag ----------------------------------------------------

uint64_t mr_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int mr_get_error(mr_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MR_ERR_CUDA;
  unsigned int flag = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&flag, g_mr_error_flag, sizeof(flag)) != cudaSuccess) return MR_ERR_CUDA;
  if (flag == 0) return MR_OK;
  if (cudaMemcpyToSymbol(g_mr_error_flag, &zero, sizeof(zero)) != cudaSuccess) return MR_ERR_CUDA;
  if (flag & MR_FLAG_TIMEOUT) return MR_ERR_TIMEOUT;
  return (flag & MR_FLAG_BAD_INDEX) ? MR_ERR_DEVICE : MR_ERR_OVERFLOW;
}

}  // extern "C"
