// TokenGate pruned-prefill library: the C ABI declared in include/tg.h.
//
// Host code validates every argument before anything is enqueued, builds TMA
// descriptors for the tensor-core kernels and launches the kernels on the
// caller's stream.  Nothing here allocates device memory or synchronises,
// except tg_check_device_error.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <cstring>
#include <functional>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include "../../include/tg.h"
#include "attn_bwd.cuh"
#include "attn_bwd_tc.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "gate_tc.cuh"
#include "decode.cuh"
#include "gather.cuh"
#include "gemm_tc.cuh"
#include "select.cuh"
#include "simt.cuh"

#define TG_VERSION "tokengate-b200 0.1.0"

namespace {

thread_local char g_last_error[512] = "";

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return status;
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return TG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream is finishing, does its set-up, and
// waits in pdl_wait() (griddepcontrol.wait) before touching global memory.
// Every kernel launched here calls pdl_wait() before its first global access.
template <typename... KArgs, typename... Args>
int launch_pdl(const char* what, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
               Args... args) {
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
  return check_launch(what);
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// ---------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point (no -lcuda needed).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor [rows][inner] with a row stride in bytes; box {box_inner, box_rows}.  Operand
// tiles use a 64-column box with the 128-byte swizzle; L2-prefetch maps use wider unswizzled boxes.
int make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t row_stride_bytes,
             uint32_t box_rows, uint32_t box_inner = 64, bool swizzle = true) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(TG_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return TG_OK;
}

// 1-D fp32 vector of n elements, box of `box` elements, no swizzle (bounds fill: zeros).
int make_map_1d_f32(CUtensorMap* map, const void* base, uint64_t n, uint32_t box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(TG_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[1] = {n};
  cuuint64_t strides[1] = {0};
  cuuint32_t bx[1] = {box};
  cuuint32_t estr[1] = {1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<void*>(base), dims, strides, bx, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TG_ERR_CUDA, "cuTensorMapEncodeTiled (1-D) failed (%d)", static_cast<int>(r));
  return TG_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device): the
// attribute call is host work that would otherwise repeat on every launch.
std::mutex g_smem_mu;
std::map<std::pair<const void*, int>, size_t> g_smem_set;

template <typename Kern>
int set_smem(Kern k, size_t bytes) {
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_pair(reinterpret_cast<const void*>(k), dev);
  {
    std::lock_guard<std::mutex> lock(g_smem_mu);
    auto it = g_smem_set.find(key);
    if (it != g_smem_set.end() && it->second >= bytes) return TG_OK;
  }
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lock(g_smem_mu);
  size_t& v = g_smem_set[key];
  if (bytes > v) v = bytes;
  return TG_OK;
}

// ---------------------------------------------------------------------------
// tcgen05 launches
// ---------------------------------------------------------------------------
constexpr int kGemmStages = 4;

int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// Persistent GEMM: grid = min(tiles, SMs); B has b_rows rows of K elements.
// MH = 2 takes 256-row tiles (half the B traffic per FLOP) when they still
// give every SM a tile; otherwise 128-row tiles keep all SMs busy.
template <int BN, int EPI, int MH>
int launch_gemm_tc(const void* A, int64_t lda, const void* B, int64_t b_rows, int M, int K, int tiles_n,
                   const tg::GemmParams& p0, cudaStream_t st) {
  constexpr int kStages = MH == 2 ? 3 : kGemmStages;
  using Cfg = tg::GemmCfg<BN, kStages, MH>;
  CUtensorMap ta, tb;
  int rc = make_map(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(lda) * 2, 128);
  if (rc) return rc;
  rc = make_map(&tb, B, static_cast<uint64_t>(K), static_cast<uint64_t>(b_rows), static_cast<uint64_t>(K) * 2,
                Cfg::kBBox);
  if (rc) return rc;
  auto kern = tg::k_gemm_tc<BN, kStages, EPI, MH>;
  rc = set_smem(kern, Cfg::kSmem);
  if (rc) return rc;
  tg::GemmParams p = p0;
  p.M = M;
  p.K = K;
  p.tiles_m = (M + Cfg::kBM - 1) / Cfg::kBM;
  p.tiles_n = tiles_n;
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < sm_count() ? tiles : sm_count();
  return launch_pdl("k_gemm_tc", kern, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmem, st, ta, tb, p);
}

// TG_GEMM_SINGLE_SM=1 in the environment selects the single-SM tcgen05 GEMM
// even where two-SM clusters fit (read at every launch, so a test can run
// both kernels in one process).
bool force_single_sm_gemm() {
  const char* e = std::getenv("TG_GEMM_SINGLE_SM");
  return e && e[0] == '1';
}

// Pair GEMM (two-SM clusters, 256 x 256 tiles): the number of clusters that
// can be resident at once, queried once per (kernel, device); 0 if the pair
// kernel cannot be launched here.
constexpr int kGemmPairStages = 3;

template <typename Kern>
int pair_clusters(Kern kern, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const auto key = std::make_pair(reinterpret_cast<const void*>(kern), dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int clusters = 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) clusters = 0;
  }
  cudaGetLastError();  // a refused query leaves no sticky error behind
  cache[key] = clusters;
  return clusters;
}

template <int EPI>
int launch_gemm_pair(const void* A, int64_t lda, const void* B, int64_t b_rows, int M, int K, int tiles_n,
                     const tg::GemmParams& p0, cudaStream_t st, int clusters) {
  using Cfg = tg::GemmPairCfg<kGemmPairStages>;
  CUtensorMap ta, tb;
  int rc = make_map(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(lda) * 2, 128);
  if (rc) return rc;
  rc = make_map(&tb, B, static_cast<uint64_t>(K), static_cast<uint64_t>(b_rows), static_cast<uint64_t>(K) * 2, 128);
  if (rc) return rc;
  // the epilogue writes through TMA: boxes of 32 rows x 64 columns
  CUtensorMap to;
  rc = make_map(&to, p0.out, static_cast<uint64_t>(p0.N), static_cast<uint64_t>(M), static_cast<uint64_t>(p0.ldo) * 2, 32);
  if (rc) return rc;
  auto kern = tg::k_gemm_pair<kGemmPairStages, EPI>;
  rc = set_smem(kern, Cfg::kSmem);
  if (rc) return rc;
  tg::GemmParams p = p0;
  p.M = M;
  p.K = K;
  p.tiles_m = (M + 255) / 256;
  p.tiles_n = tiles_n;
  const int tiles = p.tiles_m * p.tiles_n;
  const int pairs = tiles < clusters ? tiles : clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, to, p);
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "k_gemm_pair launch: %s", cudaGetErrorString(e));
  return check_launch("k_gemm_pair");
}

// Tile choice: the pair kernel (256 x 256 per two SMs, epilogue overlapped)
// wherever two-SM clusters can be resident; otherwise 256-row single-SM tiles
// when they give every SM a tile, else 128-row tiles.
template <int BN, int EPI>
int launch_gemm_auto(const void* A, int64_t lda, const void* B, int64_t b_rows, int M, int K, int tiles_n,
                     const tg::GemmParams& p0, cudaStream_t st) {
  static_assert(BN == 256, "the pair kernel's tile is 256 columns wide");
  const int clusters = pair_clusters(tg::k_gemm_pair<kGemmPairStages, EPI>, tg::GemmPairCfg<kGemmPairStages>::kThreads,
                                     tg::GemmPairCfg<kGemmPairStages>::kSmem);
  if (clusters > 0 && !force_single_sm_gemm())
    return launch_gemm_pair<EPI>(A, lda, B, b_rows, M, K, tiles_n, p0, st, clusters);
  const int64_t tiles256 = int64_t((M + 255) / 256) * tiles_n;
  if (tiles256 >= sm_count() - sm_count() / 16)
    return launch_gemm_tc<BN, EPI, 2>(A, lda, B, b_rows, M, K, tiles_n, p0, st);
  return launch_gemm_tc<BN, EPI, 1>(A, lda, B, b_rows, M, K, tiles_n, p0, st);
}

template <int BN>
int launch_gate_tc(const void* A, const void* W1, int M, int K, const tg::GateParams& p0, cudaStream_t st) {
  using Cfg = tg::GateCfg<BN>;
  CUtensorMap ta, tb;
  int rc = make_map(&ta, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, 128);
  if (rc) return rc;
  rc = make_map(&tb, W1, static_cast<uint64_t>(K), static_cast<uint64_t>(p0.N), static_cast<uint64_t>(K) * 2,
                Cfg::kBBox);
  if (rc) return rc;
  rc = set_smem(tg::k_gate_tc<BN>, Cfg::kSmem);
  if (rc) return rc;
  tg::GateParams p = p0;
  p.M = M;
  p.K = K;
  p.hidden = static_cast<const __nv_bfloat16*>(A);
  // persistent: one CTA per SM (or per tile when there are fewer tiles)
  const int tiles = (M + tg::kGateBM - 1) / tg::kGateBM;
  return launch_pdl("k_gate_tc", tg::k_gate_tc<BN>, dim3(tiles < sm_count() ? tiles : sm_count()), dim3(tg::kGateThreads),
                    Cfg::kSmem, st, ta, tb, p);
}

int dtype_size(int dtype) { return dtype == TG_BF16 ? 2 : (dtype == TG_F32 ? 4 : 0); }

// Whether tg_gate_score takes the tensor-core kernel (the only path that uses
// its workspace); other shapes and fp32 run on CUDA cores without scratch.
bool gate_uses_tc(const void* hidden, int dtype, int32_t d_model, const void* w1, int32_t h) {
  return dtype == TG_BF16 && d_model % 8 == 0 && h <= 256 && h % 16 == 0 && aligned16(hidden) && aligned16(w1);
}

// workspace layout of tg_gate_score (256-byte aligned pieces):
//   [per-CTA partial sums of s^2][completion counter][W1 scaled by the norm weight, bf16 [h][d]]
// and of tg_gate_score_select, the selector's first-digit histogram right
// after the counter so that one memset clears both:
//   [partial sums][completion counter][histogram, 2048 x u32][scaled W1]
size_t gate_partials_bytes(int64_t n) { return ((static_cast<size_t>((n + 127) / 128) * 4 + 255) / 256) * 256; }
constexpr size_t kGateHistBytes = tg::kGateHistBins * sizeof(uint32_t);
size_t gate_ws_bytes(int64_t n, int32_t d, int32_t h) {
  return gate_partials_bytes(n) + 256 + ((static_cast<size_t>(d) * h * 2 + 255) / 256) * 256;
}
size_t gate_select_ws_bytes(int64_t n, int32_t d, int32_t h) { return gate_ws_bytes(n, d, h) + kGateHistBytes; }

}  // namespace

// RMSNorm of m rows: one warp per row when the row fits in a warp's registers
// (and the weight is 16-byte aligned), else one block per row.
// words of a later kernel's workspace (counters) that the launched kernel
// clears as a side job
struct ZeroSpan {
  uint32_t* p = nullptr;
  int n = 0;
};

template <typename T>
int launch_rmsnorm(const void* x, void* y, const float* w, int64_t m, int d, float eps, cudaStream_t st,
                   ZeroSpan z = ZeroSpan{}) {
  constexpr int V = 16 / sizeof(T);
  const int nv = d / V;
  const T* xa = static_cast<const T*>(x);
  T* ya = static_cast<T*>(y);
  const unsigned blocks = static_cast<unsigned>((m + 7) / 8);
  if (!w || aligned16(w)) {
    if (nv <= 32 * 4) {
      return launch_pdl("k_rmsnorm_warp", tg::k_rmsnorm_warp<T, 4>, dim3(blocks), dim3(256), 0, st, xa, ya, w, m, d, eps,
                        z.p, z.n);
    }
    if (nv <= 32 * 8) {
      return launch_pdl("k_rmsnorm_warp", tg::k_rmsnorm_warp<T, 8>, dim3(blocks), dim3(256), 0, st, xa, ya, w, m, d, eps,
                        z.p, z.n);
    }
    if (nv <= 32 * 16) {
      return launch_pdl("k_rmsnorm_warp", tg::k_rmsnorm_warp<T, 16>, dim3(blocks), dim3(256), 0, st, xa, ya, w, m, d, eps,
                        z.p, z.n);
    }
  }
  if (z.n && cudaMemsetAsync(z.p, 0, size_t(z.n) * 4, st) != cudaSuccess)
    return fail(TG_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(cudaGetLastError()));
  return launch_pdl("k_rmsnorm", tg::k_rmsnorm<T>, dim3(unsigned(m)), dim3(256), 0, st, xa, ya, w, d, eps);
}

// Whether a 16-CTA cluster of the selector can be resident on this device
// (a non-portable cluster size): checked once per device.
bool select_cluster16_ok() {
  static std::mutex mu;
  static std::map<int, bool> ok;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  auto it = ok.find(dev);
  if (it != ok.end()) return it->second;
  bool good = cudaFuncSetAttribute(tg::k_topk_select, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  if (good) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16);
    cfg.blockDim = dim3(tg::kSelThreads);
    cfg.dynamicSmemBytes = tg::select_smem_bytes(tg::kSelMaxKpt, 1);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    good = cudaFuncSetAttribute(tg::k_topk_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(tg::select_smem_bytes(tg::kSelMaxKpt, 1))) == cudaSuccess &&
           cudaOccupancyMaxActiveClusters(&clusters, tg::k_topk_select, &cfg) == cudaSuccess && clusters >= 1;
  }
  cudaGetLastError();  // a refused query leaves no sticky error behind
  ok[dev] = good;
  return good;
}

// decode kernel for a group size (query heads per KV head) fixed at compile time
template <typename T, int D>
int launch_decode(int group, dim3 grid, cudaStream_t st, const tg::DecodeParams& p) {
  switch (group) {
    case 1: return launch_pdl("k_decode_attn", tg::k_decode_attn<T, D, 1>, grid, dim3(tg::kDecThreads), 0, st, p);
    case 2: return launch_pdl("k_decode_attn", tg::k_decode_attn<T, D, 2>, grid, dim3(tg::kDecThreads), 0, st, p);
    case 3: return launch_pdl("k_decode_attn", tg::k_decode_attn<T, D, 3>, grid, dim3(tg::kDecThreads), 0, st, p);
    case 4: return launch_pdl("k_decode_attn", tg::k_decode_attn<T, D, 4>, grid, dim3(tg::kDecThreads), 0, st, p);
    case 5: return launch_pdl("k_decode_attn", tg::k_decode_attn<T, D, 5>, grid, dim3(tg::kDecThreads), 0, st, p);
    case 6: return launch_pdl("k_decode_attn", tg::k_decode_attn<T, D, 6>, grid, dim3(tg::kDecThreads), 0, st, p);
    case 7: return launch_pdl("k_decode_attn", tg::k_decode_attn<T, D, 7>, grid, dim3(tg::kDecThreads), 0, st, p);
    default: return launch_pdl("k_decode_attn", tg::k_decode_attn<T, D, 8>, grid, dim3(tg::kDecThreads), 0, st, p);
  }
}

// TMA decode kernel: tensor maps of the KV head columns of K and V (64-row
// boxes of 64 dimensions, 128-byte swizzle; rows past the cache read as zeros)
template <int D, int G>
int launch_decode_tma_g(dim3 grid, cudaStream_t st, const tg::DecodeParams& p) {
  using Cfg = tg::DecTmaCfg<D>;
  CUtensorMap tk, tv, tb;
  const uint64_t cols = static_cast<uint64_t>(p.hkv) * D;
  int rc = make_map(&tk, p.k, cols, static_cast<uint64_t>(p.length), static_cast<uint64_t>(p.ldk) * 2, tg::kDtRows);
  if (rc) return rc;
  rc = make_map(&tv, p.v, cols, static_cast<uint64_t>(p.length), static_cast<uint64_t>(p.ldv) * 2, tg::kDtRows);
  if (rc) return rc;
  if (p.bias) {
    rc = make_map_1d_f32(&tb, p.bias, static_cast<uint64_t>(p.length), tg::kDtRows);
    if (rc) return rc;
  } else {
    tb = tk;  // not read
  }
  rc = set_smem(tg::k_decode_tma<D, G>, Cfg::kSmem);
  if (rc) return rc;
  return launch_pdl("k_decode_tma", tg::k_decode_tma<D, G>, grid, dim3(tg::kDtThreads), Cfg::kSmem, st, tk, tv, tb, p);
}

template <int D>
int launch_decode_tma(int group, dim3 grid, cudaStream_t st, const tg::DecodeParams& p) {
  switch (group) {
    case 1: return launch_decode_tma_g<D, 1>(grid, st, p);
    case 2: return launch_decode_tma_g<D, 2>(grid, st, p);
    case 3: return launch_decode_tma_g<D, 3>(grid, st, p);
    case 4: return launch_decode_tma_g<D, 4>(grid, st, p);
    case 5: return launch_decode_tma_g<D, 5>(grid, st, p);
    case 6: return launch_decode_tma_g<D, 6>(grid, st, p);
    case 7: return launch_decode_tma_g<D, 7>(grid, st, p);
    default: return launch_decode_tma_g<D, 8>(grid, st, p);
  }
}

// the layer's own buffers (normed rows, qkv, attention output, MLP activation)
static size_t layer_buffers_bytes(int64_t m, const tg_layer_shape* S) {
  const int es = dtype_size(S->dtype);
  const size_t qkv = static_cast<size_t>(S->hq + 2 * S->hkv) * S->head_dim;
  const size_t rows = static_cast<size_t>(m);
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  // x (normed rows), qkv, attention output, MLP activation (room for the
  // un-fused gate/up product, twice as wide as the fused SwiGLU output)
  const size_t act = static_cast<size_t>(S->d_ff) * 2;
  return al(rows * S->d_model * es) + al(rows * qkv * es) + al(rows * S->hq * S->head_dim * es) +
         al(rows * act * es);
}

// Where the layer's first RMSNorm reads its rows from when the gather is
// folded into it: hidden_kept[r] = hidden[idx[r]] is written in the same pass
// (with pos, bias and ratio, as tg_gather writes them).
struct LayerGather {
  const void* hidden;
  int64_t n;
  const int32_t* idx;
  const float* scores;
  const float* sumsq;
  int64_t n_prunable;
  float seq_eps;
  int32_t* pos;
  float* bias;
  float* ratio;
};

static int prefill_layer_impl(const tg_layer_weights* W, const tg_layer_shape* S, int parts, void* hidden_kept,
                              const int32_t* pos, const float* bias, const float* ratio, int64_t m,
                              const int64_t* seg_rows, int32_t nseg, const LayerGather* gather, void* ws,
                              size_t ws_bytes, void* stream);
static int launch_gather_rmsnorm(const LayerGather& g, int dtype, void* hidden_kept, void* xn, const float* w,
                                 int64_t m, int d, float eps, cudaStream_t st, ZeroSpan z);
static int gate_score_impl(const void* hidden, int dtype, int64_t n, int32_t d_model, const float* norm_w,
                           float norm_eps, const void* w1, const float* b1, const float* w2, float b2, int32_t h,
                           const uint8_t* prunable, float* scores, float* sumsq, void* ws, size_t ws_bytes,
                           bool with_hist, void* stream, bool ws_clean = false);
static int topk_select_impl(const float* scores, const uint8_t* prunable, int64_t n, int64_t n_prunable, int64_t k,
                            int32_t* kept_idx, int64_t m, const uint32_t* hist_top, void* stream,
                            uint32_t* hist_clear = nullptr);

extern "C" {

const char* tg_version(void) { return TG_VERSION; }

const char* tg_status_string(int status) {
  switch (status) {
    case TG_OK: return "ok";
    case TG_ERR_INVALID_ARG: return "invalid argument";
    case TG_ERR_SHAPE: return "inconsistent shape";
    case TG_ERR_ALIGN: return "misaligned pointer or leading dimension";
    case TG_ERR_UNSUPPORTED: return "unsupported configuration";
    case TG_ERR_WORKSPACE: return "workspace missing or too small";
    case TG_ERR_CUDA: return "CUDA error";
    case TG_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case TG_ERR_DEVICE_CHECK: return "device-side consistency check failed";
    default: return "unknown status";
  }
}

const char* tg_last_error(void) { return g_last_error; }

int tg_debug_set_flag_wait(uint64_t limit_ns, uint32_t merge_ready_target) {
  const uint64_t lim = limit_ns ? limit_ns : tg::kWaitLimitNs;
  const uint32_t tgt = merge_ready_target ? merge_ready_target : tg::kMergeReadyTarget;
  cudaError_t e = cudaMemcpyToSymbol(tg::g_flag_wait_limit_ns, &lim, sizeof(lim));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(tg::g_merge_ready_target, &tgt, sizeof(tgt));
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "tg_debug_set_flag_wait: %s", cudaGetErrorString(e));
  return TG_OK;
}

int tg_check_device_error(void* stream, uint32_t* detail) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  uint32_t word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, tg::g_error_word, sizeof(word));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(tg::g_error_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "error word: %s", cudaGetErrorString(e));
  if (detail) *detail = word;
  if (word == 0) return TG_OK;
  const uint32_t site = word & 0xffu;
  if (site >= tg::kErrTimeoutFirst && site <= tg::kErrTimeoutLast)
    return fail(TG_ERR_DEVICE_TIMEOUT, "device wait timed out at site %u", site);
  return fail(TG_ERR_DEVICE_CHECK, "device check failed at site %u (payload %u)", site, word >> 8);
}

// Schedule of the tensor-core attention kernel.  A CTA owns one 128-row query
// block of two query heads; its causal work is the number of 64-key tiles up
// to the diagonal, which grows with the block index, and every CTA also pays a
// fixed cost (start-up, first loads, epilogue) worth about kAttnCtaFixed tiles.
// When the launch is about a wave of the GPU, the longest blocks set its
// length; splitting a block into two CTAs (first and second half of its key
// tiles, merged by the CTA that finishes second) shortens them but adds a
// fixed cost.  The plan splits the k longest blocks for the k whose simulated
// longest-first schedule on the SMs ends first (k = 0: no split), and launches
// the CTAs longest first.
constexpr int kAttnCtaFixed = 4;

struct AttnPlan {
  int T = 0, per_tile = 0, ts = 0;
  bool table = false;
  std::vector<uint16_t> items;  // AttnWork encoding, longest first
  size_t part_off = 0, ml_off = 0, ctr_off = 0, bytes = 0;  // workspace layout
};

struct AttnItem {
  int size, t, code;
};

// items of the schedule that splits blocks t >= ts, longest first; a 128-row
// block t has (t + 1) * 128 / bn causal key tiles of bn keys (at most kt)
std::vector<AttnItem> attn_items(int T, int kt, int ts, int bn) {
  std::vector<AttnItem> it;
  it.reserve(2 * T);
  for (int t = 0; t < T; ++t) {
    const int u = std::min((t + 1) * (128 / bn), kt);
    if (t >= ts) {
      it.push_back({u / 2, t, 1});
      it.push_back({u - u / 2, t, 2});
    } else {
      it.push_back({u, t, 0});
    }
  }
  std::stable_sort(it.begin(), it.end(), [](const AttnItem& a, const AttnItem& b) {
    if (a.size != b.size) return a.size > b.size;
    if (a.t != b.t) return a.t > b.t;
    return a.code > b.code;
  });
  return it;
}

// end of the greedy in-order schedule of `per_tile` copies of each item on `sms` SMs
int64_t attn_makespan(const std::vector<AttnItem>& it, int per_tile, int sms, int fixed) {
  std::vector<int64_t> busy(static_cast<size_t>(sms), 0);  // min-heap of SM finish times
  for (const AttnItem& x : it)
    for (int r = 0; r < per_tile; ++r) {
      std::pop_heap(busy.begin(), busy.end(), std::greater<int64_t>());
      busy.back() += x.size + fixed;
      std::push_heap(busy.begin(), busy.end(), std::greater<int64_t>());
    }
  return *std::max_element(busy.begin(), busy.end());
}

AttnPlan attn_plan_compute(int64_t m, int hkv, int group, int head_dim, int sms) {
  constexpr int bn = tg::AttnCfg<128>::BN;  // key-tile width of k_attn_tc
  AttnPlan pl;
  pl.T = static_cast<int>((m + 127) / 128);
  pl.per_tile = hkv * (group / 2);
  pl.ts = pl.T;
  const int kt = static_cast<int>((m + bn - 1) / bn);
  // fixed cost per CTA in key tiles, and the fewest tiles a split block may have
  // (each half keeps a visible key in every row)
  const int fixed = kAttnCtaFixed;
  const int min_split = 2;
  sms = std::max(sms, 1);
  // only short launches gain from splitting: at most about two waves of CTAs,
  // and blocks of at least 4 tiles (each half keeps a visible key per row)
  if (int64_t(pl.T) * pl.per_tile > 2 * int64_t(sms) || 2 * pl.T > tg::kAttnWorkCap || pl.T >= (1 << 14)) return pl;
  int64_t best = attn_makespan(attn_items(pl.T, kt, pl.T, bn), pl.per_tile, sms, fixed);
  int best_ts = pl.T;
  for (int ts = pl.T - 1; ts >= 1 && std::min((ts + 1) * (128 / bn), kt) >= min_split; --ts) {
    const int64_t span = attn_makespan(attn_items(pl.T, kt, ts, bn), pl.per_tile, sms, fixed);
    if (span < best) {
      best = span;
      best_ts = ts;
    }
  }
  if (best_ts == pl.T) return pl;
  pl.ts = best_ts;
  const std::vector<AttnItem> it = attn_items(pl.T, kt, pl.ts, bn);
  pl.table = true;
  pl.items.reserve(it.size());
  for (const AttnItem& x : it) pl.items.push_back(static_cast<uint16_t>((x.t << 2) | x.code));
  const size_t slots = size_t(pl.T - pl.ts) * pl.per_tile;
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  pl.part_off = 0;
  pl.ml_off = al(slots * 2 * 2 * 128 * size_t(head_dim) * 4);
  pl.ctr_off = pl.ml_off + al(slots * 2 * 2 * 128 * 8);
  pl.bytes = pl.ctr_off + al(slots * 4);
  return pl;
}

// The plan depends only on the shape and the SM count; it is computed once
// per key (the schedule simulation costs tens of microseconds of host time).
const AttnPlan& attn_plan(int64_t m, int hkv, int group, int head_dim, int sms) {
  static std::mutex mu;
  static std::map<std::tuple<int64_t, int, int, int, int>, AttnPlan> cache;
  const auto key = std::make_tuple(m, hkv, group, head_dim, sms);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it == cache.end()) {
    if (cache.size() > 4096) cache.clear();
    it = cache.emplace(key, attn_plan_compute(m, hkv, group, head_dim, sms)).first;
  }
  return it->second;
}

// workspace of tg_gated_attention (0 when the launch is long enough to need no split)
size_t attn_ws_bytes(int64_t m, int hq, int hkv, int head_dim, int dtype) {
  if (dtype != TG_BF16 || m <= 0 || hq <= 0 || hkv <= 0 || hq % hkv || (hq / hkv) % 2) return 0;
  return attn_plan(m, hkv, hq / hkv, head_dim, sm_count()).bytes;
}

// Decode attention: key chunks of a multiple of 64 keys (at most
// kDecMaxChunk), about two CTAs per SM over all KV heads; the workspace holds
// each chunk's (O, max, sum) per query head, then one counter per KV head.
struct DecodePlan {
  int chunk = 0, nchunks = 0;
  size_t part_bytes = 0, bytes = 0;
};

// TG_DECODE_SIMT=1 in the environment sends bf16 decode to the CUDA-core
// kernel too (read at every call, so a test can run both kernels in one process).
bool force_simt_decode() {
  const char* e = std::getenv("TG_DECODE_SIMT");
  return e && e[0] == '1';
}

// tma: the bf16 kernel that streams the cache through shared memory (one CTA
// per SM over all KV heads, chunks of whole 64-row tiles); otherwise about two
// CTAs per SM with chunks of at most kDecMaxChunk rows.  Both keep at most
// kDecMaxChunks chunks per KV head.
DecodePlan decode_plan(int64_t length, int hkv, int group, int head_dim, bool tma) {
  DecodePlan pl;
  if (length <= 0 || hkv <= 0 || group <= 0) return pl;
  const int64_t sms = sm_count();
  int64_t chunk;
  if (tma) {
    const int64_t per_head = std::max<int64_t>(1, std::min<int64_t>(sms / hkv, tg::kDecMaxChunks));
    chunk = (length + per_head - 1) / per_head;
    chunk = std::max<int64_t>((chunk + tg::kDtRows - 1) / tg::kDtRows * tg::kDtRows, tg::kDtRows);
  } else {
    chunk = (length * hkv + 2 * sms - 1) / (2 * sms);
    chunk = std::max<int64_t>(chunk, (length + tg::kDecMaxChunks - 1) / tg::kDecMaxChunks);  // <= 256 chunks
    chunk = std::min<int64_t>(std::max<int64_t>((chunk + 63) / 64 * 64, 64), tg::kDecMaxChunk);
  }
  pl.chunk = static_cast<int>(chunk);
  pl.nchunks = static_cast<int>((length + chunk - 1) / chunk);
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  pl.part_bytes = al(static_cast<size_t>(hkv) * pl.nchunks * group * (head_dim + 2) * sizeof(float));
  pl.bytes = pl.part_bytes + al(static_cast<size_t>(hkv) * sizeof(uint32_t));
  return pl;
}

// workspace that covers either decode kernel (the query does not see the
// pointers that decide between them)
size_t decode_ws_bytes(int64_t length, int hkv, int group, int head_dim) {
  return std::max(decode_plan(length, hkv, group, head_dim, false).bytes,
                  decode_plan(length, hkv, group, head_dim, true).bytes);
}

size_t tg_workspace_bytes(int op, int64_t n, int64_t m, int32_t d_model, int32_t h, const tg_layer_shape* shape) {
  if (op == TG_OP_GATE_SCORE) return (n > 0 && d_model > 0 && h > 0) ? gate_ws_bytes(n, d_model, h) : 0;
  if (op == TG_OP_GATE_SELECT) return (n > 0 && d_model > 0 && h > 0) ? gate_select_ws_bytes(n, d_model, h) : 0;
  if (op == TG_OP_LAYER) {
    if (!shape || m <= 0 || !dtype_size(shape->dtype)) return 0;
    return layer_buffers_bytes(m, shape) + attn_ws_bytes(m, shape->hq, shape->hkv, shape->head_dim, shape->dtype);
  }
  if (op == TG_OP_ATTENTION) {
    if (!shape || m <= 0) return 0;
    return attn_ws_bytes(m, shape->hq, shape->hkv, shape->head_dim, shape->dtype);
  }
  if (op == TG_OP_ATTENTION_BWD) {
    if (!shape || m <= 0 || shape->hq <= 0 || shape->hkv <= 0) return 0;
    auto al = [](size_t b) { return (b + 255) / 256 * 256; };
    const size_t nkb = static_cast<size_t>((m + tg::kBwdBlk - 1) / tg::kBwdBlk);
    const size_t m_pad = static_cast<size_t>((m + 127) / 128 * 128);
    const size_t hd = static_cast<size_t>(shape->head_dim > 0 ? shape->head_dim : 128);
    return al(size_t(shape->hq) * m * 4) + al(size_t(shape->hkv) * m * 4) + al(size_t(shape->hq) * nkb * 2 * 4) +
           al(size_t(shape->hq) * m_pad * 16) + al(size_t(shape->hq) * m_pad * 2 * hd * 4) +
           al(2 * size_t(shape->hkv) * (m_pad / 128) * 4);
  }
  if (op == TG_OP_DECODE) {
    if (!shape || m <= 0 || shape->hkv <= 0 || shape->hq % shape->hkv) return 0;
    return decode_ws_bytes(m, shape->hkv, shape->hq / shape->hkv, shape->head_dim);
  }
  return 0;
}

int tg_gate_score(const void* hidden, int dtype, int64_t n, int32_t d_model, const float* norm_w, float norm_eps,
                  const void* w1, const float* b1, const float* w2, float b2, int32_t h, const uint8_t* prunable,
                  float* scores, float* sumsq, void* ws, size_t ws_bytes, void* stream) {
  return gate_score_impl(hidden, dtype, n, d_model, norm_w, norm_eps, w1, b1, w2, b2, h, prunable, scores, sumsq, ws,
                         ws_bytes, false, stream);
}

}  // extern "C"

// tg_gate_score; with_hist (the tg_gate_score_select workspace layout) has the
// tensor-core kernel also count order_key(s) >> 21 over the prunable tokens
// (the selector's first digit) into the workspace's histogram.  Returns
// TG_ERR_UNSUPPORTED with with_hist on the CUDA-core path, which does not
// build it.
static int gate_score_impl(const void* hidden, int dtype, int64_t n, int32_t d_model, const float* norm_w,
                           float norm_eps, const void* w1, const float* b1, const float* w2, float b2, int32_t h,
                           const uint8_t* prunable, float* scores, float* sumsq, void* ws, size_t ws_bytes,
                           bool with_hist, void* stream, bool ws_clean) {
  if (!hidden || !w1 || !w2 || !prunable || !scores || !sumsq) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (n <= 0 || d_model <= 0 || h <= 0) return fail(TG_ERR_INVALID_ARG, "n, d_model and h must be positive");
  if (n >= (int64_t(1) << 31)) return fail(TG_ERR_UNSUPPORTED, "n must be < 2^31");
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "dtype");
  cudaStream_t st = as_stream(stream);
  if (gate_uses_tc(hidden, dtype, d_model, w1, h)) {
    const size_t need = with_hist ? gate_select_ws_bytes(n, d_model, h) : gate_ws_bytes(n, d_model, h);
    if (!ws || ws_bytes < need) return fail(TG_ERR_WORKSPACE, "gate score needs %zu workspace bytes", need);
    if (!aligned16(ws)) return fail(TG_ERR_ALIGN, "workspace must be 16-byte aligned");
    float* partials = static_cast<float*>(ws);
    uint8_t* counter_at = static_cast<uint8_t*>(ws) + gate_partials_bytes(n);
    uint32_t* counter = reinterpret_cast<uint32_t*>(counter_at);
    uint32_t* key_hist = with_hist ? reinterpret_cast<uint32_t*>(counter_at + 256) : nullptr;
    // (ws_clean: the counter and histogram are zero already, as the previous
    // call left them: the last CTA resets the counter, the selector clears
    // the histogram after reading it)
    if (!ws_clean) {
      cudaError_t e = cudaMemsetAsync(counter, 0, with_hist ? 256 + kGateHistBytes : sizeof(uint32_t), st);
      if (e != cudaSuccess) return fail(TG_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    }
    const void* w1_eff = w1;
    if (norm_w) {
      // RMSNorm(h) * w_n feeds W1, so (h * w_n) W1^T = h (W1 diag(w_n))^T: fold the weight into W1
      __nv_bfloat16* w1f = reinterpret_cast<__nv_bfloat16*>(counter_at + 256 + (with_hist ? kGateHistBytes : 0));
      const int64_t total = int64_t(h) * d_model;
      tg::k_fold_norm<<<unsigned((total + 255) / 256), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w1), norm_w,
                                                                   w1f, total, d_model);
      int rc = check_launch("k_fold_norm");
      if (rc) return rc;
      w1_eff = w1f;
    }
    tg::GateParams p{};
    p.N = h;
    p.b1 = b1;
    p.w2 = w2;
    p.b2 = b2;
    p.norm_eps = norm_eps;
    p.prunable = prunable;
    p.scores = scores;
    p.partials = partials;
    p.counter = counter;
    p.sumsq = sumsq;
    p.key_hist = key_hist;
    const int nn = static_cast<int>(n);
    if (h <= 64) return launch_gate_tc<64>(hidden, w1_eff, nn, d_model, p, st);
    if (h <= 128) return launch_gate_tc<128>(hidden, w1_eff, nn, d_model, p, st);
    return launch_gate_tc<256>(hidden, w1_eff, nn, d_model, p, st);
  }
  if (with_hist) return fail(TG_ERR_UNSUPPORTED, "the key histogram comes only from the tensor-core gate kernel");
  if (h > 1024) return fail(TG_ERR_UNSUPPORTED, "h > 1024");
  const unsigned blocks = static_cast<unsigned>((n + 7) / 8);
  if (dtype == TG_F32)
    tg::k_gate_score_simt<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(hidden), n, d_model, norm_w,
                                                          norm_eps, static_cast<const float*>(w1), b1, w2, b2, h,
                                                          prunable, scores);
  else
    tg::k_gate_score_simt<__nv_bfloat16><<<blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(hidden), n, d_model, norm_w, norm_eps,
        static_cast<const __nv_bfloat16*>(w1), b1, w2, b2, h, prunable, scores);
  int rc = check_launch("k_gate_score_simt");
  if (rc) return rc;
  tg::k_sumsq_ordered<<<1, 1024, 0, st>>>(scores, prunable, n, sumsq);
  return check_launch("k_sumsq_ordered");
}

extern "C" {

int tg_topk_select(const float* scores, const uint8_t* prunable, int64_t n, int64_t n_prunable, int64_t k,
                   int32_t* kept_idx, int64_t m, void* stream) {
  return topk_select_impl(scores, prunable, n, n_prunable, k, kept_idx, m, nullptr, stream);
}

}  // extern "C"

// tg_topk_select; with hist_top (device [2048] counts of order_key >> 21 over
// the prunable tokens) the cluster selector starts from that histogram.
static int topk_select_impl(const float* scores, const uint8_t* prunable, int64_t n, int64_t n_prunable, int64_t k,
                            int32_t* kept_idx, int64_t m, const uint32_t* hist_top, void* stream,
                            uint32_t* hist_clear) {
  if (!scores || !prunable || (!kept_idx && m > 0)) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (n <= 0 || n_prunable < 0 || n_prunable > n) return fail(TG_ERR_INVALID_ARG, "bad n / n_prunable");
  if (k < 0) return fail(TG_ERR_INVALID_ARG, "k must be >= 0");
  if (n >= (int64_t(1) << 31)) return fail(TG_ERR_UNSUPPORTED, "n must be < 2^31");
  const int64_t want = (k < n_prunable ? k : n_prunable) + (n - n_prunable);
  if (m != want) return fail(TG_ERR_SHAPE, "m = %lld but min(k, n_prunable) + n - n_prunable = %lld",
                             static_cast<long long>(m), static_cast<long long>(want));
  tg::SelectParams p{};
  p.scores = scores;
  p.prunable = prunable;
  p.n = n;
  p.n_prunable = n_prunable;
  p.k = k;
  p.out = kept_idx;
  p.m = m;
  p.hist_top = nullptr;
  if (n <= tg::kSelSmallBest) {
    // short prompt: one CTA, keys resident in shared memory
    const int need = static_cast<int>((n + tg::kSelSmallThreads - 1) / tg::kSelSmallThreads);
    const int kpt = need <= 4 ? 4 : (need <= 8 ? 8 : (need <= 16 ? 16 : 32));
    const size_t smem = static_cast<size_t>(kpt) * tg::kSelSmallStride * 5 + 16;
    const int vec = (aligned16(scores) && (reinterpret_cast<uintptr_t>(prunable) & 3u) == 0) ? 1 : 0;
    cudaStream_t st = as_stream(stream);
    int rc;
    switch (kpt) {
      case 4:
        if ((rc = set_smem(tg::k_topk_select_cta<4>, smem))) return rc;
        return launch_pdl("k_topk_select_cta", tg::k_topk_select_cta<4>, dim3(1), dim3(tg::kSelSmallThreads), smem,
                          st, p, vec);
      case 8:
        if ((rc = set_smem(tg::k_topk_select_cta<8>, smem))) return rc;
        return launch_pdl("k_topk_select_cta", tg::k_topk_select_cta<8>, dim3(1), dim3(tg::kSelSmallThreads), smem,
                          st, p, vec);
      case 16:
        if ((rc = set_smem(tg::k_topk_select_cta<16>, smem))) return rc;
        return launch_pdl("k_topk_select_cta", tg::k_topk_select_cta<16>, dim3(1), dim3(tg::kSelSmallThreads), smem,
                          st, p, vec);
      default:
        if ((rc = set_smem(tg::k_topk_select_cta<32>, smem))) return rc;
        return launch_pdl("k_topk_select_cta", tg::k_topk_select_cta<32>, dim3(1), dim3(tg::kSelSmallThreads), smem,
                          st, p, vec);
    }
  }
  // cluster of 2 .. 16 CTAs of about kSelSlice tokens each, while the cluster can grow
  int csize = 1;
  while (csize < tg::kSelCluster && (n + csize - 1) / csize > tg::kSelSlice) csize *= 2;
  if (csize > 8 && !select_cluster16_ok()) csize = 8;
  p.slice = (n + csize - 1) / csize;
  int kpt = 1;
  while (static_cast<int64_t>(kpt) * tg::kSelThreads < p.slice) kpt *= 2;
  p.kpt = kpt;
  p.cached = kpt <= tg::kSelMaxKpt ? 1 : 0;
  p.hist_top = hist_top;
  p.hist_clear = hist_top ? hist_clear : nullptr;
  const size_t smem = tg::select_smem_bytes(kpt, p.cached);
  int rc = set_smem(tg::k_topk_select, smem);
  if (rc) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(csize);
  cfg.blockDim = dim3(tg::kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = as_stream(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, tg::k_topk_select, p);
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "k_topk_select launch: %s", cudaGetErrorString(e));
  return check_launch("k_topk_select");
}

extern "C" {

int tg_gate_score_select(const void* hidden, int dtype, int64_t n, int32_t d_model, const float* norm_w,
                         float norm_eps, const void* w1, const float* b1, const float* w2, float b2, int32_t h,
                         const uint8_t* prunable, int64_t n_prunable, int64_t k, float* scores, float* sumsq,
                         int32_t* kept_idx, int64_t m, void* ws, size_t ws_bytes, uint32_t flags, void* stream) {
  if (flags & ~uint32_t(TG_WS_KEPT_ZERO)) return fail(TG_ERR_INVALID_ARG, "unknown flags");
  const bool ws_clean = (flags & TG_WS_KEPT_ZERO) != 0;
  if (!scores || !prunable || (!kept_idx && m > 0)) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (n <= 0 || n_prunable < 0 || n_prunable > n) return fail(TG_ERR_INVALID_ARG, "bad n / n_prunable");
  if (k < 0) return fail(TG_ERR_INVALID_ARG, "k must be >= 0");
  const int64_t want = (k < n_prunable ? k : n_prunable) + (n - n_prunable);
  if (m != want) return fail(TG_ERR_SHAPE, "m = %lld but min(k, n_prunable) + n - n_prunable = %lld",
                             static_cast<long long>(m), static_cast<long long>(want));
  const size_t need = gate_select_ws_bytes(n, d_model, h);
  if (!ws || ws_bytes < need) return fail(TG_ERR_WORKSPACE, "gate score + select needs %zu workspace bytes", need);
  if (!aligned16(ws)) return fail(TG_ERR_ALIGN, "workspace must be 16-byte aligned");
  // the selector's first-digit histogram rides with the gate kernel when the
  // tensor cores score and the cluster selector runs (longer prompts)
  const bool with_hist = n > tg::kSelSmallBest && gate_uses_tc(hidden, dtype, d_model, w1, h);
  uint32_t* hist =
      with_hist ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + gate_partials_bytes(n) + 256) : nullptr;
  int rc = gate_score_impl(hidden, dtype, n, d_model, norm_w, norm_eps, w1, b1, w2, b2, h, prunable, scores, sumsq,
                           ws, ws_bytes, with_hist, stream, ws_clean);
  if (rc) return rc;
  return topk_select_impl(scores, prunable, n, n_prunable, k, kept_idx, m, hist, stream, ws_clean ? hist : nullptr);
}

}  // extern "C"

extern "C" {

int tg_gather(const void* hidden, int dtype, int64_t n, int32_t d_model, const int32_t* kept_idx, int64_t m,
              const float* scores, const float* sumsq, int64_t n_prunable, float seq_eps, void* hidden_kept,
              int32_t* pos, float* bias, float* ratio, void* stream) {
  if (!hidden || !kept_idx || !hidden_kept) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (bias && (!scores || !sumsq)) return fail(TG_ERR_INVALID_ARG, "bias needs scores and sumsq");
  if (n <= 0 || m <= 0 || m > n || d_model <= 0) return fail(TG_ERR_INVALID_ARG, "bad sizes");
  if (bias && n_prunable <= 0) return fail(TG_ERR_INVALID_ARG, "n_prunable must be > 0 for bias");
  const int es = dtype_size(dtype);
  if (!es) return fail(TG_ERR_INVALID_ARG, "dtype");
  const int64_t row_bytes = static_cast<int64_t>(d_model) * es;
  if (row_bytes % 16 != 0 || !aligned16(hidden) || !aligned16(hidden_kept))
    return fail(TG_ERR_ALIGN, "rows must be 16-byte multiples on 16-byte aligned buffers");
  tg::GatherParams p{};
  p.hidden = static_cast<const uint8_t*>(hidden);
  p.n = n;
  p.row_bytes = row_bytes;
  p.idx = kept_idx;
  p.m = m;
  p.scores = scores;
  p.sumsq = sumsq;
  p.n_prunable = n_prunable;
  p.eps = seq_eps;
  p.out = static_cast<uint8_t*>(hidden_kept);
  p.pos = pos;
  p.bias = bias;
  p.ratio = ratio;
  const int rows_per_batch =
      static_cast<int>(std::min<int64_t>(tg::kGatherBatch, static_cast<int64_t>(tg::kGatherStageBytes / 2) / row_bytes));
  if (rows_per_batch >= 1) {
    // bulk copies: about eight rows per CTA, at most three CTAs per SM
    const int64_t want = (m + 7) / 8;
    const int64_t cap = 3 * static_cast<int64_t>(sm_count());
    const unsigned blocks = static_cast<unsigned>(want < cap ? want : cap);
    const size_t smem = static_cast<size_t>(2) * rows_per_batch * row_bytes;
    int rc = set_smem(tg::k_gather_bulk, smem);
    if (rc) return rc;
    return launch_pdl("k_gather_bulk", tg::k_gather_bulk, dim3(blocks), dim3(tg::kGatherBulkThreads), smem,
                      as_stream(stream), p, rows_per_batch);
  }
  const unsigned blocks = static_cast<unsigned>((m + tg::kGatherRows - 1) / tg::kGatherRows);
  return launch_pdl("k_gather", tg::k_gather, dim3(blocks), dim3(tg::kGatherThreads), 0, as_stream(stream), p);
}

// tg_gated_attention; counters_zeroed: the caller has already cleared the
// split-merge counters in ws (attn_counter_span) in an earlier kernel on the
// stream, so no memset is issued here
static int gated_attention_impl(const void* q, int64_t ldq, const void* k, int64_t ldk, const void* v, int64_t ldv,
                                int dtype, int64_t m, int32_t hq, int32_t hkv, int32_t head_dim, const float* bias,
                                const float* head_gain, const float* head_temp, const float* ratio, float sm_scale,
                                void* out, int64_t ldo, float* lse, void* ws, size_t ws_bytes, void* stream,
                                bool counters_zeroed) {
  if (!q || !k || !v || !out || !head_gain || !head_temp) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (m <= 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0) return fail(TG_ERR_INVALID_ARG, "bad m / heads");
  if (m >= (int64_t(1) << 31)) return fail(TG_ERR_UNSUPPORTED, "m must be < 2^31");
  if (head_dim != 64 && head_dim != 128) return fail(TG_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (ldq < int64_t(hq) * head_dim || ldk < int64_t(hkv) * head_dim || ldv < int64_t(hkv) * head_dim ||
      ldo < int64_t(hq) * head_dim)
    return fail(TG_ERR_SHAPE, "leading dimension smaller than the heads it holds");
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "dtype");
  cudaStream_t st = as_stream(stream);
  const int group = hq / hkv;
  if (dtype == TG_BF16) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || ldq % 8 || ldk % 8 || ldv % 8 ||
        ldo % 8)
      return fail(TG_ERR_ALIGN, "bf16 attention operands need 16-byte alignment");
  }
  if (dtype == TG_BF16 && group % 2 == 0) {
    tg::AttnTcParams p{};
    p.m = static_cast<int>(m);
    p.hq = hq;
    p.hkv = hkv;
    p.group = group;
    p.num_qtiles = static_cast<int>((m + 127) / 128);
    p.bias = bias;
    p.gain = head_gain;
    p.temp = head_temp;
    p.ratio = ratio;
    p.scale_log2 = sm_scale * 1.4426950408889634f;
    p.out = static_cast<__nv_bfloat16*>(out);
    p.ldo = ldo;
    p.lse = lse;
    CUtensorMap tq, tk, tv, tb, to;
    std::memset(&tb, 0, sizeof(tb));
    int rc = make_map(&tq, q, uint64_t(hq) * head_dim, uint64_t(m), uint64_t(ldq) * 2, 128);
    // the output tile of a head is stored by TMA from shared memory, 128 rows x 64 columns per box
    if (!rc) rc = make_map(&to, out, uint64_t(hq) * head_dim, uint64_t(m), uint64_t(ldo) * 2, 128);
    // keys and values come in tiles of AttnCfg::BN = 128 rows
    constexpr int kBN = tg::AttnCfg<128>::BN;
    if (!rc) rc = make_map(&tk, k, uint64_t(hkv) * head_dim, uint64_t(m), uint64_t(ldk) * 2, kBN);
    if (!rc) rc = make_map(&tv, v, uint64_t(hkv) * head_dim, uint64_t(m), uint64_t(ldv) * 2, kBN);
    if (rc) return rc;
    p.has_bias = bias != nullptr;
    if (bias) {
      if (!aligned16(bias)) return fail(TG_ERR_ALIGN, "bias must be 16-byte aligned");
      if ((rc = make_map_1d_f32(&tb, bias, uint64_t(m), kBN))) return rc;
    }
    // key-range split of the longest row blocks when a workspace is given
    const AttnPlan& pl = attn_plan(m, hkv, group, head_dim, sm_count());
    static thread_local tg::AttnWork work;  // 3.75 KiB: passed by value as a kernel parameter
    p.ts = p.num_qtiles;
    if (pl.table && ws && ws_bytes >= pl.bytes) {
      if (!aligned16(ws)) return fail(TG_ERR_ALIGN, "attention workspace must be 16-byte aligned");
      uint8_t* wb = static_cast<uint8_t*>(ws);
      p.use_table = 1;
      p.ts = pl.ts;
      p.part = reinterpret_cast<float4*>(wb + pl.part_off);
      p.part_ml = reinterpret_cast<float2*>(wb + pl.ml_off);
      p.counters = reinterpret_cast<unsigned*>(wb + pl.ctr_off);
      std::fill(std::begin(work.item), std::end(work.item), uint16_t(0));
      std::copy(pl.items.begin(), pl.items.end(), work.item);
      if (!counters_zeroed && cudaMemsetAsync(p.counters, 0, pl.bytes - pl.ctr_off, st) != cudaSuccess)
        return fail(TG_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(cudaGetLastError()));
    }
    const int items = p.use_table ? static_cast<int>(pl.items.size()) : p.num_qtiles;
    const unsigned blocks = static_cast<unsigned>(items * hkv * (group / 2));
    if (head_dim == 128) {
      rc = set_smem(tg::k_attn_tc<128>, tg::AttnCfg<128>::kSmem);
      if (rc) return rc;
      return launch_pdl("k_attn_tc", tg::k_attn_tc<128>, dim3(blocks), dim3(tg::kAttnThreads), tg::AttnCfg<128>::kSmem, st, tq, tk,
                        tv, tb, to, p, work);
    } else {
      rc = set_smem(tg::k_attn_tc<64>, tg::AttnCfg<64>::kSmem);
      if (rc) return rc;
      return launch_pdl("k_attn_tc", tg::k_attn_tc<64>, dim3(blocks), dim3(tg::kAttnThreads), tg::AttnCfg<64>::kSmem, st, tq, tk,
                        tv, tb, to, p, work);
    }
  }
  tg::AttnSimtParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.ldq = ldq;
  p.ldk = ldk;
  p.ldv = ldv;
  p.ldo = ldo;
  p.m = static_cast<int>(m);
  p.hq = hq;
  p.hkv = hkv;
  p.bias = bias;
  p.gain = head_gain;
  p.temp = head_temp;
  p.ratio = ratio;
  p.sm_scale = sm_scale;
  p.out = out;
  p.lse = lse;
  dim3 grid(static_cast<unsigned>((m + 15) / 16), static_cast<unsigned>(hq));
  if (dtype == TG_F32) {
    if (head_dim == 128) tg::k_attn_simt<float, 128><<<grid, 128, 0, st>>>(p);
    else tg::k_attn_simt<float, 64><<<grid, 128, 0, st>>>(p);
  } else {
    if (head_dim == 128) tg::k_attn_simt<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(p);
    else tg::k_attn_simt<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(p);
  }
  return check_launch("k_attn_simt");
}

int tg_gated_attention(const void* q, int64_t ldq, const void* k, int64_t ldk, const void* v, int64_t ldv, int dtype,
                       int64_t m, int32_t hq, int32_t hkv, int32_t head_dim, const float* bias,
                       const float* head_gain, const float* head_temp, const float* ratio, float sm_scale, void* out,
                       int64_t ldo, float* lse, void* ws, size_t ws_bytes, void* stream) {
  return gated_attention_impl(q, ldq, k, ldk, v, ldv, dtype, m, hq, hkv, head_dim, bias, head_gain, head_temp, ratio,
                              sm_scale, out, ldo, lse, ws, ws_bytes, stream, false);
}

// The split-merge counters a tensor-core attention call over m rows would use
// in ws (empty when it splits nothing or takes the CUDA-core path)
static ZeroSpan attn_counter_span(int64_t m, int32_t hq, int32_t hkv, int32_t head_dim, int dtype, void* ws,
                                  size_t ws_bytes) {
  ZeroSpan z;
  if (dtype != TG_BF16 || hkv <= 0 || hq % hkv || (hq / hkv) % 2 || !ws || !aligned16(ws)) return z;
  const AttnPlan& pl = attn_plan(m, hkv, hq / hkv, head_dim, sm_count());
  if (!pl.table || ws_bytes < pl.bytes) return z;
  z.p = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + pl.ctr_off);
  z.n = static_cast<int>((pl.bytes - pl.ctr_off) / 4);
  return z;
}

int tg_linear(const void* x, int64_t ldx, const void* w, void* y, int64_t ldy, int dtype, int64_t m, int32_t n_out,
              int32_t k_in, int epilogue, void* stream) {
  if (!x || !w || !y) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (m <= 0 || n_out <= 0 || k_in <= 0 || ldx < k_in || ldy < n_out) return fail(TG_ERR_INVALID_ARG, "bad sizes");
  if (epilogue < TG_EPI_STORE || epilogue > TG_EPI_SWIGLU) return fail(TG_ERR_INVALID_ARG, "epilogue");
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "dtype");
  if (m >= (int64_t(1) << 31)) return fail(TG_ERR_UNSUPPORTED, "m must be < 2^31");
  cudaStream_t st = as_stream(stream);
  const int mm = static_cast<int>(m);
  if (dtype == TG_BF16) {
    if (!aligned16(x) || !aligned16(w) || !aligned16(y) || ldx % 8 || ldy % 8 || k_in % 8)
      return fail(TG_ERR_ALIGN, "bf16 linear operands need 16-byte alignment");
    tg::GemmParams p{};
    p.N = n_out;
    p.out = static_cast<__nv_bfloat16*>(y);
    p.ldo = ldy;
    if (epilogue == TG_EPI_SWIGLU) {
      if (n_out % 128 != 0) return fail(TG_ERR_UNSUPPORTED, "SwiGLU epilogue needs n_out %% 128 == 0");
      p.up_row0 = n_out;
      return launch_gemm_auto<256, tg::kEpiSwiGLU>(x, ldx, w, 2 * int64_t(n_out), mm, k_in, n_out / 128, p, st);
    }
    if (n_out % 32 == 0) {
      const int gn = (n_out + 255) / 256;
      if (epilogue == TG_EPI_RESIDUAL)
        return launch_gemm_auto<256, tg::kEpiResidual>(x, ldx, w, n_out, mm, k_in, gn, p, st);
      return launch_gemm_auto<256, tg::kEpiStore>(x, ldx, w, n_out, mm, k_in, gn, p, st);
    }
  }
  if (epilogue == TG_EPI_SWIGLU) return fail(TG_ERR_UNSUPPORTED, "SwiGLU epilogue needs bf16");
  const bool res = epilogue == TG_EPI_RESIDUAL;
  dim3 grid(static_cast<unsigned>((n_out + 63) / 64), static_cast<unsigned>((m + 63) / 64));
  if (dtype == TG_F32) {
    const float* xa = static_cast<const float*>(x);
    const float* wa = static_cast<const float*>(w);
    float* ya = static_cast<float*>(y);
    if (res) tg::k_gemm_simt<float, true><<<grid, 256, 0, st>>>(xa, ldx, wa, ya, ldy, mm, n_out, k_in);
    else tg::k_gemm_simt<float, false><<<grid, 256, 0, st>>>(xa, ldx, wa, ya, ldy, mm, n_out, k_in);
  } else {
    using B = __nv_bfloat16;
    const B* xa = static_cast<const B*>(x);
    const B* wa = static_cast<const B*>(w);
    B* ya = static_cast<B*>(y);
    if (res) tg::k_gemm_simt<B, true><<<grid, 256, 0, st>>>(xa, ldx, wa, ya, ldy, mm, n_out, k_in);
    else tg::k_gemm_simt<B, false><<<grid, 256, 0, st>>>(xa, ldx, wa, ya, ldy, mm, n_out, k_in);
  }
  return check_launch("k_gemm_simt");
}

int tg_gated_attention_backward(const void* q, int64_t ldq, const void* k, int64_t ldk, const void* v, int64_t ldv,
                                const void* out, int64_t ldo, const void* dout, int64_t lddo, int dtype, int64_t m,
                                int32_t hq, int32_t hkv, int32_t head_dim, const float* bias, const float* head_gain,
                                const float* head_temp, const float* ratio, float sm_scale, const float* lse, float* dq,
                                float* dk, float* dv, float* dbias, float* dgain, float* dtemp, void* ws,
                                size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !out || !dout || !head_gain || !head_temp || !lse || !dq || !dk || !dv)
    return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (m <= 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0) return fail(TG_ERR_INVALID_ARG, "bad m / heads");
  if (m >= (int64_t(1) << 31)) return fail(TG_ERR_UNSUPPORTED, "m must be < 2^31");
  if (head_dim != 64 && head_dim != 128) return fail(TG_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "dtype");
  if (ldq < int64_t(hq) * head_dim || ldo < int64_t(hq) * head_dim || lddo < int64_t(hq) * head_dim ||
      ldk < int64_t(hkv) * head_dim || ldv < int64_t(hkv) * head_dim)
    return fail(TG_ERR_SHAPE, "leading dimension smaller than the heads it holds");
  tg_layer_shape sh{};
  sh.hq = hq;
  sh.hkv = hkv;
  sh.head_dim = head_dim;
  sh.dtype = dtype;
  const size_t need = tg_workspace_bytes(TG_OP_ATTENTION_BWD, 0, m, 0, 0, &sh);
  if (!ws || ws_bytes < need) return fail(TG_ERR_WORKSPACE, "attention backward needs %zu workspace bytes", need);
  if (!aligned16(ws)) return fail(TG_ERR_ALIGN, "workspace must be 16-byte aligned");
  cudaStream_t st = as_stream(stream);
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  tg::AttnBwdParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = out;
  p.dout = dout;
  p.ldq = ldq;
  p.ldk = ldk;
  p.ldv = ldv;
  p.ldo = ldo;
  p.lddo = lddo;
  p.m = static_cast<int>(m);
  p.hq = hq;
  p.hkv = hkv;
  p.group = hq / hkv;
  p.bias = bias;
  p.gain = head_gain;
  p.temp = head_temp;
  p.ratio = ratio;
  p.lse = lse;
  p.sm_scale = sm_scale;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dbias = dbias;
  p.dgain = dgain;
  p.dtemp = dtemp;
  p.nkb = static_cast<int>((m + tg::kBwdBlk - 1) / tg::kBwdBlk);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  p.rowdot = reinterpret_cast<float*>(wb);
  wb += al(size_t(hq) * m * 4);
  p.dbias_part = reinterpret_cast<float*>(wb);
  wb += al(size_t(hkv) * m * 4);
  p.dgt_part = reinterpret_cast<float*>(wb);
  wb += al(size_t(hq) * p.nkb * 2 * 4);
  p.m_pad = static_cast<int>((m + 127) / 128 * 128);
  p.rowpar = reinterpret_cast<float*>(wb);
  wb += al(size_t(hq) * p.m_pad * 16);
  p.kv_part = reinterpret_cast<float*>(wb);
  wb += al(size_t(hq) * p.m_pad * 2 * head_dim * 4);
  p.kv_ctr = reinterpret_cast<unsigned*>(wb);
  p.dbias_nparts = hkv;
  const int nqb = p.nkb;
  // bf16 operands that TMA can read go to the tensor cores
  const bool tc = dtype == TG_BF16 && aligned16(q) && aligned16(k) && aligned16(v) && aligned16(dout) &&
                  aligned16(out) && ldq % 8 == 0 && ldk % 8 == 0 && ldv % 8 == 0 && lddo % 8 == 0 &&
                  ldo % 8 == 0 && aligned16(dq) &&
                  aligned16(dk) && aligned16(dv) && (!bias || aligned16(bias));
  if (tc) {
    auto run_tc = [&](auto prep, auto kv, auto qk, size_t smem_kv, size_t smem_q, int D) -> int {
      CUtensorMap tq128, tdo128, tk64, tv64, tk128, tv128, tq64, tdo64, tb, tpar;
      std::memset(&tb, 0, sizeof(tb));
      int rc = make_map(&tq128, q, uint64_t(hq) * D, uint64_t(m), uint64_t(ldq) * 2, 128);
      if (!rc) rc = make_map(&tdo128, dout, uint64_t(hq) * D, uint64_t(m), uint64_t(lddo) * 2, 128);
      if (!rc) rc = make_map(&tq64, q, uint64_t(hq) * D, uint64_t(m), uint64_t(ldq) * 2, 64);
      if (!rc) rc = make_map(&tdo64, dout, uint64_t(hq) * D, uint64_t(m), uint64_t(lddo) * 2, 64);
      if (!rc) rc = make_map(&tk64, k, uint64_t(hkv) * D, uint64_t(m), uint64_t(ldk) * 2, 64);
      if (!rc) rc = make_map(&tv64, v, uint64_t(hkv) * D, uint64_t(m), uint64_t(ldv) * 2, 64);
      if (!rc) rc = make_map(&tk128, k, uint64_t(hkv) * D, uint64_t(m), uint64_t(ldk) * 2, 128);
      if (!rc) rc = make_map(&tv128, v, uint64_t(hkv) * D, uint64_t(m), uint64_t(ldv) * 2, 128);
      if (!rc && bias) rc = make_map_1d_f32(&tb, bias, uint64_t(m), 64);
      if (!rc) rc = make_map_1d_f32(&tpar, p.rowpar, uint64_t(hq) * p.m_pad * 4, 256);
      if (!rc) rc = set_smem(kv, smem_kv);
      if (!rc) rc = set_smem(qk, smem_q);
      if (rc) return rc;
      const int nqb128 = static_cast<int>((m + 127) / 128);
      // per-head dbias partials in the row-dot region; group tickets start at zero
      p.dbias_part = p.rowdot;
      p.dbias_nparts = hq;
      if (cudaMemsetAsync(p.kv_ctr, 0, 2 * size_t(hkv) * nqb128 * 4, st) != cudaSuccess)
        return fail(TG_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(cudaGetLastError()));
      prep<<<unsigned((p.m_pad + 7) / 8), 256, 0, st>>>(p);
      if ((rc = check_launch("k_attn_bwd_prep"))) return rc;
      kv<<<unsigned(hq * nqb128), tg::kBwdTcThreads, smem_kv, st>>>(tk128, tv128, tq64, tdo64, tpar, p);
      if ((rc = check_launch("k_attn_bwd_kv_tc"))) return rc;
      p.nkb = nqb128;  // dgain / dtemp partials per block of 128 rows
      qk<<<unsigned(hq * nqb128), tg::kBwdTcThreads, smem_q, st>>>(tq128, tdo128, tk64, tv64, tb, p);
      if ((rc = check_launch("k_attn_bwd_dq_tc"))) return rc;
      tg::k_attn_bwd_final<<<unsigned((std::max<int64_t>(m, hq) + 255) / 256), 256, 0, st>>>(p);
      return check_launch("k_attn_bwd_final");
    };
    return head_dim == 128
               ? run_tc(tg::k_attn_bwd_prep<128>, tg::k_attn_bwd_kv_tc<128>,
                        tg::k_attn_bwd_dq_tc<128>, tg::BwdKvCfg<128>::kSmem, tg::BwdDqCfg<128>::kSmem, 128)
               : run_tc(tg::k_attn_bwd_prep<64>, tg::k_attn_bwd_kv_tc<64>,
                        tg::k_attn_bwd_dq_tc<64>, tg::BwdKvCfg<64>::kSmem, tg::BwdDqCfg<64>::kSmem, 64);
  }
  auto run = [&](auto rowdot, auto kv, auto qk, int D) -> int {
    const size_t DP = size_t(D) + 1;
    const size_t smem_kv = (4 * tg::kBwdBlk * DP + 3 * tg::kBwdBlk * (tg::kBwdBlk + 1) + tg::kBwdThreads) * 4;
    const size_t smem_q = (4 * tg::kBwdBlk * DP + tg::kBwdBlk * (tg::kBwdBlk + 1)) * 4;
    int rc = set_smem(kv, smem_kv);
    if (!rc) rc = set_smem(qk, smem_q);
    if (rc) return rc;
    rowdot<<<unsigned((m * hq + 7) / 8), 256, 0, st>>>(p);
    if ((rc = check_launch("k_attn_bwd_rowdot"))) return rc;
    kv<<<unsigned(hkv * p.nkb), tg::kBwdThreads, smem_kv, st>>>(p);
    if ((rc = check_launch("k_attn_bwd_kv"))) return rc;
    qk<<<unsigned(hq * nqb), tg::kBwdThreads, smem_q, st>>>(p);
    if ((rc = check_launch("k_attn_bwd_q"))) return rc;
    tg::k_attn_bwd_final<<<unsigned((std::max<int64_t>(m, hq) + 255) / 256), 256, 0, st>>>(p);
    return check_launch("k_attn_bwd_final");
  };
  if (dtype == TG_BF16)
    return head_dim == 128 ? run(tg::k_attn_bwd_rowdot<__nv_bfloat16, 128>, tg::k_attn_bwd_kv<__nv_bfloat16, 128>,
                                 tg::k_attn_bwd_q<__nv_bfloat16, 128>, 128)
                           : run(tg::k_attn_bwd_rowdot<__nv_bfloat16, 64>, tg::k_attn_bwd_kv<__nv_bfloat16, 64>,
                                 tg::k_attn_bwd_q<__nv_bfloat16, 64>, 64);
  return head_dim == 128 ? run(tg::k_attn_bwd_rowdot<float, 128>, tg::k_attn_bwd_kv<float, 128>,
                               tg::k_attn_bwd_q<float, 128>, 128)
                         : run(tg::k_attn_bwd_rowdot<float, 64>, tg::k_attn_bwd_kv<float, 64>,
                               tg::k_attn_bwd_q<float, 64>, 64);
}

float tg_decode_temperature_ratio(int64_t m_kept, int64_t n_prompt, int64_t t) {
  if (m_kept < 0 || n_prompt < 0 || t < 0) return 0.0f;
  const double m = static_cast<double>(m_kept + t + 1), p = static_cast<double>(n_prompt + t + 1);
  return static_cast<float>(std::log(m) / std::log(std::max(2.0, p)));
}

int tg_gated_decode_attention(const void* q, const void* k, int64_t ldk, const void* v, int64_t ldv, int dtype,
                              int64_t length, int32_t hq, int32_t hkv, int32_t head_dim, const float* bias,
                              const float* head_gain, const float* head_temp, float ratio, float sm_scale, void* out,
                              float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !out || !head_gain || !head_temp) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (length <= 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0) return fail(TG_ERR_INVALID_ARG, "bad length / heads");
  if (length > int64_t(tg::kDecMaxChunks) * tg::kDecMaxChunk)
    return fail(TG_ERR_UNSUPPORTED, "cache length must be <= %d", tg::kDecMaxChunks * tg::kDecMaxChunk);
  if (head_dim != 64 && head_dim != 128) return fail(TG_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (hq / hkv > tg::kDecMaxGroup) return fail(TG_ERR_UNSUPPORTED, "at most %d query heads per KV head", tg::kDecMaxGroup);
  if (dtype != TG_F32 && dtype != TG_BF16) return fail(TG_ERR_INVALID_ARG, "dtype");
  if (ldk < int64_t(hkv) * head_dim || ldv < int64_t(hkv) * head_dim)
    return fail(TG_ERR_SHAPE, "leading dimension smaller than the heads it holds");
  const int es = dtype_size(dtype);
  if (!aligned16(k) || !aligned16(v) || (ldk * es) % 16 || (ldv * es) % 16)
    return fail(TG_ERR_ALIGN, "cache rows need 16-byte alignment");
  const int group = hq / hkv;
  // bf16 caches stream through shared memory by TMA (16-byte aligned rows,
  // checked above, and a 16-byte aligned bias vector); fp32 caches take the
  // CUDA-core kernel
  const bool tma = dtype == TG_BF16 && (!bias || aligned16(bias)) && !force_simt_decode();
  const DecodePlan pl = decode_plan(length, hkv, group, head_dim, tma);
  const size_t need = decode_ws_bytes(length, hkv, group, head_dim);
  if (!ws || ws_bytes < need) return fail(TG_ERR_WORKSPACE, "decode attention needs %zu workspace bytes", need);
  if (!aligned16(ws)) return fail(TG_ERR_ALIGN, "workspace must be 16-byte aligned");
  cudaStream_t st = as_stream(stream);
  tg::DecodeParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.ldk = ldk;
  p.ldv = ldv;
  p.length = static_cast<int>(length);
  p.hq = hq;
  p.hkv = hkv;
  p.group = group;
  p.chunk = pl.chunk;
  p.nchunks = pl.nchunks;
  p.bias = bias;
  p.gain = head_gain;
  p.temp = head_temp;
  p.ratio_scale_log2 = ratio * sm_scale * tg::kLog2e;
  p.out = out;
  p.lse = lse;
  p.part = static_cast<float*>(ws);
  p.counters = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) + pl.part_bytes);
  if (cudaMemsetAsync(p.counters, 0, pl.bytes - pl.part_bytes, st) != cudaSuccess)
    return fail(TG_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(cudaGetLastError()));
  const dim3 grid(static_cast<unsigned>(hkv * pl.nchunks));
  if (tma) return head_dim == 128 ? launch_decode_tma<128>(group, grid, st, p) : launch_decode_tma<64>(group, grid, st, p);
  if (dtype == TG_BF16)
    return head_dim == 128 ? launch_decode<__nv_bfloat16, 128>(group, grid, st, p)
                           : launch_decode<__nv_bfloat16, 64>(group, grid, st, p);
  return head_dim == 128 ? launch_decode<float, 128>(group, grid, st, p) : launch_decode<float, 64>(group, grid, st, p);
}

int tg_pruned_prefill_layer(const tg_layer_weights* W, const tg_layer_shape* S, void* hidden_kept,
                            const int32_t* pos, const float* bias, const float* ratio, int64_t m, void* ws,
                            size_t ws_bytes, void* stream) {
  return prefill_layer_impl(W, S, TG_LAYER_FULL, hidden_kept, pos, bias, ratio, m, nullptr, 0, nullptr, ws, ws_bytes,
                            stream);
}

int tg_layer_attention_block(const tg_layer_weights* W, const tg_layer_shape* S, void* hidden, const int32_t* pos,
                             const float* bias, const float* ratio, int64_t m, void* ws, size_t ws_bytes,
                             void* stream) {
  return prefill_layer_impl(W, S, TG_LAYER_ATTENTION, hidden, pos, bias, ratio, m, nullptr, 0, nullptr, ws, ws_bytes,
                            stream);
}

int tg_layer_mlp_block(const tg_layer_weights* W, const tg_layer_shape* S, void* hidden, int64_t m, void* ws,
                       size_t ws_bytes, void* stream) {
  return prefill_layer_impl(W, S, TG_LAYER_MLP, hidden, nullptr, nullptr, nullptr, m, nullptr, 0, nullptr, ws,
                            ws_bytes, stream);
}

int tg_gather_rmsnorm(const void* hidden, int dtype, int64_t n, int32_t d_model, const int32_t* kept_idx, int64_t m,
                      const float* scores, const float* sumsq, int64_t n_prunable, float seq_eps, const float* norm_w,
                      float norm_eps, void* hidden_kept, void* x_norm, int32_t* pos, float* bias, float* ratio,
                      void* stream) {
  if (!hidden || !kept_idx || !hidden_kept || !x_norm) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (bias && (!scores || !sumsq)) return fail(TG_ERR_INVALID_ARG, "bias needs scores and sumsq");
  if (n <= 0 || m <= 0 || m > n || d_model <= 0) return fail(TG_ERR_INVALID_ARG, "bad sizes");
  if (bias && n_prunable <= 0) return fail(TG_ERR_INVALID_ARG, "n_prunable must be > 0 for bias");
  const int es = dtype_size(dtype);
  if (!es) return fail(TG_ERR_INVALID_ARG, "dtype");
  if ((int64_t(d_model) * es) % 16 != 0 || !aligned16(hidden) || !aligned16(hidden_kept) || !aligned16(x_norm))
    return fail(TG_ERR_ALIGN, "rows must be 16-byte multiples on 16-byte aligned buffers");
  const LayerGather g{hidden, n, kept_idx, scores, sumsq, n_prunable, seq_eps, pos, bias, ratio};
  return launch_gather_rmsnorm(g, dtype, hidden_kept, x_norm, norm_w, m, d_model, norm_eps, as_stream(stream),
                               ZeroSpan{});
}

int tg_gather_prefill_layer(const tg_layer_weights* W, const tg_layer_shape* S, int part, const void* hidden,
                            int64_t n, const int32_t* kept_idx, int64_t m, const float* scores, const float* sumsq,
                            int64_t n_prunable, float seq_eps, void* hidden_kept, int32_t* pos, float* bias,
                            float* ratio, void* ws, size_t ws_bytes, void* stream) {
  if (part != TG_LAYER_FULL && part != TG_LAYER_MLP) return fail(TG_ERR_INVALID_ARG, "part must be full or MLP");
  if (!hidden || !kept_idx || !hidden_kept) return fail(TG_ERR_INVALID_ARG, "null pointer");
  if (part == TG_LAYER_FULL && !pos) return fail(TG_ERR_INVALID_ARG, "the attention half needs pos");
  if (bias && (!scores || !sumsq)) return fail(TG_ERR_INVALID_ARG, "bias needs scores and sumsq");
  if (n <= 0 || m <= 0 || m > n) return fail(TG_ERR_INVALID_ARG, "bad sizes");
  if (bias && n_prunable <= 0) return fail(TG_ERR_INVALID_ARG, "n_prunable must be > 0 for bias");
  if (!aligned16(hidden) || !aligned16(hidden_kept)) return fail(TG_ERR_ALIGN, "rows must be 16-byte aligned");
  const LayerGather g{hidden, n, kept_idx, scores, sumsq, n_prunable, seq_eps, pos, bias, ratio};
  return prefill_layer_impl(W, S, part, hidden_kept, pos, bias, ratio, m, nullptr, 0, &g, ws, ws_bytes, stream);
}

size_t tg_layer_varlen_workspace_bytes(const tg_layer_shape* shape, const int64_t* seg_rows, int32_t nseg) {
  if (!shape || !seg_rows || nseg <= 0 || seg_rows[0] != 0) return 0;
  int64_t longest = 0;
  for (int32_t r = 0; r < nseg; ++r) {
    if (seg_rows[r + 1] < seg_rows[r]) return 0;
    longest = std::max(longest, seg_rows[r + 1] - seg_rows[r]);
  }
  const int64_t m = seg_rows[nseg];
  if (m <= 0 || !dtype_size(shape->dtype)) return 0;
  // + a staging copy of one request's key bias: attention loads the bias with
  // TMA, which needs a 16-byte aligned start, and a request's rows may begin anywhere
  return layer_buffers_bytes(m, shape) + attn_ws_bytes(longest, shape->hq, shape->hkv, shape->head_dim, shape->dtype) +
         (static_cast<size_t>(longest) * sizeof(float) + 255) / 256 * 256;
}

int tg_pruned_prefill_layer_varlen(const tg_layer_weights* W, const tg_layer_shape* S, void* hidden_kept,
                                   const int32_t* pos, const float* bias, const float* ratio,
                                   const int64_t* seg_rows, int32_t nseg, void* ws, size_t ws_bytes, void* stream) {
  if (!seg_rows || nseg <= 0) return fail(TG_ERR_INVALID_ARG, "segments");
  if (seg_rows[0] != 0) return fail(TG_ERR_INVALID_ARG, "seg_rows[0] must be 0");
  for (int32_t r = 0; r < nseg; ++r)
    if (seg_rows[r + 1] < seg_rows[r]) return fail(TG_ERR_INVALID_ARG, "seg_rows must not decrease");
  return prefill_layer_impl(W, S, TG_LAYER_FULL, hidden_kept, pos, bias, ratio, seg_rows[nseg], seg_rows, nseg,
                            nullptr, ws, ws_bytes, stream);
}

}  // extern "C"

static int mlp_half(const tg_layer_weights* W, const tg_layer_shape* S, void* hidden_kept, void* xn, void* act,
                    int64_t m, void* stream);

// The gather fused with an RMSNorm (k_gather_rmsnorm_warp): rows whose 16-byte
// vectors fit a warp's registers; other shapes gather first and normalise after.
static int launch_gather_rmsnorm(const LayerGather& g, int dtype, void* hidden_kept, void* xn, const float* w,
                                 int64_t m, int d, float eps, cudaStream_t st, ZeroSpan z) {
  const int es = dtype_size(dtype);
  tg::GatherParams p{};
  p.zero = z.p;
  p.zero_n = z.n;
  p.hidden = static_cast<const uint8_t*>(g.hidden);
  p.n = g.n;
  p.row_bytes = int64_t(d) * es;
  p.idx = g.idx;
  p.m = m;
  p.scores = g.scores;
  p.sumsq = g.sumsq;
  p.n_prunable = g.n_prunable;
  p.eps = g.seq_eps;
  p.out = static_cast<uint8_t*>(hidden_kept);
  p.pos = g.pos;
  p.bias = g.bias;
  p.ratio = g.ratio;
  const int nv = d * es / 16;
  const dim3 grid(unsigned((m + 7) / 8)), block(256);
  if (!w || aligned16(w)) {
    if (dtype == TG_BF16) {
      auto* y = static_cast<__nv_bfloat16*>(xn);
      if (nv <= 32 * 4) return launch_pdl("k_gather_rmsnorm_warp", tg::k_gather_rmsnorm_warp<__nv_bfloat16, 4>, grid, block, 0, st, p, y, w, d, eps);
      if (nv <= 32 * 8) return launch_pdl("k_gather_rmsnorm_warp", tg::k_gather_rmsnorm_warp<__nv_bfloat16, 8>, grid, block, 0, st, p, y, w, d, eps);
      if (nv <= 32 * 16) return launch_pdl("k_gather_rmsnorm_warp", tg::k_gather_rmsnorm_warp<__nv_bfloat16, 16>, grid, block, 0, st, p, y, w, d, eps);
    } else {
      auto* y = static_cast<float*>(xn);
      if (nv <= 32 * 4) return launch_pdl("k_gather_rmsnorm_warp", tg::k_gather_rmsnorm_warp<float, 4>, grid, block, 0, st, p, y, w, d, eps);
      if (nv <= 32 * 8) return launch_pdl("k_gather_rmsnorm_warp", tg::k_gather_rmsnorm_warp<float, 8>, grid, block, 0, st, p, y, w, d, eps);
      if (nv <= 32 * 16) return launch_pdl("k_gather_rmsnorm_warp", tg::k_gather_rmsnorm_warp<float, 16>, grid, block, 0, st, p, y, w, d, eps);
    }
  }
  int rc = tg_gather(g.hidden, dtype, g.n, d, g.idx, m, g.scores, g.sumsq, g.n_prunable, g.seq_eps, hidden_kept, g.pos,
                     g.bias, g.ratio, st);
  if (rc) return rc;
  return dtype == TG_BF16 ? launch_rmsnorm<__nv_bfloat16>(hidden_kept, xn, w, m, d, eps, st, z)
                          : launch_rmsnorm<float>(hidden_kept, xn, w, m, d, eps, st, z);
}

// One decoder layer over m rows; with seg_rows (host, nseg + 1 offsets) the
// rows are nseg independent requests and attention runs per request.
static int prefill_layer_impl(const tg_layer_weights* W, const tg_layer_shape* S, int parts, void* hidden_kept,
                              const int32_t* pos, const float* bias, const float* ratio, int64_t m,
                              const int64_t* seg_rows, int32_t nseg, const LayerGather* gather, void* ws,
                              size_t ws_bytes, void* stream) {
  if (!W || !S || !hidden_kept) return fail(TG_ERR_INVALID_ARG, "null pointer");
  const bool do_attn = (parts & TG_LAYER_ATTENTION) != 0, do_mlp = (parts & TG_LAYER_MLP) != 0;
  if (do_attn && (!W->w_in_norm || !W->w_qkv || !W->w_o || !W->head_gain || !W->head_temp))
    return fail(TG_ERR_INVALID_ARG, "null weight pointer");
  if (do_mlp && (!W->w_post_norm || !W->w_gate_up || !W->w_down)) return fail(TG_ERR_INVALID_ARG, "null weight pointer");
  if (do_attn && !pos) return fail(TG_ERR_INVALID_ARG, "null pointer (pos)");
  if (do_attn && S->qk_norm && (!W->w_q_norm || !W->w_k_norm)) return fail(TG_ERR_INVALID_ARG, "qk_norm needs its weights");
  if (m <= 0 || S->d_model <= 0 || S->hq <= 0 || S->hkv <= 0 || S->hq % S->hkv || S->d_ff <= 0)
    return fail(TG_ERR_INVALID_ARG, "bad layer shape");
  if (S->head_dim != 64 && S->head_dim != 128) return fail(TG_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  const int es = dtype_size(S->dtype);
  if (!es) return fail(TG_ERR_INVALID_ARG, "dtype");
  if ((S->d_model * es) % 16 != 0) return fail(TG_ERR_UNSUPPORTED, "d_model rows must be a multiple of 16 bytes");
  const size_t need = seg_rows ? tg_layer_varlen_workspace_bytes(S, seg_rows, nseg)
                               : tg_workspace_bytes(TG_OP_LAYER, 0, m, 0, 0, S);
  if (!ws || ws_bytes < need) return fail(TG_ERR_WORKSPACE, "layer needs %zu workspace bytes", need);
  cudaStream_t st = as_stream(stream);
  const int d = S->d_model, D = S->head_dim, hq = S->hq, hkv = S->hkv, dff = S->d_ff;
  const int64_t qkv_w = int64_t(hq + 2 * hkv) * D;
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  uint8_t* base = static_cast<uint8_t*>(ws);
  void* xn = base;
  base += al(size_t(m) * d * es);
  void* qkv = base;
  base += al(size_t(m) * qkv_w * es);
  void* att = base;
  base += al(size_t(m) * hq * D * es);
  void* act = base;
  base += al(size_t(m) * dff * 2 * es);
  void* attn_ws = base;
  int64_t longest = m;
  if (seg_rows) {
    longest = 0;
    for (int32_t r = 0; r < nseg; ++r) longest = std::max(longest, seg_rows[r + 1] - seg_rows[r]);
  }
  const size_t bias_stage_sz = seg_rows ? (static_cast<size_t>(longest) * sizeof(float) + 255) / 256 * 256 : 0;
  const size_t attn_ws_sz = need - layer_buffers_bytes(m, S) - bias_stage_sz;
  float* bias_stage = reinterpret_cast<float*>(static_cast<uint8_t*>(attn_ws) + attn_ws_sz);
  const bool bf = S->dtype == TG_BF16;
  int rc;
  // the first RMSNorm of the parts run here: from the rows in place, or
  // gathering them from the full sequence in the same pass
  auto first_norm = [&](const float* w, ZeroSpan z) -> int {
    if (!gather)
      return bf ? launch_rmsnorm<__nv_bfloat16>(hidden_kept, xn, w, m, d, S->norm_eps, st, z)
                : launch_rmsnorm<float>(hidden_kept, xn, w, m, d, S->norm_eps, st, z);
    return launch_gather_rmsnorm(*gather, S->dtype, hidden_kept, xn, w, m, d, S->norm_eps, st, z);
  };
  if (!do_attn) {
    if ((rc = first_norm(W->w_post_norm, ZeroSpan{}))) return rc;
    return mlp_half(W, S, hidden_kept, xn, act, m, stream);
  }
  // the attention split-merge counters of a single request are cleared by the
  // layer's first kernel, so no memset node sits between the q/k-norm kernel
  // and attention (it would stop attention's launch from overlapping it)
  const ZeroSpan attn_ctr =
      seg_rows ? ZeroSpan{} : attn_counter_span(m, hq, hkv, D, S->dtype, attn_ws_sz ? attn_ws : nullptr, attn_ws_sz);
  // 1. x = RMSNorm(h)
  if ((rc = first_norm(W->w_in_norm, attn_ctr))) return rc;
  // 2. qkv = x Wqkv^T
  if ((rc = tg_linear(xn, d, W->w_qkv, qkv, qkv_w, S->dtype, m, int32_t(qkv_w), d, TG_EPI_STORE, stream))) return rc;
  // 3. per-head q/k norm and RoPE at the original positions (one warp per row)
  {
    tg::RopeTable tab{};
    for (int i = 0; i < D / 2; ++i) tab.inv_freq[i] = std::pow(static_cast<double>(S->rope_theta), -2.0 * i / D);
    const unsigned blocks = unsigned((m + 7) / 8);
    const dim3 g(blocks), b(256);
    if (bf) {
      auto* x = static_cast<__nv_bfloat16*>(qkv);
      rc = D == 128 ? launch_pdl("k_qk_norm_rope_warp", tg::k_qk_norm_rope_warp<__nv_bfloat16, 128>, g, b, 0, st, x,
                                 qkv_w, int(m), hq, hkv, pos, W->w_q_norm, W->w_k_norm, S->qk_norm, S->norm_eps, tab)
                    : launch_pdl("k_qk_norm_rope_warp", tg::k_qk_norm_rope_warp<__nv_bfloat16, 64>, g, b, 0, st, x,
                                 qkv_w, int(m), hq, hkv, pos, W->w_q_norm, W->w_k_norm, S->qk_norm, S->norm_eps, tab);
    } else {
      auto* x = static_cast<float*>(qkv);
      rc = D == 128 ? launch_pdl("k_qk_norm_rope_warp", tg::k_qk_norm_rope_warp<float, 128>, g, b, 0, st, x, qkv_w,
                                 int(m), hq, hkv, pos, W->w_q_norm, W->w_k_norm, S->qk_norm, S->norm_eps, tab)
                    : launch_pdl("k_qk_norm_rope_warp", tg::k_qk_norm_rope_warp<float, 64>, g, b, 0, st, x, qkv_w,
                                 int(m), hq, hkv, pos, W->w_q_norm, W->w_k_norm, S->qk_norm, S->norm_eps, tab);
    }
    if (rc) return rc;
  }
  // 4. token-gated attention, request by request (rows of one request only
  //    see keys of the same request)
  for (int32_t r = 0; r < (seg_rows ? nseg : 1); ++r) {
    const int64_t r0 = seg_rows ? seg_rows[r] : 0, mr = seg_rows ? seg_rows[r + 1] - r0 : m;
    if (mr == 0) continue;
    const uint8_t* qb = static_cast<const uint8_t*>(qkv) + r0 * qkv_w * es;
    uint8_t* ab = static_cast<uint8_t*>(att) + r0 * int64_t(hq) * D * es;
    const float* br = bias ? bias + r0 : nullptr;
    if (br && !aligned16(br)) {
      if (cudaMemcpyAsync(bias_stage, br, size_t(mr) * sizeof(float), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return fail(TG_ERR_CUDA, "bias staging copy: %s", cudaGetErrorString(cudaGetLastError()));
      br = bias_stage;
    }
    if ((rc = gated_attention_impl(qb, qkv_w, qb + int64_t(hq) * D * es, qkv_w, qb + int64_t(hq + hkv) * D * es,
                                   qkv_w, S->dtype, mr, hq, hkv, D, br, W->head_gain, W->head_temp,
                                   ratio ? ratio + r0 : nullptr, 1.0f / sqrtf(float(D)), ab, int64_t(hq) * D, nullptr,
                                   attn_ws_sz ? attn_ws : nullptr, attn_ws_sz, stream, attn_ctr.n > 0)))
      return rc;
  }
  // 5. h += a Wo^T
  if ((rc = tg_linear(att, int64_t(hq) * D, W->w_o, hidden_kept, d, S->dtype, m, d, hq * D, TG_EPI_RESIDUAL, stream)))
    return rc;
  if (!do_mlp) return TG_OK;
  // 6. y = RMSNorm(h)
  rc = bf ? launch_rmsnorm<__nv_bfloat16>(hidden_kept, xn, W->w_post_norm, m, d, S->norm_eps, st)
          : launch_rmsnorm<float>(hidden_kept, xn, W->w_post_norm, m, d, S->norm_eps, st);
  if (rc) return rc;
  return mlp_half(W, S, hidden_kept, xn, act, m, stream);
}

// Steps 7-8 of the layer on rows already normalised into xn: act = SiLU(y Wg^T)
// * (y Wu^T), h += act Wd^T.
static int mlp_half(const tg_layer_weights* W, const tg_layer_shape* S, void* hidden_kept, void* xn, void* act,
                    int64_t m, void* stream) {
  cudaStream_t st = as_stream(stream);
  const int d = S->d_model, dff = S->d_ff;
  const bool bf = S->dtype == TG_BF16;
  int rc;
  // 7. act = SiLU(y Wg^T) * (y Wu^T)
  if (bf && dff % 128 == 0) {
    if ((rc = tg_linear(xn, d, W->w_gate_up, act, dff, S->dtype, m, dff, d, TG_EPI_SWIGLU, stream))) return rc;
  } else {
    // un-fused: gate/up product into the activation buffer, then SiLU(g) * u
    // written over the gate half of each row (every element reads only its
    // own gate/up pair), and the down projection reads rows of stride 2*d_ff
    void* gu = act;
    if ((rc = tg_linear(xn, d, W->w_gate_up, gu, 2 * int64_t(dff), S->dtype, m, 2 * dff, d, TG_EPI_STORE, stream)))
      return rc;
    const int64_t total = m * dff;
    const unsigned blocks = unsigned((total + 255) / 256);
    if (bf)
      tg::k_swiglu<__nv_bfloat16><<<blocks, 256, 0, st>>>(static_cast<__nv_bfloat16*>(gu), m, dff);
    else
      tg::k_swiglu<float><<<blocks, 256, 0, st>>>(static_cast<float*>(gu), m, dff);
    if ((rc = check_launch("k_swiglu"))) return rc;
    return tg_linear(gu, 2 * int64_t(dff), W->w_down, hidden_kept, d, S->dtype, m, d, dff, TG_EPI_RESIDUAL, stream);
  }
  // 8. h += act Wd^T
  return tg_linear(act, dff, W->w_down, hidden_kept, d, S->dtype, m, d, dff, TG_EPI_RESIDUAL, stream);
}

// ---------------------------------------------------------------------------
// Gate scores without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they score a
// prompt: a serving runtime that hands the library only the tensors of the
// request and owns every other byte of HBM through its own pool, a plugin
// host whose interface has no workspace argument, or a latency-critical path
// that must not take cudaMalloc's implicit device-wide synchronisation.  For
// them tg_gate_score_noalloc keeps its scratch (per-CTA partial sums, the
// completion counter and the norm-folded W1) in a fixed array compiled into
// the library instead of in `ws`.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = (2u << 20) + (64u << 10);  // 2 MiB + 64 KiB per device
constexpr int kNoAllocMaxDevices = 64;

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_gate_scratch[kNoAllocScratchBytes];

std::mutex g_gate_scratch_mu;
void* g_gate_scratch_addr[kNoAllocMaxDevices] = {};

// Device address of g_gate_scratch on the current device.  Host code cannot
// use the symbol itself (on the host it names a stand-in, not device memory),
// so the address is looked up once per device, with that device current.
int gate_scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(TG_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(TG_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_gate_scratch_mu);
  if (!g_gate_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gate_scratch);
    if (e != cudaSuccess || !p) return fail(TG_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_gate_scratch_addr[dev] = p;
  }
  *out = g_gate_scratch_addr[dev];
  return TG_OK;
}

}  // namespace

extern "C" {

int tg_gate_score_noalloc(const void* hidden, int dtype, int64_t n, int32_t d_model, const float* norm_w,
                          float norm_eps, const void* w1, const float* b1, const float* w2, float b2, int32_t h,
                          const uint8_t* prunable, float* scores, float* sumsq, void* stream) {
  if (n > 0 && d_model > 0 && h > 0 && gate_uses_tc(hidden, dtype, d_model, w1, h)) {
    // only the tensor-core path uses scratch; the CUDA-core path needs none
    const size_t need = gate_ws_bytes(n, d_model, h);
    if (need > kNoAllocScratchBytes)
      return fail(TG_ERR_UNSUPPORTED,
                  "tg_gate_score_noalloc: n = %lld, d_model = %d, h = %d need %zu scratch bytes, more than the "
                  "%zu built into the library (n/32 + 2*d_model*h bytes must stay below it); use tg_gate_score "
                  "with a workspace",
                  static_cast<long long>(n), d_model, h, need, kNoAllocScratchBytes);
  }
  void* scratch = nullptr;
  const int rc = gate_scratch_address(&scratch);
  if (rc) return rc;
  return tg_gate_score(hidden, dtype, n, d_model, norm_w, norm_eps, w1, b1, w2, b2, h, prunable, scores, sumsq,
                       scratch, kNoAllocScratchBytes, stream);
}

size_t tg_gate_score_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

}  // extern "C"
