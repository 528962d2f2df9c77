// awq_lib.cu — the C ABI of libawq_w4a16 (declared in include/awq_w4a16.h).
//
// Host side only: argument checks, launch configuration, TMA descriptors and
// the device status word. Every step of the path runs in the kernels
// included below; there is no host or CPU fallback.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "awq_act.cuh"
#include "awq_common.cuh"
#include "awq_gemm.cuh"
#include "awq_gemv.cuh"
#include "awq_quant.cuh"
#include "awq_w4a16.h"

namespace awq {

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::atomic<int> state{0};   // 0 unknown, 1 supported, 2 unsupported
  int num_sms = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mutex;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device, checked to be compute capability 10.0 (B200 / sm_100a).
awq_status_t current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return AWQ_ERR_UNSUPPORTED;
  DeviceInfo& d = g_devices[dev];
  int st = d.state.load(std::memory_order_acquire);
  if (st == 0) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    st = d.state.load(std::memory_order_relaxed);
    if (st == 0) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return AWQ_ERR_CUDA;
      d.num_sms = sms;
      st = (major == 10 && minor == 0) ? 1 : 2;
      d.state.store(st, std::memory_order_release);
    }
  }
  if (st != 1) return AWQ_ERR_UNSUPPORTED;
  *dev_out = dev;
  if (sms_out) *sms_out = d.num_sms;
  return AWQ_OK;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
template <typename Kernel>
awq_status_t ensure_smem(Kernel kernel, int bytes, int dev, std::atomic<uint64_t>& done_mask) {
  const uint64_t bit = 1ull << dev;
  if (done_mask.load(std::memory_order_acquire) & bit) return AWQ_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return AWQ_ERR_CUDA;
  done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return AWQ_OK;
}

// --------------------------------------------------------------------------- TMA descriptor
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// x' [M, K] fp16 row-major, box {64 k, BT tokens}, 128-byte swizzle, zero fill out of bounds.
awq_status_t make_x_map(CUtensorMap* map, const void* x, int M, int K, int BT) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return AWQ_ERR_CUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kKTile), static_cast<cuuint32_t>(BT)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? AWQ_OK : AWQ_ERR_CUDA;
}

// --------------------------------------------------------------------------- launch helper
// Every kernel is launched with programmatic stream serialization (PDL): it may start while the
// previous kernel of the stream drains, runs its prologue, and waits (griddepcontrol.wait) before
// touching global memory. cluster_y > 1 adds a (1, cluster_y, 1) thread-block cluster.
template <typename... KArgs, typename... Args>
awq_status_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, int cluster_y, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster_y > 0) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = static_cast<unsigned>(cluster_y);
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
    cudaGetLastError();
    return AWQ_ERR_CUDA;
  }
  return AWQ_OK;
}

// --------------------------------------------------------------------------- decode dispatch
// Max co-resident clusters of a kernel for a cluster size and a dynamic shared-memory size;
// cached (per kernel instantiation) because the occupancy query costs host time.
struct ClusterOccCache {
  std::mutex mu;
  struct Entry { int dev, cl; size_t smem; int clusters; };
  Entry e[256];
  int n = 0;
};
template <typename Kernel>
int max_active_clusters(Kernel kernel, int threads, size_t smem, int cl, int dev, ClusterOccCache& cache) {
  {
    std::lock_guard<std::mutex> lock(cache.mu);
    for (int i = 0; i < cache.n; ++i)
      if (cache.e[i].dev == dev && cache.e[i].cl == cl && cache.e[i].smem == smem) return cache.e[i].clusters;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cl, cl, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(cl);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lock(cache.mu);
  if (cache.n < 256) cache.e[cache.n++] = {dev, cl, smem, n};
  return n;
}

template <int MT, int S, int KS, int CW, bool kSumX = false>
awq_status_t launch_gemv_cfg(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr, __half* y,
                             int M, int N, int K, int dev, int num_sms, cudaStream_t stream) {
  using Cfg = GemvCfg<MT, S, KS, CW>;
  static_assert(!kSumX || MT == 1, "activation sums are taken for tokens 0 and 1 only");
  auto kernel = gemv_kernel<MT, S, KS, CW, kSumX>;
  constexpr int kMaxSmem = 227 * 1024;
  static std::atomic<uint64_t> smem_done{0};
  awq_status_t st = ensure_smem(kernel, kMaxSmem, dev, smem_done);
  if (st != AWQ_OK) return st;
  CUtensorMap map;
  st = make_x_map(&map, x, M, K, Cfg::kMP);
  if (st != AWQ_OK) return st;
  const int NST = padded_rows(N) / kSuperRows;
  const int G = K / kGroup;
  static ClusterOccCache cache;
  // For each cluster size (K-split), find the co-resident cluster count C whose per-CTA partial
  // buffers (ceil(NST / C) super-tiles) still let C clusters fit; cost = rounds x K-slice + a
  // constant for the final reduction. The stream never synchronises before the end.
  int best_cl = 0, best_clusters = 0, best_units = 0;
  double best_cost = 1e300;
  for (int cl = 1; cl <= 8; cl *= 2) {
    if (cl > G) break;
#ifdef AWQ_GEMV_FORCE_CL
    if (cl != AWQ_GEMV_FORCE_CL) continue;
#endif
    int clusters = max_active_clusters(kernel, Cfg::kThreads, Cfg::smem_bytes(M, 1), cl, dev, cache);
    int units = 0;
    for (int it = 0; it < 6 && clusters > 0; ++it) {
      clusters = std::min(clusters, NST);
      units = (NST + clusters - 1) / clusters;
      const size_t smem = Cfg::smem_bytes(M, units);
      if (smem > static_cast<size_t>(kMaxSmem)) { clusters = 0; break; }
      const int c2 = max_active_clusters(kernel, Cfg::kThreads, smem, cl, dev, cache);
      if (c2 >= clusters) break;
      clusters = c2;
    }
    if (clusters <= 0) continue;
    const double cost = units * static_cast<double>((G + cl - 1) / cl) + 4.0;
    if (cost < best_cost) { best_cost = cost; best_cl = cl; best_clusters = clusters; best_units = units; }
  }
  if (best_cl == 0) return AWQ_ERR_UNSUPPORTED;
  return launch_ex(kernel, dim3(best_clusters, best_cl, 1), dim3(Cfg::kThreads, 1, 1), best_cl,
                   Cfg::smem_bytes(M, best_units), stream, map, qw, sc, zr, y, M, N, K, best_units);
}

// Compile-time tuning of the decode kernel per token tile: stages, 64-k tiles per stage,
// consumer warps. Measured on the Llama-2-7B and 70B decode shapes: larger stages (fewer
// barrier round trips per weight) win as long as two CTAs still fit on an SM; 4 consumer
// warps up to M = 16, 8 above, where the extra warps hide the longer mma chains.
#ifndef AWQ_GEMV1_STAGES
#define AWQ_GEMV1_STAGES 2
#endif
#ifndef AWQ_GEMV1_KS
#define AWQ_GEMV1_KS 8
#endif
#ifndef AWQ_GEMV1_CW
#define AWQ_GEMV1_CW 4
#endif
#ifndef AWQ_GEMV2_STAGES
#define AWQ_GEMV2_STAGES 3
#endif
#ifndef AWQ_GEMV2_KS
#define AWQ_GEMV2_KS 4
#endif
#ifndef AWQ_GEMV4_STAGES
#define AWQ_GEMV4_STAGES 3
#endif
#ifndef AWQ_GEMV4_KS
#define AWQ_GEMV4_KS 4
#endif

awq_status_t launch_gemv(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr, __half* y, int M,
                         int N, int K, int dev, int num_sms, cudaStream_t stream) {
  const int mt = (M + 7) / 8;
  switch (mt) {
    case 1:
      // M <= 2: codes as fp16 subnormals (one AND per pair) and the zero point through the
      // activation sums, which the warp takes from the activation box at little cost
      if (M <= 2)
        return launch_gemv_cfg<1, AWQ_GEMV1_STAGES, AWQ_GEMV1_KS, AWQ_GEMV1_CW, true>(x, qw, sc, zr, y, M, N, K, dev,
                                                                                     num_sms, stream);
      return launch_gemv_cfg<1, AWQ_GEMV1_STAGES, AWQ_GEMV1_KS, AWQ_GEMV1_CW>(x, qw, sc, zr, y, M, N, K, dev, num_sms,
                                                                             stream);
    case 2:
      return launch_gemv_cfg<2, AWQ_GEMV2_STAGES, AWQ_GEMV2_KS, 4>(x, qw, sc, zr, y, M, N, K, dev, num_sms, stream);
    case 3: return launch_gemv_cfg<3, 3, 4, 8>(x, qw, sc, zr, y, M, N, K, dev, num_sms, stream);
    default:
      return launch_gemv_cfg<4, AWQ_GEMV4_STAGES, AWQ_GEMV4_KS, 8>(x, qw, sc, zr, y, M, N, K, dev, num_sms, stream);
  }
}

// --------------------------------------------------------------------------- prefill dispatch
template <int BT, int STAGES, int NDQ, int CPS = 1>
awq_status_t launch_gemm_cfg(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr, __half* y,
                             int M, int N, int K, int dev, int num_sms, cudaStream_t stream) {
  using C = GemmCfg<BT, STAGES, NDQ, CPS>;
  auto kernel = gemm_kernel<BT, STAGES, NDQ, CPS>;
  static std::atomic<uint64_t> smem_done{0};
  awq_status_t st = ensure_smem(kernel, C::kSmem, dev, smem_done);
  if (st != AWQ_OK) return st;
  CUtensorMap map;
  st = make_x_map(&map, x, M, K, BT);
  if (st != AWQ_OK) return st;
  const long long tiles = static_cast<long long>(padded_rows(N) / kSuperRows) * ((M + BT - 1) / BT);
  const int grid = static_cast<int>(std::min<long long>(tiles, static_cast<long long>(CPS) * num_sms));
  return launch_ex(kernel, dim3(grid, 1, 1), dim3(C::kThreads, 1, 1), 0, C::kSmem, stream, map, qw, sc, zr, y, M, N,
                   K);
}

// Compile-time tuning of the prefill kernel: dequantization warps, ring stages per token tile
// (the deepest ring that fits in shared memory).
#ifndef AWQ_GEMM_NDQ
#define AWQ_GEMM_NDQ 8
#endif
#ifndef AWQ_GEMM_S256
#define AWQ_GEMM_S256 4
#endif
#ifndef AWQ_GEMM_S128
#define AWQ_GEMM_S128 6
#endif
#ifndef AWQ_GEMM_S64
#define AWQ_GEMM_S64 7
#endif

awq_status_t launch_gemm(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr, __half* y, int M,
                         int N, int K, int dev, int num_sms, cudaStream_t stream) {
  if (M <= 32) return launch_gemm_cfg<32, 8, AWQ_GEMM_NDQ>(x, qw, sc, zr, y, M, N, K, dev, num_sms, stream);
  if (M <= 64)
    return launch_gemm_cfg<64, AWQ_GEMM_S64, AWQ_GEMM_NDQ>(x, qw, sc, zr, y, M, N, K, dev, num_sms, stream);
  // Token tile by a round model: the persistent CTAs (one per SM) take tiles round-robin, so a
  // launch costs ceil(tiles / SMs) rounds, and a tile's time grows only slowly with BT because
  // dequantizing its 128-row weight block dominates (per-tile time 0.75 + 0.35 BT/256, fitted
  // on the Llama-3-8B prefill and Llama-2-70B layers at M = 512 and 2048).
  const long long nst = padded_rows(N) / kSuperRows;
  int best_bt = 64;
  double best = 1e300;
  for (int bt : {256, 128, 64}) {
    const long long tiles = nst * ((M + bt - 1) / bt);
    const double cost = static_cast<double>((tiles + num_sms - 1) / num_sms) * (0.75 + 0.35 * bt / 256.0);
    if (cost < best - 1e-9) { best = cost; best_bt = bt; }
  }
#ifdef AWQ_GEMM_FORCE_BT
  best_bt = AWQ_GEMM_FORCE_BT;
#endif
  switch (best_bt) {
    case 256:
      return launch_gemm_cfg<256, AWQ_GEMM_S256, AWQ_GEMM_NDQ>(x, qw, sc, zr, y, M, N, K, dev, num_sms, stream);
    case 128:
      return launch_gemm_cfg<128, AWQ_GEMM_S128, AWQ_GEMM_NDQ>(x, qw, sc, zr, y, M, N, K, dev, num_sms, stream);
    default:
      return launch_gemm_cfg<64, AWQ_GEMM_S64, AWQ_GEMM_NDQ>(x, qw, sc, zr, y, M, N, K, dev, num_sms, stream);
  }
}

awq_status_t check_linear_args(const void* x, const void* qw, const void* sc, const void* zr, const void* y, int M,
                               int N, int K) {
  if (!x || !qw || !sc || !zr || !y) return AWQ_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < kGroup || K % kGroup != 0) return AWQ_ERR_INVALID_ARG;
  if (static_cast<long long>(M) * K > (1ll << 31) - 1 || static_cast<long long>(padded_rows(N)) * K > (1ll << 34))
    return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(qw) || !aligned16(sc) || !aligned16(zr) || !aligned16(y)) return AWQ_ERR_MISALIGNED;
  return AWQ_OK;
}

}  // namespace
}  // namespace awq

using namespace awq;

extern "C" {

int awq_layout_version(void) { return 1; }

const char* awq_status_string(int status) {
  switch (status) {
    case AWQ_OK: return "AWQ_OK";
    case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG: null pointer or size out of range";
    case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED: configuration or device not supported";
    case AWQ_ERR_MISALIGNED: return "AWQ_ERR_MISALIGNED: pointer not 16-byte aligned";
    case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA: CUDA runtime error";
    case AWQ_ERR_TIMEOUT: return "AWQ_ERR_TIMEOUT: a kernel gave up a bounded wait";
    default: return "AWQ_ERR_UNKNOWN";
  }
}

awq_status_t awq_check_config(int bits, int group_size, int zero_point) {
  return (bits == 4 && group_size == kGroup && zero_point == 1) ? AWQ_OK : AWQ_ERR_UNSUPPORTED;
}

size_t awq_qweight_bytes(int N, int K) {
  if (N < 1 || K < kGroup || K % kGroup) return 0;
  return static_cast<size_t>(padded_rows(N)) * K / 2;
}
size_t awq_scales_bytes(int N, int K) {
  if (N < 1 || K < kGroup || K % kGroup) return 0;
  return static_cast<size_t>(padded_rows(N)) * (K / kGroup) * 2;
}
size_t awq_zeros_bytes(int N, int K) {
  if (N < 1 || K < kGroup || K % kGroup) return 0;
  return static_cast<size_t>(padded_rows(N)) * (K / kGroup) / 2;
}

awq_status_t awq_activation_scale(const uint16_t* x, int M, int K, float alpha, float* s_out, uint16_t* x_scaled,
                                  awq_stream_t stream) {
  if (!x || !s_out) return AWQ_ERR_INVALID_ARG;
  if (M < 1 || K < 1 || K % 8 != 0 || static_cast<long long>(M) * K > (1ll << 40)) return AWQ_ERR_INVALID_ARG;
  if (!(alpha == alpha) || alpha > 3.0e38f || alpha < -3.0e38f) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_scaled) || (reinterpret_cast<uintptr_t>(s_out) & 3u)) return AWQ_ERR_MISALIGNED;
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  if (M <= kActSmallMaxM)
    return launch_ex(act_scale_small_kernel, dim3((K + 127) / 128, 1, 1), dim3(128, 1, 1), 0, 0,
                     reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const __half*>(x), M, K, alpha, s_out,
                     reinterpret_cast<__half*>(x_scaled));
  int cl = 1;
  while (cl < 8 && cl * 256 < M) cl *= 2;
  const int slabs = (K + kActCols - 1) / kActCols;
  return launch_ex(act_scale_kernel, dim3(slabs, cl, 1), dim3(kActThreads, 1, 1), cl, 0,
                        reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const __half*>(x), M, K, alpha,
                        s_out, reinterpret_cast<__half*>(x_scaled));
}

awq_status_t awq_scale_activations(const uint16_t* x, const float* s, int M, int K, uint16_t* x_scaled,
                                   awq_stream_t stream) {
  if (!x || !s || !x_scaled) return AWQ_ERR_INVALID_ARG;
  if (M < 1 || K < 1 || K % 8 != 0 || static_cast<long long>(M) * K > (1ll << 40)) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(s) || !aligned16(x_scaled)) return AWQ_ERR_MISALIGNED;
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  const long long total8 = static_cast<long long>(M) * K / 8;
  const long long blocks = (total8 + 255) / 256;
  if (blocks > 2147483647ll) return AWQ_ERR_INVALID_ARG;
  return launch_ex(scale_activations_kernel, dim3(static_cast<unsigned>(blocks), 1, 1), dim3(256, 1, 1), 0, 0,
                   reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const __half*>(x), s, total8, K,
                   reinterpret_cast<__half*>(x_scaled));
}

awq_status_t awq_quantize_g128(const uint16_t* W, const float* fold_scale, int N, int K, uint32_t* qweight,
                               uint16_t* scales, uint8_t* zeros, awq_stream_t stream) {
  if (!W || !qweight || !scales || !zeros) return AWQ_ERR_INVALID_ARG;
  if (N < 1 || K < kGroup || K % kGroup != 0) return AWQ_ERR_INVALID_ARG;
  if (static_cast<long long>(padded_rows(N)) * K > (1ll << 34)) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(fold_scale))
    return AWQ_ERR_MISALIGNED;
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  // W [N, K] fp16 as a 2-D tensor: boxes of 64 k x 128 rows, 128-byte swizzle, rows >= N read as 0
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return AWQ_ERR_CUDA;
  CUtensorMap map;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kSuperRows)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(W), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return AWQ_ERR_CUDA;
  }
  static std::atomic<uint64_t> done_f{0}, done_n{0};
  st = fold_scale ? ensure_smem(quantize_g128_kernel<true>, kQSmem, dev, done_f)
                  : ensure_smem(quantize_g128_kernel<false>, kQSmem, dev, done_n);
  if (st != AWQ_OK) return st;
  const long long units = static_cast<long long>(padded_rows(N) / kSuperRows) * (K / kGroup);
  const int grid = static_cast<int>(std::min<long long>(units, static_cast<long long>(AWQ_QUANT_MINBLOCKS) * sms));
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (fold_scale)
    return launch_ex(quantize_g128_kernel<true>, dim3(grid, 1, 1), dim3(kQThreads, 1, 1), 0, kQSmem, s, map,
                     fold_scale, N, K, qweight, reinterpret_cast<__half*>(scales), zeros);
  return launch_ex(quantize_g128_kernel<false>, dim3(grid, 1, 1), dim3(kQThreads, 1, 1), 0, kQSmem, s, map,
                   static_cast<const float*>(nullptr), N, K, qweight, reinterpret_cast<__half*>(scales), zeros);
}

awq_status_t awq_w4a16_gemv(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros,
                            uint16_t* y, int M, int N, int K, awq_stream_t stream) {
  awq_status_t st = check_linear_args(x, qweight, scales, zeros, y, M, N, K);
  if (st != AWQ_OK) return st;
  if (M > 32) return AWQ_ERR_INVALID_ARG;
  int dev, sms;
  st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  return launch_gemv(reinterpret_cast<const __half*>(x), qweight, reinterpret_cast<const __half*>(scales), zeros,
                     reinterpret_cast<__half*>(y), M, N, K, dev, sms, reinterpret_cast<cudaStream_t>(stream));
}

awq_status_t awq_w4a16_gemm(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros,
                            uint16_t* y, int M, int N, int K, awq_stream_t stream) {
  awq_status_t st = check_linear_args(x, qweight, scales, zeros, y, M, N, K);
  if (st != AWQ_OK) return st;
  int dev, sms;
  st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  return launch_gemm(reinterpret_cast<const __half*>(x), qweight, reinterpret_cast<const __half*>(scales), zeros,
                     reinterpret_cast<__half*>(y), M, N, K, dev, sms, reinterpret_cast<cudaStream_t>(stream));
}

awq_status_t awq_w4a16_linear(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros,
                              uint16_t* y, int M, int N, int K, awq_stream_t stream) {
  if (M >= 1 && M <= 32) return awq_w4a16_gemv(x, qweight, scales, zeros, y, M, N, K, stream);
  return awq_w4a16_gemm(x, qweight, scales, zeros, y, M, N, K, stream);
}

awq_status_t awq_poll_device_status(awq_stream_t stream) {
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return AWQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(int)) != cudaSuccess) return AWQ_ERR_CUDA;
  if (v == 0) return AWQ_OK;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_dev_status, &zero, sizeof(int)) != cudaSuccess) return AWQ_ERR_CUDA;
  return (v & kDevStatusTimeout) ? AWQ_ERR_TIMEOUT : AWQ_ERR_CUDA;
}

awq_status_t awq_debug_drop_first_copy(int enable) {
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  const int v = enable ? 1 : 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return AWQ_ERR_CUDA;
  return cudaMemcpyToSymbol(g_debug_drop_first_copy, &v, sizeof(v)) == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status_t awq_debug_set_wait_budget_ns(unsigned long long ns) {
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  const unsigned long long v = ns ? ns : kDefaultWaitBudgetNs;
  if (cudaDeviceSynchronize() != cudaSuccess) return AWQ_ERR_CUDA;
  return cudaMemcpyToSymbol(g_wait_budget_ns, &v, sizeof(v)) == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // extern "C"
