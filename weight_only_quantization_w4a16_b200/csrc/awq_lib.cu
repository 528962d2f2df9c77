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
#include "awq_search.cuh"
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

// The packed arrays of layout v2 as 3-D tensors for the prefill kernel's producer; a box is
// 8 tiles (one super-tile) of one 64-k tile (codes), one group (scales) or one group pair
// (zeros), so it lands in shared memory as [tile][...] exactly like a 128-row block.
//   codes  uint32 {128 words, KTp k-tiles, ntiles}  box {128, 1, 8}
//   scales uint16 {16, 2*G2 groups, ntiles}         box {16, 1, 8}
//   zeros  uint8  {16, G2 pairs, ntiles}            box {16, 1, 8}
awq_status_t make_weight_maps(CUtensorMap* qm, CUtensorMap* sm, CUtensorMap* zm, const void* qw, const void* sc,
                              const void* zr, int N, int K, int box_tiles = 8) {
  const cuuint32_t bt = static_cast<cuuint32_t>(box_tiles);
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return AWQ_ERR_CUDA;
  const cuuint64_t nt = static_cast<cuuint64_t>(ceil_div(N, kTileRows));
  const cuuint64_t g2 = static_cast<cuuint64_t>(ceil_div(K / kGroup, 2));
  const cuuint32_t estr[3] = {1, 1, 1};
  {
    const cuuint64_t dims[3] = {128, 4 * g2, nt};
    const cuuint64_t strides[2] = {512, 4 * g2 * 512};
    const cuuint32_t box[3] = {128, 1, bt};
    if (enc(qm, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(qw), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return AWQ_ERR_CUDA;
  }
  {
    const cuuint64_t dims[3] = {16, 2 * g2, nt};
    const cuuint64_t strides[2] = {32, 2 * g2 * 32};
    const cuuint32_t box[3] = {16, 1, bt};
    if (enc(sm, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(sc), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return AWQ_ERR_CUDA;
  }
  {
    const cuuint64_t dims[3] = {16, g2, nt};
    const cuuint64_t strides[2] = {16, g2 * 16};
    const cuuint32_t box[3] = {16, 1, bt};
    if (enc(zm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(zr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return AWQ_ERR_CUDA;
  }
  return AWQ_OK;
}

// --------------------------------------------------------------------------- launch helper
// Every kernel is launched with programmatic stream serialization (PDL): it may start while the
// previous kernel of the stream drains, runs its prologue, and waits (griddepcontrol.wait) before
// touching data a predecessor may write. A cluster shape with x > 0 adds a thread-block cluster.
template <typename... KArgs, typename... Args>
awq_status_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, dim3 cluster, size_t smem,
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
  if (cluster.x > 0) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster.x;
    attr[na].val.clusterDim.y = cluster.y;
    attr[na].val.clusterDim.z = cluster.z;
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
  cfg.gridDim = dim3(cl * 64, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
  attr[0].val.clusterDim.y = 1;
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

// x' [M, K] fp16 for the decode kernel as a 3-D tensor {64 k, M tokens, K/64 k-tiles}; a box is
// {64, M, kt_box}: one stage's k-tiles for every token, laid out [k-tile][token][64 k] in shared
// memory (128-byte rows; 128-byte swizzle when `swizzle`), zero fill past K.
awq_status_t make_x_map_decode(CUtensorMap* map, const void* x, int M, int K, int kt_box, bool swizzle) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return AWQ_ERR_CUDA;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kKTile), static_cast<cuuint64_t>(M),
                              static_cast<cuuint64_t>(K / kKTile)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, static_cast<cuuint64_t>(kKTile) * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kKTile), static_cast<cuuint32_t>(M),
                             static_cast<cuuint32_t>(kt_box)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? AWQ_OK : AWQ_ERR_CUDA;
}

inline int round_up(int v, int a) { return (v + a - 1) / a * a; }

#ifndef AWQ_GEMV_CL
#define AWQ_GEMV_CL 2
#endif
static_assert(AWQ_GEMV_CL == 1 || AWQ_GEMV_CL == 2, "the decode epilogue shares blocks between at most two CTAs");

// The decode kernel: CL-CTA clusters over 16-row units, each CTA a contiguous item range streamed
// by one producer lane into S stages of up to CW * SBW group pairs; CW consumer warps.
template <int MT, int CW, int S, int SBW, bool kSwz, int EPI = kEpiPlain, int MINB = 1>
awq_status_t launch_gemv_cfg(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr,
                             const EpiArgs& epi, int M, int N, int K, int dev, int num_sms, cudaStream_t stream) {
  using Cfg = GemvCfg<CW, SBW, kSwz>;
  auto kernel = awq_gemv_kernel<MT, CW, S, SBW, kSwz, EPI, MINB>;
  constexpr int kMaxSmem = 227 * 1024;
  static std::atomic<uint64_t> smem_done{0};
  awq_status_t st = ensure_smem(kernel, kMaxSmem, dev, smem_done);
  if (st != AWQ_OK) return st;
  GemvArgs a = {};
  a.qweight = reinterpret_cast<const uint8_t*>(qw);
  a.scales = reinterpret_cast<const uint8_t*>(sc);
  a.zeros = zr;
  a.y = epi.y0;
  a.y1 = epi.y1;
  a.y2 = epi.y2;
  a.n0 = epi.n0;
  a.n1 = epi.n1;
  a.M = M;
  a.N = N;
  a.g2 = ceil_div(K / kGroup, 2);
  a.units = EPI == kEpiSiluMul ? 2 * (N / 32) : ceil_div(N, kTileRows);
  const int upc = EPI == kEpiSiluMul ? 2 : 1;   // units per indivisible cluster share
  a.x_box_bytes = 4 * Cfg::kSB * M * 128;
  a.stage_bytes = round_up(Cfg::kOffX + a.x_box_bytes, Cfg::kAlignX);
  CUtensorMap map;
  st = make_x_map_decode(&map, x, M, K, 4 * Cfg::kSB, kSwz);
  if (st != AWQ_OK) return st;
  const int shares = a.units / upc;
  int cl = AWQ_GEMV_CL;
  while (cl > 1 && shares < cl) cl /= 2;
  int clusters = std::max(1, std::min(num_sms / cl, shares));
  auto records = [&](int C) {
    int R = 1;
    for (int c = 0; c < C; ++c) {
      const long long u0 = upc * (static_cast<long long>(c) * shares / C);
      const long long u1 = upc * (static_cast<long long>(c + 1) * shares / C);
      const long long L = (u1 - u0) * a.g2;
      for (int r = 0; r < cl; ++r) {
        const long long lo = r * L / cl, hi = (r + 1) * L / cl;
        if (hi > lo) R = std::max(R, static_cast<int>((hi - 1) / a.g2 - lo / a.g2 + 1));
      }
    }
    return R;
  };
  auto smem_of = [&](int R) {
    return static_cast<size_t>(S) * a.stage_bytes + static_cast<size_t>(CW) * R * kTileRows * M * 4 +
           static_cast<size_t>(2) * kTileRows * M * 4 + static_cast<size_t>(2 * S) * 8 + 16 + 1024;
  };
  int R = records(clusters);
  if (smem_of(R) > static_cast<size_t>(kMaxSmem)) return AWQ_ERR_UNSUPPORTED;
  static ClusterOccCache cache;
  const int fit = max_active_clusters(kernel, Cfg::kThreads, smem_of(R), cl, dev, cache);
  if (fit < 1) return AWQ_ERR_UNSUPPORTED;
  if (clusters > fit) {
    clusters = fit;
    R = records(clusters);
    if (smem_of(R) > static_cast<size_t>(kMaxSmem)) return AWQ_ERR_UNSUPPORTED;
  }
  a.clusters = clusters;
  a.rec_per_warp = R;
  return launch_ex(kernel, dim3(clusters * cl, 1, 1), dim3(Cfg::kThreads, 1, 1), dim3(cl, 1, 1), smem_of(R), stream,
                   map, a);
}

// Compile-time tuning of the decode kernel for M <= 2 (the decode shape of one sequence):
// consumer warps, ring stages, group pairs per warp and stage, CTAs per SM the registers allow.
#ifndef AWQ_GEMV_CW
#define AWQ_GEMV_CW 8
#endif
#ifndef AWQ_GEMV_S
#define AWQ_GEMV_S 2
#endif
#ifndef AWQ_GEMV_SBW
#define AWQ_GEMV_SBW 2
#endif
#ifndef AWQ_GEMV_MINB
// One CTA per SM by registers (118 per thread): 9% slower than a register cap that lets the next
// decode launch's CTAs become resident early when decode launches follow one another directly,
// but 28% faster in a decode layer chain, where activation kernels sit between the launches.
#define AWQ_GEMV_MINB 1
#endif

// Stage shapes per token count: the x' box grows with M, so larger M takes fewer group pairs per
// stage and fewer stages, keeping shared memory near half an SM. For very wide layers at M > 8 the
// per-warp records outgrow shared memory and only a smaller configuration (fewer consumer warps,
// shorter ring) fits; with `fallback` false that case returns AWQ_ERR_UNSUPPORTED instead, so that
// the layer-level dispatch can take the prefill kernel, which measures faster there (M = 32 on the
// 22016- and 28672-row layers).
template <int EPI>
awq_status_t launch_gemv_epi(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr,
                             const EpiArgs& epi, int M, int N, int K, int dev, int num_sms, cudaStream_t stream,
                             bool fallback = true) {
  switch ((M + 7) / 8) {
    case 1:
      if (M <= 2)
        return launch_gemv_cfg<1, AWQ_GEMV_CW, AWQ_GEMV_S, AWQ_GEMV_SBW, false, EPI, AWQ_GEMV_MINB>(
            x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
      return launch_gemv_cfg<1, 4, 4, 1, true, EPI>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
    case 2: {
      const awq_status_t st = launch_gemv_cfg<2, 4, 3, 1, true, EPI>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
      if (st != AWQ_ERR_UNSUPPORTED || !fallback) return st;
      // very wide layers: fewer consumer warps (smaller per-warp records), shorter ring
      return launch_gemv_cfg<2, 2, 2, 1, true, EPI>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
    }
    case 3: {
      const awq_status_t st = launch_gemv_cfg<3, 4, 2, 1, true, EPI>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
      if (st != AWQ_ERR_UNSUPPORTED || !fallback) return st;
      return launch_gemv_cfg<3, 2, 2, 1, true, EPI>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
    }
    default: {
      const awq_status_t st = launch_gemv_cfg<4, 4, 2, 1, true, EPI>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
      if (st != AWQ_ERR_UNSUPPORTED || !fallback) return st;
      return launch_gemv_cfg<4, 2, 2, 1, true, EPI>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
    }
  }
}

awq_status_t launch_gemv(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr, __half* y, int M,
                         int N, int K, int dev, int num_sms, cudaStream_t stream, bool fallback = true) {
  const EpiArgs epi = {y, nullptr, nullptr, 0, 0};
  return launch_gemv_epi<kEpiPlain>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream, fallback);
}

// --------------------------------------------------------------------------- prefill dispatch
// KS = 2: `mixed` runs whole rounds of one tile per CTA first and splits only the tiles left for
// the last round; `max_clusters` (> 0) caps the grid (a test hook).
template <int BT, int STAGES, int NDQ, int CPS = 1, int EPI = kEpiPlain, int KS = 1>
awq_status_t launch_gemm_cfg(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr,
                             const EpiArgs& epi, int M, int N, int K, int dev, int num_sms, cudaStream_t stream,
                             bool mixed = false, int max_clusters = 0) {
  using C = GemmCfg<BT, STAGES, NDQ, CPS, KS, EPI>;
  auto kernel = awq_gemm_kernel<BT, STAGES, NDQ, CPS, EPI, KS>;
  static std::atomic<uint64_t> smem_done{0};
  awq_status_t st = ensure_smem(kernel, C::kSmem, dev, smem_done);
  if (st != AWQ_OK) return st;
  CUtensorMap xmap, qmap, smap, zmap;
  st = make_x_map(&xmap, x, M, K, BT);
  if (st != AWQ_OK) return st;
  st = make_weight_maps(&qmap, &smap, &zmap, qw, sc, zr, N, K, EPI == kEpiSiluMul ? 4 : 8);
  if (st != AWQ_OK) return st;
  const long long nst = EPI == kEpiSiluMul ? ceil_div(N / 32, 4) : padded_rows(N) / kSuperRows;
  const long long tiles = nst * ((M + BT - 1) / BT);
  if (KS == 2) {   // CTA pairs, as many as can be co-resident
    static ClusterOccCache cache;
    int fit = max_active_clusters(kernel, C::kThreads, C::kSmem, 2, dev, cache);
    if (max_clusters > 0) fit = std::min(fit, max_clusters);
    if (fit < 1) return AWQ_ERR_UNSUPPORTED;
    // mixed: every CTA takes whole tiles for tiles / (2 fit) rounds, the rest are split
    const int solo = mixed ? static_cast<int>(tiles / (2ll * fit)) : 0;
    const long long split_tiles = tiles - 2ll * fit * solo;
    const int clusters = solo > 0 ? fit : static_cast<int>(std::min<long long>(split_tiles, fit));
    return launch_ex(kernel, dim3(2 * clusters, 1, 1), dim3(C::kThreads, 1, 1), dim3(2, 1, 1), C::kSmem, stream,
                     xmap, qmap, smap, zmap, epi, M, N, K, solo);
  }
  const int grid = static_cast<int>(std::min<long long>(tiles, static_cast<long long>(CPS) * num_sms));
  return launch_ex(kernel, dim3(grid, 1, 1), dim3(C::kThreads, 1, 1), dim3(0, 0, 0), C::kSmem, stream, xmap, qmap,
                   smap, zmap, epi, M, N, K, 0);
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

// With the K split (KS = 2) the exchange slots (16 KB each) share the shared memory with the ring.
#ifndef AWQ_GEMM_KS_S256
#define AWQ_GEMM_KS_S256 4
#endif
#ifndef AWQ_GEMM_KS_S128
#define AWQ_GEMM_KS_S128 5
#endif
#ifndef AWQ_GEMM_KS_S64
#define AWQ_GEMM_KS_S64 6
#endif
#ifndef AWQ_GEMM_KS_S32
#define AWQ_GEMM_KS_S32 8
#endif
// Relative cost of a K-split tile beyond half a tile (the partial-sum exchange, the shorter ring).
#ifndef AWQ_GEMM_KS_OVERHEAD
#define AWQ_GEMM_KS_OVERHEAD 0.1
#endif
// A split form is taken only when the model prices it at least this factor below the best form
// without the split. Measured against predicted gains of the mixed form: 10% predicted gave 5% and
// 9% (Llama-3-8B and Llama-2-70B gate/up at M = 512), 3% predicted lost 3% (8B gate/up, M = 2048).
#ifndef AWQ_GEMM_KS_MARGIN
#define AWQ_GEMM_KS_MARGIN 1.08
#endif

// Test hook (awq_debug_set_gemm_split): 0 lets the round model choose the K split, 1 or 2 forces it.
std::atomic<int> g_force_ks{0};

// Token tile BT and K split of the prefill kernel by a round model: the persistent CTAs (one per
// SM; with the split, one CTA pair per two SMs) take tiles round-robin, so a launch costs
// ceil(tiles / slots) rounds, and a tile's time grows only slowly with BT because dequantizing its
// 128-row weight block dominates (per-tile time 0.75 + 0.35 BT/256, fitted on the Llama-3-8B
// prefill and Llama-2-70B layers at M = 512 and 2048). A split tile takes half a tile's time plus
// the exchange. Three forms: no split; every tile split (ks 2); whole rounds of one tile per SM
// and only the last round's tiles split (ks 2, mixed). BT = 32 serves M <= 32 and BT = 64 M <= 64.
// `force`: 0 the model, 1 no split, 2 every tile split, 3 the mixed form on a grid of 3 CTA pairs
// (a test hook that makes small layers take both kinds of work item).
struct GemmPlan {
  int bt, ks;
  bool mixed;
  int max_clusters;          // > 0: grid cap (force 3)
  long long split_tiles;     // tiles split across a CTA pair, on num_sms SMs
};
GemmPlan gemm_plan(int M, int N, int epi, int num_sms, int force) {
  const long long nst = epi == kEpiSiluMul ? ceil_div(N / 32, 4) : padded_rows(N) / kSuperRows;
  GemmPlan best_plan = {64, 1, false, 0, 0};
  double best = 1e300;
  const int bts_small[1] = {M <= 32 ? 32 : 64};
  const int bts_large[3] = {256, 128, 64};
  const int* bts = M <= 64 ? bts_small : bts_large;
  const int nbt = M <= 64 ? 1 : 3;
  const long long pairs = force == 3 ? 3 : std::max(1, num_sms / 2);
  const long long slots1 = std::max(1, num_sms);
  auto consider = [&](double cost, const GemmPlan& p) {
    if (cost < best - 1e-9) { best = cost; best_plan = p; }
  };
  for (int i = 0; i < nbt; ++i) {
    const int bt = bts[i];
    const long long tiles = nst * ((M + bt - 1) / bt);
    const double t_tile = 0.75 + 0.35 * bt / 256.0, t_split = t_tile * (0.5 + AWQ_GEMM_KS_OVERHEAD);
    if (force == 0 || force == 1)
      consider(static_cast<double>((tiles + slots1 - 1) / slots1) * t_tile, {bt, 1, false, 0, 0});
    const double margin = force == 0 ? AWQ_GEMM_KS_MARGIN : 1.0;
    if (force == 0 || force == 2)
      consider(margin * static_cast<double>((tiles + pairs - 1) / pairs) * t_split, {bt, 2, false, 0, tiles});
    if (force == 0 || force == 3) {
      const long long solo = tiles / (2 * pairs), rest = tiles - 2 * pairs * solo;
      if (force == 3 || (solo > 0 && rest > 0))
        consider(margin * (static_cast<double>(solo) * t_tile +
                           static_cast<double>((rest + pairs - 1) / pairs) * t_split),
                 {bt, 2, true, force == 3 ? 3 : 0, rest});
    }
  }
  return best_plan;
}

template <int EPI>
awq_status_t launch_gemm_epi(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr,
                             const EpiArgs& epi, int M, int N, int K, int dev, int num_sms, cudaStream_t stream) {
  const GemmPlan plan = gemm_plan(M, N, EPI, num_sms, g_force_ks.load());
  int best_bt = plan.bt;
  const int best_ks = plan.ks;
#ifdef AWQ_GEMM_FORCE_BT
  best_bt = AWQ_GEMM_FORCE_BT;
#endif
#define AWQ_GEMM_ARGS x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream
#define AWQ_GEMM_SPLIT_ARGS AWQ_GEMM_ARGS, plan.mixed, plan.max_clusters
  if (best_ks == 2) {
    switch (best_bt) {
      case 256:   // kEpiSiluMul's wider zeros slots leave room for 3 stages only
        return launch_gemm_cfg<256, EPI == kEpiSiluMul ? 3 : AWQ_GEMM_KS_S256, AWQ_GEMM_NDQ, 1, EPI, 2>(
            AWQ_GEMM_SPLIT_ARGS);
      case 128: return launch_gemm_cfg<128, AWQ_GEMM_KS_S128, AWQ_GEMM_NDQ, 1, EPI, 2>(AWQ_GEMM_SPLIT_ARGS);
      case 64: return launch_gemm_cfg<64, AWQ_GEMM_KS_S64, AWQ_GEMM_NDQ, 1, EPI, 2>(AWQ_GEMM_SPLIT_ARGS);
      default: return launch_gemm_cfg<32, AWQ_GEMM_KS_S32, AWQ_GEMM_NDQ, 1, EPI, 2>(AWQ_GEMM_SPLIT_ARGS);
    }
  }
  switch (best_bt) {
    case 256: return launch_gemm_cfg<256, AWQ_GEMM_S256, AWQ_GEMM_NDQ, 1, EPI>(AWQ_GEMM_ARGS);
    case 128: return launch_gemm_cfg<128, AWQ_GEMM_S128, AWQ_GEMM_NDQ, 1, EPI>(AWQ_GEMM_ARGS);
    case 64: return launch_gemm_cfg<64, AWQ_GEMM_S64, AWQ_GEMM_NDQ, 1, EPI>(AWQ_GEMM_ARGS);
    default: return launch_gemm_cfg<32, 8, AWQ_GEMM_NDQ, 1, EPI>(AWQ_GEMM_ARGS);
  }
#undef AWQ_GEMM_SPLIT_ARGS
#undef AWQ_GEMM_ARGS
}

awq_status_t launch_gemm(const __half* x, const uint32_t* qw, const __half* sc, const uint8_t* zr, __half* y, int M,
                         int N, int K, int dev, int num_sms, cudaStream_t stream) {
  EpiArgs epi = {y, nullptr, nullptr, 0, 0};
  return launch_gemm_epi<kEpiPlain>(x, qw, sc, zr, epi, M, N, K, dev, num_sms, stream);
}

// Rows are limited so that every count below fits an int: N <= 2^31 - 2^7 and N * K <= 2^34.
constexpr long long kMaxRows = (1ll << 31) - 128;
inline bool rows_ok(int N, int K) {
  return N >= 1 && N <= kMaxRows && static_cast<long long>(ceil_div(N, kTileRows)) * kTileRows * K <= (1ll << 34);
}

awq_status_t check_linear_args(const void* x, const void* qw, const void* sc, const void* zr, const void* y, int M,
                               int N, int K) {
  if (!x || !qw || !sc || !zr || !y) return AWQ_ERR_INVALID_ARG;
  if (M < 1 || K < kGroup || K % kGroup != 0 || !rows_ok(N, K)) return AWQ_ERR_INVALID_ARG;
  if (static_cast<long long>(M) * K > (1ll << 31) - 1) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(qw) || !aligned16(sc) || !aligned16(zr) || !aligned16(y)) return AWQ_ERR_MISALIGNED;
  return AWQ_OK;
}

// Packed sizes of layout v2: per (16-row tile, group pair) 2048 + 64 + 16 bytes.
inline size_t tile_pairs(int N, int K) {
  return static_cast<size_t>(ceil_div(N, kTileRows)) * static_cast<size_t>(ceil_div(K / kGroup, 2));
}

// Workspace of the scale search, each piece 256-byte aligned: y_ref fp32 [M,N], y fp16 [M,N], s fp32 [K],
// x' fp16 [M,K], the packed weights, and the error reduction's partial sums.
struct SearchWs {
  size_t y_ref, y, s, xs, qw, sc, zr, partial, total;
};
inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }
SearchWs search_ws(int M, int N, int K) {
  SearchWs w{};
  size_t o = 0;
  w.y_ref = o; o = align256(o + static_cast<size_t>(M) * N * 4);
  w.y = o; o = align256(o + static_cast<size_t>(M) * N * 2);
  w.s = o; o = align256(o + static_cast<size_t>(K) * 4);
  w.xs = o; o = align256(o + static_cast<size_t>(M) * K * 2);
  w.qw = o; o = align256(o + tile_pairs(N, K) * kPairCodeBytes);
  w.sc = o; o = align256(o + tile_pairs(N, K) * kPairScaleBytes);
  w.zr = o; o = align256(o + tile_pairs(N, K) * kPairZeroBytes);
  w.partial = o; o = align256(o + static_cast<size_t>(kSearchMaxBlocks) * 8);
  w.total = o;
  return w;
}
inline bool search_shape_ok(int M, int N, int K) {
  return M >= 1 && M <= 65535 * 16 && K >= kGroup && K % kGroup == 0 && rows_ok(N, K) &&
         static_cast<long long>(M) * K <= (1ll << 31) - 1 && static_cast<long long>(M) * N <= (1ll << 31) - 1;
}


// Scratch of awq_search_alpha_noalloc: a file-scope device array, so that callers which cannot
// allocate device memory can still run the search. Every device on which this library's kernels
// are loaded holds it until the process exits. In host code `g_search_scratch` only names the
// symbol; its address on a device comes from cudaGetSymbolAddress with that device current.
static __device__ __align__(256) unsigned char g_search_scratch[AWQ_SEARCH_NOALLOC_SCRATCH_BYTES];
std::atomic<void*> g_search_scratch_ptr[kMaxDevices];
std::mutex g_search_scratch_mutex;

// Device address of g_search_scratch on `dev` (the current device), looked up once per device.
awq_status_t search_scratch(int dev, void** out) {
  void* p = g_search_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_search_scratch_mutex);
    p = g_search_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_search_scratch) != cudaSuccess || p == nullptr) {
        (void)cudaGetLastError();
        return AWQ_ERR_CUDA;
      }
      g_search_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return AWQ_OK;
}

}  // namespace
}  // namespace awq

using namespace awq;

extern "C" {

int awq_layout_version(void) { return 2; }

const char* awq_status_string(int status) {
  switch (status) {
    case AWQ_OK: return "AWQ_OK";
    case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG: null pointer or size out of range";
    case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED: configuration or device not supported";
    case AWQ_ERR_MISALIGNED: return "AWQ_ERR_MISALIGNED: pointer not 16-byte aligned";
    case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA: CUDA runtime error";
    case AWQ_ERR_TIMEOUT: return "AWQ_ERR_TIMEOUT: a kernel gave up a bounded wait";
    case AWQ_ERR_BOUNDS: return "AWQ_ERR_BOUNDS: a bounds check of the debug build failed";
    default: return "AWQ_ERR_UNKNOWN";
  }
}

awq_status_t awq_check_config(int bits, int group_size, int zero_point) {
  return ((bits == 4 || bits == 3) && group_size == kGroup && (zero_point == 0 || zero_point == 1))
             ? AWQ_OK
             : AWQ_ERR_UNSUPPORTED;
}

size_t awq_qweight_bytes(int N, int K) {
  if (K < kGroup || K % kGroup || !rows_ok(N, K)) return 0;
  return tile_pairs(N, K) * kPairCodeBytes;
}
size_t awq_scales_bytes(int N, int K) {
  if (K < kGroup || K % kGroup || !rows_ok(N, K)) return 0;
  return tile_pairs(N, K) * kPairScaleBytes;
}
size_t awq_zeros_bytes(int N, int K) {
  if (K < kGroup || K % kGroup || !rows_ok(N, K)) return 0;
  return tile_pairs(N, K) * kPairZeroBytes;
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
    return launch_ex(awq_act_scale_small_kernel, dim3((K + 127) / 128, 1, 1), dim3(128, 1, 1), dim3(0, 0, 0), 0,
                     reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const __half*>(x), M, K, alpha, s_out,
                     reinterpret_cast<__half*>(x_scaled));
  int cl = 1;
  while (cl < 8 && cl * 256 < M) cl *= 2;
  const int slabs = (K + kActCols - 1) / kActCols;
  return launch_ex(awq_act_scale_kernel, dim3(slabs, cl, 1), dim3(kActThreads, 1, 1), dim3(1, cl, 1), 0,
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
  return launch_ex(awq_scale_activations_kernel, dim3(static_cast<unsigned>(blocks), 1, 1), dim3(256, 1, 1),
                   dim3(0, 0, 0), 0,
                   reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const __half*>(x), s, total8, K,
                   reinterpret_cast<__half*>(x_scaled));
}

awq_status_t awq_quantize(const uint16_t* W, const float* fold_scale, int N, int K, int bits, int group_size,
                          int zero_point, uint32_t* qweight, uint16_t* scales, uint8_t* zeros, awq_stream_t stream) {
  if (!W || !qweight || !scales || !zeros) return AWQ_ERR_INVALID_ARG;
  if (K < kGroup || K % kGroup != 0 || !rows_ok(N, K)) return AWQ_ERR_INVALID_ARG;
  if (awq_check_config(bits, group_size, zero_point) != AWQ_OK) return AWQ_ERR_UNSUPPORTED;
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
  const long long units = static_cast<long long>(padded_rows(N) / kSuperRows) * (K / kGroup);
  const int grid = static_cast<int>(std::min<long long>(units, static_cast<long long>(AWQ_QUANT_MINBLOCKS) * sms));
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto run = [&](auto kernel, std::atomic<uint64_t>& done) -> awq_status_t {
    const awq_status_t e = ensure_smem(kernel, kQSmem, dev, done);
    if (e != AWQ_OK) return e;
    return launch_ex(kernel, dim3(grid, 1, 1), dim3(kQThreads, 1, 1), dim3(0, 0, 0), kQSmem, s, map, fold_scale, N, K,
                     qweight, reinterpret_cast<__half*>(scales), zeros);
  };
  static std::atomic<uint64_t> done[8];
  const bool f = fold_scale != nullptr;
  const int variant = (bits == 3 ? 2 : 0) + (zero_point ? 0 : 1);
  switch (variant) {
    case 0: return f ? run(awq_quantize_g128_kernel<true, 4, false>, done[0]) : run(awq_quantize_g128_kernel<false, 4, false>, done[1]);
    case 1: return f ? run(awq_quantize_g128_kernel<true, 4, true>, done[2]) : run(awq_quantize_g128_kernel<false, 4, true>, done[3]);
    case 2: return f ? run(awq_quantize_g128_kernel<true, 3, false>, done[4]) : run(awq_quantize_g128_kernel<false, 3, false>, done[5]);
    default: return f ? run(awq_quantize_g128_kernel<true, 3, true>, done[6]) : run(awq_quantize_g128_kernel<false, 3, true>, done[7]);
  }
}

awq_status_t awq_quantize_g128(const uint16_t* W, const float* fold_scale, int N, int K, uint32_t* qweight,
                               uint16_t* scales, uint8_t* zeros, awq_stream_t stream) {
  return awq_quantize(W, fold_scale, N, K, 4, kGroup, 1, qweight, scales, zeros, stream);
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
  // M <= 32: the decode kernel in its primary configuration, which measures faster than the
  // prefill kernel at every such M on the Llama-2 7B/70B shapes; otherwise the prefill kernel.
  if (M >= 1 && M <= 32) {
    awq_status_t st = check_linear_args(x, qweight, scales, zeros, y, M, N, K);
    if (st != AWQ_OK) return st;
    int dev, sms;
    if ((st = current_device(&dev, &sms)) != AWQ_OK) return st;
    st = launch_gemv(reinterpret_cast<const __half*>(x), qweight, reinterpret_cast<const __half*>(scales), zeros,
                     reinterpret_cast<__half*>(y), M, N, K, dev, sms, reinterpret_cast<cudaStream_t>(stream), false);
    if (st != AWQ_ERR_UNSUPPORTED) return st;
  }
  return awq_w4a16_gemm(x, qweight, scales, zeros, y, M, N, K, stream);
}

size_t awq_search_workspace_bytes(int M, int N, int K) {
  if (!search_shape_ok(M, N, K)) return 0;
  return search_ws(M, N, K).total;
}

awq_status_t awq_search_alpha(const uint16_t* x, const uint16_t* W, int M, int N, int K, const float* alphas,
                              int n_alpha, double* err, int* best, void* workspace, size_t workspace_bytes,
                              awq_stream_t stream) {
  if (!x || !W || !alphas || !err || !best || !workspace) return AWQ_ERR_INVALID_ARG;
  if (!search_shape_ok(M, N, K) || n_alpha < 1 || n_alpha > 4096) return AWQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_alpha; ++i)
    if (!(alphas[i] == alphas[i]) || alphas[i] > 3.0e38f || alphas[i] < -3.0e38f) return AWQ_ERR_INVALID_ARG;
  const SearchWs w = search_ws(M, N, K);
  if (workspace_bytes < w.total) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(W) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(err) & 7u) ||
      (reinterpret_cast<uintptr_t>(best) & 3u))
    return AWQ_ERR_MISALIGNED;
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* y_ref = reinterpret_cast<float*>(ws + w.y_ref);
  uint16_t* y = reinterpret_cast<uint16_t*>(ws + w.y);
  float* s = reinterpret_cast<float*>(ws + w.s);
  uint16_t* xs = reinterpret_cast<uint16_t*>(ws + w.xs);
  uint32_t* qw = reinterpret_cast<uint32_t*>(ws + w.qw);
  uint16_t* sc = reinterpret_cast<uint16_t*>(ws + w.sc);
  uint8_t* zr = ws + w.zr;
  double* partial = reinterpret_cast<double*>(ws + w.partial);
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // the layer's unquantized output on the calibration rows, once
  st = launch_ex(awq_ref_gemm_kernel, dim3(static_cast<unsigned>(ceil_div(N, 128)), static_cast<unsigned>(ceil_div(M, 16)), 1),
                 dim3(128, 1, 1), dim3(0, 0, 0), 0, cs, reinterpret_cast<const __half*>(x),
                 reinterpret_cast<const __half*>(W), y_ref, M, N, K);
  if (st != AWQ_OK) return st;
  const long long count = static_cast<long long>(M) * N;
  const int nb = static_cast<int>(std::min<long long>(kSearchMaxBlocks, (count + kSearchThreads - 1) / kSearchThreads));
  for (int i = 0; i < n_alpha; ++i) {
    if ((st = awq_activation_scale(x, M, K, alphas[i], s, xs, stream)) != AWQ_OK) return st;
    if ((st = awq_quantize_g128(W, s, N, K, qw, sc, zr, stream)) != AWQ_OK) return st;
    if ((st = awq_w4a16_linear(xs, qw, sc, zr, y, M, N, K, stream)) != AWQ_OK) return st;
    if ((st = launch_ex(awq_sq_error_kernel, dim3(nb, 1, 1), dim3(kSearchThreads, 1, 1), dim3(0, 0, 0), 0, cs, y_ref,
                        reinterpret_cast<const __half*>(y), count, partial)) != AWQ_OK)
      return st;
    if ((st = launch_ex(awq_sq_error_final_kernel, dim3(1, 1, 1), dim3(32, 1, 1), dim3(0, 0, 0), 0, cs,
                        static_cast<const double*>(partial), nb, err, i, i == n_alpha - 1 ? best : nullptr,
                        n_alpha)) != AWQ_OK)
      return st;
  }
  return AWQ_OK;
}

awq_status_t awq_search_alpha_noalloc(const uint16_t* x, const uint16_t* W, int M, int N, int K, const float* alphas,
                                      int n_alpha, double* err, int* best, awq_stream_t stream) {
  if (!search_shape_ok(M, N, K) || search_ws(M, N, K).total > static_cast<size_t>(AWQ_SEARCH_NOALLOC_SCRATCH_BYTES))
    return AWQ_ERR_INVALID_ARG;
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  void* scratch = nullptr;
  if ((st = search_scratch(dev, &scratch)) != AWQ_OK) return st;
  return awq_search_alpha(x, W, M, N, K, alphas, n_alpha, err, best, scratch,
                          static_cast<size_t>(AWQ_SEARCH_NOALLOC_SCRATCH_BYTES), stream);
}

awq_status_t awq_w4a16_linear_qkv(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                                  const uint8_t* zeros, uint16_t* yq, uint16_t* yk, uint16_t* yv, int M, int Nq,
                                  int Nkv, int K, awq_stream_t stream) {
  if (!yk || !yv || Nq < 1 || Nkv < 1) return AWQ_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(Nq) + 2ll * Nkv;
  if (N > kMaxRows) return AWQ_ERR_INVALID_ARG;
  awq_status_t st = check_linear_args(x, qweight, scales, zeros, yq, M, static_cast<int>(N), K);
  if (st != AWQ_OK) return st;
  if (!aligned16(yk) || !aligned16(yv)) return AWQ_ERR_MISALIGNED;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != AWQ_OK) return st;
  const EpiArgs epi = {reinterpret_cast<__half*>(yq), reinterpret_cast<__half*>(yk), reinterpret_cast<__half*>(yv),
                       Nq, Nkv};
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const __half* xh = reinterpret_cast<const __half*>(x);
  const __half* sh = reinterpret_cast<const __half*>(scales);
  if (M <= 32) {
    st = launch_gemv_epi<kEpiSplit3>(xh, qweight, sh, zeros, epi, M, static_cast<int>(N), K, dev, sms, cs, false);
    if (st != AWQ_ERR_UNSUPPORTED) return st;
  }
  return launch_gemm_epi<kEpiSplit3>(xh, qweight, sh, zeros, epi, M, static_cast<int>(N), K, dev, sms, cs);
}

awq_status_t awq_w4a16_linear_silu_mul(const uint16_t* x, const uint32_t* qweight, const uint16_t* scales,
                                       const uint8_t* zeros, uint16_t* h, int M, int I, int K, awq_stream_t stream) {
  if (I < 16 || I % 16 != 0 || I > kMaxRows / 2) return AWQ_ERR_INVALID_ARG;
  awq_status_t st = check_linear_args(x, qweight, scales, zeros, h, M, 2 * I, K);
  if (st != AWQ_OK) return st;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != AWQ_OK) return st;
  const EpiArgs epi = {reinterpret_cast<__half*>(h), nullptr, nullptr, 0, 0};
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const __half* xh = reinterpret_cast<const __half*>(x);
  const __half* sh = reinterpret_cast<const __half*>(scales);
  if (M <= 32) {
    st = launch_gemv_epi<kEpiSiluMul>(xh, qweight, sh, zeros, epi, M, 2 * I, K, dev, sms, cs, false);
    if (st != AWQ_ERR_UNSUPPORTED) return st;
  }
  return launch_gemm_epi<kEpiSiluMul>(xh, qweight, sh, zeros, epi, M, 2 * I, K, dev, sms, cs);
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
  if (v & kDevStatusTimeout) return AWQ_ERR_TIMEOUT;
  return (v & kDevStatusBounds) ? AWQ_ERR_BOUNDS : AWQ_ERR_CUDA;
}

awq_status_t awq_debug_drop_first_copy(int enable) {
  int dev, sms;
  awq_status_t st = current_device(&dev, &sms);
  if (st != AWQ_OK) return st;
  const int v = enable ? 1 : 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return AWQ_ERR_CUDA;
  return cudaMemcpyToSymbol(g_debug_drop_first_copy, &v, sizeof(v)) == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status_t awq_gemm_plan(int M, int N, int K, int epilogue, int num_sms, int* token_tile, int* k_split,
                           long long* split_tiles) {
  if (!token_tile || !k_split || !split_tiles || M < 1 || K < kGroup || K % kGroup != 0 || !rows_ok(N, K) ||
      num_sms < 1 || epilogue < kEpiPlain || epilogue > kEpiSiluMul)
    return AWQ_ERR_INVALID_ARG;
  if (epilogue == kEpiSiluMul && N % 32 != 0) return AWQ_ERR_INVALID_ARG;
  const GemmPlan p = gemm_plan(M, N, epilogue, num_sms, g_force_ks.load());
  *token_tile = p.bt;
  *k_split = p.ks;
  *split_tiles = p.split_tiles;
  return AWQ_OK;
}

awq_status_t awq_debug_set_gemm_split(int ks) {
  if (ks < 0 || ks > 3) return AWQ_ERR_INVALID_ARG;
  g_force_ks.store(ks);
  return AWQ_OK;
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
