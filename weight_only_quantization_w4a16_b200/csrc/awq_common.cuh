// awq_common.cuh — device helpers shared by the kernels of libawq_w4a16.
//
// Inline PTX wrappers for sm_100a (mbarrier, bulk and tensor TMA copies,
// tcgen05 tensor memory and MMA, mma.sync), the packed-layout index helpers
// and the device status word used by bounded waits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "awq_w4a16.h"

namespace awq {

// ---------------------------------------------------------------------------
// Packed layout v2 constants (see include/awq_w4a16.h): 16-row tiles, each tile's codes, scales
// and zeros contiguous along K in group pairs (2048 + 64 + 16 bytes per tile and pair).
// ---------------------------------------------------------------------------
constexpr int kGroup = 128;        // quantization group along K
constexpr int kKTile = 64;         // k per packed tile
constexpr int kSuperRows = 128;    // rows per super-tile
constexpr int kTileRows = 16;      // rows per mma tile
constexpr int kChunkWords = 128;   // words of one (16-row, 64-k) tile = 512 bytes
constexpr int kSuperChunkWords = 8 * kChunkWords;  // (128-row, 64-k) = 4096 bytes
constexpr int kPairCodeBytes = 2048;   // codes of one (tile, group pair)
constexpr int kPairScaleBytes = 64;    // scales of one (tile, group pair)
constexpr int kPairZeroBytes = 16;     // zeros of one (tile, group pair)

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
// Rows rounded up to whole 128-row super-tiles (the prefill kernel's and the quantizer's row blocks).
__host__ __device__ inline int padded_rows(int N) { return ceil_div(N, kSuperRows) * kSuperRows; }

// ---------------------------------------------------------------------------
// Device status word and the wait budget for bounded spin-waits.
// ---------------------------------------------------------------------------
constexpr int kDevStatusTimeout = 1;
constexpr int kDevStatusBounds = 2;   // debug builds: a kernel's bounds check failed
constexpr unsigned long long kDefaultWaitBudgetNs = 2000000000ull;   // 2 s
constexpr unsigned long long kDrainBudgetNs = 1000000000ull;         // 1 s for teardown waits

// Defined here: the library is built as one translation unit (awq_lib.cu).
__device__ int g_dev_status = 0;
__device__ unsigned long long g_wait_budget_ns = kDefaultWaitBudgetNs;
// Test hook: nonzero makes the producer of each pipelined kernel skip the copies of its first
// ring stage, so the consumers' wait on that stage can only end by running out its budget.
__device__ int g_debug_drop_first_copy = 0;

// Debug builds (-DAWQ_DEBUG_BOUNDS) check the kernels' computed offsets against the extents of the
// buffers they address: a failed check records kDevStatusBounds in the device status word and the
// access is skipped (no trap, no fault). In normal builds AWQ_CHECK(cond) is the constant true.
#ifdef AWQ_DEBUG_BOUNDS
__device__ __forceinline__ bool awq_check(bool ok) {
  if (!ok) atomicOr(&g_dev_status, kDevStatusBounds);
  return ok;
}
#define AWQ_CHECK(cond) ::awq::awq_check(cond)
#else
#define AWQ_CHECK(cond) true
#endif

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch: wait until the preceding kernel of the stream has completed
// and its writes are visible (a no-op when there is none), then let the next kernel launch
// early so its prologue overlaps this kernel's tail. Every kernel calls pdl_wait() before its
// first global-memory access.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_launch_dependents();
}
// The same for kernels that write nothing the next kernel may read before its own wait (it reads
// this kernel's outputs only after griddepcontrol.wait, which returns once this grid has
// completed): the next kernel launches at once, so a decode kernel after an activation kernel
// can already stream its packed weights while the kernels before it run.
__device__ __forceinline__ void pdl_enter_early() {
  pdl_launch_dependents();
  pdl_wait();
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with an explicit bound (ns) on how long the thread may stay suspended in it.
__device__ __forceinline__ bool mbar_try_wait_for(uint64_t* bar, uint32_t parity, uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}
// The same two waits with acquire semantics at cluster scope: for phases completed by arrivals
// of the other CTA of a cluster, whose shared-memory stores into this CTA they make visible.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_for_cluster(uint64_t* bar, uint32_t parity, uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// Budgets below this (set only through the test hook) also bound each suspended try_wait, so
// that the budget is honoured even when the hardware's own suspend window is longer.
constexpr unsigned long long kShortBudgetNs = 1000000ull;

// Bounded wait: returns true when the phase with `parity` has completed.
// Gives up (returns false) when *abort is set by another warp, or after
// `budget_ns` of waiting, in which case it sets *abort and the device status.
// kCluster: acquire at cluster scope (arrivals from the other CTA of a cluster).
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                  unsigned long long budget_ns) {
  const bool short_budget = budget_ns < kShortBudgetNs;
  const uint32_t hint = static_cast<uint32_t>(budget_ns);
  auto try_once = [&]() {
    if (kCluster)
      return short_budget ? mbar_try_wait_for_cluster(bar, parity, hint) : mbar_try_wait_cluster(bar, parity);
    return short_budget ? mbar_try_wait_for(bar, parity, hint) : mbar_try_wait(bar, parity);
  };
  if (try_once()) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (try_once()) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > budget_ns) {
      *abort = 1;
      atomicOr(&g_dev_status, kDevStatusTimeout);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// Thread-block clusters: the cluster barrier, split into arrive and wait (all 32 lanes of a warp
// execute each together), and shared-memory access to the other CTAs of the cluster.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The shared::cluster address of this CTA's shared-memory object `p` in the CTA of rank `rank`.
__device__ __forceinline__ uint32_t cluster_smem_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// One arrival, with release semantics at cluster scope, on an mbarrier of another CTA.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// An asynchronous 16-byte store into another CTA's shared memory that completes 16 bytes of the
// transaction count of `cluster_bar`, an mbarrier in that same CTA.
__device__ __forceinline__ void st_async_v4(uint32_t cluster_addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                            uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   cluster_addr),
               "r"(a), "r"(b), "r"(c), "r"(d), "r"(cluster_bar)
               : "memory");
}

// ---------------------------------------------------------------------------
// Bulk / tensor copies (TMA). No multicast anywhere in this library.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst_smem, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst_smem)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst_smem, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst_smem)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, tensor memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] . B[smem desc]^T, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on `bar` when all tcgen05 operations issued so far by this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base + i), columns col..col+31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 bytes,
// 8-row atoms 1024 bytes apart (SBO), atom base 1024-byte aligned.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;               // leading byte offset (unused for swizzled K-major), 16 B
  d |= static_cast<uint64_t>(1024 >> 4) << 32;       // stride byte offset: 8 rows x 128 B
  d |= static_cast<uint64_t>(1) << 46;               // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;               // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: fp16 A and B (K-major), fp32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (0u << 7) | (0u << 10)                    // A, B format: f16
         | (0u << 15) | (0u << 16)                   // A, B K-major
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// ---------------------------------------------------------------------------
// Legacy warp-level MMA (register operands), used by the decode kernel.
// ---------------------------------------------------------------------------
// A pure register-to-register operation: not volatile, so the compiler may interleave independent
// accumulator chains.
__device__ __forceinline__ void mma_m16n8k16_f32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A . B with a zero accumulator operand (the first product of an accumulator chain), so the
// chain needs no zeroed registers.
__device__ __forceinline__ void mma_m16n8k16_f32_zero(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                      uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t lop_or(uint32_t q, uint32_t mask, uint32_t bits) {
  uint32_t r;
  // r = (q & mask) | bits in one LOP3 (immediate LUT 0xEA = (a & b) | c)
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(q), "r"(mask), "r"(bits));
  return r;
}

// fp16 pair -> two fp32 values through the mixed-precision add f32(h) + (-0.0) (an FMA-pipe
// instruction; exact for every fp16 value, signed zeros and non-finite values included).
__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t v) {
  float a, b;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.f16 %0, l, %3;\n\tadd.rn.f32.f16 %1, h, %3;\n\t}"
      : "=f"(a), "=f"(b)
      : "r"(v), "f"(-0.0f));
  return make_float2(a, b);
}

// A small non-negative integer v < 2^23 as fp32 without the conversion unit: the bits of 2^23 + v
// minus 2^23 (exact).
__device__ __forceinline__ float small_uint_to_float(uint32_t v) {
  return __int_as_float(0x4B000000 | v) - 8388608.0f;
}

__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

}  // namespace awq
