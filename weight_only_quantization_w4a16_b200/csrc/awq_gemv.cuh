// awq_gemv.cuh — a3: decode W4A16 linear layer, 1 <= M <= 32.
//
// llm-awq README, "Installation" step 3: W4A16 (4-bit weight, 16-bit
// activation) kernels for the decode stage. y[M,N] = x'[M,K] . ((q-z)*S)^T,
// fp32 accumulation, fp16 output.
//
// The layer is HBM-bound (0.52 bytes of packed weight per weight, about
// 3.85*M flop per byte). Design for B200:
//  * work items are (unit, group pair): a unit is NT 16-row tiles, a group
//    pair is 256 k (2128 bytes of codes, scales and zeros per tile in packed
//    layout v2, where every tile's data runs contiguously along K);
//  * every warp is an independent stream-K worker: the units are split
//    evenly over the thread-block clusters (unit-aligned), and a cluster's
//    items are split evenly over all warps of its CTAs, so each warp owns one
//    contiguous item range: three contiguous byte ranges of the packed arrays;
//  * a warp streams its range through a private D-stage ring of 1-D bulk
//    copies (weights) and one 3-D TMA box per stage (the stage's x' k-tiles,
//    zero fill past K); there is no producer warp and no cross-warp handoff;
//  * the weights of a warp's first ring pass are requested before the kernel
//    waits on its stream predecessor (programmatic dependent launch), so
//    consecutive decode launches overlap their weight streams;
//  * dequantization yields exact small integers: a code pair is masked out of
//    its word and OR-ed into the mantissa of fp16 1024 (one LOP3), one HSUB2
//    of 1024 + z leaves q - z (or 16 (q - z) for the odd nibbles), and the
//    m16n8k16 tensor-core product with x' is exact; S is applied in fp32 to
//    each group's sums;
//  * a warp writes one partial-sum record per unit it touched into shared
//    memory; after one cluster barrier the cluster's CTAs add the records of
//    each unit in worker order through distributed shared memory
//    (deterministic, no global scratch, no atomics) and store y.
#pragma once

#include <cooperative_groups.h>

#include "awq_common.cuh"
#include "awq_gemm.cuh"

namespace awq {

// ------------------------------------------------------------------------------------
// Cluster barrier (all 32 lanes of a warp execute it together).
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Per-launch arguments of the decode kernel (the stage layout is computed on the host).
struct GemvArgs {
  const uint8_t* qweight;   // packed codes (layout v2), 2048 bytes per (tile, group pair)
  const uint8_t* scales;    // 64 bytes per (tile, group pair)
  const uint8_t* zeros;     // 16 bytes per (tile, group pair)
  __half* y;                // [M, N]
  int M, N;
  int ntiles;               // ceil(N / 16)
  int g2;                   // group pairs per tile: ceil(K / 256)
  int units;                // ceil(ntiles / NT)
  int clusters;             // clusters in the grid
  int rec_per_warp;         // partial-sum records per warp (max units a warp's range touches)
  int stage_bytes;          // bytes of one ring stage (multiple of 1024)
  int off_scales, off_zeros, off_x;   // offsets inside a stage
  int x_box_bytes;          // bytes of the stage's x' box (4*SB k-tiles x M tokens x 128)
  int x_swizzle;            // the x' box uses the 128-byte swizzle (M > 2)
  // fused epilogues (ring form): kEpiSplit3 writes y, y1, y2 with widths n0, n1, N - n0 - n1;
  // kEpiSiluMul pairs logical unit 2j (gate tile j) with 2j + 1 (up tile P + j), P = N / 32
  __half* y1;
  __half* y2;
  int n0, n1;
};

// Worker (warp) w of W that holds item i of a cluster's L items, when worker w owns items
// [floor(w L / W), floor((w+1) L / W)).
__host__ __device__ inline long long gemv_worker_of(long long i, long long L, long long W) {
  return ((i + 1) * W - 1) / L;
}

// MT: 8-token tiles (M <= 8*MT); NT: 16-row tiles per unit; CW: warps per CTA; D: ring stages
// per warp; SB: group pairs per stage.
template <int MT, int NT, int CW, int D, int SB>
struct GemvCfg {
  static constexpr int kThreads = 32 * CW;
  static constexpr int kCodes = NT * SB * 2048;
  static constexpr int kScales = NT * SB * 64;
  static constexpr int kZeros = NT * SB * 16;
};

// Loads the B fragments (x') of one 64-k tile for the lane's token rows: 32 bytes per 8-token
// tile (chunks 2t and 2t+1 of row kt_local*M + m of the x' box), zero for tokens >= M.
template <int MT>
__device__ __forceinline__ void gemv_load_x(uint4 (&xv)[MT][2], const uint8_t* xs, int kt_local, int M, int r, int t,
                                            bool swz) {
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    const int m = 8 * j + r;
    if (m < M) {
      const int row = kt_local * M + m;
      const int c0 = swz ? ((2 * t) ^ (row & 7)) : 2 * t;
      const int c1 = swz ? ((2 * t + 1) ^ (row & 7)) : 2 * t + 1;
      xv[j][0] = *reinterpret_cast<const uint4*>(xs + row * 128 + c0 * 16);
      xv[j][1] = *reinterpret_cast<const uint4*>(xs + row * 128 + c1 * 16);
    } else {
      xv[j][0] = make_uint4(0, 0, 0, 0);
      xv[j][1] = make_uint4(0, 0, 0, 0);
    }
  }
}

// Adds one group (two 64-k tiles) of the stage to acc.
//   cw[kk][j]: the lane's 16 bytes of codes of k-tile kk of the group, tile j;
//   xv[kk]:    the x' fragments of k-tile kk;
//   sv[j], zz[j]: the scale pair (rows r, r+8) and zero byte of tile j for this group;
//   sx[2]:     (kSumX) the group's activation sums of tokens 0 and 1.
// Two exact dequantizations:
//  * kSumX == false (any M): a code pair is masked out of its word and OR-ed into the mantissa
//    of fp16 1024 (0x6400), giving 1024 + q (even nibbles) or 1024 + 16q (odd nibbles, 4 bits
//    higher); subtracting 1024 + z, resp. 1024 + 16z, leaves q - z or 16 (q - z), small
//    integers exact in fp16. The group's fp32 sums are scaled by S and S/16.
//  * kSumX == true (M <= 2): one AND per pair gives the codes as exact fp16 subnormals q 2^-24
//    (16q 2^-24 for the odd nibbles), and the zero point enters once per group as
//    -S z sum_k x'_mk. The group's fp32 sums are scaled by S 2^24 and S 2^20.
// Either way every tensor-core product is exact. NACC independent accumulator chains per tile
// shorten the dependent-MMA chains.
template <int MT, int NT, int NACC, bool kSumX>
__device__ __forceinline__ void gemv_group(float (&acc)[NT][MT][4], const uint4 (&cw)[2][NT],
                                           const uint4 (&xv)[2][MT][2], const uint32_t (&sv)[NT],
                                           const uint32_t (&zz)[NT], const float (&sx)[2]) {
  float tq[NACC][NT][MT][4];
#pragma unroll
  for (int a = 0; a < NACC; ++a)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int j = 0; j < MT; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) tq[a][n][j][c] = 0.f;
  uint32_t zlo[NT], zhi[NT];   // fp16 pairs 1024 + z (row r) and 1024 + 16 z (row r+8)
  if (!kSumX) {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      zlo[n] = 0x64006400u + (zz[n] & 0xFu) * 0x00010001u;
      zhi[n] = 0x64006400u + (zz[n] >> 4) * 0x00100010u;
    }
  }
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
    for (int s4 = 0; s4 < 4; ++s4) {
      const int ac = (4 * kk + s4) % NACC;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const uint4& wv = cw[kk][n];
        const uint32_t q = (s4 == 0) ? wv.x : (s4 == 1) ? wv.y : (s4 == 2) ? wv.z : wv.w;
        const uint32_t q8 = q >> 8;
        uint32_t a[4];
        if (kSumX) {
          a[0] = q & 0x000F000Fu;     // row r,   slots e0 e1:  q 2^-24
          a[1] = q & 0x00F000F0u;     // row r+8, slots e0 e1: 16q 2^-24
          a[2] = q8 & 0x000F000Fu;    // row r,   slots e2 e3
          a[3] = q8 & 0x00F000F0u;    // row r+8, slots e2 e3
        } else {
          a[0] = hsub2_u32(lop_or(q, 0x000F000Fu, 0x64006400u), zlo[n]);    // row r,   e0 e1: q - z
          a[1] = hsub2_u32(lop_or(q, 0x00F000F0u, 0x64006400u), zhi[n]);    // row r+8, e0 e1: 16 (q - z)
          a[2] = hsub2_u32(lop_or(q8, 0x000F000Fu, 0x64006400u), zlo[n]);   // row r,   e2 e3
          a[3] = hsub2_u32(lop_or(q8, 0x00F000F0u, 0x64006400u), zhi[n]);   // row r+8, e2 e3
        }
#pragma unroll
        for (int j = 0; j < MT; ++j) {
          const uint4& xq = xv[kk][j][s4 >> 1];
          mma_m16n8k16_f32(tq[ac][n][j], a, (s4 & 1) ? xq.z : xq.x, (s4 & 1) ? xq.w : xq.y);
        }
      }
    }
  }
#pragma unroll
  for (int a = 1; a < NACC; ++a)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int j = 0; j < MT; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) tq[0][n][j][c] += tq[a][n][j][c];
  if (kSumX) {
    // acc element c holds token 2t + (c & 1); only tokens 0 and 1 exist here (M <= 2)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const float2 sf = half2_bits_to_float2(sv[n]);
      const float c_lo = sf.x * 16777216.0f, c_hi = sf.y * 1048576.0f;
      const float d_lo = -sf.x * small_uint_to_float(zz[n] & 0xFu);
      const float d_hi = -sf.y * small_uint_to_float(zz[n] >> 4);
      acc[n][0][0] = fmaf(d_lo, sx[0], fmaf(c_lo, tq[0][n][0][0], acc[n][0][0]));
      acc[n][0][1] = fmaf(d_lo, sx[1], fmaf(c_lo, tq[0][n][0][1], acc[n][0][1]));
      acc[n][0][2] = fmaf(d_hi, sx[0], fmaf(c_hi, tq[0][n][0][2], acc[n][0][2]));
      acc[n][0][3] = fmaf(d_hi, sx[1], fmaf(c_hi, tq[0][n][0][3], acc[n][0][3]));
    }
  } else {
    // acc += S (sum x (q - z)); rows r+8 carry 16 (q - z)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const float2 sf = half2_bits_to_float2(sv[n]);
      const float c_lo = sf.x, c_hi = sf.y * 0.0625f;
#pragma unroll
      for (int j = 0; j < MT; ++j) {
        acc[n][j][0] = fmaf(c_lo, tq[0][n][j][0], acc[n][j][0]);
        acc[n][j][1] = fmaf(c_lo, tq[0][n][j][1], acc[n][j][1]);
        acc[n][j][2] = fmaf(c_hi, tq[0][n][j][2], acc[n][j][2]);
        acc[n][j][3] = fmaf(c_hi, tq[0][n][j][3], acc[n][j][3]);
      }
    }
  }
}

// The activation sums of tokens 0 and 1 over one group (k-tiles kt0, kt0 + 1 of the stage's x'
// box, M <= 2 rows per k-tile, no swizzle): each lane adds 4 values, then a butterfly.
__device__ __forceinline__ void gemv_group_xsums(float (&sx)[2], const uint8_t* xs, int kt0, int M, int lane) {
  const int kt = kt0 + (lane >> 4), k4 = 4 * (lane & 15);
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    float v = 0.f;
    if (m < M) {
      const uint2 q = *reinterpret_cast<const uint2*>(xs + (kt * M + m) * 128 + k4 * 2);
      const float2 a0 = half2_bits_to_float2(q.x);
      const float2 a1 = half2_bits_to_float2(q.y);
      v = (a0.x + a0.y) + (a1.x + a1.y);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    }
    sx[m] = v;
  }
}

template <int MT, int NT, int CW, int D, int SB, int NACC, bool kSumX>
__global__ void __launch_bounds__(GemvCfg<MT, NT, CW, D, SB>::kThreads, 1)
    awq_gemv_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemvArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int cid = static_cast<int>(blockIdx.x) / CL;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = a.M, G2 = a.g2;
  const int rec_elems = NT * 16 * M;   // floats per record
  uint8_t* ring = smem + static_cast<size_t>(warp) * D * a.stage_bytes;
  float* rec_all = reinterpret_cast<float*>(smem + static_cast<size_t>(CW) * D * a.stage_bytes);
  float* rec = rec_all + static_cast<size_t>(warp) * a.rec_per_warp * rec_elems;
  uint64_t* bars = reinterpret_cast<uint64_t*>(rec_all + static_cast<size_t>(CW) * a.rec_per_warp * rec_elems);
  uint64_t* full = bars + warp * D;
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + CW * D);

  // ---- this cluster's units and this warp's item range
  const long long u0 = static_cast<long long>(cid) * a.units / a.clusters;
  const long long u1 = static_cast<long long>(cid + 1) * a.units / a.clusters;
  const long long L = (u1 - u0) * G2;
  const long long Wc = static_cast<long long>(CL) * CW;
  const long long wk = static_cast<long long>(rank) * CW + warp;
  const long long i0 = wk * L / Wc, i1 = (wk + 1) * L / Wc;

  if (threadIdx.x == 0) *s_abort = 0;
  if (lane == 0) {
    for (int d = 0; d < D; ++d) mbar_init(&full[d], 1);
    mbar_fence_init();
  }
  __syncthreads();
  // The next kernel of the stream may launch at once: it reads only its own packed weights before
  // its griddepcontrol.wait, which returns after this grid has completed. Chained decode launches
  // thereby overlap their weight streams with this one's tail.
  pdl_launch_dependents();
  const unsigned long long budget = g_wait_budget_ns;

  // Walk of a warp's items in stages: a stage starts at (unit u, pair p) and holds
  // min(SB, pairs left in the unit, items left) pairs. Cursors advance without divisions.
  struct Cursor {
    long long it;   // item index within the cluster's range
    int u;          // unit (absolute)
    int p;          // group pair within the unit
  };
  auto stage_np = [&](const Cursor& c) -> int {
    const long long left = i1 - c.it;
    const int left_unit = G2 - c.p;
    return static_cast<int>(min(static_cast<long long>(min(SB, left_unit)), left));
  };
  auto advance = [&](Cursor& c, int np) {
    c.it += np;
    c.p += np;
    if (c.p == G2) { c.p = 0; ++c.u; }
  };
  auto issue_weights = [&](int slot, const Cursor& c) {   // one lane
    const int np = stage_np(c);
    const int nvalid = min(NT, a.ntiles - c.u * NT);
    uint8_t* sb = ring + static_cast<size_t>(slot) * a.stage_bytes;
    mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nvalid * np * (2048 + 64 + 16) + a.x_box_bytes));
    for (int j = 0; j < nvalid; ++j) {
      const size_t tp = static_cast<size_t>(c.u * NT + j) * G2 + c.p;   // (tile, pair) index
      bulk_g2s(sb + j * SB * 2048, a.qweight + tp * 2048, np * 2048, &full[slot]);
      bulk_g2s(sb + a.off_scales + j * SB * 64, a.scales + tp * 64, np * 64, &full[slot]);
      bulk_g2s(sb + a.off_zeros + j * SB * 16, a.zeros + tp * 16, np * 16, &full[slot]);
    }
  };
  auto issue_x = [&](int slot, const Cursor& c) {   // one lane
    tma_load_3d(ring + static_cast<size_t>(slot) * a.stage_bytes + a.off_x, &tmap_x, 0, 0, 4 * c.p, &full[slot]);
  };
  const Cursor start = {i0, static_cast<int>(u0 + i0 / G2), static_cast<int>(i0 % G2)};

  // ---- prologue: the first ring pass of weights, before waiting on the previous kernel
  const bool drop0 = g_debug_drop_first_copy != 0;
  Cursor isc = start;   // next stage to issue
  int npro = 0;
  for (; npro < D && isc.it < i1; ++npro) {
    if (lane == 0 && !(drop0 && npro == 0)) issue_weights(npro, isc);
    advance(isc, stage_np(isc));
  }
  if (lane == 0 && i0 < i1) tma_prefetch_desc(&tmap_x);
  __syncwarp();
  pdl_wait();
  if (lane == 0) {
    Cursor c = start;
    for (int s = 0; s < npro; ++s) {
      if (!(drop0 && s == 0)) issue_x(s, c);
      advance(c, stage_np(c));
    }
  }
  __syncwarp();

  // ---- stream the range
  const int r = lane >> 2, t = lane & 3;
  const bool swz = a.x_swizzle != 0;
  float acc[NT][MT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[n][j][c] = 0.f;
  int ri = 0;
  auto flush = [&]() {
    float* pr = rec + static_cast<size_t>(ri) * rec_elems;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int j = 0; j < MT; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int m = 8 * j + 2 * t + (c & 1);
          const int row = 16 * n + r + 8 * (c >> 1);
          if (m < M) pr[row * M + m] = acc[n][j][c];
          acc[n][j][c] = 0.f;
        }
  };
  bool ok = true;
  int slot = 0;
  uint32_t phase = 0;
  Cursor cs = start;   // next stage to consume
  while (cs.it < i1) {
    const int np = stage_np(cs);
    ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[slot], phase, s_abort, budget));
    if (!ok) break;
    const uint8_t* sb = ring + static_cast<size_t>(slot) * a.stage_bytes;
#pragma unroll
    for (int pp = 0; pp < SB; ++pp) {
      if (pp < np) {
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          uint4 xv[2][MT][2];
          uint4 cw[2][NT];
          uint32_t sv[NT], zz[NT];
          float sx[2] = {0.f, 0.f};
          if (kSumX) gemv_group_xsums(sx, sb + a.off_x, 4 * pp + 2 * gg, M, lane);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            gemv_load_x<MT>(xv[kk], sb + a.off_x, 4 * pp + 2 * gg + kk, M, r, t, swz);
#pragma unroll
            for (int n = 0; n < NT; ++n)
              cw[kk][n] = *reinterpret_cast<const uint4*>(sb + (n * SB + pp) * 2048 + (2 * gg + kk) * 512 + lane * 16);
          }
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            sv[n] = *reinterpret_cast<const uint32_t*>(sb + a.off_scales + (n * SB + pp) * 64 + gg * 32 + r * 4);
            zz[n] = sb[a.off_zeros + (n * SB + pp) * 16 + gg * 8 + r];
          }
          gemv_group<MT, NT, NACC, kSumX>(acc, cw, xv, sv, zz, sx);
        }
      }
    }
    // the stage is consumed: refill it with the next stage of the range
    __syncwarp();
    fence_proxy_async_smem();
    if (isc.it < i1) {
      if (lane == 0) {
        issue_weights(slot, isc);
        issue_x(slot, isc);
      }
      advance(isc, stage_np(isc));
    }
    __syncwarp();
    const int u_before = cs.u;
    advance(cs, np);
    if (cs.u != u_before && cs.it < i1) {   // the next stage starts a new unit: record this one
      flush();
      ++ri;
    }
    if (++slot == D) { slot = 0; phase ^= 1; }
  }
  if (ok) {
    if (i0 < i1) flush();
  } else {
    // drain the copies still in flight (stages cs .. isc) before the CTA may exit
    int never = 0;
    Cursor q = cs;
    int s = slot;
    uint32_t ph = phase;
    while (q.it < isc.it) {
      if (lane == 0 && !(drop0 && q.it == i0)) mbar_wait_bounded(&full[s], ph, &never, kDrainBudgetNs);
      advance(q, stage_np(q));
      if (++s == D) { s = 0; ph ^= 1; }
    }
    __syncwarp();
  }

  // ---- cluster reduction: each output of the cluster's units is the sum of the records of
  // the workers that touched its unit, in worker order. One warp per unit: its lanes find the
  // contributing workers (32-bit arithmetic: a cluster holds fewer than 2^23 items and at most
  // 256 workers), then add their records element by element.
  cluster_arrive();
  cluster_wait();
  if (*s_abort == 0) {
    const uint32_t Lu = static_cast<uint32_t>(L), W32 = static_cast<uint32_t>(Wc);
    const int R = a.rec_per_warp;
    const int nunits = static_cast<int>(u1 - u0);
    const int per_unit = M * NT * 16;
    for (int ur = rank * CW + warp; ur < nunits; ur += CL * CW) {
      const uint32_t first = static_cast<uint32_t>(ur) * G2, last = first + G2 - 1;
      const uint32_t wf = ((first + 1) * W32 - 1) / Lu, wl = ((last + 1) * W32 - 1) / Lu;
      const int ncontrib = static_cast<int>(wl - wf) + 1;
      const size_t ybase = static_cast<size_t>(u0 + ur) * (NT * 16);
      // lane l describes contributor wf + l (at most 32: the host keeps CL * CW <= 32): its CTA and
      // the float offset of its record for this unit
      const uint32_t w = wf + lane;
      int cta = -1, off = 0;
      if (lane < ncontrib) {
        const uint32_t aw = w * Lu / W32, bw = (w + 1) * Lu / W32;
        if (bw > aw) {
          cta = static_cast<int>(w / CW);
          off = (static_cast<int>(w % CW) * R + (ur - static_cast<int>(aw / G2))) * rec_elems;
        }
      }
      // every lane runs every iteration (the shuffles need the whole warp); lanes past the unit's
      // outputs only skip the loads and the store
      for (int e0 = 0; e0 < per_unit; e0 += 32) {
        const int e = e0 + lane;
        const bool live = e < per_unit;
        const int m = live ? e / (NT * 16) : 0, row = live ? e - m * (NT * 16) : 0;
        float v = 0.f;
        for (int c = 0; c < ncontrib; ++c) {
          const int cc = __shfl_sync(0xFFFFFFFFu, cta, c);
          const int oo = __shfl_sync(0xFFFFFFFFu, off, c);
          if (live && cc >= 0) v += cluster.map_shared_rank(rec_all, cc)[oo + row * M + m];
        }
        const size_t n = ybase + row;
        if (live && n < static_cast<size_t>(a.N)) a.y[static_cast<size_t>(m) * a.N + n] = __float2half_rn(v);
      }
    }
  }
  // no CTA leaves while another may still read its shared memory
  cluster_arrive();
  cluster_wait();
}


// ------------------------------------------------------------------------------------
// Shared-ring form: one producer lane streams the CTA's contiguous item range (with 16-row
// units a CTA's range is one contiguous byte range of each packed array in layout v2) into a
// ring of S stages of up to SB group pairs of one tile; CW consumer warps split each stage's
// group pairs. Every consumer warp writes a record for every unit of the CTA's range (zeros
// where it had no item), the CTA adds its warps' records in warp order, and the cluster adds
// the CTAs' records of each unit in rank order through distributed shared memory.
template <int CW, int SB>
struct GemvRingCfg {
  static constexpr int kThreads = 32 * (CW + 1);
  static constexpr int kCodes = SB * 2048;
  static constexpr int kScales = SB * 64;
  static constexpr int kZeros = SB * 16;
};

template <int MT, int CW, int S, int SB, int NACC, bool kSumX, int EPI>
__global__ void __launch_bounds__(GemvRingCfg<CW, SB>::kThreads, 1)
    awq_gemv_ring_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemvArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int cid = static_cast<int>(blockIdx.x) / CL;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = a.M, G2 = a.g2;
  const int rec_elems = 16 * M;   // floats per record (one 16-row unit)
  const int R = a.rec_per_warp;   // units a CTA's range touches at most
  float* rec_all = reinterpret_cast<float*>(smem + static_cast<size_t>(S) * a.stage_bytes);   // [CW][R][16][M]
  uint64_t* full = reinterpret_cast<uint64_t*>(rec_all + static_cast<size_t>(CW) * R * rec_elems);
  uint64_t* empty = full + S;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + S);

  // ---- this cluster's units and this CTA's item range (kEpiSiluMul: whole gate/up unit pairs)
  const int P = a.N / 32;
  const long long upc = EPI == kEpiSiluMul ? 2 : 1;
  const long long u0 = upc * (static_cast<long long>(cid) * (a.units / upc) / a.clusters);
  const long long u1 = upc * (static_cast<long long>(cid + 1) * (a.units / upc) / a.clusters);
  const long long L = (u1 - u0) * G2;
  const long long i0 = static_cast<long long>(rank) * L / CL, i1 = static_cast<long long>(rank + 1) * L / CL;
  // physical tile of a (logical) unit
  auto tile_of = [&](int u) -> int { return EPI == kEpiSiluMul ? ((u & 1) ? P + (u >> 1) : (u >> 1)) : u; };

  if (threadIdx.x == 0) {
    for (int d = 0; d < S; ++d) {
      mbar_init(&full[d], 1);
      mbar_init(&empty[d], CW);
    }
    *s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  const unsigned long long budget = g_wait_budget_ns;

  struct Cursor {
    long long it;   // item index within the cluster's range
    int u;          // unit (absolute)
    int p;          // group pair within the unit
  };
  auto stage_np = [&](const Cursor& c) -> int {
    const long long left = i1 - c.it;
    return static_cast<int>(min(static_cast<long long>(min(SB, G2 - c.p)), left));
  };
  auto advance = [&](Cursor& c, int np) {
    c.it += np;
    c.p += np;
    if (c.p == G2) { c.p = 0; ++c.u; }
  };
  const Cursor start = {i0, static_cast<int>(u0 + i0 / G2), static_cast<int>(i0 % G2)};
  const bool drop0 = g_debug_drop_first_copy != 0;
  bool ok = true;

  if (warp == CW) {
    // ---------------------------------------------------------------- producer lane
    if (lane == 0) {
      auto issue_weights = [&](int slot, const Cursor& c) {
        const int np = stage_np(c);
        uint8_t* sb = smem + static_cast<size_t>(slot) * a.stage_bytes;
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(np * (2048 + 64 + 16) + a.x_box_bytes));
        const size_t tp = static_cast<size_t>(tile_of(c.u)) * G2 + c.p;   // (tile, pair) index
        bulk_g2s(sb, a.qweight + tp * 2048, np * 2048, &full[slot]);
        bulk_g2s(sb + a.off_scales, a.scales + tp * 64, np * 64, &full[slot]);
        bulk_g2s(sb + a.off_zeros, a.zeros + tp * 16, np * 16, &full[slot]);
      };
      auto issue_x = [&](int slot, const Cursor& c) {
        tma_load_3d(smem + static_cast<size_t>(slot) * a.stage_bytes + a.off_x, &tmap_x, 0, 0, 4 * c.p, &full[slot]);
      };
      // first ring pass of weights before waiting on the previous kernel
      Cursor isc = start;
      int npro = 0;
      for (; npro < S && isc.it < i1; ++npro) {
        if (!(drop0 && npro == 0)) issue_weights(npro, isc);
        advance(isc, stage_np(isc));
      }
      if (i0 < i1) tma_prefetch_desc(&tmap_x);
      pdl_wait();
      {
        Cursor c = start;
        for (int s = 0; s < npro; ++s) {
          if (!(drop0 && s == 0)) issue_x(s, c);
          advance(c, stage_np(c));
        }
      }
      int slot = 0;
      uint32_t phase = 0;
      for (int s = npro; isc.it < i1; ++s) {
        // refill the slot of stage s - S once its consumers have released it
        if (!mbar_wait_bounded(&empty[slot], phase, s_abort, budget)) { ok = false; break; }
        issue_weights(slot, isc);
        issue_x(slot, isc);
        advance(isc, stage_np(isc));
        if (++slot == S) { slot = 0; phase ^= 1; }
      }
      // drain: the last S stages this lane issued may still be in flight if the consumers stopped
      // early; wait for each (their phases are the most recent of their slots)
      int n_issued = 0;
      for (Cursor q = start; q.it < isc.it; advance(q, stage_np(q))) ++n_issued;
      int never = 0;
      for (int s2 = max(0, n_issued - S); s2 < n_issued; ++s2)
        if (!(drop0 && s2 == 0)) mbar_wait_bounded(&full[s2 % S], static_cast<uint32_t>((s2 / S) & 1), &never,
                                                   kDrainBudgetNs);
    }
  } else {
    // ---------------------------------------------------------------- consumer warps
    pdl_wait();
    const int r = lane >> 2, t = lane & 3;
    const bool swz = a.x_swizzle != 0;
    float acc[1][MT][4];
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[0][j][c] = 0.f;
    float* rec = rec_all + static_cast<size_t>(warp) * R * rec_elems;
    int ri = 0;
    auto flush = [&]() {
      float* pr = rec + static_cast<size_t>(ri) * rec_elems;
#pragma unroll
      for (int j = 0; j < MT; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int m = 8 * j + 2 * t + (c & 1);
          const int row = r + 8 * (c >> 1);
          if (m < M) pr[row * M + m] = acc[0][j][c];
          acc[0][j][c] = 0.f;
        }
    };
    int slot = 0;
    uint32_t phase = 0;
    Cursor cs = start;
    while (cs.it < i1) {
      const int np = stage_np(cs);
      ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[slot], phase, s_abort, budget));
      if (!ok) break;
      const uint8_t* sb = smem + static_cast<size_t>(slot) * a.stage_bytes;
#pragma unroll
      for (int pi = 0; pi < (SB + CW - 1) / CW; ++pi) {
        const int pp = warp + pi * CW;
        if (pp < np) {
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            uint4 xv[2][MT][2];
            uint4 cw[2][1];
            uint32_t sv[1], zz[1];
            float sx[2] = {0.f, 0.f};
            if (kSumX) gemv_group_xsums(sx, sb + a.off_x, 4 * pp + 2 * gg, M, lane);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              gemv_load_x<MT>(xv[kk], sb + a.off_x, 4 * pp + 2 * gg + kk, M, r, t, swz);
              cw[kk][0] = *reinterpret_cast<const uint4*>(sb + pp * 2048 + (2 * gg + kk) * 512 + lane * 16);
            }
            sv[0] = *reinterpret_cast<const uint32_t*>(sb + a.off_scales + pp * 64 + gg * 32 + r * 4);
            zz[0] = sb[a.off_zeros + pp * 16 + gg * 8 + r];
            gemv_group<MT, 1, NACC, kSumX>(acc, cw, xv, sv, zz, sx);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      const int u_before = cs.u;
      advance(cs, np);
      if (cs.u != u_before && cs.it < i1) {   // the next stage starts a new unit: record this one
        flush();
        ++ri;
      }
      if (++slot == S) { slot = 0; phase ^= 1; }
    }
    if (ok && i0 < i1) flush();
  }

  // ---- the CTA adds its consumer warps' records, in warp order (all threads of the CTA)
  __syncthreads();
  if (*s_abort == 0) {
    const int n_rec = (i0 < i1) ? static_cast<int>((i1 - 1) / G2 - i0 / G2) + 1 : 0;
    for (int e = threadIdx.x; e < n_rec * rec_elems; e += blockDim.x) {
      float v = 0.f;
      for (int w = 0; w < CW; ++w) v += rec_all[static_cast<size_t>(w) * R * rec_elems + e];
      rec_all[e] = v;   // warp 0's records now hold the CTA's sums
    }
  }
  // ---- cluster reduction: each output is the sum of the records of the CTAs that touched its
  // unit, in rank order. One warp per unit (per gate/up pair with kEpiSiluMul).
  cluster_arrive();
  cluster_wait();
  if (*s_abort == 0) {
    const uint32_t Lu = static_cast<uint32_t>(L), CLu = static_cast<uint32_t>(CL);
    const int nunits = static_cast<int>(u1 - u0);
    const int nwarps = CW + 1;
    // the sum over the contributing CTAs of element (row, m) of relative unit ur
    auto unit_sum = [&](int ur, int row, int m) -> float {
      const uint32_t first = static_cast<uint32_t>(ur) * G2, last = first + G2 - 1;
      const uint32_t cf = ((first + 1) * CLu - 1) / Lu, cl_ = ((last + 1) * CLu - 1) / Lu;
      float v = 0.f;
      for (uint32_t c = cf; c <= cl_; ++c) {
        const uint32_t ac = c * Lu / CLu, bc = (c + 1) * Lu / CLu;
        if (bc == ac) continue;
        const int rr = ur - static_cast<int>(ac / G2);
        v += cluster.map_shared_rank(rec_all, static_cast<int>(c))[rr * rec_elems + row * M + m];
      }
      return v;
    };
    if (EPI == kEpiSiluMul) {
      const int I = a.N / 2;
      for (int pr = rank * nwarps + warp; 2 * pr < nunits; pr += CL * nwarps) {
        const int j = static_cast<int>(u0 / 2) + pr;   // gate tile j, up tile P + j
        for (int e = lane; e < rec_elems; e += 32) {
          const int row = e / M, m = e - row * M;
          const float g = unit_sum(2 * pr, row, m), u = unit_sum(2 * pr + 1, row, m);
          const int i = 16 * j + row;
          if (i < I) a.y[static_cast<size_t>(m) * I + i] = __float2half_rn(silu_mul(g, u));
        }
      }
    } else {
      EpiArgs epi = {a.y, a.y1, a.y2, a.n0, a.n1};
      for (int ur = rank * nwarps + warp; ur < nunits; ur += CL * nwarps) {
        const long long nbase = static_cast<long long>(u0 + ur) * 16;
        for (int e = lane; e < rec_elems; e += 32) {
          const int row = e / M, m = e - row * M;
          const float v = unit_sum(ur, row, m);
          const long long n = nbase + row;
          if (n < a.N) epi_store<EPI>(epi, m, n, a.N, v);
        }
      }
    }
  }
  // no CTA leaves while another may still read its shared memory
  cluster_arrive();
  cluster_wait();
}

}  // namespace awq
