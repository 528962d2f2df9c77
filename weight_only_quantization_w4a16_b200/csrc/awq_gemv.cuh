// awq_gemv.cuh — a3: decode W4A16 linear layer, 1 <= M <= 32.
//
// llm-awq README, "Installation" step 3: W4A16 (4-bit weight, 16-bit
// activation) kernels for the decode stage. y[M,N] = x'[M,K] . ((q-z)*S)^T,
// fp32 accumulation, fp16 output.
//
// The layer is HBM-bound (0.52 bytes of packed weight per weight, about
// 3.85*M flop per byte). Design for B200:
//  * work items are (16-row unit, group pair): 2048 bytes of codes, 64 of scales
//    and 16 of zeros per item in packed layout v2, where every tile's data runs
//    contiguously along K, so a run of items is one contiguous byte range of
//    each packed array;
//  * stream-K split: the units are divided evenly over thread-block clusters
//    (unit-aligned), and a cluster's items evenly over its CTAs, so each CTA owns
//    one contiguous item range;
//  * one producer lane per CTA streams that range into a ring of S stages, each
//    a run of up to CW * SBW group pairs of one unit: three 1-D bulk copies
//    (codes, scales, zeros; copies of several KB keep HBM efficient) and one 3-D
//    TMA box of the stage's x' k-tiles (zero fill past K);
//  * the weights of the first ring pass are requested before the kernel waits
//    on its stream predecessor, and the kernel lets its dependents launch at
//    once (programmatic dependent launch), so consecutive decode launches
//    overlap their weight streams;
//  * CW consumer warps split each stage's group pairs (SBW each). The packed
//    layout makes a lane's 16 bytes exactly the m16n8k16 A-fragments of 4
//    k-steps for rows r, r+8; a code pair is masked out of its word and OR-ed
//    into the mantissa of fp16 1024 (one LOP3), one HSUB2 of 1024 + z leaves
//    q - z (16 (q - z) for the odd nibbles), so every tensor-core product is
//    exact; S is applied in fp32 to each group's sums. The integer pipe runs at
//    half rate and dequantization alone needs a large part of it at HBM speed,
//    so the rest of the loop is kept lean: compile-time stage offsets, 32-bit
//    cursors, accumulator chains that start from a zero operand;
//  * every consumer warp writes a partial-sum record for every unit of its
//    CTA's range; the CTA adds its warps' records in warp order, then the
//    cluster adds the CTAs' records of each unit in rank order through
//    distributed shared memory (deterministic, no global scratch, no atomics).
#pragma once

#include <cooperative_groups.h>

#include "awq_common.cuh"
#include "awq_gemm.cuh"

namespace awq {

// Per-launch arguments of the decode kernel.
struct GemvArgs {
  const uint8_t* qweight;   // packed codes (layout v2), 2048 bytes per (tile, group pair)
  const uint8_t* scales;    // 64 bytes per (tile, group pair)
  const uint8_t* zeros;     // 16 bytes per (tile, group pair)
  __half* y;                // [M, N] (kEpiSplit3: the first output; kEpiSiluMul: h [M, N/2])
  __half* y1;               // kEpiSplit3: second and third outputs
  __half* y2;
  int n0, n1;               // kEpiSplit3: widths of the first and second outputs
  int M, N;
  int g2;                   // group pairs per tile: ceil(K / 256)
  int units;                // 16-row units (tiles; kEpiSiluMul: 2 per gate/up pair)
  int clusters;             // clusters in the grid
  int rec_per_warp;         // units a CTA's item range touches at most
  int stage_bytes;          // bytes of one ring stage (multiple of 128, or 1024 with swizzle)
  int x_box_bytes;          // bytes of the stage's x' box (4 * SB k-tiles x M tokens x 128)
};

template <int CW, int SBW, bool kSwz>
struct GemvCfg {
  static constexpr int kThreads = 32 * (CW + 1);
  static constexpr int kSB = CW * SBW;                       // group pairs per stage
  static constexpr int kOffS = kSB * 2048;                   // scales after the codes
  static constexpr int kOffZ = kOffS + kSB * 64;             // zeros after the scales
  static constexpr int kAlignX = kSwz ? 1024 : 128;
  static constexpr int kOffX = (kOffZ + kSB * 16 + kAlignX - 1) / kAlignX * kAlignX;
};

// Loads the B fragments (x') of one 64-k tile for the lane's token rows: 32 bytes per 8-token
// tile (chunks 2t and 2t+1 of row kt_local*M + m of the x' box). With one token tile, lanes of
// tokens m >= M read token M-1 instead: those MMA columns are never stored, so they need no
// zeroing. (With more tiles the select keeps register pressure lower.)
template <int MT, bool kSwz>
__device__ __forceinline__ void gemv_load_x(uint4 (&xv)[MT][2], const uint8_t* xs, int kt_local, int M, int r, int t) {
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    const int m = MT == 1 ? min(r, M - 1) : 8 * j + r;
    const int row = kt_local * M + m;
    const int c0 = kSwz ? ((2 * t) ^ (row & 7)) : 2 * t;
    const int c1 = kSwz ? ((2 * t + 1) ^ (row & 7)) : 2 * t + 1;
    const bool live = MT == 1 || m < M;
    xv[j][0] = live ? *reinterpret_cast<const uint4*>(xs + row * 128 + c0 * 16) : make_uint4(0, 0, 0, 0);
    xv[j][1] = live ? *reinterpret_cast<const uint4*>(xs + row * 128 + c1 * 16) : make_uint4(0, 0, 0, 0);
  }
}

// Adds one group (two 64-k tiles) to acc.
//   c0, c1: the lane's 16 bytes of codes of the group's two k-tiles;
//   xv[kk]: the x' fragments of k-tile kk;   sv, zz: scale pair (rows r, r+8) and zero byte.
// Exact dequantization (see the file header); two accumulator chains of four MMAs, each
// starting from a zero operand.
template <int MT>
__device__ __forceinline__ void gemv_group(float (&acc)[MT][4], const uint4& c0, const uint4& c1,
                                           const uint4 (&xv)[2][MT][2], uint32_t sv, uint32_t zz) {
  float tq[2][MT][4];
  const uint32_t zlo = 0x64006400u + (zz & 0xFu) * 0x00010001u;   // fp16 pair 1024 + z (row r)
  const uint32_t zhi = 0x64006400u + (zz >> 4) * 0x00100010u;    // 1024 + 16 z (row r+8)
#pragma unroll
  for (int kk = 0; kk < 2; ++kk) {
    const uint4& wv = kk ? c1 : c0;
#pragma unroll
    for (int s4 = 0; s4 < 4; ++s4) {
      const int ac = s4 & 1;
      const uint32_t q = (s4 == 0) ? wv.x : (s4 == 1) ? wv.y : (s4 == 2) ? wv.z : wv.w;
      const uint32_t q8 = __umulhi(q, 1u << 24);   // q >> 8 on the multiply pipe
      uint32_t a[4];
      a[0] = hsub2_u32(lop_or(q, 0x000F000Fu, 0x64006400u), zlo);    // row r,   e0 e1: q - z
      a[1] = hsub2_u32(lop_or(q, 0x00F000F0u, 0x64006400u), zhi);    // row r+8, e0 e1: 16 (q - z)
      a[2] = hsub2_u32(lop_or(q8, 0x000F000Fu, 0x64006400u), zlo);   // row r,   e2 e3
      a[3] = hsub2_u32(lop_or(q8, 0x00F000F0u, 0x64006400u), zhi);   // row r+8, e2 e3
#pragma unroll
      for (int j = 0; j < MT; ++j) {
        const uint4& xq = xv[kk][j][s4 >> 1];
        const uint32_t b0 = (s4 & 1) ? xq.z : xq.x, b1 = (s4 & 1) ? xq.w : xq.y;
        if (kk == 0 && s4 < 2) mma_m16n8k16_f32_zero(tq[ac][j], a, b0, b1);
        else mma_m16n8k16_f32(tq[ac][j], a, b0, b1);
      }
    }
  }
  // acc += S (sum x (q - z)); rows r+8 carry 16 (q - z)
  const float2 sf = half2_bits_to_float2(sv);
  const float c_lo = sf.x, c_hi = sf.y * 0.0625f;
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    acc[j][0] = fmaf(c_lo, tq[0][j][0] + tq[1][j][0], acc[j][0]);
    acc[j][1] = fmaf(c_lo, tq[0][j][1] + tq[1][j][1], acc[j][1]);
    acc[j][2] = fmaf(c_hi, tq[0][j][2] + tq[1][j][2], acc[j][2]);
    acc[j][3] = fmaf(c_hi, tq[0][j][3] + tq[1][j][3], acc[j][3]);
  }
}

// MT: 8-token tiles (M <= 8 MT); CW: consumer warps; S: ring stages; SBW: group pairs per consumer
// warp and stage; kSwz: the x' box uses the 128-byte swizzle (M > 2); EPI: epilogue; MINB: CTAs
// per SM the registers must allow (2 lets the next decode launch's CTAs become resident, and
// prefetch their weights, while this one runs).
template <int MT, int CW, int S, int SBW, bool kSwz, int EPI, int MINB>
__global__ void __launch_bounds__(GemvCfg<CW, SBW, kSwz>::kThreads, MINB)
    awq_gemv_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemvArgs a) {
  using C = GemvCfg<CW, SBW, kSwz>;
  constexpr int SB = C::kSB;
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
  const int R = a.rec_per_warp;
  float* rec_all = reinterpret_cast<float*>(smem + static_cast<size_t>(S) * a.stage_bytes);   // [CW][R][16][M]
  float* recv = rec_all + static_cast<size_t>(CW) * R * rec_elems;   // [2][16][M]: partials pushed by rank 1
  uint64_t* full = reinterpret_cast<uint64_t*>(recv + 2 * rec_elems);
  uint64_t* empty = full + S;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + S);

  // ---- this cluster's units and this CTA's item range (kEpiSiluMul: whole gate/up unit pairs).
  // A cluster holds fewer than 2^23 items, so 32-bit arithmetic suffices from here on.
  const int P = a.N / 32;
  const int upc = EPI == kEpiSiluMul ? 2 : 1;
  const int shares = a.units / upc;
  const int u0 = upc * static_cast<int>(static_cast<long long>(cid) * shares / a.clusters);
  const int u1 = upc * static_cast<int>(static_cast<long long>(cid + 1) * shares / a.clusters);
  const int L = (u1 - u0) * G2;
  const int i0 = static_cast<int>(static_cast<long long>(rank) * L / CL);
  const int i1 = static_cast<int>(static_cast<long long>(rank + 1) * L / CL);
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
  if (CL == 2) cluster_arrive_relaxed();   // first cluster phase: this CTA has started
  // The next kernel of the stream may launch at once: it reads only its own packed weights before
  // its griddepcontrol.wait, which returns after this grid has completed.
  pdl_launch_dependents();
  const unsigned long long budget = g_wait_budget_ns;

  // Stages: a stage starts at item `it` of the cluster range, unit u, pair p, and holds
  // min(SB, pairs left in the unit, items left) pairs.
  struct Cursor {
    int it, u, p;
  };
  auto stage_np = [&](const Cursor& c) -> int { return min(min(SB, G2 - c.p), i1 - c.it); };
  auto advance = [&](Cursor& c, int np) {
    c.it += np;
    c.p += np;
    if (c.p == G2) { c.p = 0; ++c.u; }
  };
  const Cursor start = {i0, u0 + i0 / G2, i0 % G2};
  const bool drop0 = g_debug_drop_first_copy != 0;
  bool ok = true;

  if (warp == CW) {
    // ---------------------------------------------------------------- producer lane
    if (lane == 0) {
      auto issue_weights = [&](int slot, const Cursor& c) {
        const int np = stage_np(c);
        // the stage's (tile, pair) range lies inside the packed arrays and the ring slot
        if (!AWQ_CHECK(tile_of(c.u) >= 0 && tile_of(c.u) < a.units && c.p >= 0 && np >= 1 && c.p + np <= G2 &&
                       np <= SB && slot >= 0 && slot < S))
          return;
        uint8_t* sb = smem + static_cast<size_t>(slot) * a.stage_bytes;
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(np * (2048 + 64 + 16) + a.x_box_bytes));
        const size_t tp = static_cast<size_t>(tile_of(c.u)) * G2 + c.p;   // (tile, pair) index
        bulk_g2s(sb, a.qweight + tp * 2048, np * 2048, &full[slot]);
        bulk_g2s(sb + C::kOffS, a.scales + tp * 64, np * 64, &full[slot]);
        bulk_g2s(sb + C::kOffZ, a.zeros + tp * 16, np * 16, &full[slot]);
      };
      auto issue_x = [&](int slot, const Cursor& c) {
        tma_load_3d(smem + static_cast<size_t>(slot) * a.stage_bytes + C::kOffX, &tmap_x, 0, 0, 4 * c.p, &full[slot]);
      };
      // first ring pass of weights before waiting on the previous kernel
      Cursor isc = start;
      int n_issued = 0;
      for (; n_issued < S && isc.it < i1; ++n_issued) {
        if (!(drop0 && n_issued == 0)) issue_weights(n_issued, isc);
        advance(isc, stage_np(isc));
      }
      if (i0 < i1) tma_prefetch_desc(&tmap_x);
      pdl_wait();
      {
        Cursor c = start;
        for (int s = 0; s < n_issued; ++s) {
          if (!(drop0 && s == 0)) issue_x(s, c);
          advance(c, stage_np(c));
        }
      }
      int slot = 0;
      uint32_t phase = 0;
      for (; isc.it < i1; ++n_issued) {
        // refill the slot of stage n_issued - S once its consumers have released it
        if (!mbar_wait_bounded(&empty[slot], phase, s_abort, budget)) { ok = false; break; }
        issue_weights(slot, isc);
        issue_x(slot, isc);
        advance(isc, stage_np(isc));
        if (++slot == S) { slot = 0; phase ^= 1; }
      }
      // drain: the last S stages issued may still be in flight if the consumers stopped early;
      // wait for each (their phases are the most recent of their slots)
      int never = 0;
      for (int s2 = max(0, n_issued - S); s2 < n_issued; ++s2)
        if (!(drop0 && s2 == 0))
          mbar_wait_bounded(&full[s2 % S], static_cast<uint32_t>((s2 / S) & 1), &never, kDrainBudgetNs);
    }
  } else {
    // ---------------------------------------------------------------- consumer warps
    pdl_wait();
    const int r = lane >> 2, t = lane & 3;
    float acc[MT][4];
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
    float* rec = rec_all + static_cast<size_t>(warp) * R * rec_elems;
    int ri = 0;
    auto flush = [&]() {
      if (!AWQ_CHECK(ri >= 0 && ri < R)) return;
      float* pr = rec + ri * rec_elems;
#pragma unroll
      for (int j = 0; j < MT; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int m = 8 * j + 2 * t + (c & 1);
          const int row = r + 8 * (c >> 1);
          if (m < M) pr[row * M + m] = acc[j][c];
          acc[j][c] = 0.f;
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
      for (int pi = 0; pi < SBW; ++pi) {
        const int pp = warp + pi * CW;
        if (pp < np) {
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const uint8_t* cb = sb + pp * 2048 + gg * 1024 + lane * 16;
            const uint4 c0 = *reinterpret_cast<const uint4*>(cb);
            const uint4 c1 = *reinterpret_cast<const uint4*>(cb + 512);
            uint4 xv[2][MT][2];
            gemv_load_x<MT, kSwz>(xv[0], sb + C::kOffX, 4 * pp + 2 * gg, M, r, t);
            gemv_load_x<MT, kSwz>(xv[1], sb + C::kOffX, 4 * pp + 2 * gg + 1, M, r, t);
            const uint32_t sv = *reinterpret_cast<const uint32_t*>(sb + C::kOffS + pp * 64 + gg * 32 + r * 4);
            const uint32_t zz = sb[C::kOffZ + pp * 16 + gg * 8 + r];
            gemv_group<MT>(acc, c0, c1, xv, sv, zz);
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

  // ---- epilogue. The cluster's items are split at L/2 between its two CTAs, so at most one
  // block of units (one unit; one gate/up unit pair with kEpiSiluMul) is shared. Each CTA adds its
  // consumer warps' records in warp order and stores the blocks it holds alone; for the shared
  // block, rank 1 pushes its sums into rank 0's shared memory, and rank 0 adds them after its own
  // (rank order: deterministic, no global scratch, no atomics).
  __syncthreads();
  const int bsz = upc * G2;                                  // items per block
  const int split = L / 2;
  const bool shared_blk = CL == 2 && split > 0 && split < L && (split - 1) / bsz == split / bsz;
  const int bb = split / bsz;                                // the shared block (relative)
  const bool live = *s_abort == 0 && i0 < i1;
  const int uf = i0 / G2, ul = (i1 - 1) / G2;                // units of this CTA's records (relative)
  // element e of relative unit ur summed over this CTA's warps (zero for a unit it did not touch)
  auto cta_sum = [&](int ur, int e) -> float {
    if (ur < uf || ur > ul) return 0.f;
    if (!AWQ_CHECK(ur - uf < R && e >= 0 && e < rec_elems)) return 0.f;
    const float* pr = rec_all + static_cast<size_t>(ur - uf) * rec_elems + e;
    float v = 0.f;
#pragma unroll 4
    for (int w = 0; w < CW; ++w) v += pr[static_cast<size_t>(w) * R * rec_elems];
    return v;
  };
  // stores block b; `extra` (rank 0, shared block) holds rank 1's sums of the block's units
  auto finalize = [&](int b, int e, const float* extra) {
    const int row = e / M, m = e - row * M;
    if (EPI == kEpiSiluMul) {
      float g = cta_sum(2 * b, e), u = cta_sum(2 * b + 1, e);
      if (extra != nullptr) { g += extra[e]; u += extra[rec_elems + e]; }
      const int I = a.N / 2;
      const int i = 16 * (u0 / 2 + b) + row;
      if (i < I) a.y[static_cast<size_t>(m) * I + i] = __float2half_rn(silu_mul(g, u));
    } else {
      float v = cta_sum(b, e);
      if (extra != nullptr) v += extra[e];
      const long long n = static_cast<long long>(u0 + b) * 16 + row;
      if (n < a.N) epi_store<EPI>(EpiArgs{a.y, a.y1, a.y2, a.n0, a.n1}, m, n, a.N, v);
    }
  };
  if (CL == 2) {
    cluster_wait();                                          // both CTAs have started
    if (rank == 0) cluster_arrive_relaxed();                 // second phase: rank 0 only receives
    else {
      if (live && shared_blk) {
        float* dst = cluster.map_shared_rank(recv, 0);
        for (int idx = threadIdx.x; idx < upc * rec_elems && AWQ_CHECK(idx < 2 * rec_elems); idx += blockDim.x)
          dst[idx] = cta_sum(bb * upc + idx / rec_elems, idx % rec_elems);
      }
      cluster_arrive();                                      // release: the pushed sums
    }
  }
  if (live) {
    const int fb = uf / upc, lb = ul / upc;
    const int b0 = (shared_blk && rank == 1) ? fb + 1 : fb;  // rank 1's first block is the shared one
    const int b1 = (shared_blk && rank == 0) ? lb - 1 : lb;  // rank 0's last block is the shared one
    for (int idx = threadIdx.x; idx < (b1 - b0 + 1) * rec_elems; idx += blockDim.x)
      finalize(b0 + idx / rec_elems, idx % rec_elems, nullptr);
  }
  if (CL == 2) {
    cluster_wait();                                          // rank 1's sums are in `recv`
    if (rank == 0 && live && shared_blk)
      for (int e = threadIdx.x; e < rec_elems; e += blockDim.x) finalize(bb, e, recv);
  }
}

}  // namespace awq
