// awq_gemv.cuh — a3: decode W4A16 linear layer, 1 <= M <= 32.
//
// llm-awq README, "Installation" step 3: W4A16 (4-bit weight, 16-bit
// activation) kernels for the decode stage. y[M,N] = x'[M,K] . ((q-z)*S)^T,
// fp32 accumulation, fp16 output.
//
// The layer is HBM-bound (0.52 bytes of packed weight per weight, about
// 3.85*M flop per byte). Design for B200:
//  * packed layout v1 makes one 16-byte load per lane exactly the m16n8k16
//    A-fragments of 4 k-steps for rows r, r+8 of a 16-row tile, and the
//    matching activation slots a contiguous 32-byte run of x' per token;
//  * codes become exact fp16 integers (q - z) with one LOP3 (OR-ing the
//    0x6400 exponent) and one HSUB2 per pair; odd nibbles are left x16 and
//    compensated in fp32; the per-group scale S is applied in fp32 to the
//    group's partial sums, so the tensor-core products are exact;
//  * weights stream through a register ring D k-tiles deep with
//    L1::no_allocate 128-bit loads; activations come through L1;
//  * a thread-block cluster of CL CTAs splits K; the CTAs add their partial
//    sums through distributed shared memory in rank order (deterministic, no
//    global scratch, no atomics).
#pragma once

#include <cooperative_groups.h>

#include "awq_common.cuh"

namespace awq {

// MT: 8-token tiles (M <= 8*MT); NT: 16-row tiles per warp; RW: warps per CTA; D: ring depth (k-tiles, even)
template <int MT, int NT, int RW, int D>
struct GemvCfg {
  static constexpr int kRows = RW * NT * kTileRows;   // rows per CTA
  static constexpr int kThreads = RW * 32;
  static_assert(D % 2 == 0, "ring depth must cover whole groups");
  static_assert(kSuperRows % kRows == 0, "a CTA must not straddle super-tiles");
};

template <int MT, int NT, int RW, int D>
__global__ void __launch_bounds__(GemvCfg<MT, NT, RW, D>::kThreads) gemv_kernel(
    const __half* __restrict__ x, const uint32_t* __restrict__ qweight, const __half* __restrict__ scales,
    const uint8_t* __restrict__ zeros, __half* __restrict__ y, int M, int N, int K) {
  using Cfg = GemvCfg<MT, NT, RW, D>;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());

  extern __shared__ __align__(16) float s_part[];   // [kRows][M]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, t = lane & 3;               // mma fragment row / column block
  const int G = K / kGroup, KT = K / kKTile;
  const int g0 = static_cast<int>((static_cast<long long>(G) * rank) / CL);
  const int g1 = static_cast<int>((static_cast<long long>(G) * (rank + 1)) / CL);
  const int kt0 = 2 * g0;
  const int nkt = 2 * (g1 - g0);

  const int row0 = blockIdx.x * Cfg::kRows + warp * NT * kTileRows;   // first row of this warp
  const int st = row0 / kSuperRows;
  const int ntl0 = (row0 % kSuperRows) / kTileRows;

  const uint32_t* wbase = qweight + static_cast<size_t>(st) * KT * kSuperChunkWords +
                          static_cast<size_t>(ntl0) * kChunkWords + lane * 4;
  const uint32_t* sbase = reinterpret_cast<const uint32_t*>(scales) +
                          (static_cast<size_t>(st) * G * 8 + ntl0) * 8 + r;   // u32 = (S_r, S_{r+8})
  const uint8_t* zbase = zeros + (static_cast<size_t>(st) * G * 8 + ntl0) * 8 + r;

  // activations: lane (g = r, t) of token tile j reads x'[8j + r][64kt + 16t .. +16]
  const __half* xrow[MT];
  bool xok[MT];
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    const int m = 8 * j + r;
    xok[j] = m < M;
    xrow[j] = x + static_cast<size_t>(xok[j] ? m : 0) * K + 16 * t;
  }

  uint4 wring[D][NT];                 // packed weights, D k-tiles ahead
  uint32_t sring[D / 2][NT], zring[D / 2][NT];   // per-group scale pair and zero byte
  uint4 xring[2][MT][2];              // activations, 2 k-tiles ahead (L1/L2 hits)

  auto issue_w = [&](int kl, uint4 (&w)[NT]) {
    const int kt = kt0 + kl;
#pragma unroll
    for (int i = 0; i < NT; ++i)
      w[i] = ldg_stream_v4(wbase + static_cast<size_t>(kt) * kSuperChunkWords + i * kChunkWords);
  };
  auto issue_meta = [&](int kl, uint32_t (&sv)[NT], uint32_t (&zv)[NT]) {
    const int g = (kt0 + kl) >> 1;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      sv[i] = __ldg(sbase + static_cast<size_t>(g) * 64 + i * 8);
      zv[i] = __ldg(zbase + static_cast<size_t>(g) * 64 + i * 8);
    }
  };
  auto issue_x = [&](int kl, uint4 (&xv)[MT][2]) {
    const int kt = kt0 + kl;
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      if (xok[j]) {
        const uint4* p = reinterpret_cast<const uint4*>(xrow[j] + static_cast<size_t>(kt) * kKTile);
        xv[j][0] = __ldg(p);
        xv[j][1] = __ldg(p + 1);
      } else {
        xv[j][0] = make_uint4(0, 0, 0, 0);
        xv[j][1] = make_uint4(0, 0, 0, 0);
      }
    }
  };

  float acc[NT][MT][4], tmp[NT][MT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i)
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][j][c] = tmp[i][j][c] = 0.f;

  // prologue: fill the rings (nkt is even and >= 2)
#pragma unroll
  for (int u = 0; u < D; ++u) {
    if (u < nkt) {
      issue_w(u, wring[u]);
      if ((u & 1) == 0) issue_meta(u, sring[u / 2], zring[u / 2]);
    }
  }
  issue_x(0, xring[0]);
  issue_x(1, xring[1]);

  for (int base = 0; base < nkt; base += D) {
#pragma unroll
    for (int u = 0; u < D; ++u) {
      const int kl = base + u;
      if (kl < nkt) {
        // zero-point constants for this group: (1024 + z_r) and (1024 + 16 z_{r+8}) as half2
        uint32_t za[NT], zb[NT];
#pragma unroll
        for (int i = 0; i < NT; ++i) {
          const uint32_t zz = zring[u / 2][i];
          za[i] = 0x64006400u | ((zz & 0xFu) * 0x00010001u);
          zb[i] = 0x64006400u | (((zz >> 4) & 0xFu) * 0x00100010u);
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
#pragma unroll
          for (int i = 0; i < NT; ++i) {
            const uint32_t q = (s == 0) ? wring[u][i].x : (s == 1) ? wring[u][i].y : (s == 2) ? wring[u][i].z : wring[u][i].w;
            const uint32_t q8 = q >> 8;
            uint32_t a[4];
            a[0] = hsub2_u32(lop_or(q, 0x000F000Fu, 0x64006400u), za[i]);    // row r,   slots e0 e1
            a[1] = hsub2_u32(lop_or(q, 0x00F000F0u, 0x64006400u), zb[i]);    // row r+8, slots e0 e1 (x16)
            a[2] = hsub2_u32(lop_or(q8, 0x000F000Fu, 0x64006400u), za[i]);   // row r,   slots e2 e3
            a[3] = hsub2_u32(lop_or(q8, 0x00F000F0u, 0x64006400u), zb[i]);   // row r+8, slots e2 e3 (x16)
#pragma unroll
            for (int j = 0; j < MT; ++j) {
              const uint4& xv = xring[u & 1][j][s >> 1];
              const uint32_t b0 = (s & 1) ? xv.z : xv.x;
              const uint32_t b1 = (s & 1) ? xv.w : xv.y;
              mma_m16n8k16_f32(tmp[i][j], a, b0, b1);
            }
          }
        }
        if (u & 1) {
          // end of a group: acc += S * partial (row r+8 carries the x16 of the odd nibbles)
#pragma unroll
          for (int i = 0; i < NT; ++i) {
            const uint32_t sv = sring[u / 2][i];
            const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sv));
            const float s_lo = sf.x, s_hi = sf.y * 0.0625f;
#pragma unroll
            for (int j = 0; j < MT; ++j) {
              acc[i][j][0] = fmaf(s_lo, tmp[i][j][0], acc[i][j][0]);
              acc[i][j][1] = fmaf(s_lo, tmp[i][j][1], acc[i][j][1]);
              acc[i][j][2] = fmaf(s_hi, tmp[i][j][2], acc[i][j][2]);
              acc[i][j][3] = fmaf(s_hi, tmp[i][j][3], acc[i][j][3]);
              tmp[i][j][0] = tmp[i][j][1] = tmp[i][j][2] = tmp[i][j][3] = 0.f;
            }
          }
        }
        // refill: activations 2 k-tiles ahead, weights D k-tiles ahead; a group's scale and
        // zero slot is refilled only after the group's second k-tile has used it
        if (kl + 2 < nkt) issue_x(kl + 2, xring[u & 1]);
        if (kl + D < nkt) issue_w(kl + D, wring[u]);
        if ((u & 1) && kl + D - 1 < nkt) issue_meta(kl + D - 1, sring[u / 2], zring[u / 2]);
      }
    }
  }

  // ---- partial sums to shared memory: s_part[row][m]
  const int rl0 = warp * NT * kTileRows;
#pragma unroll
  for (int i = 0; i < NT; ++i) {
#pragma unroll
    for (int j = 0; j < MT; ++j) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int m = 8 * j + 2 * t + (c & 1);
        const int rl = rl0 + i * kTileRows + r + 8 * (c >> 1);
        if (m < M) s_part[rl * M + m] = acc[i][j][c];
      }
    }
  }
  cluster.sync();
  // ---- rank `rank` reduces rows [rank*R/CL, (rank+1)*R/CL) over the cluster, in rank order
  const int rb = (Cfg::kRows * rank) / CL, re = (Cfg::kRows * (rank + 1)) / CL;
  const int nelem = (re - rb) * M;
  const int nrow0 = blockIdx.x * Cfg::kRows;
  for (int e = threadIdx.x; e < nelem; e += Cfg::kThreads) {
    const int rl = rb + e / M, m = e % M;
    float v = 0.f;
    for (int q = 0; q < CL; ++q) v += cluster.map_shared_rank(s_part, q)[rl * M + m];
    const int n = nrow0 + rl;
    if (n < N) y[static_cast<size_t>(m) * N + n] = __float2half_rn(v);
  }
  cluster.sync();   // no CTA leaves while another still reads its shared memory
}

}  // namespace awq
