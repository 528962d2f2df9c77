// awq_gemv.cuh — a3: decode W4A16 linear layer, 1 <= M <= 32.
//
// llm-awq README, "Installation" step 3: W4A16 (4-bit weight, 16-bit
// activation) kernels for the decode stage. y[M,N] = x'[M,K] . ((q-z)*S)^T,
// fp32 accumulation, fp16 output.
//
// The layer is HBM-bound (0.52 bytes of packed weight per weight, about
// 3.85*M flop per byte). Design for B200:
//  * a producer warp streams each stage with TMA: one 1-D bulk copy of KS
//    contiguous 4 KB (super-tile, 64-k) blocks of packed codes, the stage's
//    scales and zeros, and KS 2-D boxes of x' (64 k x 8*MT tokens, 128-byte
//    swizzle, zero fill past M) into an S-deep shared-memory ring, so HBM
//    reads stay in flight while the consumer warps compute;
//  * packed layout v1 makes each consumer lane's 16-byte read exactly the
//    m16n8k16 A-fragments of 4 k-steps for rows r, r+8 of a 16-row tile, and
//    the matching activation slots a contiguous 32-byte run of x' per token;
//  * codes enter the tensor core as exact fp16 subnormals: one AND per pair
//    gives q * 2^-24 (odd nibbles 16q * 2^-24, compensated in fp32), with no
//    subtraction; the zero point is applied per group as -S z sum_k x'_mk,
//    where the sums come from one extra mma per k-step against an all-ones
//    A fragment (shared by the warp's two 16-row tiles, and already in the
//    accumulator layout); S is applied in fp32 to the group's partial sums,
//    so every tensor-core product is exact;
//  * persistent clusters: cluster c walks super-tiles c, c + C, ...; its CL
//    CTAs split K and keep every super-tile's partial sums in shared memory,
//    so the stream never stops for a barrier; one cluster barrier at the end
//    precedes the reduction through distributed shared memory, in rank order
//    (deterministic, no global scratch, no atomics).
#pragma once

#include <cooperative_groups.h>

#include "awq_common.cuh"

namespace awq {

// ------------------------------------------------------------------------------------
// Cluster barrier (all 32 lanes of a warp execute it together).
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// MT: 8-token tiles (M <= 8*MT); S: pipeline stages; KS: 64-k tiles per stage (even).
// A CTA is one producer warp plus four consumer warps; consumer warp w owns rows
// 32w .. 32w+31 of a 128-row super-tile (two 16-row mma tiles).
template <int MT, int S, int KS>
struct GemvCfg {
  static_assert(KS % 2 == 0, "a stage must hold whole groups");
  static constexpr int kMP = 8 * MT;                         // token rows of the activation boxes
  static constexpr int kX = KS * kMP * 128;                  // activations: KS boxes of 64 k x kMP rows
  static constexpr int kW = KS * kSuperChunkWords * 4;       // packed codes: KS x 4 KB
  static constexpr int kSc = (KS / 2) * 256;                 // scales of KS/2 groups
  static constexpr int kZ = (KS / 2) * 64;                   // zeros of KS/2 groups
  static constexpr int kStage = (kX + kW + kSc + kZ + 1023) / 1024 * 1024;
  static constexpr int kThreads = 5 * 32;
  // + partial sums (units x 128 rows x M floats) + barriers + alignment slack
  static size_t smem_bytes(int M, int units) {
    return static_cast<size_t>(S) * kStage + static_cast<size_t>(units) * kSuperRows * M * 4 + 2 * S * 8 + 1024;
  }
};

template <int MT, int S, int KS>
__global__ void __launch_bounds__(GemvCfg<MT, S, KS>::kThreads, 1) gemv_kernel(
    const __grid_constant__ CUtensorMap tmap_x, const uint32_t* __restrict__ qweight,
    const __half* __restrict__ scales, const uint8_t* __restrict__ zeros, __half* __restrict__ y, int M, int N,
    int K, int max_units) {
  using C = GemvCfg<MT, S, KS>;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* part = reinterpret_cast<float*>(smem + S * C::kStage);              // [max_units][128][M]
  uint64_t* full = reinterpret_cast<uint64_t*>(part + static_cast<size_t>(max_units) * kSuperRows * M);
  uint64_t* empty = full + S;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + S);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = K / kGroup, KT = K / kKTile;
  const int NST = padded_rows(N) / kSuperRows;
  const int g0 = static_cast<int>((static_cast<long long>(G) * rank) / CL);
  const int g1 = static_cast<int>((static_cast<long long>(G) * (rank + 1)) / CL);
  const int kt0 = 2 * g0;
  const int nkt = 2 * (g1 - g0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    *s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  pdl_enter();
  const unsigned long long budget = g_wait_budget_ns;
  bool ok = true;
  int stage = 0;
  uint32_t phase = 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer warp
    if (lane == 0) tma_prefetch_desc(&tmap_x);
    uint32_t issued_mask = 0, last_par = 0;
    for (int st = blockIdx.x; st < NST; st += gridDim.x) {
      for (int kb = 0; kb < nkt && ok; kb += KS) {
        const int nk = min(KS, nkt - kb);
        ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[stage], phase ^ 1, s_abort, budget));
        if (!ok) break;
        if (lane == 0) {
          uint8_t* sb = smem + stage * C::kStage;
          mbar_arrive_expect_tx(&full[stage], nk * (kSuperChunkWords * 4 + 160 + C::kMP * 128));
          bulk_g2s(sb + C::kX, qweight + (static_cast<size_t>(st) * KT + kt0 + kb) * kSuperChunkWords,
                   nk * kSuperChunkWords * 4, &full[stage]);
          bulk_g2s(sb + C::kX + C::kW, scales + (static_cast<size_t>(st) * G + g0 + kb / 2) * 128, nk * 128,
                   &full[stage]);
          bulk_g2s(sb + C::kX + C::kW + C::kSc, zeros + (static_cast<size_t>(st) * G + g0 + kb / 2) * 64, nk * 32,
                   &full[stage]);
          for (int i = 0; i < nk; ++i)
            tma_load_2d(sb + i * C::kMP * 128, &tmap_x, (kt0 + kb + i) * kKTile, 0, &full[stage]);
        }
        __syncwarp();
        issued_mask |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
    // drain every copy this warp issued before the CTA can exit
    int never = 0;
    for (int s = 0; s < S; ++s)
      if (issued_mask & (1u << s)) mbar_wait_bounded(&full[s], (last_par >> s) & 1u, &never, kDrainBudgetNs);
  } else {
    // ---------------------------------------------------------------- consumer warps
    const int cw = warp - 1;
    const int r = lane >> 2, t = lane & 3;     // mma fragment row / column block
    int ui = 0;
    for (int st = blockIdx.x; st < NST; st += gridDim.x, ++ui) {
      float acc[2][MT][4];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[i][j][c] = 0.f;

      for (int kb = 0; kb < nkt && ok; kb += KS) {
        const int nk = min(KS, nkt - kb);
        ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[stage], phase, s_abort, budget));
        if (!ok) break;
        const uint8_t* sb = smem + stage * C::kStage;
        const uint8_t* sw = sb + C::kX + (2 * cw) * 512 + lane * 16;
        const uint8_t* ssc = sb + C::kX + C::kW + (2 * cw) * 32 + r * 4;
        const uint8_t* szr = sb + C::kX + C::kW + C::kSc + (2 * cw) * 8 + r;
#pragma unroll
        for (int i = 0; i < KS; i += 2) {
          if (i < nk) {
            // group of k-tiles i, i+1. Codes enter the mma as exact fp16 subnormals q * 2^-24 (odd
            // nibbles 16q * 2^-24); an extra mma against an all-ones A fragment gives sum_k x'_mk
            // for the zero-point term: sum x (q - z) S = S (sum x q) - S z (sum x).
            // NACC independent accumulator chains per tile shorten the dependent-mma chains
#ifdef AWQ_GEMV_NACC
            constexpr int NACC = MT == 1 ? AWQ_GEMV_NACC : 1;
#else
            constexpr int NACC = MT == 1 ? 4 : (MT == 2 ? 2 : 1);
#endif
            float tq[NACC][2][MT][4], tx[NACC][MT][4];
#pragma unroll
            for (int a = 0; a < NACC; ++a)
#pragma unroll
              for (int j = 0; j < MT; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  tq[a][0][j][c] = tq[a][1][j][c] = 0.f;
                  tx[a][j][c] = 0.f;
                }
#pragma unroll
            for (int ii = 0; ii < 2; ++ii) {
              const int kl = i + ii;
              uint4 w[2];
#pragma unroll
              for (int n = 0; n < 2; ++n) w[n] = *reinterpret_cast<const uint4*>(sw + kl * 4096 + n * 512);
              uint4 xv[MT][2];
#pragma unroll
              for (int j = 0; j < MT; ++j) {
                const int m = 8 * j + r;
                const uint8_t* row = sb + kl * C::kMP * 128 + m * 128;
                xv[j][0] = *reinterpret_cast<const uint4*>(row + (((2 * t) ^ (m & 7)) << 4));
                xv[j][1] = *reinterpret_cast<const uint4*>(row + (((2 * t + 1) ^ (m & 7)) << 4));
              }
#pragma unroll
              for (int s4 = 0; s4 < 4; ++s4) {
                const int ac = (ii * 4 + s4) % NACC;
#pragma unroll
                for (int n = 0; n < 2; ++n) {
                  const uint32_t q = (s4 == 0) ? w[n].x : (s4 == 1) ? w[n].y : (s4 == 2) ? w[n].z : w[n].w;
                  const uint32_t q8 = q >> 8;
                  uint32_t a[4];
                  a[0] = q & 0x000F000Fu;     // row r,   slots e0 e1:  q * 2^-24
                  a[1] = q & 0x00F000F0u;     // row r+8, slots e0 e1: 16q * 2^-24
                  a[2] = q8 & 0x000F000Fu;    // row r,   slots e2 e3
                  a[3] = q8 & 0x00F000F0u;    // row r+8, slots e2 e3
#pragma unroll
                  for (int j = 0; j < MT; ++j) {
                    const uint4& xq = xv[j][s4 >> 1];
                    mma_m16n8k16_f32(tq[ac][n][j], a, (s4 & 1) ? xq.z : xq.x, (s4 & 1) ? xq.w : xq.y);
                  }
                }
                const uint32_t ones[4] = {0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u};
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                  const uint4& xq = xv[j][s4 >> 1];
                  mma_m16n8k16_f32(tx[ac][j], ones, (s4 & 1) ? xq.z : xq.x, (s4 & 1) ? xq.w : xq.y);
                }
              }
            }
#pragma unroll
            for (int a = 1; a < NACC; ++a)
#pragma unroll
              for (int j = 0; j < MT; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  tq[0][0][j][c] += tq[a][0][j][c];
                  tq[0][1][j][c] += tq[a][1][j][c];
                  tx[0][j][c] += tx[a][j][c];
                }
            // end of the group: acc += S 2^24 (sum x q) - S z (sum x); rows r+8 use S 2^20 for the x16
#pragma unroll
            for (int n = 0; n < 2; ++n) {
              const uint32_t sv = *reinterpret_cast<const uint32_t*>(ssc + (i / 2) * 256 + n * 32);
              const uint32_t zz = szr[(i / 2) * 64 + n * 8];
              const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sv));
              const float c_lo = sf.x * 16777216.0f, c_hi = sf.y * 1048576.0f;
              const float d_lo = -sf.x * static_cast<float>(zz & 0xFu);
              const float d_hi = -sf.y * static_cast<float>(zz >> 4);
#pragma unroll
              for (int j = 0; j < MT; ++j) {
                acc[n][j][0] = fmaf(d_lo, tx[0][j][0], fmaf(c_lo, tq[0][n][j][0], acc[n][j][0]));
                acc[n][j][1] = fmaf(d_lo, tx[0][j][1], fmaf(c_lo, tq[0][n][j][1], acc[n][j][1]));
                acc[n][j][2] = fmaf(d_hi, tx[0][j][2], fmaf(c_hi, tq[0][n][j][2], acc[n][j][2]));
                acc[n][j][3] = fmaf(d_hi, tx[0][j][3], fmaf(c_hi, tq[0][n][j][3], acc[n][j][3]));
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      // ---- partial sums of this unit: part[ui][row][m] (reduced over the cluster at the end)
      float* pu = part + static_cast<size_t>(ui) * kSuperRows * M;
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int m = 8 * j + 2 * t + (c & 1);
            const int rl = 32 * cw + 16 * n + r + 8 * (c >> 1);
            if (m < M) pu[rl * M + m] = acc[n][j][c];
          }
    }
  }
  // ---- one cluster reduction for all units: rank `rank` owns rows [rank*128/CL, (rank+1)*128/CL)
  // of every super-tile and adds the CL partial sums in rank order (deterministic)
  cluster_arrive();
  cluster_wait();
  if (warp != 0) {
    const int rb = (kSuperRows * rank) / CL, re = (kSuperRows * (rank + 1)) / CL;
    const int per_unit = (re - rb) * M;
    int ui = 0;
    for (int st = blockIdx.x; st < NST; st += gridDim.x, ++ui) {
      const float* pu = part + static_cast<size_t>(ui) * kSuperRows * M;
      for (int e = threadIdx.x - 32; e < per_unit; e += 128) {
        const int rl = rb + e / M, m = e % M;
        float v = 0.f;
        for (int q = 0; q < CL; ++q) v += cluster.map_shared_rank(pu, q)[rl * M + m];
        const int nn = st * kSuperRows + rl;
        if (nn < N) y[static_cast<size_t>(m) * N + nn] = __float2half_rn(v);
      }
    }
  }
  // no CTA leaves while another may still read its shared memory
  cluster_arrive();
  cluster_wait();
}

}  // namespace awq
