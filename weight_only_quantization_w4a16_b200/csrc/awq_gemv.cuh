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
//  * the weights of the first ring pass are requested before the kernel waits
//    on its stream predecessor (programmatic dependent launch): packed weights
//    are static inputs, so their stream overlaps the previous kernel's tail;
//  * packed layout v1 makes each consumer lane's 16-byte read exactly the
//    m16n8k16 A-fragments of 4 k-steps for rows r, r+8 of a 16-row tile, and
//    the matching activation slots a contiguous 32-byte run of x' per token;
//  * dequantization yields exact small integers, so every tensor-core product
//    is exact: for M >= 3 two instructions per code pair (LOP3 into the fp16
//    mantissa of 1024, HSUB2 of 1024 + z) give q - z; for M <= 2 one AND per
//    pair gives q as an fp16 subnormal and the zero point is applied per
//    group through the activation sums; S is applied in fp32 to each group's
//    sums;
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

// Independent accumulator chains per 16-row tile in gemv_group_math (shorter dependent-mma chains).
template <int MT>
constexpr int kGemvNacc =
#ifdef AWQ_GEMV_NACC
    MT == 1 ? AWQ_GEMV_NACC : 1;
#else
    MT == 2 ? 2 : 1;
#endif

// One quantization group (two 64-k tiles) of a consumer warp's fragments, in registers
// (loaded from the stage right before the group's math):
//   w[ii][n]     the lane's 16 bytes of codes of k-tile ii, 16-row tile n (packed layout v1:
//                exactly the m16n8k16 A fragments of 4 k-steps for rows r, r+8);
//   xv[ii][j][2] the lane's 32 bytes of x' of k-tile ii, token tile j (B fragments);
//   sv[n], zz[n] the scale pair (rows r, r+8) and the zero-point byte of tile n;
//   sx[2]        (kSumX) the group's activation sums of tokens 0 and 1.
template <int MT, int NT>
struct GemvGroupRegs {
  uint4 w[2][NT];
  uint4 xv[2][MT][2];
  uint32_t sv[NT];
  uint32_t zz[NT];
  uint2 sx[2];   // raw fp16 quads for the activation sums (kSumX)
};

// Loads a group's fragments from the stage in shared memory.
//   xg: the group's two activation boxes (8*MT tokens x 64 k fp16 each, 128-byte swizzle, 1024
//       bytes per 8 tokens), back to back;
//   wg: the group's two 4 KB super-chunks of packed codes, offset to the warp's first 16-row
//       tile and to this lane's 16 bytes (each further tile is 512 bytes further);
//   scg / zg: the warp's scales / zeros of the group, offset to this lane's fragment row r.
template <int MT, int NT, bool kSumX>
__device__ __forceinline__ void gemv_group_load(GemvGroupRegs<MT, NT>& g, const uint8_t* xg, const uint8_t* wg,
                                                const uint8_t* scg, const uint8_t* zg, int r, int t) {
  constexpr int kBox = 8 * MT * 128;
#pragma unroll
  for (int ii = 0; ii < 2; ++ii) {
#pragma unroll
    for (int n = 0; n < NT; ++n) g.w[ii][n] = *reinterpret_cast<const uint4*>(wg + ii * 4096 + n * 512);
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      const int m = 8 * j + r;
      const uint8_t* row = xg + ii * kBox + m * 128;
      g.xv[ii][j][0] = *reinterpret_cast<const uint4*>(row + (((2 * t) ^ (m & 7)) << 4));
      g.xv[ii][j][1] = *reinterpret_cast<const uint4*>(row + (((2 * t + 1) ^ (m & 7)) << 4));
    }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    g.sv[n] = *reinterpret_cast<const uint32_t*>(scg + n * 32);
    g.zz[n] = zg[n * 8];
  }
  if (kSumX) {
    // tokens 0 and 1 of the group: lane l reads 4 values of k-tile l >> 4 at k = 4 (l & 15);
    // box row 1 sits in 16-byte chunks swizzled by c ^ 1
    const int lane = 4 * r + t;
    const uint8_t* box = xg + (lane >> 4) * kBox;
    const int c16 = (lane & 15) >> 1, off = (lane & 1) << 3;
    g.sx[0] = *reinterpret_cast<const uint2*>(box + (c16 << 4) + off);
    g.sx[1] = *reinterpret_cast<const uint2*>(box + 128 + ((c16 ^ 1) << 4) + off);
  }
}

// Adds one group to acc. Two exact dequantizations:
//  * kSumX == false (any M): a code pair is masked out of its word and OR-ed into the mantissa
//    of fp16 1024 (0x6400), giving 1024 + q (even nibbles) or 1024 + 16q (odd nibbles, 4 bits
//    higher); subtracting 1024 + z, resp. 1024 + 16z, leaves q - z or 16 (q - z), small
//    integers exact in fp16. The group's fp32 sums are scaled by S and S/16.
//  * kSumX == true (M <= 2): one AND per pair gives the codes as exact fp16 subnormals q 2^-24
//    (16q 2^-24 for the odd nibbles), and the zero point enters once per group as
//    -S z sum_k x'_mk, with the activation sums of tokens 0 and 1 added up by the warp
//    (4 values per lane and a butterfly). The group's fp32 sums are scaled by S 2^24, S 2^20.
// Either way every tensor-core product is exact.
template <int MT, int NACC, int NT, bool kSumX>
__device__ __forceinline__ void gemv_group_math(float (&acc)[NT][MT][4], const GemvGroupRegs<MT, NT>& g, int t) {
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
      zlo[n] = 0x64006400u + (g.zz[n] & 0xFu) * 0x00010001u;
      zhi[n] = 0x64006400u + (g.zz[n] >> 4) * 0x00100010u;
    }
  }
#pragma unroll
  for (int ii = 0; ii < 2; ++ii) {
#pragma unroll
    for (int s4 = 0; s4 < 4; ++s4) {
      const int ac = (ii * 4 + s4) % NACC;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const uint4& wv = g.w[ii][n];
        const uint32_t q = (s4 == 0) ? wv.x : (s4 == 1) ? wv.y : (s4 == 2) ? wv.z : wv.w;
        const uint32_t q8 = q >> 8;
        uint32_t a[4];
        if (kSumX) {
          a[0] = q & 0x000F000Fu;     // row r,   slots e0 e1:  q * 2^-24
          a[1] = q & 0x00F000F0u;     // row r+8, slots e0 e1: 16q * 2^-24
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
          const uint4& xq = g.xv[ii][j][s4 >> 1];
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
    const float2 a0 = __half22float2(*reinterpret_cast<const __half2*>(&g.sx[0].x));
    const float2 a1 = __half22float2(*reinterpret_cast<const __half2*>(&g.sx[0].y));
    const float2 b0 = __half22float2(*reinterpret_cast<const __half2*>(&g.sx[1].x));
    const float2 b1 = __half22float2(*reinterpret_cast<const __half2*>(&g.sx[1].y));
    float sx0 = (a0.x + a0.y) + (a1.x + a1.y), sx1 = (b0.x + b0.y) + (b1.x + b1.y);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sx0 += __shfl_xor_sync(0xFFFFFFFFu, sx0, o);
      sx1 += __shfl_xor_sync(0xFFFFFFFFu, sx1, o);
    }
    // acc element c holds token 2t + (c & 1); tokens >= 2 only exist for M > 2 (unused here)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&g.sv[n]));
      const float c_lo = sf.x * 16777216.0f, c_hi = sf.y * 1048576.0f;
      const float d_lo = -sf.x * static_cast<float>(g.zz[n] & 0xFu);
      const float d_hi = -sf.y * static_cast<float>(g.zz[n] >> 4);
      acc[n][0][0] = fmaf(d_lo, sx0, fmaf(c_lo, tq[0][n][0][0], acc[n][0][0]));
      acc[n][0][1] = fmaf(d_lo, sx1, fmaf(c_lo, tq[0][n][0][1], acc[n][0][1]));
      acc[n][0][2] = fmaf(d_hi, sx0, fmaf(c_hi, tq[0][n][0][2], acc[n][0][2]));
      acc[n][0][3] = fmaf(d_hi, sx1, fmaf(c_hi, tq[0][n][0][3], acc[n][0][3]));
    }
  } else {
    // acc += S (sum x (q - z)); rows r+8 carry 16 (q - z)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&g.sv[n]));
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

// MT: 8-token tiles (M <= 8*MT); S: pipeline stages; KS: 64-k tiles per stage (even);
// CW: consumer warps (2, 4 or 8). A CTA is one producer warp plus CW consumer warps; consumer
// warp w owns rows (128/CW) w .. (128/CW)(w+1) - 1 of a 128-row super-tile (8/CW mma tiles).
template <int MT, int S, int KS, int CW>
struct GemvCfg {
  static_assert(KS % 2 == 0, "a stage must hold whole groups");
  static_assert(CW == 2 || CW == 4 || CW == 8, "2, 4 or 8 consumer warps");
  static constexpr int kNT = 8 / CW;                         // 16-row tiles per consumer warp
  static constexpr int kMP = 8 * MT;                         // token rows of the activation boxes
  static constexpr int kX = KS * kMP * 128;                  // activations: KS boxes of 64 k x kMP rows
  static constexpr int kW = KS * kSuperChunkWords * 4;       // packed codes: KS x 4 KB
  static constexpr int kSc = (KS / 2) * 256;                 // scales of KS/2 groups
  static constexpr int kZ = (KS / 2) * 64;                   // zeros of KS/2 groups
  static constexpr int kStage = (kX + kW + kSc + kZ + 1023) / 1024 * 1024;
  static constexpr int kThreads = (1 + CW) * 32;
  // + partial sums (units x 128 rows x M floats) + barriers + abort flag + alignment slack
  static size_t smem_bytes(int M, int units) {
    return static_cast<size_t>(S) * kStage + static_cast<size_t>(units) * kSuperRows * M * 4 + 2 * S * 8 + 16 + 1024;
  }
};

template <int MT, int S, int KS, int CW, bool kSumX>
__global__ void __launch_bounds__(GemvCfg<MT, S, KS, CW>::kThreads, 1) gemv_kernel(
    const __grid_constant__ CUtensorMap tmap_x, const uint32_t* __restrict__ qweight,
    const __half* __restrict__ scales, const uint8_t* __restrict__ zeros, __half* __restrict__ y, int M, int N,
    int K, int max_units) {
  using C = GemvCfg<MT, S, KS, CW>;
  constexpr int NT = C::kNT;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = K / kGroup, KT = K / kKTile;
  const int NST = padded_rows(N) / kSuperRows;
  const int g0 = static_cast<int>((static_cast<long long>(G) * rank) / CL);
  const int g1 = static_cast<int>((static_cast<long long>(G) * (rank + 1)) / CL);
  const int kt0 = 2 * g0;
  const int nkt = 2 * (g1 - g0);

  float* part = reinterpret_cast<float*>(smem + S * C::kStage);              // [max_units][128][M]
  uint64_t* full = reinterpret_cast<uint64_t*>(part + static_cast<size_t>(max_units) * kSuperRows * M);
  uint64_t* empty = full + S;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + S);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    *s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  const unsigned long long budget = g_wait_budget_ns;
  bool ok = true;
  int stage = 0;
  uint32_t phase = 0;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer warp
    // Stage i of this CTA: super-tile blockIdx.x + (i / spu) * gridDim.x, k-tiles [kb, kb + nk).
    const int spu = (nkt + KS - 1) / KS;
    const int nunits = (NST - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                       static_cast<int>(gridDim.x);
    const int total = nunits * spu;
    auto issue_weights = [&](int slot, int i) {
      const int st = blockIdx.x + (i / spu) * gridDim.x, kb = (i % spu) * KS, nk = min(KS, nkt - kb);
      uint8_t* sb = smem + slot * C::kStage;
      mbar_arrive_expect_tx(&full[slot], nk * (kSuperChunkWords * 4 + 160 + C::kMP * 128));
      bulk_g2s(sb + C::kX, qweight + (static_cast<size_t>(st) * KT + kt0 + kb) * kSuperChunkWords,
               nk * kSuperChunkWords * 4, &full[slot]);
      bulk_g2s(sb + C::kX + C::kW, scales + (static_cast<size_t>(st) * G + g0 + kb / 2) * 128, nk * 128, &full[slot]);
      bulk_g2s(sb + C::kX + C::kW + C::kSc, zeros + (static_cast<size_t>(st) * G + g0 + kb / 2) * 64, nk * 32,
               &full[slot]);
    };
    auto issue_x = [&](int slot, int i) {
      const int kb = (i % spu) * KS, nk = min(KS, nkt - kb);
      uint8_t* sb = smem + slot * C::kStage;
      for (int k = 0; k < nk; ++k) tma_load_2d(sb + k * C::kMP * 128, &tmap_x, (kt0 + kb + k) * kKTile, 0, &full[slot]);
    };
    // first ring pass: packed weights only, before waiting on the previous kernel
    const bool drop0 = g_debug_drop_first_copy != 0;
    const int npre = min(S, total);
    uint32_t issued_mask = 0, last_par = 0;
    if (lane == 0) {
      tma_prefetch_desc(&tmap_x);
      for (int i = 0; i < npre; ++i)
        if (!(drop0 && i == 0)) issue_weights(i, i);
    }
    for (int i = 0; i < npre; ++i)
      if (!(drop0 && i == 0)) issued_mask |= 1u << i;
    __syncwarp();
    pdl_enter();
    if (lane == 0)
      for (int i = 0; i < npre; ++i)
        if (!(drop0 && i == 0)) issue_x(i, i);
    __syncwarp();
    stage = npre % S;
    phase = npre == S ? 1u : 0u;
    for (int i = npre; i < total; ++i) {
      ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[stage], phase ^ 1, s_abort, budget));
      if (!ok) break;
      if (lane == 0) {
        issue_weights(stage, i);
        issue_x(stage, i);
      }
      __syncwarp();
      issued_mask |= 1u << stage;
      last_par = (last_par & ~(1u << stage)) | (phase << stage);
      if (++stage == S) { stage = 0; phase ^= 1; }
    }
    // drain every copy this warp issued before the CTA can exit
    int never = 0;
    for (int s = 0; s < S; ++s)
      if (issued_mask & (1u << s)) mbar_wait_bounded(&full[s], (last_par >> s) & 1u, &never, kDrainBudgetNs);
  } else {
    // ---------------------------------------------------------------- consumer warps
    pdl_enter();
    const int cw = warp - 1;
    const int r = lane >> 2, t = lane & 3;     // mma fragment row / column block
    int ui = 0;
    for (int st = blockIdx.x; st < NST; st += gridDim.x, ++ui) {
      float acc[NT][MT][4];
#pragma unroll
      for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[i][j][c] = 0.f;

      for (int kb = 0; kb < nkt && ok; kb += KS) {
        const int nk = min(KS, nkt - kb);
        ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[stage], phase, s_abort, budget));
        if (!ok) break;
        const uint8_t* sb = smem + stage * C::kStage;
        const uint8_t* sw = sb + C::kX + (NT * cw) * 512 + lane * 16;
        const uint8_t* ssc = sb + C::kX + C::kW + (NT * cw) * 32 + r * 4;
        const uint8_t* szr = sb + C::kX + C::kW + C::kSc + (NT * cw) * 8 + r;
#pragma unroll
        for (int i = 0; i < KS; i += 2)
          if (i < nk) {
            GemvGroupRegs<MT, NT> gr;
            gemv_group_load<MT, NT, kSumX>(gr, sb + i * C::kMP * 128, sw + i * 4096, ssc + (i / 2) * 256,
                                           szr + (i / 2) * 64, r, t);
            gemv_group_math<MT, kGemvNacc<MT>, NT, kSumX>(acc, gr, t);
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      // ---- partial sums of this unit: part[ui][row][m] (reduced over the cluster at the end)
      float* pu = part + static_cast<size_t>(ui) * kSuperRows * M;
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int m = 8 * j + 2 * t + (c & 1);
            const int rl = 16 * (NT * cw + n) + r + 8 * (c >> 1);
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
      for (int e = threadIdx.x - 32; e < per_unit; e += CW * 32) {
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
