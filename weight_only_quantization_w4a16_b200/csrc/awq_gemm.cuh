// awq_gemm.cuh — a4: prefill W4A16 linear layer on tcgen05 tensor cores.
//
// llm-awq README, "Installation" step 3 (W4A16 kernels for the context
// stage) and HF "transformers - AWQ" section 2 ("version": "gemm").
// y[M,N] = x'[M,K] . ((q-z)*S)^T with fp16 operands and fp32 accumulation.
//
// The contraction runs "swapped": the dequantized weight tile is the MMA's
// 128-row A operand (one 128-row super-tile of the packed layout), and a
// tile of BT tokens of x' is the B operand, so every dequantized weight feeds
// BT tokens. Per CTA (persistent, one per SM):
//   warp NDQ+4 (one lane): producer — 3-D TMA boxes of the packed codes
//       (8 tiles x one 64-k tile = 4 KB), scales (8 x 32 B) and zeros
//       (8 x 16 B) of a (super-tile, 64-k) block of packed layout v2, and a
//       2-D TMA load of the x' tile (BT x 64, 128-byte swizzle) into a
//       STAGES-deep shared-memory ring (mbarrier transaction counts; tiles
//       past the last one read as zeros);
//   warps 0..NDQ-1: dequantize codes to fp16 (q - z) * S straight into the
//       A tile in the canonical K-major 128-byte-swizzle layout (bank-conflict
//       free 8-byte stores), then fence.proxy.async and arrive;
//   warp NDQ+5 (one lane): issues tcgen05.mma kind::f16 128 x BT x 16 into a
//       TMEM accumulator, commits each stage back to the producer;
//   warps NDQ..NDQ+3: epilogue — tcgen05.ld of the accumulator (each warp its
//       32-lane quarter), fp16 convert, coalesced stores of y; two TMEM
//       accumulators let the epilogue of one tile overlap the next mainloop.
// K split (KS = 2, clusters of two CTAs): when the tiles are too few to fill
// the SMs, or a few are left over for a last round, the CTA pair of a cluster
// shares a tile, rank r running 64-k steps [r KB/2, (r+1) KB/2). Rank 1's
// epilogue sends its fp32 sums, 32 columns at a time, into rank 0's shared
// memory with st.async stores that count down an mbarrier of rank 0; rank 0
// adds them to its own (a fixed order) and stores the tile. A launch may
// first run whole-tile rounds (one tile per CTA, all of K) and split only the
// tiles left for the last round: every role walks the same work-item sequence.
// Every mbarrier wait is bounded by %globaltimer; on expiry the CTA records
// AWQ_ERR_TIMEOUT in the device status word, every role stops, the producer
// waits for its copies in flight, the MMA thread for its MMAs, and TMEM is
// freed before the CTA returns.
#pragma once

#include "awq_common.cuh"

namespace awq {

// Epilogue of the linear kernels ("transformers - AWQ" section 3, fused modules):
//   kEpiPlain  y[M, N]
//   kEpiSplit3 the fused q/k/v output split into y0 [M, n0], y1 [M, n1], y2 [M, N - n0 - n1]
//   kEpiSiluMul the fused gate+up layer (weight rows: I gate rows, then I up rows, I % 16 == 0):
//              h[M, I] = SiLU(gate) * up, written to y0; the prefill kernel loads each 128-row
//              block as 4 gate tiles and the 4 matching up tiles, interleaved by 16 rows, so a
//              gate row and its up row sit 16 accumulator lanes apart in one warp
constexpr int kEpiPlain = 0;
constexpr int kEpiSplit3 = 1;
constexpr int kEpiSiluMul = 2;
struct EpiArgs {
  __half* y0;
  __half* y1;
  __half* y2;
  int n0, n1;   // kEpiSplit3: widths of y0 and y1 (y2 takes the rest of N)
};

// Stores one fp32 output of row n (of N), token m, per the epilogue (kEpiPlain / kEpiSplit3).
template <int EPI>
__device__ __forceinline__ void epi_store(const EpiArgs& e, int m, long long n, int N, float v) {
  if (EPI == kEpiSplit3) {
    if (n < e.n0) {
      e.y0[static_cast<size_t>(m) * e.n0 + n] = __float2half_rn(v);
    } else if (n < e.n0 + e.n1) {
      e.y1[static_cast<size_t>(m) * e.n1 + (n - e.n0)] = __float2half_rn(v);
    } else {
      const int n2 = N - e.n0 - e.n1;
      e.y2[static_cast<size_t>(m) * n2 + (n - e.n0 - e.n1)] = __float2half_rn(v);
    }
  } else {
    e.y0[static_cast<size_t>(m) * N + n] = __float2half_rn(v);
  }
}

// SiLU(g) * u in fp32 (SiLU(g) = g / (1 + e^-g)).
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// CPS: resident CTAs per SM. With 2, each CTA keeps one TMEM accumulator (the other CTA's
// epilogue and mainloop interleave with its own); with 1, two accumulators let the epilogue of
// one tile overlap the mainloop of the next.
// KS: CTAs that share one output tile, each over its part of K (a cluster of KS = 2 CTAs; rank 1
// pushes its fp32 partial sums into rank 0's shared memory with asynchronous stores that count
// down rank 0's mbarrier, 32 columns at a time, through an exchange buffer of two or more slots).
template <int BT, int STAGES, int NDQ, int CPS = 1, int KS = 1, int EPI = kEpiPlain>
struct GemmCfg {
  static_assert(BT % 32 == 0 && BT >= 32 && BT <= 256, "token tile");
  static_assert(CPS == 1 || CPS == 2, "CTAs per SM");
  static_assert(NDQ == 4 || NDQ == 8, "dequant warps");
  static_assert(KS == 1 || (KS == 2 && CPS == 1), "K split across a CTA pair");
  static constexpr int kA = kSuperRows * kKTile * 2;        // 16 KB dequantized weights
  static constexpr int kB = BT * kKTile * 2;                // x' tile
  static constexpr int kRawQ = kSuperChunkWords * 4;        // 4096 B
  static constexpr int kRawS = 8 * 16 * 2;                  // 256 B
  static constexpr int kZeroBytes = 8 * 16;                 // 128 B: zeros of the group pair, 8 tiles
  // zeros slot: kEpiSiluMul loads the gate and the up tiles' zeros into two 128-byte-aligned halves
  static constexpr int kRawZ = EPI == kEpiSiluMul ? 256 : 128;
  static constexpr int kTx = kB + kRawQ + kRawS + kZeroBytes;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + STAGES * kA;
  static constexpr int kOffQ = kOffB + STAGES * kB;
  static constexpr int kOffS = kOffQ + STAGES * kRawQ;
  static constexpr int kOffZ = kOffS + STAGES * kRawS;
  static constexpr int kXChunk = kSuperRows * 32 * 4;          // 16 KB: 32 fp32 columns of 128 rows
  static constexpr int kOffX = (kOffZ + STAGES * kRawZ + 127) / 128 * 128;   // KS = 2: exchange slots
  // KS = 2: as many exchange slots (up to one per 32-column chunk of the tile) as shared memory
  // holds beside the ring
  static constexpr int kXFree = (232448 - 1024 - 512 - kOffX) / kXChunk;
  static constexpr int kXSlots = KS != 2 ? 0 : (BT / 32 < kXFree ? BT / 32 : kXFree);
  static_assert(KS != 2 || kXSlots >= 1, "exchange slots");
  static constexpr int kOffBar = kOffX + kXSlots * kXChunk;
  // barriers: full[S], aready[S], empty[S], accfull[2], accempty[2], drain[1]; KS = 2: xfull[X], xempty[X]
  static constexpr int kNumBars = 3 * STAGES + 5 + 2 * kXSlots;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16 + 1024;        // + slack for 1024-byte alignment
  // two accumulators of BT columns; tcgen05.alloc takes a power of two >= 32 columns
  static constexpr int kNAcc = CPS == 2 ? 1 : 2;   // TMEM accumulators of BT columns
  // tcgen05.alloc takes a power of two >= 32 columns; all CTAs of an SM share its 512
  static constexpr int kTmemCols = kNAcc * BT <= 32 ? 32 : kNAcc * BT <= 64 ? 64 : kNAcc * BT <= 128 ? 128
                                   : kNAcc * BT <= 256 ? 256 : 512;
  static_assert(kTmemCols * CPS <= 512, "tensor memory");
  static constexpr int kThreads = (NDQ + 6) * 32;
  static constexpr int kWarpEpi0 = NDQ;
  static constexpr int kWarpProd = NDQ + 4;
  static constexpr int kWarpMma = NDQ + 5;
  static_assert(kSmem <= 232448, "shared memory");
  static_assert(CPS == 1 || (kSmem + 1024) * 2 <= 233472, "two CTAs per SM must fit in shared memory");
};

// One work item of a CTA: a tile over 64-k steps [kb0, kb1), shared with the other CTA of the
// cluster when `split`.
struct GemmWork {
  int tile, kb0, kb1;
  bool split;
};

// solo (KS = 2 only): rounds in which every CTA of the grid takes a tile of its own over all of K
// before the remaining tiles are split across the CTA pairs (0: every tile is split).
template <int BT, int STAGES, int NDQ, int CPS, int EPI, int KS = 1>
__global__ void __launch_bounds__(GemmCfg<BT, STAGES, NDQ, CPS, KS, EPI>::kThreads, CPS)
    awq_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_s, const __grid_constant__ CUtensorMap tmap_z,
                    const EpiArgs epi, int M, int N, int K, int solo) {
  using C = GemmCfg<BT, STAGES, NDQ, CPS, KS, EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* aready = bars + STAGES;
  uint64_t* empty = bars + 2 * STAGES;
  uint64_t* accfull = bars + 3 * STAGES;
  uint64_t* accempty = accfull + 2;
  uint64_t* drain = accfull + 4;
  uint64_t* xfull = drain + 1;                 // KS = 2, rank 0: rank 1's partial sums are in slot b
  uint64_t* xempty = drain + 1 + C::kXSlots;   // KS = 2, rank 1: rank 0 has read slot b
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // kEpiSiluMul: N = 2I rows, P = I/16 tile pairs; super-tile st = gate tiles 4st..4st+3 and up
  // tiles P + 4st..P + 4st + 3
  const int P = N / 32;
  const int NST = EPI == kEpiSiluMul ? ceil_div(P, 4) : padded_rows(N) / kSuperRows;
  const int MTT = (M + BT - 1) / BT;
  const int ntiles = NST * MTT;
  const int KB = K / kKTile;
  // The CTA's work items in order; every role walks the same sequence. KS = 1: tiles blockIdx.x,
  // + gridDim.x, ... over all of K. KS = 2: first `solo` rounds of one tile per CTA over all of K,
  // then the remaining tiles striped over the clusters, the CTA pair of a cluster sharing each
  // (rank r: steps [r KB / 2, (r + 1) KB / 2)).
  const int G = static_cast<int>(gridDim.x);
  const int rank = KS == 2 ? static_cast<int>(blockIdx.x % KS) : 0;
  const int nsolo = KS == 2 ? solo : 0;
  auto work = [&](int i, GemmWork& w) -> bool {
    if (KS == 1 || i < nsolo) {
      w.tile = KS == 1 ? static_cast<int>(blockIdx.x) + i * G : i * G + static_cast<int>(blockIdx.x);
      w.kb0 = 0;
      w.kb1 = KB;
      w.split = false;
    } else {
      w.tile = nsolo * G + static_cast<int>(blockIdx.x) / KS + (i - nsolo) * (G / KS);
      w.kb0 = rank * KB / KS;
      w.kb1 = (rank + 1) * KB / KS;
      w.split = true;
    }
    return w.tile < ntiles;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&aready[s], NDQ);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(drain, 1);
    if (KS == 2)
      for (int b = 0; b < C::kXSlots; ++b) {
        mbar_init(&xfull[b], 1);    // rank 0's expect_tx arrival + 16 KB of rank 1's stores
        mbar_init(&xempty[b], 4);   // one arrival per epilogue warp of rank 0
      }
    *s_abort = 0;
    mbar_fence_init();
  }
  if (warp == C::kWarpProd && lane == 0) {
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_s);
    tma_prefetch_desc(&tmap_z);
  }
  if (warp == C::kWarpMma) {
    tmem_alloc(s_tmem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (KS == 2) {   // the partner's barriers are initialised before any arrival on them
    cluster_arrive();
    cluster_wait();
  }
  pdl_enter();
  const uint32_t tmem_base = *s_tmem;
  const unsigned long long budget = g_wait_budget_ns;

  if (warp == C::kWarpProd) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, last_par = 0;   // per stage: loaded at least once / parity of last load
      bool ok = true;
      GemmWork w;
      for (int i = 0; ok && work(i, w); ++i) {
        const int st = w.tile % NST, mt = w.tile / NST;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, s_abort, budget)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], C::kTx);
          if (EPI == kEpiSiluMul) {   // 4-tile boxes: gate tiles to slots 0..3, up tiles to slots 4..7
            tma_load_3d(smem + C::kOffQ + stage * C::kRawQ, &tmap_q, 0, kb, 4 * st, &full[stage]);
            tma_load_3d(smem + C::kOffQ + stage * C::kRawQ + C::kRawQ / 2, &tmap_q, 0, kb, P + 4 * st, &full[stage]);
            tma_load_3d(smem + C::kOffS + stage * C::kRawS, &tmap_s, 0, kb >> 1, 4 * st, &full[stage]);
            tma_load_3d(smem + C::kOffS + stage * C::kRawS + C::kRawS / 2, &tmap_s, 0, kb >> 1, P + 4 * st,
                        &full[stage]);
            tma_load_3d(smem + C::kOffZ + stage * C::kRawZ, &tmap_z, 0, kb >> 2, 4 * st, &full[stage]);
            tma_load_3d(smem + C::kOffZ + stage * C::kRawZ + 128, &tmap_z, 0, kb >> 2, P + 4 * st,
                        &full[stage]);
          } else {
            tma_load_3d(smem + C::kOffQ + stage * C::kRawQ, &tmap_q, 0, kb, 8 * st, &full[stage]);
            tma_load_3d(smem + C::kOffS + stage * C::kRawS, &tmap_s, 0, kb >> 1, 8 * st, &full[stage]);
            tma_load_3d(smem + C::kOffZ + stage * C::kRawZ, &tmap_z, 0, kb >> 2, 8 * st, &full[stage]);
          }
          tma_load_2d(smem + C::kOffB + stage * C::kB, &tmap_x, kb * kKTile, mt * BT, &full[stage]);
          issued_mask |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // drain: every copy this thread issued has landed before the CTA may exit
      int never = 0;
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s))
          mbar_wait_bounded(&full[s], (last_par >> s) & 1u, &never, kDrainBudgetNs);
    }
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(kSuperRows, BT);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, any = false;
      int it = 0;
      GemmWork w;
      for (; ok && work(it, w); ++it) {
        const int b = it % C::kNAcc;
        const uint32_t use = static_cast<uint32_t>(it / C::kNAcc);
        if (!mbar_wait_bounded(&accempty[b], (use & 1) ^ 1, s_abort, budget)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BT);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, s_abort, budget) ||
              !mbar_wait_bounded(&aready[stage], phase, s_abort, budget)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + C::kOffA + stage * C::kA);
          const uint32_t b0 = smem_u32(smem + C::kOffB + stage * C::kB);
#pragma unroll
          for (int kk = 0; kk < kKTile / 16; ++kk)
            tc_mma_f16(d_tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), idesc,
                       (kb != w.kb0 || kk != 0) ? 1u : 0u);
          any = true;
          tc_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(&accfull[b]);
      }
      if (any) {
        int never = 0;
        tc_commit(drain);
        mbar_wait_bounded(drain, 0, &never, kDrainBudgetNs);
      }
    }
  } else if (warp < NDQ) {
    // ------------------------------------------------------------ dequantize
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    GemmWork w;
    for (int i = 0; ok && work(i, w); ++i) {
      for (int kb = w.kb0; kb < w.kb1; ++kb) {
        // warp-uniform result: the code below needs the whole warp
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[stage], phase, s_abort, budget))) { ok = false; break; }
        const uint32_t* rq = reinterpret_cast<const uint32_t*>(smem + C::kOffQ + stage * C::kRawQ);
        const uint32_t* rs = reinterpret_cast<const uint32_t*>(smem + C::kOffS + stage * C::kRawS);
        const uint8_t* rz = smem + C::kOffZ + stage * C::kRawZ;
        uint8_t* A = smem + C::kOffA + stage * C::kA;
#pragma unroll
        for (int u = 0; u < 8 / NDQ; ++u) {
          const int c = warp * 32 + lane + u * 32 * NDQ;   // (16-row tile, lane) chunk
          const int nt = c >> 5, lw = c & 31, r = lw >> 2, t = lw & 3;
          // 16-row block nt of the A tile comes from shared-memory slot sl (kEpiSiluMul interleaves
          // gate and up tiles: blocks 2e and 2e+1 are gate tile e and up tile e)
          const int sl = EPI == kEpiSiluMul ? ((nt & 1) ? 4 + (nt >> 1) : (nt >> 1)) : nt;
          const uint4 words = *reinterpret_cast<const uint4*>(rq + sl * kChunkWords + lw * 4);
          const uint32_t sp = rs[sl * 8 + r];                        // (S_r, S_{r+8})
          const int zoff = (EPI == kEpiSiluMul && sl >= 4) ? 128 + (sl - 4) * 16 : sl * 16;
          const uint32_t zb = rz[zoff + ((kb >> 1) & 1) * 8 + r];
          const uint32_t s_r = __byte_perm(sp, 0, 0x1010);          // (S_r, S_r)
          const uint32_t s_r8 = __byte_perm(sp, 0, 0x3232);         // (S_{r+8}, S_{r+8})
          const uint32_t za = 0x64006400u | ((zb & 0xFu) * 0x00010001u);
          const uint32_t zc = 0x64006400u | ((zb >> 4) * 0x00010001u);
          uint8_t* rowA = A + (nt * 16 + r) * 128;
          uint8_t* rowB = rowA + 8 * 128;
#pragma unroll
          for (int ii = 0; ii < 4; ++ii) {
            const int s = ii ^ ((r >> 1) & 1);                      // rotation keeps 8-byte stores conflict free
            const uint32_t q = (s == 0) ? words.x : (s == 1) ? words.y : (s == 2) ? words.z : words.w;
            const uint32_t p0 = hmul2_u32(hsub2_u32(lop_or(q, 0x000F000Fu, 0x64006400u), za), s_r);
            const uint32_t p1 = hmul2_u32(hsub2_u32(lop_or(q >> 4, 0x000F000Fu, 0x64006400u), zc), s_r8);
            const uint32_t p2 = hmul2_u32(hsub2_u32(lop_or(q >> 8, 0x000F000Fu, 0x64006400u), za), s_r);
            const uint32_t p3 = hmul2_u32(hsub2_u32(lop_or(q >> 12, 0x000F000Fu, 0x64006400u), zc), s_r8);
            const int off = (((2 * t + (s >> 1)) ^ r) << 4) + (s & 1) * 8;
            *reinterpret_cast<uint2*>(rowA + off) = make_uint2(p0, p2);
            *reinterpret_cast<uint2*>(rowB + off) = make_uint2(p1, p3);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&aready[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - C::kWarpEpi0;   // == warp % 4: TMEM lane quarter of this warp
    bool ok = true;
    int it = 0;
    uint32_t xq = 0;   // KS = 2: exchange chunks so far (slot xq % X, phase parity (xq / X) & 1)
    GemmWork w;
    for (; ok && work(it, w); ++it) {
      const int st = w.tile % NST, mt = w.tile / NST;
      const int b = it % C::kNAcc;
      const uint32_t use = static_cast<uint32_t>(it / C::kNAcc);
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&accfull[b], use & 1, s_abort, budget))) { ok = false; break; }
      tc_fence_after();
      const int n = st * kSuperRows + 32 * e + lane;
      const bool n_ok = n < N;
      // kEpiSiluMul: lanes 0..15 of this quarter hold gate row i, lanes 16..31 the up row i
      const int i_gu = 16 * (4 * st + e) + (lane & 15);
#pragma unroll 1
      for (int cc = 0; cc < BT / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * e) << 16) + static_cast<uint32_t>(b * BT + 32 * cc), v);
        tc_wait_ld();
        if (KS == 2 && w.split) {
          // row 32 e + lane of the chunk: 8 16-byte pieces, piece j at position j ^ (lane & 7) of
          // the row's 128 bytes (the 8 lanes of a shared-memory phase hit distinct banks)
          constexpr int kXS = C::kXSlots > 0 ? C::kXSlots : 1;
          const int xs = static_cast<int>(xq % kXS);
          const uint32_t xpar = (xq / kXS) & 1;
          ++xq;
          uint8_t* xrow = smem + C::kOffX + xs * C::kXChunk + (32 * e + lane) * 128;
          if (rank == 1) {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded<true>(&xempty[xs], xpar ^ 1, s_abort, budget))) {
              ok = false;
              break;
            }
            const uint32_t dst = cluster_smem_addr(xrow, 0);
            const uint32_t bar = cluster_smem_addr(&xfull[xs], 0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_async_v4(dst + ((j ^ (lane & 7)) << 4), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3], bar);
            continue;   // rank 0 stores the tile
          }
          // one thread announces the chunk's bytes (rank 1's stores may count down before this)
          if (e == 0 && lane == 0) mbar_arrive_expect_tx(&xfull[xs], C::kXChunk);
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded<true>(&xfull[xs], xpar, s_abort, budget))) {
            ok = false;
            break;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {   // own partial sums first, then rank 1's (a fixed order)
            const float4 p = *reinterpret_cast<const float4*>(xrow + ((j ^ (lane & 7)) << 4));
            v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + p.x);
            v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + p.y);
            v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + p.z);
            v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + p.w);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(cluster_smem_addr(&xempty[xs], 1));
        }
        const int mb = mt * BT + 32 * cc;
        if (EPI == kEpiSiluMul) {
          const int I = N / 2;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float g = __uint_as_float(v[j]);
            const float u = __shfl_down_sync(0xFFFFFFFFu, g, 16);
            const int m = mb + j;
            if (lane < 16 && i_gu < I && m < M) epi.y0[static_cast<size_t>(m) * I + i_gu] = __float2half_rn(silu_mul(g, u));
          }
        } else if (n_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = mb + j;
            if (m < M) epi_store<EPI>(epi, m, n, N, __uint_as_float(v[j]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  if (KS == 2) {   // neither CTA exits while the other may still write to or arrive on it
    cluster_arrive();
    cluster_wait();
  }
}

}  // namespace awq
