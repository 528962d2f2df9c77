// awq_quant.cuh — a2: AWQ scale fold + asymmetric 4-bit group quantizer (g = 128).
//
// llm-awq README "Usage" steps 1-3 (--w_bit 4 --q_group_size 128, real
// quantization), HF "transformers - AWQ" section 2 (zero_point true, bits 4,
// group_size 128), CSDN "02.02 AWQ" (salient weight channels scaled up by s).
//
// Per group of 128 weights along K (all IEEE fp32, round to nearest even):
//   w'  = fp16(fp32(W) * s_k)
//   lo, hi = min, max of w'
//   S   = fp16(max(hi - lo, 1e-5) / 15)
//   z   = clamp(rint(-lo / S), 0, 15)
//   q   = clamp(rint(w' / S) + z, 0, 15)
// Variants (template arguments kBits, kSym; the llm-awq README's model zoo lists INT3-g128
// next to INT4-g128, the llmstudio.ru AutoAWQ section names w_bit and zero_point): 3-bit codes
// take qmax = 7 in place of 15 in the same rules (stored in the same 4-bit slots); the symmetric
// form (zero_point false) takes S = fp16(max(max|w'|, 1e-5) / (2^(b-1) - 1)) and the fixed
// z = 2^(b-1), then the same q = clamp(rint(w' / S) + z, 0, qmax).
//
// w'/S is computed as va = w'*r, rho = fma(-S, va, w'), v = fma(rho, r, va)
// with r = RN(1/S), on packed fp32 pairs. This equals the IEEE quotient RN(w'/S) for every fp16
// pair: w' and S carry at most 11 significant bits, so their exact quotient
// is never a rounding midpoint of fp32 and lies at least 2^-12 ulp away from
// one, while va is within 1.5 ulp of the quotient, rho is exact (at most 12
// significant bits), and va + rho*r is within 2^-23 ulp of the quotient.
// (S = inf gives NaN here and 0 in the IEEE quotient; both end as code 0
// because z = 0 whenever S = inf.) Rounding is a magic-constant addition
// (1.5*2^23 + 16, even, so ties go to even). Clamping: when every lane's
// group keeps |w'/S| inside a 16-bit window (all groups of finite weights
// whose range is above the 1e-5 floor), the low 16 bits of the rounded sum
// are clamped as packed integers by one DPX instruction; otherwise
// clamp(rint(v) + z, 0, 15) == rint(clamp(v, -z, 15 - z)) + z is taken in
// fp32 before rounding (a clamped NaN becomes -z, i.e. code 0, as in the
// IEEE form). Measured alternatives that were slower on B200 and are not
// used: clamping w' on fp16 pairs before the division, a tree of min/max
// chains, and scalar fp32 in place of the packed f32x2 pairs.
//
// Work decomposition: persistent CTAs walk (super-tile, group) units. A
// producer lane streams each unit (128 rows x 128 k of fp16 W as two 2-D TMA
// boxes with 128-byte swizzle, plus the group's fold scales) into a 3-stage
// shared-memory ring, so HBM reads stay in flight while the 8 compute warps
// (16 rows each) work. Lanes l and l^8 hold the two halves of one row's group
// (their swizzled 16-byte reads are bank-conflict free); rows r and r+8 live
// in lanes l and l^16, which trade 4-code quads with one shuffle per word to
// assemble packed layout v2.
#pragma once

#include "awq_common.cuh"

namespace awq {

constexpr int kQuantThreads = 256;

// Packed fp32 pairs (sm_100 f32x2 arithmetic): one instruction for two IEEE
// fp32 operations, each rounded to nearest even exactly as the scalar form.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// fp16 pair -> two fp32 values through the mixed-precision add f32(h) + (-0.0), exact for every
// fp16 value (signed zeros and non-finite values included); measured slightly faster than the
// conversion instruction here.
__device__ __forceinline__ float2 h2_to_f2(uint32_t v) {
  float a, b;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.f16 %0, l, %3;\n\tadd.rn.f32.f16 %1, h, %3;\n\t}"
      : "=f"(a), "=f"(b)
      : "r"(v), "f"(-0.0f));
  return make_float2(a, b);
}

// Rounding by magic addition: for |v| <= 16, v + (1.5*2^23 + 16) rounds v to the
// nearest integer n (ties to even, since the constant is even) and leaves 16 + n in the
// low byte of the float's bits.
constexpr float kRoundMagic = 12582928.0f;   // 1.5 * 2^23 + 16

// One (super-tile, group) unit: 128 rows x 128 k of W, two 64-k TMA boxes with 128-byte
// swizzle (16 KB each), plus the group's 128 fold scales.
#ifndef AWQ_QUANT_STAGES
#define AWQ_QUANT_STAGES 3
#endif
#ifndef AWQ_QUANT_MINBLOCKS
#define AWQ_QUANT_MINBLOCKS 2
#endif
constexpr int kQStages = AWQ_QUANT_STAGES;
constexpr int kQBox = kSuperRows * 64 * 2;                  // 16 KB
// stage bases must stay 1024-byte aligned: the 128-byte swizzle pattern is a function of the address
constexpr int kQStageBytes = (2 * kQBox + kGroup * 4 + 1023) / 1024 * 1024;   // 32 KB + 512 B, rounded up
constexpr int kQComputeWarps = 8;
constexpr int kQThreads = (kQComputeWarps + 1) * 32;        // + 1 producer warp
constexpr int kQSmem = kQStages * kQStageBytes + 2 * kQStages * 8 + 16 + 1024;

// kBits: 4 or 3 (codes 0..2^kBits - 1 in the same 4-bit slots); kSym: symmetric variant
// (S = fp16(max(max|w'|, 1e-5) / (2^(kBits-1) - 1)), z = 2^(kBits-1)), the asymmetric rules otherwise.
template <bool kFold, int kBits = 4, bool kSym = false>
__global__ void __launch_bounds__(kQThreads, AWQ_QUANT_MINBLOCKS) awq_quantize_g128_kernel(const __grid_constant__ CUtensorMap tmap_w,
                                                                 const float* __restrict__ fold, int N, int K,
                                                                 uint32_t* __restrict__ qweight,
                                                                 __half* __restrict__ scales,
                                                                 uint8_t* __restrict__ zeros) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQStages * kQStageBytes);
  uint64_t* empty = full + kQStages;
  volatile int* s_abort = reinterpret_cast<volatile int*>(empty + kQStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = K / kGroup;
  const int G2 = ceil_div(G, 2);
  const int KTp = 4 * G2;              // k-tiles per tile in packed layout v2 (padded to group pairs)
  const int ntiles = ceil_div(N, kTileRows);
  const int ST = padded_rows(N) / kSuperRows;
  const int units = ST * G;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kQComputeWarps);
    }
    *s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();
  // Wait for the previous kernel, but do not let the next one start early: kernels that read
  // packed weights before their own wait (the decode kernel) may follow, so the next
  // kernel launches only once this grid has completed and every write below is visible.
  pdl_wait();
  const unsigned long long budget = g_wait_budget_ns;

  if (warp == kQComputeWarps) {
    // ---------------------------------------------------------------- producer
    if (lane != 0) return;
    tma_prefetch_desc(&tmap_w);
    int stage = 0;
    uint32_t phase = 0, issued_mask = 0, last_par = 0;
    bool drop = g_debug_drop_first_copy != 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const int st = u / G, g = u % G;
      if (!mbar_wait_bounded(&empty[stage], phase ^ 1, s_abort, budget)) break;
      if (drop) {   // test hook: this stage's copies are never issued
        drop = false;
        if (++stage == kQStages) { stage = 0; phase ^= 1; }
        continue;
      }
      uint8_t* dst = smem + stage * kQStageBytes;
      mbar_arrive_expect_tx(&full[stage], 2 * kQBox + (kFold ? kGroup * 4 : 0));
      tma_load_2d(dst, &tmap_w, g * kGroup, st * kSuperRows, &full[stage]);
      tma_load_2d(dst + kQBox, &tmap_w, g * kGroup + 64, st * kSuperRows, &full[stage]);
      if (kFold) bulk_g2s(dst + 2 * kQBox, fold + static_cast<size_t>(g) * kGroup, kGroup * 4, &full[stage]);
      issued_mask |= 1u << stage;
      last_par = (last_par & ~(1u << stage)) | (phase << stage);
      if (++stage == kQStages) { stage = 0; phase ^= 1; }
    }
    int never = 0;
    for (int s = 0; s < kQStages; ++s)
      if (issued_mask & (1u << s)) mbar_wait_bounded(&full[s], (last_par >> s) & 1u, &never, kDrainBudgetNs);
    return;
  }

  // ------------------------------------------------------------------ compute warps
  // lanes l and l^8 share a row (two halves of the group); lanes l and l^16 hold rows r, r+8
  const int nt = warp;
  const int r = lane & 7;
  const int half = (lane >> 3) & 1;
  const int h = lane >> 4;
  const int rr = r + 8 * h;                 // row in the 16-row tile
  const int row_s = nt * kTileRows + rr;    // row in the super-tile (TMA box row)
  int stage = 0;
  uint32_t phase = 0;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int st = u / G, g = u % G;
    // warp-uniform result: the shuffles below need the whole warp
    if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[stage], phase, s_abort, budget))) break;
    const uint8_t* sb = smem + stage * kQStageBytes;
    // ---- 64 weights of this lane: chunks c = 2i + half (16 B each), box c>>3, unit c&7 ^ (row & 7)
    uint4 raw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = 2 * i + half;
      raw[i] = *reinterpret_cast<const uint4*>(sb + (c >> 3) * kQBox + row_s * 128 + (((c & 7) ^ (row_s & 7)) << 4));
    }
    float4 sv[8][2];
    if (kFold) {
      const float* sfold = reinterpret_cast<const float*>(sb + 2 * kQBox);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sv[i][0] = *reinterpret_cast<const float4*>(&sfold[8 * (2 * i + half)]);
        sv[i][1] = *reinterpret_cast<const float4*>(&sfold[8 * (2 * i + half) + 4]);
      }
    }
    // the stage is in registers: hand it back to the producer
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    if (++stage == kQStages) { stage = 0; phase ^= 1; }

    const int n = st * kSuperRows + row_s;
    const bool valid = n < N;

    // ---- fold (fp32 multiply, RNE to fp16) and min/max on half2
    __half2 mn = __halves2half2(__ushort_as_half(0x7C00), __ushort_as_half(0x7C00));   // +inf
    __half2 mx = __halves2half2(__ushort_as_half(0xFC00), __ushort_as_half(0xFC00));   // -inf
    uint32_t wq[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t v[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __half2 hv = *reinterpret_cast<const __half2*>(&v[j]);
        if (kFold) {
          const float2 f = h2_to_f2(v[j]);
          const float4& a = sv[i][j >> 1];
          const float s0 = (j & 1) ? a.z : a.x;
          const float s1 = (j & 1) ? a.w : a.y;
          const float2 p = f2_unpack(f2_mul(f2_pack(f.x, f.y), f2_pack(s0, s1)));
          hv = __floats2half2_rn(p.x, p.y);
        }
        wq[i][j] = *reinterpret_cast<uint32_t*>(&hv);
        mn = __hmin2(mn, hv);
        mx = __hmax2(mx, hv);
      }
    }
    float lo = fminf(__low2float(mn), __high2float(mn));
    float hi = fmaxf(__low2float(mx), __high2float(mx));
    lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, 8));
    hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, 8));

    // ---- scale, zero point, reciprocal
    constexpr int kQMax = (1 << kBits) - 1;
    constexpr float kQMaxF = static_cast<float>(kQMax);
    __half S;
    float zf;
    if constexpr (kSym) {
      const float amax = fmaxf(fmaxf(fabsf(lo), fabsf(hi)), 1e-5f);
      S = __float2half_rn(__fdiv_rn(amax, static_cast<float>((1 << (kBits - 1)) - 1)));
      zf = static_cast<float>(1 << (kBits - 1));
    } else {
      const float range = fmaxf(__fsub_rn(hi, lo), 1e-5f);
      S = __float2half_rn(__fdiv_rn(range, kQMaxF));
      zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, __half2float(S))), 0.0f), kQMaxF);
    }
    const float Sf = __half2float(S);
    const float rcp = __frcp_rn(Sf);
    // clamp(rint(v) + z, 0, qmax) == rint(clamp(v, -z, qmax - z)) + z, as -z and qmax - z are integers
    const float vlo = -zf, vhi = __fsub_rn(kQMaxF, zf);
    const uint64_t rcp2 = f2_pack(rcp, rcp), nS2 = f2_pack(-Sf, -Sf), magic2 = f2_pack(kRoundMagic, kRoundMagic);
    const uint32_t zsub = (16u - static_cast<uint32_t>(__float2int_rz(zf))) * 0x01010101u;

    // ---- codes: one quad (4 consecutive k = slots e0..e3) per (chunk i, step-half sb)
    uint32_t quad[8][2];
    // Packed-integer clamp: for |v| < 2^15 - 16 the low 16 bits of v + (1.5*2^23 + 16) are
    // 16 + rint(v) (two's complement); one DPX add-min-relu on 16-bit pairs, max(min(a + b, 15), 0)
    // with b = z - 16, then gives clamp(rint(v) + z, 0, 15). Every group of finite fp16 weights whose range is not the
    // 1e-5 floor has |v| <= 15 * 2^11 (range >= one fp16 ulp of max(|lo|, |hi|)); groups beyond
    // the 16-bit window (range at the floor, non-finite values) take the fp32 clamp below.
    const bool fast = fmaxf(fabsf(lo), fabsf(hi)) * rcp < 32000.0f;
    if (__all_sync(0xFFFFFFFFu, fast)) {
      const uint32_t zoff2 = (static_cast<uint32_t>(__float2int_rz(zf) - 16) & 0xFFFFu) * 0x00010001u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int sbh = 0; sbh < 2; ++sbh) {
          uint32_t code2[2];
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {
            const float2 w = h2_to_f2(wq[i][2 * sbh + pr]);
            const uint64_t w2 = f2_pack(w.x, w.y);
            const uint64_t va = f2_mul(w2, rcp2);
            const uint64_t rho = f2_fma(nS2, va, w2);
            const uint64_t v2 = f2_fma(rho, rcp2, va);
            const float2 tq = f2_unpack(f2_add(v2, magic2));
            const uint32_t t16 = __byte_perm(__float_as_uint(tq.x), __float_as_uint(tq.y), 0x5410);
            code2[pr] = __viaddmin_s16x2_relu(t16, zoff2, kQMax * 0x00010001u);   // max(min(n + z, qmax), 0)
          }
          // padding rows (n >= N) read as zeros: code 0 unless the zero point is fixed (symmetric)
          if constexpr (kSym) quad[i][sbh] = valid ? __byte_perm(code2[0], code2[1], 0x6420) : 0u;
          else quad[i][sbh] = __byte_perm(code2[0], code2[1], 0x6420);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int sbh = 0; sbh < 2; ++sbh) {
          uint32_t lowbytes[2];
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {
            const float2 w = h2_to_f2(wq[i][2 * sbh + pr]);
            // IEEE quotient w / S: va = w * r, rho = w - S * va (exact), v = va + rho * r
            const uint64_t w2 = f2_pack(w.x, w.y);
            const uint64_t va = f2_mul(w2, rcp2);
            const uint64_t rho = f2_fma(nS2, va, w2);
            float2 v = f2_unpack(f2_fma(rho, rcp2, va));
            if constexpr (kSym) {
              // S = inf (an overflowed fold) gives rcp = 0: the IEEE quotient is w * 0 (0 for finite w,
              // NaN for infinite w), while the correction term above is NaN; with the fixed zero point
              // the two give different codes, so take the quotient itself
              if (rcp == 0.0f) v = f2_unpack(va);
            }
            v.x = fminf(fmaxf(v.x, vlo), vhi);
            v.y = fminf(fmaxf(v.y, vlo), vhi);
            const float2 tq = f2_unpack(f2_add(f2_pack(v.x, v.y), magic2));
            lowbytes[pr] = __byte_perm(__float_as_uint(tq.x), __float_as_uint(tq.y), 0x0040);
          }
          // bytes (16 + n) for slots e0..e3, minus (16 - z) per byte: n + z in [0, qmax], no borrows
          const uint32_t q4 = __byte_perm(lowbytes[0], lowbytes[1], 0x5410) - zsub;
          quad[i][sbh] = valid ? q4 : 0u;
        }
      }
    }

    // ---- assemble words: lane with h = 0 builds k-tile 2g, lane with h = 1 builds k-tile 2g+1.
    // Chunk i covers k-tile (i >> 2), column block t = (i & 3), steps s = 2*half + sbh.
    // Tile T = 8 st + nt of packed layout v2: its k-tiles follow one another (KTp per tile).
    const int T = st * 8 + nt;
    // the group's codes lie inside the packed arrays (ntiles x KTp chunks of 512 bytes)
    if (T < ntiles && AWQ_CHECK(g >= 0 && g < G && 2 * g + h < KTp)) {
      uint32_t* out = qweight + (static_cast<size_t>(T) * KTp + 2 * g + h) * kChunkWords;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        uint32_t w2[2];
#pragma unroll
        for (int sbh = 0; sbh < 2; ++sbh) {
          const uint32_t send = h ? quad[t][sbh] : quad[4 + t][sbh];
          const uint32_t mine = h ? quad[4 + t][sbh] : quad[t][sbh];
          const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, send, 16);
          const uint32_t a = h ? recv : mine;   // row r
          const uint32_t b = h ? mine : recv;   // row r + 8
          w2[sbh] = __byte_perm(a | (b << 4), 0u, 0x3120);
        }
        *reinterpret_cast<uint2*>(out + (4 * r + t) * 4 + 2 * half) = make_uint2(w2[0], w2[1]);
      }
      // ---- scales and zero points
      const size_t meta = static_cast<size_t>(T) * 2 * G2 + g;
      const int zi = valid ? __float2int_rz(zf) : 0;
      const int z_hi = __shfl_xor_sync(0xFFFFFFFFu, zi, 16);
      if (half == 0) {
        scales[meta * 16 + 2 * r + h] = valid ? S : __ushort_as_half(0);
        if (h == 0) zeros[meta * 8 + r] = static_cast<uint8_t>(zi | (z_hi << 4));
      }
      // an odd group count leaves one padding group per tile: code 0, scale 0, zero 0
      if ((G & 1) && g == G - 1) {
        uint32_t* pad = qweight + (static_cast<size_t>(T) * KTp + 2 * G + h) * kChunkWords;
#pragma unroll
        for (int t = 0; t < 4; ++t) *reinterpret_cast<uint2*>(pad + (4 * r + t) * 4 + 2 * half) = make_uint2(0u, 0u);
        if (half == 0) {
          scales[(meta + 1) * 16 + 2 * r + h] = __ushort_as_half(0);
          if (h == 0) zeros[(meta + 1) * 8 + r] = 0;
        }
      }
    }
  }
  __threadfence();   // this thread's codes, scales and zeros are visible device-wide before it exits
}

}  // namespace awq
