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
//
// w'/S is computed as va = w'*r, rho = fma(-S, va, w'), v = fma(rho, r, va)
// with r = RN(1/S). This equals the IEEE quotient RN(w'/S) for every fp16
// pair: w' and S carry at most 11 significant bits, so their exact quotient
// is never a rounding midpoint of fp32 and lies at least 2^-12 ulp away from
// one, while va is within 1.5 ulp of the quotient, rho is exact (at most 12
// significant bits), and va + rho*r is within 2^-23 ulp of the quotient.
// (S = inf gives NaN here and 0 in the IEEE quotient; both end as code 0
// because z = 0 whenever S = inf.)
//
// Work decomposition: a CTA of 8 warps owns one 128-row super-tile and one
// group; warp nt owns rows nt*16 .. nt*16+15. Lane l loads row l/2, 16-byte
// chunks c = 2i + (l&1) of the group (two lanes read one 32-byte sector per
// instruction). Rows r and r+8 live in lanes l and l^16, which trade 4-code
// quads with one shuffle per word to assemble packed layout v1.
#pragma once

#include "awq_common.cuh"

namespace awq {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint32_t quad_of_codes(float q0, float q1, float q2, float q3) {
  // codes are integer-valued floats in [0, 15]; byte e = code of slot e
  const uint32_t a = static_cast<uint32_t>(__float2int_rz(q0)) | (static_cast<uint32_t>(__float2int_rz(q1)) << 8);
  const uint32_t b = static_cast<uint32_t>(__float2int_rz(q2)) | (static_cast<uint32_t>(__float2int_rz(q3)) << 8);
  return a | (b << 16);
}

template <bool kFold>
__global__ void __launch_bounds__(kQuantThreads) quantize_g128_kernel(const __half* __restrict__ W,
                                                                     const float* __restrict__ fold, int N, int K,
                                                                     uint32_t* __restrict__ qweight,
                                                                     __half* __restrict__ scales,
                                                                     uint8_t* __restrict__ zeros) {
  __shared__ __align__(16) float s_fold[kGroup];
  const int g = blockIdx.x;
  const int st = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = warp;
  const int G = K / kGroup;
  const int KT = K / kKTile;
  if (kFold) {
    if (threadIdx.x < kGroup / 4)
      reinterpret_cast<float4*>(s_fold)[threadIdx.x] =
          __ldg(reinterpret_cast<const float4*>(fold + static_cast<size_t>(g) * kGroup) + threadIdx.x);
    __syncthreads();
  }
  const int rr = lane >> 1;              // row in the 16-row tile
  const int half = lane & 1;
  const int h = rr >> 3;                 // 0: rows 0-7 (lanes 0-15), 1: rows 8-15
  const int r = rr & 7;
  const int n = st * kSuperRows + nt * kTileRows + rr;
  const bool valid = n < N;

  // ---- load 64 weights: chunks c = 2i + half, k = 128g + 8c .. 8c+7
  uint4 raw[8];
  const __half* wrow = W + static_cast<size_t>(valid ? n : 0) * K + static_cast<size_t>(g) * kGroup;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    raw[i] = valid ? ldg_stream_v4(wrow + 8 * (2 * i + half)) : make_uint4(0, 0, 0, 0);

  // ---- fold and min/max
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
        const int kk = 8 * (2 * i + half) + 2 * j;
        const float2 f = __half22float2(hv);
        hv = __floats2half2_rn(__fmul_rn(f.x, s_fold[kk]), __fmul_rn(f.y, s_fold[kk + 1]));
      }
      wq[i][j] = *reinterpret_cast<uint32_t*>(&hv);
      mn = __hmin2(mn, hv);
      mx = __hmax2(mx, hv);
    }
  }
  float lo = fminf(__low2float(mn), __high2float(mn));
  float hi = fmaxf(__low2float(mx), __high2float(mx));
  lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, 1));
  hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, 1));

  // ---- scale, zero point, reciprocal
  const float range = fmaxf(__fsub_rn(hi, lo), 1e-5f);
  const __half S = __float2half_rn(__fdiv_rn(range, 15.0f));
  const float Sf = __half2float(S);
  const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, Sf)), 0.0f), 15.0f);
  const float rcp = __frcp_rn(Sf);

  // ---- codes: one quad (4 consecutive k = slots e0..e3) per (chunk i, step-half sb)
  uint32_t quad[8][2];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int sb = 0; sb < 2; ++sb) {
      float qf[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t pair = wq[i][2 * sb + (e >> 1)];
        const unsigned short hb = static_cast<unsigned short>((e & 1) ? (pair >> 16) : (pair & 0xFFFFu));
        const float w = __half2float(__ushort_as_half(hb));
        const float va = __fmul_rn(w, rcp);
        const float rho = __fmaf_rn(-Sf, va, w);
        const float v = __fmaf_rn(rho, rcp, va);
        qf[e] = fminf(fmaxf(__fadd_rn(rintf(v), zf), 0.0f), 15.0f);
      }
      quad[i][sb] = valid ? quad_of_codes(qf[0], qf[1], qf[2], qf[3]) : 0u;
    }
  }

  // ---- assemble words: lane with h = 0 builds k-tile 2g, lane with h = 1 builds k-tile 2g+1.
  // Chunk i covers k-tile (i >> 2), column block t = (i & 3), steps s = 2*half + sb.
  uint32_t* out = qweight + (static_cast<size_t>(st) * KT + 2 * g + h) * kSuperChunkWords +
                  static_cast<size_t>(nt) * kChunkWords;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    uint32_t w2[2];
#pragma unroll
    for (int sb = 0; sb < 2; ++sb) {
      const uint32_t send = h ? quad[t][sb] : quad[4 + t][sb];
      const uint32_t mine = h ? quad[4 + t][sb] : quad[t][sb];
      const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, send, 16);
      const uint32_t a = h ? recv : mine;   // row r
      const uint32_t b = h ? mine : recv;   // row r + 8
      w2[sb] = __byte_perm(a | (b << 4), 0u, 0x3120);
    }
    *reinterpret_cast<uint2*>(out + (4 * r + t) * 4 + 2 * half) = make_uint2(w2[0], w2[1]);
  }

  // ---- scales and zero points
  const size_t meta = (static_cast<size_t>(st) * G + g) * 8 + nt;
  const int zi = valid ? __float2int_rz(zf) : 0;
  const int z_hi = __shfl_xor_sync(0xFFFFFFFFu, zi, 16);
  if (half == 0) {
    scales[meta * 16 + 2 * r + h] = valid ? S : __ushort_as_half(0);
    if (h == 0) zeros[meta * 8 + r] = static_cast<uint8_t>(zi | (z_hi << 4));
  }
}

}  // namespace awq
