// awq_act.cuh — a1: per-input-channel activation statistic and activation scaling.
//
// CSDN VPTQ blog, section "02.02 AWQ": the scale of a salient channel comes
// from offline activation statistics; the equivalent transform scales weight
// channels up by s and activations down by s. This file computes
//   s_k  = max(mean_m |x_mk|, 1e-8)^alpha      (float64, rounded to fp32)
//   x'_mk = fp16_rn(fp32(x_mk) / s_k)          (IEEE fp32 division)
//
// Design: one CTA owns a slab of 64 columns; a thread-block cluster of CL
// CTAs splits the rows of the slab. The column sums are exact integers in
// units of 2^-24 (every fp16 magnitude is an integer multiple of 2^-24), so
// the sum is independent of order; the CTAs of a cluster combine their
// partial sums through distributed shared memory, each computes the same s,
// and each scales its own rows. No global scratch, no atomics.
#pragma once

#include <cooperative_groups.h>

#include "awq_common.cuh"

namespace awq {

constexpr int kActCols = 64;       // columns per CTA slab
constexpr int kActThreads = 256;   // 8 warps; a warp covers 4 rows x 64 columns per step

// |fp16| as an integer number of 2^-24 units (exact for finite values).
__device__ __forceinline__ uint64_t f16_abs_units(uint32_t bits) {
  const uint32_t b = bits & 0x7FFFu;
  const uint32_t e = b >> 10;
  const uint32_t m = b & 0x3FFu;
  return e == 0 ? static_cast<uint64_t>(m) : (static_cast<uint64_t>(m | 0x400u) << (e - 1));
}

__global__ void __launch_bounds__(kActThreads) awq_act_scale_kernel(const __half* __restrict__ x, int M, int K,
                                                               float alpha, float* __restrict__ s_out,
                                                               __half* __restrict__ x_scaled) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());

  __shared__ uint64_t s_part[kActThreads / 32][kActCols];
  __shared__ uint64_t s_csum[kActCols];
  __shared__ float s_scale[kActCols];

  pdl_enter_early();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = blockIdx.x * kActCols;
  const int rsub = lane >> 3;         // 0..3: row within the warp's 4-row step
  const int c8 = lane & 7;            // 8-column block within the slab
  const int kc = k0 + 8 * c8;
  const bool col_ok = kc < K;         // K % 8 == 0, so a block is all in or all out
  const int m_begin = static_cast<int>((static_cast<long long>(M) * rank) / CL);
  const int m_end = static_cast<int>((static_cast<long long>(M) * (rank + 1)) / CL);

  // ---- pass 1: exact column sums of |x| over this CTA's rows
  uint64_t acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0;
  for (int m0 = m_begin + warp * 4; m0 < m_end; m0 += 32 * 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int m = m0 + u * 32 + rsub;
      if (col_ok && m < m_end) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K + kc));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[2 * j] += f16_abs_units(w[j] & 0xFFFFu);
          acc[2 * j + 1] += f16_abs_units(w[j] >> 16);
        }
      }
    }
  }
  // reduce the 4 row-lanes that share a column block (lanes c8, c8+8, c8+16, c8+24)
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    acc[j] += __shfl_xor_sync(0xFFFFFFFFu, acc[j], 8);
    acc[j] += __shfl_xor_sync(0xFFFFFFFFu, acc[j], 16);
  }
  if (rsub == 0) {
#pragma unroll
    for (int j = 0; j < 8; ++j) s_part[warp][8 * c8 + j] = acc[j];
  }
  __syncthreads();
  if (threadIdx.x < kActCols) {
    uint64_t t = 0;
#pragma unroll
    for (int w = 0; w < kActThreads / 32; ++w) t += s_part[w][threadIdx.x];
    s_csum[threadIdx.x] = t;
  }
  // ---- combine the cluster's partial sums (distributed shared memory)
  cluster.sync();
  if (threadIdx.x < kActCols) {
    uint64_t tot = 0;
    for (int r = 0; r < CL; ++r) {
      const uint64_t* remote = cluster.map_shared_rank(s_csum, r);
      tot += remote[threadIdx.x];
    }
    const int k = k0 + threadIdx.x;
    float sf = 1.0f;
    if (k < K) {
      // exact: tot < 2^53 for M < 2^13 (and rounded once beyond), times 2^-24 is exact
      const double sum = __dmul_rn(static_cast<double>(tot), 0x1p-24);
      double mean = __ddiv_rn(sum, static_cast<double>(M));
      mean = fmax(mean, 1e-8);
      const double p = (alpha == 0.5f) ? __dsqrt_rn(mean) : pow(mean, static_cast<double>(alpha));
      sf = __double2float_rn(p);
      if (rank == 0) s_out[k] = sf;
    }
    s_scale[threadIdx.x] = sf;
  }
  cluster.sync();   // remote reads done before any CTA of the cluster may exit; s_scale visible
  if (x_scaled == nullptr) return;

  // ---- pass 2: x' = fp16(fp32(x) / s) for this CTA's rows
  float sc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) sc[j] = s_scale[8 * c8 + j];
  for (int m0 = m_begin + warp * 4; m0 < m_end; m0 += 32 * 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int m = m0 + u * 32 + rsub;
      if (col_ok && m < m_end) {
        const size_t off = static_cast<size_t>(m) * K + kc;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + off));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] & 0xFFFFu)));
          const float b = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] >> 16)));
          const __half ha = __float2half_rn(__fdiv_rn(a, sc[2 * j]));
          const __half hb = __float2half_rn(__fdiv_rn(b, sc[2 * j + 1]));
          o[j] = static_cast<uint32_t>(__half_as_ushort(ha)) | (static_cast<uint32_t>(__half_as_ushort(hb)) << 16);
        }
        *reinterpret_cast<uint4*>(x_scaled + off) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// Small M (decode): one thread per column, no cluster. The same exact integer column sum,
// the same float64 statistic and the same fp32 division as awq_act_scale_kernel.
constexpr int kActSmallMaxM = 32;
__global__ void __launch_bounds__(128) awq_act_scale_small_kernel(const __half* __restrict__ x, int M, int K,
                                                             float alpha, float* __restrict__ s_out,
                                                             __half* __restrict__ x_scaled) {
  pdl_enter_early();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const unsigned short* xb = reinterpret_cast<const unsigned short*>(x);
  uint64_t tot = 0;
  for (int m = 0; m < M; ++m) tot += f16_abs_units(__ldg(xb + static_cast<size_t>(m) * K + k));
  const double sum = __dmul_rn(static_cast<double>(tot), 0x1p-24);
  double mean = __ddiv_rn(sum, static_cast<double>(M));
  mean = fmax(mean, 1e-8);
  const double p = (alpha == 0.5f) ? __dsqrt_rn(mean) : pow(mean, static_cast<double>(alpha));
  const float sf = __double2float_rn(p);
  s_out[k] = sf;
  if (x_scaled == nullptr) return;
  for (int m = 0; m < M; ++m) {
    const size_t off = static_cast<size_t>(m) * K + k;
    x_scaled[off] = __float2half_rn(__fdiv_rn(__half2float(__ushort_as_half(__ldg(xb + off))), sf));
  }
}

// x'[m, k] = fp16_rn(fp32(x[m, k]) / s[k]) with a given s (the activation half of the
// equivalent transform at inference time, s fixed by calibration). One thread per 8 values.
__global__ void __launch_bounds__(256) awq_scale_activations_kernel(const __half* __restrict__ x,
                                                               const float* __restrict__ s, long long total8, int K,
                                                               __half* __restrict__ xs) {
  pdl_enter_early();
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= total8) return;
  const long long off = i * 8;
  const int k = static_cast<int>(off % K);
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + off));
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k));
  const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k + 4));
  const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float a = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] & 0xFFFFu)));
    const float b = __half2float(__ushort_as_half(static_cast<unsigned short>(w[j] >> 16)));
    const __half ha = __float2half_rn(__fdiv_rn(a, sc[2 * j]));
    const __half hb = __float2half_rn(__fdiv_rn(b, sc[2 * j + 1]));
    o[j] = static_cast<uint32_t>(__half_as_ushort(ha)) | (static_cast<uint32_t>(__half_as_ushort(hb)) << 16);
  }
  *reinterpret_cast<uint4*>(xs + off) = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace awq
