// awq_search.cuh — the AWQ scale search: pick the exponent alpha of s = mean|x|^alpha.
//
// llm-awq README, "Usage" step 1: the AWQ search picks the scales on calibration data and dumps
// them; CSDN VPTQ blog, "02.02 AWQ": the scales come from offline activation statistics, with no
// backpropagation. For each candidate alpha the library runs the path it already has (activation
// statistic and scaling, fold + quantizer, the W4A16 linear layer) on the calibration rows and
// measures the squared output error against the layer's unquantized output x . W^T. This file
// holds the two kernels the search adds:
//  * awq_ref_gemm_kernel: y_ref[M,N] = x[M,K] . W[N,K]^T, fp16 inputs, fp32 accumulation and
//    output, on legacy warp MMAs with fragments loaded straight from global memory (an offline
//    step, run once per search);
//  * awq_sq_error_kernel / awq_sq_error_final_kernel: err = sum (y_ref - y)^2 in float64. The
//    first kernel writes one partial sum per block into scratch memory, the second adds them in
//    block order (deterministic) and, after the last candidate, picks the first minimum.
#pragma once

#include "awq_common.cuh"

namespace awq {

constexpr int kSearchMaxBlocks = 1024;   // partial sums of the error reduction
constexpr int kSearchThreads = 256;

// Each warp computes a 16 x 32 block of y_ref (four m16n8k16 tiles along N), CTA = 4 warps along N.
__global__ void __launch_bounds__(128) awq_ref_gemm_kernel(const __half* __restrict__ x, const __half* __restrict__ W,
                                                          float* __restrict__ y_ref, int M, int N, int K) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int m0 = blockIdx.y * 16;
  const int n0 = (blockIdx.x * 4 + warp) * 32;
  pdl_enter();
  float acc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
  const uint32_t* xw = reinterpret_cast<const uint32_t*>(x);
  const uint32_t* Ww = reinterpret_cast<const uint32_t*>(W);
  const int K2 = K / 2;   // 32-bit words per row
  auto ldx = [&](int m, int kw) -> uint32_t { return m < M ? __ldg(xw + static_cast<size_t>(m) * K2 + kw) : 0u; };
  auto ldw = [&](int n, int kw) -> uint32_t { return n < N ? __ldg(Ww + static_cast<size_t>(n) * K2 + kw) : 0u; };
  for (int k0 = 0; k0 < K; k0 += 16) {
    const int kw = k0 / 2 + t;
    uint32_t a[4];
    a[0] = ldx(m0 + g, kw);
    a[1] = ldx(m0 + g + 8, kw);
    a[2] = ldx(m0 + g, kw + 4);
    a[3] = ldx(m0 + g + 8, kw + 4);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + 8 * j + g;
      mma_m16n8k16_f32(acc[j], a, ldw(n, kw), ldw(n, kw + 4));
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int m = m0 + g + 8 * (c >> 1), n = n0 + 8 * j + 2 * t + (c & 1);
      if (m < M && n < N) y_ref[static_cast<size_t>(m) * N + n] = acc[j][c];
    }
}

// partial[b] = sum over this block's elements of (y_ref - y)^2, float64; elements are taken in a
// fixed order for a fixed grid, so the result is reproducible.
__global__ void __launch_bounds__(kSearchThreads) awq_sq_error_kernel(const float* __restrict__ y_ref,
                                                                     const __half* __restrict__ y, long long count,
                                                                     double* __restrict__ partial) {
  __shared__ double s_red[kSearchThreads / 32];
  pdl_enter();
  double v = 0.0;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const double d = static_cast<double>(y_ref[i]) - static_cast<double>(__half2float(y[i]));
    v = fma(d, d, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < kSearchThreads / 32; ++w) tot += s_red[w];
    partial[blockIdx.x] = tot;
  }
}

// err[i] = sum of the nblocks partials in block order. With best != nullptr (after the last
// candidate) also writes the index of the first smallest err[0..n_err).
__global__ void awq_sq_error_final_kernel(const double* __restrict__ partial, int nblocks, double* __restrict__ err,
                                          int i, int* __restrict__ best, int n_err) {
  pdl_enter();
  if (threadIdx.x != 0) return;
  double tot = 0.0;
  for (int b = 0; b < nblocks; ++b) tot += partial[b];
  err[i] = tot;
  if (best != nullptr) {
    int bi = 0;
    for (int j = 1; j < n_err; ++j)
      if (err[j] < err[bi]) bi = j;
    *best = bi;
  }
}

}  // namespace awq
