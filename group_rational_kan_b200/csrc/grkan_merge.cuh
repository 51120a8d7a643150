// grkan_merge.cuh -- second stage of the coefficient-gradient reduction.
//
// The first stage leaves one float32 partial per (row tile, group,
// coefficient). This kernel adds the T partials of each (group, coefficient)
// in double precision in a fixed order and writes dA / dB: a second-stage
// merge in a set order takes the place of per-element atomic adds (the
// two-stage reduction of "PolyKAN: Efficient Fused GPU Operators for
// Polynomial Kolmogorov-Arnold Network Variants", abstract, technique (iii)).
// The order never depends on timing, so the result is identical from run to
// run.
#pragma once

#include "grkan_common.cuh"

namespace grk {

constexpr int kMergeThreads = 256;

// One CTA per (group, coefficient): thread t adds tiles t, t + 256, ... in
// float64, then the CTA adds the 256 thread sums in a fixed tree (xor
// butterfly inside each warp, warps in index order).
__global__ void __launch_bounds__(kMergeThreads)
merge_partials(const float* __restrict__ ws, float* __restrict__ dA, float* __restrict__ dB,
               double* __restrict__ sums64, long long T, int n_g, int m, int n) {
  __shared__ double part[kMergeThreads / 32];
  const int K = m + 1 + n;
  const long long o = blockIdx.x;
  const float* p = ws + o * T;
  double s = 0.0;
  for (long long t = threadIdx.x; t < T; t += kMergeThreads) s += (double)p[t];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
#pragma unroll
    for (int w = 0; w < kMergeThreads / 32; ++w) tot += part[w];
    const int g = (int)(o / K);
    const int k = (int)(o - (long long)g * K);
    if (k <= m)
      dA[(long long)g * (m + 1) + k] = (float)tot;
    else
      dB[(long long)g * n + (k - m - 1)] = (float)tot;
    if (sums64) sums64[o] = tot;
  }
}

// Data-parallel merge across devices: gathered holds `world` blocks of
// n_g * K float64 sums in rank order (one block per device, e.g. after an
// all-gather). Adds them in rank order and writes dA / dB.
__global__ void merge_ranks(const double* __restrict__ gathered, int world,
                            float* __restrict__ dA, float* __restrict__ dB, int n_g, int m,
                            int n) {
  const int K = m + 1 + n;
  const long long per = (long long)n_g * K;
  const long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= per) return;
  double s = 0.0;
  for (int r = 0; r < world; ++r) s += gathered[(long long)r * per + o];
  const int g = (int)(o / K);
  const int k = (int)(o - (long long)g * K);
  if (k <= m)
    dA[(long long)g * (m + 1) + k] = (float)s;
  else
    dB[(long long)g * n + (k - m - 1)] = (float)s;
}

}  // namespace grk
