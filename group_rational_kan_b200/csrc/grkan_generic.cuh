// grkan_generic.cuh -- plain kernels for any shape, alignment and degree.
//
// One CTA per work unit (row tile x group), the two-dimensional decomposition
// of the FlashKAT backward ("FlashKAT ...", paper notes, section
// "3. FlashKAT kernel restructuring (Algorithm 2)": first grid dimension over
// ceil(B*N / S_block) row tiles, second over the n_g groups). The group's
// coefficients are loaded once per CTA; the backward folds its per-thread
// partial sums through warp shuffles and shared memory into one workspace slot
// per (unit, coefficient), with no atomics. Scalar loads: these kernels carry
// shapes the TMA-pipelined kernels do not take (unaligned rows, odd group
// widths, other degrees).
#pragma once

#include "grkan_common.cuh"

namespace grk {

constexpr int kGenericThreads = 256;

template <class IO, int MM, int NM>
__global__ void __launch_bounds__(kGenericThreads)
fwd_generic(const typename IO::T* x, typename IO::T* y, const float* __restrict__ a,
            const float* __restrict__ b, long long rows, long long d, int dg, int n_g, int m, int n,
            int S) {
  const long long unit = blockIdx.x;
  const long long tile = unit / n_g;
  const int g = (int)(unit - tile * n_g);
  GroupCoef<MM, NM> c;
  c.load(a, b, g, m, n);
  const long long r0 = tile * S;
  const long long nr = (rows - r0) < S ? (rows - r0) : S;
  const long long cnt = nr * dg;
  for (long long l = threadIdx.x; l < cnt; l += blockDim.x) {
    const long long r = r0 + l / dg;
    const long long e = r * d + (long long)g * dg + (l % dg);
    y[e] = IO::cvt(forward_point<MM, NM>(c, IO::ld(x, e), m, n));
  }
}

// Partial sums of one unit -> ws[(g*K + k) * ws_T + tile0 + tile], K = m + 1 + n.
template <class IO, int MM, int NM>
__global__ void __launch_bounds__(kGenericThreads)
bwd_generic(const typename IO::T* x, const typename IO::T* dy, typename IO::T* dx,
            const float* __restrict__ a, const float* __restrict__ b, float* __restrict__ ws,
            long long rows, long long d, int dg, int n_g, int m, int n, int S, long long ws_T,
            long long tile0) {
  __shared__ float red[kGenericThreads / 32][MM + 1 + NM];
  const long long unit = blockIdx.x;
  const long long tile = unit / n_g;
  const int g = (int)(unit - tile * n_g);
  GroupCoef<MM, NM> c;
  c.load(a, b, g, m, n);
  float accA[MM + 1], accB[NM > 0 ? NM : 1];
#pragma unroll
  for (int i = 0; i <= MM; ++i) accA[i] = 0.f;
#pragma unroll
  for (int j = 0; j < (NM > 0 ? NM : 1); ++j) accB[j] = 0.f;

  const long long r0 = tile * S;
  const long long nr = (rows - r0) < S ? (rows - r0) : S;
  const long long cnt = nr * dg;
  for (long long l = threadIdx.x; l < cnt; l += blockDim.x) {
    const long long r = r0 + l / dg;
    const long long e = r * d + (long long)g * dg + (l % dg);
    const float xv = IO::ld(x, e);
    const float gv = IO::ld(dy, e);
    dx[e] = IO::cvt(backward_point<MM, NM>(c, xv, gv, m, n, accA, accB));
  }

  // Fixed-order block reduction: xor butterfly inside each warp, then warps in
  // index order.
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i <= MM; ++i) {
    float v = accA[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][i] = v;
  }
#pragma unroll
  for (int j = 0; j < NM; ++j) {
    float v = accB[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][MM + 1 + j] = v;
  }
  __syncthreads();
  const int K = m + 1 + n;
  if (threadIdx.x < K) {
    const int k = threadIdx.x;
    const int slot = (k <= m) ? k : (MM + 1 + (k - m - 1));
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kGenericThreads / 32; ++w) s += red[w][slot];
    ws[((long long)g * K + k) * ws_T + tile0 + tile] = s;
  }
}

}  // namespace grk
