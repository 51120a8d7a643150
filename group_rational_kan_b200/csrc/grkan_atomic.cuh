// grkan_atomic.cuh -- the coefficient-gradient accumulation schemes that the
// FlashKAT study compares, kept for error and speed measurements only:
//
//   per element  every thread handles one element and adds each of its m+1+n
//                gradient terms straight into dA / dB in global memory with a
//                float32 atomic add ("FlashKAT ...", paper notes, section
//                "2. The atomic-add problem of the original KAT", Algorithm 1);
//   per block    a block owns S_block rows x d_g elements of one group, sums
//                their terms on chip, then adds each of its m+1+n sums into
//                dA / dB with one atomic add (section "3. FlashKAT kernel
//                restructuring (Algorithm 2)": a 2-D grid of row tiles x
//                groups).
//
// Both depend on the order in which the atomics land, so their results change
// from run to run; the library's own backward (two stages, fixed order) does
// not. dx is written exactly as by the other kernels.
#pragma once

#include "grkan_common.cuh"

namespace grk {

constexpr int kAtomicThreads = 256;

template <class IO, int MM, int NM>
__global__ void __launch_bounds__(kAtomicThreads)
bwd_atomic_element(const typename IO::T* x, const typename IO::T* dy, typename IO::T* dx,
                   const float* __restrict__ a, const float* __restrict__ b, float* dA,
                   float* dB, long long elems, long long d, int dg, int m, int n) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < elems; e += stride) {
    const int g = (int)((e % d) / dg);
    GroupCoef<MM, NM> c;
    c.load(a, b, g, m, n);  // every thread reads its group's coefficients itself
    float accA[MM + 1], accB[NM > 0 ? NM : 1];
#pragma unroll
    for (int i = 0; i <= MM; ++i) accA[i] = 0.f;
#pragma unroll
    for (int j = 0; j < (NM > 0 ? NM : 1); ++j) accB[j] = 0.f;
    dx[e] = IO::cvt(backward_point<MM, NM>(c, IO::ld(x, e), IO::ld(dy, e), m, n, accA, accB));
#pragma unroll
    for (int i = 0; i <= MM; ++i)
      if (i <= m) atomicAdd(dA + (long long)g * (m + 1) + i, accA[i]);
#pragma unroll
    for (int j = 0; j < NM; ++j)
      if (j < n) atomicAdd(dB + (long long)g * n + j, accB[j]);
  }
}

// One block per (row tile of S_block rows, group); blockIdx.x = tile * n_g + g.
template <class IO, int MM, int NM>
__global__ void __launch_bounds__(kAtomicThreads)
bwd_atomic_block(const typename IO::T* x, const typename IO::T* dy, typename IO::T* dx,
                 const float* __restrict__ a, const float* __restrict__ b, float* dA, float* dB,
                 long long rows, long long d, int dg, int n_g, int m, int n, int s_block) {
  __shared__ float red[kAtomicThreads / 32][MM + 1 + NM];
  const long long tile = blockIdx.x / n_g;
  const int g = (int)(blockIdx.x - tile * n_g);
  GroupCoef<MM, NM> c;
  c.load(a, b, g, m, n);
  float accA[MM + 1], accB[NM > 0 ? NM : 1];
#pragma unroll
  for (int i = 0; i <= MM; ++i) accA[i] = 0.f;
#pragma unroll
  for (int j = 0; j < (NM > 0 ? NM : 1); ++j) accB[j] = 0.f;
  const long long r0 = tile * s_block;
  const long long nr = (rows - r0) < s_block ? (rows - r0) : s_block;
  const long long cnt = nr * dg;
  for (long long l = threadIdx.x; l < cnt; l += blockDim.x) {
    const long long e = (r0 + l / dg) * d + (long long)g * dg + (l % dg);
    dx[e] = IO::cvt(backward_point<MM, NM>(c, IO::ld(x, e), IO::ld(dy, e), m, n, accA, accB));
  }
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
    for (int w = 0; w < kAtomicThreads / 32; ++w) s += red[w][slot];
    if (k <= m) atomicAdd(dA + (long long)g * (m + 1) + k, s);
    else atomicAdd(dB + (long long)g * n + (k - m - 1), s);
  }
}

}  // namespace grk
