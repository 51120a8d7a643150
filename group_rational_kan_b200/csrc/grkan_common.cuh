// grkan_common.cuh -- element types and per-element math of the GR-KAN
// group-rational activation (device side).
//
// y = P(x) / (1 + |Q(x)|), P(x) = sum_{i<=m} a_i x^i, Q(x) = sum_{1<=j<=n} b_j x^j
// ("FlashKAT: Understanding and Addressing Performance Bottlenecks in the
// Kolmogorov-Arnold Transformer", paper notes, section "KAT's breakthrough":
// grouped inputs sharing the coefficients of a safe Pade activation unit).
// Backward with D = 1 + |Q|, r = 1/D, s = sign(Q) (sign(0) = 0), t = dy*r:
//   dx = t P'(x) - t y s Q'(x);  dA_i += t x^i;  dB_j += -t y s x^j.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace grk {

// ---------------------------------------------------------------------------
// Element types of x, y, dy, dx. Arithmetic is always float32.
struct IoF32 {
  using T = float;
  static constexpr int kBytes = 4;
  static __device__ __forceinline__ float ld(const T* p, long long i) { return p[i]; }
  static __device__ __forceinline__ T cvt(float v) { return v; }
};

struct IoBF16 {
  using T = unsigned short;  // bf16 bit pattern
  static constexpr int kBytes = 2;
  static __device__ __forceinline__ float ld(const T* p, long long i) {
    return __uint_as_float(static_cast<unsigned>(p[i]) << 16);
  }
  static __device__ __forceinline__ T cvt(float v) {
    unsigned short h;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(v));
    return h;
  }
};

// ---------------------------------------------------------------------------
// Scalar helpers.

// Reciprocal of D = 1 + |Q| >= 1 (hardware approximation, max 1 ulp).
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// -y * sign(q) with sign(0) = 0, by flipping y's sign bit unless q is negative.
__device__ __forceinline__ float neg_y_sign(float y, float q) {
  const unsigned r = __float_as_uint(y) ^ (~__float_as_uint(q) & 0x80000000u);
  return (q != 0.f) ? __uint_as_float(r) : 0.f;
}

// ---------------------------------------------------------------------------
// Coefficients of one group in registers. ca[i] = a_i (i <= m), cb[j] = b_j
// (1 <= j <= n; cb[0] unused). Degrees are runtime values bounded by the
// template maxima; every loop is unrolled to the maxima with guards so the
// arrays stay in registers (for the exact-degree kernels the guards fold away).
template <int MM, int NM>
struct GroupCoef {
  float ca[MM + 1];
  float cb[NM + 1];

  __device__ __forceinline__ void load(const float* a, const float* b, int g, int m, int n) {
#pragma unroll
    for (int i = 0; i <= MM; ++i) ca[i] = (i <= m) ? __ldg(a + (long long)g * (m + 1) + i) : 0.f;
    cb[0] = 0.f;
#pragma unroll
    for (int j = 1; j <= NM; ++j) cb[j] = (j <= n) ? __ldg(b + (long long)g * n + (j - 1)) : 0.f;
  }
};

// Forward value at one point: Horner for P and for Q / x.
template <int MM, int NM>
__device__ __forceinline__ float forward_point(const GroupCoef<MM, NM>& c, float x, int m, int n) {
  float P = 0.f;
#pragma unroll
  for (int i = MM; i >= 0; --i) {
    if (i == m) P = c.ca[i];
    else if (i < m) P = fmaf(P, x, c.ca[i]);
  }
  float q = 0.f;  // Q(x) / x = b_1 + b_2 x + ... + b_n x^(n-1)
#pragma unroll
  for (int j = NM; j >= 1; --j) {
    if (j == n) q = c.cb[j];
    else if (j < n) q = fmaf(q, x, c.cb[j]);
  }
  const float Q = q * x;
  return P * rcp_approx(1.f + fabsf(Q));
}

// Backward at one point. Returns dx; adds t x^i to accA[i] and
// -t y s x^j to accB[j-1].
template <int MM, int NM>
__device__ __forceinline__ float backward_point(const GroupCoef<MM, NM>& c, float x, float dy,
                                                int m, int n, float* accA, float* accB) {
  // P and P' together by Horner.
  float P = 0.f, dP = 0.f;
#pragma unroll
  for (int i = MM; i >= 0; --i) {
    if (i == m) {
      P = c.ca[i];
    } else if (i < m) {
      dP = fmaf(dP, x, P);
      P = fmaf(P, x, c.ca[i]);
    }
  }
  // q = Q / x and q' by Horner; Q = q x, Q' = q + x q'.
  float q = 0.f, dq = 0.f;
#pragma unroll
  for (int j = NM; j >= 1; --j) {
    if (j == n) {
      q = c.cb[j];
    } else if (j < n) {
      dq = fmaf(dq, x, q);
      q = fmaf(q, x, c.cb[j]);
    }
  }
  const float Q = q * x;
  const float dQ = fmaf(dq, x, q);
  const float r = rcp_approx(1.f + fabsf(Q));
  const float y = P * r;
  const float t = dy * r;
  const float nu = t * neg_y_sign(y, Q);  // -t y s
  float xi = 1.f;
#pragma unroll
  for (int i = 0; i <= MM; ++i) {
    if (i <= m) {
      accA[i] = fmaf(t, xi, accA[i]);
      xi *= x;
    }
  }
  xi = x;
#pragma unroll
  for (int j = 1; j <= NM; ++j) {
    if (j <= n) {
      accB[j - 1] = fmaf(nu, xi, accB[j - 1]);
      xi *= x;
    }
  }
  return fmaf(nu, dQ, t * dP);
}

}  // namespace grk
