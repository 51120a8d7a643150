// grkan_tma.cuh -- persistent, TMA-pipelined forward and backward kernels.
//
// Work decomposition: (row tile x group) units as in the FlashKAT backward
// ("FlashKAT ...", paper notes, section "3. FlashKAT kernel restructuring
// (Algorithm 2)"), realised as a persistent grid of one CTA per SM (16 warps;
// 12 for the bf16 backward) in which every warp runs its own pipeline:
//   - a warp owns a ring of shared-memory stages (one 2-D TMA box of every input
//     tensor each) with its own full / empty mbarriers; its lane 0 issues the
//     box loads `stages` boxes ahead and refills a slot as soon as the warp has
//     read it; nothing couples the warps of a CTA after start-up, so one warp's
//     loads overlap another's arithmetic;
//   - work items (forward: boxes; backward: units of 8 boxes) are taken by the
//     warps in a fixed stride over a warp-major numbering, with division-free
//     mixed-radix cursors;
//   - the lanes evaluate the rational function on pairs of elements with packed
//     float32x2 arithmetic from coefficients kept in a CTA-wide table, and write
//     y or dx with 16-byte streaming stores after computing a pass's values (in
//     float32 the lanes instead stage the box in a per-warp slot that one TMA
//     tensor store per box writes out);
//   - the backward keeps the m + 1 + n coefficient-gradient sums in registers;
//     at the end of a unit the warp folds them in a fixed order (recursive
//     halving over shuffles) into one float32 partial per (unit, coefficient)
//     in the workspace -- no atomics (section "3. ...": accumulate inside the
//     block, one global write per block).
// Every wait is bounded: a wait that runs out records a code in
// g_grkan_device_error and the kernel winds down instead of hanging.
#pragma once

#include <atomic>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "grkan_common.cuh"

namespace grk {

struct TmaGeom {
  long long rows;       // B * N
  long long T;          // row tiles (units per group)
  long long ws_T;       // workspace stride between coefficients (tiles of the whole tensor)
  long long ws_tile0;   // workspace tile of this call's first tile
  long long d;          // channels (row length)
  long long S;          // rows per tile
  int dg;               // channels per group
  int n_g;              // groups
  int SCw;              // rows per TMA box
  int bw;               // TMA box width (channels)
  int nbox;             // boxes per group row = dg / bw
  unsigned box_bytes;   // SCw * bw * element size
  int m, n;             // degrees
  int nrb_full;         // row blocks (boxes of SCw rows) of a full tile: ceil(S / SCw)
  int nrb_last;         // row blocks of the last tile
};

// Launch shape (compile-time; the defaults are the tuned configuration).
// One CTA of independent warps per SM (16 for the forward; for the backward 16 in
// float32, HBM-bound, and 12 in bf16, whose arithmetic-bound loop runs faster with
// up to 168 registers per thread). Every warp owns, per element
// type, a ring of forward stages (one box of x each) and of backward stages
// (one box of x and one of dy each). The float32 forward streams 3 KiB boxes
// through three stages beside a staging slot for its TMA stores; the float32
// backward, 1.5 KiB boxes through four. The bf16 forward streams 2 KiB boxes
// through four stages (measured faster than 1.5 KiB x 4 or x 6, 1 KiB x 8 and
// 3 KiB x 3). The bf16 backward is
// bound by arithmetic issue: 3 KiB boxes read in three passes of two 16-byte
// vectors per lane, two stages.
#ifndef GRK_FWD_WARPS
#define GRK_FWD_WARPS 16
#endif
#ifndef GRK_F32_BWD_WARPS
#define GRK_F32_BWD_WARPS 16
#endif
#ifndef GRK_BF16_BWD_WARPS
#define GRK_BF16_BWD_WARPS 12
#endif
#ifndef GRK_F32_FWD_VEC
#define GRK_F32_FWD_VEC 6
#endif
#ifndef GRK_F32_FWD_STAGES
#define GRK_F32_FWD_STAGES 3
#endif
#ifndef GRK_F32_BWD_VEC
#define GRK_F32_BWD_VEC 3
#endif
#ifndef GRK_F32_BWD_HALVES
#define GRK_F32_BWD_HALVES 1
#endif
#ifndef GRK_F32_BWD_STAGES
#define GRK_F32_BWD_STAGES 4
#endif
#ifndef GRK_BF16_FWD_VEC
#define GRK_BF16_FWD_VEC 4
#endif
#ifndef GRK_BF16_FWD_STAGES
#define GRK_BF16_FWD_STAGES 4
#endif
#ifndef GRK_BF16_BWD_VEC
#define GRK_BF16_BWD_VEC 2
#endif
#ifndef GRK_BF16_BWD_HALVES
#define GRK_BF16_BWD_HALVES 3
#endif
#ifndef GRK_BF16_BWD_STAGES
#define GRK_BF16_BWD_STAGES 2
#endif

// How the backward writes dx, per element type: 0 = 16-byte streaming stores
// from the lanes (each pass's values first, then its stores, each guarded by its
// row); 2 = the lanes stage the box in a shared-memory slot and one TMA tensor
// store per box writes it (rows past the tensor are clipped by the tensor map).
// Measured on B200: bf16 (arithmetic-bound) is fastest with 0, float32
// (HBM-bound) with 2.
#ifndef GRK_F32_BWD_STORE
#define GRK_F32_BWD_STORE 2
#endif
#ifndef GRK_BF16_BWD_STORE
#define GRK_BF16_BWD_STORE 0
#endif
// How the forward writes y: 0 = each vector computed and stored under its row
// guard; 1 = all of a box's values first, then the guarded stores (bf16: 2.5 %
// faster than 0 on B200); 2 = staged and written by one TMA store per box
// (float32, with three ring stages to make room for the slot: 3-4 % faster than
// 0 with four).
#ifndef GRK_F32_FWD_STORE
#define GRK_F32_FWD_STORE 2
#endif
#ifndef GRK_BF16_FWD_STORE
#define GRK_BF16_FWD_STORE 1
#endif
constexpr int kFwdWarps = GRK_FWD_WARPS;  // forward: 16 warps x 128 registers
constexpr int kFwdThreads = kFwdWarps * 32;

template <class IO>
struct Shape;
template <>
struct Shape<IoF32> {
  static constexpr int kFwdVec = GRK_F32_FWD_VEC;        // vectors per lane in a forward box
  static constexpr int kFwdStages = GRK_F32_FWD_STAGES;  // forward ring depth
  static constexpr int kBwdVec = GRK_F32_BWD_VEC;        // vectors per lane and tensor in one pass
  static constexpr int kBwdHalves = GRK_F32_BWD_HALVES;  // passes over a backward box
  static constexpr int kBwdStages = GRK_F32_BWD_STAGES;  // backward ring depth
  static constexpr int kBwdWarps = GRK_F32_BWD_WARPS;    // backward warps per CTA
  static constexpr int kBwdStore = GRK_F32_BWD_STORE;    // how dx is written (see above)
  static constexpr int kFwdStore = GRK_F32_FWD_STORE;    // how y is written (see above)
};
template <>
struct Shape<IoBF16> {
  static constexpr int kFwdVec = GRK_BF16_FWD_VEC;
  static constexpr int kFwdStages = GRK_BF16_FWD_STAGES;
  static constexpr int kBwdVec = GRK_BF16_BWD_VEC;
  static constexpr int kBwdHalves = GRK_BF16_BWD_HALVES;
  static constexpr int kBwdStages = GRK_BF16_BWD_STAGES;
  static constexpr int kBwdWarps = GRK_BF16_BWD_WARPS;
  static constexpr int kBwdStore = GRK_BF16_BWD_STORE;
  static constexpr int kFwdStore = GRK_BF16_FWD_STORE;
};
template <class IO>
constexpr unsigned fwd_box_bytes() {
  return 32u * Shape<IO>::kFwdVec * 16u;
}
template <class IO>
constexpr unsigned bwd_box_bytes() {
  return 32u * Shape<IO>::kBwdVec * Shape<IO>::kBwdHalves * 16u;
}
inline unsigned fwd_box_target(bool bf16) {
  return bf16 ? fwd_box_bytes<IoBF16>() : fwd_box_bytes<IoF32>();
}
inline unsigned bwd_box_target(bool bf16) {
  return bf16 ? bwd_box_bytes<IoBF16>() : bwd_box_bytes<IoF32>();
}
#ifndef GRK_BOXES_PER_UNIT
#define GRK_BOXES_PER_UNIT 8
#endif
constexpr int kBoxesPerUnit = GRK_BOXES_PER_UNIT;  // backward boxes per (tile, group) unit
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s
// Backstop: a wait also gives up after this many polls, whatever the timer says.
constexpr unsigned kMaxPolls = 1u << 26;

// Error codes written to g_grkan_device_error (bit-or).
constexpr unsigned kErrFullWait = 1u;
constexpr unsigned kErrEmptyWait = 2u;
constexpr unsigned kErrReduceWait = 4u;
constexpr unsigned kErrDrainWait = 8u;
constexpr unsigned kErrSelfTest = 16u;  // grkan_selftest_wait_timeout's wait ran out

__device__ unsigned int g_grkan_device_error = 0;

// Degrees (m, n) with TMA-pipelined kernels: the KAT degree (5, 4) and m = n
// from 3 to 8 (for degree sweeps); every other degree takes the generic kernels.
#define GRK_TMA_DEGREES(X) X(3, 3) X(4, 4) X(5, 4) X(5, 5) X(6, 6) X(7, 7) X(8, 8)

inline bool tma_has_degree(int m, int n) {
#define GRK_DEG_CASE(M, N) \
  if (m == M && n == N) return true;
  GRK_TMA_DEGREES(GRK_DEG_CASE)
#undef GRK_DEG_CASE
  return false;
}
// The forward-and-backward (recompute) variant of the backward kernel exists for
// the KAT degree only.
inline bool tma_has_fused_degree(int m, int n) { return m == 5 && n == 4; }

// --- PTX wrappers --------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity; false after limit_ns (or
// kMaxPolls polls).
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity,
                                              unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned polls = 0; !mbar_try_wait(bar, parity); ++polls) {
    if (global_ns() - t0 > limit_ns || polls > kMaxPolls) return false;
  }
  return true;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  return mbar_wait_for(bar, parity, kWaitTimeoutNs);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// TMA tensor store of a box from shared memory (bulk async-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int c0, int c1,
                                             uint32_t src) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk store has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk store is complete.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void report(unsigned code) { atomicOr(&g_grkan_device_error, code); }

// --- packed float32x2 arithmetic -------------------------------------------------

__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// Two bf16 -> float32 exactly: the low half moved to the top by a byte permute,
// the high half by a mask (both integer-pipe operations).
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(__byte_perm(w, 0u, 0x1044)),
                     __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf16x2(float2 v) {
  __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);  // .x -> low half
  return *reinterpret_cast<uint32_t*>(&h);
}

// Coefficients of the (5, 4) fast path, broadcast to both lanes of a pair.
struct Coef54 {
  float2 a0, a1, a2, a3, a4, a5;      // a_i
  float2 ia2, ia3, ia4, ia5;          // i * a_i  (P')
  float2 b1, b2, b3, b4;              // b_j
  float2 jb2, jb3, jb4;               // j * b_j  (Q')

};

// y for a pair of elements: Horner for P and for Q / x.
__device__ __forceinline__ float2 fwd_pair(const Coef54& c, float2 x) {
  float2 P = fma2(c.a5, x, c.a4);
  P = fma2(P, x, c.a3);
  P = fma2(P, x, c.a2);
  P = fma2(P, x, c.a1);
  P = fma2(P, x, c.a0);
  float2 q = fma2(c.b4, x, c.b3);
  q = fma2(q, x, c.b2);
  q = fma2(q, x, c.b1);
  const float2 Q = mul2(q, x);
  const float2 r = make_float2(rcp_approx(1.f + fabsf(Q.x)), rcp_approx(1.f + fabsf(Q.y)));
  return mul2(P, r);
}

struct Acc54 {
  float2 a0, a1, a2, a3, a4, a5, b1, b2, b3, b4;
  __device__ __forceinline__ void zero() {
    a0 = a1 = a2 = a3 = a4 = a5 = b1 = b2 = b3 = b4 = make_float2(0.f, 0.f);
  }
};

// dx for a pair of elements; adds t x^i and -t y s x^j to the sums.
__device__ __forceinline__ float2 bwd_pair(const Coef54& c, float2 x, float2 dy, Acc54& acc,
                                           float2* y_out = nullptr) {
  const float2 x2 = mul2(x, x);
  const float2 x3 = mul2(x2, x);
  const float2 x4 = mul2(x2, x2);
  const float2 x5 = mul2(x4, x);
  // Horner's rule for P, P', Q / x and Q' (the operation count of Estrin's
  // scheme, fewer live temporaries: measured faster here). P and Q follow the
  // forward's order exactly, so the recomputed y is the forward's y bit for bit.
  const float2 P = fma2(fma2(fma2(fma2(fma2(c.a5, x, c.a4), x, c.a3), x, c.a2), x, c.a1), x, c.a0);
  const float2 dP = fma2(fma2(fma2(fma2(c.ia5, x, c.ia4), x, c.ia3), x, c.ia2), x, c.a1);
  const float2 Q = mul2(fma2(fma2(fma2(c.b4, x, c.b3), x, c.b2), x, c.b1), x);
  const float2 dQ = fma2(fma2(fma2(c.jb4, x, c.jb3), x, c.jb2), x, c.b1);
  const float2 r = make_float2(rcp_approx(1.f + fabsf(Q.x)), rcp_approx(1.f + fabsf(Q.y)));
  const float2 y = mul2(P, r);
  if (y_out) *y_out = y;
  const float2 t = mul2(dy, r);
  const float2 nu = mul2(t, make_float2(neg_y_sign(y.x, Q.x), neg_y_sign(y.y, Q.y)));
  acc.a0 = add2(acc.a0, t);
  acc.a1 = fma2(t, x, acc.a1);
  acc.a2 = fma2(t, x2, acc.a2);
  acc.a3 = fma2(t, x3, acc.a3);
  acc.a4 = fma2(t, x4, acc.a4);
  acc.a5 = fma2(t, x5, acc.a5);
  acc.b1 = fma2(nu, x, acc.b1);
  acc.b2 = fma2(nu, x2, acc.b2);
  acc.b3 = fma2(nu, x3, acc.b3);
  acc.b4 = fma2(nu, x4, acc.b4);
  return fma2(nu, dQ, mul2(t, dP));
}

__host__ __device__ constexpr unsigned round_up(unsigned v, unsigned a) {
  return (v + a - 1) / a * a;
}

// --- degree traits ------------------------------------------------------------------
//
// Deg<M, N> gives the packed kernels their coefficient registers, sums and
// per-pair arithmetic. The generic form evaluates in the power basis (x^k by
// balanced products, then one FMA per term); Deg<5, 4> is the hand-written
// Horner form above.

// Floats per group in the coefficient table: a_0..a_M, i a_i (i = 2..M),
// b_1..b_N, j b_j (j = 2..N), padded to a multiple of four.
template <int M, int N>
__host__ __device__ constexpr int tab_floats() {
  return ((M + 1) + (M - 1) + N + (N - 1) + 3) / 4 * 4;
}

// Table entry k of group g (the layout above), from the coefficient arrays.
template <int M, int N>
__device__ __forceinline__ float coef_value(const float* a, const float* b, int g, int k) {
  if (k <= M) return __ldg(a + g * (M + 1) + k);
  if (k < 2 * M) {
    const int i = k - (M + 1) + 2;
    return (float)i * __ldg(a + g * (M + 1) + i);
  }
  if (k < 2 * M + N) return __ldg(b + g * N + (k - 2 * M));
  if (k < 2 * M + 2 * N - 1) {
    const int j = k - (2 * M + N) + 2;
    return (float)j * __ldg(b + g * N + (j - 1));
  }
  return 0.f;
}

template <int M, int N>
struct Deg {
  static constexpr int K = M + 1 + N;
  static constexpr int TF = tab_floats<M, N>();
  struct Coef {
    float2 a[M + 1];   // a_i
    float2 ia[M + 1];  // i a_i, i >= 2
    float2 b[N + 1];   // b_j, j >= 1
    float2 jb[N + 1];  // j b_j, j >= 2
  };
  struct Acc {
    float2 a[M + 1], b[N];
    __device__ __forceinline__ void zero() {
#pragma unroll
      for (int i = 0; i <= M; ++i) a[i] = make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < N; ++j) b[j] = make_float2(0.f, 0.f);
    }
  };
  __device__ static __forceinline__ void assign(const float (&v)[TF], Coef& c) {
    int o = 0;
#pragma unroll
    for (int i = 0; i <= M; ++i) c.a[i] = f2(v[o++]);
#pragma unroll
    for (int i = 2; i <= M; ++i) c.ia[i] = f2(v[o++]);
#pragma unroll
    for (int j = 1; j <= N; ++j) c.b[j] = f2(v[o++]);
#pragma unroll
    for (int j = 2; j <= N; ++j) c.jb[j] = f2(v[o++]);
  }
  __device__ static __forceinline__ float2 fwd(const Coef& c, float2 x) {
    float2 P = c.a[M];
#pragma unroll
    for (int i = M - 1; i >= 0; --i) P = fma2(P, x, c.a[i]);
    float2 q = c.b[N];
#pragma unroll
    for (int j = N - 1; j >= 1; --j) q = fma2(q, x, c.b[j]);
    const float2 Q = mul2(q, x);
    const float2 r = make_float2(rcp_approx(1.f + fabsf(Q.x)), rcp_approx(1.f + fabsf(Q.y)));
    return mul2(P, r);
  }
  __device__ static __forceinline__ float2 bwd(const Coef& c, float2 x, float2 dy, Acc& acc,
                                               float2* y_out) {
    constexpr int KP = M > N ? M : N;
    float2 p[KP + 1];  // p[k] = x^k
    p[1] = x;
#pragma unroll
    for (int k = 2; k <= KP; ++k) p[k] = mul2(p[k / 2], p[k - k / 2]);
    float2 P = fma2(c.a[1], x, c.a[0]);
#pragma unroll
    for (int i = 2; i <= M; ++i) P = fma2(c.a[i], p[i], P);
    float2 dP = c.a[1];
#pragma unroll
    for (int i = 2; i <= M; ++i) dP = fma2(c.ia[i], p[i - 1], dP);
    float2 Q = mul2(c.b[1], x);
#pragma unroll
    for (int j = 2; j <= N; ++j) Q = fma2(c.b[j], p[j], Q);
    float2 dQ = c.b[1];
#pragma unroll
    for (int j = 2; j <= N; ++j) dQ = fma2(c.jb[j], p[j - 1], dQ);
    const float2 r = make_float2(rcp_approx(1.f + fabsf(Q.x)), rcp_approx(1.f + fabsf(Q.y)));
    const float2 y = mul2(P, r);
    if (y_out) *y_out = y;
    const float2 t = mul2(dy, r);
    const float2 nu = mul2(t, make_float2(neg_y_sign(y.x, Q.x), neg_y_sign(y.y, Q.y)));
    acc.a[0] = add2(acc.a[0], t);
#pragma unroll
    for (int i = 1; i <= M; ++i) acc.a[i] = fma2(t, p[i], acc.a[i]);
#pragma unroll
    for (int j = 1; j <= N; ++j) acc.b[j - 1] = fma2(nu, p[j], acc.b[j - 1]);
    return fma2(nu, dQ, mul2(t, dP));
  }
  template <int NS>
  __device__ static __forceinline__ void sums(const Acc& acc, float (&v)[NS]) {
#pragma unroll
    for (int i = 0; i <= M; ++i) v[i] = acc.a[i].x + acc.a[i].y;
#pragma unroll
    for (int j = 0; j < N; ++j) v[M + 1 + j] = acc.b[j].x + acc.b[j].y;
#pragma unroll
    for (int k = K; k < NS; ++k) v[k] = 0.f;
  }
};

template <>
struct Deg<5, 4> {
  static constexpr int K = 10;
  static constexpr int TF = tab_floats<5, 4>();
  using Coef = Coef54;
  using Acc = Acc54;
  __device__ static __forceinline__ void assign(const float (&v)[TF], Coef54& c) {
    c.a0 = f2(v[0]); c.a1 = f2(v[1]); c.a2 = f2(v[2]); c.a3 = f2(v[3]);
    c.a4 = f2(v[4]); c.a5 = f2(v[5]); c.ia2 = f2(v[6]); c.ia3 = f2(v[7]);
    c.ia4 = f2(v[8]); c.ia5 = f2(v[9]); c.b1 = f2(v[10]); c.b2 = f2(v[11]);
    c.b3 = f2(v[12]); c.b4 = f2(v[13]); c.jb2 = f2(v[14]); c.jb3 = f2(v[15]);
    c.jb4 = f2(v[16]);
  }
  __device__ static __forceinline__ float2 fwd(const Coef54& c, float2 x) { return fwd_pair(c, x); }
  __device__ static __forceinline__ float2 bwd(const Coef54& c, float2 x, float2 dy, Acc54& acc,
                                               float2* y_out) {
    return bwd_pair(c, x, dy, acc, y_out);
  }
  template <int NS>
  __device__ static __forceinline__ void sums(const Acc54& acc, float (&v)[NS]) {
    v[0] = acc.a0.x + acc.a0.y;
    v[1] = acc.a1.x + acc.a1.y;
    v[2] = acc.a2.x + acc.a2.y;
    v[3] = acc.a3.x + acc.a3.y;
    v[4] = acc.a4.x + acc.a4.y;
    v[5] = acc.a5.x + acc.a5.y;
    v[6] = acc.b1.x + acc.b1.y;
    v[7] = acc.b2.x + acc.b2.y;
    v[8] = acc.b3.x + acc.b3.y;
    v[9] = acc.b4.x + acc.b4.y;
#pragma unroll
    for (int k = 10; k < NS; ++k) v[k] = 0.f;
  }
};

// Coefficients of every group in the CTA's shared memory after the warps'
// regions (tab_floats per group), used when n_g <= kTableGroups; with more
// groups every lane reads its group's entries from global memory (broadcast
// loads). Scalars, not pairs: a pair built in registers from one scalar lets the
// compiler keep one register per coefficient.
constexpr int kTableGroups = 64;
template <int M, int N>
__host__ __device__ constexpr unsigned coef_table_bytes() {
  return (unsigned)(kTableGroups * tab_floats<M, N>() * 4);
}

template <int M, int N>
__device__ __forceinline__ void build_coef_table(float* tab, const float* a, const float* b,
                                                 int n_g) {
  constexpr int TF = tab_floats<M, N>();
  for (int e = threadIdx.x; e < n_g * TF; e += blockDim.x) {
    const int g = e / TF;
    tab[e] = coef_value<M, N>(a, b, g, e - g * TF);
  }
}

template <int M, int N>
__device__ __forceinline__ void load_coef(bool use_tab, const float* tab, const float* a,
                                          const float* b, int g, typename Deg<M, N>::Coef& c) {
  using D = Deg<M, N>;
  float v[D::TF];
  if (use_tab) {
    const float4* q = reinterpret_cast<const float4*>(tab + g * D::TF);
#pragma unroll
    for (int k = 0; k < D::TF / 4; ++k) {
      const float4 w = q[k];
      v[4 * k] = w.x;
      v[4 * k + 1] = w.y;
      v[4 * k + 2] = w.z;
      v[4 * k + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < D::TF; ++k) v[k] = coef_value<M, N>(a, b, g, k);
  }
  D::assign(v, c);
}

// --- per-warp pipeline geometry ----------------------------------------------------
//
// Every warp runs its own pipeline: it owns kStages stage slots in shared
// memory, each holding one TMA box (SCw rows x bw channels) of every input
// tensor, and its own full / empty mbarriers. Nothing couples the warps of a
// CTA after initialisation, so they drift out of phase and one warp's loads
// and reductions overlap another's arithmetic.

// Per-warp shared memory: [stages][tensors][box, 128-byte rounded], then the
// 8-byte barriers.
struct WarpLayout {
  unsigned box_slot;   // bytes of one box slot
  unsigned stage;      // bytes of one stage (all tensors)
  unsigned out_off;    // output staging slots (boxes written back by TMA stores)
  unsigned bar_off;    // full[stages] then empty[stages]
  unsigned per_warp;   // bytes per warp (multiple of 128)
  __host__ __device__ WarpLayout(unsigned box_bytes, int tensors, int stages, int outs = 0) {
    box_slot = round_up(box_bytes, 128);
    stage = box_slot * (unsigned)tensors;
    out_off = stage * (unsigned)stages;
    bar_off = out_off + box_slot * (unsigned)outs;
    per_warp = round_up(bar_off + (unsigned)(2 * stages) * 8, 128);
  }
};

// Where the vectors a lane owns in every box go in global memory: vector v of
// the box (16 bytes) is row v / vpr, vector column v % vpr; off = element
// offset from the box origin, row = row in the box (huge for unused slots).
template <class IO, int NV>
struct LaneMap {
  int off[NV];
  int row[NV];
  __device__ __forceinline__ void init(const TmaGeom& g, int lane, long long d) {
    constexpr int ve = 16 / IO::kBytes;  // elements per vector
    const int vpr = g.bw / ve;
    const int nvec = (int)(g.box_bytes / 16);
#pragma unroll
    for (int it = 0; it < NV; ++it) {
      const int v = lane + it * 32;
      if (v < nvec) {
        const int r = v / vpr;
        row[it] = r;
        off[it] = (int)((long long)r * d) + (v - r * vpr) * ve;
      } else {
        row[it] = 0x3fffffff;
        off[it] = 0;
      }
    }
  }
};

__device__ __forceinline__ void store16(void* p, uint4 v) {
  __stcs(reinterpret_cast<uint4*>(p), v);
}

// Sum NS (16 or 32) per-lane values over the warp in a fixed order.
// Recursive halving: at each step a lane keeps half of its values (those of its
// own half of the index range) and adds the partner's. Afterwards lane l holds
// in v[0] the sum of value (l >> 1) & 15 (NS = 16: the last step adds the two
// lanes of a pair) or of value l (NS = 32).
template <int NS>
__device__ __forceinline__ void warp_sum(float (&v)[NS], int lane) {
  static_assert(NS == 16 || NS == 32, "16 or 32 slots");
  constexpr int kSteps = NS == 16 ? 4 : 5;
#pragma unroll
  for (int step = 0; step < kSteps; ++step) {
    const int half = (NS / 2) >> step;  // values kept after this step
    const int mask = 16 >> step;        // partner distance
    const bool upper = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float recv = __shfl_xor_sync(0xffffffffu, send, mask);
      v[i] = (upper ? v[i + half] : v[i]) + recv;
    }
  }
  if constexpr (NS == 16) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// Mixed-radix counter (hi, mid, lo) with radices (unbounded, nmid, nlo), stepped
// by a fixed stride without any division in the loop.
struct Cursor3 {
  long long hi;
  int mid, lo;
  long long s_hi;
  int s_mid, s_lo, nmid, nlo;
  __device__ __forceinline__ void init(long long first, long long stride, int nmid_, int nlo_) {
    nmid = nmid_;
    nlo = nlo_;
    const long long per = (long long)nmid * nlo;
    hi = first / per;
    const int r = (int)(first - hi * per);
    mid = r / nlo;
    lo = r - mid * nlo;
    s_hi = stride / per;
    const int sr = (int)(stride - s_hi * per);
    s_mid = sr / nlo;
    s_lo = sr - s_mid * nlo;
  }
  __device__ __forceinline__ void next() {
    lo += s_lo;
    int carry = lo >= nlo;
    lo -= carry ? nlo : 0;
    mid += s_mid + carry;
    carry = mid >= nmid;
    mid -= carry ? nmid : 0;
    hi += s_hi + carry;
  }
};

// --- forward -------------------------------------------------------------------------
// Work items are boxes (row block, group, column box), taken by warp gw of the
// grid (numbered warp-major) as item gw, gw + total warps, ... in
// row-block-major order.


template <class IO, int M, int N>
__global__ void __launch_bounds__(kFwdThreads, 1)
fwd_tma(const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap my,
        typename IO::T* __restrict__ y,
        const float* __restrict__ a, const float* __restrict__ b, const TmaGeom geom) {
  using S_ = Shape<IO>;
  using D = Deg<M, N>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const WarpLayout L(geom.box_bytes, 1, S_::kFwdStages, S_::kFwdStore == 2 ? 1 : 0);
  unsigned char* base = smem + warp * L.per_warp;
  float* ctab = reinterpret_cast<float*>(smem + kFwdWarps * L.per_warp);
  const bool use_tab = geom.n_g <= kTableGroups;
  const uint32_t full0 = smem_addr(base + L.bar_off);
  const uint32_t empty0 = full0 + 8 * S_::kFwdStages;
  const long long row_blocks = (geom.rows + geom.SCw - 1) / geom.SCw;
  // warp-major numbering: consecutive work items go to different SMs, so the
  // items left over after whole rounds spread over every SM instead of
  // filling the first SMs' warps
  const long long gw = (long long)warp * gridDim.x + blockIdx.x;
  const long long GW = (long long)gridDim.x * kFwdWarps;

  if (lane == 0) {
    for (int s = 0; s < S_::kFwdStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
    if (warp == 0) {
      prefetch_map(&mx);
      if (S_::kFwdStore == 2) prefetch_map(&my);
    }
  }
  if (use_tab) build_coef_table<M, N>(ctab, a, b, geom.n_g);
  __syncthreads();

  Cursor3 ic;  // issue cursor (lane 0): (row block, group, box)
  ic.init(gw, GW, geom.n_g, geom.nbox);
  int iq = 0;
  auto issue = [&]() {
    const int s = iq % S_::kFwdStages;
    mbar_arrive_expect_tx(full0 + 8 * s, geom.box_bytes);
    tma_load_2d(smem_addr(base + s * L.stage), &mx, ic.mid * geom.dg + ic.lo * geom.bw,
                (int)(ic.hi * geom.SCw), full0 + 8 * s);
    ic.next();
    ++iq;
  };
  if (lane == 0)
    for (int s = 0; s < S_::kFwdStages && ic.hi < row_blocks; ++s) issue();
  __syncwarp();

  LaneMap<IO, S_::kFwdVec> lm;
  lm.init(geom, lane, geom.d);
  typename D::Coef c;
  int cur_g = -1;
  bool ok = true;
  int q = 0;
  Cursor3 cc;  // consumer cursor
  cc.init(gw, GW, geom.n_g, geom.nbox);
  for (; cc.hi < row_blocks; cc.next(), ++q) {
    const int s = q % S_::kFwdStages;
    const uint32_t ph = (uint32_t)(q / S_::kFwdStages) & 1;
    if (!mbar_wait(full0 + 8 * s, ph)) {
      report(kErrFullWait);
      ok = false;
      break;
    }
    const int g = cc.mid;
    if (g != cur_g) {
      load_coef<M, N>(use_tab, ctab, a, b, g, c);
      cur_g = g;
    }
    const uint4* buf = reinterpret_cast<const uint4*>(base + s * L.stage);
    uint4 v[S_::kFwdVec];
#pragma unroll
    for (int it = 0; it < S_::kFwdVec; ++it)  // slots past the box: zeros, never stored
      v[it] = lm.row[it] < geom.SCw ? buf[lane + 32 * it] : make_uint4(0u, 0u, 0u, 0u);
    // release the slot and refill it with the item S_::kFwdStages ahead
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(empty0 + 8 * s);
      if (ic.hi < row_blocks) {
        if (!mbar_wait(empty0 + 8 * s, ph)) {
          report(kErrEmptyWait);
          ok = false;
        } else {
          issue();
        }
      }
    }
    const long long row0 = cc.hi * geom.SCw;
    typename IO::T* yo = y + row0 * geom.d + (g * geom.dg + cc.lo * geom.bw);
    auto fwd_vec = [&](const uint4& xv) {
      uint4 o;
      if constexpr (IO::kBytes == 2) {
        o.x = f2_to_bf16x2(D::fwd(c, bf16x2_to_f2(xv.x)));
        o.y = f2_to_bf16x2(D::fwd(c, bf16x2_to_f2(xv.y)));
        o.z = f2_to_bf16x2(D::fwd(c, bf16x2_to_f2(xv.z)));
        o.w = f2_to_bf16x2(D::fwd(c, bf16x2_to_f2(xv.w)));
      } else {
        const float2 p0 = D::fwd(c, make_float2(__uint_as_float(xv.x), __uint_as_float(xv.y)));
        const float2 p1 = D::fwd(c, make_float2(__uint_as_float(xv.z), __uint_as_float(xv.w)));
        o = make_uint4(__float_as_uint(p0.x), __float_as_uint(p0.y), __float_as_uint(p1.x),
                       __float_as_uint(p1.y));
      }
      return o;
    };
    if constexpr (S_::kFwdStore == 0) {
#pragma unroll
      for (int it = 0; it < S_::kFwdVec; ++it)
        if (row0 + lm.row[it] < geom.rows) store16(yo + lm.off[it], fwd_vec(v[it]));
    } else if constexpr (S_::kFwdStore == 1) {
      // every vector's values first (rows past the tensor arrive zero-filled),
      // then the guarded stores: the arithmetic stays one basic block
      uint4 o[S_::kFwdVec];
#pragma unroll
      for (int it = 0; it < S_::kFwdVec; ++it) o[it] = fwd_vec(v[it]);
#pragma unroll
      for (int it = 0; it < S_::kFwdVec; ++it)
        if (row0 + lm.row[it] < geom.rows) store16(yo + lm.off[it], o[it]);
    } else {
      // staged in the warp's output slot, written by one TMA store (clipped rows)
      uint4 o[S_::kFwdVec];
#pragma unroll
      for (int it = 0; it < S_::kFwdVec; ++it) o[it] = fwd_vec(v[it]);
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      uint4* outs = reinterpret_cast<uint4*>(base + L.out_off) + lane;
#pragma unroll
      for (int it = 0; it < S_::kFwdVec; ++it)
        if (lm.row[it] < geom.SCw) outs[32 * it] = o[it];
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&my, g * geom.dg + cc.lo * geom.bw, (int)row0, smem_addr(base + L.out_off));
        bulk_commit();
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
    if (!ok) break;
  }
  if (!ok && lane == 0) {
    // wind down: let every issued load land before the CTA's memory goes away
    for (int j = q; j < iq; ++j)
      if (!mbar_wait(full0 + 8 * (j % S_::kFwdStages), (uint32_t)(j / S_::kFwdStages) & 1))
        report(kErrDrainWait);
  }
  if (S_::kFwdStore == 2 && lane == 0) bulk_wait_all();  // stores done before the CTA ends
}

// --- backward ------------------------------------------------------------------------
// Units (tile, g) (tile = S rows) are taken by warp gw of the grid (numbered
// warp-major, gw = warp * grid + CTA) as unit gw, gw + total warps, ... in
// tile-major order; a unit's boxes are its row blocks (SCw rows) times the
// group's column boxes. The partial sum of unit (tile, g), coefficient k goes to
// ws[(g * K + k) * ws_T + ws_tile0 + tile], K = m + 1 + n.


// Row blocks of tile `tile`: ceil(min(S, rows - tile * S) / SCw); only the last
// tile can be short.
__device__ __forceinline__ int tile_row_blocks(const TmaGeom& g, long long tile) {
  return tile == g.T - 1 ? g.nrb_last : g.nrb_full;
}

// kWithY: also write y (the forward output recomputed on the way), for
// training that recomputes the activation during the backward pass.
// kFull: every 16-byte vector slot of a lane holds box data (the box is exactly
// 32 * NV vectors), so the loads need no guard.
template <class IO, int M, int N, bool kWithY, bool kFull>
__global__ void __launch_bounds__(Shape<IO>::kBwdWarps * 32, 1)
bwd_tma(const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mdy,
        const __grid_constant__ CUtensorMap mdx,
        typename IO::T* __restrict__ dx, typename IO::T* __restrict__ yout,
        const float* __restrict__ a,
        const float* __restrict__ b, float* __restrict__ ws, const TmaGeom geom) {
  using S_ = Shape<IO>;
  using T = typename IO::T;
  using D = Deg<M, N>;
  constexpr int NV = S_::kBwdVec * S_::kBwdHalves;  // 16-byte vectors per lane in a box
  // vectors per pass: fewer for high degrees, whose per-pair state is larger
  constexpr int kBwdVec = (M + N > 9) ? 1 : S_::kBwdVec;
  constexpr int kPasses = NV / kBwdVec;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  constexpr bool kTmaOut = S_::kBwdStore == 2;  // dx leaves through a staging slot and TMA
  const WarpLayout L(geom.box_bytes, 2, S_::kBwdStages, kTmaOut ? 1 : 0);
  unsigned char* base = smem + warp * L.per_warp;
  float* ctab = reinterpret_cast<float*>(smem + S_::kBwdWarps * L.per_warp);
  const bool use_tab = geom.n_g <= kTableGroups;
  const uint32_t full0 = smem_addr(base + L.bar_off);
  const uint32_t empty0 = full0 + 8 * S_::kBwdStages;
  // warp-major numbering: consecutive work items go to different SMs, so the
  // items left over after whole rounds spread over every SM instead of
  // filling the first SMs' warps
  const long long gw = (long long)warp * gridDim.x + blockIdx.x;
  const long long GW = (long long)gridDim.x * S_::kBwdWarps;

  if (lane == 0) {
    for (int s = 0; s < S_::kBwdStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
    if (warp == 0) {
      prefetch_map(&mx);
      prefetch_map(&mdy);
      if (kTmaOut) prefetch_map(&mdx);
    }
  }
  if (use_tab) build_coef_table<M, N>(ctab, a, b, geom.n_g);
  __syncthreads();

  // issue cursor (lane 0): unit (tile, g) = iu.hi, iu.lo; box (irb, ibx) of inrb
  // row blocks; the box origin (icol, irow) and the ring slot advance by addition
  Cursor3 iu;
  iu.init(gw, GW, 1, geom.n_g);
  int irb = 0, ibx = 0, inrb = 0, icol = 0, irow = 0, islot = 0;
  int iq = 0;
  auto unit_start = [&]() {
    if (iu.hi < geom.T) {
      inrb = tile_row_blocks(geom, iu.hi);
      icol = iu.lo * geom.dg;
      irow = (int)(iu.hi * geom.S);
    } else {
      inrb = 0;
    }
  };
  unit_start();
  const uint32_t stage0 = smem_addr(base);
  const uint32_t tx_bytes = 2u * geom.box_bytes;
  auto issue = [&]() {
    const uint32_t bar = full0 + 8u * (uint32_t)islot;
    const uint32_t dst = stage0 + (uint32_t)islot * L.stage;
    mbar_arrive_expect_tx(bar, tx_bytes);
    tma_load_2d(dst, &mx, icol, irow, bar);
    tma_load_2d(dst + L.box_slot, &mdy, icol, irow, bar);
    ++iq;
    islot = (islot + 1 == S_::kBwdStages) ? 0 : islot + 1;
    icol += geom.bw;
    if (++ibx == geom.nbox) {
      ibx = 0;
      icol -= geom.dg;  // nbox * bw == dg: back to the group's first column
      irow += geom.SCw;
      if (++irb == inrb) {
        irb = 0;
        iu.next();
        unit_start();
      }
    }
  };
  if (lane == 0)
    for (int s = 0; s < S_::kBwdStages && iu.hi < geom.T; ++s) issue();
  __syncwarp();

  // per-lane byte offsets of the lane's vectors from a box's origin in global memory
  LaneMap<IO, NV> lm;
  lm.init(geom, lane, geom.d);
  int boff[NV];
#pragma unroll
  for (int sl = 0; sl < NV; ++sl) boff[sl] = lm.off[sl] * (int)sizeof(T);
  const long long row_bytes = geom.d * (long long)sizeof(T);
  typename D::Coef c;
  int cur_g = -1;
  typename D::Acc acc;
  bool ok = true;
  int q = 0, rslot = 0;  // boxes consumed; ring slot and phase of the next one
  uint32_t rphase = 0;
  Cursor3 cu;
  cu.init(gw, GW, 1, geom.n_g);
  for (; cu.hi < geom.T && ok; cu.next()) {
    const long long tile = cu.hi;
    const int g = cu.lo;
    const int nrb = tile_row_blocks(geom, tile);
    if (g != cur_g) {
      load_coef<M, N>(use_tab, ctab, a, b, g, c);
      cur_g = g;
    }
    acc.zero();
    const long long left = geom.rows - tile * geom.S;
    const int rows_left = left < geom.S ? (int)left : (int)geom.S;
    const long long tile_off = (tile * geom.S * geom.d + (long long)g * geom.dg) * sizeof(T);
    char* dxt = reinterpret_cast<char*>(dx) + tile_off;
    char* yt = kWithY ? reinterpret_cast<char*>(yout) + tile_off : nullptr;
    for (int rb = 0; rb < nrb && ok; ++rb) {
      const int r0 = rb * geom.SCw;     // row of the box within the tile
      const int lim = rows_left - r0;   // lane vectors in rows >= lim are past the end
      for (int bx = 0; bx < geom.nbox; ++bx, ++q) {
        const int s = rslot;
        const uint32_t ph = rphase;
        if (++rslot == S_::kBwdStages) {
          rslot = 0;
          rphase ^= 1u;
        }
        if (!mbar_wait(full0 + 8 * s, ph)) {
          report(kErrFullWait);
          ok = false;
          break;
        }
        const uint4* xl = reinterpret_cast<const uint4*>(base + s * L.stage) + lane;
        const uint4* gl = reinterpret_cast<const uint4*>(base + s * L.stage + L.box_slot) + lane;
        const long long box_off = (long long)r0 * row_bytes + (long long)bx * geom.bw * sizeof(T);
        char* dxo = dxt + box_off;
        char* yo = kWithY ? yt + box_off : nullptr;
        uint4* outs = reinterpret_cast<uint4*>(base + L.out_off) + lane;  // staging (kTmaOut)
#pragma unroll
        for (int h = 0; h < kPasses; ++h) {
          uint4 xv[kBwdVec], gv[kBwdVec];
#pragma unroll
          for (int it = 0; it < kBwdVec; ++it) {
            const int sl = h * kBwdVec + it;
            if (kFull || lm.row[sl] < geom.SCw) {
              xv[it] = xl[32 * sl];
              gv[it] = gl[32 * sl];
            } else {
              xv[it] = make_uint4(0, 0, 0, 0);
              gv[it] = make_uint4(0, 0, 0, 0);
            }
          }
          if (h == kPasses - 1) {
            // release the slot (every lane has read it) and refill it
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(empty0 + 8 * s);
              if (iu.hi < geom.T) {
                if (!mbar_wait(empty0 + 8 * s, ph)) {
                  report(kErrEmptyWait);
                  ok = false;
                } else {
                  issue();
                }
              }
            }
          }
          uint4 ov[kBwdVec], oyv[kBwdVec];
#pragma unroll
          for (int it = 0; it < kBwdVec; ++it) {
            const int sl = h * kBwdVec + it;
            // rows past the end arrive zero-filled from TMA: they add exact
            // zeros to the sums and are not stored
            uint4 o, oy;
            float2 y0, y1, y2, y3;
            if constexpr (IO::kBytes == 2) {
              o.x = f2_to_bf16x2(
                  D::bwd(c, bf16x2_to_f2(xv[it].x), bf16x2_to_f2(gv[it].x), acc, kWithY ? &y0 : nullptr));
              o.y = f2_to_bf16x2(
                  D::bwd(c, bf16x2_to_f2(xv[it].y), bf16x2_to_f2(gv[it].y), acc, kWithY ? &y1 : nullptr));
              o.z = f2_to_bf16x2(
                  D::bwd(c, bf16x2_to_f2(xv[it].z), bf16x2_to_f2(gv[it].z), acc, kWithY ? &y2 : nullptr));
              o.w = f2_to_bf16x2(
                  D::bwd(c, bf16x2_to_f2(xv[it].w), bf16x2_to_f2(gv[it].w), acc, kWithY ? &y3 : nullptr));
              if constexpr (kWithY)
                oy = make_uint4(f2_to_bf16x2(y0), f2_to_bf16x2(y1), f2_to_bf16x2(y2),
                                f2_to_bf16x2(y3));
            } else {
              const float2 p0 = D::bwd(
                  c, make_float2(__uint_as_float(xv[it].x), __uint_as_float(xv[it].y)),
                  make_float2(__uint_as_float(gv[it].x), __uint_as_float(gv[it].y)), acc,
                  kWithY ? &y0 : nullptr);
              const float2 p1 = D::bwd(
                  c, make_float2(__uint_as_float(xv[it].z), __uint_as_float(xv[it].w)),
                  make_float2(__uint_as_float(gv[it].z), __uint_as_float(gv[it].w)), acc,
                  kWithY ? &y1 : nullptr);
              o = make_uint4(__float_as_uint(p0.x), __float_as_uint(p0.y), __float_as_uint(p1.x),
                             __float_as_uint(p1.y));
              if constexpr (kWithY)
                oy = make_uint4(__float_as_uint(y0.x), __float_as_uint(y0.y),
                                __float_as_uint(y1.x), __float_as_uint(y1.y));
            }
            ov[it] = o;
            if constexpr (kWithY) oyv[it] = oy;
          }
          if constexpr (kTmaOut) {
            // the slot is free once the previous box's store has read it
            if (h == 0) {
              if (lane == 0) bulk_wait_read_all();
              __syncwarp();
            }
#pragma unroll
            for (int it = 0; it < kBwdVec; ++it) {
              const int sl = h * kBwdVec + it;
              if (kFull || lm.row[sl] < geom.SCw) outs[32 * sl] = ov[it];
              if constexpr (kWithY)
                if (lm.row[sl] < lim) store16(yo + boff[sl], oyv[it]);
            }
          } else {
#pragma unroll
            for (int it = 0; it < kBwdVec; ++it) {
              const int sl = h * kBwdVec + it;
              if (lm.row[sl] < lim) {
                store16(dxo + boff[sl], ov[it]);
                if constexpr (kWithY) store16(yo + boff[sl], oyv[it]);
              }
            }
          }
        }
        if constexpr (kTmaOut) {
          // the lanes' shared-memory writes become visible to the async proxy,
          // then one store writes the box (rows past the tensor are clipped)
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&mdx, g * geom.dg + bx * geom.bw, (int)(tile * geom.S) + r0,
                         smem_addr(base + L.out_off));
            bulk_commit();
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
        if (!ok) break;
      }
    }
    if (!ok) break;
    // Unit reduction, fixed order: the two lanes of each pair, then a
    // recursive-halving exchange over the warp.
    constexpr int NS = D::K <= 16 ? 16 : 32;
    float v[NS];
    D::template sums<NS>(acc, v);
    warp_sum<NS>(v, lane);
    const int k = NS == 16 ? ((lane >> 1) & 15) : lane;
    if ((NS == 32 || (lane & 1) == 0) && k < D::K)
      ws[((long long)g * D::K + k) * geom.ws_T + geom.ws_tile0 + tile] = v[0];
  }
  if (!ok && lane == 0) {
    for (int j = q; j < iq; ++j)
      if (!mbar_wait(full0 + 8 * (j % S_::kBwdStages), (uint32_t)(j / S_::kBwdStages) & 1))
        report(kErrDrainWait);
  }
  if (kTmaOut && lane == 0) bulk_wait_all();  // stores done before the CTA's memory goes
}

// --- host-side launchers ---------------------------------------------------------

// Raise a kernel's dynamic shared-memory limit to what it uses and ask for the
// largest shared-memory carveout; once per kernel and device (the cache is keyed
// on the kernel itself).
template <auto Kernel>
inline cudaError_t ensure_smem(unsigned bytes) {
  static std::atomic<unsigned long long> done_devices{0};  // bit d: set on device d
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done_devices.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const void* fn = reinterpret_cast<const void*>(Kernel);
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && bit) done_devices.fetch_or(bit, std::memory_order_release);
  return e;
}

// Shared memory of a launch: one region per warp for the largest box, then
// the coefficient table.
template <class IO, int M, int N>
inline unsigned fwd_smem_bytes() {
  return kFwdWarps *
             WarpLayout(fwd_box_bytes<IO>(), 1, Shape<IO>::kFwdStages,
                        Shape<IO>::kFwdStore == 2 ? 1 : 0)
                 .per_warp +
         coef_table_bytes<M, N>();
}
template <class IO, int M, int N>
inline unsigned bwd_smem_bytes() {
  return Shape<IO>::kBwdWarps *
             WarpLayout(bwd_box_bytes<IO>(), 2, Shape<IO>::kBwdStages,
                        Shape<IO>::kBwdStore == 2 ? 1 : 0)
                 .per_warp +
         coef_table_bytes<M, N>();
}

template <class IO, int M, int N>
inline cudaError_t launch_fwd_tma_t(const TmaGeom& g, const CUtensorMap& mx,
                                    const CUtensorMap& my, void* y, const float* a,
                                    const float* b, long long grid, cudaStream_t st) {
  const unsigned smem = fwd_smem_bytes<IO, M, N>();
  cudaError_t e = ensure_smem<fwd_tma<IO, M, N>>(smem);
  if (e != cudaSuccess) return e;
  fwd_tma<IO, M, N><<<(unsigned)grid, kFwdThreads, smem, st>>>(mx, my, (typename IO::T*)y, a, b,
                                                                g);
  return cudaGetLastError();
}

// my maps y with the forward box (used when y is written by TMA stores).
inline cudaError_t launch_fwd_tma(bool bf16, const TmaGeom& g, const CUtensorMap& mx,
                                  const CUtensorMap& my, void* y, const float* a,
                                  const float* b, int sms, cudaStream_t st) {
  if (g.box_bytes > fwd_box_target(bf16)) return cudaErrorInvalidValue;
  const long long items = ((g.rows + g.SCw - 1) / g.SCw) * g.n_g * g.nbox;
  long long grid = sms;
  if (grid * kFwdWarps > items) grid = (items + kFwdWarps - 1) / kFwdWarps;
#define GRK_FWD_CASE(M, N)                                                          \
  if (g.m == M && g.n == N)                                                         \
    return bf16 ? launch_fwd_tma_t<IoBF16, M, N>(g, mx, my, y, a, b, grid, st)      \
                : launch_fwd_tma_t<IoF32, M, N>(g, mx, my, y, a, b, grid, st);
  GRK_TMA_DEGREES(GRK_FWD_CASE)
#undef GRK_FWD_CASE
  return cudaErrorNotSupported;
}

template <class IO, int M, int N, bool kWithY, bool kFull>
inline cudaError_t launch_bwd_tma_t(const TmaGeom& g, const CUtensorMap& mx,
                                    const CUtensorMap& mdy, const CUtensorMap& mdx, void* dx,
                                    void* y, const float* a, const float* b, float* ws,
                                    long long grid, cudaStream_t st) {
  const unsigned smem = bwd_smem_bytes<IO, M, N>();
  cudaError_t e = ensure_smem<bwd_tma<IO, M, N, kWithY, kFull>>(smem);
  if (e != cudaSuccess) return e;
  bwd_tma<IO, M, N, kWithY, kFull><<<(unsigned)grid, Shape<IO>::kBwdWarps * 32, smem, st>>>(
      mx, mdy, mdx, (typename IO::T*)dx, (typename IO::T*)y, a, b, ws, g);
  return cudaGetLastError();
}

template <class IO, int M, int N>
inline cudaError_t launch_bwd_tma_io(const TmaGeom& g, const CUtensorMap& mx,
                                     const CUtensorMap& mdy, const CUtensorMap& mdx, void* dx,
                                     void* y, const float* a, const float* b, float* ws,
                                     long long grid, cudaStream_t st) {
  // every lane vector slot used: the box is exactly 32 lanes x NV vectors
  const bool full = g.box_bytes == bwd_box_bytes<IO>();
  if (y) {
    if constexpr (M == 5 && N == 4) {
      return full ? launch_bwd_tma_t<IO, M, N, true, true>(g, mx, mdy, mdx, dx, y, a, b, ws, grid,
                                                            st)
                  : launch_bwd_tma_t<IO, M, N, true, false>(g, mx, mdy, mdx, dx, y, a, b, ws,
                                                             grid, st);
    } else {
      return cudaErrorNotSupported;
    }
  }
  return full ? launch_bwd_tma_t<IO, M, N, false, true>(g, mx, mdy, mdx, dx, y, a, b, ws, grid, st)
              : launch_bwd_tma_t<IO, M, N, false, false>(g, mx, mdy, mdx, dx, y, a, b, ws, grid,
                                                          st);
}

// y == nullptr: backward only; otherwise also write the recomputed forward y
// (degree (5, 4) only). mdx maps dx with the backward box (used when dx is
// written by TMA stores).
inline cudaError_t launch_bwd_tma(bool bf16, const TmaGeom& g, const CUtensorMap& mx,
                                  const CUtensorMap& mdy, const CUtensorMap& mdx, void* dx,
                                  void* y, const float* a, const float* b, float* ws, int sms,
                                  cudaStream_t st) {
  if (g.box_bytes > bwd_box_target(bf16)) return cudaErrorInvalidValue;
  const long long units = g.T * g.n_g;
  const int warps = bf16 ? Shape<IoBF16>::kBwdWarps : Shape<IoF32>::kBwdWarps;
  long long grid = sms;
  if (grid * warps > units) grid = (units + warps - 1) / warps;
#define GRK_BWD_CASE(M, N)                                                                   \
  if (g.m == M && g.n == N)                                                                  \
    return bf16 ? launch_bwd_tma_io<IoBF16, M, N>(g, mx, mdy, mdx, dx, y, a, b, ws, grid, st) \
                : launch_bwd_tma_io<IoF32, M, N>(g, mx, mdy, mdx, dx, y, a, b, ws, grid, st);
  GRK_TMA_DEGREES(GRK_BWD_CASE)
#undef GRK_BWD_CASE
  return cudaErrorNotSupported;
}

// One warp waits on an mbarrier phase that nothing completes, with the same
// bounded wait as the pipelined kernels and a short limit: the wait runs out,
// the kernel records kErrSelfTest and returns, and the context stays usable.
__global__ void selftest_wait_timeout(unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const bool got = mbar_wait_for(b, 0, limit_ns);  // phase 0 never completes
  if (!__any_sync(0xffffffffu, got) && threadIdx.x == 0) report(kErrSelfTest);
}

inline cudaError_t read_device_error(uint32_t* out, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_grkan_device_error, sizeof(uint32_t), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

inline cudaError_t clear_device_error(cudaStream_t st) {
  static const uint32_t zero = 0;
  return cudaMemcpyToSymbolAsync(g_grkan_device_error, &zero, sizeof(uint32_t), 0,
                                 cudaMemcpyHostToDevice, st);
}

}  // namespace grk
