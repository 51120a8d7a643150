// grkan_tma.cuh -- persistent, TMA-pipelined forward and backward kernels.
//
// Work decomposition: (row tile x group) units as in the FlashKAT backward
// ("FlashKAT ...", paper notes, section "3. FlashKAT kernel restructuring
// (Algorithm 2)"), realised as a persistent grid of one 16-warp CTA per SM that
// walks the unit list in a fixed stride. A unit is split into chunks of SC rows
// x d_g channels (24 KiB of one tensor) that stream through a ring of shared-
// memory stages filled by 2-D TMA tile loads:
//   - thread 0 also acts as the issuer: it stages the group's coefficients in
//     the stage header and issues the loads, keeping the ring full by refilling
//     the stage of chunk q-1 (once every warp has read it) when it starts q;
//   - every warp reads its vectors of the chunk into registers, releases the
//     stage, evaluates the rational function on pairs of elements with packed
//     float32x2 arithmetic, and writes y or dx with 16-byte global stores;
//   - the backward keeps the ten coefficient-gradient sums in registers; at the
//     end of a unit they are folded in a fixed order through shared memory and
//     warp shuffles into one float32 partial per (unit, coefficient) in the
//     workspace -- no atomics (section "3. ...": accumulate inside the block,
//     one global write per block).
// Every wait is bounded: a wait that runs out records a code in
// g_grkan_device_error and the kernel winds down instead of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "grkan_common.cuh"

namespace grk {

struct TmaGeom {
  long long rows;       // B * N
  long long T;          // row tiles
  long long d;          // channels (row length)
  int dg;               // channels per group
  int n_g;              // groups
  int SC;               // rows per chunk (TMA box height)
  int chunks_per_unit;  // chunks per row tile
  int bw;               // TMA box width (channels)
  int nbox;             // boxes per chunk row = dg / bw
  unsigned chunk_bytes; // SC * dg * element size (one tensor)
  int m, n;             // degrees
};

// Launch shape (compile-time; the defaults are the tuned configuration).
#ifndef GRK_WARPS
#define GRK_WARPS 16
#endif
#ifndef GRK_FWD_STAGES
#define GRK_FWD_STAGES 8
#endif
#ifndef GRK_BWD_STAGES
#define GRK_BWD_STAGES 4
#endif
#ifndef GRK_CHUNK_BYTES
#define GRK_CHUNK_BYTES 24576
#endif

constexpr int kWarps = GRK_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kFwdStages = GRK_FWD_STAGES;
constexpr int kBwdStages = GRK_BWD_STAGES;
constexpr unsigned kMaxChunkBytes = GRK_CHUNK_BYTES;
constexpr int kVec = (int)((kMaxChunkBytes / 16 + kThreads - 1) / kThreads);  // vectors/thread
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;                 // 2 s

// Error codes written to g_grkan_device_error (bit-or).
constexpr unsigned kErrFullWait = 1u;
constexpr unsigned kErrEmptyWait = 2u;
constexpr unsigned kErrReduceWait = 4u;
constexpr unsigned kErrDrainWait = 8u;

__device__ unsigned int g_grkan_device_error = 0;

inline bool tma_has_degree(int m, int n) { return m == 5 && n == 4; }

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

// Wait for the phase with the given parity; false after kWaitTimeoutNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitTimeoutNs) return false;
  }
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
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

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
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

  __device__ __forceinline__ void set(const float* c) {  // c = a_0..a_5, b_1..b_4
    a0 = f2(c[0]); a1 = f2(c[1]); a2 = f2(c[2]); a3 = f2(c[3]); a4 = f2(c[4]); a5 = f2(c[5]);
    ia2 = f2(2.f * c[2]); ia3 = f2(3.f * c[3]); ia4 = f2(4.f * c[4]); ia5 = f2(5.f * c[5]);
    b1 = f2(c[6]); b2 = f2(c[7]); b3 = f2(c[8]); b4 = f2(c[9]);
    jb2 = f2(2.f * c[7]); jb3 = f2(3.f * c[8]); jb4 = f2(4.f * c[9]);
  }
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
__device__ __forceinline__ float2 bwd_pair(const Coef54& c, float2 x, float2 dy, Acc54& acc) {
  const float2 x2 = mul2(x, x);
  const float2 x3 = mul2(x2, x);
  const float2 x4 = mul2(x2, x2);
  const float2 x5 = mul2(x4, x);
  float2 P = fma2(c.a1, x, c.a0);
  P = fma2(c.a2, x2, P);
  P = fma2(c.a3, x3, P);
  P = fma2(c.a4, x4, P);
  P = fma2(c.a5, x5, P);
  float2 dP = fma2(c.ia2, x, c.a1);
  dP = fma2(c.ia3, x2, dP);
  dP = fma2(c.ia4, x3, dP);
  dP = fma2(c.ia5, x4, dP);
  float2 Q = mul2(c.b1, x);
  Q = fma2(c.b2, x2, Q);
  Q = fma2(c.b3, x3, Q);
  Q = fma2(c.b4, x4, Q);
  float2 dQ = fma2(c.jb2, x, c.b1);
  dQ = fma2(c.jb3, x2, dQ);
  dQ = fma2(c.jb4, x3, dQ);
  const float2 r = make_float2(rcp_approx(1.f + fabsf(Q.x)), rcp_approx(1.f + fabsf(Q.y)));
  const float2 y = mul2(P, r);
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

// --- shared-memory layout ------------------------------------------------------

constexpr int kCoefSlot = 16;  // floats per stage header (10 used)

__host__ __device__ constexpr unsigned round_up(unsigned v, unsigned a) {
  return (v + a - 1) / a * a;
}

// [stages x tensors x chunk] [stages x header coef] [full bars] [empty bars]
// [two reduction bars] [reduction buffer 10 x kThreads floats]
struct Layout {
  unsigned stage_stride;  // bytes of one stage (all tensors)
  unsigned coef_off, bar_off, red_off, total;
  __host__ __device__ Layout(unsigned chunk_bytes, int tensors, int stages, bool reduce) {
    const unsigned cb = round_up(chunk_bytes, 128);
    stage_stride = cb * (unsigned)tensors;
    coef_off = stage_stride * (unsigned)stages;
    bar_off = coef_off + (unsigned)(stages * kCoefSlot * 4);
    red_off = round_up(bar_off + (unsigned)(2 * stages + 2) * 8, 128);
    total = red_off + (reduce ? (unsigned)(10 * kThreads * 4) : 0u);
  }
};

// Chunks in unit (tile): ceil(min(S, rows - tile*S) / SC).
__device__ __forceinline__ int unit_chunks(const TmaGeom& g, long long tile) {
  const long long S = (long long)g.SC * g.chunks_per_unit;
  long long left = g.rows - tile * S;
  if (left > S) left = S;
  return (int)((left + g.SC - 1) / g.SC);
}

// Where the vectors a thread owns in every chunk go in global memory. The
// chunk is stored in shared memory as nbox boxes of SC rows x bw channels;
// vector v (16 bytes) of the chunk is box v / (SC*vpr), row (v % (SC*vpr)) /
// vpr, vector column v % vpr. off = element offset from the chunk's origin
// (first row, first channel of the group); row = row within the chunk, or a
// huge value for a slot past the end of the chunk.
template <class IO>
struct VecMap {
  long long off[kVec];
  int row[kVec];
  __device__ __forceinline__ void init(const TmaGeom& g, int tid) {
    constexpr int ve = 16 / IO::kBytes;  // elements per vector
    const int vpr = g.bw / ve;
    const int vpb = vpr * g.SC;
    const int nvec = (int)(g.chunk_bytes / 16);
#pragma unroll
    for (int it = 0; it < kVec; ++it) {
      const int v = tid + it * kThreads;
      if (v < nvec) {
        const int bx = v / vpb;
        const int rem = v - bx * vpb;
        const int r = rem / vpr;
        const int c = rem - r * vpr;
        row[it] = r;
        off[it] = (long long)r * g.d + (long long)bx * g.bw + (long long)c * ve;
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

// --- forward -----------------------------------------------------------------------
// Work items are (row chunk, group) pairs, item w -> chunk w / n_g, group w % n_g,
// taken by CTA i as w = i, i + grid, ...

template <class IO>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tma(const __grid_constant__ CUtensorMap mx, typename IO::T* __restrict__ y,
        const float* __restrict__ a, const float* __restrict__ b, const TmaGeom geom) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const Layout L(geom.chunk_bytes, 1, kFwdStages, false);
  float* coef = reinterpret_cast<float*>(smem + L.coef_off);
  const uint32_t full0 = smem_addr(smem + L.bar_off);
  const uint32_t empty0 = full0 + 8 * kFwdStages;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const long long row_chunks = (geom.rows + geom.SC - 1) / geom.SC;
  const long long items = row_chunks * geom.n_g;
  const int box_bytes = geom.SC * geom.bw * IO::kBytes;

  if (tid == 0) {
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
    prefetch_map(&mx);
  }
  __syncthreads();

  // issue cursor (thread 0): next item to load and its sequence number
  long long iw = blockIdx.x, iq = 0;
  auto issue = [&]() {
    const int s = (int)(iq % kFwdStages);
    const long long rc = iw / geom.n_g;
    const int g = (int)(iw - rc * geom.n_g);
    float* cs = coef + s * kCoefSlot;
#pragma unroll
    for (int i = 0; i < 6; ++i) cs[i] = __ldg(a + g * 6 + i);
#pragma unroll
    for (int j = 0; j < 4; ++j) cs[6 + j] = __ldg(b + g * 4 + j);
    mbar_arrive_expect_tx(full0 + 8 * s, geom.chunk_bytes);
    for (int bx = 0; bx < geom.nbox; ++bx)
      tma_load_2d(smem_addr(smem + s * L.stage_stride + bx * box_bytes), &mx,
                  g * geom.dg + bx * geom.bw, (int)(rc * geom.SC), full0 + 8 * s);
    iw += gridDim.x;
    ++iq;
  };
  if (tid == 0)
    for (int s = 0; s < kFwdStages && iw < items; ++s) issue();

  VecMap<IO> vm;
  vm.init(geom, tid);
  const int nvec = (int)(geom.chunk_bytes / 16);
  Coef54 c;
  int cur_g = -1;
  bool ok = true;
  long long q = 0;
  for (long long w = blockIdx.x; w < items; w += gridDim.x, ++q) {
    const int s = (int)(q % kFwdStages);
    if (tid == 0 && q >= 1 && iw < items) {
      // refill the stage of chunk q-1 once every warp has read it
      if (!mbar_wait(empty0 + 8 * (int)((q - 1) % kFwdStages),
                     (uint32_t)((q - 1) / kFwdStages) & 1)) {
        report(kErrEmptyWait);
        ok = false;
        break;
      }
      issue();
    }
    if (!mbar_wait(full0 + 8 * s, (uint32_t)(q / kFwdStages) & 1)) {
      report(kErrFullWait);
      ok = false;
      break;
    }
    const long long rc = w / geom.n_g;
    const int g = (int)(w - rc * geom.n_g);
    if (g != cur_g) {
      c.set(coef + s * kCoefSlot);
      cur_g = g;
    }
    const uint4* buf = reinterpret_cast<const uint4*>(smem + s * L.stage_stride);
    uint4 v[kVec];
#pragma unroll
    for (int it = 0; it < kVec; ++it) {
      const int vi = tid + it * kThreads;
      if (vi < nvec) v[it] = buf[vi];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
    const long long row0 = rc * geom.SC;
    typename IO::T* yo = y + row0 * geom.d + (long long)g * geom.dg;
#pragma unroll
    for (int it = 0; it < kVec; ++it) {
      if (row0 + vm.row[it] < geom.rows) {
        uint4 o;
        if constexpr (IO::kBytes == 2) {
          o.x = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v[it].x)));
          o.y = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v[it].y)));
          o.z = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v[it].z)));
          o.w = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v[it].w)));
        } else {
          const float2 p0 =
              fwd_pair(c, make_float2(__uint_as_float(v[it].x), __uint_as_float(v[it].y)));
          const float2 p1 =
              fwd_pair(c, make_float2(__uint_as_float(v[it].z), __uint_as_float(v[it].w)));
          o = make_uint4(__float_as_uint(p0.x), __float_as_uint(p0.y), __float_as_uint(p1.x),
                         __float_as_uint(p1.y));
        }
        store16(yo + vm.off[it], o);
      }
    }
  }
  if (!ok && tid == 0) {
    // wind down: let every issued load land before the CTA's memory goes away
    for (long long j = q; j < iq; ++j)
      if (!mbar_wait(full0 + 8 * (int)(j % kFwdStages), (uint32_t)(j / kFwdStages) & 1))
        report(kErrDrainWait);
  }
}

// --- backward ------------------------------------------------------------------------
// Units u = tile * n_g + g, taken by CTA i as u = i, i + grid, ...; the partial
// sum of unit (tile, g), coefficient k goes to ws[(g * 10 + k) * T + tile].

template <class IO>
__global__ void __launch_bounds__(kThreads, 1)
bwd_tma(const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mdy,
        typename IO::T* __restrict__ dx, const float* __restrict__ a,
        const float* __restrict__ b, float* __restrict__ ws, const TmaGeom geom) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const Layout L(geom.chunk_bytes, 2, kBwdStages, true);
  const unsigned cbytes = round_up(geom.chunk_bytes, 128);  // x at +0, dy at +cbytes
  float* coef = reinterpret_cast<float*>(smem + L.coef_off);
  const uint32_t full0 = smem_addr(smem + L.bar_off);
  const uint32_t empty0 = full0 + 8 * kBwdStages;
  const uint32_t redbar = empty0 + 8 * kBwdStages;  // two: "written", "read"
  float* red = reinterpret_cast<float*>(smem + L.red_off);  // [10][kThreads]
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const long long units = geom.T * geom.n_g;
  const int box_bytes = geom.SC * geom.bw * IO::kBytes;

  if (tid == 0) {
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kWarps);
    }
    mbar_init(redbar, kWarps);
    mbar_init(redbar + 8, kWarps);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
    prefetch_map(&mx);
    prefetch_map(&mdy);
  }
  __syncthreads();

  // issue cursor (thread 0): unit iu, chunk ick of nick, sequence number iq
  long long iu = blockIdx.x, iq = 0;
  int ick = 0, inck = 0;
  float cv[10];
  auto start_unit = [&]() {
    if (iu < units) {
      const long long tile = iu / geom.n_g;
      const int g = (int)(iu - tile * geom.n_g);
      inck = unit_chunks(geom, tile);
#pragma unroll
      for (int i = 0; i < 6; ++i) cv[i] = __ldg(a + g * 6 + i);
#pragma unroll
      for (int j = 0; j < 4; ++j) cv[6 + j] = __ldg(b + g * 4 + j);
    }
  };
  auto issue = [&]() {
    const int s = (int)(iq % kBwdStages);
    const long long tile = iu / geom.n_g;
    const int g = (int)(iu - tile * geom.n_g);
    unsigned char* stage = smem + s * L.stage_stride;
    float* cs = coef + s * kCoefSlot;
#pragma unroll
    for (int k = 0; k < 10; ++k) cs[k] = cv[k];
    const int col = g * geom.dg;
    const int row = (int)(tile * (long long)geom.SC * geom.chunks_per_unit + (long long)ick * geom.SC);
    mbar_arrive_expect_tx(full0 + 8 * s, 2u * geom.chunk_bytes);
    for (int bx = 0; bx < geom.nbox; ++bx) {
      tma_load_2d(smem_addr(stage + bx * box_bytes), &mx, col + bx * geom.bw, row, full0 + 8 * s);
      tma_load_2d(smem_addr(stage + cbytes + bx * box_bytes), &mdy, col + bx * geom.bw, row,
                  full0 + 8 * s);
    }
    ++iq;
    if (++ick == inck) {
      ick = 0;
      iu += gridDim.x;
      start_unit();
    }
  };
  if (tid == 0) {
    start_unit();
    for (int s = 0; s < kBwdStages && iu < units; ++s) issue();
  }

  VecMap<IO> vm;
  vm.init(geom, tid);
  const int nvec = (int)(geom.chunk_bytes / 16);
  Coef54 c;
  Acc54 acc;
  bool ok = true;
  long long q = 0;
  uint32_t nred = 0;  // reductions done (phase of the reduction barriers)
  for (long long u = blockIdx.x; u < units && ok; u += gridDim.x) {
    const long long tile = u / geom.n_g;
    const int g = (int)(u - tile * geom.n_g);
    const int nck = unit_chunks(geom, tile);
    const long long S = (long long)geom.SC * geom.chunks_per_unit;
    acc.zero();
    for (int ck = 0; ck < nck; ++ck, ++q) {
      const int s = (int)(q % kBwdStages);
      if (tid == 0 && q >= 1 && iu < units) {
        if (!mbar_wait(empty0 + 8 * (int)((q - 1) % kBwdStages),
                       (uint32_t)((q - 1) / kBwdStages) & 1)) {
          report(kErrEmptyWait);
          ok = false;
          break;
        }
        issue();
      }
      if (!mbar_wait(full0 + 8 * s, (uint32_t)(q / kBwdStages) & 1)) {
        report(kErrFullWait);
        ok = false;
        break;
      }
      if (ck == 0) c.set(coef + s * kCoefSlot);
      const uint4* xb = reinterpret_cast<const uint4*>(smem + s * L.stage_stride);
      const uint4* gb = reinterpret_cast<const uint4*>(smem + s * L.stage_stride + cbytes);
      uint4 xv[kVec], gv[kVec];
#pragma unroll
      for (int it = 0; it < kVec; ++it) {
        const int vi = tid + it * kThreads;
        if (vi < nvec) {
          xv[it] = xb[vi];
          gv[it] = gb[vi];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
      const long long row0 = tile * S + (long long)ck * geom.SC;
      typename IO::T* dxo = dx + row0 * geom.d + (long long)g * geom.dg;
#pragma unroll
      for (int it = 0; it < kVec; ++it) {
        // rows past the end were zero-filled by TMA: they add exact zeros to
        // the sums but must not be stored
        if (tid + it * kThreads < nvec) {
          uint4 o;
          if constexpr (IO::kBytes == 2) {
            o.x = f2_to_bf16x2(bwd_pair(c, bf16x2_to_f2(xv[it].x), bf16x2_to_f2(gv[it].x), acc));
            o.y = f2_to_bf16x2(bwd_pair(c, bf16x2_to_f2(xv[it].y), bf16x2_to_f2(gv[it].y), acc));
            o.z = f2_to_bf16x2(bwd_pair(c, bf16x2_to_f2(xv[it].z), bf16x2_to_f2(gv[it].z), acc));
            o.w = f2_to_bf16x2(bwd_pair(c, bf16x2_to_f2(xv[it].w), bf16x2_to_f2(gv[it].w), acc));
          } else {
            const float2 p0 = bwd_pair(
                c, make_float2(__uint_as_float(xv[it].x), __uint_as_float(xv[it].y)),
                make_float2(__uint_as_float(gv[it].x), __uint_as_float(gv[it].y)), acc);
            const float2 p1 = bwd_pair(
                c, make_float2(__uint_as_float(xv[it].z), __uint_as_float(xv[it].w)),
                make_float2(__uint_as_float(gv[it].z), __uint_as_float(gv[it].w)), acc);
            o = make_uint4(__float_as_uint(p0.x), __float_as_uint(p0.y), __float_as_uint(p1.x),
                           __float_as_uint(p1.y));
          }
          if (row0 + vm.row[it] < geom.rows) store16(dxo + vm.off[it], o);
        }
      }
    }
    if (!ok) break;

    // Unit reduction, fixed order: lanes of a pair, then red[k][thread], then
    // warp k sums coefficient k over threads lane, lane + 32, ... (in order)
    // and an xor butterfly.
    float* rk = red + tid;
    rk[0 * kThreads] = acc.a0.x + acc.a0.y;
    rk[1 * kThreads] = acc.a1.x + acc.a1.y;
    rk[2 * kThreads] = acc.a2.x + acc.a2.y;
    rk[3 * kThreads] = acc.a3.x + acc.a3.y;
    rk[4 * kThreads] = acc.a4.x + acc.a4.y;
    rk[5 * kThreads] = acc.a5.x + acc.a5.y;
    rk[6 * kThreads] = acc.b1.x + acc.b1.y;
    rk[7 * kThreads] = acc.b2.x + acc.b2.y;
    rk[8 * kThreads] = acc.b3.x + acc.b3.y;
    rk[9 * kThreads] = acc.b4.x + acc.b4.y;
    __syncwarp();
    if (lane == 0) mbar_arrive(redbar);
    if (!mbar_wait(redbar, nred & 1)) {
      report(kErrReduceWait);
      ok = false;
      break;
    }
    for (int k = warp; k < 10; k += kWarps) {
      const float* col = red + k * kThreads;
      float v = col[lane];
#pragma unroll
      for (int i = 1; i < kWarps; ++i) v += col[lane + 32 * i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) ws[((long long)g * 10 + k) * geom.T + tile] = v;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(redbar + 8);
    if (!mbar_wait(redbar + 8, nred & 1)) {
      report(kErrReduceWait);
      ok = false;
      break;
    }
    ++nred;
  }
  if (!ok && tid == 0) {
    for (long long j = q; j < iq; ++j)
      if (!mbar_wait(full0 + 8 * (int)(j % kBwdStages), (uint32_t)(j / kBwdStages) & 1))
        report(kErrDrainWait);
  }
}

// --- host-side launchers ---------------------------------------------------------

// Raise a kernel's dynamic shared-memory limit to the largest layout it can
// need and ask for the largest shared-memory carveout. One cache per kernel
// instantiation (the instantiations share a function-pointer type, so the
// cache is keyed on the template arguments); set once per device.
template <class IO, bool kBackward>
inline cudaError_t ensure_smem(unsigned most) {
  static int done_for_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (done_for_device == dev) return cudaSuccess;
  const void* fn = kBackward ? reinterpret_cast<const void*>(bwd_tma<IO>)
                             : reinterpret_cast<const void*>(fwd_tma<IO>);
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done_for_device = dev;
  return e;
}

inline cudaError_t launch_fwd_tma(bool bf16, const TmaGeom& g, const CUtensorMap& mx, void* y,
                                  const float* a, const float* b, int sms, cudaStream_t st) {
  const Layout L(g.chunk_bytes, 1, kFwdStages, false);
  const unsigned most = Layout(kMaxChunkBytes, 1, kFwdStages, false).total;
  if (L.total > most) return cudaErrorInvalidValue;
  const long long items = ((g.rows + g.SC - 1) / g.SC) * g.n_g;
  long long grid = sms;
  if (grid > items) grid = items;
  cudaError_t e;
  if (bf16) {
    if ((e = ensure_smem<IoBF16, false>(most)) != cudaSuccess) return e;
    fwd_tma<IoBF16><<<(unsigned)grid, kThreads, L.total, st>>>(mx, (IoBF16::T*)y, a, b, g);
  } else {
    if ((e = ensure_smem<IoF32, false>(most)) != cudaSuccess) return e;
    fwd_tma<IoF32><<<(unsigned)grid, kThreads, L.total, st>>>(mx, (IoF32::T*)y, a, b, g);
  }
  return cudaGetLastError();
}

inline cudaError_t launch_bwd_tma(bool bf16, const TmaGeom& g, const CUtensorMap& mx,
                                  const CUtensorMap& mdy, void* dx, const float* a,
                                  const float* b, float* ws, int sms, cudaStream_t st) {
  const Layout L(g.chunk_bytes, 2, kBwdStages, true);
  const unsigned most = Layout(kMaxChunkBytes, 2, kBwdStages, true).total;
  if (L.total > most) return cudaErrorInvalidValue;
  const long long units = g.T * g.n_g;
  long long grid = sms;
  if (grid > units) grid = units;
  cudaError_t e;
  if (bf16) {
    if ((e = ensure_smem<IoBF16, true>(most)) != cudaSuccess) return e;
    bwd_tma<IoBF16><<<(unsigned)grid, kThreads, L.total, st>>>(mx, mdy, (IoBF16::T*)dx, a, b,
                                                                ws, g);
  } else {
    if ((e = ensure_smem<IoF32, true>(most)) != cudaSuccess) return e;
    bwd_tma<IoF32><<<(unsigned)grid, kThreads, L.total, st>>>(mx, mdy, (IoF32::T*)dx, a, b, ws,
                                                               g);
  }
  return cudaGetLastError();
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
