// grkan_linear.cuh -- the GR-KAN activation fused into the linear layer that
// follows it, on the fifth-generation tensor cores:
//
//   out[r, o] = sum_k y[r, k] W[o, k] (+ bias[o]),   y = P(x) / (1 + |Q(x)|)
//
// A KAT layer is a group-rational activation followed by a linear map
// ("FlashKAT ...", paper notes, section "Insight 2": the GR-KAN term next to the
// linear layer's 2 d_in d_out operations), and the pages locate what remains of
// the training time after their fix in the GR-KAN forward. Here the activation
// is computed while the tile of x waits in shared memory for the matrix
// multiply, so y never goes to HBM.
//
// One CTA computes a 128 x 512 tile of out (bf16 in, float32 accumulate in all
// 512 TMEM columns, bf16 out), in K steps of 32, so that the activation of an x
// tile serves 512 output features:
//   warp 0       lane 0 issues the TMA loads of the x tile (128 x 32) and of
//                the W tile (two 256 x 32 halves), 64-byte swizzled, into a
//                ring of stages;
//   warps 2..17  apply the activation to the x tile in place (same swizzled
//                positions), then signal the stage ready;
//   warp 1       allocates the TMEM columns; lane 0 issues two tcgen05.mma
//                (M 128, N 256, K 16) per half and stage and returns the stage
//                to the producer with tcgen05.commit;
//   warps 2..5   at the end read the accumulators (tcgen05.ld, one 32-lane
//                quarter each), add the bias, convert to bf16 and write the
//                tile through 128-byte-swizzled staging buffers with TMA
//                stores.
// A tile whose second half lies past n_out issues neither its loads nor its
// MMAs.
// Every wait is bounded (device error word, as in the other kernels); TMEM is
// freed on every path.
#pragma once

#include "grkan_tma.cuh"

namespace grk {
namespace lin {

constexpr int BM = 128;   // rows of a tile (UMMA M)
constexpr int BNH = 256;  // output features of one MMA (UMMA N), a tile half
constexpr int BN = 2 * BNH;
constexpr int BK = 32;    // K per stage: one 64-byte swizzle row of bf16
constexpr int kStages = 5;
#ifndef GRK_LIN_XFORM_WARPS
#define GRK_LIN_XFORM_WARPS 16
#endif
constexpr int kXformWarps = GRK_LIN_XFORM_WARPS;  // warps applying the activation
constexpr int kChunksPerRow = BK * 2 / 16;                        // 16-byte chunks per row
constexpr int kXformRows = BM * kChunksPerRow / (kXformWarps * 32);  // rows per transform thread
constexpr int kWarps = 2 + kXformWarps;
constexpr int kThreads = kWarps * 32;
constexpr unsigned kATile = BM * BK * 2;    // 8 KiB
constexpr unsigned kBHalf = BNH * BK * 2;   // 16 KiB
constexpr unsigned kBTile = 2 * kBHalf;     // 32 KiB
constexpr unsigned kStage = kATile + kBTile;
constexpr unsigned kEpiRows = 32;         // rows per epilogue warp
constexpr unsigned kEpiCols = 64;         // columns per TMA store box (128 bytes of bf16)
constexpr unsigned kEpiBuf = kEpiRows * kEpiCols * 2;  // 4 KiB staging buffer

// Shared memory: [stages][A | B] at a 1024-byte boundary, then the barriers
// (full, ready, empty per stage; accumulator full), the TMEM address slot and
// the coefficient table.
struct Layout {
  static constexpr unsigned kBarOff = kStages * kStage;
  static constexpr unsigned kNumBars = 3 * kStages + 1;
  static constexpr unsigned kTmemSlot = kBarOff + kNumBars * 8;
  static constexpr unsigned kTabOff = (kTmemSlot + 4 + 15) / 16 * 16;
  static constexpr unsigned kBytes = kTabOff + coef_table_bytes<5, 4>();
  static constexpr unsigned kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

// As mbar_try_wait, but the thread may sleep in the instruction until the phase
// completes (at most kSuspendHintNs per call): a waiting thread issues almost
// nothing, which leaves the issue slots to the warps that compute.
constexpr uint32_t kSuspendHintNs = 10000000u;  // 10 ms
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Sleeping wait for the phase with the given parity; false after kWaitTimeoutNs.
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait_sleep(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned polls = 0; !mbar_try_wait_sleep(bar, parity); ++polls) {
    if (global_ns() - t0 > kWaitTimeoutNs || polls > kMaxPolls) return false;
  }
  return true;
}

// --- tcgen05 wrappers ---------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] B[smem]^T, kind::f16 (bf16 inputs, float32 accumulator)
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on an mbarrier once every tcgen05 operation issued so far by this thread is done
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// 16 consecutive float32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}


// Shared-memory matrix descriptor of a K-major bf16 tile written by TMA with
// 64-byte swizzling: rows of 64 bytes, 8-row atoms of 512 bytes one after
// another (stride byte offset 512), descriptor version 1, layout SWIZZLE_64B.
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(512u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)4u << 61);
}

// Instruction descriptor: float32 accumulator, bf16 A and B, both K-major,
// M = BM, and N (a multiple of 16 up to BNH) in bits [17, 23) as N / 8.
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BM >> 4) << 24);
__host__ __device__ constexpr uint32_t idesc_n(int n) {
  return kIdescBase | ((uint32_t)(n >> 3) << 17);
}

struct LinGeom {
  long long rows;  // R = B * N
  int d;           // K: input features (the activation's channels)
  int nout;        // output features
  int dg;          // channels per group
  int n_g;
  int kt;          // K steps = d / BK
};

__global__ void __launch_bounds__(kThreads, 1)
linear_fwd(const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mw,
           const __grid_constant__ CUtensorMap mo, const float* __restrict__ a,
           const float* __restrict__ b, const float* __restrict__ bias, const LinGeom geom) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + Layout::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * (uint32_t)s; };
  auto ready_bar = [&](int s) { return bar0 + 8u * (uint32_t)(kStages + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(2 * kStages + s); };
  const uint32_t acc_bar = bar0 + 8u * (uint32_t)(3 * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Layout::kTmemSlot);
  float* ctab = reinterpret_cast<float*>(smem + Layout::kTabOff);
  const bool use_tab = geom.n_g <= kTableGroups;

  const int n_tiles = (geom.nout + BN - 1) / BN;
  const int n0 = (int)(blockIdx.x % n_tiles) * BN;
  const long long m0 = (long long)(blockIdx.x / n_tiles) * BM;
  const bool two = n0 + BNH < geom.nout;  // the tile's second half holds outputs
  // MMA widths of the two halves: the valid columns rounded up to 16, so a
  // narrow last tile does not multiply zero-filled W rows
  const int w0 = geom.nout - n0 < BNH ? geom.nout - n0 : BNH;
  const int w1 = two ? (geom.nout - n0 - BNH < BNH ? geom.nout - n0 - BNH : BNH) : 0;
  const uint32_t idesc0 = idesc_n((w0 + 15) / 16 * 16);
  const uint32_t idesc1 = idesc_n(two ? (w1 + 15) / 16 * 16 : 16);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(ready_bar(s), kXformWarps);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
    prefetch_map(&mx);
    prefetch_map(&mw);
    prefetch_map(&mo);
  }
  if (warp == 1) {
    tmem_alloc(sbase + Layout::kTmemSlot, (uint32_t)BN);  // 512 columns: both halves
    tmem_relinquish();
  }
  if (use_tab) build_coef_table<5, 4>(ctab, a, b, geom.n_g);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ---- TMA producer -------------------------------------------------------------
    if (lane == 0) {
      int issued = 0;
      for (int kt = 0; kt < geom.kt; ++kt) {
        const int s = kt % kStages;
        if (kt >= kStages &&
            !mbar_wait(empty_bar(s), (uint32_t)((kt / kStages) - 1) & 1u)) {
          report(kErrEmptyWait);
          ok = false;
          break;
        }
        const uint32_t sa = sbase + (uint32_t)s * kStage;
        mbar_arrive_expect_tx(full_bar(s), two ? kStage : kATile + kBHalf);
        tma_load_2d(sa, &mx, kt * BK, (int)m0, full_bar(s));
        tma_load_2d(sa + kATile, &mw, kt * BK, n0, full_bar(s));
        if (two) tma_load_2d(sa + kATile + kBHalf, &mw, kt * BK, n0 + BNH, full_bar(s));
        ++issued;
      }
      if (!ok) {  // let the issued loads land before the CTA's memory goes away
        for (int j = 0; j < issued; ++j)
          if (!mbar_wait(full_bar(j % kStages), (uint32_t)(j / kStages) & 1u)) report(kErrDrainWait);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issue ----------------------------------------------------------------
    if (lane == 0) {
      for (int kt = 0; kt < geom.kt; ++kt) {
        const int s = kt % kStages;
        const uint32_t ph = (uint32_t)(kt / kStages) & 1u;
        if (!mbar_wait(full_bar(s), ph) || !mbar_wait(ready_bar(s), ph)) {
          report(kErrFullWait);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = sbase + (uint32_t)s * kStage;
        const uint64_t ad = sw64_desc(sa);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 1 && !two) break;
          const uint64_t bd = sw64_desc(sa + kATile + (uint32_t)h * kBHalf);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // 16 bf16 = 32 bytes = 2 descriptor units per step
            umma_bf16(tmem_d + (uint32_t)(h * BNH), ad + 2u * (uint64_t)k, bd + 2u * (uint64_t)k,
                      h == 0 ? idesc0 : idesc1, (kt > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(empty_bar(s));
      }
      umma_commit(acc_bar);  // every MMA issued above is done when this arrives
      // and none may still write TMEM when the columns are freed
      if (!mbar_wait(acc_bar, 0)) report(kErrReduceWait);
    }
  } else {
    // ---- activation in place, then the epilogue -----------------------------------
    const int t = threadIdx.x - 64;      // 0 .. 32 kXformWarps - 1
    const int j = t % kChunksPerRow;     // logical 16-byte chunk (8 channels) of a row
    const int rb = t / kChunksPerRow;    // rows rb + i kRowStep, i < kXformRows
    constexpr int kRowStep = kXformWarps * 32 / kChunksPerRow;
    Coef54 c;
    int cur_g = -1;
    for (int kt = 0; kt < geom.kt; ++kt) {
      const int s = kt % kStages;
      const uint32_t ph = (uint32_t)(kt / kStages) & 1u;
      if (!mbar_wait(full_bar(s), ph)) {
        report(kErrFullWait);
        ok = false;
        break;
      }
      const int g = (kt * BK + j * 8) / geom.dg;  // a chunk lies in one group (d_g % 8 == 0)
      if (g != cur_g) {
        load_coef<5, 4>(use_tab, ctab, a, b, g, c);
        cur_g = g;
      }
      unsigned char* at = smem + (size_t)s * kStage;
      // all loads first, then the arithmetic, then all stores: independent chunks
      // in flight together
      uint4* p[kXformRows];
      uint4 v[kXformRows];
#pragma unroll
      for (int i = 0; i < kXformRows; ++i) {
        const int r = rb + kRowStep * i;
        // 64-byte swizzle: chunk bits [4, 6) of the offset xor row bits [1, 3)
        p[i] = reinterpret_cast<uint4*>(at + r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
        v[i] = *p[i];
      }
#pragma unroll
      for (int i = 0; i < kXformRows; ++i) {
        v[i].x = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v[i].x)));
        v[i].y = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v[i].y)));
        v[i].z = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v[i].z)));
        v[i].w = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v[i].w)));
      }
#pragma unroll
      for (int i = 0; i < kXformRows; ++i) *p[i] = v[i];
      fence_proxy_async_smem();  // generic-proxy writes before the tensor core's reads
      __syncwarp();
      if (lane == 0) mbar_arrive(ready_bar(s));
    }
    // epilogue: warps 2..5, TMEM lane quarter = warp % 4
    if (warp < 6) {
      const int q = warp & 3;
      if (!mbar_wait(acc_bar, 0)) {
        report(kErrReduceWait);
        ok = false;
      }
      tc_fence_after();
      if (ok) {
        // staging buffer of this warp inside the (now idle) stage ring, 1024-aligned
        unsigned char* stg = smem + (size_t)(warp - 2) * 2 * kEpiBuf;
        const uint32_t stg_a = sbase + (uint32_t)(warp - 2) * 2u * kEpiBuf;
        for (int cb = 0; cb < BN / (int)kEpiCols; ++cb) {
          const int col0 = n0 + cb * (int)kEpiCols;
          if (col0 >= geom.nout) break;
          const int buf = cb & 1;
          if (cb >= 2) {  // the store that used this buffer has read it
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
          }
          unsigned char* sb = stg + buf * kEpiBuf;
#pragma unroll
          for (int h = 0; h < (int)kEpiCols / 16; ++h) {
            float v[16];
            tmem_ld16(tmem_d + ((uint32_t)(q * 32) << 16) + (uint32_t)(cb * kEpiCols + h * 16), v);
            if (bias) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int col = col0 + h * 16 + e;
                v[e] += col < geom.nout ? __ldg(bias + col) : 0.f;
              }
            }
            // two 16-byte chunks (logical 2h, 2h + 1) of this row, swizzled
            uint4 w0, w1;
            w0.x = f2_to_bf16x2(make_float2(v[0], v[1]));
            w0.y = f2_to_bf16x2(make_float2(v[2], v[3]));
            w0.z = f2_to_bf16x2(make_float2(v[4], v[5]));
            w0.w = f2_to_bf16x2(make_float2(v[6], v[7]));
            w1.x = f2_to_bf16x2(make_float2(v[8], v[9]));
            w1.y = f2_to_bf16x2(make_float2(v[10], v[11]));
            w1.z = f2_to_bf16x2(make_float2(v[12], v[13]));
            w1.w = f2_to_bf16x2(make_float2(v[14], v[15]));
            *reinterpret_cast<uint4*>(sb + lane * 128 + (((2 * h) ^ (lane & 7)) << 4)) = w0;
            *reinterpret_cast<uint4*>(sb + lane * 128 + (((2 * h + 1) ^ (lane & 7)) << 4)) = w1;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&mo, col0, (int)m0 + q * 32, stg_a + (uint32_t)buf * kEpiBuf);
            bulk_commit();
          }
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
      }
    }
  }
  // teardown: every tcgen05.ld has completed; free the accumulator columns
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, (uint32_t)BN);
  }
}

}  // namespace lin
}  // namespace grk
