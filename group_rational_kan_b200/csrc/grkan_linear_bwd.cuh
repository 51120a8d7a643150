// grkan_linear_bwd.cuh -- the GR-KAN backward fused into the data-gradient
// matrix multiply of the linear layer that follows the activation:
//
//   dy[r, c] = sum_o dout[r, o] W[o, c]            (the activation's output gradient)
//   dx[r, c] = dy (P'(x) - y s Q'(x)) / D          (as grkan_backward)
//   dA[g, i] = sum t x^i,  dB[g, j] = -sum t y s x^j,  t = dy / D
//
// The pages fuse the activation's backward into one kernel per element stream
// ("FlashKAT ...", paper notes, section "3. FlashKAT kernel restructuring
// (Algorithm 2)"); a KAT layer pairs it with a linear map (section "Insight 2").
// Here dy never exists in memory: it is the float32 accumulator of the tensor
// core product, and the activation's backward runs as that product's epilogue.
//
// Persistent kernel, one CTA per SM, tiles of 128 rows x 192 channels taken in
// the order tile = blockIdx.x + i gridDim.x (row-tile major, so the CTAs working
// at the same time share their dout rows and W columns in L2):
//   warp 0       lane 0 issues the TMA loads: per tile the x tile (six 32-channel
//                boxes, 64-byte swizzled, double-buffered), then per K step of 64
//                output features the dout tile (128 x 64, K-major) and the W tile
//                (three 64-channel x 64-feature boxes, channel-major), 128-byte
//                swizzled, into a three-stage ring;
//   warp 1       allocates 512 TMEM columns (two 192-column accumulators) and
//                lane 0 issues four tcgen05.mma (M 128, N 192, K 16; W read
//                channel-major, i.e. MN-major) per stage;
//   warps 2..13  the epilogue: warp w reads TMEM lane quarter w % 4 (32 rows)
//                and 64 channels ((w - 2) / 4), runs the (5, 4) backward on
//                each element pair with dy from the accumulator and x from the
//                shared tile, writes dx over x in place, stores it with TMA, and
//                sums t x^i, -t y s x^j over its 32 x 64 block into one float32
//                partial per coefficient.
// The accumulator and the x buffer of a tile go back to the MMA and TMA warps
// as soon as the epilogue is done with them, so the product of tile i + 1 runs
// under the epilogue of tile i. Every wait is bounded (device error word), and
// TMEM is freed on every path.
#pragma once

#include "grkan_linear.cuh"

namespace grk {
namespace lin {
namespace dg {

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
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (global_ns() - t0 > kWaitTimeoutNs) return false;
  }
  return true;
}

constexpr int BM = 128;            // rows per tile (UMMA M)
constexpr int BN = 192;            // channels per tile (UMMA N)
constexpr int BK = 64;             // output features per stage: one 128-byte swizzle row
constexpr int kStages = 3;
constexpr int kEpiWarps = 12;      // three per TMEM lane quarter
constexpr int kWarps = 2 + kEpiWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kWarpCols = BN / (kEpiWarps / 4);  // 64 channels per epilogue warp
constexpr int kAccStride = 256;    // TMEM column offset of the second accumulator
constexpr unsigned kATile = BM * BK * 2;          // 16 KiB: dout, 128 rows x 64 features
constexpr unsigned kWBox = 64 * BK * 2;           // 8 KiB: 64 features x 64 channels
constexpr unsigned kWTile = (BN / 64) * kWBox;    // 24 KiB
constexpr unsigned kStage = kATile + kWTile;      // 40 KiB
constexpr unsigned kXBox = BM * 32 * 2;           // 8 KiB: 128 rows x 32 channels
constexpr unsigned kXTile = (BN / 32) * kXBox;    // 48 KiB
constexpr unsigned kXSub = 32 * 32 * 2;           // 2 KiB: one warp's 32 rows of a box
static_assert(kWarpCols == 64, "an epilogue warp covers two 32-channel x boxes");

// Shared memory: [stages][dout | W] and the two x / dx tiles (all at 1024-byte
// boundaries), then the barriers, the TMEM address slot and the coefficient
// table.
struct Layout {
  static constexpr unsigned kXOff = kStages * kStage;
  static constexpr unsigned kBarOff = kXOff + 2 * kXTile;
  // full[S], empty[S], acc_full[2], acc_empty[2], x_full[2], x_empty[2], done
  static constexpr unsigned kNumBars = 2 * kStages + 9;
  static constexpr unsigned kTmemSlot = kBarOff + kNumBars * 8;
  static constexpr unsigned kTabOff = (kTmemSlot + 4 + 15) / 16 * 16;
  static constexpr unsigned kBytes = kTabOff + coef_table_bytes<5, 4>();
  static constexpr unsigned kAlloc = kBytes + 1024;  // slack to align the base to 1024
};
static_assert(Layout::kAlloc <= 232448, "shared memory per CTA");

// K-major bf16 tile written by TMA with 128-byte swizzling: 128-byte rows,
// 8-row atoms of 1024 bytes one after another (stride byte offset 1024),
// descriptor version 1, layout SWIZZLE_128B. A K step of 16 elements moves the
// start address 32 bytes along the row.
__device__ __forceinline__ uint64_t sw128_k_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// MN-major bf16 tile of 64-channel boxes, 128-byte swizzled: each K index is a
// 128-byte row of 64 channels, 8 K rows make a 1024-byte atom (stride byte
// offset: the next 8 K rows), and the next 64 channels sit one box further on
// (leading byte offset kWBox). A K step of 16 moves the start two atoms.
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(kWBox >> 4) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// Instruction descriptor: float32 accumulator, bf16 A and B, A K-major, B
// MN-major (bit 16), M = 128, N in bits [17, 23) as N / 8.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                            ((uint32_t)(BM >> 4) << 24);
__host__ __device__ constexpr uint32_t idesc_n(int n) { return kIdesc | ((uint32_t)(n >> 3) << 17); }

// 32 consecutive float32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct DgGeom {
  long long rows;     // R = B * N
  long long n_tiles;  // row tiles x column tiles
  long long ws_T;     // partial slots per (group, coefficient)
  int d;              // channels (the product's N)
  int nout;           // output features of the linear layer (the product's K)
  int dg;             // channels per group (a multiple of 64)
  int n_g;
  int kt;             // K steps = ceil(nout / BK)
  int n_ct;           // column tiles = ceil(d / BN)
  int nbg;            // 64-channel blocks per group = dg / 64
};

__global__ void __launch_bounds__(kThreads, 1)
linear_dgrad(const __grid_constant__ CUtensorMap mdo, const __grid_constant__ CUtensorMap mw,
             const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mdx,
             const float* __restrict__ a, const float* __restrict__ b, float* __restrict__ ws,
             const DgGeom geom) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + Layout::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * (uint32_t)s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(kStages + s); };
  auto accf_bar = [&](int j) { return bar0 + 8u * (uint32_t)(2 * kStages + j); };
  auto acce_bar = [&](int j) { return bar0 + 8u * (uint32_t)(2 * kStages + 2 + j); };
  auto xf_bar = [&](int j) { return bar0 + 8u * (uint32_t)(2 * kStages + 4 + j); };
  auto xe_bar = [&](int j) { return bar0 + 8u * (uint32_t)(2 * kStages + 6 + j); };
  const uint32_t done_bar = bar0 + 8u * (uint32_t)(2 * kStages + 8);
  auto stage_addr = [&](int s) { return sbase + (uint32_t)s * kStage; };
  auto xtile_addr = [&](int j) { return sbase + Layout::kXOff + (uint32_t)j * kXTile; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Layout::kTmemSlot);
  float* ctab = reinterpret_cast<float*>(smem + Layout::kTabOff);
  const bool use_tab = geom.n_g <= kTableGroups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(accf_bar(j), 1);
      mbar_init(acce_bar(j), kEpiWarps);
      mbar_init(xf_bar(j), 1);
      mbar_init(xe_bar(j), kEpiWarps);
    }
    mbar_init(done_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
    prefetch_map(&mdo);
    prefetch_map(&mw);
    prefetch_map(&mx);
    prefetch_map(&mdx);
  }
  if (warp == 1) {
    tmem_alloc(sbase + Layout::kTmemSlot, 512u);
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
      long long kc = 0;  // K steps issued over all tiles (the ring position)
      int i = 0;         // tiles issued
      for (long long tile = blockIdx.x; tile < geom.n_tiles; tile += gridDim.x, ++i) {
        const long long mt = tile / geom.n_ct;
        const int n0 = (int)(tile - mt * geom.n_ct) * BN;
        const int m0 = (int)(mt * BM);
        const int ncols = geom.d - n0 < BN ? geom.d - n0 : BN;  // a multiple of 64
        const int xb = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (use >= 1 && !mbar_wait_sleep(xe_bar(xb), (use - 1) & 1u)) {
          report(kErrEmptyWait);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(xf_bar(xb), (uint32_t)(ncols / 32) * kXBox);
        for (int j = 0; j < ncols / 32; ++j)
          tma_load_2d(xtile_addr(xb) + (uint32_t)j * kXBox, &mx, n0 + 32 * j, m0, xf_bar(xb));
        for (int kt = 0; kt < geom.kt; ++kt, ++kc) {
          const int s = (int)(kc % kStages);
          const uint32_t round = (uint32_t)(kc / kStages);
          if (kc >= kStages && !mbar_wait_sleep(empty_bar(s), (round + 1) & 1u)) {
            report(kErrEmptyWait);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(s), kATile + (uint32_t)(ncols / 64) * kWBox);
          tma_load_2d(stage_addr(s), &mdo, kt * BK, m0, full_bar(s));
          for (int j = 0; j < ncols / 64; ++j)
            tma_load_2d(stage_addr(s) + kATile + (uint32_t)j * kWBox, &mw, n0 + 64 * j, kt * BK,
                        full_bar(s));
        }
        if (!ok) {
          ++i;  // this tile's x load was issued
          break;
        }
      }
      // the last load issued into each ring slot and x buffer has landed before
      // the CTA's shared memory can go away (immediate on the normal path)
      for (long long j = kc > kStages ? kc - kStages : 0; j < kc; ++j)
        if (!mbar_wait(full_bar((int)(j % kStages)), (uint32_t)(j / kStages) & 1u))
          report(kErrDrainWait);
      for (int j = i > 2 ? i - 2 : 0; j < i; ++j)
        if (!mbar_wait(xf_bar(j & 1), (uint32_t)(j >> 1) & 1u)) report(kErrDrainWait);
    }
  } else if (warp == 1) {
    // ---- MMA issue ----------------------------------------------------------------
    if (lane == 0) {
      long long kc = 0;
      int i = 0;
      for (long long tile = blockIdx.x; tile < geom.n_tiles; tile += gridDim.x, ++i) {
        const long long mt = tile / geom.n_ct;
        const int n0 = (int)(tile - mt * geom.n_ct) * BN;
        const int ncols = geom.d - n0 < BN ? geom.d - n0 : BN;
        const uint32_t idesc = idesc_n(ncols);
        const int ab = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (use >= 1 && !mbar_wait_sleep(acce_bar(ab), (use - 1) & 1u)) {
          report(kErrEmptyWait);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem_d + (uint32_t)(ab * kAccStride);
        for (int kt = 0; kt < geom.kt; ++kt, ++kc) {
          const int s = (int)(kc % kStages);
          if (!mbar_wait_sleep(full_bar(s), (uint32_t)(kc / kStages) & 1u)) {
            report(kErrFullWait);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_k_desc(stage_addr(s));
          const uint64_t bd = sw128_mn_desc(stage_addr(s) + kATile);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // A: 32 bytes along the row; B: two 1024-byte atoms
            umma_bf16(dt, ad + 2u * (uint64_t)k, bd + 128u * (uint64_t)k, idesc,
                      (kt > 0 || k > 0) ? 1u : 0u);
          umma_commit(empty_bar(s));
        }
        if (!ok) break;
        umma_commit(accf_bar(ab));
      }
      // no MMA may still write TMEM when the columns are freed
      umma_commit(done_bar);
      if (!mbar_wait(done_bar, 0)) report(kErrReduceWait);
    }
  } else {
    // ---- epilogue: the GR-KAN backward on the accumulator -----------------------------
    const int q = warp & 3;           // TMEM lane quarter: rows 32 q .. 32 q + 31
    const int w3 = (warp - 2) >> 2;   // channels 64 w3 .. 64 w3 + 63 of the tile
    const int r = 32 * q + lane;      // this thread's row in the tile
    const int swz = (r >> 1) & 3;     // 64-byte swizzle of the row
    Coef54 c;
    int cur_g = -1;
    int i = 0;
    for (long long tile = blockIdx.x; tile < geom.n_tiles; tile += gridDim.x, ++i) {
      const long long mt = tile / geom.n_ct;
      const int n0 = (int)(tile - mt * geom.n_ct) * BN;
      const int m0 = (int)(mt * BM);
      const int ncols = geom.d - n0 < BN ? geom.d - n0 : BN;
      const int ab = i & 1;
      const uint32_t use = (uint32_t)(i >> 1);
      const bool got = mbar_wait_sleep(accf_bar(ab), use & 1u) && mbar_wait_sleep(xf_bar(ab), use & 1u);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) report(kErrFullWait);
        ok = false;
        break;
      }
      tc_fence_after();
      if (i >= 1 && lane == 0) {  // the previous tile's dx stores have read its buffer
        bulk_wait_read0();
        mbar_arrive(xe_bar((i - 1) & 1));
      }
      const bool active = 64 * w3 < ncols;
      const int cb = n0 / 64 + w3;  // 64-channel block of d
      const int g = cb / geom.nbg;
      Acc54 acc;
      acc.zero();
      if (active) {
        if (g != cur_g) {
          load_coef<5, 4>(use_tab, ctab, a, b, g, c);
          cur_g = g;
        }
        unsigned char* xt = smem + Layout::kXOff + (size_t)ab * kXTile;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {  // one 32-channel x box at a time
          float v[32];
          tmem_ld32(tmem_d + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * kAccStride + 64 * w3 + 32 * hh),
                    v);
          unsigned char* row = xt + (size_t)(2 * w3 + hh) * kXBox + (size_t)r * 64;
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // 16-byte chunks: 8 channels
            uint4* p = reinterpret_cast<uint4*>(row + ((j ^ swz) << 4));
            const uint4 xv = *p;
            uint4 o;
            o.x = f2_to_bf16x2(bwd_pair(c, bf16x2_to_f2(xv.x), make_float2(v[8 * j], v[8 * j + 1]), acc));
            o.y = f2_to_bf16x2(
                bwd_pair(c, bf16x2_to_f2(xv.y), make_float2(v[8 * j + 2], v[8 * j + 3]), acc));
            o.z = f2_to_bf16x2(
                bwd_pair(c, bf16x2_to_f2(xv.z), make_float2(v[8 * j + 4], v[8 * j + 5]), acc));
            o.w = f2_to_bf16x2(
                bwd_pair(c, bf16x2_to_f2(xv.w), make_float2(v[8 * j + 6], v[8 * j + 7]), acc));
            *p = o;
          }
        }
      }
      // the accumulator columns are read: hand them back to the MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(ab));
      if (active) {
        fence_proxy_async_smem();  // generic-proxy dx writes before the TMA store reads them
        __syncwarp();
        if (lane == 0 && (long long)m0 + 32 * q < geom.rows) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            tma_store_2d(&mdx, xtile_addr(ab) + (uint32_t)(2 * w3 + hh) * kXBox + (uint32_t)q * kXSub,
                         n0 + 64 * w3 + 32 * hh, m0 + 32 * q);
          bulk_commit();
        }
        // the block's partial sums, fixed order: the two lanes of each pair, then
        // a recursive-halving exchange over the warp's 32 rows
        float sv[16];
        Deg<5, 4>::sums<16>(acc, sv);
        warp_sum<16>(sv, lane);
        const int k = (lane >> 1) & 15;
        const long long slot = (mt * geom.nbg + (cb - g * geom.nbg)) * 4 + q;
        if ((lane & 1) == 0 && k < 10) ws[((long long)g * 10 + k) * geom.ws_T + slot] = sv[0];
      }
    }
    if (lane == 0) bulk_wait0();  // this warp's stores are complete
    __syncwarp();
  }
  // teardown: every tcgen05.ld has completed; free the accumulator columns
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, 512u);
  }
}

}  // namespace dg
}  // namespace lin
}  // namespace grk
