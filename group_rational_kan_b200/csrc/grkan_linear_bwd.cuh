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
// Persistent kernel on CTA pairs (clusters of two, tcgen05 cta_group::2), one
// CTA per SM. A pair computes a 256-row x 192-channel tile, each CTA 128 rows;
// pair tiles are taken in the order tile = pair + i pairs (row-tile major, so
// the pairs working at the same time share their dout rows and W columns in L2).
// In each CTA:
//   warp 0       lane 0 issues the TMA loads: per K step of 64 output
//                features the CTA's 128 dout rows (K-major, 128-byte swizzled)
//                and its half of the W tile (96 channels as three 32-channel
//                boxes, channel-major, 64-byte swizzled) into a ring of stages,
//                and per tile, after the first ring's worth of those, the CTA's
//                x tile (six 32-channel boxes, 64-byte swizzled,
//                double-buffered);
//   warp 1       allocates 512 TMEM columns (two 192-column accumulators). In
//                the leader (rank 0) lane 0 issues four tcgen05.mma (M 256, N
//                192, K 16; A rows from both CTAs, W from both halves, read
//                channel-major i.e. MN-major) per stage and releases the stage
//                in both CTAs with one multicast commit; in the other CTA lane
//                0 tells the leader when each of its stages has landed;
//   warps 2..13  the epilogue: warp w reads TMEM lane quarter w % 4 (32 rows)
//                and 64 channels ((w - 2) / 4), runs the (5, 4) backward on
//                each element pair with dy from the accumulator and x from the
//                shared tile, writes dx over x in place, stores it with TMA, and
//                sums t x^i, -t y s x^j over its 32 x 64 block into one float32
//                partial per coefficient.
// Each W tile crosses L2 once per 256 rows: 14 bytes of operands per output
// element (8 of dout, 6 of W) instead of 20 for single-CTA 128 x 192 tiles.
// The accumulator and the x buffer of a tile go back to the MMA and TMA warps
// as soon as the epilogue is done with them, so the product of tile i + 1 runs
// under the epilogue of tile i. Every wait is bounded (device error word), and
// TMEM is freed on every path.
#pragma once

#include "grkan_linear.cuh"

namespace grk {
namespace lin {
namespace dg {

constexpr int BM = 128;            // rows per CTA (a pair covers 256: UMMA M)
constexpr int BN = 192;            // channels per tile (UMMA N)
constexpr int BK = 64;             // output features per stage: one 128-byte swizzle row of dout
#ifndef GRK_DG_STAGES
#define GRK_DG_STAGES 4
#endif
constexpr int kStages = GRK_DG_STAGES;
constexpr int kEpiWarps = 12;      // three per TMEM lane quarter
constexpr int kWarps = 2 + kEpiWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kWarpCols = BN / (kEpiWarps / 4);  // 64 channels per epilogue warp
constexpr int kAccStride = 256;    // TMEM column offset of the second accumulator
constexpr unsigned kATile = BM * BK * 2;          // 16 KiB: dout, 128 rows x 64 features
constexpr unsigned kWBox = 32 * BK * 2;           // 4 KiB: 64 features x 32 channels
constexpr unsigned kWHalf = (BN / 2 / 32) * kWBox;  // 12 KiB: this CTA's 96 channels
constexpr unsigned kStage = kATile + kWHalf;      // 28 KiB (a multiple of 1024)
constexpr unsigned kXBox = BM * 32 * 2;           // 8 KiB: 128 rows x 32 channels
constexpr unsigned kXTile = (BN / 32) * kXBox;    // 48 KiB
constexpr unsigned kXSub = 32 * 32 * 2;           // 2 KiB: one warp's 32 rows of a box
static_assert(kWarpCols == 64, "an epilogue warp covers two 32-channel x boxes");
static_assert(kStage % 1024 == 0, "stages keep the 128-byte swizzle atoms aligned");

// Shared memory: [stages][dout | W half] and the two x / dx tiles (at 1024-byte
// boundaries), then the barriers, the TMEM address slot and the coefficient
// table.
struct Layout {
  static constexpr unsigned kXOff = kStages * kStage;
  static constexpr unsigned kBarOff = kXOff + 2 * kXTile;
  // full[S], empty[S], peer_full[S], acc_full[2], acc_empty[2], x_full[2],
  // x_empty[2], done
  static constexpr unsigned kNumBars = 3 * kStages + 9;
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
// MN-major bf16 tile of 32-channel boxes, 64-byte swizzled: each K index is a
// 64-byte row of 32 channels, 8 K rows make a 512-byte atom (stride byte
// offset: the next 8 K rows), and the next 32 channels sit one box further on
// (leading byte offset kWBox). A K step of 16 moves the start two atoms.
__device__ __forceinline__ uint64_t sw64_mn_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(kWBox >> 4) << 16) |
         ((uint64_t)(512u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)4u << 61);
}
// Instruction descriptor: float32 accumulator, bf16 A and B, A K-major, B
// MN-major (bit 16), M = 256 (the pair), N in bits [17, 23) as N / 8.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                            ((uint32_t)(2 * BM >> 4) << 24);
__host__ __device__ constexpr uint32_t idesc_n(int n) { return kIdesc | ((uint32_t)(n >> 3) << 17); }

// --- CTA-pair primitives ---------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
// the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// arrive on an mbarrier of either CTA of the pair (a shared::cluster address)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D[tmem of both CTAs] (+)= A[smem of both] B[smem of both]^T, issued by the leader
__device__ __forceinline__ void umma2_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this offset in both CTAs of the pair once the
// leader's MMAs issued so far are done
__device__ __forceinline__ void umma2_commit_both(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], m;\n\t}" ::"r"(bar)
      : "memory");
}

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
  long long n_tiles;  // pair tiles: 256-row tiles x column tiles
  long long n_mt;     // 128-row tiles
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
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const long long pair0 = blockIdx.x >> 1;
  const long long npairs = gridDim.x >> 1;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + Layout::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * (uint32_t)s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(kStages + s); };
  auto pfull_bar = [&](int s) { return bar0 + 8u * (uint32_t)(2 * kStages + s); };
  auto accf_bar = [&](int j) { return bar0 + 8u * (uint32_t)(3 * kStages + j); };
  auto acce_bar = [&](int j) { return bar0 + 8u * (uint32_t)(3 * kStages + 2 + j); };
  auto xf_bar = [&](int j) { return bar0 + 8u * (uint32_t)(3 * kStages + 4 + j); };
  auto xe_bar = [&](int j) { return bar0 + 8u * (uint32_t)(3 * kStages + 6 + j); };
  const uint32_t done_bar = bar0 + 8u * (uint32_t)(3 * kStages + 8);
  auto stage_addr = [&](int s) { return sbase + (uint32_t)s * kStage; };
  auto xtile_addr = [&](int j) { return sbase + Layout::kXOff + (uint32_t)j * kXTile; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Layout::kTmemSlot);
  float* ctab = reinterpret_cast<float*>(smem + Layout::kTabOff);
  const bool use_tab = geom.n_g <= kTableGroups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(pfull_bar(s), 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(accf_bar(j), 1);
      mbar_init(acce_bar(j), 2 * kEpiWarps);  // the leader's: both CTAs' epilogue warps
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
    tmem_alloc2(sbase + Layout::kTmemSlot, 512u);
    tmem_relinquish2();
  }
  if (use_tab) build_coef_table<5, 4>(ctab, a, b, geom.n_g);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any remote arrival or commit
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ---- TMA producer (each CTA: its x tile, its dout rows, its half of W) ------------
    if (lane == 0) {
      long long kc = 0;  // K steps issued over all tiles (the ring position)
      int i = 0;         // x tiles issued
      for (long long tile = pair0; tile < geom.n_tiles; tile += npairs) {
        const long long pm = tile / geom.n_ct;
        const int n0 = (int)(tile - pm * geom.n_ct) * BN;
        const int m0 = (int)(pm * 2 * BM) + (int)rank * BM;
        const int ncols = geom.d - n0 < BN ? geom.d - n0 : BN;  // a multiple of 64
        const int half = ncols / 2;                              // this CTA's W channels
        const int xb = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        // The x tile goes in after the first ring's worth of this tile's operand
        // loads: its buffer frees when the epilogue of tile i - 1 starts, i.e.
        // when the product of tile i - 1 is done, and waiting for that first
        // would drain the ring at every tile.
        const int xpos = geom.kt < kStages ? geom.kt : kStages;
        auto load_x = [&]() -> bool {
          if (use >= 1 && !mbar_wait_sleep(xe_bar(xb), (use - 1) & 1u)) return false;
          mbar_arrive_expect_tx(xf_bar(xb), (uint32_t)(ncols / 32) * kXBox);
          for (int j = 0; j < ncols / 32; ++j)
            tma_load_2d(xtile_addr(xb) + (uint32_t)j * kXBox, &mx, n0 + 32 * j, m0, xf_bar(xb));
          return true;
        };
        for (int kt = 0; kt <= geom.kt; ++kt, ++kc) {
          if (kt == xpos) {
            if (!load_x()) {
              report(kErrEmptyWait);
              ok = false;
              break;
            }
            ++i;  // x loads issued
          }
          if (kt == geom.kt) break;
          const int s = (int)(kc % kStages);
          const uint32_t round = (uint32_t)(kc / kStages);
          if (kc >= kStages && !mbar_wait_sleep(empty_bar(s), (round + 1) & 1u)) {
            report(kErrEmptyWait);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(s), kATile + (uint32_t)(half / 32) * kWBox);
          tma_load_2d(stage_addr(s), &mdo, kt * BK, m0, full_bar(s));
          for (int j = 0; j < half / 32; ++j)
            tma_load_2d(stage_addr(s) + kATile + (uint32_t)j * kWBox, &mw,
                        n0 + (int)rank * half + 32 * j, kt * BK, full_bar(s));
        }
        if (!ok) break;
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
    if (leader && lane == 0) {
      // ---- MMA issue (leader) -------------------------------------------------------
      long long kc = 0;
      int i = 0;
      for (long long tile = pair0; tile < geom.n_tiles; tile += npairs, ++i) {
        const long long pm = tile / geom.n_ct;
        const int n0 = (int)(tile - pm * geom.n_ct) * BN;
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
          const uint32_t ph = (uint32_t)(kc / kStages) & 1u;
          if (!mbar_wait_sleep(full_bar(s), ph) || !mbar_wait_sleep(pfull_bar(s), ph)) {
            report(kErrFullWait);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_k_desc(stage_addr(s));
          const uint64_t bd = sw64_mn_desc(stage_addr(s) + kATile);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // A: 32 bytes along the row; B: two 512-byte atoms
            umma2_bf16(dt, ad + 2u * (uint64_t)k, bd + 64u * (uint64_t)k, idesc,
                       (kt > 0 || k > 0) ? 1u : 0u);
          umma2_commit_both(empty_bar(s));  // the stage is free in both CTAs
        }
        if (!ok) break;
        umma2_commit_both(accf_bar(ab));
      }
      // no MMA may still write TMEM when the columns are freed
      umma2_commit_both(done_bar);
      if (!mbar_wait(done_bar, 0)) report(kErrReduceWait);
    } else if (!leader && lane == 0) {
      // ---- tell the leader when each of this CTA's stages has landed -------------------
      long long kc = 0;
      const uint32_t lead_pfull0 = peer_addr(pfull_bar(0), 0);
      for (long long tile = pair0; tile < geom.n_tiles && ok; tile += npairs) {
        for (int kt = 0; kt < geom.kt; ++kt, ++kc) {
          const int s = (int)(kc % kStages);
          if (!mbar_wait_sleep(full_bar(s), (uint32_t)(kc / kStages) & 1u)) {
            report(kErrFullWait);
            ok = false;
            break;
          }
          mbar_arrive_cluster(lead_pfull0 + 8u * (uint32_t)s);
        }
      }
    }
  } else {
    // ---- epilogue: the GR-KAN backward on the accumulator -----------------------------
    const int q = warp & 3;           // TMEM lane quarter: rows 32 q .. 32 q + 31
    const int w3 = (warp - 2) >> 2;   // channels 64 w3 .. 64 w3 + 63 of the tile
    const int r = 32 * q + lane;      // this thread's row in the CTA's 128
    const int swz = (r >> 1) & 3;     // 64-byte swizzle of the row
    const uint32_t lead_acce0 = peer_addr(acce_bar(0), 0);
    Coef54 c;
    int cur_g = -1;
    int i = 0;
    for (long long tile = pair0; tile < geom.n_tiles; tile += npairs, ++i) {
      const long long pm = tile / geom.n_ct;
      const int n0 = (int)(tile - pm * geom.n_ct) * BN;
      const long long mt = pm * 2 + rank;  // this CTA's 128-row tile
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
        bulk_wait_read_all();
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
      // the accumulator columns are read: tell the leader's MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_acce0 + 8u * (uint32_t)ab);
      if (active) {
        fence_proxy_async_smem();  // generic-proxy dx writes before the TMA store reads them
        __syncwarp();
        if (lane == 0 && (long long)m0 + 32 * q < geom.rows) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            tma_store_2d(&mdx, n0 + 64 * w3 + 32 * hh, m0 + 32 * q,
                         xtile_addr(ab) + (uint32_t)(2 * w3 + hh) * kXBox + (uint32_t)q * kXSub);
          bulk_commit();
        }
        // the block's partial sums, fixed order: the two lanes of each pair, then
        // a recursive-halving exchange over the warp's 32 rows
        float sv[16];
        Deg<5, 4>::sums<16>(acc, sv);
        warp_sum<16>(sv, lane);
        const int k = (lane >> 1) & 15;
        const long long slot = (mt * geom.nbg + (cb - g * geom.nbg)) * 4 + q;
        if (mt < geom.n_mt && (lane & 1) == 0 && k < 10)
          ws[((long long)g * 10 + k) * geom.ws_T + slot] = sv[0];
      }
    }
    if (lane == 0) bulk_wait_all();  // this warp's stores are complete
    __syncwarp();
  }
  // teardown: both CTAs are done with the accumulators and with each other's
  // barriers; free the accumulator columns
  __syncwarp();  // the cluster barrier is warp-aligned
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_d, 512u);
  }
}

}  // namespace dg
}  // namespace lin
}  // namespace grk
