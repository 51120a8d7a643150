// grkan_linear_quad.cuh -- the GR-KAN activation fused into the following linear
// layer on clusters of four CTAs, so that every element of x is activated once
// for up to 1024 outputs and W crosses L2 once per 256 rows:
//
//   out[r, o] = sum_k y[r, k] W[o, k] (+ bias[o]),   y = P(x) / (1 + |Q(x)|)
//
// The cluster is two tcgen05 CTA pairs (cta_group::2, M = 256). Rank 2p + h:
// pair p computes outputs [p NP, (p + 1) NP) of the cluster's column tile, half
// h holds rows [128 h, 128 h + 128) of the cluster's 256-row tile. The two CTAs
// with the same h (ranks h and h + 2, "partners") need the same activated rows:
// each loads 64 of them raw, activates them into its own operand tile and
// copies the result into the partner's with one bulk shared-to-shared copy, so
// the activation of a tile is split four ways and done once.
//
// Three rings per CTA, each with its own depth, so that no load waits for the
// activation and the activation never waits for a load:
//   raw   the CTA's 64 raw x rows of a K step of 64 (8 KiB), TMA-loaded;
//   A     the activated 128 x 64 operand tile of the pair MMA (16 KiB): one
//         half written by this CTA's transform threads, the other copied in by
//         the partner;
//   W     the CTA's NP / 2 rows of W for the K step (NP / 2 x 128 bytes),
//         TMA-loaded with completion counted on the pair leader's barrier.
// All operand tiles are K-major with the 128-byte swizzle.
//
// Persistent: the cluster walks its tiles (256 rows x 2 NP outputs) in a fixed
// stride. Per CTA:
//   warp 0       lane 0 loads the raw ring;
//   warp 1       allocates 512 TMEM columns (one NP-column accumulator). In the
//                pair leader (h = 0) lane 0 issues the MMAs (M 256, N up to
//                256 each, K 16) once the W stage and both CTAs' A stages are
//                complete, then releases the W stage in the pair and the A stage
//                in all four CTAs with multicast commits. In the other CTA lane
//                0 tells the leader when its A stage is complete;
//   warp 2       lane 0 loads the W ring;
//   8 warps      activate two 16-byte chunks each per K step: raw slot ->
//                registers -> activation -> this CTA's half of the A stage. The
//                last of the eight warps to finish a stage (a shared counter)
//                copies the half into the partner's stage and marks it ready;
//   4 warps      the epilogue: read the accumulator (one TMEM lane quarter
//                each), add the bias, convert to bf16 and write the tile with
//                TMA stores through 128-byte-swizzled staging buffers, then free
//                the accumulator for the next tile.
// Warp w runs on scheduler w % 4. The transform warps are placed off warp 1's
// scheduler: they wake on the same stage releases that the MMA issuer waits
// for, and sharing its scheduler slowed the issue of the next K step's MMAs.
// Every wait is bounded (device error word), and TMEM is freed on every path.
#pragma once

#include "grkan_linear_bwd.cuh"

// 1: grkan_linear_forward takes this kernel for n_out > 512 (use_linear_quad in
// grkan_api.cu); 2: whenever d is a multiple of 64; 0: never.
#ifndef GRK_LIN_QUAD
#define GRK_LIN_QUAD 1
#endif

namespace grk {
namespace lin {
namespace qd {

using dg::cluster_rank;
using dg::cluster_sync;
using dg::peer_addr;
using dg::sw128_k_desc;
using dg::tmem_alloc2;
using dg::tmem_dealloc2;
using dg::tmem_relinquish2;
using dg::umma2_bf16;

constexpr int BM = 128;          // rows per CTA; a pair covers 256 (UMMA M)
constexpr int BK = 64;           // K per stage: one 128-byte swizzle row of bf16
// Ring depths and epilogue staging buffers per warp (launch-shape knobs). The
// operand ring is GRK_QD_A_STAGES deep for pair tiles of up to 384 outputs and
// 5 deep for 512 (whose W stages are larger); the W ring takes what shared
// memory is left.
#ifndef GRK_QD_RAW_STAGES
#define GRK_QD_RAW_STAGES 2
#endif
#ifndef GRK_QD_A_STAGES
#define GRK_QD_A_STAGES 7
#endif
#ifndef GRK_QD_EPI_BUFS
#define GRK_QD_EPI_BUFS 1
#endif
constexpr int kRawStages = GRK_QD_RAW_STAGES;
constexpr int kAStagesMax = GRK_QD_A_STAGES;
static_assert(kAStagesMax >= 5, "the operand ring's depth at the widest tiles");
constexpr int kEpiBufs = GRK_QD_EPI_BUFS;
constexpr int kWStagesMax = 6;
constexpr int kNPMax = 512;      // outputs per pair: the TMEM columns
constexpr int kXformWarps = 8;
constexpr int kEpiWarps = 4;
// Warp roles: 0 x producer, 1 MMA issue (leader) or forwarder, 2 W producer;
// transform warps 4, 8, 12, 6, 10, 14, 3, 7 (in their index order); epilogue
// warps 16, 5, 18, 15 (an epilogue warp reads TMEM lane quarter warp % 4, so
// these cover the 128 lanes); warps 9, 11, 13, 17, 19 idle. Warp 1's scheduler
// (warps 1, 5, 9, ...) holds no transform warp.
constexpr int kWarps = 20;
constexpr int kThreads = kWarps * 32;
__device__ __forceinline__ int xform_index(int w) {
  switch (w) {
    case 4: return 0;
    case 8: return 1;
    case 12: return 2;
    case 6: return 3;
    case 10: return 4;
    case 14: return 5;
    case 3: return 6;
    case 7: return 7;
    default: return -1;
  }
}
__device__ __forceinline__ int epi_index(int w) {
  return w == 16 ? 0 : w == 5 ? 1 : w == 18 ? 2 : w == 15 ? 3 : -1;
}
constexpr unsigned kRaw = 64 * BK * 2;            // 8 KiB: the CTA's 64 raw rows
constexpr unsigned kATile = 2 * kRaw;             // 16 KiB: the CTA's 128 operand rows
constexpr unsigned kWBox = 64 * BK * 2;           // 8 KiB: 64 W rows
constexpr unsigned kEpiBuf = 32 * 64 * 2;         // 4 KiB: 32 rows x 64 outputs
static_assert(kXformWarps * 32 * 2 == 64 * (BK / 8), "two 16-byte chunks per transform thread");
static_assert(kEpiBufs == 1 || kEpiBufs == 2, "one or two staging buffers per epilogue warp");

// Shared memory, from a 1024-byte aligned base: raw ring, A ring, epilogue
// staging, then the W ring (its stage size depends on NP, its depth is chosen
// to fill what is left), the barriers, the TMEM slot, the per-A-stage counters
// of finished transform warps and the coefficient table. Everything after the
// raw ring depends on NP.
struct Layout {
  static constexpr unsigned kAOff = kRawStages * kRaw;
  // xfull[R], xempty[R], aready[Amax], aempty[Amax], wfull[Wmax], wempty[Wmax],
  // acc_full, acc_empty, done
  static constexpr unsigned kNumBars = 2 * kRawStages + 2 * kAStagesMax + 2 * kWStagesMax + 3;
  static constexpr unsigned kTail = kNumBars * 8 + 16 + 4 * kAStagesMax + 16 + coef_table_bytes<5, 4>();
  static constexpr unsigned kMaxBytes = 232448 - 1024;  // the opt-in limit less the alignment slack
  __host__ __device__ static constexpr int a_stages(int np) { return np > 384 ? 5 : kAStagesMax; }
  __host__ __device__ static constexpr unsigned stg_off(int np) {
    return kAOff + (unsigned)a_stages(np) * kATile;
  }
  __host__ __device__ static constexpr unsigned w_off(int np) {
    return stg_off(np) + kEpiWarps * kEpiBufs * kEpiBuf;
  }
  // bytes of a W stage (the CTA's NP / 2 rows) and the ring depth that fits
  __host__ __device__ static constexpr unsigned w_stage(int np) { return (unsigned)(np / 2) * BK * 2; }
  __host__ __device__ static constexpr int w_stages(int np) {
    return (int)((kMaxBytes - w_off(np) - kTail) / w_stage(np)) < kWStagesMax
               ? (int)((kMaxBytes - w_off(np) - kTail) / w_stage(np))
               : kWStagesMax;
  }
  __host__ __device__ static constexpr unsigned bar_off(int np) {
    return w_off(np) + (unsigned)w_stages(np) * w_stage(np);
  }
  __host__ __device__ static constexpr unsigned tmem_slot(int np) { return bar_off(np) + kNumBars * 8; }
  __host__ __device__ static constexpr unsigned cnt_off(int np) { return (tmem_slot(np) + 4 + 15) / 16 * 16; }
  __host__ __device__ static constexpr unsigned tab_off(int np) {
    return (cnt_off(np) + 4 * kAStagesMax + 15) / 16 * 16;
  }
  __host__ __device__ static constexpr unsigned alloc(int np) {
    return tab_off(np) + coef_table_bytes<5, 4>() + 1024;
  }
};
// the largest of Layout::alloc over the four widths (the launch attribute)
constexpr unsigned kAllocMax =
    Layout::alloc(128) > Layout::alloc(256)
        ? (Layout::alloc(128) > Layout::alloc(384)
               ? (Layout::alloc(128) > Layout::alloc(512) ? Layout::alloc(128) : Layout::alloc(512))
               : (Layout::alloc(384) > Layout::alloc(512) ? Layout::alloc(384) : Layout::alloc(512)))
        : (Layout::alloc(256) > Layout::alloc(384)
               ? (Layout::alloc(256) > Layout::alloc(512) ? Layout::alloc(256) : Layout::alloc(512))
               : (Layout::alloc(384) > Layout::alloc(512) ? Layout::alloc(384) : Layout::alloc(512)));
static_assert(Layout::w_off(128) % 1024 == 0 && Layout::w_off(512) % 1024 == 0,
              "the W ring starts on a swizzle-atom boundary");
static_assert(Layout::w_stages(kNPMax) >= 3 && Layout::w_stages(384) >= 3,
              "three W stages at the widest tiles");
static_assert(kAllocMax <= 232448, "shared memory per CTA");

// Instruction descriptor: float32 accumulator, bf16 A and B, both K-major,
// M = 256 (the pair), N in bits [17, 23) as N / 8.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(2 * BM >> 4) << 24);
__host__ __device__ constexpr uint32_t idesc_n(int n) { return kIdesc | ((uint32_t)(n >> 3) << 17); }

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.cta_group::2"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster)
      : "memory");
}
// Copy `bytes` of this CTA's shared memory to another CTA of the cluster
// (shared::cluster addresses), completing on that CTA's mbarrier.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, uint32_t src, uint32_t bytes,
                                                  uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "r"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Arrive on the barrier at this offset in the CTAs of `mask` once the leader's
// MMAs issued so far are done.
__device__ __forceinline__ void umma2_commit_mask(uint32_t bar, uint16_t mask) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, %1;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], m;\n\t}" ::"r"(bar),
      "h"(mask)
      : "memory");
}
// Arrival on a barrier of any CTA of the cluster, ordering this thread's
// earlier memory operations before it at cluster scope.
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// Two 16-column TMEM loads of this thread's lane, one wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
#pragma unroll
  for (int c = 0; c < 2; ++c)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[16 * c + 0]), "=r"(r[16 * c + 1]), "=r"(r[16 * c + 2]), "=r"(r[16 * c + 3]),
          "=r"(r[16 * c + 4]), "=r"(r[16 * c + 5]), "=r"(r[16 * c + 6]), "=r"(r[16 * c + 7]),
          "=r"(r[16 * c + 8]), "=r"(r[16 * c + 9]), "=r"(r[16 * c + 10]), "=r"(r[16 * c + 11]),
          "=r"(r[16 * c + 12]), "=r"(r[16 * c + 13]), "=r"(r[16 * c + 14]), "=r"(r[16 * c + 15])
        : "r"(taddr + 16u * (uint32_t)c));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Position in a ring of stages: the slot and the parity of its current use. A
// producer waits for the slot's release with the parity flipped, which a fresh
// barrier reports complete, so the first use of every slot does not wait.
struct Ring {
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next(int n) {
    if (++s == n) {
      s = 0;
      ph ^= 1u;
    }
  }
};

struct QGeom {
  long long rows;     // R = B * N
  long long n_tiles;  // 256-row tiles x column tiles
  int d;              // K: input features (the activation's channels), a multiple of 64
  int nout;           // output features
  int dg;             // channels per group
  int n_g;
  int kt;             // K steps = d / BK
  int np;             // outputs per pair: 128, 256, 384 or 512
  int n1, n2;         // the pair's two MMA widths: n1 = min(np, 256), n2 = np - n1
  int n_ct;           // column tiles = ceil(nout / (2 np))
  int ws;             // W ring depth: Layout::w_stages(np)
};

__global__ void __launch_bounds__(kThreads, 1)
linear_fwd_quad(const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mw,
                const __grid_constant__ CUtensorMap mo, const float* __restrict__ a,
                const float* __restrict__ b, const float* __restrict__ bias, const QGeom geom) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t p = rank >> 1;        // outputs [p np, (p + 1) np) of the column tile
  const uint32_t h = rank & 1;         // rows [128 h, 128 h + 128) of the 256-row tile
  const bool leader = h == 0;          // issues the pair's MMAs
  const uint32_t partner = rank ^ 2u;  // same rows, the other pair
  const uint32_t lead = rank & ~1u;    // this pair's leader
  const long long cl0 = blockIdx.x >> 2;
  const long long ncl = gridDim.x >> 2;
  const int WS = geom.ws;
  const uint32_t wbytes = Layout::w_stage(geom.np);  // this CTA's W rows of a K step
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + Layout::bar_off(geom.np);
  constexpr int R = kRawStages;
  const int A = Layout::a_stages(geom.np);
  auto xfull_bar = [&](int s) { return bar0 + 8u * (uint32_t)s; };
  auto xempty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(R + s); };
  auto aready_bar = [&](int s) { return bar0 + 8u * (uint32_t)(2 * R + s); };
  constexpr int AM = kAStagesMax;
  auto aempty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(2 * R + AM + s); };
  auto wfull_bar = [&](int s) { return bar0 + 8u * (uint32_t)(2 * R + 2 * AM + s); };
  auto wempty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(2 * R + 2 * AM + kWStagesMax + s); };
  const uint32_t accf_bar = bar0 + 8u * (uint32_t)(2 * R + 2 * AM + 2 * kWStagesMax);
  const uint32_t acce_bar = accf_bar + 8u;
  const uint32_t done_bar = accf_bar + 16u;
  auto raw_addr = [&](int s) { return sbase + (uint32_t)s * kRaw; };
  auto a_addr = [&](int s) { return sbase + Layout::kAOff + (uint32_t)s * kATile; };
  auto w_addr = [&](int s) { return sbase + Layout::w_off(geom.np) + (uint32_t)s * wbytes; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Layout::tmem_slot(geom.np));
  unsigned* xcnt = reinterpret_cast<unsigned*>(smem + Layout::cnt_off(geom.np));
  float* ctab = reinterpret_cast<float*>(smem + Layout::tab_off(geom.np));
  const bool use_tab = geom.n_g <= kTableGroups;
  const uint16_t pair_mask = (uint16_t)(3u << (2 * p));

  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(xfull_bar(s), 1);             // the producer's arming; the raw bytes
      mbar_init(xempty_bar(s), kXformWarps);  // every transform warp has read the slot
    }
    for (int s = 0; s < A; ++s) {
      xcnt[s] = 0u;
      // the last transform warp's arming (this half; the partner's half as
      // bytes), and in the leader the other CTA's forwarder
      mbar_init(aready_bar(s), leader ? 2 : 1);
      mbar_init(aempty_bar(s), 2);           // both leaders' MMAs are done with it
    }
    for (int s = 0; s < WS; ++s) {
      mbar_init(wfull_bar(s), 1);   // the leader's: its producer's arming; both CTAs' bytes
      mbar_init(wempty_bar(s), 1);  // the pair's MMAs are done with it
    }
    mbar_init(accf_bar, 1);
    mbar_init(acce_bar, 2 * kEpiWarps);  // the leader's: both CTAs' epilogue warps
    mbar_init(done_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async_smem();
    prefetch_map(&mx);
    prefetch_map(&mw);
    prefetch_map(&mo);
  }
  if (warp == 1) {
    tmem_alloc2(smem_addr(tmem_slot), (uint32_t)kNPMax);
    tmem_relinquish2();
  }
  if (use_tab) build_coef_table<5, 4>(ctab, a, b, geom.n_g);
  tc_fence_before();
  cluster_sync();  // every CTA's barriers exist before any remote arrival, copy or commit
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      // ---- raw x producer: this CTA's 64 rows of each K step ---------------------------
      long long kc = 0;
      Ring rx;
      for (long long tile = cl0; tile < geom.n_tiles && ok; tile += ncl) {
        const long long mt = tile / geom.n_ct;
        const int xrow = (int)(mt * 2 * BM) + (int)h * BM + (int)p * 64;
        for (int kt = 0; kt < geom.kt; ++kt, ++kc, rx.next(R)) {
          if (!mbar_wait_sleep(xempty_bar(rx.s), rx.ph ^ 1u)) {
            report(kErrEmptyWait);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(xfull_bar(rx.s), kRaw);
          tma_load_2d(raw_addr(rx.s), &mx, kt * BK, xrow, xfull_bar(rx.s));
        }
      }
      // the last load into each slot has landed before the memory can go away
      // (immediate on the normal path)
      for (long long j = kc > R ? kc - R : 0; j < kc; ++j)
        if (!mbar_wait(xfull_bar((int)(j % R)), (uint32_t)(j / R) & 1u)) report(kErrDrainWait);
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // ---- W producer: this CTA's half of the pair's W rows, counted on the leader -----
      const uint32_t lead_wfull0 = peer_addr(wfull_bar(0), lead);
      long long kc = 0;
      Ring rw;
      for (long long tile = cl0; tile < geom.n_tiles && ok; tile += ncl) {
        const long long mt = tile / geom.n_ct;
        const int ct = (int)(tile - mt * geom.n_ct);
        const int wrow = ct * 2 * geom.np + (int)p * geom.np;
        for (int kt = 0; kt < geom.kt; ++kt, ++kc, rw.next(WS)) {
          const int s = rw.s;
          if (!mbar_wait_sleep(wempty_bar(s), rw.ph ^ 1u)) {
            report(kErrEmptyWait);
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(wfull_bar(s), 2u * wbytes);  // both CTAs' rows
          const uint32_t fb = lead_wfull0 + 8u * (uint32_t)s;
          // rows of the first MMA (n1 / 2 from this CTA), then of the second
          for (int j = 0; j < geom.n1 / 128; ++j)
            tma_load_2d_pair(w_addr(s) + (uint32_t)j * kWBox, &mw, kt * BK,
                             wrow + (int)h * (geom.n1 / 2) + 64 * j, fb);
          for (int j = 0; j < geom.n2 / 128; ++j)
            tma_load_2d_pair(w_addr(s) + (uint32_t)(geom.n1 / 2) * (BK * 2) + (uint32_t)j * kWBox,
                             &mw, kt * BK, wrow + geom.n1 + (int)h * (geom.n2 / 2) + 64 * j, fb);
        }
      }
      // The leader waits for the last phase of each slot (both CTAs' bytes).
      // The other CTA cannot see its loads complete; on the normal path the
      // leader's MMAs consumed them before the teardown barrier, and an error
      // path reaches the teardown only after a wait of seconds has run out.
      if (leader)
        for (long long j = kc > WS ? kc - WS : 0; j < kc; ++j)
          if (!mbar_wait(wfull_bar((int)(j % WS)), (uint32_t)(j / WS) & 1u)) report(kErrDrainWait);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ---- MMA issue (pair leader) ------------------------------------------------------
      const uint32_t idesc1 = idesc_n(geom.n1);
      const uint32_t idesc2 = idesc_n(geom.n2 > 0 ? geom.n2 : 16);
      Ring rw, ra;
      int i = 0;
      for (long long tile = cl0; tile < geom.n_tiles; tile += ncl, ++i) {
        if (i >= 1 && !mbar_wait_sleep(acce_bar, (uint32_t)(i - 1) & 1u)) {
          report(kErrEmptyWait);
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < geom.kt; ++kt, rw.next(WS), ra.next(A)) {
          const int sw = rw.s;
          const int sa = ra.s;
          if (!mbar_wait_sleep(wfull_bar(sw), rw.ph) || !mbar_wait_sleep(aready_bar(sa), ra.ph)) {
            report(kErrFullWait);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_k_desc(a_addr(sa));
          const uint64_t bd1 = sw128_k_desc(w_addr(sw));
          const uint64_t bd2 = sw128_k_desc(w_addr(sw) + (uint32_t)(geom.n1 / 2) * (BK * 2));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {  // 16 bf16 = 32 bytes along the row
            const uint32_t acc = (kt > 0 || k > 0) ? 1u : 0u;
            umma2_bf16(tmem_d, ad + 2u * (uint64_t)k, bd1 + 2u * (uint64_t)k, idesc1, acc);
            if (geom.n2 > 0)
              umma2_bf16(tmem_d + (uint32_t)geom.n1, ad + 2u * (uint64_t)k,
                         bd2 + 2u * (uint64_t)k, idesc2, acc);
          }
          umma2_commit_mask(wempty_bar(sw), pair_mask);      // the W stage, in this pair
          umma2_commit_mask(aempty_bar(sa), (uint16_t)0xF);  // the A stage, in all four
        }
        if (!ok) break;
        umma2_commit_mask(accf_bar, pair_mask);
      }
      // no MMA may still write TMEM when the columns are freed
      umma2_commit_mask(done_bar, pair_mask);
      if (!mbar_wait(done_bar, 0)) report(kErrReduceWait);
    } else if (!leader && lane == 0) {
      // ---- forwarder: this CTA's A stage is complete, on the leader's barrier ----------
      const uint32_t lead_ready0 = peer_addr(aready_bar(0), lead);
      const long long n_kc = ((geom.n_tiles - cl0 + ncl - 1) / ncl) * (long long)geom.kt;
      Ring ra;
      for (long long kc = 0; kc < n_kc; ++kc, ra.next(A)) {
        if (!mbar_wait_sleep(aready_bar(ra.s), ra.ph)) {
          report(kErrFullWait);
          break;
        }
        mbar_arrive_release_cluster(lead_ready0 + 8u * (uint32_t)ra.s);
      }
    }
  } else if (xform_index(warp) >= 0) {
    // ---- activation: two 16-byte chunks per thread and K step (rows rr and
    // rr + 32), into this CTA's half of the A stage -----------------------------------------
    const int t = xform_index(warp) * 32 + lane;  // 0 .. 255
    const int rr = t >> 3;  // rows rr and rr + 32 of the CTA's 64 raw rows
    const int j = t & 7;    // logical 16-byte chunk (8 channels) of the 128-byte row
    // 128-byte swizzle (8-row atoms): rows rr and rr + 32 share the xor pattern
    const uint32_t sw = (uint32_t)(j ^ (rr & 7)) << 4;
    const uint32_t raw_off = (uint32_t)rr * 128u + sw;
    const uint32_t a_off = ((uint32_t)p * 64u + (uint32_t)rr) * 128u + sw;
    const uint32_t part_a0 = peer_addr(a_addr(0), partner) + p * kRaw;
    const uint32_t part_ready0 = peer_addr(aready_bar(0), partner);
    long long kc = 0;  // K steps done
    Coef54 c;
    int cur_g = -1;
    Ring rx, ra;
    for (long long tile = cl0; tile < geom.n_tiles && ok; tile += ncl) {
      // the group of this thread's chunk, advanced by 64 channels per K step
      int ch = j * 8;
      int g = ch / geom.dg;
      int gend = (g + 1) * geom.dg;
      for (int kt = 0; kt < geom.kt; ++kt, rx.next(R), ra.next(A), ch += BK) {
        const int sx = rx.s;
        const int sa = ra.s;
        bool got = mbar_wait_sleep(xfull_bar(sx), rx.ph);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) report(kErrFullWait);
          ok = false;
          break;
        }
        const unsigned char* raw = smem + (size_t)sx * kRaw + raw_off;
        uint4 v = *reinterpret_cast<const uint4*>(raw);
        uint4 v2 = *reinterpret_cast<const uint4*>(raw + 32u * 128u);
        __syncwarp();
        if (lane == 0) mbar_arrive(xempty_bar(sx));  // the slot is read
        while (ch >= gend) {  // a chunk lies in one group (d_g % 8 == 0)
          ++g;
          gend += geom.dg;
        }
        if (g != cur_g) {
          load_coef<5, 4>(use_tab, ctab, a, b, g, c);
          cur_g = g;
        }
        v.x = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v.x)));
        v.y = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v.y)));
        v.z = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v.z)));
        v.w = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v.w)));
        v2.x = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v2.x)));
        v2.y = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v2.y)));
        v2.z = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v2.z)));
        v2.w = f2_to_bf16x2(fwd_pair(c, bf16x2_to_f2(v2.w)));
        // the A stage is free in this CTA and the partner once both pairs' MMAs
        // of its previous use are done
        got = mbar_wait_sleep(aempty_bar(sa), ra.ph ^ 1u);
        if (!__all_sync(0xffffffffu, got)) {
          if (lane == 0) report(kErrEmptyWait);
          ok = false;
          break;
        }
        unsigned char* at = smem + Layout::kAOff + (size_t)sa * kATile + a_off;
        *reinterpret_cast<uint4*>(at) = v;
        *reinterpret_cast<uint4*>(at + 32u * 128u) = v2;
        fence_proxy_async_smem();  // before the copy's and the tensor cores' reads
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();  // this warp's writes before its count
          if (atomicAdd(&xcnt[sa], 1u) == (unsigned)kXformWarps - 1u) {
            // the last warp of the stage: every warp's writes are in place;
            // copy this CTA's half into the partner's stage, then mark it ready
            // (the partner's half arrives as bytes on the same barrier)
            __threadfence_block();
            xcnt[sa] = 0u;  // next used after this stage's release
            bulk_copy_to_peer(part_a0 + (uint32_t)sa * kATile, a_addr(sa) + p * kRaw, kRaw,
                              part_ready0 + 8u * (uint32_t)sa);
            mbar_arrive_expect_tx(aready_bar(sa), kRaw);
          }
        }
        ++kc;
      }
    }
    // the partner's last copies into this CTA have landed before its memory can
    // go away (immediate on the normal path)
    if (t == 0)
      for (long long u = kc > A ? kc - A : 0; u < kc; ++u)
        if (!mbar_wait(aready_bar((int)(u % A)), (uint32_t)(u / A) & 1u)) report(kErrDrainWait);
  } else if (epi_index(warp) >= 0) {
    // ---- epilogue: accumulator -> bf16 -> TMA stores --------------------------------------
    const int q = warp & 3;  // TMEM lane quarter: rows 32 q .. 32 q + 31 of the CTA's 128
    const int e = epi_index(warp);
    const unsigned stg_off = Layout::stg_off(geom.np) + (unsigned)e * (unsigned)kEpiBufs * kEpiBuf;
    unsigned char* stg = smem + stg_off;
    const uint32_t stg_a = sbase + stg_off;
    const uint32_t lead_acce = peer_addr(acce_bar, lead);
    long long sc = 0;  // stores issued by this warp
    int i = 0;
    for (long long tile = cl0; tile < geom.n_tiles; tile += ncl, ++i) {
      const bool got = mbar_wait_sleep(accf_bar, (uint32_t)i & 1u);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) report(kErrReduceWait);
        ok = false;
        break;
      }
      tc_fence_after();
      const long long mt = tile / geom.n_ct;
      const int ct = (int)(tile - mt * geom.n_ct);
      const long long row = mt * 2 * BM + (long long)h * BM + 32 * q;
      const int colb = ct * 2 * geom.np + (int)p * geom.np;
      // a quarter wholly past the last row (ragged last tile) has nothing to store
      const int ncb = row < geom.rows ? geom.np / 64 : 0;
      for (int cb = 0; cb < ncb; ++cb, ++sc) {
        const int col0 = colb + 64 * cb;
        if (col0 >= geom.nout) break;
        const int buf = (int)(sc % kEpiBufs);
        if (sc >= kEpiBufs) {  // the store that used this buffer has read it
          if (lane == 0) {
            if (kEpiBufs == 2)
              asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            else
              bulk_wait_read_all();
          }
          __syncwarp();
        }
        unsigned char* sb = stg + buf * kEpiBuf;
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          float v[32];
          tmem_ld32(tmem_d + ((uint32_t)(32 * q) << 16) + (uint32_t)(64 * cb + 32 * hq), v);
          if (bias) {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              const int col = col0 + 32 * hq + x;
              v[x] += col < geom.nout ? __ldg(bias + col) : 0.f;
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {  // 16-byte chunk 4 hq + u of row `lane`
            uint4 w;
            w.x = f2_to_bf16x2(make_float2(v[8 * u + 0], v[8 * u + 1]));
            w.y = f2_to_bf16x2(make_float2(v[8 * u + 2], v[8 * u + 3]));
            w.z = f2_to_bf16x2(make_float2(v[8 * u + 4], v[8 * u + 5]));
            w.w = f2_to_bf16x2(make_float2(v[8 * u + 6], v[8 * u + 7]));
            // 128-byte swizzle: chunk c of row `lane` at ((c ^ (lane & 7)) << 4)
            *reinterpret_cast<uint4*>(sb + lane * 128 + (((4 * hq + u) ^ (lane & 7)) << 4)) = w;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&mo, col0, (int)row, stg_a + (uint32_t)buf * kEpiBuf);
          bulk_commit();
        }
      }
      // the accumulator is read: tell the pair leader's MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_release_cluster(lead_acce);
    }
    if (lane == 0) bulk_wait_all();  // this warp's stores are complete
    __syncwarp();
  }
  // teardown: all four CTAs are done with each other's barriers and stages, and
  // the pair's MMAs are done; free the accumulator columns
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_d, (uint32_t)kNPMax);
  }
}

}  // namespace qd
}  // namespace lin
}  // namespace grk
