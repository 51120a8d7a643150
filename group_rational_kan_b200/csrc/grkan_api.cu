// grkan_api.cu -- the C ABI declared in include/grkan.h: argument checks,
// work partition, kernel selection and launches. No allocation, no host
// synchronisation (except grkan_device_error, which says so).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "grkan.h"
#include "grkan_atomic.cuh"
#include "grkan_common.cuh"
#include "grkan_generic.cuh"
#include "grkan_linear.cuh"
#include "grkan_linear_bwd.cuh"
#include "grkan_linear_quad.cuh"
#include "grkan_merge.cuh"
#include "grkan_tma.cuh"

namespace {

thread_local char g_last_error[256] = "no error";

void set_last_error(const char* where, const char* what, int code) {
  snprintf(g_last_error, sizeof g_last_error, "%s: %s (%d)", where, what, code);
}

// GRKAN_OK, or GRKAN_ERR_CUDA with the failing call recorded for
// grkan_last_error().
grkan_status_t cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return GRKAN_OK;
  set_last_error(where, cudaGetErrorString(e), (int)e);
  return GRKAN_ERR_CUDA;
}

// Work partition. The backward reduces over (row tile x group) units of S rows;
// S depends only on the shape, never on the device or the pointers, so the
// float32 partials -- and therefore dA and dB -- are the same bits on every run.
// For shapes the TMA kernels take, a unit is grk::kBoxesPerUnit TMA boxes of
// the backward (SCw rows x bw channels, about 1.5 KiB); otherwise about 12 KiB
// of rows of one group.
constexpr long long kGenericTileBytes = 12288;
constexpr int kMaxBoxRows = 256;

struct Box {
  int bw = 0;   // channels (0: no box fits)
  int scw = 0;  // rows
  int nbox = 0; // boxes per group row
  unsigned bytes = 0;
};

// The TMA box for a group: width a divisor of d_g of at most 256 elements and a
// whole number of 16-byte vectors, height as many rows as fit in `target` bytes
// (at most 256). Wide rows stream better, so the widest box that fills at least
// three quarters of the target wins; if none does, the fullest box.
Box choose_box(long long dg, int es, unsigned target) {
  Box wide, full;
  if (dg <= 0) return wide;
  for (long long w = dg < 256 ? dg : 256; w >= 1; --w) {
    if (dg % w != 0 || (w * es) % 16 != 0 || (unsigned)(w * es) > target) continue;
    long long rows = target / (unsigned)(w * es);
    if (rows > kMaxBoxRows) rows = kMaxBoxRows;
    Box b;
    b.bw = (int)w;
    b.scw = (int)rows;
    b.nbox = (int)(dg / w);
    b.bytes = (unsigned)(rows * w * es);
    if (wide.bw == 0 && 4ull * b.bytes >= 3ull * target) wide = b;
    if (b.bytes > full.bytes) full = b;
  }
  return wide.bw ? wide : full;
}

struct Plan {
  long long rows = 0, d = 0, dg = 0;
  int n_g = 1, m = 0, n = 0, K = 1, es = 4;
  grkan_dtype_t dtype = GRKAN_F32;
  Box fbox, bbox;   // forward / backward TMA boxes
  long long S = 1;  // rows per tile (unit)
  long long T = 0;  // number of row tiles
  size_t ws_bytes = 0;
};

grkan_status_t make_plan(int64_t B, int64_t N, int64_t d, int32_t n_g, int32_t m, int32_t n,
                         grkan_dtype_t dtype, Plan* p) {
  if (dtype != GRKAN_F32 && dtype != GRKAN_BF16) return GRKAN_ERR_DTYPE;
  if (m < 0 || m > GRKAN_MAX_M || n < 0 || n > GRKAN_MAX_N) return GRKAN_ERR_DEGREE;
  if (B < 0 || N < 0 || d < 0 || n_g < 1) return GRKAN_ERR_SHAPE;
  if (d % n_g != 0) return GRKAN_ERR_SHAPE;
  const long long lim = (1LL << 62);
  if (B != 0 && N > lim / B) return GRKAN_ERR_SHAPE;
  const long long rows = (long long)B * N;
  if (rows != 0 && d > lim / 4 / rows) return GRKAN_ERR_SHAPE;
  p->rows = rows;
  p->d = d;
  p->n_g = n_g;
  p->dg = d / n_g;
  p->m = m;
  p->n = n;
  p->K = m + 1 + n;
  p->dtype = dtype;
  p->es = dtype == GRKAN_F32 ? 4 : 2;
  p->fbox = choose_box(p->dg, p->es, grk::fwd_box_target(dtype == GRKAN_BF16));
  p->bbox = choose_box(p->dg, p->es, grk::bwd_box_target(dtype == GRKAN_BF16));
  if (p->bbox.bw > 0) {
    int per = grk::kBoxesPerUnit / p->bbox.nbox;
    if (per < 1) per = 1;
    p->S = (long long)p->bbox.scw * per;
  } else {
    const long long row_bytes = p->dg * p->es;
    long long s = row_bytes > 0 ? kGenericTileBytes / row_bytes : kMaxBoxRows;
    if (s < 1) s = 1;
    if (s > kMaxBoxRows) s = kMaxBoxRows;
    p->S = s;
  }
  p->T = (rows + p->S - 1) / p->S;
  if (rows == 0 || d == 0) p->T = 0;
  p->ws_bytes = (size_t)p->T * (size_t)n_g * (size_t)p->K * sizeof(float);
  if (p->T > 0 && (long long)n_g * p->T > (1LL << 31) - 1) return GRKAN_ERR_SHAPE;
  return GRKAN_OK;
}

bool overlaps(const void* p, size_t pb, const void* q, size_t qb) {
  if (!p || !q || pb == 0 || qb == 0) return false;
  const uintptr_t a = (uintptr_t)p, b = (uintptr_t)q;
  return a < b + qb && b < a + pb;
}

// Partial overlap is an error; exact aliasing is allowed where documented.
bool bad_alias(const void* in, const void* out, size_t bytes) {
  return in != out && overlaps(in, bytes, out, bytes);
}

bool is_sm100() {
  static std::once_flag once;
  static int ok = 0;
  std::call_once(once, [] {
    int dev = 0;
    cudaDeviceProp prop;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaGetDeviceProperties(&prop, dev) == cudaSuccess)
      ok = (prop.major == 10) ? 1 : 0;
  });
  return ok != 0;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Dispatch of the generic kernels on the element type.
template <class IO>
cudaError_t launch_generic_fwd(const Plan& p, const void* x, void* y, const float* a,
                               const float* b, cudaStream_t st) {
  const long long units = p.T * p.n_g;
  grk::fwd_generic<IO, GRKAN_MAX_M, GRKAN_MAX_N><<<(unsigned)units, grk::kGenericThreads, 0, st>>>(
      (const typename IO::T*)x, (typename IO::T*)y, a, b, p.rows, p.d, (int)p.dg, p.n_g, p.m, p.n,
      (int)p.S);
  return cudaGetLastError();
}

template <class IO>
cudaError_t launch_generic_bwd(const Plan& p, const void* x, const void* dy, void* dx,
                               const float* a, const float* b, float* ws, long long ws_T,
                               long long tile0, cudaStream_t st) {
  const long long units = p.T * p.n_g;
  grk::bwd_generic<IO, GRKAN_MAX_M, GRKAN_MAX_N><<<(unsigned)units, grk::kGenericThreads, 0, st>>>(
      (const typename IO::T*)x, (const typename IO::T*)dy, (typename IO::T*)dx, a, b, ws, p.rows,
      p.d, (int)p.dg, p.n_g, p.m, p.n, (int)p.S, ws_T, tile0);
  return cudaGetLastError();
}

cudaError_t launch_merge(const Plan& p, const float* ws, float* dA, float* dB, double* sums64,
                         cudaStream_t st) {
  const long long outs = (long long)p.n_g * p.K;
  grk::merge_partials<<<(unsigned)outs, grk::kMergeThreads, 0, st>>>(ws, dA, dB, sums64, p.T,
                                                                      p.n_g, p.m, p.n);
  return cudaGetLastError();
}

// --- path selection ----------------------------------------------------------

bool tma_degree_supported(int m, int n) { return grk::tma_has_degree(m, n); }

bool tma_shape_ok(const Plan& p) {
  if (p.rows <= 0 || p.d <= 0) return false;
  if ((p.d * p.es) % 16 != 0 || (p.dg * p.es) % 16 != 0) return false;
  if (p.rows > 0x7fffffffLL || p.d > 0x7fffffffLL) return false;
  // the kernels keep a lane's byte offsets inside a box (up to scw rows of d
  // elements) in 32-bit integers
  const long long scw = p.fbox.scw > p.bbox.scw ? p.fbox.scw : p.bbox.scw;
  if (scw * p.d * p.es >= 0x7fffffffLL) return false;
  // both boxes exist and every box starts on a 128-byte shared-memory boundary
  // (slots are rounded up to 128 bytes)
  return p.fbox.bw > 0 && p.bbox.bw > 0;
}

int choose_fwd_path(const Plan& p, const void* x, const void* y, uint32_t flags) {
  if (flags & GRKAN_FLAG_GENERIC) return 0;
  if (!tma_degree_supported(p.m, p.n) || !tma_shape_ok(p)) return 0;
  if (!aligned16(x) || !aligned16(y)) return 0;
  return 1;
}

int choose_bwd_path(const Plan& p, const void* x, const void* dy, const void* dx,
                    uint32_t flags) {
  if (flags & GRKAN_FLAG_GENERIC) return 0;
  if (!tma_degree_supported(p.m, p.n) || !tma_shape_ok(p)) return 0;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx)) return 0;
  return 1;
}

// --- TMA tensor maps -----------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

// 2-D map over the (rows, d) tensor, box = (bw columns, scw rows).
bool make_map(CUtensorMap* map, const void* base, const Plan& p, const Box& bx) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_last_error("cudaGetDriverEntryPoint", "cuTensorMapEncodeTiled not found", 0);
    return false;
  }
  const cuuint64_t dims[2] = {(cuuint64_t)p.d, (cuuint64_t)p.rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(p.d * p.es)};
  const cuuint32_t box[2] = {(cuuint32_t)bx.bw, (cuuint32_t)bx.scw};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      p.dtype == GRKAN_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) set_last_error("cuTensorMapEncodeTiled", "failed", (int)r);
  return r == CUDA_SUCCESS;
}

grk::TmaGeom make_geom(const Plan& p, const Box& bx) {
  grk::TmaGeom g;
  g.rows = p.rows;
  g.T = p.T;
  g.ws_T = p.T;
  g.ws_tile0 = 0;
  g.d = p.d;
  g.S = p.S;
  g.dg = (int)p.dg;
  g.n_g = p.n_g;
  g.SCw = bx.scw;
  g.bw = bx.bw;
  g.nbox = bx.nbox;
  g.box_bytes = bx.bytes;
  g.m = p.m;
  g.n = p.n;
  g.nrb_full = (int)((p.S + bx.scw - 1) / bx.scw);
  const long long last = p.T > 0 ? p.rows - (p.T - 1) * p.S : 0;
  g.nrb_last = (int)((last + bx.scw - 1) / bx.scw);
  return g;
}

int sm_count() {
  static std::once_flag once;
  static int sms = 148;
  std::call_once(once, [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      sms = v;
  });
  return sms;
}

grkan_status_t launch_tma_fwd(const Plan& p, const void* x, void* y, const float* a,
                              const float* b, cudaStream_t st) {
  CUtensorMap mx, my;
  if (!make_map(&mx, x, p, p.fbox) || !make_map(&my, y, p, p.fbox)) return GRKAN_ERR_CUDA;
  const grk::TmaGeom geom = make_geom(p, p.fbox);
  cudaError_t e =
      grk::launch_fwd_tma(p.dtype == GRKAN_BF16, geom, mx, my, y, a, b, sm_count(), st);
  return cuda_status(e, "forward (TMA) launch");
}

grkan_status_t launch_tma_bwd(const Plan& p, const void* x, const void* dy, void* dx, void* y,
                              const float* a, const float* b, float* ws, long long ws_T,
                              long long tile0, cudaStream_t st) {
  CUtensorMap mx, mdy, mdx;
  if (!make_map(&mx, x, p, p.bbox) || !make_map(&mdy, dy, p, p.bbox) ||
      !make_map(&mdx, dx, p, p.bbox))
    return GRKAN_ERR_CUDA;
  grk::TmaGeom geom = make_geom(p, p.bbox);
  geom.ws_T = ws_T;
  geom.ws_tile0 = tile0;
  cudaError_t e = grk::launch_bwd_tma(p.dtype == GRKAN_BF16, geom, mx, mdy, mdx, dx, y, a, b, ws,
                                      sm_count(), st);
  return cuda_status(e, "backward (TMA) launch");
}

grkan_status_t check_coef_ptrs(const Plan& p, const float* a, const float* b) {
  if (!a) return GRKAN_ERR_NULL;
  if (p.n > 0 && !b) return GRKAN_ERR_NULL;
  return GRKAN_OK;
}

grkan_status_t do_forward(const void* x, void* y, const float* a, const float* b, int64_t B,
                          int64_t N, int64_t d, int32_t n_g, int32_t m, int32_t n,
                          grkan_dtype_t dtype, uint32_t flags, void* stream) {
  if (flags & ~GRKAN_FLAG_GENERIC) return GRKAN_ERR_FLAGS;
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if (p.rows == 0 || p.d == 0) return GRKAN_OK;
  if (!x || !y) return GRKAN_ERR_NULL;
  if ((s = check_coef_ptrs(p, a, b)) != GRKAN_OK) return s;
  const size_t bytes = (size_t)p.rows * (size_t)p.d * (size_t)p.es;
  if (bad_alias(x, y, bytes)) return GRKAN_ERR_ALIAS;
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  cudaStream_t st = (cudaStream_t)stream;
  if (choose_fwd_path(p, x, y, flags) == 1) return launch_tma_fwd(p, x, y, a, b, st);
  cudaError_t e = (dtype == GRKAN_F32) ? launch_generic_fwd<grk::IoF32>(p, x, y, a, b, st)
                                       : launch_generic_fwd<grk::IoBF16>(p, x, y, a, b, st);
  return cuda_status(e, "forward (generic) launch");
}

// Stage 1 into the workspace; the partials of this call's tiles go to tiles
// [tile0, tile0 + p.T) of a workspace laid out for ws_T tiles (a whole tensor).
// With y != nullptr the forward output is written too (one pass over x, dy on the
// TMA path; a forward kernel first on the generic path).
grkan_status_t do_partials_at(const Plan& p, const void* x, const void* dy, const float* a,
                              const float* b, void* dx, void* y, void* ws, long long ws_T,
                              long long tile0, uint32_t flags, cudaStream_t st) {
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  if (choose_bwd_path(p, x, dy, dx, flags) == 1 &&
      (!y || (aligned16(y) && grk::tma_has_fused_degree(p.m, p.n))))
    return launch_tma_bwd(p, x, dy, dx, y, a, b, (float*)ws, ws_T, tile0, st);
  if (y) {
    cudaError_t e = (p.dtype == GRKAN_F32) ? launch_generic_fwd<grk::IoF32>(p, x, y, a, b, st)
                                           : launch_generic_fwd<grk::IoBF16>(p, x, y, a, b, st);
    grkan_status_t s = cuda_status(e, "forward (generic) launch");
    if (s != GRKAN_OK) return s;
  }
  cudaError_t e =
      (p.dtype == GRKAN_F32)
          ? launch_generic_bwd<grk::IoF32>(p, x, dy, dx, a, b, (float*)ws, ws_T, tile0, st)
          : launch_generic_bwd<grk::IoBF16>(p, x, dy, dx, a, b, (float*)ws, ws_T, tile0, st);
  return cuda_status(e, "backward (generic) launch");
}

grkan_status_t do_partials(const Plan& p, const void* x, const void* dy, const float* a,
                           const float* b, void* dx, void* ws, size_t ws_bytes, uint32_t flags,
                           cudaStream_t st) {
  if (!x || !dy || !dx) return GRKAN_ERR_NULL;
  grkan_status_t s = check_coef_ptrs(p, a, b);
  if (s != GRKAN_OK) return s;
  if (!ws || ws_bytes < p.ws_bytes || !aligned16(ws)) return GRKAN_ERR_WORKSPACE;
  const size_t bytes = (size_t)p.rows * (size_t)p.d * (size_t)p.es;
  // dx may replace dy (read before written) but never x, which stays readable
  if (overlaps(x, bytes, dx, bytes) || bad_alias(dy, dx, bytes)) return GRKAN_ERR_ALIAS;
  if (overlaps(ws, p.ws_bytes, x, bytes) || overlaps(ws, p.ws_bytes, dy, bytes) ||
      overlaps(ws, p.ws_bytes, dx, bytes))
    return GRKAN_ERR_ALIAS;
  return do_partials_at(p, x, dy, a, b, dx, nullptr, ws, p.T, 0, flags, st);
}

grkan_status_t do_merge(const Plan& p, const void* ws, size_t ws_bytes, float* dA, float* dB,
                        double* sums64, cudaStream_t st) {
  if (!dA || (p.n > 0 && !dB)) return GRKAN_ERR_NULL;
  if (p.T > 0 && (!ws || ws_bytes < p.ws_bytes)) return GRKAN_ERR_WORKSPACE;
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  cudaError_t e = launch_merge(p, (const float*)ws, dA, dB, sums64, st);
  return cuda_status(e, "merge launch");
}

// Scratch for grkan_backward_noalloc: file-scope static device memory, one copy
// per device that loads the library. Host code must not pass the symbol itself
// to a kernel (in host code it names a host-side stand-in); it looks up the
// device address once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_ws[GRKAN_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_ws on the current device (looked up on first use).
grkan_status_t noalloc_workspace(void** out) {
  int dev = 0;
  grkan_status_t s = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (s != GRKAN_OK) return s;
  if (dev < 0 || dev >= kMaxDevices) return GRKAN_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    s = cuda_status(cudaGetSymbolAddress(&p, g_noalloc_ws), "cudaGetSymbolAddress");
    if (s != GRKAN_OK) return s;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return GRKAN_OK;
}

// --- host-buffer step: row chunks streamed through device staging -------------------
//
// Three streams per device (created on first use and kept): host-to-device
// copies, kernels, device-to-host copies. Chunk c uses staging slot c % kSlots;
// a slot is refilled only after its previous results have left the device.
// Chunks are whole row tiles, so the partial sums land exactly where a single
// grkan_backward would put them and the merged gradients are the same bits.

constexpr int kSlots = 3;
constexpr long long kChunkTarget = 32LL << 20;  // bytes of one tensor chunk

struct HostPipe {
  cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr, comp_done = nullptr, out_done = nullptr;
  cudaEvent_t in[kSlots] = {}, comp[kSlots] = {}, out[kSlots] = {};
  bool ready = false;
};

std::mutex g_pipe_mutex;
HostPipe g_pipe[kMaxDevices];

grkan_status_t pipe_for_device(int dev, HostPipe** out) {
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    const unsigned fl = cudaStreamNonBlocking;
    grkan_status_t s = cuda_status(cudaStreamCreateWithFlags(&hp.s_in, fl), "cudaStreamCreate");
    if (s == GRKAN_OK) s = cuda_status(cudaStreamCreateWithFlags(&hp.s_comp, fl), "cudaStreamCreate");
    if (s == GRKAN_OK) s = cuda_status(cudaStreamCreateWithFlags(&hp.s_out, fl), "cudaStreamCreate");
    cudaEvent_t* evs[] = {&hp.start, &hp.comp_done, &hp.out_done};
    for (cudaEvent_t* e : evs)
      if (s == GRKAN_OK)
        s = cuda_status(cudaEventCreateWithFlags(e, cudaEventDisableTiming), "cudaEventCreate");
    for (int i = 0; i < kSlots && s == GRKAN_OK; ++i) {
      s = cuda_status(cudaEventCreateWithFlags(&hp.in[i], cudaEventDisableTiming), "cudaEventCreate");
      if (s == GRKAN_OK)
        s = cuda_status(cudaEventCreateWithFlags(&hp.comp[i], cudaEventDisableTiming),
                        "cudaEventCreate");
      if (s == GRKAN_OK)
        s = cuda_status(cudaEventCreateWithFlags(&hp.out[i], cudaEventDisableTiming),
                        "cudaEventCreate");
    }
    if (s != GRKAN_OK) return s;
    hp.ready = true;
  }
  *out = &hp;
  return GRKAN_OK;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Rows per chunk: a whole number of row tiles, about kChunkTarget bytes of one
// tensor (or what the caller asked for, rounded up to whole tiles).
long long chunk_rows_for(const Plan& p, long long want) {
  long long rows = want > 0 ? want : kChunkTarget / (p.d * p.es > 0 ? p.d * p.es : 1);
  if (rows < p.S) rows = p.S;
  rows = (rows + p.S - 1) / p.S * p.S;
  if (rows > p.rows) rows = (p.rows + p.S - 1) / p.S * p.S;
  return rows < 1 ? 1 : rows;
}

struct StagingLayout {
  long long chunk_rows = 0;
  size_t tensor = 0;  // bytes of one chunk buffer
  size_t ws_off = 0, grad_off = 0, total = 0;
};

StagingLayout staging_layout(const Plan& p, long long want_rows) {
  StagingLayout L;
  L.chunk_rows = chunk_rows_for(p, want_rows);
  L.tensor = align256((size_t)L.chunk_rows * (size_t)p.d * (size_t)p.es);
  L.ws_off = (size_t)kSlots * 4 * L.tensor;  // per slot: x, dy, y, dx
  L.grad_off = L.ws_off + align256(p.ws_bytes);
  L.total = L.grad_off + align256((size_t)p.n_g * (size_t)p.K * sizeof(float));
  return L;
}

}  // namespace

extern "C" {

grkan_status_t grkan_forward(const void* x, void* y, const float* a, const float* b, int64_t B,
                             int64_t N, int64_t d, int32_t n_g, int32_t m, int32_t n,
                             grkan_dtype_t dtype, void* stream) {
  return do_forward(x, y, a, b, B, N, d, n_g, m, n, dtype, 0u, stream);
}

grkan_status_t grkan_forward_ex(const void* x, void* y, const float* a, const float* b, int64_t B,
                                int64_t N, int64_t d, int32_t n_g, int32_t m, int32_t n,
                                grkan_dtype_t dtype, uint32_t flags, void* stream) {
  return do_forward(x, y, a, b, B, N, d, n_g, m, n, dtype, flags, stream);
}

size_t grkan_backward_workspace_bytes(int64_t B, int64_t N, int64_t d, int32_t n_g, int32_t m,
                                      int32_t n, grkan_dtype_t dtype) {
  Plan p;
  if (make_plan(B, N, d, n_g, m, n, dtype, &p) != GRKAN_OK) return 0;
  return p.ws_bytes;
}

grkan_status_t grkan_backward_partials(const void* x, const void* dy, const float* a,
                                       const float* b, void* dx, int64_t B, int64_t N, int64_t d,
                                       int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                                       void* workspace, size_t workspace_bytes, uint32_t flags,
                                       void* stream) {
  if (flags & ~GRKAN_FLAG_GENERIC) return GRKAN_ERR_FLAGS;
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if (p.T == 0) return GRKAN_OK;
  return do_partials(p, x, dy, a, b, dx, workspace, workspace_bytes, flags,
                     (cudaStream_t)stream);
}

grkan_status_t grkan_backward_merge(const void* workspace, size_t workspace_bytes, float* dA,
                                    float* dB, double* sums64, int64_t B, int64_t N, int64_t d,
                                    int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                                    void* stream) {
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  return do_merge(p, workspace, workspace_bytes, dA, dB, sums64, (cudaStream_t)stream);
}

grkan_status_t grkan_backward_ex(const void* x, const void* dy, const float* a, const float* b,
                                 void* dx, float* dA, float* dB, int64_t B, int64_t N, int64_t d,
                                 int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                                 void* workspace, size_t workspace_bytes, uint32_t flags,
                                 void* stream) {
  if (flags & ~GRKAN_FLAG_GENERIC) return GRKAN_ERR_FLAGS;
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if (!dA || (p.n > 0 && !dB)) return GRKAN_ERR_NULL;
  cudaStream_t st = (cudaStream_t)stream;
  if (p.T > 0) {
    s = do_partials(p, x, dy, a, b, dx, workspace, workspace_bytes, flags, st);
    if (s != GRKAN_OK) return s;
  }
  return do_merge(p, workspace, workspace_bytes, dA, dB, nullptr, st);
}

grkan_status_t grkan_backward(const void* x, const void* dy, const float* a, const float* b,
                              void* dx, float* dA, float* dB, int64_t B, int64_t N, int64_t d,
                              int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                              void* workspace, size_t workspace_bytes, void* stream) {
  return grkan_backward_ex(x, dy, a, b, dx, dA, dB, B, N, d, n_g, m, n, dtype, workspace,
                           workspace_bytes, 0u, stream);
}

grkan_status_t grkan_backward_atomic(const void* x, const void* dy, const float* a,
                                     const float* b, void* dx, float* dA, float* dB, int64_t B,
                                     int64_t N, int64_t d, int32_t n_g, int32_t m, int32_t n,
                                     grkan_dtype_t dtype, int32_t mode, int32_t block_rows,
                                     void* stream) {
  if (mode != GRKAN_ATOMIC_PER_ELEMENT && mode != GRKAN_ATOMIC_PER_BLOCK) return GRKAN_ERR_FLAGS;
  if (block_rows < 0) return GRKAN_ERR_SHAPE;
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if (!dA || (p.n > 0 && !dB)) return GRKAN_ERR_NULL;
  const size_t bytes = (size_t)p.rows * (size_t)p.d * (size_t)p.es;
  if (p.T > 0) {
    // every check before anything is enqueued
    if (!x || !dy || !dx) return GRKAN_ERR_NULL;
    if ((s = check_coef_ptrs(p, a, b)) != GRKAN_OK) return s;
    if (overlaps(x, bytes, dx, bytes) || bad_alias(dy, dx, bytes)) return GRKAN_ERR_ALIAS;
    if (mode == GRKAN_ATOMIC_PER_BLOCK) {
      const long long sb = block_rows > 0 ? block_rows : 1024;
      if (((p.rows + sb - 1) / sb) * p.n_g > 0x7fffffffLL) return GRKAN_ERR_SHAPE;
    }
  }
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(dA, 0, sizeof(float) * p.n_g * (p.m + 1), st);
  if (e == cudaSuccess && p.n > 0) e = cudaMemsetAsync(dB, 0, sizeof(float) * p.n_g * p.n, st);
  if ((s = cuda_status(e, "grkan_backward_atomic zeroing")) != GRKAN_OK) return s;
  if (p.T == 0) return GRKAN_OK;
  const bool f32 = p.dtype == GRKAN_F32;
  if (mode == GRKAN_ATOMIC_PER_ELEMENT) {
    const long long elems = p.rows * p.d;
    long long blocks = (elems + grk::kAtomicThreads - 1) / grk::kAtomicThreads;
    const long long cap = (long long)sm_count() * 32;
    if (blocks > cap) blocks = cap;
    if (f32)
      grk::bwd_atomic_element<grk::IoF32, GRKAN_MAX_M, GRKAN_MAX_N>
          <<<(unsigned)blocks, grk::kAtomicThreads, 0, st>>>(
              (const float*)x, (const float*)dy, (float*)dx, a, b, dA, dB, elems, p.d,
              (int)p.dg, p.m, p.n);
    else
      grk::bwd_atomic_element<grk::IoBF16, GRKAN_MAX_M, GRKAN_MAX_N>
          <<<(unsigned)blocks, grk::kAtomicThreads, 0, st>>>(
              (const grk::IoBF16::T*)x, (const grk::IoBF16::T*)dy, (grk::IoBF16::T*)dx, a, b,
              dA, dB, elems, p.d, (int)p.dg, p.m, p.n);
  } else {
    const int sb = block_rows > 0 ? block_rows : 1024;
    const long long tiles = (p.rows + sb - 1) / sb;
    const long long blocks = tiles * p.n_g;  // fits in 31 bits (checked above)
    if (f32)
      grk::bwd_atomic_block<grk::IoF32, GRKAN_MAX_M, GRKAN_MAX_N>
          <<<(unsigned)blocks, grk::kAtomicThreads, 0, st>>>(
              (const float*)x, (const float*)dy, (float*)dx, a, b, dA, dB, p.rows, p.d,
              (int)p.dg, p.n_g, p.m, p.n, sb);
    else
      grk::bwd_atomic_block<grk::IoBF16, GRKAN_MAX_M, GRKAN_MAX_N>
          <<<(unsigned)blocks, grk::kAtomicThreads, 0, st>>>(
              (const grk::IoBF16::T*)x, (const grk::IoBF16::T*)dy, (grk::IoBF16::T*)dx, a, b,
              dA, dB, p.rows, p.d, (int)p.dg, p.n_g, p.m, p.n, sb);
  }
  return cuda_status(cudaGetLastError(), "grkan_backward_atomic launch");
}

namespace {

// 2-D bf16 tensor map with the given shared-memory swizzle (the inner box must
// span no more bytes than the swizzle width).
bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                   uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    set_last_error("cudaGetDriverEntryPoint", "cuTensorMapEncodeTiled not found", 0);
    return false;
  }
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)(inner * 2)};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) set_last_error("cuTensorMapEncodeTiled", "failed (linear)", (int)r);
  return r == CUDA_SUCCESS;
}

// Clusters of `size` CTAs of `kernel` (with `smem` bytes of dynamic shared
// memory) that are resident at once on the current device (0 if none fits),
// looked up once per device (for the one kernel that asks: the cluster fused
// forward).
cudaError_t resident_clusters(const void* kernel, int size, int threads, unsigned smem, int* out) {
  static std::mutex mu;
  static int cached[64];  // clusters + 1 once looked up
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && cached[dev] > 0) {
    *out = cached[dev] - 1;
    return cudaSuccess;
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sms / size * size), 1, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)size;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
  if (e != cudaSuccess) return e;
  if (n < 0) n = 0;
  if (dev >= 0 && dev < 64) cached[dev] = n + 1;
  *out = n;
  return cudaSuccess;
}

// Column tiling of the cluster fused forward: n_ct tiles of at most 2 x 512
// outputs, split evenly between the two CTA pairs of a cluster, each pair's
// share rounded up to 128 (two MMAs of at most 256, W boxes of 64 rows per CTA).
void quad_cols(int64_t nout, int* np, int* n_ct) {
  namespace qd = grk::lin::qd;
  const long long ct = (nout + 2LL * qd::kNPMax - 1) / (2LL * qd::kNPMax);
  const long long share = (nout + 2 * ct - 1) / (2 * ct);
  *n_ct = (int)ct;
  *np = (int)((share + 127) / 128 * 128);
}

// Whether grkan_linear_forward takes the cluster kernel: for n_out > 512 (d a
// multiple of its K step). Measured on the KAT-B rows (100,864 x 3072): n_out 576
// to 2048 are faster than or level with the one-CTA kernel (768: 0.53 against
// 0.68 ms; 1536, two column tiles of 768: 1.02 against 1.06), and at d = 768
// n_out 1536 and 3072 are 24-37 % faster; n_out 512 and below are slower (512:
// 0.50 against 0.41), where the one-CTA kernel already activates each element
// once.
bool use_linear_quad(const Plan& p, int64_t nout) {
  if (!GRK_LIN_QUAD || p.d % grk::lin::qd::BK != 0) return false;
  return GRK_LIN_QUAD == 2 || nout > 512;
}

// The cluster fused forward: d a multiple of its K step (64); the plan, the
// pointers and the other shapes are checked by the caller. Returns
// cudaErrorNotSupported, having launched nothing, when no cluster of four fits
// on the device.
cudaError_t launch_linear_quad(const void* x, const void* W, void* out, const Plan& p,
                               int64_t nout, const float* a, const float* b, const float* bias,
                               cudaStream_t st) {
  namespace qd = grk::lin::qd;
  CUtensorMap mx, mw, mo;
  if (!make_map_bf16(&mx, x, (uint64_t)p.d, (uint64_t)p.rows, qd::BK, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_bf16(&mw, W, (uint64_t)p.d, (uint64_t)nout, qd::BK, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_bf16(&mo, out, (uint64_t)nout, (uint64_t)p.rows, 64, 32,
                     CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  qd::QGeom g;
  g.rows = p.rows;
  g.d = (int)p.d;
  g.nout = (int)nout;
  g.dg = (int)p.dg;
  g.n_g = p.n_g;
  g.kt = (int)(p.d / qd::BK);
  quad_cols(nout, &g.np, &g.n_ct);
  g.n1 = g.np < 256 ? g.np : 256;
  g.n2 = g.np - g.n1;
  g.n_tiles = ((p.rows + 2 * qd::BM - 1) / (2 * qd::BM)) * g.n_ct;
  g.ws = qd::Layout::w_stages(g.np);
  cudaError_t e = grk::ensure_smem<qd::linear_fwd_quad>(qd::kAllocMax);
  if (e != cudaSuccess) return e;
  int clusters = 0;
  if (resident_clusters(reinterpret_cast<const void*>(qd::linear_fwd_quad), 4, qd::kThreads,
                        qd::kAllocMax, &clusters) != cudaSuccess) {
    (void)cudaGetLastError();  // the query failed: no cluster can be placed
    return cudaErrorNotSupported;
  }
  if (clusters < 1) return cudaErrorNotSupported;
  if ((long long)clusters > g.n_tiles) clusters = (int)g.n_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(4 * clusters), 1, 1);
  cfg.blockDim = dim3(qd::kThreads, 1, 1);
  cfg.dynamicSmemBytes = qd::Layout::alloc(g.np);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 4;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qd::linear_fwd_quad, mx, mw, mo, a, b, bias, g);
}

}  // namespace

namespace {

// Shape checks of grkan_linear_forward (the plan is valid).
grkan_status_t linear_fwd_shape(const Plan& p, int64_t nout) {
  if (p.dtype != GRKAN_BF16) return GRKAN_ERR_DTYPE;
  if (p.m != 5 || p.n != 4) return GRKAN_ERR_DEGREE;
  if (nout < 0 || p.d == 0 || p.d % grk::lin::BK != 0 || p.dg % 8 != 0 || nout % 8 != 0 ||
      p.rows > 0x7fffffffLL || nout > 0x7fffffffLL)
    return GRKAN_ERR_SHAPE;
  return GRKAN_OK;
}

}  // namespace

int32_t grkan_linear_forward_path(int64_t B, int64_t N, int64_t d, int32_t n_g, int32_t m,
                                  int32_t n, int64_t nout, grkan_dtype_t dtype) {
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s == GRKAN_OK) s = linear_fwd_shape(p, nout);
  if (s != GRKAN_OK) return -(int32_t)s;
  return use_linear_quad(p, nout) ? 1 : 0;
}

grkan_status_t grkan_linear_forward(const void* x, const float* a, const float* b, const void* W,
                                    const float* bias, void* out, int64_t B, int64_t N,
                                    int64_t d, int32_t n_g, int32_t m, int32_t n, int64_t nout,
                                    grkan_dtype_t dtype, void* stream) {
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if ((s = linear_fwd_shape(p, nout)) != GRKAN_OK) return s;
  if (p.rows == 0 || nout == 0) return GRKAN_OK;
  if (!x || !W || !out) return GRKAN_ERR_NULL;
  if ((s = check_coef_ptrs(p, a, b)) != GRKAN_OK) return s;
  if (!aligned16(x) || !aligned16(W) || !aligned16(out)) return GRKAN_ERR_SHAPE;
  const size_t xbytes = (size_t)p.rows * (size_t)p.d * 2;
  const size_t wbytes = (size_t)nout * (size_t)p.d * 2;
  const size_t obytes = (size_t)p.rows * (size_t)nout * 2;
  if (overlaps(out, obytes, x, xbytes) || overlaps(out, obytes, W, wbytes)) return GRKAN_ERR_ALIAS;
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  if (use_linear_quad(p, nout)) {
    const cudaError_t eq =
        launch_linear_quad(x, W, out, p, nout, a, b, bias, (cudaStream_t)stream);
    // no cluster of four fits on this device: the one-CTA kernel below
    if (eq != cudaErrorNotSupported) return cuda_status(eq, "grkan_linear_forward launch");
  }
  CUtensorMap mx, mw, mo;
  if (!make_map_bf16(&mx, x, (uint64_t)p.d, (uint64_t)p.rows, grk::lin::BK, grk::lin::BM,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_bf16(&mw, W, (uint64_t)p.d, (uint64_t)nout, grk::lin::BK, grk::lin::BNH,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_bf16(&mo, out, (uint64_t)nout, (uint64_t)p.rows, grk::lin::kEpiCols,
                     grk::lin::kEpiRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return GRKAN_ERR_CUDA;
  grk::lin::LinGeom g;
  g.rows = p.rows;
  g.d = (int)p.d;
  g.nout = (int)nout;
  g.dg = (int)p.dg;
  g.n_g = p.n_g;
  g.kt = (int)(p.d / grk::lin::BK);
  const long long tiles = ((p.rows + grk::lin::BM - 1) / grk::lin::BM) *
                          ((nout + grk::lin::BN - 1) / grk::lin::BN);
  if (tiles > 0x7fffffffLL) return GRKAN_ERR_SHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = grk::ensure_smem<grk::lin::linear_fwd>(grk::lin::Layout::kAlloc);
  if (e == cudaSuccess) {
    grk::lin::linear_fwd<<<(unsigned)tiles, grk::lin::kThreads, grk::lin::Layout::kAlloc, st>>>(
        mx, mw, mo, a, b, bias, g);
    e = cudaGetLastError();
  }
  return cuda_status(e, "grkan_linear_forward launch");
}

namespace {

// Partial slots of the fused data-gradient kernel per (group, coefficient): one
// per (128-row tile, 64-channel block of the group, 32-row quarter).
long long dgrad_slots(const Plan& p) {
  return ((p.rows + grk::lin::dg::BM - 1) / grk::lin::dg::BM) * (p.dg / 64) * 4;
}

// CTA pairs of the fused data-gradient kernel that are resident at once on the
// current device (a pair needs two SMs of one GPC), looked up once per device.
cudaError_t dgrad_pairs(int* out) {
  static std::mutex mu;
  static int cached[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && cached[dev] > 0) {
    *out = cached[dev];
    return cudaSuccess;
  }
  namespace dg = grk::lin::dg;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sms / 2 * 2), 1, 1);
  cfg.blockDim = dim3(dg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = dg::Layout::kAlloc;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, dg::linear_dgrad, &cfg);
  if (e != cudaSuccess) return e;
  if (n < 1) n = 1;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  *out = n;
  return cudaSuccess;
}

// Shape checks of grkan_linear_backward (the plan is valid).
grkan_status_t dgrad_shape(const Plan& p, int64_t nout) {
  if (p.dtype != GRKAN_BF16) return GRKAN_ERR_DTYPE;
  if (p.m != 5 || p.n != 4) return GRKAN_ERR_DEGREE;
  if (nout < 0 || nout % 8 != 0 || nout > 0x7fffffffLL || p.dg % 64 != 0 ||
      p.rows > 0x7fffffffLL || p.d > 0x7fffffffLL)
    return GRKAN_ERR_SHAPE;
  if (p.rows > 0 && p.d > 0 && (long long)p.n_g * dgrad_slots(p) > (1LL << 31) - 1)
    return GRKAN_ERR_SHAPE;
  return GRKAN_OK;
}

}  // namespace

size_t grkan_linear_backward_workspace_bytes(int64_t B, int64_t N, int64_t d, int32_t n_g,
                                             int32_t m, int32_t n, int64_t nout,
                                             grkan_dtype_t dtype) {
  Plan p;
  if (make_plan(B, N, d, n_g, m, n, dtype, &p) != GRKAN_OK || dgrad_shape(p, nout) != GRKAN_OK)
    return 0;
  if (p.rows == 0 || p.d == 0 || nout == 0) return 0;
  return (size_t)dgrad_slots(p) * (size_t)p.n_g * (size_t)p.K * sizeof(float);
}

grkan_status_t grkan_linear_backward(const void* x, const void* dout, const void* W,
                                     const float* a, const float* b, void* dx, float* dA,
                                     float* dB, int64_t B, int64_t N, int64_t d, int32_t n_g,
                                     int32_t m, int32_t n, int64_t nout, grkan_dtype_t dtype,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if ((s = dgrad_shape(p, nout)) != GRKAN_OK) return s;
  if (!dA || !dB) return GRKAN_ERR_NULL;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t xbytes = (size_t)p.rows * (size_t)p.d * 2;
  if (p.rows == 0 || p.d == 0 || nout == 0) {
    // no rows: empty sums; no output features: dy = 0, so dx = 0 and the sums are 0
    if (xbytes > 0 && !dx) return GRKAN_ERR_NULL;
    if (!is_sm100()) return GRKAN_ERR_DEVICE;
    cudaError_t e = cudaSuccess;
    if (xbytes > 0) e = cudaMemsetAsync(dx, 0, xbytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dA, 0, sizeof(float) * p.n_g * (p.m + 1), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, sizeof(float) * p.n_g * p.n, st);
    return cuda_status(e, "grkan_linear_backward zeroing");
  }
  if (!x || !dout || !W || !dx) return GRKAN_ERR_NULL;
  if ((s = check_coef_ptrs(p, a, b)) != GRKAN_OK) return s;
  if (!aligned16(x) || !aligned16(dout) || !aligned16(W) || !aligned16(dx))
    return GRKAN_ERR_SHAPE;
  const long long T = dgrad_slots(p);
  const size_t ws_bytes = (size_t)T * (size_t)p.n_g * (size_t)p.K * sizeof(float);
  if (!workspace || workspace_bytes < ws_bytes || !aligned16(workspace)) return GRKAN_ERR_WORKSPACE;
  const size_t dobytes = (size_t)p.rows * (size_t)nout * 2;
  const size_t wbytes = (size_t)nout * (size_t)p.d * 2;
  if (overlaps(dx, xbytes, x, xbytes) || overlaps(dx, xbytes, dout, dobytes) ||
      overlaps(dx, xbytes, W, wbytes) || overlaps(workspace, ws_bytes, x, xbytes) ||
      overlaps(workspace, ws_bytes, dout, dobytes) || overlaps(workspace, ws_bytes, W, wbytes) ||
      overlaps(workspace, ws_bytes, dx, xbytes))
    return GRKAN_ERR_ALIAS;
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  namespace dg = grk::lin::dg;
  CUtensorMap mdo, mw, mx, mdx;
  if (!make_map_bf16(&mdo, dout, (uint64_t)nout, (uint64_t)p.rows, dg::BK, dg::BM,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_bf16(&mw, W, (uint64_t)p.d, (uint64_t)nout, 32, dg::BK,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_bf16(&mx, x, (uint64_t)p.d, (uint64_t)p.rows, 32, dg::BM,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_bf16(&mdx, dx, (uint64_t)p.d, (uint64_t)p.rows, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B))
    return GRKAN_ERR_CUDA;
  dg::DgGeom g;
  g.rows = p.rows;
  g.d = (int)p.d;
  g.nout = (int)nout;
  g.dg = (int)p.dg;
  g.n_g = p.n_g;
  g.kt = (int)((nout + dg::BK - 1) / dg::BK);
  g.n_ct = (int)((p.d + dg::BN - 1) / dg::BN);
  g.n_tiles = ((p.rows + 2 * dg::BM - 1) / (2 * dg::BM)) * g.n_ct;
  g.n_mt = (p.rows + dg::BM - 1) / dg::BM;
  g.ws_T = T;
  g.nbg = (int)(p.dg / 64);
  cudaError_t e = grk::ensure_smem<dg::linear_dgrad>(dg::Layout::kAlloc);
  int pairs = 0;
  if (e == cudaSuccess) e = dgrad_pairs(&pairs);
  if (e == cudaSuccess) {
    if ((long long)pairs > g.n_tiles) pairs = (int)g.n_tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    cfg.blockDim = dim3(dg::kThreads, 1, 1);
    cfg.dynamicSmemBytes = dg::Layout::kAlloc;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, dg::linear_dgrad, mdo, mw, mx, mdx, a, b, (float*)workspace, g);
  }
  if ((s = cuda_status(e, "grkan_linear_backward launch")) != GRKAN_OK) return s;
  Plan pm = p;
  pm.T = T;
  return cuda_status(launch_merge(pm, (const float*)workspace, dA, dB, nullptr, st),
                     "grkan_linear_backward merge");
}

grkan_status_t grkan_merge_ranks(const double* gathered, int32_t world, float* dA, float* dB,
                                 int32_t n_g, int32_t m, int32_t n, void* stream) {
  if (m < 0 || m > GRKAN_MAX_M || n < 0 || n > GRKAN_MAX_N) return GRKAN_ERR_DEGREE;
  if (n_g < 1 || world < 1) return GRKAN_ERR_SHAPE;
  if (!gathered || !dA || (n > 0 && !dB)) return GRKAN_ERR_NULL;
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  const long long per = (long long)n_g * (m + 1 + n);
  const unsigned threads = 128;
  grk::merge_ranks<<<(unsigned)((per + threads - 1) / threads), threads, 0,
                     (cudaStream_t)stream>>>(gathered, world, dA, dB, n_g, m, n);
  return cuda_status(cudaGetLastError(), "merge_ranks launch");
}

grkan_status_t grkan_backward_noalloc(const void* x, const void* dy, const float* a,
                                      const float* b, void* dx, float* dA, float* dB, int64_t B,
                                      int64_t N, int64_t d, int32_t n_g, int32_t m, int32_t n,
                                      grkan_dtype_t dtype, void* stream) {
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if (!dA || (p.n > 0 && !dB)) return GRKAN_ERR_NULL;
  if (p.ws_bytes > (size_t)GRKAN_NOALLOC_WORKSPACE_BYTES) {
    set_last_error("grkan_backward_noalloc", "workspace needed exceeds the static scratch",
                   (int)(p.ws_bytes >> 20));
    return GRKAN_ERR_WORKSPACE;
  }
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  void* ws = nullptr;
  s = noalloc_workspace(&ws);
  if (s != GRKAN_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (p.T > 0) {
    s = do_partials(p, x, dy, a, b, dx, ws, GRKAN_NOALLOC_WORKSPACE_BYTES, 0u, st);
    if (s != GRKAN_OK) return s;
  }
  return do_merge(p, ws, GRKAN_NOALLOC_WORKSPACE_BYTES, dA, dB, nullptr, st);
}

grkan_status_t grkan_forward_backward(const void* x, const void* dy, const float* a,
                                      const float* b, void* y, void* dx, float* dA, float* dB,
                                      int64_t B, int64_t N, int64_t d, int32_t n_g, int32_t m,
                                      int32_t n, grkan_dtype_t dtype, void* workspace,
                                      size_t workspace_bytes, uint32_t flags, void* stream) {
  if (flags & ~GRKAN_FLAG_GENERIC) return GRKAN_ERR_FLAGS;
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if (!dA || (p.n > 0 && !dB)) return GRKAN_ERR_NULL;
  cudaStream_t st = (cudaStream_t)stream;
  if (p.T > 0) {
    if (!x || !dy || !dx || !y) return GRKAN_ERR_NULL;
    if ((s = check_coef_ptrs(p, a, b)) != GRKAN_OK) return s;
    if (!workspace || workspace_bytes < p.ws_bytes || !aligned16(workspace))
      return GRKAN_ERR_WORKSPACE;
    const size_t bytes = (size_t)p.rows * (size_t)p.d * (size_t)p.es;
    if (overlaps(x, bytes, dx, bytes) || bad_alias(dy, dx, bytes) || overlaps(y, bytes, x, bytes) ||
        overlaps(y, bytes, dy, bytes) || overlaps(y, bytes, dx, bytes))
      return GRKAN_ERR_ALIAS;
    if (overlaps(workspace, p.ws_bytes, x, bytes) || overlaps(workspace, p.ws_bytes, dy, bytes) ||
        overlaps(workspace, p.ws_bytes, dx, bytes) || overlaps(workspace, p.ws_bytes, y, bytes))
      return GRKAN_ERR_ALIAS;
    s = do_partials_at(p, x, dy, a, b, dx, y, workspace, p.T, 0, flags, st);
    if (s != GRKAN_OK) return s;
  }
  return do_merge(p, workspace, workspace_bytes, dA, dB, nullptr, st);
}

size_t grkan_step_host_scratch_bytes(int64_t B, int64_t N, int64_t d, int32_t n_g, int32_t m,
                                     int32_t n, grkan_dtype_t dtype, int64_t chunk_rows) {
  Plan p;
  if (make_plan(B, N, d, n_g, m, n, dtype, &p) != GRKAN_OK) return 0;
  if (p.rows == 0 || p.d == 0) return 256;
  return staging_layout(p, chunk_rows).total;
}

grkan_status_t grkan_step_host(const void* x_host, const void* dy_host, const float* a,
                               const float* b, void* y_host, void* dx_host, float* dA_host,
                               float* dB_host, double* sums64, int64_t B, int64_t N, int64_t d,
                               int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype, void* scratch,
                               size_t scratch_bytes, int64_t chunk_rows, void* stream) {
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return s;
  if (!dA_host || (p.n > 0 && !dB_host)) return GRKAN_ERR_NULL;
  if ((s = check_coef_ptrs(p, a, b)) != GRKAN_OK) return s;
  const bool empty = p.rows == 0 || p.d == 0;
  if (!empty && (!x_host || !dy_host || !y_host || !dx_host)) return GRKAN_ERR_NULL;
  const StagingLayout L = empty ? StagingLayout() : staging_layout(p, chunk_rows);
  const size_t need = empty ? 256 : L.total;
  if (!scratch || scratch_bytes < need || ((uintptr_t)scratch & 255u)) return GRKAN_ERR_WORKSPACE;
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  int dev = 0;
  if ((s = cuda_status(cudaGetDevice(&dev), "cudaGetDevice")) != GRKAN_OK) return s;
  if (dev < 0 || dev >= kMaxDevices) return GRKAN_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  HostPipe* hp = nullptr;
  if ((s = pipe_for_device(dev, &hp)) != GRKAN_OK) return s;
  cudaStream_t caller = (cudaStream_t)stream;
  unsigned char* base = (unsigned char*)scratch;
  float* ws = (float*)(base + L.ws_off);
  float* dA = (float*)(base + L.grad_off);
  float* dB = dA + (size_t)p.n_g * (p.m + 1);
  const size_t ka = (size_t)p.n_g * (p.m + 1) * sizeof(float);
  const size_t kb = (size_t)p.n_g * p.n * sizeof(float);

#define GRK_TRY(expr, what)                                   \
  do {                                                        \
    if ((s = cuda_status((expr), what)) != GRKAN_OK) return s; \
  } while (0)

  // everything issued before on the caller's stream happens first
  GRK_TRY(cudaEventRecord(hp->start, caller), "cudaEventRecord");
  GRK_TRY(cudaStreamWaitEvent(hp->s_in, hp->start, 0), "cudaStreamWaitEvent");
  GRK_TRY(cudaStreamWaitEvent(hp->s_comp, hp->start, 0), "cudaStreamWaitEvent");
  GRK_TRY(cudaStreamWaitEvent(hp->s_out, hp->start, 0), "cudaStreamWaitEvent");
  if (empty) {
    s = do_merge(p, ws, 0, dA, dB, sums64, hp->s_comp);
    if (s != GRKAN_OK) return s;
  } else {
    const long long nchunks = (p.rows + L.chunk_rows - 1) / L.chunk_rows;
    const size_t row_bytes = (size_t)p.d * (size_t)p.es;
    for (long long c = 0; c < nchunks; ++c) {
      const int slot = (int)(c % kSlots);
      const long long r0 = c * L.chunk_rows;
      const long long rows = (p.rows - r0) < L.chunk_rows ? (p.rows - r0) : L.chunk_rows;
      const size_t bytes = (size_t)rows * row_bytes;
      const size_t off = (size_t)r0 * row_bytes;
      unsigned char* sx = base + (size_t)slot * 4 * L.tensor;
      unsigned char* sdy = sx + L.tensor;
      unsigned char* sy = sdy + L.tensor;
      unsigned char* sdx = sy + L.tensor;
      // inputs in, once the slot's previous outputs have left
      if (c >= kSlots) GRK_TRY(cudaStreamWaitEvent(hp->s_in, hp->out[slot], 0), "cudaStreamWaitEvent");
      GRK_TRY(cudaMemcpyAsync(sx, (const unsigned char*)x_host + off, bytes,
                              cudaMemcpyHostToDevice, hp->s_in), "cudaMemcpyAsync");
      GRK_TRY(cudaMemcpyAsync(sdy, (const unsigned char*)dy_host + off, bytes,
                              cudaMemcpyHostToDevice, hp->s_in), "cudaMemcpyAsync");
      GRK_TRY(cudaEventRecord(hp->in[slot], hp->s_in), "cudaEventRecord");
      // forward and backward of the chunk; its tiles go to their place in ws
      GRK_TRY(cudaStreamWaitEvent(hp->s_comp, hp->in[slot], 0), "cudaStreamWaitEvent");
      Plan pc;
      if ((s = make_plan(rows, 1, p.d, p.n_g, p.m, p.n, p.dtype, &pc)) != GRKAN_OK) return s;
      if (choose_fwd_path(pc, sx, sy, 0) == 1) {
        s = launch_tma_fwd(pc, sx, sy, a, b, hp->s_comp);
      } else {
        cudaError_t e = (p.dtype == GRKAN_F32)
                            ? launch_generic_fwd<grk::IoF32>(pc, sx, sy, a, b, hp->s_comp)
                            : launch_generic_fwd<grk::IoBF16>(pc, sx, sy, a, b, hp->s_comp);
        s = cuda_status(e, "forward (generic) launch");
      }
      if (s != GRKAN_OK) return s;
      s = do_partials_at(pc, sx, sdy, a, b, sdx, nullptr, ws, p.T, r0 / p.S, 0u, hp->s_comp);
      if (s != GRKAN_OK) return s;
      GRK_TRY(cudaEventRecord(hp->comp[slot], hp->s_comp), "cudaEventRecord");
      // outputs out
      GRK_TRY(cudaStreamWaitEvent(hp->s_out, hp->comp[slot], 0), "cudaStreamWaitEvent");
      GRK_TRY(cudaMemcpyAsync((unsigned char*)y_host + off, sy, bytes, cudaMemcpyDeviceToHost,
                              hp->s_out), "cudaMemcpyAsync");
      GRK_TRY(cudaMemcpyAsync((unsigned char*)dx_host + off, sdx, bytes, cudaMemcpyDeviceToHost,
                              hp->s_out), "cudaMemcpyAsync");
      GRK_TRY(cudaEventRecord(hp->out[slot], hp->s_out), "cudaEventRecord");
    }
    s = do_merge(p, ws, p.ws_bytes, dA, dB, sums64, hp->s_comp);
    if (s != GRKAN_OK) return s;
  }
  GRK_TRY(cudaMemcpyAsync(dA_host, dA, ka, cudaMemcpyDeviceToHost, hp->s_comp), "cudaMemcpyAsync");
  if (kb) GRK_TRY(cudaMemcpyAsync(dB_host, dB, kb, cudaMemcpyDeviceToHost, hp->s_comp), "cudaMemcpyAsync");
  GRK_TRY(cudaEventRecord(hp->comp_done, hp->s_comp), "cudaEventRecord");
  GRK_TRY(cudaEventRecord(hp->out_done, hp->s_out), "cudaEventRecord");
  // the caller's stream continues after both
  GRK_TRY(cudaStreamWaitEvent(caller, hp->comp_done, 0), "cudaStreamWaitEvent");
  GRK_TRY(cudaStreamWaitEvent(caller, hp->out_done, 0), "cudaStreamWaitEvent");
#undef GRK_TRY
  return GRKAN_OK;
}

int32_t grkan_forward_path(const void* x, const void* y, int64_t B, int64_t N, int64_t d,
                           int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                           uint32_t flags) {
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return -(int32_t)s;
  if (flags & ~GRKAN_FLAG_GENERIC) return -(int32_t)GRKAN_ERR_FLAGS;
  return choose_fwd_path(p, x, y, flags);
}

int32_t grkan_backward_path(const void* x, const void* dy, const void* dx, int64_t B, int64_t N,
                            int64_t d, int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                            uint32_t flags) {
  Plan p;
  grkan_status_t s = make_plan(B, N, d, n_g, m, n, dtype, &p);
  if (s != GRKAN_OK) return -(int32_t)s;
  if (flags & ~GRKAN_FLAG_GENERIC) return -(int32_t)GRKAN_ERR_FLAGS;
  return choose_bwd_path(p, x, dy, dx, flags);
}

grkan_status_t grkan_device_error(uint32_t* code, void* stream) {
  if (!code) return GRKAN_ERR_NULL;
  cudaStream_t st = (cudaStream_t)stream;
  return cuda_status(grk::read_device_error(code, st), "grkan_device_error");
}

grkan_status_t grkan_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 2000000u) return GRKAN_ERR_SHAPE;
  if (!is_sm100()) return GRKAN_ERR_DEVICE;
  static_assert(grk::kErrSelfTest == GRKAN_DEVICE_ERROR_SELFTEST, "error bit");
  grk::selftest_wait_timeout<<<1, 32, 0, (cudaStream_t)stream>>>(1000ull * limit_us);
  return cuda_status(cudaGetLastError(), "grkan_selftest_wait_timeout launch");
}

grkan_status_t grkan_clear_device_error(void* stream) {
  return cuda_status(grk::clear_device_error((cudaStream_t)stream), "grkan_clear_device_error");
}

const char* grkan_status_string(grkan_status_t s) {
  switch (s) {
    case GRKAN_OK: return "GRKAN_OK";
    case GRKAN_ERR_NULL: return "GRKAN_ERR_NULL: a required pointer is NULL";
    case GRKAN_ERR_SHAPE: return "GRKAN_ERR_SHAPE: invalid sizes or d % n_g != 0";
    case GRKAN_ERR_DEGREE: return "GRKAN_ERR_DEGREE: m or n out of range";
    case GRKAN_ERR_DTYPE: return "GRKAN_ERR_DTYPE: unknown dtype";
    case GRKAN_ERR_WORKSPACE: return "GRKAN_ERR_WORKSPACE: workspace missing, small or unaligned";
    case GRKAN_ERR_CUDA: return "GRKAN_ERR_CUDA: CUDA error while enqueueing";
    case GRKAN_ERR_ALIAS: return "GRKAN_ERR_ALIAS: an output overlaps an input it may not overlap";
    case GRKAN_ERR_FLAGS: return "GRKAN_ERR_FLAGS: unknown flag bits";
    case GRKAN_ERR_DEVICE: return "GRKAN_ERR_DEVICE: current device is not sm_100";
  }
  return "GRKAN_ERR_UNKNOWN";
}

int32_t grkan_abi_version(void) { return GRKAN_ABI_VERSION; }

const char* grkan_last_error(void) { return g_last_error; }

}  // extern "C"
