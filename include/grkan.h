/*
 * grkan.h -- C ABI of the B200 (sm_100a) GR-KAN group-rational activation.
 *
 * The operation. The Kolmogorov-Arnold Transformer replaces the MLP's fixed
 * activation by a Group-Rational KAN: channels are split into n_g groups and
 * every group shares the coefficients of one "safe" Pade activation unit
 * ("FlashKAT: Understanding and Addressing Performance Bottlenecks in the
 * Kolmogorov-Arnold Transformer", paper notes, section "KAT's breakthrough and
 * remaining problem"; 8 groups, 6 numerator and 4 denominator coefficients in
 * section "Loss / training strategy"):
 *
 *   x : row-major (B, N, d) tensor, rows = B*N; channel c is in group
 *       g = c / d_g with d_g = d / n_g (contiguous channel blocks)
 *   P(x) = a[g][0] + a[g][1] x + ... + a[g][m] x^m
 *   Q(x) = b[g][0] x + b[g][1] x^2 + ... + b[g][n-1] x^n   (b_1..b_n, no b_0)
 *   y    = P(x) / (1 + |Q(x)|)
 *
 * The backward pass (gradient equations cited, not printed, in section
 * "2. The atomic-add problem of the original KAT"; derived here by calculus,
 * with D = 1 + |Q|, s = sign(Q), sign(0) = 0, g = dL/dy):
 *   dx        = g (P'(x) - y s Q'(x)) / D
 *   dA[g][i]  = sum over every row and every channel of group g of  g x^i / D
 *   dB[g][j]  = sum over the same elements of  -g y s x^(j+1) / D
 * The sums run over all batch x sequence x in-group elements (same section).
 * They are computed without atomics, in two stages (cf. the two-stage reduction
 * of "PolyKAN: Efficient Fused GPU Operators for Polynomial Kolmogorov-Arnold
 * Network Variants", abstract, technique (iii)): per (row tile, group) partial
 * sums into a caller-owned workspace, then a fixed-order merge in double
 * precision. dA and dB are therefore bit-identical from run to run for a given
 * shape and a given pointer alignment class (16-byte aligned or not).
 *
 * Conventions shared by every entry point:
 *  - Pointers named x, y, dy, dx, a, b, dA, dB, workspace are DEVICE pointers
 *    (or managed memory) of the current CUDA device; the caller owns them.
 *    The compute entry points allocate no device memory and keep no state
 *    between calls; the exceptions are named where they are declared:
 *    grkan_step_host creates three streams and a few events per device on its
 *    first call, grkan_backward_noalloc uses a static device array that the
 *    library holds, and the fused linear entry points look up a per-device
 *    occupancy figure once.
 *  - dtype selects the element type of x, y, dy, dx: float32 or bfloat16.
 *    Coefficients a (n_g x (m+1)), b (n_g x n) and gradients dA, dB are always
 *    float32, row-major. Arithmetic is float32; the merge is float64.
 *  - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous: it validates, enqueues kernels and returns.
 *  - 0 <= m <= GRKAN_MAX_M, 0 <= n <= GRKAN_MAX_N, n_g >= 1, d % n_g == 0.
 *    With n = 0, b may be NULL and Q = 0. B*N*d == 0 is a valid no-op
 *    (the backward then writes zeros to dA and dB).
 *  - Aliasing: y may equal x (in place) and dx may equal dy (dy is read
 *    before dx is written at the same place). dx may not equal or overlap x,
 *    which has to stay readable for the caller; that, and any other overlap
 *    between an input and an output, returns GRKAN_ERR_ALIAS.
 *  - Errors are returned, never thrown; on error nothing is enqueued.
 *    GRKAN_ERR_CUDA reports a launch failure (cudaGetLastError); a fault that
 *    happens later on the GPU surfaces at the caller's next synchronisation.
 */
#ifndef GRKAN_H
#define GRKAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GRKAN_API __attribute__((visibility("default")))
#else
#define GRKAN_API
#endif

/* 3: grkan_linear_forward_path added. */
#define GRKAN_ABI_VERSION 3
#define GRKAN_MAX_M 8
#define GRKAN_MAX_N 8

typedef enum grkan_dtype { GRKAN_F32 = 0, GRKAN_BF16 = 1 } grkan_dtype_t;

typedef enum grkan_status {
  GRKAN_OK = 0,
  GRKAN_ERR_NULL = 1,      /* a required pointer is NULL */
  GRKAN_ERR_SHAPE = 2,     /* negative size, n_g < 1, d % n_g != 0, or size overflow */
  GRKAN_ERR_DEGREE = 3,    /* m or n outside [0, GRKAN_MAX_M] / [0, GRKAN_MAX_N] */
  GRKAN_ERR_DTYPE = 4,     /* unknown dtype */
  GRKAN_ERR_WORKSPACE = 5, /* workspace NULL or smaller than the query says */
  GRKAN_ERR_CUDA = 6,      /* CUDA reported an error while enqueueing */
  GRKAN_ERR_ALIAS = 7,     /* an output overlaps an input it may not overlap */
  GRKAN_ERR_FLAGS = 8,     /* unknown flag bits */
  GRKAN_ERR_DEVICE = 9     /* the current device is not sm_100 (B200 class) */
} grkan_status_t;

/* Flag bits for the *_ex entry points. */
#define GRKAN_FLAG_GENERIC 1u /* use the plain grid-stride kernels even where the
                                 TMA-pipelined kernels apply (for testing) */

/* Forward: y = P(x) / (1 + |Q(x)|) elementwise, group coefficients a, b. */
GRKAN_API grkan_status_t grkan_forward(const void* x, void* y, const float* a, const float* b, int64_t B,
                             int64_t N, int64_t d, int32_t n_g, int32_t m, int32_t n,
                             grkan_dtype_t dtype, void* stream);

GRKAN_API grkan_status_t grkan_forward_ex(const void* x, void* y, const float* a, const float* b, int64_t B,
                                int64_t N, int64_t d, int32_t n_g, int32_t m, int32_t n,
                                grkan_dtype_t dtype, uint32_t flags, void* stream);

/* Bytes of device workspace grkan_backward needs for this shape (0 when the
 * input is empty). The layout is private; its size depends only on the shape. */
GRKAN_API size_t grkan_backward_workspace_bytes(int64_t B, int64_t N, int64_t d, int32_t n_g, int32_t m,
                                      int32_t n, grkan_dtype_t dtype);

/* Backward: dx (same shape and dtype as x), dA (n_g x (m+1)) and dB (n_g x n),
 * both overwritten (not accumulated). workspace must hold at least
 * grkan_backward_workspace_bytes(...) bytes, 16-byte aligned; its previous
 * contents do not matter. Equivalent to grkan_backward_partials followed by
 * grkan_backward_merge on the same stream. */
GRKAN_API grkan_status_t grkan_backward(const void* x, const void* dy, const float* a, const float* b,
                              void* dx, float* dA, float* dB, int64_t B, int64_t N, int64_t d,
                              int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                              void* workspace, size_t workspace_bytes, void* stream);

GRKAN_API grkan_status_t grkan_backward_ex(const void* x, const void* dy, const float* a, const float* b,
                                 void* dx, float* dA, float* dB, int64_t B, int64_t N, int64_t d,
                                 int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                                 void* workspace, size_t workspace_bytes, uint32_t flags,
                                 void* stream);

/* Forward and backward fused in one pass over x and dy, for training that
 * recomputes the activation in the backward pass (activation checkpointing):
 * writes y (as grkan_forward) and dx, dA, dB (as grkan_backward). Reads x and dy
 * once and writes y and dx once: 4 element sizes of traffic per element instead
 * of 5 for the two separate calls. y may not overlap x, dy or dx; dx may equal
 * dy. flags: 0 or GRKAN_FLAG_GENERIC. */
GRKAN_API grkan_status_t grkan_forward_backward(const void* x, const void* dy, const float* a,
                                                const float* b, void* y, void* dx, float* dA,
                                                float* dB, int64_t B, int64_t N, int64_t d,
                                                int32_t n_g, int32_t m, int32_t n,
                                                grkan_dtype_t dtype, void* workspace,
                                                size_t workspace_bytes, uint32_t flags,
                                                void* stream);

/* The GR-KAN activation fused into the linear layer that follows it (a KAT
 * layer: "FlashKAT: Understanding and Addressing Performance Bottlenecks in the
 * Kolmogorov-Arnold Transformer", paper notes, section "Insight 2"):
 *   out[r, o] = sum_k y[r, k] W[o, k] + bias[o],   y = grkan_forward(x),
 * on the tensor cores, with y computed in shared memory and never written.
 * x: bf16 (B*N rows x d), row-major. W: bf16 (nout x d), row-major (a linear
 * layer's weight). bias: float32 (nout) or NULL. out: bf16 (B*N x nout),
 * row-major, overwritten. y is rounded to bf16 before the product, as when
 * grkan_forward's output feeds a bf16 matrix multiply; the sum is float32.
 * Requires dtype GRKAN_BF16 (else GRKAN_ERR_DTYPE), (m, n) = (5, 4) (else
 * GRKAN_ERR_DEGREE), d > 0, d % 32 == 0, d_g % 8 == 0, nout % 8 == 0 and
 * 16-byte aligned x, W, out (else GRKAN_ERR_SHAPE); out may not overlap x or W.
 * B*N == 0 or nout == 0: nothing to do. */
GRKAN_API grkan_status_t grkan_linear_forward(const void* x, const float* a, const float* b,
                                              const void* W, const float* bias, void* out,
                                              int64_t B, int64_t N, int64_t d, int32_t n_g,
                                              int32_t m, int32_t n, int64_t nout,
                                              grkan_dtype_t dtype, void* stream);

/* Which kernel grkan_linear_forward takes for these shapes: 1 = clusters of four
 * CTAs (two tcgen05 CTA pairs sharing each 256-row tile; n_out > 512 and
 * d % 64 == 0), 0 = one CTA per 128 x 512 output tile, < 0 = the negated status
 * the call would return for these shapes. Both kernels give the same bits. No
 * device is queried: on a device where no cluster of four fits, a 1 runs as 0. */
GRKAN_API int32_t grkan_linear_forward_path(int64_t B, int64_t N, int64_t d, int32_t n_g,
                                            int32_t m, int32_t n, int64_t nout,
                                            grkan_dtype_t dtype);

/* The GR-KAN backward fused into the data-gradient product of the linear layer
 * that follows the activation (the backward of grkan_linear_forward without its
 * weight gradient):
 *   dy[r, c] = sum_o dout[r, o] W[o, c]      (float32, on the tensor cores)
 *   dx, dA, dB = grkan_backward(x, dy)        (with this float32 dy)
 * dy is the product's accumulator and never goes to memory. x: bf16 (B*N rows x
 * d), row-major. dout: bf16 (B*N x nout), row-major (the layer output's
 * gradient). W: bf16 (nout x d), row-major (the linear layer's weight). dx: bf16
 * like x, overwritten; dA (n_g x 6), dB (n_g x 4) float32, overwritten. dA and dB
 * are reduced in a fixed order, as grkan_backward's (the same bits on every
 * run). workspace: device memory of at least
 * grkan_linear_backward_workspace_bytes (which returns 0 for shapes this call
 * rejects and when nothing needs reducing), 16-byte aligned, owned by the caller
 * and free for the call's duration on its stream. nout == 0 gives dx = 0 and
 * zero gradients; B*N == 0 gives zero gradients.
 * Requires dtype GRKAN_BF16 (else GRKAN_ERR_DTYPE), (m, n) = (5, 4) (else
 * GRKAN_ERR_DEGREE), d_g % 64 == 0, nout % 8 == 0 and 16-byte aligned x, dout,
 * W, dx (else GRKAN_ERR_SHAPE); dx and the workspace may not overlap x, dout, W
 * or each other (GRKAN_ERR_ALIAS). */
GRKAN_API size_t grkan_linear_backward_workspace_bytes(int64_t B, int64_t N, int64_t d,
                                                       int32_t n_g, int32_t m, int32_t n,
                                                       int64_t nout, grkan_dtype_t dtype);

GRKAN_API grkan_status_t grkan_linear_backward(const void* x, const void* dout, const void* W,
                                               const float* a, const float* b, void* dx,
                                               float* dA, float* dB, int64_t B, int64_t N,
                                               int64_t d, int32_t n_g, int32_t m, int32_t n,
                                               int64_t nout, grkan_dtype_t dtype,
                                               void* workspace, size_t workspace_bytes,
                                               void* stream);

/* Coefficient gradients accumulated with float32 atomic adds, the two schemes
 * that "FlashKAT: Understanding and Addressing Performance Bottlenecks in the
 * Kolmogorov-Arnold Transformer" compares (paper notes, sections "2. The
 * atomic-add problem of the original KAT" and "3. FlashKAT kernel restructuring
 * (Algorithm 2)"), for error and speed studies against grkan_backward:
 *   GRKAN_ATOMIC_PER_ELEMENT  every element adds its m+1+n terms to dA / dB in
 *                             global memory (one thread per element);
 *   GRKAN_ATOMIC_PER_BLOCK    a block sums block_rows rows of one group on chip,
 *                             then adds each of its m+1+n sums once
 *                             (block_rows = 0: 1024, the paper's typical S_block).
 * dx is the same as grkan_backward's. dA and dB are zeroed on the stream first
 * and then depend on the order in which the atomics land: they can differ from
 * run to run. No workspace. Unknown mode: GRKAN_ERR_FLAGS. */
typedef enum grkan_atomic_mode {
  GRKAN_ATOMIC_PER_ELEMENT = 1,
  GRKAN_ATOMIC_PER_BLOCK = 2
} grkan_atomic_mode_t;

GRKAN_API grkan_status_t grkan_backward_atomic(const void* x, const void* dy, const float* a,
                                               const float* b, void* dx, float* dA, float* dB,
                                               int64_t B, int64_t N, int64_t d, int32_t n_g,
                                               int32_t m, int32_t n, grkan_dtype_t dtype,
                                               int32_t mode, int32_t block_rows, void* stream);

/* Stage 1 alone: dx, plus one float32 partial sum per (row tile, group,
 * coefficient) into the workspace. */
GRKAN_API grkan_status_t grkan_backward_partials(const void* x, const void* dy, const float* a,
                                       const float* b, void* dx, int64_t B, int64_t N, int64_t d,
                                       int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                                       void* workspace, size_t workspace_bytes, uint32_t flags,
                                       void* stream);

/* Stage 2 alone: fixed-order float64 sum of the workspace partials written by
 * grkan_backward_partials for the same shape; writes dA and dB (float32).
 * If sums64 is not NULL it also receives the float64 sums, laid out
 * [n_g][m+1+n] (a_0..a_m then b_1..b_n), for a later cross-device merge. */
GRKAN_API grkan_status_t grkan_backward_merge(const void* workspace, size_t workspace_bytes, float* dA,
                                    float* dB, double* sums64, int64_t B, int64_t N, int64_t d,
                                    int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                                    void* stream);

/* Data-parallel merge across devices. Each device runs the backward on its
 * own rows and grkan_backward_merge with sums64; the caller gathers the
 * world blocks of n_g*(m+1+n) float64 sums into `gathered` in rank order (for
 * example with an all-gather). This adds them in rank order -- the same order
 * on every device, independent of the transport -- and writes dA and dB
 * (float32), so all devices hold bit-identical gradients. gathered, dA and dB
 * are device pointers; world >= 1. */
GRKAN_API grkan_status_t grkan_merge_ranks(const double* gathered, int32_t world, float* dA,
                                           float* dB, int32_t n_g, int32_t m, int32_t n,
                                           void* stream);

/* Backward without a caller-supplied workspace (no counterpart in the paper;
 * an addition for callers that cannot allocate device memory per call, such as
 * a plugin whose host framework owns all device memory and forbids allocation
 * while enqueueing work, or a process that must keep its device footprint fixed
 * after start-up). Same arguments and results as grkan_backward, minus the
 * workspace: the partial sums go to a scratch array of
 * GRKAN_NOALLOC_WORKSPACE_BYTES that the library holds in static device memory
 * on every GPU that loads it, until the process exits. Shapes whose workspace
 * (grkan_backward_workspace_bytes) exceeds that size return GRKAN_ERR_WORKSPACE.
 * Nothing is allocated: the first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current, so make that first
 * call before any stream capture. All calls share the one array: calls whose
 * kernels overlap on the GPU (different streams without ordering) race and give
 * wrong gradients; calls ordered on one stream are safe. The array keeps the
 * last call's partials; every call overwrites all it reads. */
#define GRKAN_NOALLOC_WORKSPACE_BYTES (4u << 20)
GRKAN_API grkan_status_t grkan_backward_noalloc(const void* x, const void* dy, const float* a,
                                                const float* b, void* dx, float* dA, float* dB,
                                                int64_t B, int64_t N, int64_t d, int32_t n_g,
                                                int32_t m, int32_t n, grkan_dtype_t dtype,
                                                void* stream);

/* One forward + backward step on HOST-resident tensors. x_host, dy_host (in) and
 * y_host, dx_host (out) are host pointers to row-major (B, N, d) tensors (page-
 * locked memory lets the copies overlap; pageable memory works but serialises);
 * dA_host, dB_host receive the coefficient gradients (host pointers). a and b
 * are device pointers, as everywhere. The rows stream through `scratch`, a
 * device buffer of at least grkan_step_host_scratch_bytes(...) bytes (256-byte
 * aligned, owned by the caller), in chunks of about 32 MiB per tensor (or
 * chunk_rows rows, rounded up to whole reduction tiles) on three internal
 * streams, so that the host-to-device copies, the kernels and the
 * device-to-host copies of consecutive chunks overlap. The result is the same,
 * bit for bit, as grkan_forward + grkan_backward on device copies of the same
 * data. sums64 (a DEVICE pointer, may be NULL) also receives the float64 sums
 * [n_g][m+1+n] that grkan_backward_merge would give, for a data-parallel merge
 * with grkan_merge_ranks. Asynchronous with respect to the host: the outputs are
 * complete once `stream` reaches the point of the call. The first call on a
 * device creates three streams and a few events that live until the process
 * exits; calls are serialised per device while they enqueue. */
GRKAN_API size_t grkan_step_host_scratch_bytes(int64_t B, int64_t N, int64_t d, int32_t n_g,
                                               int32_t m, int32_t n, grkan_dtype_t dtype,
                                               int64_t chunk_rows);
GRKAN_API grkan_status_t grkan_step_host(const void* x_host, const void* dy_host, const float* a,
                                         const float* b, void* y_host, void* dx_host,
                                         float* dA_host, float* dB_host, double* sums64,
                                         int64_t B, int64_t N, int64_t d, int32_t n_g, int32_t m,
                                         int32_t n, grkan_dtype_t dtype, void* scratch,
                                         size_t scratch_bytes, int64_t chunk_rows, void* stream);

/* Which kernels a call with these arguments would run: 1 = TMA-pipelined
 * persistent kernels, 0 = generic grid-stride kernels, < 0 = invalid arguments
 * (the negated status). x, y are only inspected for alignment. */
GRKAN_API int32_t grkan_forward_path(const void* x, const void* y, int64_t B, int64_t N, int64_t d,
                           int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype, uint32_t flags);
GRKAN_API int32_t grkan_backward_path(const void* x, const void* dy, const void* dx, int64_t B, int64_t N,
                            int64_t d, int32_t n_g, int32_t m, int32_t n, grkan_dtype_t dtype,
                            uint32_t flags);

/* Device-side error word. The pipelined kernels bound every wait; a wait that
 * runs out (which correct inputs never cause) sets a nonzero code here and the
 * kernel returns early instead of hanging. grkan_device_error copies the word
 * to *code (host pointer) and synchronises the stream; grkan_clear_device_error
 * resets it (stream-ordered). */
GRKAN_API grkan_status_t grkan_device_error(uint32_t* code, void* stream);
GRKAN_API grkan_status_t grkan_clear_device_error(void* stream);

/* Self-test of the bounded waits: launches one warp that waits, with the same
 * wait routine as the pipelined kernels and a limit of limit_us microseconds
 * (1 .. 2,000,000; else GRKAN_ERR_SHAPE), on an mbarrier phase that nothing
 * completes. The wait runs out, the kernel ORs GRKAN_DEVICE_ERROR_SELFTEST into
 * the device error word and returns; the context stays usable. */
#define GRKAN_DEVICE_ERROR_SELFTEST 16u
GRKAN_API grkan_status_t grkan_selftest_wait_timeout(uint32_t limit_us, void* stream);

/* Human-readable name of a status code (static string). */
GRKAN_API const char* grkan_status_string(grkan_status_t status);

/* Text of the last CUDA-level failure on the calling thread (the failing call
 * and CUDA's message) behind a GRKAN_ERR_CUDA return; static storage, valid
 * until the thread's next failing call. */
GRKAN_API const char* grkan_last_error(void);

/* GRKAN_ABI_VERSION of the built library. */
GRKAN_API int32_t grkan_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GRKAN_H */
