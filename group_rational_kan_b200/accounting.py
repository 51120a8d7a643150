"""Algorithmic work of the GR-KAN hot path: bytes that must cross HBM and
floating-point operations per element.

Bytes (element size es = 4 for float32 I/O, 2 for bf16):
  forward   read x, write y                   2 es
  backward  read x and dy, write dx           3 es   (stage 1; the partials,
            coefficients and the merge add < 1 MB per call and are left out)
  step      forward + backward                5 es
  forward_backward  read x and dy, write y and dx   4 es   (the recompute
            variant: one pass over x and dy for both outputs)
Floating point: the forward's extra operations per input are 2m + 2n + 3
("FlashKAT: Understanding and Addressing Performance Bottlenecks in the
Kolmogorov-Arnold Transformer", paper notes, section "Insight 2": the GR-KAN
term (2m+2n+3) d_in next to a linear layer's 2 d_in d_out).
"""


def element_size(dtype):
    """0 = float32, 1 = bf16."""
    return 4 if dtype == 0 else 2


def bytes_per_element(phase, dtype):
    es = element_size(dtype)
    return {"forward": 2 * es, "backward": 3 * es, "step": 5 * es,
            "forward_backward": 4 * es}[phase]


def forward_flops_per_element(m, n):
    return 2 * m + 2 * n + 3


def backward_flops_per_element(m, n):
    """Operations of the backward as this library evaluates it, an FMA counted
    as two: powers x^2..x^max (max(m, n) - 1 products), P, P', Q, Q' from the
    powers (2m, 2(m-1), 2n - 1, 2(n-1)), D and the reciprocal (2), y, t,
    -t y s (3), dx (3), the m+1 + n gradient sums (2(m+1) - 1 + 2n)."""
    k = max(m, n)
    powers = max(k - 1, 0)
    polys = 2 * m + 2 * max(m - 1, 0) + max(2 * n - 1, 0) + 2 * max(n - 1, 0)
    return powers + polys + 2 + 3 + 3 + (2 * (m + 1) - 1) + 2 * n


def flashkat_access_reduction(s_block, d_g):
    """Factor by which accumulating inside a block before one global update cuts
    the global accesses for the gradient (section "3. FlashKAT kernel
    restructuring (Algorithm 2)")."""
    return s_block * d_g


def backward_fma_ops_per_element(m, n):
    """FP32 FMA-pipe lane operations per element of the backward kernel (a packed
    f32x2 operation counts two, one per element): powers x^2..x^k (k = max(m, n),
    k - 1), P (m), P' (m - 1), Q (n), Q' (n - 1), y, t, -t y s (3), dx (2), the
    m + 1 + n sums, and the scalar 1 + |Q|: k + 3m + 3n + 4. For (5, 4) that is 36,
    which the instruction-class counters of the (5, 4) kernel confirm (25 FFMA2 +
    9 FMUL2 + 1 FADD2 per element pair, plus 2 FADD)."""
    return max(m, n) + 3 * m + 3 * n + 4


def fma_pipe_peak(sms, sm_mhz):
    """FP32 FMA-pipe lane operations per second: 128 per SM and cycle (a packed
    f32x2 instruction issues 64 lane operations and holds the pipe two cycles)."""
    return 128.0 * sms * sm_mhz * 1e6

