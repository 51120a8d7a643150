/*
 * grkan_oracle.h -- plain fp64 CPU oracle for the GR-KAN group-rational
 * ("safe Pade") activation: forward y, backward dx, and the per-group
 * coefficient gradients dA, dB.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library. It shares no code,
 * header, table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes (the activation of the Kolmogorov-Arnold Transformer's
 * Group-Rational KAN, as summarised in "FlashKAT: Understanding and Addressing
 * Performance Bottlenecks in the Kolmogorov-Arnold Transformer" (paper notes),
 * section "KAT's breakthrough": inputs are grouped and each group shares the
 * coefficients of a safe Pade activation unit):
 *
 *   x is a row-major (rows, d) tensor; channel c belongs to group g = c / d_g,
 *   d_g = d / n_g (contiguous channel blocks).
 *   P(x) = a_{g,0} + a_{g,1} x + ... + a_{g,m} x^m
 *   Q(x) = b_{g,1} x + ... + b_{g,n} x^n           (no constant term)
 *   y    = P(x) / (1 + |Q(x)|)
 *
 * Backward, by ordinary calculus (the notes cite equations 10-11 for the
 * gradient without printing them, section "2. The atomic-add problem of the
 * original KAT"; they state only that dA and dB sum contributions over every
 * batch, sequence and in-group element). With D = 1 + |Q|, s = sign(Q)
 * (sign(0) = 0) and g = dL/dy:
 *   dx         = g (P'(x) - y s Q'(x)) / D
 *   dA[g][i]  += g x^i / D                       i = 0..m
 *   dB[g][j]  += -g y s x^j / D                  j = 1..n
 *
 * Inputs are float32 or bf16 (passed as uint16 bit patterns); they are widened
 * exactly to double. Coefficients are passed as double (the caller widens the
 * float32 parameters exactly). All arithmetic is double precision.
 *
 * Reductions run over fixed row chunks whose partial sums are added in chunk
 * order, so results do not depend on the number of threads.
 */
#ifndef GRKAN_ORACLE_H
#define GRKAN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GRO_F32 0
#define GRO_BF16 1

/* Return codes: 0 ok, 1 bad shape (d % n_g != 0, negative sizes), 2 bad degree,
 * 3 bad dtype, 4 null pointer. */

/* y[e] for every element (idx == NULL) or for the flat indices idx[0..count)
 * (x is then the full tensor). kappa_y (nullable) receives the error scale
 * (sum_i |a_i||x|^i + |y| sum_j |b_j||x|^j) / D. */
int gro_forward(const void* x, int dtype, int64_t rows, int64_t d, int n_g, int m, int n,
                const double* a, const double* b, const int64_t* idx, int64_t count, double* y,
                double* kappa_y);

/* Element-wise backward: dx for every element (idx == NULL) or for idx[0..count).
 * Nullable extras per element:
 *   kappa_dx : |g| (sum_i i|a_i||x|^{i-1} + |y| sum_j j|b_j||x|^{j-1} + kappa_y |Q'|) / D
 *   dx_sign  : 3 values per element, dx evaluated with s forced to -1, 0, +1
 *   q, kappa_q : Q(x) and sum_j |b_j||x|^j  (the sign decision and its scale) */
int gro_backward_elem(const void* x, const void* dy, int dtype, int64_t rows, int64_t d, int n_g,
                      int m, int n, const double* a, const double* b, const int64_t* idx,
                      int64_t count, double* dx, double* kappa_dx, double* dx_sign, double* q,
                      double* kappa_q);

/* Coefficient gradients over all rows:
 *   dA[n_g][m+1], dB[n_g][n]           the sums
 *   sabs_a, sabs_b (nullable)          sums of |term| (condition scale)
 *   c2_a, c2_b (nullable)              sums of (|term| (1 + c))^2, c the
 *                                      term's sensitivity to float32 rounding
 *                                      of the polynomials it depends on:
 *                                      c = kappa_q / D for a dA term
 *                                      (kappa_q = sum_j |b_j||x|^j), and
 *                                      |term| (1 + c) = |term| + |g x^j / D^2|
 *                                      (kappa_p + 2 |P| kappa_q / D) for a dB
 *                                      term (kappa_p = sum_i |a_i||x|^i); the
 *                                      square root is the size of the float32
 *                                      rounding noise of the sum
 *   amb_b (nullable)                   sum over elements whose sign decision is
 *                                      ambiguous (|Q| < amb_rel * kappa_q) of
 *                                      2 |g y x^j / D|: the most a flipped sign
 *                                      there can move dB
 *   amb_count (nullable)               number of such elements
 * nthreads <= 0 uses every available thread. */
int gro_coef_grads(const void* x, const void* dy, int dtype, int64_t rows, int64_t d, int n_g,
                   int m, int n, const double* a, const double* b, double amb_rel, double* dA,
                   double* dB, double* sabs_a, double* sabs_b, double* c2_a, double* c2_b,
                   double* amb_b, int64_t* amb_count, int nthreads);

int gro_max_threads(void);

#ifdef __cplusplus
}
#endif

#endif
