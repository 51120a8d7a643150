/*
 * grkan_oracle.c -- plain fp64 CPU oracle for the GR-KAN group-rational
 * activation. TEST INFRASTRUCTURE ONLY (see grkan_oracle.h for the contract,
 * the formulas and the citations). Slow on purpose: one element at a time,
 * Horner's rule in double precision, no blocking or fusion.
 */
#include "grkan_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Rows per reduction chunk. Chunk partial sums are combined in chunk order. */
#define GRO_CHUNK_ROWS 64

static double load_input(const void* p, int dtype, int64_t i) {
  if (dtype == GRO_F32) return (double)((const float*)p)[i];
  /* bf16 is the upper half of a float32: widen by placing it there. */
  uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static int check_args(int64_t rows, int64_t d, int n_g, int m, int n, int dtype) {
  if (rows < 0 || d < 0 || n_g <= 0) return 1;
  if (d % n_g != 0) return 1;
  if (m < 0 || m > 16 || n < 0 || n > 16) return 2;
  if (dtype != GRO_F32 && dtype != GRO_BF16) return 3;
  return 0;
}

/* The rational function and its pieces at one point x, group coefficients
 * a[0..m] = a_0..a_m and b[0..n-1] = b_1..b_n. */
typedef struct {
  double P;  /* numerator P(x) */
  double Q;  /* inner denominator sum Q(x) = b_1 x + ... + b_n x^n */
  double dP; /* P'(x) */
  double dQ; /* Q'(x) */
  double D;  /* 1 + |Q(x)| */
  double y;  /* P / D */
  double s;  /* sign(Q), with sign(0) = 0 */
} point_t;

static void eval_point(double x, const double* a, int m, const double* b, int n, point_t* o) {
  double P = a[m];
  for (int i = m - 1; i >= 0; --i) P = P * x + a[i];

  double Q = 0.0;
  for (int j = n; j >= 1; --j) Q = (Q + b[j - 1]) * x;

  double dP = 0.0;
  for (int i = m; i >= 1; --i) dP = dP * x + (double)i * a[i];

  double dQ = 0.0;
  for (int j = n; j >= 1; --j) dQ = dQ * x + (double)j * b[j - 1];

  o->P = P;
  o->Q = Q;
  o->dP = dP;
  o->dQ = dQ;
  o->D = 1.0 + fabs(Q);
  o->y = P / o->D;
  o->s = (Q > 0.0) ? 1.0 : ((Q < 0.0) ? -1.0 : 0.0);
}

/* Error scales: the same expressions evaluated with absolute values. */
static double kappa_y_at(double x, const double* a, int m, const double* b, int n,
                         const point_t* p) {
  double ax = fabs(x), sa = 0.0, sb = 0.0, xi = 1.0;
  for (int i = 0; i <= m; ++i) {
    sa += fabs(a[i]) * xi;
    xi *= ax;
  }
  xi = ax;
  for (int j = 1; j <= n; ++j) {
    sb += fabs(b[j - 1]) * xi;
    xi *= ax;
  }
  return (sa + fabs(p->y) * sb) / p->D;
}

static double kappa_q_at(double x, const double* b, int n) {
  double ax = fabs(x), sb = 0.0, xi = ax;
  for (int j = 1; j <= n; ++j) {
    sb += fabs(b[j - 1]) * xi;
    xi *= ax;
  }
  return sb;
}

int gro_forward(const void* x, int dtype, int64_t rows, int64_t d, int n_g, int m, int n,
                const double* a, const double* b, const int64_t* idx, int64_t count, double* y,
                double* kappa_y) {
  int rc = check_args(rows, d, n_g, m, n, dtype);
  if (rc) return rc;
  int64_t total = rows * d;
  int64_t cnt = idx ? count : total;
  if (cnt > 0 && (!x || !a || (n > 0 && !b) || !y)) return 4;
  int64_t dg = d / n_g;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int64_t k = 0; k < cnt; ++k) {
    int64_t e = idx ? idx[k] : k;
    int g = (int)((e % d) / dg);
    const double* ga = a + (int64_t)g * (m + 1);
    const double* gb = b ? b + (int64_t)g * n : NULL;
    double xv = load_input(x, dtype, e);
    point_t p;
    eval_point(xv, ga, m, gb, n, &p);
    y[k] = p.y;
    if (kappa_y) kappa_y[k] = kappa_y_at(xv, ga, m, gb, n, &p);
  }
  return 0;
}

int gro_backward_elem(const void* x, const void* dy, int dtype, int64_t rows, int64_t d, int n_g,
                      int m, int n, const double* a, const double* b, const int64_t* idx,
                      int64_t count, double* dx, double* kappa_dx, double* dx_sign, double* q,
                      double* kappa_q) {
  int rc = check_args(rows, d, n_g, m, n, dtype);
  if (rc) return rc;
  int64_t total = rows * d;
  int64_t cnt = idx ? count : total;
  if (cnt > 0 && (!x || !dy || !a || (n > 0 && !b) || !dx)) return 4;
  int64_t dg = d / n_g;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int64_t k = 0; k < cnt; ++k) {
    int64_t e = idx ? idx[k] : k;
    int g = (int)((e % d) / dg);
    const double* ga = a + (int64_t)g * (m + 1);
    const double* gb = b ? b + (int64_t)g * n : NULL;
    double xv = load_input(x, dtype, e);
    double gv = load_input(dy, dtype, e);
    point_t p;
    eval_point(xv, ga, m, gb, n, &p);
    dx[k] = gv * (p.dP - p.y * p.s * p.dQ) / p.D;
    if (dx_sign) {
      for (int t = 0; t < 3; ++t) {
        double s = (double)(t - 1);
        dx_sign[3 * k + t] = gv * (p.dP - p.y * s * p.dQ) / p.D;
      }
    }
    if (q) q[k] = p.Q;
    if (kappa_q) kappa_q[k] = kappa_q_at(xv, gb, n);
    if (kappa_dx) {
      double ax = fabs(xv), sa = 0.0, sb = 0.0, xi = 1.0;
      for (int i = 1; i <= m; ++i) {
        sa += (double)i * fabs(ga[i]) * xi;
        xi *= ax;
      }
      xi = 1.0;
      for (int j = 1; j <= n; ++j) {
        sb += (double)j * fabs(gb[j - 1]) * xi;
        xi *= ax;
      }
      double ky = kappa_y_at(xv, ga, m, gb, n, &p);
      kappa_dx[k] = fabs(gv) * (sa + fabs(p.y) * sb + ky * fabs(p.dQ)) / p.D;
    }
  }
  return 0;
}

static double kappa_p_at(double x, const double* a, int m) {
  double ax = fabs(x), sa = 0.0, xi = 1.0;
  for (int i = 0; i <= m; ++i) {
    sa += fabs(a[i]) * xi;
    xi *= ax;
  }
  return sa;
}

int gro_coef_grads(const void* x, const void* dy, int dtype, int64_t rows, int64_t d, int n_g,
                   int m, int n, const double* a, const double* b, double amb_rel, double* dA,
                   double* dB, double* sabs_a, double* sabs_b, double* c2_a, double* c2_b,
                   double* amb_b, int64_t* amb_count, int nthreads) {
  int rc = check_args(rows, d, n_g, m, n, dtype);
  if (rc) return rc;
  if (!dA || (n > 0 && !dB)) return 4;
  int64_t total = rows * d;
  if (total > 0 && (!x || !dy || !a || (n > 0 && !b))) return 4;
  const int ka = m + 1;
  const int kb = n;
  const int64_t dg = d / n_g;
  /* Per chunk: sums, sums of |term|, conditioned sums of squares and the dB
   * ambiguity allowance, each n_g * (m+1+n) doubles, plus a count. */
  const int64_t width = (int64_t)n_g * (ka + kb);
  const int64_t nchunks = (rows + GRO_CHUNK_ROWS - 1) / GRO_CHUNK_ROWS;
  double* part = NULL;
  int64_t* part_cnt = NULL;
  if (nchunks > 0) {
    part = (double*)calloc((size_t)(nchunks * width * 4), sizeof(double));
    part_cnt = (int64_t*)calloc((size_t)nchunks, sizeof(int64_t));
    if (!part || !part_cnt) {
      free(part);
      free(part_cnt);
      return 5;
    }
  }
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (int64_t c = 0; c < nchunks; ++c) {
    double* sum = part + c * width * 4; /* [g][k] sums, k < ka: a_k, k >= ka: b_{k-ka+1} */
    double* sab = sum + width;          /* sums of |term| */
    double* amb = sab + width;          /* ambiguity allowance for dB */
    double* csq = amb + width;          /* conditioned sums of squares */
    int64_t r0 = c * GRO_CHUNK_ROWS;
    int64_t r1 = r0 + GRO_CHUNK_ROWS < rows ? r0 + GRO_CHUNK_ROWS : rows;
    for (int64_t r = r0; r < r1; ++r) {
      for (int64_t col = 0; col < d; ++col) {
        int64_t e = r * d + col;
        int g = (int)(col / dg);
        const double* ga = a + (int64_t)g * ka;
        const double* gb = b ? b + (int64_t)g * kb : NULL;
        double xv = load_input(x, dtype, e);
        double gv = load_input(dy, dtype, e);
        point_t p;
        eval_point(xv, ga, m, gb, n, &p);
        double* srow = sum + (int64_t)g * (ka + kb);
        double* arow = sab + (int64_t)g * (ka + kb);
        double* mrow = amb + (int64_t)g * (ka + kb);
        double* qrow = csq + (int64_t)g * (ka + kb);
        const double kq = kappa_q_at(xv, gb, n);
        const double kp = kappa_p_at(xv, ga, m);
        double xi = 1.0;
        for (int i = 0; i <= m; ++i) {
          double term = gv * xi / p.D;
          srow[i] += term;
          arow[i] += fabs(term);
          double w = fabs(term) * (1.0 + kq / p.D);
          qrow[i] += w * w;
          xi *= xv;
        }
        int ambiguous = fabs(p.Q) < amb_rel * kq;
        if (ambiguous) part_cnt[c] += 1;
        xi = xv;
        for (int j = 1; j <= n; ++j) {
          double term = -gv * p.y * p.s * xi / p.D;
          srow[ka + j - 1] += term;
          arow[ka + j - 1] += fabs(term);
          double w = fabs(term) +
                     fabs(gv * xi / (p.D * p.D)) * (kp + 2.0 * fabs(p.P) * kq / p.D);
          qrow[ka + j - 1] += w * w;
          if (ambiguous) mrow[ka + j - 1] += 2.0 * fabs(gv * p.y * xi / p.D);
          xi *= xv;
        }
      }
    }
  }
  for (int g = 0; g < n_g; ++g) {
    for (int i = 0; i < ka; ++i) {
      dA[g * ka + i] = 0.0;
      if (sabs_a) sabs_a[g * ka + i] = 0.0;
      if (c2_a) c2_a[g * ka + i] = 0.0;
    }
    for (int j = 0; j < kb; ++j) {
      dB[g * kb + j] = 0.0;
      if (sabs_b) sabs_b[g * kb + j] = 0.0;
      if (c2_b) c2_b[g * kb + j] = 0.0;
      if (amb_b) amb_b[g * kb + j] = 0.0;
    }
  }
  int64_t namb = 0;
  for (int64_t c = 0; c < nchunks; ++c) {
    const double* sum = part + c * width * 4;
    const double* sab = sum + width;
    const double* amb = sab + width;
    const double* csq = amb + width;
    namb += part_cnt[c];
    for (int g = 0; g < n_g; ++g) {
      const int64_t o = (int64_t)g * (ka + kb);
      for (int i = 0; i < ka; ++i) {
        dA[g * ka + i] += sum[o + i];
        if (sabs_a) sabs_a[g * ka + i] += sab[o + i];
        if (c2_a) c2_a[g * ka + i] += csq[o + i];
      }
      for (int j = 0; j < kb; ++j) {
        dB[g * kb + j] += sum[o + ka + j];
        if (sabs_b) sabs_b[g * kb + j] += sab[o + ka + j];
        if (c2_b) c2_b[g * kb + j] += csq[o + ka + j];
        if (amb_b) amb_b[g * kb + j] += amb[o + ka + j];
      }
    }
  }
  if (amb_count) *amb_count = namb;
  free(part);
  free(part_cnt);
  return 0;
}

int gro_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
