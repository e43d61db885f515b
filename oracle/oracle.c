/*
 * oracle.c -- plain float64 CPU reference for streaming log-domain Sinkhorn.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call this
 * file; only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header, constant or helper with the CUDA library.
 *
 * What it computes, and where each step comes from:
 *
 *  - Ground cost C_ij = sum_k (x_ik - y_jk)^2, written as the direct difference
 *    (SinkSLOT README, "Tensor Contract": squared-Euclidean ground cost).
 *  - f-update  f_i = -eps * LSE_j[(g_j - C_ij)/eps + log b_j] and the symmetric
 *    g-update  g_j = -eps * LSE_i[(f_i - C_ij)/eps + log a_i]
 *    (FlashSinkhorn summary, Methodology section 1, "Attention-Form Reformulation";
 *    the g form is the symmetric twin with the log a_i bias gamma).
 *    The LSE is taken in two passes: the maximum, then the sum of exponentials
 *    shifted by it. Terms whose weight is exactly zero are left out of the sum.
 *  - Schedule: g starts at g_init (zero when none is given); each iteration is
 *    one f-update followed by one g-update that uses the new f; a fixed number of
 *    iterations, no convergence test (SinkSLOT README, API Reference:
 *    variant="alternating", stop_mode="fixed").
 *  - Transport plan P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps).
 *  - Dual objective D(f,g) = <f,a> + <g,b> - eps*(sum_ij P_ij - m_a*m_b), the double
 *    sum evaluated term by term.
 *  - Envelope gradient grad_i = 2*(a_i x_i - sum_j Pt_ij y_j), where Pt is the plan of
 *    (ft, g) with ft = F(g), so that its row sums equal a exactly
 *    (FlashSinkhorn summary, section 3, "Transport Matrix Application"; SinkSLOT
 *    README, "Basic Usage": analytic gradient without backpropagation through the
 *    iterations).
 *  - Plan row sums r_i = sum_j P_ij (column sums by swapping the roles of the
 *    clouds), from which the marginal residuals are formed (SinkSLOT README,
 *    stop_mode "marginal").
 *  - The general solve (SinkSLOT README, API Reference: variant, alpha, stop_mode,
 *    stop_max_iter, stop_tol, stop_check_every; iters_run, converged, final_viol):
 *    variant "alternating" (Gauss-Seidel) is the schedule above; variant "symmetric"
 *    (Jacobi) computes both updates from the previous iterate and blends them,
 *    f' = (1 - alpha) f + alpha F(g), g' = (1 - alpha) g + alpha G(f), from f = 0 and
 *    g = g_init (or 0). Stop mode "fixed" runs n_iters iterations; "marginal" stops at
 *    the first check where max(|P1 - a|_inf, |P^T 1 - b|_inf) <= stop_tol; "potential"
 *    at the first check where max(|f - f_prev|_inf, |g - g_prev|_inf) < stop_tol, the
 *    previous values being those of the last check (of the start for the first one;
 *    eps * |delta phi| with phi = f / eps is |delta f|). Checks run after every
 *    stop_check_every-th iteration and after the last one allowed (stop_max_iter).
 *
 * Every function returns 0 on success or a negative code on invalid arguments.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Below this many pair terms a call runs on one thread: a parallel region costs more. */
#define ORC_PARALLEL_MIN_WORK 2000000LL

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_MASS (-2)
#define ORC_ERR_ALLOC (-3)

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Squared Euclidean distance, written as the direct difference. */
static double sq_dist(const double* p, const double* q, int32_t d) {
  double s = 0.0;
  for (int32_t k = 0; k < d; ++k) {
    double t = p[k] - q[k];
    s += t * t;
  }
  return s;
}

/*
 * One potential update for a set of "query" points P against "key" points Q:
 *   out[k] = -eps * log( sum_j wq_j * exp((pot_q_j - C(P_row, Q_j)) / eps) ),
 * with row = rows[k] (or k when rows is NULL), the sum skipping wq_j == 0.
 * With (P,Q,wq,pot_q) = (x,y,b,g) this is the f-update F(g); with (y,x,a,f) it
 * is the g-update G(f).
 */
int oracle_lse_update(const double* P, int64_t np, const double* Q, int64_t nq, int32_t d,
                      const double* wq, const double* pot_q, double eps, const int64_t* rows,
                      int64_t n_rows, double* out) {
  if (!P || !Q || !wq || !pot_q || !out || np < 1 || nq < 1 || d < 1 || !(eps > 0.0))
    return ORC_ERR_ARG;
  int bad = 0;
#pragma omp parallel if (n_rows * nq * d > ORC_PARALLEL_MIN_WORK)
  {
    double* z = (double*)malloc(sizeof(double) * (size_t)nq);
    if (!z) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 16)
    for (int64_t k = 0; k < n_rows; ++k) {
      if (!z) continue;
      int64_t i = rows ? rows[k] : k;
      const double* p = P + i * d;
      /* pass 1: exponents and their maximum */
      double zmax = -INFINITY;
      for (int64_t j = 0; j < nq; ++j) {
        if (wq[j] == 0.0) {
          z[j] = -INFINITY;
          continue;
        }
        double c = sq_dist(p, Q + j * d, d);
        z[j] = (pot_q[j] - c) / eps + log(wq[j]);
        if (z[j] > zmax) zmax = z[j];
      }
      /* pass 2: shifted sum of exponentials */
      double s = 0.0;
      for (int64_t j = 0; j < nq; ++j) {
        if (wq[j] == 0.0) continue;
        s += exp(z[j] - zmax);
      }
      out[k] = -eps * (zmax + log(s));
    }
    free(z);
  }
  return bad ? ORC_ERR_ALLOC : ORC_OK;
}

static int check_mass(const double* a, int64_t n, const double* b, int64_t m) {
  double sa = 0.0, sb = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    if (!(a[i] >= 0.0) || isinf(a[i])) return ORC_ERR_ARG;
    sa += a[i];
  }
  for (int64_t j = 0; j < m; ++j) {
    if (!(b[j] >= 0.0) || isinf(b[j])) return ORC_ERR_ARG;
    sb += b[j];
  }
  if (!(sa > 0.0) || !(sb > 0.0)) return ORC_ERR_MASS;
  double big = sa > sb ? sa : sb;
  if (fabs(sa - sb) > 1e-5 * big) return ORC_ERR_MASS;
  return ORC_OK;
}

/* Fixed-count alternating Sinkhorn: g <- g_init (or 0); repeat n_iters: f <- F(g), g <- G(f). */
int oracle_potentials(const double* x, int64_t n, const double* y, int64_t m, int32_t d,
                      const double* a, const double* b, double eps, int32_t n_iters,
                      const double* g_init, double* f_out, double* g_out) {
  if (!x || !y || !a || !b || !f_out || !g_out || n < 1 || m < 1 || d < 1 || n_iters < 1 ||
      !(eps > 0.0) || isinf(eps))
    return ORC_ERR_ARG;
  int rc = check_mass(a, n, b, m);
  if (rc) return rc;
  for (int64_t j = 0; j < m; ++j) g_out[j] = g_init ? g_init[j] : 0.0;
  for (int32_t it = 0; it < n_iters; ++it) {
    rc = oracle_lse_update(x, n, y, m, d, b, g_out, eps, NULL, n, f_out);
    if (rc) return rc;
    rc = oracle_lse_update(y, m, x, n, d, a, f_out, eps, NULL, m, g_out);
    if (rc) return rc;
  }
  return ORC_OK;
}

/*
 * Row sums of the plan for a set of rows: out[k] = sum_j P_ij, i = rows[k] (or k),
 * P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps). Column sums: call with the clouds,
 * weights and potentials swapped.
 */
int oracle_plan_row_sums(const double* x, int64_t n, const double* y, int64_t m, int32_t d,
                         const double* a, const double* b, double eps, const double* f,
                         const double* g, const int64_t* rows, int64_t n_rows, double* out) {
  if (!x || !y || !a || !b || !f || !g || !out || n < 1 || m < 1 || d < 1 || !(eps > 0.0))
    return ORC_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 16) if (n_rows * m * d > ORC_PARALLEL_MIN_WORK)
  for (int64_t k = 0; k < n_rows; ++k) {
    int64_t i = rows ? rows[k] : k;
    double s = 0.0;
    for (int64_t j = 0; j < m; ++j) {
      double c = sq_dist(x + i * d, y + j * d, d);
      s += a[i] * b[j] * exp((f[i] + g[j] - c) / eps);
    }
    out[k] = s;
  }
  return ORC_OK;
}

/* D(f,g) = <f,a> + <g,b> - eps*(sum_ij P_ij - m_a*m_b), the plan mass summed term by term. */
int oracle_cost(const double* x, int64_t n, const double* y, int64_t m, int32_t d,
                const double* a, const double* b, double eps, const double* f, const double* g,
                double* out) {
  if (!out) return ORC_ERR_ARG;
  double* r = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  if (!r) return ORC_ERR_ALLOC;
  int rc = oracle_plan_row_sums(x, n, y, m, d, a, b, eps, f, g, NULL, n, r);
  if (rc) {
    free(r);
    return rc;
  }
  double fa = 0.0, gb = 0.0, mass = 0.0, ma = 0.0, mb = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    fa += f[i] * a[i];
    mass += r[i];
    ma += a[i];
  }
  for (int64_t j = 0; j < m; ++j) {
    gb += g[j] * b[j];
    mb += b[j];
  }
  free(r);
  *out = fa + gb - eps * (mass - ma * mb);
  return ORC_OK;
}

/*
 * Envelope gradient with respect to x for a set of rows:
 *   ft_i = F(g)_i,  Pt_ij = a_i b_j exp((ft_i + g_j - C_ij)/eps),
 *   grad[k, :] = 2 * (a_i x_i - sum_j Pt_ij y_j),  i = rows[k] (or k).
 */
int oracle_grad_x(const double* x, int64_t n, const double* y, int64_t m, int32_t d,
                  const double* a, const double* b, double eps, const double* g,
                  const int64_t* rows, int64_t n_rows, double* grad) {
  if (!x || !y || !a || !b || !g || !grad || n < 1 || m < 1 || d < 1 || !(eps > 0.0))
    return ORC_ERR_ARG;
  double* ft = (double*)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1));
  if (!ft) return ORC_ERR_ALLOC;
  int rc = oracle_lse_update(x, n, y, m, d, b, g, eps, rows, n_rows, ft);
  if (rc) {
    free(ft);
    return rc;
  }
  int bad = 0;
#pragma omp parallel if (n_rows * m * d > ORC_PARALLEL_MIN_WORK)
  {
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    if (!acc) {
#pragma omp atomic write
      bad = 1;
    }
#pragma omp for schedule(dynamic, 16)
    for (int64_t k = 0; k < n_rows; ++k) {
      if (!acc) continue;
      int64_t i = rows ? rows[k] : k;
      for (int32_t c = 0; c < d; ++c) acc[c] = 0.0;
      for (int64_t j = 0; j < m; ++j) {
        double cij = sq_dist(x + i * d, y + j * d, d);
        double p = a[i] * b[j] * exp((ft[k] + g[j] - cij) / eps);
        for (int32_t c = 0; c < d; ++c) acc[c] += p * y[j * d + c];
      }
      for (int32_t c = 0; c < d; ++c) grad[k * d + c] = 2.0 * (a[i] * x[i * d + c] - acc[c]);
    }
    free(acc);
  }
  free(ft);
  return bad ? ORC_ERR_ALLOC : ORC_OK;
}

/* max(|P1 - a|_inf, |P^T 1 - b|_inf) at (f, g), from the explicit row and column sums. */
static int marginal_violation(const double* x, int64_t n, const double* y, int64_t m, int32_t d,
                              const double* a, const double* b, double eps, const double* f,
                              const double* g, double* out) {
  double* r = (double*)malloc(sizeof(double) * (size_t)n);
  double* c = (double*)malloc(sizeof(double) * (size_t)m);
  if (!r || !c) {
    free(r);
    free(c);
    return ORC_ERR_ALLOC;
  }
  int rc = oracle_plan_row_sums(x, n, y, m, d, a, b, eps, f, g, NULL, n, r);
  if (!rc) rc = oracle_plan_row_sums(y, m, x, n, d, b, a, eps, g, f, NULL, m, c);
  double v = 0.0;
  if (!rc) {
    for (int64_t i = 0; i < n; ++i) v = fmax(v, fabs(r[i] - a[i]));
    for (int64_t j = 0; j < m; ++j) v = fmax(v, fabs(c[j] - b[j]));
  }
  free(r);
  free(c);
  *out = v;
  return rc;
}

#define ORC_ALTERNATING 0
#define ORC_SYMMETRIC 1
#define ORC_STOP_FIXED 0
#define ORC_STOP_MARGINAL 1
#define ORC_STOP_POTENTIAL 2

/*
 * The general solve. Under stop_mode fixed it runs n_iters iterations and reports
 * iters_run = n_iters, converged = -1, final_viol = NaN; otherwise at most stop_max_iter
 * iterations with a check after every stop_check_every-th one and after the last one.
 */
int oracle_solve(const double* x, int64_t n, const double* y, int64_t m, int32_t d,
                 const double* a, const double* b, double eps, int32_t variant, double alpha,
                 int32_t stop_mode, int32_t n_iters, int32_t stop_max_iter, double stop_tol,
                 int32_t stop_check_every, const double* g_init, double* f_out, double* g_out,
                 int32_t* iters_run, int32_t* converged, double* final_viol) {
  if (!x || !y || !a || !b || !f_out || !g_out || !iters_run || !converged || !final_viol ||
      n < 1 || m < 1 || d < 1 || !(eps > 0.0) || isinf(eps))
    return ORC_ERR_ARG;
  if (variant != ORC_ALTERNATING && variant != ORC_SYMMETRIC) return ORC_ERR_ARG;
  if (variant == ORC_SYMMETRIC && !(alpha > 0.0 && alpha <= 1.0)) return ORC_ERR_ARG;
  if (stop_mode < ORC_STOP_FIXED || stop_mode > ORC_STOP_POTENTIAL) return ORC_ERR_ARG;
  if (stop_mode == ORC_STOP_FIXED ? n_iters < 1
                                  : (stop_max_iter < 1 || stop_check_every < 1 || !(stop_tol >= 0.0)))
    return ORC_ERR_ARG;
  int rc = check_mass(a, n, b, m);
  if (rc) return rc;
  const int32_t total = stop_mode == ORC_STOP_FIXED ? n_iters : stop_max_iter;
  double* fn = (double*)malloc(sizeof(double) * (size_t)n);
  double* gn = (double*)malloc(sizeof(double) * (size_t)m);
  double* fp = (double*)malloc(sizeof(double) * (size_t)n);
  double* gp = (double*)malloc(sizeof(double) * (size_t)m);
  if (!fn || !gn || !fp || !gp) {
    free(fn);
    free(gn);
    free(fp);
    free(gp);
    return ORC_ERR_ALLOC;
  }
  for (int64_t i = 0; i < n; ++i) f_out[i] = fp[i] = 0.0;
  for (int64_t j = 0; j < m; ++j) g_out[j] = gp[j] = g_init ? g_init[j] : 0.0;
  *iters_run = 0;
  *converged = stop_mode == ORC_STOP_FIXED ? -1 : 0;
  *final_viol = NAN;
  for (int32_t it = 1; it <= total && !rc; ++it) {
    if (variant == ORC_ALTERNATING) {
      rc = oracle_lse_update(x, n, y, m, d, b, g_out, eps, NULL, n, f_out);
      if (!rc) rc = oracle_lse_update(y, m, x, n, d, a, f_out, eps, NULL, m, g_out);
    } else {
      rc = oracle_lse_update(x, n, y, m, d, b, g_out, eps, NULL, n, fn);
      if (!rc) rc = oracle_lse_update(y, m, x, n, d, a, f_out, eps, NULL, m, gn);
      if (!rc) {
        for (int64_t i = 0; i < n; ++i) f_out[i] = (1.0 - alpha) * f_out[i] + alpha * fn[i];
        for (int64_t j = 0; j < m; ++j) g_out[j] = (1.0 - alpha) * g_out[j] + alpha * gn[j];
      }
    }
    if (rc) break;
    *iters_run = it;
    if (stop_mode == ORC_STOP_FIXED || (it % stop_check_every != 0 && it != total)) continue;
    double v = 0.0;
    if (stop_mode == ORC_STOP_MARGINAL) {
      rc = marginal_violation(x, n, y, m, d, a, b, eps, f_out, g_out, &v);
      if (rc) break;
    } else {
      for (int64_t i = 0; i < n; ++i) {
        v = fmax(v, fabs(f_out[i] - fp[i]));
        fp[i] = f_out[i];
      }
      for (int64_t j = 0; j < m; ++j) {
        v = fmax(v, fabs(g_out[j] - gp[j]));
        gp[j] = g_out[j];
      }
    }
    *final_viol = v;
    if (stop_mode == ORC_STOP_MARGINAL ? v <= stop_tol : v < stop_tol) {
      *converged = 1;
      break;
    }
  }
  free(fn);
  free(gn);
  free(fp);
  free(gp);
  return rc;
}
