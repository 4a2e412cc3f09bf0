/*
 * rlscan_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, sequential fp64 CPU reference for the seven credit-assignment
 * estimators.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load this library; the product path (librlscan) never
 * does, and the two share no code, header, table or helper.
 *
 * Every routine reads the same fp32 / uint8 / int32 host arrays the GPU path
 * reads, computes in double precision with one loop per row in the natural
 * time order of the estimator, and writes double outputs.  Nothing here is
 * blocked, fused or reassociated: each estimator is written in its textbook
 * recursive form, NOT through the (a_t, b_t) coefficients the GPU scan uses.
 *
 * Source of what is computed:
 *  - "rl-triton: High-Performance Triton GPU Kernels for Reinforcement
 *    Learning Credit Assignment" (arxivlens page), Abstract: the seven
 *    estimators, all instances of one first-order linear recurrence.
 *  - Same title (gist.science technical summary), Methodologie 1 "Unified
 *    Algebraic Framework": the backward recurrence A_t = alpha_t + beta_t *
 *    A_{t+1} and its forward-time mirror for eligibility traces.
 *  - Same page, Methodologie 3 "Expliciete Boundary Semantiek": termination
 *    means the successor value is zero; truncation means an appended
 *    bootstrap value replaces it; the end of the rollout window (t = T-1)
 *    takes the bootstrap once.
 *  - The pages name each estimator but print no formula for it, so each one
 *    follows its original paper: GAE (Schulman et al. 2016), V-trace
 *    (Espeholt et al. 2018, IMPALA), Retrace(lambda) (Munos et al. 2016),
 *    TD(lambda) lambda-returns and discounted returns (Sutton & Barto),
 *    accumulating eligibility traces (Sutton & Barto), and an episodic
 *    (reset-on-done) inclusive prefix sum.
 *
 * Conventions (layout): every per-step array is row-major [N, T] with T
 * contiguous; Retrace's q and pi are [N, T, A] with A contiguous.  Flags are
 * uint8, nonzero = true.  `truncated` may be NULL (no truncation), in which
 * case `trunc_value` is ignored.  `bootstrap` is [N]; where documented as
 * nullable, NULL means 0.
 *
 * Readings where the pages are silent (the same ones the GPU path uses):
 *  - the successor value nv_t of step t is: 0 if terminated[t]; else
 *    trunc_value[t] if truncated[t]; else bootstrap[n] if t == T-1; else the
 *    next step's value.  Termination wins over truncation on the same step.
 *  - the window end t = T-1 always takes the bootstrap in the local term of
 *    step T-1 (never in a carried-in value), so it is counted once.
 *  - eligibility traces and prefix sums reset after any done step
 *    (terminated or truncated); the reset applies from the next step on.
 *
 * Return value of every routine: 0 on success, -1 on an invalid argument.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

/* Does the transition out of step t carry on to step t+1 inside this window? */
static int continues(int64_t t, int64_t T, const uint8_t *term_row,
                     const uint8_t *trunc_row) {
  if (term_row[t]) return 0;
  if (trunc_row && trunc_row[t]) return 0;
  return t + 1 < T;
}

/* Successor value used when the step does not continue (boundary semantics). */
static double boundary_value(int64_t n, int64_t t, const uint8_t *term_row,
                             const uint8_t *trunc_row, const float *tv_row,
                             const float *bootstrap) {
  if (term_row[t]) return 0.0;
  if (trunc_row && trunc_row[t]) return (double)tv_row[t];
  return bootstrap ? (double)bootstrap[n] : 0.0; /* window end */
}

static int bad_dims(int64_t N, int64_t T) { return N < 0 || T < 0; }

/* Generalized Advantage Estimation (Schulman et al. 2016):
 *   delta_t = r_t + gamma * V(s_{t+1}) - V(s_t)
 *   A_t     = delta_t + gamma * lambda * A_{t+1}   (A cut to 0 past a boundary)
 *   R_t     = A_t + V(s_t)
 * `returns` may be NULL. */
int rlo_gae(int64_t N, int64_t T, const float *rewards, const float *values,
            const float *bootstrap, const uint8_t *terminated,
            const uint8_t *truncated, const float *trunc_value, double gamma,
            double lambda, double *advantages, double *returns) {
  if (bad_dims(N, T)) return -1;
  for (int64_t n = 0; n < N; ++n) {
    const float *r = rewards + n * T, *v = values + n * T;
    const uint8_t *te = terminated + n * T;
    const uint8_t *tr = truncated ? truncated + n * T : NULL;
    const float *tv = trunc_value ? trunc_value + n * T : NULL;
    double next_adv = 0.0;
    for (int64_t t = T - 1; t >= 0; --t) {
      int c = continues(t, T, te, tr);
      double next_v = c ? (double)v[t + 1] : boundary_value(n, t, te, tr, tv, bootstrap);
      double delta = (double)r[t] + gamma * next_v - (double)v[t];
      double adv = delta + (c ? gamma * lambda * next_adv : 0.0);
      advantages[n * T + t] = adv;
      if (returns) returns[n * T + t] = adv + (double)v[t];
      next_adv = adv;
    }
  }
  return 0;
}

/* TD(lambda) returns (lambda-returns, Sutton & Barto):
 *   G_t = r_t + gamma * ((1 - lambda) * V(s_{t+1}) + lambda * G_{t+1})
 * and at a boundary G_t = r_t + gamma * nv_t. */
int rlo_td_lambda(int64_t N, int64_t T, const float *rewards,
                  const float *values, const float *bootstrap,
                  const uint8_t *terminated, const uint8_t *truncated,
                  const float *trunc_value, double gamma, double lambda,
                  double *out) {
  if (bad_dims(N, T)) return -1;
  for (int64_t n = 0; n < N; ++n) {
    const float *r = rewards + n * T, *v = values + n * T;
    const uint8_t *te = terminated + n * T;
    const uint8_t *tr = truncated ? truncated + n * T : NULL;
    const float *tv = trunc_value ? trunc_value + n * T : NULL;
    double next_g = 0.0;
    for (int64_t t = T - 1; t >= 0; --t) {
      double g;
      if (continues(t, T, te, tr))
        g = (double)r[t] + gamma * ((1.0 - lambda) * (double)v[t + 1] + lambda * next_g);
      else
        g = (double)r[t] + gamma * boundary_value(n, t, te, tr, tv, bootstrap);
      out[n * T + t] = g;
      next_g = g;
    }
  }
  return 0;
}

/* Discounted (Monte-Carlo) return: G_t = r_t + gamma * G_{t+1}; at a
 * boundary G_t = r_t + gamma * nv_t.  `bootstrap` may be NULL (= 0). */
int rlo_discounted_return(int64_t N, int64_t T, const float *rewards,
                          const float *bootstrap, const uint8_t *terminated,
                          const uint8_t *truncated, const float *trunc_value,
                          double gamma, double *out) {
  if (bad_dims(N, T)) return -1;
  for (int64_t n = 0; n < N; ++n) {
    const float *r = rewards + n * T;
    const uint8_t *te = terminated + n * T;
    const uint8_t *tr = truncated ? truncated + n * T : NULL;
    const float *tv = trunc_value ? trunc_value + n * T : NULL;
    double next_g = 0.0;
    for (int64_t t = T - 1; t >= 0; --t) {
      double g;
      if (continues(t, T, te, tr))
        g = (double)r[t] + gamma * next_g;
      else
        g = (double)r[t] + gamma * boundary_value(n, t, te, tr, tv, bootstrap);
      out[n * T + t] = g;
      next_g = g;
    }
  }
  return 0;
}

static double dmin(double a, double b) { return a < b ? a : b; }

/* V-trace (Espeholt et al. 2018), with the trace coefficient scaled by lambda:
 *   rho_t = min(rho_bar, exp(log_rho_t)),  c_t = lambda * min(c_bar, exp(log_rho_t))
 *   vs_t - V(s_t) = rho_t * (r_t + gamma V(s_{t+1}) - V(s_t))
 *                   + gamma * c_t * (vs_{t+1} - V(s_{t+1}))
 *   pg_adv_t = rho_t * (r_t + gamma * vs_{t+1} - V(s_t))
 * At a boundary V(s_{t+1}) and vs_{t+1} are both replaced by nv_t and the
 * carried correction is cut.  `pg_advantages` may be NULL. */
int rlo_vtrace(int64_t N, int64_t T, const float *log_rhos,
               const float *rewards, const float *values,
               const float *bootstrap, const uint8_t *terminated,
               const uint8_t *truncated, const float *trunc_value,
               double gamma, double lambda, double rho_bar, double c_bar,
               double *vs, double *pg_advantages) {
  if (bad_dims(N, T)) return -1;
  for (int64_t n = 0; n < N; ++n) {
    const float *lr = log_rhos + n * T, *r = rewards + n * T, *v = values + n * T;
    const uint8_t *te = terminated + n * T;
    const uint8_t *tr = truncated ? truncated + n * T : NULL;
    const float *tv = trunc_value ? trunc_value + n * T : NULL;
    double next_vs = 0.0; /* vs_{t+1}, valid only when step t continues */
    for (int64_t t = T - 1; t >= 0; --t) {
      double ratio = exp((double)lr[t]);
      double rho = dmin(rho_bar, ratio);
      double c = lambda * dmin(c_bar, ratio);
      int cont = continues(t, T, te, tr);
      double succ_v, succ_vs, carried;
      if (cont) {
        succ_v = (double)v[t + 1];
        succ_vs = next_vs;
        carried = gamma * c * (next_vs - (double)v[t + 1]);
      } else {
        succ_v = boundary_value(n, t, te, tr, tv, bootstrap);
        succ_vs = succ_v;
        carried = 0.0;
      }
      double vs_t = (double)v[t] + rho * ((double)r[t] + gamma * succ_v - (double)v[t]) + carried;
      vs[n * T + t] = vs_t;
      if (pg_advantages)
        pg_advantages[n * T + t] = rho * ((double)r[t] + gamma * succ_vs - (double)v[t]);
      next_vs = vs_t;
    }
  }
  return 0;
}

/* Retrace(lambda) (Munos et al. 2016), recursive target form:
 *   E_t = sum_a pi_t(a) Q_t(a),  q_t = Q_t(a_t),
 *   c_t = lambda * min(1, pi_t(a_t) / mu_t)      (mu_t = behaviour prob of a_t)
 *   Qret_t = r_t + gamma * (E_{t+1} - c_{t+1} q_{t+1} + c_{t+1} Qret_{t+1})
 * and at a boundary Qret_t = r_t + gamma * nv_t, where the bootstrap and the
 * truncation values are expected values E_pi Q of the successor state.
 * Returns -2 if an action index is outside [0, A). */
int rlo_retrace(int64_t N, int64_t T, int64_t A, const float *q,
                const float *pi, const float *mu_a, const int32_t *actions,
                const float *rewards, const float *bootstrap,
                const uint8_t *terminated, const uint8_t *truncated,
                const float *trunc_value, double gamma, double lambda,
                double *q_ret) {
  if (bad_dims(N, T) || A < 1) return -1;
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t *te = terminated + n * T;
    const uint8_t *tr = truncated ? truncated + n * T : NULL;
    const float *tv = trunc_value ? trunc_value + n * T : NULL;
    double next_qret = 0.0, next_e = 0.0, next_c = 0.0, next_q = 0.0;
    for (int64_t t = T - 1; t >= 0; --t) {
      int64_t i = n * T + t;
      int32_t a = actions[i];
      if (a < 0 || (int64_t)a >= A) return -2;
      const float *qrow = q + i * A, *prow = pi + i * A;
      double e = 0.0;
      for (int64_t k = 0; k < A; ++k) e += (double)prow[k] * (double)qrow[k];
      double ratio = (double)prow[a] / (double)mu_a[i];
      double c = lambda * dmin(1.0, ratio);
      double qa = (double)qrow[a];
      double g;
      if (continues(t, T, te, tr))
        g = (double)rewards[i] + gamma * (next_e - next_c * next_q + next_c * next_qret);
      else
        g = (double)rewards[i] + gamma * boundary_value(n, t, te, tr, tv, bootstrap);
      q_ret[i] = g;
      next_qret = g;
      next_e = e;
      next_c = c;
      next_q = qa;
    }
  }
  return 0;
}

/* Accumulating eligibility trace, forward in time (Sutton & Barto):
 *   e_t = g_t + gamma * lambda * e_{t-1},  e_{-1} = init_trace[n] (NULL = 0),
 * and the trace restarts (e_{t-1} := 0) after a done step. */
int rlo_elig_trace(int64_t N, int64_t T, const float *inputs,
                   const float *init_trace, const uint8_t *terminated,
                   const uint8_t *truncated, double gamma, double lambda,
                   double *traces) {
  if (bad_dims(N, T)) return -1;
  for (int64_t n = 0; n < N; ++n) {
    const float *g = inputs + n * T;
    const uint8_t *te = terminated + n * T;
    const uint8_t *tr = truncated ? truncated + n * T : NULL;
    double prev = init_trace ? (double)init_trace[n] : 0.0;
    for (int64_t t = 0; t < T; ++t) {
      if (t > 0 && (te[t - 1] || (tr && tr[t - 1]))) prev = 0.0;
      double e = (double)g[t] + gamma * lambda * prev;
      traces[n * T + t] = e;
      prev = e;
    }
  }
  return 0;
}

/* Episodic inclusive prefix sum, forward in time: S_t = x_t + S_{t-1},
 * S_{-1} = 0, restarting after a done step.  Accumulates in int64 and stores
 * the two's-complement low 32 bits; *max_abs receives max |S| in int64 so
 * callers can confirm that no wrap-around happened. */
int rlo_episodic_prefix_sum(int64_t N, int64_t T, const int32_t *x,
                            const uint8_t *terminated, const uint8_t *truncated,
                            int32_t *out, int64_t *max_abs) {
  if (bad_dims(N, T)) return -1;
  int64_t m = 0;
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t *te = terminated + n * T;
    const uint8_t *tr = truncated ? truncated + n * T : NULL;
    int64_t s = 0;
    for (int64_t t = 0; t < T; ++t) {
      if (t > 0 && (te[t - 1] || (tr && tr[t - 1]))) s = 0;
      s += (int64_t)x[n * T + t];
      int64_t mag = s < 0 ? -s : s;
      if (mag > m) m = mag;
      out[n * T + t] = (int32_t)(uint32_t)(uint64_t)s;
    }
  }
  if (max_abs) *max_abs = m;
  return 0;
}

/* Generic first-order linear recurrence (the pages' unified form, gist.science
 * technical summary, Methodologie 1, with the coefficients given directly):
 * in scan order (t = 0..T-1 forward, t = T-1..0 when `reverse`),
 *   x_t = b_t + a_t * x_prev,
 * where x_prev is the previous step in scan order, or init[n] (NULL: 0) for
 * the row's first step; reset[t] != 0 (reset may be NULL) cuts the
 * dependency, x_t = b_t. */
int rlo_affine_scan(int64_t N, int64_t T, const float *a, const float *b,
                    const uint8_t *reset, const float *init, int reverse,
                    double *x) {
  if (bad_dims(N, T)) return -1;
  for (int64_t n = 0; n < N; ++n) {
    double carry = init ? (double)init[n] : 0.0;
    for (int64_t k = 0; k < T; ++k) {
      const int64_t t = reverse ? T - 1 - k : k;
      const int64_t i = n * T + t;
      double v = (double)b[i];
      if (!(reset && reset[i])) v += (double)a[i] * carry;
      x[i] = v;
      carry = v;
    }
  }
  return 0;
}

/* Gradient (adjoint) of rlo_affine_scan for a loss whose direct derivative
 * with respect to x_t is dy_t.  x is the forward scan's output.  In the
 * forward scan's order, with nxt(t) the following step and prv(t) the
 * preceding one:
 *   g_t   = dy_t + [nxt(t) exists and not reset] a_nxt(t) g_nxt(t)
 *   db_t  = g_t
 *   da_t  = [not reset_t] g_t * (x_prv(t), or init[n] at the first step)
 *   dinit = [not reset at the first step] a_first g_first
 * (the chain rule through the recurrence, evaluated last step first).
 * da and dinit may be NULL. */
int rlo_affine_scan_grad(int64_t N, int64_t T, const float *a, const float *x,
                         const float *dy, const uint8_t *reset, const float *init,
                         int reverse, double *da, double *db, double *dinit) {
  if (bad_dims(N, T)) return -1;
  for (int64_t n = 0; n < N; ++n) {
    double g_next = 0.0, a_next = 0.0;
    int have_next = 0, reset_next = 0;
    for (int64_t k = T - 1; k >= 0; --k) { /* scan position k, last first */
      const int64_t t = reverse ? T - 1 - k : k;
      const int64_t i = n * T + t;
      double g = (double)dy[i];
      if (have_next && !reset_next) g += a_next * g_next;
      db[i] = g;
      const int r = reset && reset[i];
      if (da) {
        double xp;
        if (k == 0)
          xp = init ? (double)init[n] : 0.0;
        else
          xp = (double)x[n * T + (reverse ? t + 1 : t - 1)];
        da[i] = r ? 0.0 : g * xp;
      }
      if (k == 0 && dinit) dinit[n] = r ? 0.0 : (double)a[i] * g;
      g_next = g;
      a_next = (double)a[i];
      reset_next = r;
      have_next = 1;
    }
  }
  return 0;
}

/* rlo_affine_scan on time-major arrays: element (t, n) of a, b, reset and x
 * at t * N + n (each time step a contiguous row of the N environments);
 * init is [N].  Same recurrence, same scan order per environment. */
int rlo_affine_scan_tm(int64_t N, int64_t T, const float *a, const float *b,
                       const uint8_t *reset, const float *init, int reverse,
                       double *x) {
  if (bad_dims(N, T)) return -1;
  for (int64_t n = 0; n < N; ++n) {
    double carry = init ? (double)init[n] : 0.0;
    for (int64_t k = 0; k < T; ++k) {
      const int64_t t = reverse ? T - 1 - k : k;
      const int64_t i = t * N + n;
      double v = (double)b[i];
      if (!(reset && reset[i])) v += (double)a[i] * carry;
      x[i] = v;
      carry = v;
    }
  }
  return 0;
}
