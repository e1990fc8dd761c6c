/*
 * s6_oracle.c -- plain, slow, fp64 CPU oracle for the selective scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library and its Python binding) shares no code with it and never
 * calls it.
 *
 * Sources (page title, section):
 *  [KN1]  "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 *         (chapterpal.com), Knowl 1 "Selective State Space Layer (S6)":
 *         steps 2-4 and the per-element loop (discretize, update, readout).
 *  [KN4]  same page, Knowl 4 "Equivalence of Zero-Order Hold Selective SSM to
 *         Gated Recurrent Units" (Theorem 1).
 *  [PG33] "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 *         (paper-graph-ui summary), section 3.4, "Algorithm 2 (Selective S6)"
 *         and "The specific functional forms" (softplus), and "The Mamba
 *         Architecture" (SiLU gate branch).
 *  [TP-II6] "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 *         (trishampatil.com engineering walk-through), Part II section 4
 *         (h_0 = 0) and section 6 (Algorithm 2 shapes).
 *  [TP-III4] same page, Part III section 4 (recomputation in the backward).
 *  [KN3]  chapterpal.com page, Knowl 3 "Mamba Block Architecture", step 3:
 *         the main branch runs a short 1D temporal convolution of width
 *         d_conv = 4, then SiLU, then the S6 layer.
 *  [PG36] paper-graph-ui summary, section 3.6 "Additional Model Details",
 *         "Parameterization of Delta's input projection" (the low-rank
 *         s_Delta(x) = Linear_D(Linear_R(x))).
 *  [PG-T8] paper-graph-ui summary, "Ablation Studies and Robustness Checks",
 *         "Parameterization of A (Table 8)": S4D-Lin, A_n = -1/2 + n i.
 *  [PG34] paper-graph-ui summary, "The Mamba Architecture (Section 3.4)",
 *         "The Mamba simplification": convolution (local context, the
 *         "shift-SSM" of H3), SiLU, selective SSM on the main branch.
 *
 * What is computed (forward), for every batch b and channel d independently:
 *     Delta_t = softplus(delta[b,d,t] + bias[d])                     [PG33]
 *     for n:  Abar = exp(Delta_t * A[d,n])                           [KN1 step 3]
 *             Bbar = (exp(Delta_t * A[d,n]) - 1) / A[d,n] * B[b,n,t] [KN1 step 3]
 *             h[n] = Abar * h[n] + Bbar * u[b,d,t]                   [KN1 step 4]
 *     y0_t = sum_n C[b,n,t] * h[n]  (+ D[d] * u[b,d,t] if D given)   [KN1 step 4]
 *     y_t  = y0_t * silu(z[b,d,t])  (if z given)                     [PG33 block]
 * with h = 0 before the first step [TP-II6 s.4] (or a given initial state, to
 * continue a sequence one call or one token at a time: the recurrent mode of
 * [TP-II6] section 4, "best for autoregressive inference") and last_state = h
 * after the last step.
 *
 * Readings where the pages are silent or ambiguous (each one is listed in the
 * design notes of the repository):
 *  - Bbar is the exact zero-order-hold value for a diagonal A, evaluated as
 *    Delta * psi(Delta*A) * B with psi(x) = expm1(x)/x (psi(0) = 1), which is
 *    the same quantity written without the cancellation of exp(x) - 1 and
 *    without the division by A (so A = 0 is the limit Delta*B).
 *  - softplus is exact (stable form, no large-argument cutoff).
 *  - The D skip and the z gate are not on the pages; y = (C.h + D*u)*silu(z).
 *
 * The backward is the adjoint of the forward above, derived by hand from it
 * (the pages give no gradient formulas).  States are recomputed forward per
 * channel and kept in fp64 (the oracle has no memory constraint), then a
 * reverse sweep accumulates gradients [TP-III4].
 *
 * Convolution prologue (s6_oracle_conv_*), [KN3] / [PG34], with the readings
 * the pages leave open: the convolution is depthwise (one filter of width W
 * per channel, as the pages apply it per channel of the branch), causal
 * (x = 0 before the first step, so that step t sees no later input, as a
 * recurrent model needs) and has an optional per-channel bias:
 *     pre[b,d,t] = conv_b[d] + sum_{k=0}^{W-1} conv_w[d,k] * x[b,d,t-(W-1)+k]
 *     u[b,d,t]   = pre * sigmoid(pre)                                (SiLU)
 * and u feeds the forward above.  Its backward is the chain rule through the
 * SiLU and the convolution after the S6 backward has given du.
 *
 * Low-rank Delta projection (s6_oracle_dtproj_*), [PG36] "Parameterization
 * of Delta's input projection": s_Delta(x) = Linear_D(Linear_R(x)) with a
 * small rank R.  The scan takes the rank-R projection dt_low = Linear_R(x)
 * (batch, R, L) and the weight W_dt (dim, R) of Linear_D, whose bias is
 * delta_bias:
 *     delta[b,d,t] = sum_r W_dt[d,r] * dt_low[b,r,t]
 * and delta feeds the forward above (softplus(delta + delta_bias)).  Its
 * backward is the chain rule through that product after the S6 backward has
 * given ddelta.
 *
 * Complex-valued diagonal A (s6_oracle_cplx_*), [PG36] "Real vs. Complex
 * parameters" and [PG-T8] (S4D-Lin, A_n = -1/2 + n i): the state, A, B and C
 * are complex, u, delta, z and y real.  Readings where the pages say no more:
 * B_t and C_t are input-dependent complex vectors; the output is the real
 * part of the readout; the same zero-order hold with complex exp and psi:
 *     Abar = exp(Delta A_n),  Bbar = (exp(Delta A_n) - 1) / A_n * B_n,
 *     h_n  = Abar h_n + Bbar u,   y0 = Re(sum_n C_n h_n) + D u.
 * A complex vector of N entries is passed as 2N doubles, real parts first
 * ("planar"): A (dim, 2N), B and C (batch, 2N, L), states (batch, dim, 2N).
 * Gradients of complex inputs are the pairs (d/d re, d/d im), stored the
 * same way.
 *
 * Parity pins (the tests check this file against): Theorem 1 closed form,
 * the LTI convolution form, brute-force unrolling, an independent ZOH via the
 * matrix exponential, the exact ODE solution for a step input, finite
 * differences and autograd for the backward, and exact hand-derived values.
 */
#include <complex.h>
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef long long i64;

/* softplus(v) = log(1 + e^v), stable form. */
static double softplus(double v) {
  if (v > 0.0) return v + log1p(exp(-v));
  return log1p(exp(v));
}

/* logistic sigmoid, stable form. */
static double sigmoid(double v) {
  if (v >= 0.0) return 1.0 / (1.0 + exp(-v));
  double e = exp(v);
  return e / (1.0 + e);
}

/* psi(x) = (exp(x) - 1) / x, psi(0) = 1. */
static double psi(double x) {
  if (x == 0.0) return 1.0;
  return expm1(x) / x;
}

/* phi(x) = d psi / dx = (x e^x - expm1(x)) / x^2; series near 0. */
static double phi(double x) {
  if (fabs(x) < 1e-2) {
    /* sum_k (k+1)/(k+2)! x^k */
    return 0.5 + x * (1.0 / 3.0 + x * (1.0 / 8.0 + x * (1.0 / 30.0 + x * (1.0 / 144.0))));
  }
  return (x * exp(x) - expm1(x)) / (x * x);
}

typedef struct {
  const double *u, *delta, *bias, *A, *B, *C, *D, *z, *dy;
  const double *h0; /* optional initial state (batch, dim, N); NULL = 0 */
  double *y, *last_state;
  double *du, *ddelta, *dz;
  double *dA_part, *dD_part, *dbias_part; /* per (b,d) partials */
  double *dB_acc, *dC_acc;                /* per-thread (batch,N,L) accumulators */
  i64 batch, dim, L, N;
  i64 first, last; /* range of flattened (b,d) this worker owns */
} job_t;

/* ---------------------------------------------------------------- forward */

static void fwd_channel(const job_t *j, i64 b, i64 d, double *h) {
  const i64 L = j->L, N = j->N, dim = j->dim;
  const double *u = j->u + (b * dim + d) * L;
  const double *dl = j->delta + (b * dim + d) * L;
  const double *z = j->z ? j->z + (b * dim + d) * L : NULL;
  const double *Bm = j->B + b * N * L;
  const double *Cm = j->C + b * N * L;
  const double *A = j->A + d * N;
  const double bias = j->bias ? j->bias[d] : 0.0;
  const double Dd = j->D ? j->D[d] : 0.0;
  double *y = j->y + (b * dim + d) * L;
  for (i64 n = 0; n < N; ++n) h[n] = j->h0 ? j->h0[(b * dim + d) * N + n] : 0.0;
  for (i64 t = 0; t < L; ++t) {
    const double Delta = softplus(dl[t] + bias);
    double y0 = 0.0;
    for (i64 n = 0; n < N; ++n) {
      const double x = Delta * A[n];
      const double Abar = exp(x);
      const double Bbar = Delta * psi(x) * Bm[n * L + t];
      h[n] = Abar * h[n] + Bbar * u[t];
      y0 += Cm[n * L + t] * h[n];
    }
    if (j->D) y0 += Dd * u[t];
    if (z) y0 *= z[t] * sigmoid(z[t]);
    y[t] = y0;
  }
  if (j->last_state) {
    double *ls = j->last_state + (b * dim + d) * N;
    for (i64 n = 0; n < N; ++n) ls[n] = h[n];
  }
}

static void *fwd_worker(void *arg) {
  job_t *j = (job_t *)arg;
  double *h = (double *)malloc(sizeof(double) * (size_t)j->N);
  for (i64 i = j->first; i < j->last; ++i) fwd_channel(j, i / j->dim, i % j->dim, h);
  free(h);
  return NULL;
}

/* --------------------------------------------------------------- backward */

static void bwd_channel(job_t *j, i64 b, i64 d, double *H, double *G) {
  const i64 L = j->L, N = j->N, dim = j->dim;
  const i64 off = (b * dim + d) * L;
  const double *u = j->u + off, *dl = j->delta + off, *dy = j->dy + off;
  const double *z = j->z ? j->z + off : NULL;
  const double *Bm = j->B + b * N * L, *Cm = j->C + b * N * L;
  const double *A = j->A + d * N;
  const double bias = j->bias ? j->bias[d] : 0.0;
  const double Dd = j->D ? j->D[d] : 0.0;

  /* Recompute the forward states; H[(t+1)*N + n] = h_t, H[n] = h_{-1} = 0. */
  for (i64 n = 0; n < N; ++n) H[n] = 0.0;
  for (i64 t = 0; t < L; ++t) {
    const double Delta = softplus(dl[t] + bias);
    for (i64 n = 0; n < N; ++n) {
      const double x = Delta * A[n];
      H[(t + 1) * N + n] = exp(x) * H[t * N + n] + Delta * psi(x) * Bm[n * L + t] * u[t];
    }
  }

  /* Reverse sweep.  G[n] is the adjoint of h_t (total derivative of the loss
   * sum_t dy_t * y_t with respect to h_t). */
  for (i64 n = 0; n < N; ++n) G[n] = 0.0;
  double dD = 0.0, dbias = 0.0;
  double *dA = j->dA_part + (b * dim + d) * N;
  for (i64 n = 0; n < N; ++n) dA[n] = 0.0;
  double *dBacc = j->dB_acc, *dCacc = j->dC_acc;
  double Abar_next[64];
  for (i64 n = 0; n < N; ++n) Abar_next[n] = 0.0; /* Abar_{L} unused: G_{L} = 0 */
  for (i64 t = L - 1; t >= 0; --t) {
    const double v = dl[t] + bias;
    const double Delta = softplus(v);
    double y0 = 0.0;
    for (i64 n = 0; n < N; ++n) y0 += Cm[n * L + t] * H[(t + 1) * N + n];
    if (j->D) y0 += Dd * u[t];
    double dy0 = dy[t];
    if (z) {
      const double s = sigmoid(z[t]);
      j->dz[off + t] = dy[t] * y0 * s * (1.0 + z[t] * (1.0 - s));
      dy0 = dy[t] * z[t] * s;
    }
    double du = j->D ? Dd * dy0 : 0.0;
    double dDelta = 0.0;
    if (j->D) dD += dy0 * u[t];
    for (i64 n = 0; n < N; ++n) {
      const double x = Delta * A[n];
      const double Abar = exp(x);
      const double hprev = H[t * N + n];
      /* G_t = C_t dy0_t + Abar_{t+1} G_{t+1} */
      G[n] = Cm[n * L + t] * dy0 + Abar_next[n] * G[n];
      Abar_next[n] = Abar;
      const double Bt = Bm[n * L + t];
      const double Ebar = Delta * psi(x); /* Bbar / B */
      du += G[n] * Ebar * Bt;
      /* d/dDelta of (Abar h_prev + Bbar u) = A Abar h_prev + Abar B u */
      dDelta += G[n] * Abar * (A[n] * hprev + Bt * u[t]);
      /* d/dA of (Abar h_prev + Bbar u) = Delta Abar h_prev + B u Delta^2 phi(x) */
      dA[n] += G[n] * (Delta * Abar * hprev + Bt * u[t] * Delta * Delta * phi(x));
      dBacc[(b * N + n) * L + t] += G[n] * u[t] * Ebar;
      dCacc[(b * N + n) * L + t] += dy0 * H[(t + 1) * N + n];
    }
    const double dd = dDelta * sigmoid(v);
    j->du[off + t] = du;
    j->ddelta[off + t] = dd;
    dbias += dd;
  }
  j->dD_part[b * dim + d] = dD;
  j->dbias_part[b * dim + d] = dbias;
}

static void *bwd_worker(void *arg) {
  job_t *j = (job_t *)arg;
  double *H = (double *)malloc(sizeof(double) * (size_t)((j->L + 1) * j->N));
  double *G = (double *)malloc(sizeof(double) * (size_t)j->N);
  for (i64 i = j->first; i < j->last; ++i) bwd_channel(j, i / j->dim, i % j->dim, H, G);
  free(H);
  free(G);
  return NULL;
}

/* ------------------------------------------------------------- driver */

static int run_workers(job_t *base, i64 nthreads, void *(*fn)(void *), int per_thread_acc) {
  const i64 total = base->batch * base->dim;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > total) nthreads = total > 0 ? total : 1;
  job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
  pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) { free(jobs); free(th); return -1; }
  const size_t accn = (size_t)(base->batch * base->N * base->L);
  int rc = 0;
  for (i64 k = 0; k < nthreads; ++k) {
    jobs[k] = *base;
    jobs[k].first = total * k / nthreads;
    jobs[k].last = total * (k + 1) / nthreads;
    if (per_thread_acc) {
      jobs[k].dB_acc = (double *)calloc(accn ? accn : 1, sizeof(double));
      jobs[k].dC_acc = (double *)calloc(accn ? accn : 1, sizeof(double));
      if (!jobs[k].dB_acc || !jobs[k].dC_acc) rc = -1;
    }
  }
  if (rc == 0) {
    for (i64 k = 1; k < nthreads; ++k) pthread_create(&th[k], NULL, fn, &jobs[k]);
    fn(&jobs[0]);
    for (i64 k = 1; k < nthreads; ++k) pthread_join(th[k], NULL);
  }
  if (per_thread_acc && rc == 0) {
    /* fixed-order reduction of the per-thread accumulators */
    for (size_t i = 0; i < accn; ++i) {
      double sb = 0.0, sc = 0.0;
      for (i64 k = 0; k < nthreads; ++k) { sb += jobs[k].dB_acc[i]; sc += jobs[k].dC_acc[i]; }
      base->dB_acc[i] = sb;
      base->dC_acc[i] = sc;
    }
  }
  if (per_thread_acc)
    for (i64 k = 0; k < nthreads; ++k) { free(jobs[k].dB_acc); free(jobs[k].dC_acc); }
  free(jobs);
  free(th);
  return rc;
}

/* Forward.  Layouts: u, delta, z, y: (batch, dim, L); B, C: (batch, N, L);
 * A: (dim, N); bias, D: (dim); initial_state, last_state: (batch, dim, N).
 * bias, D, z, initial_state (the state before the first step; NULL = 0) and
 * last_state may be NULL.  Returns 0 on success.  Continuing a sequence from
 * the state another call left is the recurrent (one token at a time) mode of
 * the selective SSM. */
int s6_oracle_fwd(const double *u, const double *delta, const double *bias, const double *A,
                  const double *B, const double *C, const double *D, const double *z,
                  const double *initial_state, double *y, double *last_state, i64 batch,
                  i64 dim, i64 L, i64 N, i64 nthreads) {
  if (batch < 0 || dim < 0 || L < 0 || N < 1 || N > 64) return -2;
  job_t j;
  memset(&j, 0, sizeof(j));
  j.u = u; j.delta = delta; j.bias = bias; j.A = A; j.B = B; j.C = C; j.D = D; j.z = z;
  j.h0 = initial_state;
  j.y = y; j.last_state = last_state;
  j.batch = batch; j.dim = dim; j.L = L; j.N = N;
  if (batch * dim == 0) return 0;
  return run_workers(&j, nthreads, fwd_worker, 0);
}

/* Backward of the loss sum(dy * y).  Outputs: du, ddelta, dz (batch, dim, L);
 * dB, dC (batch, N, L); dA (dim, N); dD, dbias (dim).  dz must be non-NULL iff
 * z is; dD must be non-NULL iff D is; dbias may be NULL.  Returns 0 on
 * success. */
int s6_oracle_bwd(const double *u, const double *delta, const double *bias, const double *A,
                  const double *B, const double *C, const double *D, const double *z,
                  const double *dy, double *du, double *ddelta, double *dA, double *dB,
                  double *dC, double *dD, double *dz, double *dbias, i64 batch, i64 dim, i64 L,
                  i64 N, i64 nthreads) {
  if (batch < 0 || dim < 0 || L < 0 || N < 1 || N > 64) return -2;
  if ((z == NULL) != (dz == NULL)) return -2;
  if ((D == NULL) != (dD == NULL)) return -2;
  const size_t bd = (size_t)(batch * dim);
  job_t j;
  memset(&j, 0, sizeof(j));
  j.u = u; j.delta = delta; j.bias = bias; j.A = A; j.B = B; j.C = C; j.D = D; j.z = z;
  j.dy = dy; j.du = du; j.ddelta = ddelta; j.dz = dz;
  j.batch = batch; j.dim = dim; j.L = L; j.N = N;
  j.dB_acc = dB; j.dC_acc = dC;
  memset(dB, 0, sizeof(double) * (size_t)(batch * N * L));
  memset(dC, 0, sizeof(double) * (size_t)(batch * N * L));
  memset(dA, 0, sizeof(double) * (size_t)(dim * N));
  if (dD) memset(dD, 0, sizeof(double) * (size_t)dim);
  if (dbias) memset(dbias, 0, sizeof(double) * (size_t)dim);
  if (bd == 0) return 0;
  j.dA_part = (double *)calloc(bd * (size_t)N, sizeof(double));
  j.dD_part = (double *)calloc(bd, sizeof(double));
  j.dbias_part = (double *)calloc(bd, sizeof(double));
  int rc = -1;
  if (j.dA_part && j.dD_part && j.dbias_part) {
    rc = run_workers(&j, nthreads, bwd_worker, 1);
    if (rc == 0) {
      /* parameters are shared over the batch: sum the per-(b,d) partials in b order */
      for (i64 b = 0; b < batch; ++b)
        for (i64 d = 0; d < dim; ++d) {
          for (i64 n = 0; n < N; ++n) dA[d * N + n] += j.dA_part[(b * dim + d) * N + n];
          if (dD) dD[d] += j.dD_part[b * dim + d];
          if (dbias) dbias[d] += j.dbias_part[b * dim + d];
        }
    }
  }
  free(j.dA_part);
  free(j.dD_part);
  free(j.dbias_part);
  return rc;
}

/* ------------------------------------------------ convolution prologue */

/* pre and u = SiLU(pre) of the causal depthwise convolution (see the header). */
static void conv_silu(const double *x, const double *w, const double *cb, i64 W, double *pre,
                      double *u, i64 batch, i64 dim, i64 L) {
  for (i64 b = 0; b < batch; ++b)
    for (i64 d = 0; d < dim; ++d) {
      const i64 off = (b * dim + d) * L;
      for (i64 t = 0; t < L; ++t) {
        double p = cb ? cb[d] : 0.0;
        for (i64 k = 0; k < W; ++k) {
          const i64 s = t - (W - 1) + k; /* the input step weight k looks at */
          if (s >= 0) p += w[d * W + k] * x[off + s];
        }
        pre[off + t] = p;
        u[off + t] = p * sigmoid(p);
      }
    }
}

/* The convolution prologue alone: u (and pre if non-NULL) from x.  Layouts:
 * x, pre, u (batch, dim, L); conv_w (dim, W); conv_b (dim) or NULL. */
int s6_oracle_conv_silu(const double *x, const double *conv_w, const double *conv_b, i64 W,
                        double *pre, double *u, i64 batch, i64 dim, i64 L) {
  if (batch < 0 || dim < 0 || L < 0 || W < 1 || W > 64) return -2;
  const size_t n = (size_t)(batch * dim * L);
  double *p = pre ? pre : (double *)malloc(sizeof(double) * (n ? n : 1));
  if (!p) return -1;
  conv_silu(x, conv_w, conv_b, W, p, u, batch, dim, L);
  if (!pre) free(p);
  return 0;
}

/* Forward with the prologue: u = SiLU(causal depthwise conv of x), then the
 * S6 forward of s6_oracle_fwd (h = 0 before the first step). */
int s6_oracle_conv_fwd(const double *x, const double *conv_w, const double *conv_b, i64 W,
                       const double *delta, const double *bias, const double *A, const double *B,
                       const double *C, const double *D, const double *z, double *y,
                       double *last_state, i64 batch, i64 dim, i64 L, i64 N, i64 nthreads) {
  if (batch < 0 || dim < 0 || L < 0 || W < 1 || W > 64) return -2;
  const size_t n = (size_t)(batch * dim * L);
  double *pre = (double *)malloc(sizeof(double) * (n ? n : 1));
  double *u = (double *)malloc(sizeof(double) * (n ? n : 1));
  int rc = -1;
  if (pre && u) {
    conv_silu(x, conv_w, conv_b, W, pre, u, batch, dim, L);
    rc = s6_oracle_fwd(u, delta, bias, A, B, C, D, z, NULL, y, last_state, batch, dim, L, N,
                       nthreads);
  }
  free(pre);
  free(u);
  return rc;
}

/* Backward of sum(dy * y) for the forward with the prologue.  Outputs as in
 * s6_oracle_bwd, with dx (batch, dim, L) in place of du, plus dconv_w (dim, W)
 * and dconv_b (dim; may be NULL).  The S6 backward gives du at u = SiLU(pre);
 * then
 *     dpre_t = du_t * sigmoid(pre_t) * (1 + pre_t * (1 - sigmoid(pre_t)))
 * and each term conv_w[d,k] * x[s], s = t-(W-1)+k, of pre_t passes dpre_t on:
 *     dx[s] += conv_w[d,k] * dpre_t,  dconv_w[d,k] += dpre_t * x[s],
 *     dconv_b[d] += dpre_t. */
int s6_oracle_conv_bwd(const double *x, const double *conv_w, const double *conv_b, i64 W,
                       const double *delta, const double *bias, const double *A, const double *B,
                       const double *C, const double *D, const double *z, const double *dy,
                       double *dx, double *dconv_w, double *dconv_b, double *ddelta, double *dA,
                       double *dB, double *dC, double *dD, double *dz, double *dbias, i64 batch,
                       i64 dim, i64 L, i64 N, i64 nthreads) {
  if (batch < 0 || dim < 0 || L < 0 || W < 1 || W > 64) return -2;
  const size_t n = (size_t)(batch * dim * L);
  double *pre = (double *)malloc(sizeof(double) * (n ? n : 1));
  double *u = (double *)malloc(sizeof(double) * (n ? n : 1));
  double *du = (double *)malloc(sizeof(double) * (n ? n : 1));
  int rc = -1;
  if (pre && u && du) {
    conv_silu(x, conv_w, conv_b, W, pre, u, batch, dim, L);
    rc = s6_oracle_bwd(u, delta, bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz, dbias,
                       batch, dim, L, N, nthreads);
  }
  if (rc == 0) {
    memset(dx, 0, sizeof(double) * n);
    memset(dconv_w, 0, sizeof(double) * (size_t)(dim * W));
    if (dconv_b) memset(dconv_b, 0, sizeof(double) * (size_t)dim);
    for (i64 b = 0; b < batch; ++b)
      for (i64 d = 0; d < dim; ++d) {
        const i64 off = (b * dim + d) * L;
        for (i64 t = 0; t < L; ++t) {
          const double s = sigmoid(pre[off + t]);
          const double dpre = du[off + t] * s * (1.0 + pre[off + t] * (1.0 - s));
          for (i64 k = 0; k < W; ++k) {
            const i64 src = t - (W - 1) + k;
            if (src < 0) continue;
            dx[off + src] += conv_w[d * W + k] * dpre;
            dconv_w[d * W + k] += dpre * x[off + src];
          }
          if (dconv_b) dconv_b[d] += dpre;
        }
      }
  }
  free(pre);
  free(u);
  free(du);
  return rc;
}

/* -------------------------------------------- low-rank Delta projection */

/* delta = W_dt . dt_low per batch row (see the header). */
static void dt_project(const double *dt_low, const double *W, i64 R, double *delta, i64 batch,
                       i64 dim, i64 L) {
  for (i64 b = 0; b < batch; ++b)
    for (i64 d = 0; d < dim; ++d)
      for (i64 t = 0; t < L; ++t) {
        double s = 0.0;
        for (i64 r = 0; r < R; ++r) s += W[d * R + r] * dt_low[(b * R + r) * L + t];
        delta[(b * dim + d) * L + t] = s;
      }
}

/* Forward with the low-rank Delta projection: delta = W_dt . dt_low, then
 * the S6 forward of s6_oracle_fwd.  Layouts: dt_low (batch, R, L); W_dt
 * (dim, R); the rest as s6_oracle_fwd. */
int s6_oracle_dtproj_fwd(const double *u, const double *dt_low, const double *W_dt, i64 R,
                         const double *bias, const double *A, const double *B, const double *C,
                         const double *D, const double *z, double *y, double *last_state,
                         i64 batch, i64 dim, i64 L, i64 N, i64 nthreads) {
  if (batch < 0 || dim < 0 || L < 0 || R < 1) return -2;
  const size_t n = (size_t)(batch * dim * L);
  double *delta = (double *)malloc(sizeof(double) * (n ? n : 1));
  if (!delta) return -1;
  dt_project(dt_low, W_dt, R, delta, batch, dim, L);
  const int rc = s6_oracle_fwd(u, delta, bias, A, B, C, D, z, NULL, y, last_state, batch, dim, L,
                               N, nthreads);
  free(delta);
  return rc;
}

/* Backward of sum(dy * y) for the forward with the projection.  Outputs as
 * in s6_oracle_bwd, with d_dt_low (batch, R, L) and dW_dt (dim, R) in place
 * of ddelta.  With ddelta from the S6 backward, every term
 * W_dt[d,r] * dt_low[b,r,t] of delta[b,d,t] passes ddelta[b,d,t] on:
 *     d_dt_low[b,r,t] += W_dt[d,r] * ddelta[b,d,t],
 *     dW_dt[d,r]      += ddelta[b,d,t] * dt_low[b,r,t]. */
int s6_oracle_dtproj_bwd(const double *u, const double *dt_low, const double *W_dt, i64 R,
                         const double *bias, const double *A, const double *B, const double *C,
                         const double *D, const double *z, const double *dy, double *du,
                         double *d_dt_low, double *dW_dt, double *dA, double *dB, double *dC,
                         double *dD, double *dz, double *dbias, i64 batch, i64 dim, i64 L, i64 N,
                         i64 nthreads) {
  if (batch < 0 || dim < 0 || L < 0 || R < 1) return -2;
  const size_t n = (size_t)(batch * dim * L);
  double *delta = (double *)malloc(sizeof(double) * (n ? n : 1));
  double *ddelta = (double *)malloc(sizeof(double) * (n ? n : 1));
  int rc = -1;
  if (delta && ddelta) {
    dt_project(dt_low, W_dt, R, delta, batch, dim, L);
    rc = s6_oracle_bwd(u, delta, bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz, dbias,
                       batch, dim, L, N, nthreads);
  }
  if (rc == 0) {
    memset(d_dt_low, 0, sizeof(double) * (size_t)(batch * R * L));
    memset(dW_dt, 0, sizeof(double) * (size_t)(dim * R));
    for (i64 b = 0; b < batch; ++b)
      for (i64 d = 0; d < dim; ++d)
        for (i64 t = 0; t < L; ++t) {
          const double g = ddelta[(b * dim + d) * L + t];
          for (i64 r = 0; r < R; ++r) {
            d_dt_low[(b * R + r) * L + t] += W_dt[d * R + r] * g;
            dW_dt[d * R + r] += g * dt_low[(b * R + r) * L + t];
          }
        }
  }
  free(delta);
  free(ddelta);
  return rc;
}

/* ------------------------------------------------ complex diagonal A */

typedef double complex cplx;

/* psi(x) = (exp(x) - 1) / x for complex x; its series near 0. */
static cplx cpsi(cplx x) {
  if (cabs(x) < 1e-3) return 1.0 + x * (0.5 + x * (1.0 / 6.0 + x * (1.0 / 24.0 + x / 120.0)));
  return (cexp(x) - 1.0) / x;
}

/* phi(x) = d psi / dx = (x e^x - (e^x - 1)) / x^2; its series near 0. */
static cplx cphi(cplx x) {
  if (cabs(x) < 1e-2)
    return 0.5 + x * (1.0 / 3.0 + x * (1.0 / 8.0 + x * (1.0 / 30.0 + x * (1.0 / 144.0))));
  return (x * cexp(x) - (cexp(x) - 1.0)) / (x * x);
}

/* element n of a planar complex row of N entries (stride between entries) */
static cplx cget(const double *p, i64 n, i64 N, i64 stride) {
  return p[n * stride] + I * p[(n + N) * stride];
}

typedef struct {
  const double *u, *delta, *bias, *A, *B, *C, *D, *z, *dy;
  double *y, *last_state, *du, *ddelta, *dz;
  double *dA_part, *dD_part, *dbias_part, *dB_acc, *dC_acc;
  i64 batch, dim, L, N, first, last;
} cjob_t;

static void cfwd_channel(const cjob_t *j, i64 b, i64 d, cplx *h) {
  const i64 L = j->L, N = j->N, dim = j->dim;
  const i64 off = (b * dim + d) * L;
  const double *Bm = j->B + b * 2 * N * L, *Cm = j->C + b * 2 * N * L;
  const double bias = j->bias ? j->bias[d] : 0.0;
  for (i64 n = 0; n < N; ++n) h[n] = 0.0;
  for (i64 t = 0; t < L; ++t) {
    const double Delta = softplus(j->delta[off + t] + bias);
    double y0 = 0.0;
    for (i64 n = 0; n < N; ++n) {
      const cplx An = cget(j->A + d * 2 * N, n, N, 1);
      const cplx x = Delta * An;
      const cplx Bbar = Delta * cpsi(x) * cget(Bm + t, n, N, L);
      h[n] = cexp(x) * h[n] + Bbar * j->u[off + t];
      y0 += creal(cget(Cm + t, n, N, L) * h[n]);
    }
    if (j->D) y0 += j->D[d] * j->u[off + t];
    if (j->z) y0 *= j->z[off + t] * sigmoid(j->z[off + t]);
    j->y[off + t] = y0;
  }
  if (j->last_state) {
    double *ls = j->last_state + (b * dim + d) * 2 * N;
    for (i64 n = 0; n < N; ++n) {
      ls[n] = creal(h[n]);
      ls[N + n] = cimag(h[n]);
    }
  }
}

static void *cfwd_worker(void *arg) {
  cjob_t *j = (cjob_t *)arg;
  cplx *h = (cplx *)malloc(sizeof(cplx) * (size_t)j->N);
  for (i64 i = j->first; i < j->last; ++i) cfwd_channel(j, i / j->dim, i % j->dim, h);
  free(h);
  return NULL;
}

/* The adjoint of the complex forward, for the real loss sum(dy * y).  The
 * gradient of a complex w is g = dl/d(re w) + i dl/d(im w); through a
 * product v = a w it is conj(a) g_v, and through y = Re(c h) it is
 * conj(c) dy.  So G_t = conj(C_t) dy0_t + conj(Abar_{t+1}) G_{t+1}, and with
 * dh_t/dDelta = Abar (A h_{t-1} + B u), dh_t/dA = Delta Abar h_{t-1} +
 * Delta^2 phi(x) B u:
 *     du     += Re(conj(G) Bbar),        dDelta += Re(conj(G) dh/dDelta),
 *     g_A    += conj(dh/dA) G,           g_B    += conj(Delta psi(x)) u G,
 *     g_C    += conj(h_t) dy0. */
static void cbwd_channel(cjob_t *j, i64 b, i64 d, cplx *H, cplx *G, cplx *Anext, cplx *gA) {
  const i64 L = j->L, N = j->N, dim = j->dim;
  const i64 off = (b * dim + d) * L;
  const double *Bm = j->B + b * 2 * N * L, *Cm = j->C + b * 2 * N * L;
  const double bias = j->bias ? j->bias[d] : 0.0;
  const double Dd = j->D ? j->D[d] : 0.0;
  for (i64 n = 0; n < N; ++n) H[n] = 0.0;
  for (i64 t = 0; t < L; ++t) {
    const double Delta = softplus(j->delta[off + t] + bias);
    for (i64 n = 0; n < N; ++n) {
      const cplx x = Delta * cget(j->A + d * 2 * N, n, N, 1);
      H[(t + 1) * N + n] = cexp(x) * H[t * N + n] +
                           Delta * cpsi(x) * cget(Bm + t, n, N, L) * j->u[off + t];
    }
  }
  for (i64 n = 0; n < N; ++n) {
    G[n] = 0.0;
    Anext[n] = 0.0;
    gA[n] = 0.0;
  }
  double dD = 0.0, dbias = 0.0;
  for (i64 t = L - 1; t >= 0; --t) {
    const double v = j->delta[off + t] + bias;
    const double Delta = softplus(v);
    const double ut = j->u[off + t];
    double y0 = 0.0;
    for (i64 n = 0; n < N; ++n) y0 += creal(cget(Cm + t, n, N, L) * H[(t + 1) * N + n]);
    if (j->D) y0 += Dd * ut;
    double dy0 = j->dy[off + t];
    if (j->z) {
      const double zt = j->z[off + t], sz = sigmoid(zt);
      j->dz[off + t] = j->dy[off + t] * y0 * sz * (1.0 + zt * (1.0 - sz));
      dy0 = j->dy[off + t] * zt * sz;
    }
    double du = j->D ? Dd * dy0 : 0.0, dDelta = 0.0;
    if (j->D) dD += dy0 * ut;
    for (i64 n = 0; n < N; ++n) {
      const cplx An = cget(j->A + d * 2 * N, n, N, 1);
      const cplx x = Delta * An;
      const cplx Abar = cexp(x);
      const cplx Bn = cget(Bm + t, n, N, L), Cn = cget(Cm + t, n, N, L);
      const cplx hprev = H[t * N + n], hcur = H[(t + 1) * N + n];
      G[n] = conj(Cn) * dy0 + conj(Anext[n]) * G[n];
      Anext[n] = Abar;
      const cplx E = Delta * cpsi(x); /* Bbar / B */
      du += creal(conj(G[n]) * E * Bn);
      dDelta += creal(conj(G[n]) * Abar * (An * hprev + Bn * ut));
      gA[n] += conj(Delta * Abar * hprev + Delta * Delta * cphi(x) * Bn * ut) * G[n];
      const cplx gB = conj(E) * ut * G[n];
      const cplx gC = conj(hcur) * dy0;
      j->dB_acc[(b * 2 * N + n) * L + t] += creal(gB);
      j->dB_acc[(b * 2 * N + N + n) * L + t] += cimag(gB);
      j->dC_acc[(b * 2 * N + n) * L + t] += creal(gC);
      j->dC_acc[(b * 2 * N + N + n) * L + t] += cimag(gC);
    }
    const double dd = dDelta * sigmoid(v);
    j->du[off + t] = du;
    j->ddelta[off + t] = dd;
    dbias += dd;
  }
  double *pa = j->dA_part + (b * dim + d) * 2 * N;
  for (i64 n = 0; n < N; ++n) {
    pa[n] = creal(gA[n]);
    pa[N + n] = cimag(gA[n]);
  }
  j->dD_part[b * dim + d] = dD;
  j->dbias_part[b * dim + d] = dbias;
}

static void *cbwd_worker(void *arg) {
  cjob_t *j = (cjob_t *)arg;
  const size_t N = (size_t)j->N;
  cplx *H = (cplx *)malloc(sizeof(cplx) * (size_t)(j->L + 1) * N);
  cplx *G = (cplx *)malloc(sizeof(cplx) * 3 * N);
  for (i64 i = j->first; i < j->last; ++i) cbwd_channel(j, i / j->dim, i % j->dim, H, G, G + N, G + 2 * N);
  free(H);
  free(G);
  return NULL;
}

static int run_cworkers(cjob_t *base, i64 nthreads, void *(*fn)(void *), int acc) {
  const i64 total = base->batch * base->dim;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > total) nthreads = total > 0 ? total : 1;
  cjob_t *jobs = (cjob_t *)calloc((size_t)nthreads, sizeof(cjob_t));
  pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) { free(jobs); free(th); return -1; }
  const size_t accn = (size_t)(base->batch * 2 * base->N * base->L);
  int rc = 0;
  for (i64 k = 0; k < nthreads; ++k) {
    jobs[k] = *base;
    jobs[k].first = total * k / nthreads;
    jobs[k].last = total * (k + 1) / nthreads;
    if (acc) {
      jobs[k].dB_acc = (double *)calloc(accn ? accn : 1, sizeof(double));
      jobs[k].dC_acc = (double *)calloc(accn ? accn : 1, sizeof(double));
      if (!jobs[k].dB_acc || !jobs[k].dC_acc) rc = -1;
    }
  }
  if (rc == 0) {
    for (i64 k = 1; k < nthreads; ++k) pthread_create(&th[k], NULL, fn, &jobs[k]);
    fn(&jobs[0]);
    for (i64 k = 1; k < nthreads; ++k) pthread_join(th[k], NULL);
  }
  if (acc && rc == 0) {
    for (size_t i = 0; i < accn; ++i) {
      double sb = 0.0, sc = 0.0;
      for (i64 k = 0; k < nthreads; ++k) { sb += jobs[k].dB_acc[i]; sc += jobs[k].dC_acc[i]; }
      base->dB_acc[i] = sb;
      base->dC_acc[i] = sc;
    }
  }
  if (acc)
    for (i64 k = 0; k < nthreads; ++k) { free(jobs[k].dB_acc); free(jobs[k].dC_acc); }
  free(jobs);
  free(th);
  return rc;
}

/* Complex forward.  Layouts: u, delta, z, y (batch, dim, L); A (dim, 2N);
 * B, C (batch, 2N, L); bias, D (dim); last_state (batch, dim, 2N); complex
 * vectors planar (real parts first).  bias, D, z, last_state may be NULL. */
int s6_oracle_cplx_fwd(const double *u, const double *delta, const double *bias, const double *A,
                       const double *B, const double *C, const double *D, const double *z,
                       double *y, double *last_state, i64 batch, i64 dim, i64 L, i64 N,
                       i64 nthreads) {
  if (batch < 0 || dim < 0 || L < 0 || N < 1 || N > 64) return -2;
  cjob_t j;
  memset(&j, 0, sizeof(j));
  j.u = u; j.delta = delta; j.bias = bias; j.A = A; j.B = B; j.C = C; j.D = D; j.z = z;
  j.y = y; j.last_state = last_state;
  j.batch = batch; j.dim = dim; j.L = L; j.N = N;
  if (batch * dim == 0) return 0;
  return run_cworkers(&j, nthreads, cfwd_worker, 0);
}

/* Complex backward of sum(dy * y).  Outputs du, ddelta, dz (batch, dim, L);
 * dA (dim, 2N); dB, dC (batch, 2N, L); dD, dbias (dim).  dz non-NULL iff z,
 * dD iff D; dbias may be NULL. */
int s6_oracle_cplx_bwd(const double *u, const double *delta, const double *bias, const double *A,
                       const double *B, const double *C, const double *D, const double *z,
                       const double *dy, double *du, double *ddelta, double *dA, double *dB,
                       double *dC, double *dD, double *dz, double *dbias, i64 batch, i64 dim,
                       i64 L, i64 N, i64 nthreads) {
  if (batch < 0 || dim < 0 || L < 0 || N < 1 || N > 64) return -2;
  if ((z == NULL) != (dz == NULL) || (D == NULL) != (dD == NULL)) return -2;
  const size_t bd = (size_t)(batch * dim);
  cjob_t j;
  memset(&j, 0, sizeof(j));
  j.u = u; j.delta = delta; j.bias = bias; j.A = A; j.B = B; j.C = C; j.D = D; j.z = z;
  j.dy = dy; j.du = du; j.ddelta = ddelta; j.dz = dz;
  j.batch = batch; j.dim = dim; j.L = L; j.N = N;
  j.dB_acc = dB; j.dC_acc = dC;
  memset(dB, 0, sizeof(double) * (size_t)(batch * 2 * N * L));
  memset(dC, 0, sizeof(double) * (size_t)(batch * 2 * N * L));
  memset(dA, 0, sizeof(double) * (size_t)(dim * 2 * N));
  if (dD) memset(dD, 0, sizeof(double) * (size_t)dim);
  if (dbias) memset(dbias, 0, sizeof(double) * (size_t)dim);
  if (bd == 0) return 0;
  j.dA_part = (double *)calloc(bd * 2 * (size_t)N, sizeof(double));
  j.dD_part = (double *)calloc(bd, sizeof(double));
  j.dbias_part = (double *)calloc(bd, sizeof(double));
  int rc = -1;
  if (j.dA_part && j.dD_part && j.dbias_part) {
    rc = run_cworkers(&j, nthreads, cbwd_worker, 1);
    if (rc == 0) {
      for (i64 b = 0; b < batch; ++b)
        for (i64 d = 0; d < dim; ++d) {
          for (i64 n = 0; n < 2 * N; ++n) dA[d * 2 * N + n] += j.dA_part[(b * dim + d) * 2 * N + n];
          if (dD) dD[d] += j.dD_part[b * dim + d];
          if (dbias) dbias[d] += j.dbias_part[b * dim + d];
        }
    }
  }
  free(j.dA_part);
  free(j.dD_part);
  free(j.dbias_part);
  return rc;
}
