/*
 * Plain fp64 CPU oracle for the ParaRNN / DEER Newton solve of diagonal and
 * 2x2 block-diagonal nonlinear recurrences.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA library; neither includes the other.
 *
 * Sources (page title, then the passage):
 *  - "ParaRNN: Unlocking Parallel Training of Nonlinear RNNs for Large Language
 *    Models" (sciencestack 2510.21450), TL;DR and Abstract: the sequence of
 *    recurrence relations is one system of equations, solved with Newton's
 *    iterations plus a parallel reduction of the block bi-diagonal system;
 *    GRU and LSTM cells adapted to have diagonal / 2x2 block-diagonal Jacobians
 *    (Figure 2 caption).  Figure 4 caption: the residual reported is the max
 *    over the batch.
 *  - DEER summary (agihunt, "Recasting nonlinear recurrences as quadratically
 *    convergent fixed-point iterations..."): the converged iteration reproduces
 *    sequential evaluation; tolerance 1e-4 suffices in float32; Newton started
 *    far from the solution may diverge (no damping is applied here).
 *  - The pages print no cell equations.  The ParaGRU cell used throughout is
 *      z = sig(Pz + az*h), r = sig(Pr + ar*h), c = tanh(Pc + ac*(r*h)),
 *      h' = (1-z)*h + z*c,
 *    i.e. a GRU whose recurrence weights are diagonal (per channel), which is
 *    what makes its Jacobian diagonal (ParaRNN, Figure 2 caption).
 *  - The LSTM cell is read as the standard LSTM with a diagonal recurrence on h
 *    only (no peepholes), biases folded into the projected inputs, gate order
 *    (i, f, g, o), state order (c, h):
 *      i = sig(Pi + ai*h), f = sig(Pf + af*h), g = tanh(Pg + ag*h),
 *      o = sig(Po + ao*h), c' = f*c + i*g, h' = o*tanh(c').
 *
 * Layouts (C order): projected inputs P[B][L][G][D]; recurrence weights a[G][D];
 * trajectories h[B][L][D] for t = 1..L (h0 is not repeated); diagonal scan
 * A, b [B][L][D]; block scan A[B][L][D][2][2] (row-major), b and x [B][L][D][2].
 *
 * Everything here is a straight transcription of the definitions: no blocking,
 * no reassociation.  Threads (pthreads) split only the independent channels
 * (b, d); every channel's arithmetic runs in the order written.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define IDX3(b, t, d, L, D) ((((size_t)(b)) * (size_t)(L) + (size_t)(t)) * (size_t)(D) + (size_t)(d))
#define IDXP(b, t, g, d, L, G, D) \
  (((((size_t)(b)) * (size_t)(L) + (size_t)(t)) * (size_t)(G) + (size_t)(g)) * (size_t)(D) + (size_t)(d))

static double sig(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ------------------------------------------------------------------------- */
/* Channel-parallel driver: contiguous ranges of channels per thread.         */
/* ------------------------------------------------------------------------- */
static int g_threads = 0; /* 0 = all CPUs in this process's affinity mask */

void oracle_set_threads(int n) { g_threads = n; }

int oracle_get_threads(void) {
  if (g_threads > 0) return g_threads;
  cpu_set_t set;
  if (sched_getaffinity(0, sizeof(set), &set) == 0) {
    int n = CPU_COUNT(&set);
    if (n > 0) return n;
  }
  return 1;
}

typedef void (*chan_body)(void* ctx, int64_t ch);
typedef struct {
  chan_body body;
  void* ctx;
  int64_t lo, hi;
} range_job;

static void* range_worker(void* p) {
  range_job* j = (range_job*)p;
  for (int64_t c = j->lo; c < j->hi; ++c) j->body(j->ctx, c);
  return NULL;
}

static void for_channels(int64_t nchan, chan_body body, void* ctx) {
  int nt = oracle_get_threads();
  if (nt > 256) nt = 256;
  if ((int64_t)nt > nchan) nt = (int)(nchan > 0 ? nchan : 1);
  if (nt <= 1) {
    for (int64_t c = 0; c < nchan; ++c) body(ctx, c);
    return;
  }
  pthread_t th[256];
  range_job jobs[256];
  int started[256];
  for (int i = 0; i < nt; ++i) {
    jobs[i].body = body;
    jobs[i].ctx = ctx;
    jobs[i].lo = nchan * i / nt;
    jobs[i].hi = nchan * (i + 1) / nt;
    started[i] = pthread_create(&th[i], NULL, range_worker, &jobs[i]) == 0;
    if (!started[i]) range_worker(&jobs[i]);
  }
  for (int i = 0; i < nt; ++i)
    if (started[i]) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------------------- */
/* Linear recurrences (the block bi-diagonal system, solved sequentially).    */
/* ------------------------------------------------------------------------- */

typedef struct {
  const double *A, *b, *x0;
  double* x;
  int64_t L, D;
} scan_ctx;

static void scan_diag_chan(void* p, int64_t ch) {
  scan_ctx* c = (scan_ctx*)p;
  int64_t bb = ch / c->D, d = ch % c->D;
  double x = c->x0 ? c->x0[bb * c->D + d] : 0.0;
  for (int64_t t = 0; t < c->L; ++t) {
    size_t i = IDX3(bb, t, d, c->L, c->D);
    x = c->A[i] * x + c->b[i];
    c->x[i] = x;
  }
}

/* h_t = A_t * h_{t-1} + b_t, t = 1..L, starting from h0 (NULL means 0). */
void oracle_scan_diag(const double* A, const double* b, const double* h0, double* h,
                      int64_t B, int64_t L, int64_t D) {
  scan_ctx c = {A, b, h0, h, L, D};
  for_channels(B * D, scan_diag_chan, &c);
}

static void scan_block2_chan(void* p, int64_t ch) {
  scan_ctx* c = (scan_ctx*)p;
  int64_t bb = ch / c->D, d = ch % c->D;
  double u0 = c->x0 ? c->x0[(bb * c->D + d) * 2 + 0] : 0.0;
  double u1 = c->x0 ? c->x0[(bb * c->D + d) * 2 + 1] : 0.0;
  for (int64_t t = 0; t < c->L; ++t) {
    size_t i = IDX3(bb, t, d, c->L, c->D);
    const double* M = c->A + 4 * i;
    double n0 = M[0] * u0 + M[1] * u1 + c->b[2 * i + 0];
    double n1 = M[2] * u0 + M[3] * u1 + c->b[2 * i + 1];
    u0 = n0;
    u1 = n1;
    c->x[2 * i + 0] = u0;
    c->x[2 * i + 1] = u1;
  }
}

/* x_t = A_t x_{t-1} + b_t with 2x2 A_t (row-major) and 2-vectors; x0 NULL = 0. */
void oracle_scan_block2(const double* A, const double* b, const double* x0, double* x,
                        int64_t B, int64_t L, int64_t D) {
  scan_ctx c = {A, b, x0, x, L, D};
  for_channels(B * D, scan_block2_chan, &c);
}

/* ------------------------------------------------------------------------- */
/* Cells and their Jacobians with respect to the previous state.              */
/* ------------------------------------------------------------------------- */

/* ParaGRU step.  p = (Pz, Pr, Pc), w = (az, ar, ac).  Returns h' in *f and
 * dh'/dh in *J.  Derivative by the chain rule:
 *   dz/dh = z(1-z) az, dr/dh = r(1-r) ar,
 *   du/dh = ac (r + h dr/dh), dc/dh = (1-c^2) du/dh,
 *   dh'/dh = (1-z) - h dz/dh + c dz/dh + z dc/dh. */
void oracle_gru_cell(const double* p, const double* w, double h, double* f, double* J) {
  double z = sig(p[0] + w[0] * h);
  double r = sig(p[1] + w[1] * h);
  double u = p[2] + w[2] * (r * h);
  double c = tanh(u);
  *f = (1.0 - z) * h + z * c;
  if (J) {
    double dz = z * (1.0 - z) * w[0];
    double dr = r * (1.0 - r) * w[1];
    double du = w[2] * (r + h * dr);
    double dc = (1.0 - c * c) * du;
    *J = (1.0 - z) - h * dz + c * dz + z * dc;
  }
}

/* ParaLSTM step with state (c, h).  p = (Pi, Pf, Pg, Po), w = (ai, af, ag, ao).
 * J is d(c', h')/d(c, h), row-major:
 *   [[dc'/dc, dc'/dh], [dh'/dc, dh'/dh]]. */
void oracle_lstm_cell(const double* p, const double* w, double c, double h,
                      double* fc, double* fh, double* J) {
  double i = sig(p[0] + w[0] * h);
  double f = sig(p[1] + w[1] * h);
  double g = tanh(p[2] + w[2] * h);
  double o = sig(p[3] + w[3] * h);
  double cn = f * c + i * g;
  double tc = tanh(cn);
  *fc = cn;
  *fh = o * tc;
  if (J) {
    double di = i * (1.0 - i) * w[0];
    double df = f * (1.0 - f) * w[1];
    double dg = (1.0 - g * g) * w[2];
    double dov = o * (1.0 - o) * w[3];
    double dcn_dc = f;
    double dcn_dh = df * c + di * g + i * dg;
    double dtc = 1.0 - tc * tc;
    J[0] = dcn_dc;
    J[1] = dcn_dh;
    J[2] = o * dtc * dcn_dc;
    J[3] = dov * tc + o * dtc * dcn_dh;
  }
}

/* ------------------------------------------------------------------------- */
/* Sequential rollout: the plain definition of the result.                   */
/* ------------------------------------------------------------------------- */

typedef struct {
  const double *P, *a, *c0, *h0;
  double *c, *h;
  int64_t L, D;
} roll_ctx;

static void rollout_gru_chan(void* p, int64_t ch) {
  roll_ctx* x = (roll_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double w[3] = {x->a[0 * D + d], x->a[1 * D + d], x->a[2 * D + d]};
  double s = x->h0 ? x->h0[bb * D + d] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    double pg[3];
    for (int g = 0; g < 3; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 3, D)];
    double f;
    oracle_gru_cell(pg, w, s, &f, NULL);
    s = f;
    x->h[IDX3(bb, t, d, L, D)] = s;
  }
}

void oracle_rollout_gru(const double* P, const double* a, const double* h0, double* h,
                        int64_t B, int64_t L, int64_t D) {
  roll_ctx x = {P, a, NULL, h0, NULL, h, L, D};
  for_channels(B * D, rollout_gru_chan, &x);
}

static void rollout_lstm_chan(void* p, int64_t ch) {
  roll_ctx* x = (roll_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double w[4] = {x->a[0 * D + d], x->a[1 * D + d], x->a[2 * D + d], x->a[3 * D + d]};
  double sc = x->c0 ? x->c0[bb * D + d] : 0.0;
  double sh = x->h0 ? x->h0[bb * D + d] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    double pg[4];
    for (int g = 0; g < 4; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 4, D)];
    double fc, fh;
    oracle_lstm_cell(pg, w, sc, sh, &fc, &fh, NULL);
    sc = fc;
    sh = fh;
    x->c[IDX3(bb, t, d, L, D)] = sc;
    x->h[IDX3(bb, t, d, L, D)] = sh;
  }
}

void oracle_rollout_lstm(const double* P, const double* a, const double* c0, const double* h0,
                         double* c, double* h, int64_t B, int64_t L, int64_t D) {
  roll_ctx x = {P, a, c0, h0, c, h, L, D};
  for_channels(B * D, rollout_lstm_chan, &x);
}

/* ------------------------------------------------------------------------- */
/* Serial Newton on the stacked system F_t(h) = h_t - f(h_{t-1}, P_t) = 0.    */
/* ------------------------------------------------------------------------- */
/*
 * Iterate k = 0, 1, ... from h^0 = 0 (t = 1..L; h_0 = h0 is fixed):
 *   r_t   = f(h^k_{t-1}, P_t) - h^k_t                (minus the residual of F)
 *   rho_k = max over every (b, t, d [, component]) of |r_t|
 *   stop with iterations = k if rho_k <= tol; stop unconverged if k == max_iters
 *   A_t   = df/dh at h^k_{t-1}
 *   delta_t = A_t delta_{t-1} + r_t, delta_0 = 0      (the linear solve)
 *   h^{k+1} = h^k + delta
 * rho_hist receives rho_0..rho_k (max_iters + 1 slots).  chan_iters, if not
 * NULL, receives per channel the first k at which that channel's own max
 * residual was <= tol (or -1 if never within the iterations run).
 * Returns the iteration count; *converged is 1 if rho_k <= tol was reached.
 * A non-finite residual stops the iteration (converged = 0, *nonfinite = 1).
 */
typedef struct {
  const double *P, *a, *c0, *h0;
  double *c, *h, *Jt, *rt, *cmax;
  int64_t L, D;
} newton_ctx;

static void newton_gru_residual_chan(void* p, int64_t ch) {
  newton_ctx* x = (newton_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double w[3] = {x->a[0 * D + d], x->a[1 * D + d], x->a[2 * D + d]};
  double m = 0.0;
  for (int64_t t = 0; t < L; ++t) {
    double hp = (t == 0) ? (x->h0 ? x->h0[bb * D + d] : 0.0) : x->h[IDX3(bb, t - 1, d, L, D)];
    double pg[3];
    for (int g = 0; g < 3; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 3, D)];
    double f, J;
    oracle_gru_cell(pg, w, hp, &f, &J);
    size_t i = IDX3(bb, t, d, L, D);
    x->rt[i] = f - x->h[i];
    x->Jt[i] = J;
    double ar = fabs(x->rt[i]);
    if (!(ar <= m)) m = ar; /* keeps a NaN */
  }
  x->cmax[ch] = m;
}

static void newton_gru_solve_chan(void* p, int64_t ch) {
  newton_ctx* x = (newton_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double delta = 0.0;
  for (int64_t t = 0; t < L; ++t) {
    size_t i = IDX3(bb, t, d, L, D);
    delta = x->Jt[i] * delta + x->rt[i];
    x->h[i] += delta;
  }
}

/* max over channels (NaN wins); records first-within-tol iteration per channel */
static double reduce_rho(const double* cmax, int64_t n, double tol, int k, int32_t* chan_iters) {
  double rho = 0.0;
  for (int64_t c = 0; c < n; ++c) {
    if (!(cmax[c] <= rho)) rho = cmax[c];
    if (chan_iters && chan_iters[c] < 0 && cmax[c] <= tol) chan_iters[c] = k;
  }
  return rho;
}

int oracle_newton_gru(const double* P, const double* a, const double* h0, double tol,
                      int max_iters, int64_t B, int64_t L, int64_t D, double* h,
                      double* rho_hist, int32_t* chan_iters, int* converged, int* nonfinite) {
  size_t N = (size_t)B * (size_t)L * (size_t)D;
  newton_ctx x = {P, a, NULL, h0, NULL, h, NULL, NULL, NULL, L, D};
  x.Jt = (double*)malloc(N * sizeof(double));
  x.rt = (double*)malloc(N * sizeof(double));
  x.cmax = (double*)malloc((size_t)(B * D) * sizeof(double));
  int k = 0;
  *converged = 0;
  *nonfinite = 0;
  for (size_t i = 0; i < N; ++i) h[i] = 0.0;
  if (chan_iters)
    for (int64_t i = 0; i < B * D; ++i) chan_iters[i] = -1;
  for (k = 0;; ++k) {
    for_channels(B * D, newton_gru_residual_chan, &x); /* r_t, A_t at h^k */
    double rho = reduce_rho(x.cmax, B * D, tol, k, chan_iters);
    rho_hist[k] = rho;
    if (!isfinite(rho)) {
      *nonfinite = 1;
      break;
    }
    if (rho <= tol) {
      *converged = 1;
      break;
    }
    if (k == max_iters) break;
    for_channels(B * D, newton_gru_solve_chan, &x); /* delta, h^{k+1} */
  }
  free(x.Jt);
  free(x.rt);
  free(x.cmax);
  return k;
}

static void newton_lstm_residual_chan(void* p, int64_t ch) {
  newton_ctx* x = (newton_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double w[4] = {x->a[0 * D + d], x->a[1 * D + d], x->a[2 * D + d], x->a[3 * D + d]};
  double m = 0.0;
  for (int64_t t = 0; t < L; ++t) {
    double cp, hp;
    if (t == 0) {
      cp = x->c0 ? x->c0[bb * D + d] : 0.0;
      hp = x->h0 ? x->h0[bb * D + d] : 0.0;
    } else {
      cp = x->c[IDX3(bb, t - 1, d, L, D)];
      hp = x->h[IDX3(bb, t - 1, d, L, D)];
    }
    double pg[4];
    for (int g = 0; g < 4; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 4, D)];
    double fc, fh;
    size_t i = IDX3(bb, t, d, L, D);
    oracle_lstm_cell(pg, w, cp, hp, &fc, &fh, x->Jt + 4 * i);
    x->rt[2 * i + 0] = fc - x->c[i];
    x->rt[2 * i + 1] = fh - x->h[i];
    double a0 = fabs(x->rt[2 * i + 0]), a1 = fabs(x->rt[2 * i + 1]);
    if (!(a0 <= m)) m = a0;
    if (!(a1 <= m)) m = a1;
  }
  x->cmax[ch] = m;
}

static void newton_lstm_solve_chan(void* p, int64_t ch) {
  newton_ctx* x = (newton_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double e0 = 0.0, e1 = 0.0;
  for (int64_t t = 0; t < L; ++t) {
    size_t i = IDX3(bb, t, d, L, D);
    const double* M = x->Jt + 4 * i;
    double n0 = M[0] * e0 + M[1] * e1 + x->rt[2 * i + 0];
    double n1 = M[2] * e0 + M[3] * e1 + x->rt[2 * i + 1];
    e0 = n0;
    e1 = n1;
    x->c[i] += e0;
    x->h[i] += e1;
  }
}

int oracle_newton_lstm(const double* P, const double* a, const double* c0, const double* h0,
                       double tol, int max_iters, int64_t B, int64_t L, int64_t D, double* c,
                       double* h, double* rho_hist, int32_t* chan_iters, int* converged,
                       int* nonfinite) {
  size_t N = (size_t)B * (size_t)L * (size_t)D;
  newton_ctx x = {P, a, c0, h0, c, h, NULL, NULL, NULL, L, D};
  x.Jt = (double*)malloc(4 * N * sizeof(double));
  x.rt = (double*)malloc(2 * N * sizeof(double));
  x.cmax = (double*)malloc((size_t)(B * D) * sizeof(double));
  int k = 0;
  *converged = 0;
  *nonfinite = 0;
  for (size_t i = 0; i < N; ++i) {
    c[i] = 0.0;
    h[i] = 0.0;
  }
  if (chan_iters)
    for (int64_t i = 0; i < B * D; ++i) chan_iters[i] = -1;
  for (k = 0;; ++k) {
    for_channels(B * D, newton_lstm_residual_chan, &x);
    double rho = reduce_rho(x.cmax, B * D, tol, k, chan_iters);
    rho_hist[k] = rho;
    if (!isfinite(rho)) {
      *nonfinite = 1;
      break;
    }
    if (rho <= tol) {
      *converged = 1;
      break;
    }
    if (k == max_iters) break;
    for_channels(B * D, newton_lstm_solve_chan, &x);
  }
  free(x.Jt);
  free(x.rt);
  free(x.cmax);
  return k;
}

/* Max-abs residual of a given trajectory, max_t |f(h_{t-1}, P_t) - h_t|, in fp64:
 * a certificate for a trajectory computed elsewhere. */
typedef struct {
  const double *P, *a, *h0, *h;
  double* cmax;
  int64_t L, D;
} resid_ctx;

static void residual_gru_chan(void* p, int64_t ch) {
  resid_ctx* x = (resid_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double w[3] = {x->a[0 * D + d], x->a[1 * D + d], x->a[2 * D + d]};
  double m = 0.0;
  for (int64_t t = 0; t < L; ++t) {
    double hp = (t == 0) ? (x->h0 ? x->h0[bb * D + d] : 0.0) : x->h[IDX3(bb, t - 1, d, L, D)];
    double pg[3];
    for (int g = 0; g < 3; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 3, D)];
    double f;
    oracle_gru_cell(pg, w, hp, &f, NULL);
    double e = fabs(f - x->h[IDX3(bb, t, d, L, D)]);
    if (!(e <= m)) m = e;
  }
  x->cmax[ch] = m;
}

double oracle_residual_gru(const double* P, const double* a, const double* h0, const double* h,
                           int64_t B, int64_t L, int64_t D) {
  resid_ctx x = {P, a, h0, h, NULL, L, D};
  x.cmax = (double*)malloc((size_t)(B * D) * sizeof(double));
  for_channels(B * D, residual_gru_chan, &x);
  double m = reduce_rho(x.cmax, B * D, 0.0, 0, NULL);
  free(x.cmax);
  return m;
}

/* ------------------------------------------------------------------------- */
/* Gradients of the solved trajectory (the backward pass).                    */
/* ------------------------------------------------------------------------- */
/*
 * For a loss whose gradient with respect to the trajectory is g_t = dl/dh_t
 * (t = 1..L), the total gradient lambda_t = dl/dh_t through the recurrence
 * obeys the adjoint recursion
 *     lambda_L = g_L,   lambda_t = g_t + J_{t+1}^T lambda_{t+1},
 * with J_t = df/dh at (h_{t-1}, P_t).  Then
 *     dl/dP_t  = lambda_t^T df/dP_t (h_{t-1}, P_t),
 *     dl/da    = sum_t lambda_t^T df/da (h_{t-1}, P_t),
 *     dl/dh0   = J_1^T lambda_1.
 * The trajectory h is the solution of the forward system (given, not
 * recomputed).  Evaluated sequentially from t = L down to 1, in fp64.
 */
typedef struct {
  const double *P, *a, *c0, *h0, *c, *h, *gc, *gh;
  double *dP, *da_part, *dc0, *dh0;
  int64_t L, D;
} bwd_ctx;

/* GRU: df/dPz = (c-h) z(1-z), df/dPc = z(1-c^2), df/dPr = z(1-c^2) ac h r(1-r);
 * df/da_g = df/dP_g * (h for z and r, r*h for c). */
static void backward_gru_chan(void* p, int64_t ch) {
  bwd_ctx* x = (bwd_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double w[3] = {x->a[0 * D + d], x->a[1 * D + d], x->a[2 * D + d]};
  double da[3] = {0.0, 0.0, 0.0};
  double lam_next = 0.0; /* J_{t+1}^T lambda_{t+1}, zero after the last step */
  double mu = 0.0;
  for (int64_t t = L - 1; t >= 0; --t) {
    double hp = (t == 0) ? (x->h0 ? x->h0[bb * D + d] : 0.0) : x->h[IDX3(bb, t - 1, d, L, D)];
    double pg[3];
    for (int g = 0; g < 3; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 3, D)];
    double lam = x->gh[IDX3(bb, t, d, L, D)] + lam_next;
    double z = sig(pg[0] + w[0] * hp);
    double r = sig(pg[1] + w[1] * hp);
    double c = tanh(pg[2] + w[2] * (r * hp));
    double dfdz = (c - hp) * z * (1.0 - z);      /* d h'/d Pz */
    double dfdu = z * (1.0 - c * c);             /* d h'/d Pc */
    double dfdr = dfdu * w[2] * hp * r * (1.0 - r); /* d h'/d Pr */
    x->dP[IDXP(bb, t, 0, d, L, 3, D)] = lam * dfdz;
    x->dP[IDXP(bb, t, 1, d, L, 3, D)] = lam * dfdr;
    x->dP[IDXP(bb, t, 2, d, L, 3, D)] = lam * dfdu;
    da[0] += lam * dfdz * hp;
    da[1] += lam * dfdr * hp;
    da[2] += lam * dfdu * r * hp;
    double f, J;
    oracle_gru_cell(pg, w, hp, &f, &J);
    mu = J * lam;
    lam_next = mu;
  }
  if (x->dh0) x->dh0[bb * D + d] = mu;
  for (int g = 0; g < 3; ++g) x->da_part[ch * 3 + g] = da[g];
}

void oracle_backward_gru(const double* P, const double* a, const double* h0, const double* h,
                         const double* gh, double* dP, double* da, double* dh0, int64_t B,
                         int64_t L, int64_t D) {
  bwd_ctx x = {P, a, NULL, h0, NULL, h, NULL, gh, dP, NULL, NULL, dh0, L, D};
  x.da_part = (double*)malloc((size_t)(B * D) * 3 * sizeof(double));
  for_channels(B * D, backward_gru_chan, &x);
  for (int64_t g = 0; g < 3; ++g)
    for (int64_t d = 0; d < D; ++d) {
      double s = 0.0;
      for (int64_t bb = 0; bb < B; ++bb) s += x.da_part[(bb * D + d) * 3 + g];
      da[g * D + d] = s;
    }
  free(x.da_part);
}

/* LSTM, state (c, h), lambda = (lambda_c, lambda_h).  With u_x = P_x + a_x h:
 *   dc'/du_i = g i(1-i), dc'/du_f = c f(1-f), dc'/du_g = i(1-g^2), dc'/du_o = 0,
 *   dh'/du_x = o (1 - tanh(c')^2) dc'/du_x  (x = i, f, g),  dh'/du_o = tanh(c') o(1-o);
 *   dl/dP_x = lambda_c dc'/du_x + lambda_h dh'/du_x,   dl/da_x += dl/dP_x * h. */
static void backward_lstm_chan(void* p, int64_t ch) {
  bwd_ctx* x = (bwd_ctx*)p;
  int64_t L = x->L, D = x->D, bb = ch / D, d = ch % D;
  double w[4] = {x->a[0 * D + d], x->a[1 * D + d], x->a[2 * D + d], x->a[3 * D + d]};
  double da[4] = {0.0, 0.0, 0.0, 0.0};
  double mc = 0.0, mh = 0.0; /* J_{t+1}^T lambda_{t+1} */
  for (int64_t t = L - 1; t >= 0; --t) {
    double cp, hp;
    if (t == 0) {
      cp = x->c0 ? x->c0[bb * D + d] : 0.0;
      hp = x->h0 ? x->h0[bb * D + d] : 0.0;
    } else {
      cp = x->c[IDX3(bb, t - 1, d, L, D)];
      hp = x->h[IDX3(bb, t - 1, d, L, D)];
    }
    double pg[4];
    for (int g = 0; g < 4; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 4, D)];
    double lc = (x->gc ? x->gc[IDX3(bb, t, d, L, D)] : 0.0) + mc;
    double lh = (x->gh ? x->gh[IDX3(bb, t, d, L, D)] : 0.0) + mh;
    double ig = sig(pg[0] + w[0] * hp);
    double fg = sig(pg[1] + w[1] * hp);
    double gg = tanh(pg[2] + w[2] * hp);
    double og = sig(pg[3] + w[3] * hp);
    double cn = fg * cp + ig * gg;
    double tc = tanh(cn);
    double dc[4] = {gg * ig * (1.0 - ig), cp * fg * (1.0 - fg), ig * (1.0 - gg * gg), 0.0};
    double dh[4];
    for (int g = 0; g < 3; ++g) dh[g] = og * (1.0 - tc * tc) * dc[g];
    dh[3] = tc * og * (1.0 - og);
    for (int g = 0; g < 4; ++g) {
      double v = lc * dc[g] + lh * dh[g];
      x->dP[IDXP(bb, t, g, d, L, 4, D)] = v;
      da[g] += v * hp;
    }
    double fc, fh, J[4];
    oracle_lstm_cell(pg, w, cp, hp, &fc, &fh, J);
    /* J^T lambda: J = [[dc'/dc, dc'/dh], [dh'/dc, dh'/dh]] */
    mc = J[0] * lc + J[2] * lh;
    mh = J[1] * lc + J[3] * lh;
  }
  if (x->dc0) x->dc0[bb * D + d] = mc;
  if (x->dh0) x->dh0[bb * D + d] = mh;
  for (int g = 0; g < 4; ++g) x->da_part[ch * 4 + g] = da[g];
}

void oracle_backward_lstm(const double* P, const double* a, const double* c0, const double* h0,
                          const double* c, const double* h, const double* gc, const double* gh,
                          double* dP, double* da, double* dc0, double* dh0, int64_t B, int64_t L,
                          int64_t D) {
  bwd_ctx x = {P, a, c0, h0, c, h, gc, gh, dP, NULL, dc0, dh0, L, D};
  x.da_part = (double*)malloc((size_t)(B * D) * 4 * sizeof(double));
  for_channels(B * D, backward_lstm_chan, &x);
  for (int64_t g = 0; g < 4; ++g)
    for (int64_t d = 0; d < D; ++d) {
      double s = 0.0;
      for (int64_t bb = 0; bb < B; ++bb) s += x.da_part[(bb * D + d) * 4 + g];
      da[g * D + d] = s;
    }
  free(x.da_part);
}

/* ------------------------------------------------------------------------
 * Input projection P = x W^T + bias: the projected gate pre-activations the
 * cells take as inputs (ParaRNN TL;DR: the recurrence keeps diagonal weights
 * only, the dense weights act on the inputs).  x [M,K], W [N,K] (one row of W
 * per output feature), bias [N] or NULL, P [M,N]; plain sums in k order.
 * ---------------------------------------------------------------------- */
typedef struct {
  const double *x, *W, *bias;
  double* P;
  int64_t N, K;
} proj_ctx;

static void projection_row(void* p, int64_t m) {
  const proj_ctx* c = (const proj_ctx*)p;
  for (int64_t n = 0; n < c->N; ++n) {
    double s = c->bias ? c->bias[n] : 0.0;
    for (int64_t k = 0; k < c->K; ++k) s += c->x[m * c->K + k] * c->W[n * c->K + k];
    c->P[m * c->N + n] = s;
  }
}

void oracle_input_projection(const double* x, const double* W, const double* bias, double* P,
                             int64_t M, int64_t N, int64_t K) {
  proj_ctx c = {x, W, bias, P, N, K};
  for_channels(M, projection_row, &c);
}

/* ------------------------------------------------------------------------
 * Multi-head GRU with dense 8x8 recurrence blocks (the "dense small-block"
 * variant: DEER summary, caveats -- dense Jacobians cost O(n^3) per step; here
 * n = 8 per head).  Channels d = 8 * head + i; per head, with U_g the head's
 * 8x8 block of gate g (row i = output channel, column j = input channel):
 *   z = sig(P_z + U_z h),  r = sig(P_r + U_r h),  c = tanh(P_c + r * (U_c h)),
 *   h' = (1 - z) * h + z * c            (elementwise products)
 * which is the ParaGRU cell when every U_g is diagonal.  Jacobian, row i:
 *   dh'_i/dh_j = [i == j] (1 - z_i) + (c_i - h_i) z_i (1 - z_i) U_z[i][j]
 *              + z_i (1 - c_i^2) (r_i U_c[i][j] + (U_c h)_i r_i (1 - r_i) U_r[i][j])
 * P is [B, L, 3, D] (gates z, r, c), U is [3, H, 8, 8], D = 8 H.
 *
 * Time strides (DEER summary, caveats paragraph: heads of 8 channels with
 * exponentially increasing strides, i.e. shorter effective sequences): head g
 * may recur at stride s_g >= 1, h_t = f(h_{t - s_g}, P_t), with h_{t - s_g} = h0
 * for t < s_g.  strides == NULL means s_g = 1 for every head.
 * ---------------------------------------------------------------------- */
#define NB 8

void oracle_mhgru_cell(const double* p /* [3][8] */, const double* U /* [3][8][8] of one head */,
                       const double* h, double* f, double* J /* [8][8] or NULL */) {
  double uz[NB], ur[NB], uc[NB];
  for (int i = 0; i < NB; ++i) {
    uz[i] = ur[i] = uc[i] = 0.0;
    for (int j = 0; j < NB; ++j) {
      uz[i] += U[(0 * NB + i) * NB + j] * h[j];
      ur[i] += U[(1 * NB + i) * NB + j] * h[j];
      uc[i] += U[(2 * NB + i) * NB + j] * h[j];
    }
  }
  for (int i = 0; i < NB; ++i) {
    double z = sig(p[0 * NB + i] + uz[i]);
    double r = sig(p[1 * NB + i] + ur[i]);
    double c = tanh(p[2 * NB + i] + r * uc[i]);
    f[i] = (1.0 - z) * h[i] + z * c;
    if (J) {
      double dz = (c - h[i]) * z * (1.0 - z);
      double dc = z * (1.0 - c * c);
      for (int j = 0; j < NB; ++j)
        J[i * NB + j] = (i == j ? 1.0 - z : 0.0) + dz * U[(0 * NB + i) * NB + j] +
                        dc * (r * U[(2 * NB + i) * NB + j] +
                              uc[i] * r * (1.0 - r) * U[(1 * NB + i) * NB + j]);
    }
  }
}

typedef struct {
  const double *P, *U, *h0;
  double *h, *Jt, *rt, *cmax;
  int64_t L, H;
  const int32_t* stride; /* [H] or NULL (all 1) */
  double* dt;            /* Newton step delta, [B, L, D] */
} mh_ctx;

static int64_t mh_stride(const mh_ctx* x, int64_t g) { return x->stride ? x->stride[g] : 1; }

/* gates of head g at (b, t): p[gate * 8 + i] */
static void mh_gates(const mh_ctx* x, int64_t bb, int64_t t, int64_t g, double* p) {
  int64_t D = NB * x->H;
  for (int k = 0; k < 3; ++k)
    for (int i = 0; i < NB; ++i) p[k * NB + i] = x->P[IDXP(bb, t, k, g * NB + i, x->L, 3, D)];
}

/* the state the step at t recurs on: h_{t - s_g}, or h0 before the sequence */
static void mh_prev(const mh_ctx* x, int64_t bb, int64_t t, int64_t g, double* hp) {
  int64_t D = NB * x->H, tp = t - mh_stride(x, g);
  for (int i = 0; i < NB; ++i)
    hp[i] = (tp < 0) ? (x->h0 ? x->h0[bb * D + g * NB + i] : 0.0)
                     : x->h[IDX3(bb, tp, g * NB + i, x->L, D)];
}

static void rollout_mhgru_head(void* p, int64_t u) {
  mh_ctx* x = (mh_ctx*)p;
  int64_t bb = u / x->H, g = u % x->H, D = NB * x->H;
  double hp[NB], f[NB], pg[3 * NB];
  for (int64_t t = 0; t < x->L; ++t) {
    mh_prev(x, bb, t, g, hp);
    mh_gates(x, bb, t, g, pg);
    oracle_mhgru_cell(pg, x->U + g * 3 * NB * NB, hp, f, NULL);
    for (int i = 0; i < NB; ++i) x->h[IDX3(bb, t, g * NB + i, x->L, D)] = f[i];
  }
}

/* U here is [3, H, 8, 8]; the cell wants one head's [3][8][8]: gather it. */
static double* mh_heads(const double* U, int64_t H) {
  double* Uh = (double*)malloc((size_t)H * 3 * NB * NB * sizeof(double));
  for (int64_t g = 0; g < H; ++g)
    for (int k = 0; k < 3; ++k)
      for (int e = 0; e < NB * NB; ++e)
        Uh[(g * 3 + k) * NB * NB + e] = U[((size_t)k * H + g) * NB * NB + e];
  return Uh;
}

void oracle_rollout_mhgru(const double* P, const double* U, const double* h0, double* h,
                          int64_t B, int64_t L, int64_t H, const int32_t* strides) {
  double* Uh = mh_heads(U, H);
  mh_ctx x = {P, Uh, h0, h, NULL, NULL, NULL, L, H, strides, NULL};
  for_channels(B * H, rollout_mhgru_head, &x);
  free(Uh);
}

static void newton_mhgru_residual_head(void* p, int64_t u) {
  mh_ctx* x = (mh_ctx*)p;
  int64_t bb = u / x->H, g = u % x->H, D = NB * x->H, L = x->L;
  double hp[NB], f[NB], pg[3 * NB], m = 0.0;
  for (int64_t t = 0; t < L; ++t) {
    mh_prev(x, bb, t, g, hp);
    mh_gates(x, bb, t, g, pg);
    double* J = x->Jt + ((size_t)u * L + t) * NB * NB;
    oracle_mhgru_cell(pg, x->U + g * 3 * NB * NB, hp, f, J);
    for (int i = 0; i < NB; ++i) {
      size_t k = IDX3(bb, t, g * NB + i, L, D);
      x->rt[k] = f[i] - x->h[k];
      double ar = fabs(x->rt[k]);
      if (!(ar <= m)) m = ar; /* keeps a NaN */
    }
  }
  x->cmax[u] = m;
}

static void newton_mhgru_solve_head(void* p, int64_t u) {
  mh_ctx* x = (mh_ctx*)p;
  int64_t bb = u / x->H, g = u % x->H, D = NB * x->H, L = x->L, st = mh_stride(x, g);
  for (int64_t t = 0; t < L; ++t) {
    /* delta_t = J_t delta_{t - s} + r_t, with delta = 0 before the sequence */
    const double* J = x->Jt + ((size_t)u * L + t) * NB * NB;
    double prev[NB], nd[NB];
    for (int j = 0; j < NB; ++j)
      prev[j] = (t - st < 0) ? 0.0 : x->dt[IDX3(bb, t - st, g * NB + j, L, D)];
    for (int i = 0; i < NB; ++i) {
      double s = x->rt[IDX3(bb, t, g * NB + i, L, D)];
      for (int j = 0; j < NB; ++j) s += J[i * NB + j] * prev[j];
      nd[i] = s;
    }
    for (int i = 0; i < NB; ++i) x->dt[IDX3(bb, t, g * NB + i, L, D)] = nd[i];
  }
  /* the update, once every delta of the head is known */
  for (int64_t t = 0; t < L; ++t)
    for (int i = 0; i < NB; ++i)
      x->h[IDX3(bb, t, g * NB + i, L, D)] += x->dt[IDX3(bb, t, g * NB + i, L, D)];
}

/* Serial Newton as oracle_newton_gru, with 8x8 blocks: the linear solve is
 * delta_t = J_t delta_{t-s} + r_t per head (s = the head's stride, 1 by
 * default).  rho_hist has max_iters + 1 slots. */
int oracle_newton_mhgru(const double* P, const double* U, const double* h0, double tol,
                        int max_iters, int64_t B, int64_t L, int64_t H, double* h,
                        double* rho_hist, int* converged, int* nonfinite,
                        const int32_t* strides) {
  size_t N = (size_t)B * (size_t)L * (size_t)(NB * H);
  double* Uh = mh_heads(U, H);
  mh_ctx x = {P, Uh, h0, h, NULL, NULL, NULL, L, H, strides, NULL};
  x.dt = (double*)malloc(N * sizeof(double));
  x.Jt = (double*)malloc(N * NB * sizeof(double));
  x.rt = (double*)malloc(N * sizeof(double));
  x.cmax = (double*)malloc((size_t)(B * H) * sizeof(double));
  int k;
  *converged = 0;
  *nonfinite = 0;
  for (size_t i = 0; i < N; ++i) h[i] = 0.0;
  for (k = 0;; ++k) {
    for_channels(B * H, newton_mhgru_residual_head, &x);
    double rho = reduce_rho(x.cmax, B * H, tol, k, NULL);
    rho_hist[k] = rho;
    if (!isfinite(rho)) {
      *nonfinite = 1;
      break;
    }
    if (rho <= tol) {
      *converged = 1;
      break;
    }
    if (k == max_iters) break;
    for_channels(B * H, newton_mhgru_solve_head, &x);
  }
  free(x.Jt);
  free(x.rt);
  free(x.cmax);
  free(x.dt);
  free(Uh);
  return k;
}
