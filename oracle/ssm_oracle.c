/*
 * ssm_oracle.c -- plain, slow, sequential fp64 CPU oracle for the Mamba
 * selective state-space scan and its single-token state update.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The product (the CUDA
 * library and its Python binding) never calls it and shares no code with it.
 *
 * What it computes, per batch b and channel d, with state h[n], n < N:
 *
 *   v      = delta[b,t,d] + bias[d]                 (bias: the dt projection's
 *                                                    bias, Mamba block, §3.4)
 *   Delta  = softplus(v) if softplus else v          (selection mechanism,
 *                                                    §3.1: Delta_t = softplus(.))
 *   h[n]   = exp(Delta * A[d,n]) * h[n]
 *            + Delta * B[b,t,n] * x[b,t,d]           (discretised recurrence,
 *                                                    §2.2, with the simplified
 *                                                    deltaB = Delta*B of the
 *                                                    §3.3 selective_scan; the
 *                                                    _zoh entry points use the
 *                                                    exact ZOH B-bar of §2.2)
 *   y      = sum_n C[b,t,n] * h[n] + D[d] * x[b,t,d] (readout, §2.2 y_t = C h_t,
 *                                                    plus the block's D skip)
 *   y     *= z / (1 + exp(-z))   if z is given       (block gate y * SiLU(z), §3.4)
 *
 * with h = h0[b,d,:] (or 0) before t = 0 and h_last[b,d,:] = h after t = L-1.
 * Section numbers refer to the page "Mamba 논문 리뷰: Selective State Space
 * Models로 Transformer를 넘어서" (youngju.dev): §2.2 Zero-Order Hold
 * discretisation, §3.1 Selection Mechanism, §3.3 Hardware-Aware algorithm
 * (the simplified selective_scan), §3.4 Mamba Block.
 *
 * Readings where the pages are silent or inconsistent (each also listed in
 * the design notes):
 *   - B-bar: the simplified Delta*B of the §3.3 scan, not the exact ZOH form
 *     of §2.2.
 *   - softplus(v) = log1p(exp(v)) for v <= 20 and v itself above 20.
 *   - The skip term D*x is added before the gate: y = (C.h + D x) * SiLU(z).
 *   - y_t reads the state after x_t has entered it.
 *
 * Inputs are read in their storage type (bf16 or fp32) and widened exactly
 * to double; every operation after that is fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_MAX_N 1024

/* Widen element i of an input tensor to double. bf16 is the upper half of an
 * IEEE binary32, so shifting it into place is exact. */
static double widen(const void* p, int64_t i, int is_bf16) {
  if (is_bf16) {
    uint32_t w = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
  }
  return (double)((const float*)p)[i];
}

/* softplus(v) = log(1 + e^v) (§3.1); the identity above 20, where the
 * difference is below 2.1e-9 relative. */
static double softplus(double v) { return v > 20.0 ? v : log1p(exp(v)); }

/* SiLU(z) = z * sigmoid(z) (§3.4 gate). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* The factor that multiplies B[n] x in the state update: Delta (the
 * simplified deltaB = Delta*B of the §3.3 selective_scan), or, for the exact
 * zero-order hold of §2.2, B-bar = (Delta A)^-1 (exp(Delta A) - 1) Delta B,
 * which for a diagonal A is (exp(Delta A_n) - 1) / A_n (Delta at A_n = 0). */
static double input_coef(double dt, double An, int zoh) {
  if (!zoh) return dt;
  return An == 0.0 ? dt : expm1(dt * An) / An;
}

typedef struct {
  int64_t batch, seqlen, dim, dstate;
  int is_bf16;
  const void* x;       /* (batch, seqlen, dim)    io type */
  const void* delta;   /* (batch, seqlen, dim)    io type */
  const float* A;      /* (dim, dstate)           fp32    */
  const void* B;       /* (batch, seqlen, dstate) io type */
  const void* C;       /* (batch, seqlen, dstate) io type */
  const float* D;      /* (dim) fp32 or NULL              */
  const void* z;       /* (batch, seqlen, dim) io or NULL */
  const float* bias;   /* (dim) fp32 or NULL              */
  int softplus;
  const float* h0;     /* (batch, dim, dstate) fp32 or NULL */
  const int64_t* chans;/* nchan pairs (b, d)              */
  int64_t nchan;
  double* y;           /* (nchan, seqlen)                 */
  double* h_last;      /* (nchan, dstate) or NULL         */
  int zoh;             /* input term: 0 Delta*B (§3.3), 1 exact ZOH (§2.2) */
} scan_job;

/* One channel (b, d), sequentially in t: the loop of the §3.3 selective_scan
 * for a single (b, d) row, without materialising deltaA / deltaB. */
static void scan_one_channel(const scan_job* j, int64_t k) {
  const int64_t b = j->chans[2 * k], d = j->chans[2 * k + 1];
  const int64_t L = j->seqlen, Dm = j->dim, N = j->dstate;
  double h[ORACLE_MAX_N];
  for (int64_t n = 0; n < N; ++n)
    h[n] = j->h0 ? (double)j->h0[(b * Dm + d) * N + n] : 0.0;
  const double bias = j->bias ? (double)j->bias[d] : 0.0;
  const double Dd = j->D ? (double)j->D[d] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    const int64_t i_bld = (b * L + t) * Dm + d;
    const int64_t i_bln = (b * L + t) * N;
    const double xv = widen(j->x, i_bld, j->is_bf16);
    const double v = widen(j->delta, i_bld, j->is_bf16) + bias;
    const double dt = j->softplus ? softplus(v) : v;
    double y = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const double dA = exp(dt * (double)j->A[d * N + n]);
      const double dB = input_coef(dt, (double)j->A[d * N + n], j->zoh) *
                        widen(j->B, i_bln + n, j->is_bf16);
      h[n] = dA * h[n] + dB * xv;
      y += widen(j->C, i_bln + n, j->is_bf16) * h[n];
    }
    y += Dd * xv;
    if (j->z) y *= silu(widen(j->z, i_bld, j->is_bf16));
    j->y[k * L + t] = y;
  }
  if (j->h_last)
    for (int64_t n = 0; n < N; ++n) j->h_last[k * N + n] = h[n];
}

typedef struct {
  const scan_job* job;
  int64_t lo, hi;
} scan_slice;

static void* scan_worker(void* arg) {
  const scan_slice* s = (const scan_slice*)arg;
  for (int64_t k = s->lo; k < s->hi; ++k) scan_one_channel(s->job, k);
  return NULL;
}

/*
 * oracle_selective_scan -- run the scan for `nchan` channels given as
 * (b, d) pairs in `chans`, splitting the channels over `nthreads` threads
 * (each channel stays sequential in t). Returns 0, or -1 on bad arguments.
 */
static int scan_impl(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int is_bf16,
                     const void* x, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* bias,
                     int softplus_on, const float* h0, const int64_t* chans, int64_t nchan,
                     double* y, double* h_last, int nthreads, int zoh);

int oracle_selective_scan(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                          int is_bf16, const void* x, const void* delta, const float* A,
                          const void* B, const void* C, const float* D, const void* z,
                          const float* bias, int softplus_on, const float* h0,
                          const int64_t* chans, int64_t nchan, double* y, double* h_last,
                          int nthreads) {
  return scan_impl(batch, seqlen, dim, dstate, is_bf16, x, delta, A, B, C, D, z, bias,
                   softplus_on, h0, chans, nchan, y, h_last, nthreads, 0);
}

/* oracle_selective_scan_zoh -- the same scan with the exact zero-order-hold
 * input term of §2.2 (B-bar = (exp(Delta A) - 1) / A * B per state). */
int oracle_selective_scan_zoh(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                              int is_bf16, const void* x, const void* delta, const float* A,
                              const void* B, const void* C, const float* D, const void* z,
                              const float* bias, int softplus_on, const float* h0,
                              const int64_t* chans, int64_t nchan, double* y, double* h_last,
                              int nthreads) {
  return scan_impl(batch, seqlen, dim, dstate, is_bf16, x, delta, A, B, C, D, z, bias,
                   softplus_on, h0, chans, nchan, y, h_last, nthreads, 1);
}

static int scan_impl(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate, int is_bf16,
                     const void* x, const void* delta, const float* A, const void* B,
                     const void* C, const float* D, const void* z, const float* bias,
                     int softplus_on, const float* h0, const int64_t* chans, int64_t nchan,
                     double* y, double* h_last, int nthreads, int zoh) {
  if (batch < 0 || seqlen < 0 || dim < 0 || dstate <= 0 || dstate > ORACLE_MAX_N) return -1;
  if (!x || !delta || !A || !B || !C || !chans || !y) return -1;
  for (int64_t k = 0; k < nchan; ++k)
    if (chans[2 * k] < 0 || chans[2 * k] >= batch || chans[2 * k + 1] < 0 ||
        chans[2 * k + 1] >= dim)
      return -1;
  scan_job job = {batch, seqlen, dim, dstate, is_bf16, x, delta, A, B, C, D, z,
                  bias, softplus_on, h0, chans, nchan, y, h_last, zoh};
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (nthreads == 1 || nchan < 2) {
    for (int64_t k = 0; k < nchan; ++k) scan_one_channel(&job, k);
    return 0;
  }
  pthread_t tid[256];
  scan_slice sl[256];
  int started = 0;
  for (int w = 0; w < nthreads; ++w) {
    sl[w].job = &job;
    sl[w].lo = nchan * w / nthreads;
    sl[w].hi = nchan * (w + 1) / nthreads;
    if (pthread_create(&tid[w], NULL, scan_worker, &sl[w]) == 0) {
      ++started;
    } else {
      scan_worker(&sl[w]);
      tid[w] = 0;
    }
  }
  for (int w = 0; w < nthreads; ++w)
    if (tid[w]) pthread_join(tid[w], NULL);
  (void)started;
  return 0;
}

/*
 * oracle_state_update -- one decode step (the recurrent, O(1)-per-token form
 * of the same recurrence: the scan's loop body with L = 1). `state` is the
 * oracle's own fp64 (batch, dim, dstate) state, updated in place; y is
 * (batch, dim). x, delta, z are (batch, dim); B, C are (batch, dstate).
 */
static int state_update_impl(int64_t batch, int64_t dim, int64_t dstate, int is_bf16,
                             double* state, const void* x, const void* delta, const float* A,
                             const void* B, const void* C, const float* D, const void* z,
                             const float* bias, int softplus_on, double* y, int zoh);

int oracle_state_update(int64_t batch, int64_t dim, int64_t dstate, int is_bf16,
                        double* state, const void* x, const void* delta, const float* A,
                        const void* B, const void* C, const float* D, const void* z,
                        const float* bias, int softplus_on, double* y) {
  return state_update_impl(batch, dim, dstate, is_bf16, state, x, delta, A, B, C, D, z, bias,
                           softplus_on, y, 0);
}

/* oracle_state_update_zoh -- one decode step with the exact ZOH input term. */
int oracle_state_update_zoh(int64_t batch, int64_t dim, int64_t dstate, int is_bf16,
                            double* state, const void* x, const void* delta, const float* A,
                            const void* B, const void* C, const float* D, const void* z,
                            const float* bias, int softplus_on, double* y) {
  return state_update_impl(batch, dim, dstate, is_bf16, state, x, delta, A, B, C, D, z, bias,
                           softplus_on, y, 1);
}

static int state_update_impl(int64_t batch, int64_t dim, int64_t dstate, int is_bf16,
                             double* state, const void* x, const void* delta, const float* A,
                             const void* B, const void* C, const float* D, const void* z,
                             const float* bias, int softplus_on, double* y, int zoh) {
  if (batch < 0 || dim < 0 || dstate <= 0 || !state || !x || !delta || !A || !B || !C || !y)
    return -1;
  for (int64_t b = 0; b < batch; ++b) {
    for (int64_t d = 0; d < dim; ++d) {
      const int64_t i_bd = b * dim + d;
      const double xv = widen(x, i_bd, is_bf16);
      const double v = widen(delta, i_bd, is_bf16) + (bias ? (double)bias[d] : 0.0);
      const double dt = softplus_on ? softplus(v) : v;
      double* h = state + i_bd * dstate;
      double acc = 0.0;
      for (int64_t n = 0; n < dstate; ++n) {
        const double dA = exp(dt * (double)A[d * dstate + n]);
        const double dB = input_coef(dt, (double)A[d * dstate + n], zoh) *
                          widen(B, b * dstate + n, is_bf16);
        h[n] = dA * h[n] + dB * xv;
        acc += widen(C, b * dstate + n, is_bf16) * h[n];
      }
      acc += (D ? (double)D[d] : 0.0) * xv;
      if (z) acc *= silu(widen(z, i_bd, is_bf16));
      y[i_bd] = acc;
    }
  }
  return 0;
}

/* ------------------------------------------------------------------------
 * Backward pass: the gradient of the scan above, by reverse-mode
 * differentiation of its loop (the recomputation-based training of the
 * §3.3 Hardware-Aware algorithm needs exactly these gradients; the pages give
 * no formulas for them, so they are derived here from the forward loop by the
 * chain rule). For the loss  sum dy[b,t,d] y[b,t,d] + sum dh_last[b,d,n]
 * h_last[b,d,n], with per-step quantities of one channel (b, d):
 *
 *   v_t = delta_t + bias,  Dt_t = softplus(v_t) (or v_t),  a_tn = exp(Dt_t A_n)
 *   h_tn = a_tn h_(t-1)n + Dt_t B_tn x_t,   s_t = sum_n C_tn h_tn + D x_t
 *   y_t = s_t SiLU(z_t)  (or s_t)
 *
 * the adjoint of the state, lam_tn = dLoss/dh_tn, obeys
 *   lam_(L-1)n = C_(L-1)n g_(L-1) + dh_last_n,
 *   lam_tn     = C_tn g_t + a_(t+1)n lam_(t+1)n,   g_t = dy_t SiLU(z_t)
 * and the input gradients are
 *   dz_t     = dy_t s_t SiLU'(z_t),   SiLU'(z) = sig(z) (1 + z (1 - sig(z)))
 *   dx_t     = D g_t + Dt_t sum_n lam_tn B_tn
 *   dDt_t    = x_t sum_n lam_tn B_tn + sum_n lam_tn A_n a_tn h_(t-1)n
 *   ddelta_t = dDt_t softplus'(v_t) = dDt_t sig(v_t)  (1 above the cutoff 20,
 *              where the forward uses the identity; 1 without softplus)
 *   dbias    = sum_(b,t) ddelta_t,  dD = sum_(b,t) g_t x_t
 *   dA_n     = sum_(b,t) lam_tn Dt_t a_tn h_(t-1)n
 *   dB_tn    = sum_d lam_tn Dt_t x_t,   dC_tn = sum_d g_t h_tn
 *   dh0_n    = a_0n lam_0n.
 * ------------------------------------------------------------------------ */

typedef struct {
  scan_job fwd;         /* inputs; fwd.y / fwd.h_last unused */
  const void* dy;       /* (batch, seqlen, dim) io type */
  const float* dh_last; /* (batch, dim, dstate) fp32 or NULL */
  /* per listed channel k */
  double* dx;           /* (nchan, seqlen) */
  double* ddelta;       /* (nchan, seqlen) */
  double* dz;           /* (nchan, seqlen) or NULL */
  double* dh0;          /* (nchan, dstate) */
} bwd_job;

/* Per-thread accumulators of the gradients summed over channels. */
typedef struct {
  double* dA;    /* (dim, dstate) */
  double* dB;    /* (batch, seqlen, dstate) */
  double* dC;    /* (batch, seqlen, dstate) */
  double* dD;    /* (dim) */
  double* dbias; /* (dim) */
} bwd_acc;

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* One channel: the forward loop again, keeping every state, then the adjoint
 * loop backwards in t. `hist` holds (seqlen + 1) * dstate doubles. */
static void bwd_one_channel(const bwd_job* j, const bwd_acc* acc, int64_t k, double* hist,
                            double* s_hist) {
  const scan_job* f = &j->fwd;
  const int64_t b = f->chans[2 * k], d = f->chans[2 * k + 1];
  const int64_t L = f->seqlen, Dm = f->dim, N = f->dstate;
  const double bias = f->bias ? (double)f->bias[d] : 0.0;
  const double Dd = f->D ? (double)f->D[d] : 0.0;
  /* hist[0] = h_(-1), hist[t + 1] = h_t */
  for (int64_t n = 0; n < N; ++n)
    hist[n] = f->h0 ? (double)f->h0[(b * Dm + d) * N + n] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    const int64_t i_bld = (b * L + t) * Dm + d, i_bln = (b * L + t) * N;
    const double xv = widen(f->x, i_bld, f->is_bf16);
    const double v = widen(f->delta, i_bld, f->is_bf16) + bias;
    const double dt = f->softplus ? softplus(v) : v;
    double s = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const double a = exp(dt * (double)f->A[d * N + n]);
      hist[(t + 1) * N + n] = a * hist[t * N + n] + dt * widen(f->B, i_bln + n, f->is_bf16) * xv;
      s += widen(f->C, i_bln + n, f->is_bf16) * hist[(t + 1) * N + n];
    }
    s_hist[t] = s + Dd * xv;
  }
  double lam[ORACLE_MAX_N];
  for (int64_t n = 0; n < N; ++n)
    lam[n] = j->dh_last ? (double)j->dh_last[(b * Dm + d) * N + n] : 0.0;
  for (int64_t t = L - 1; t >= 0; --t) {
    const int64_t i_bld = (b * L + t) * Dm + d, i_bln = (b * L + t) * N;
    const double xv = widen(f->x, i_bld, f->is_bf16);
    const double v = widen(f->delta, i_bld, f->is_bf16) + bias;
    const double dt = f->softplus ? softplus(v) : v;
    const double dyv = widen(j->dy, i_bld, f->is_bf16);
    double g = dyv;
    if (f->z) {
      const double zv = widen(f->z, i_bld, f->is_bf16);
      const double sg = sigmoid(zv);
      g = dyv * zv * sg;
      if (j->dz) j->dz[k * L + t] = dyv * s_hist[t] * sg * (1.0 + zv * (1.0 - sg));
    }
    acc->dD[d] += g * xv;
    double sum_lb = 0.0, sum_la = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const double An = (double)f->A[d * N + n];
      const double a = exp(dt * An);
      const double hprev = hist[t * N + n];
      lam[n] += widen(f->C, i_bln + n, f->is_bf16) * g;
      acc->dC[i_bln + n] += g * hist[(t + 1) * N + n];
      acc->dB[i_bln + n] += lam[n] * dt * xv;
      sum_lb += lam[n] * widen(f->B, i_bln + n, f->is_bf16);
      sum_la += lam[n] * An * a * hprev;
      acc->dA[d * N + n] += lam[n] * dt * a * hprev;
      lam[n] *= a;
    }
    j->dx[k * L + t] = Dd * g + dt * sum_lb;
    const double ddt = xv * sum_lb + sum_la;
    const double dv = !f->softplus ? ddt : (v > 20.0 ? ddt : ddt * sigmoid(v));
    j->ddelta[k * L + t] = dv;
    acc->dbias[d] += dv;
  }
  for (int64_t n = 0; n < N; ++n) j->dh0[k * N + n] = lam[n];
}

typedef struct {
  const bwd_job* job;
  bwd_acc acc;
  int64_t lo, hi;
  int failed;
} bwd_slice;

static void* bwd_worker(void* arg) {
  bwd_slice* s = (bwd_slice*)arg;
  const scan_job* f = &s->job->fwd;
  double* hist = (double*)malloc((size_t)(f->seqlen + 1) * (size_t)f->dstate * sizeof(double));
  double* s_hist = (double*)malloc((size_t)(f->seqlen > 0 ? f->seqlen : 1) * sizeof(double));
  if (!hist || !s_hist) {
    s->failed = 1;
  } else {
    for (int64_t k = s->lo; k < s->hi; ++k) bwd_one_channel(s->job, &s->acc, k, hist, s_hist);
  }
  free(hist);
  free(s_hist);
  return NULL;
}

/*
 * oracle_selective_scan_bwd -- gradients of the scan for the `nchan`
 * channels listed in `chans` (pairs (b, d)), over `nthreads` threads.
 * Per-channel outputs dx, ddelta, dz (NULL when z is NULL), dh0 are indexed
 * by list position. dA, dB, dC, dD, dbias are sums over the listed channels
 * (all of a row b's channels give dB, dC of row b; all rows b of channel d
 * give dA[d], dD[d], dbias[d]); they are overwritten. Threads accumulate
 * privately and the sums are added in thread order, so results do not depend
 * on timing. Returns 0, -1 on bad arguments, -2 when memory runs out.
 */
int oracle_selective_scan_bwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                              int is_bf16, const void* x, const void* delta, const float* A,
                              const void* B, const void* C, const float* D, const void* z,
                              const float* bias, int softplus_on, const float* h0,
                              const void* dy, const float* dh_last, const int64_t* chans,
                              int64_t nchan, double* dx, double* ddelta, double* dz,
                              double* dh0, double* dA, double* dB, double* dC, double* dD,
                              double* dbias, int nthreads) {
  if (batch < 0 || seqlen < 0 || dim < 0 || dstate <= 0 || dstate > ORACLE_MAX_N) return -1;
  if (!x || !delta || !A || !B || !C || !dy || !chans || !dx || !ddelta || !dh0 || !dA ||
      !dB || !dC || !dD || !dbias || (z && !dz))
    return -1;
  for (int64_t k = 0; k < nchan; ++k)
    if (chans[2 * k] < 0 || chans[2 * k] >= batch || chans[2 * k + 1] < 0 ||
        chans[2 * k + 1] >= dim)
      return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 64) nthreads = 64;
  if (nchan < nthreads) nthreads = nchan > 0 ? (int)nchan : 1;
  bwd_job job;
  scan_job f = {batch, seqlen, dim, dstate, is_bf16, x, delta, A, B, C, D, z,
                bias, softplus_on, h0, chans, nchan, NULL, NULL, 0};
  job.fwd = f;
  job.dy = dy;
  job.dh_last = dh_last;
  job.dx = dx;
  job.ddelta = ddelta;
  job.dz = z ? dz : NULL;
  job.dh0 = dh0;
  const size_t nA = (size_t)dim * dstate, nBC = (size_t)batch * seqlen * dstate;
  const size_t per = nA + 2 * nBC + 2 * (size_t)dim;
  bwd_slice sl[64];
  pthread_t tid[64];
  int rc = 0;
  for (int w = 0; w < nthreads; ++w) {
    double* m = (double*)calloc(per > 0 ? per : 1, sizeof(double));
    sl[w].job = &job;
    sl[w].lo = nchan * w / nthreads;
    sl[w].hi = nchan * (w + 1) / nthreads;
    sl[w].failed = m == NULL;
    sl[w].acc.dA = m;
    sl[w].acc.dB = m ? m + nA : NULL;
    sl[w].acc.dC = m ? m + nA + nBC : NULL;
    sl[w].acc.dD = m ? m + nA + 2 * nBC : NULL;
    sl[w].acc.dbias = m ? m + nA + 2 * nBC + dim : NULL;
    tid[w] = 0;
  }
  for (int w = 0; w < nthreads; ++w) {
    if (sl[w].failed) continue;
    if (nthreads == 1 || pthread_create(&tid[w], NULL, bwd_worker, &sl[w]) != 0) {
      tid[w] = 0;
      bwd_worker(&sl[w]);
    }
  }
  for (int w = 0; w < nthreads; ++w)
    if (tid[w]) pthread_join(tid[w], NULL);
  memset(dA, 0, nA * sizeof(double));
  memset(dB, 0, nBC * sizeof(double));
  memset(dC, 0, nBC * sizeof(double));
  memset(dD, 0, (size_t)dim * sizeof(double));
  memset(dbias, 0, (size_t)dim * sizeof(double));
  for (int w = 0; w < nthreads; ++w) {
    if (sl[w].failed) rc = -2;
    if (!sl[w].acc.dA) continue;
    for (size_t i = 0; i < nA; ++i) dA[i] += sl[w].acc.dA[i];
    for (size_t i = 0; i < nBC; ++i) dB[i] += sl[w].acc.dB[i];
    for (size_t i = 0; i < nBC; ++i) dC[i] += sl[w].acc.dC[i];
    for (int64_t i = 0; i < dim; ++i) dD[i] += sl[w].acc.dD[i];
    for (int64_t i = 0; i < dim; ++i) dbias[i] += sl[w].acc.dbias[i];
    free(sl[w].acc.dA);
  }
  return rc;
}

/* ------------------------------------------------------------------------
 * The block's causal depthwise convolution and SiLU (page "Mamba 논문 리뷰",
 * §3.4 Mamba Block: conv1d = nn.Conv1d(d_inner, d_inner, d_conv,
 * padding=d_conv-1, groups=d_inner), its output cut to the first L steps,
 * then SiLU). Per batch row b, channel d and step t, with taps k < width:
 *
 *   u[b,t,d]   = bias[d] + sum_k w[d,k] * x[b, t - (width-1) + k, d]
 *                (x at negative steps is the zero padding)
 *   out[b,t,d] = SiLU(u[b,t,d])  (or u without SiLU)
 *
 * The backward, for the loss sum dout * out, is
 *   du[t]    = dout[t] * SiLU'(u[t])  (or dout[t])
 *   dx[s]    = sum_k w[d,k] * du[s + (width-1) - k]   (terms with t >= L are 0)
 *   dw[d,k]  = sum_(b,t) du[b,t,d] * x[b, t - (width-1) + k, d]
 *   dbias[d] = sum_(b,t) du[b,t,d]
 * ------------------------------------------------------------------------ */

static double conv_u(const void* x, const float* w, const float* bias, int is_bf16, int64_t b,
                     int64_t t, int64_t d, int64_t L, int64_t Dm, int64_t width) {
  double u = bias ? (double)bias[d] : 0.0;
  for (int64_t k = 0; k < width; ++k) {
    const int64_t s = t - (width - 1) + k;
    if (s < 0) continue;
    u += (double)w[d * width + k] * widen(x, (b * L + s) * Dm + d, is_bf16);
  }
  return u;
}

/* oracle_conv1d_silu -- out (batch, seqlen, dim) fp64. Returns 0 or -1. */
int oracle_conv1d_silu(int64_t batch, int64_t seqlen, int64_t dim, int64_t width, int is_bf16,
                       const void* x, const float* w, const float* bias, int silu_on,
                       double* out) {
  if (batch < 0 || seqlen < 0 || dim < 0 || width < 1 || !x || !w || !out) return -1;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t t = 0; t < seqlen; ++t)
      for (int64_t d = 0; d < dim; ++d) {
        const double u = conv_u(x, w, bias, is_bf16, b, t, d, seqlen, dim, width);
        out[(b * seqlen + t) * dim + d] = silu_on ? silu(u) : u;
      }
  return 0;
}

/* oracle_conv1d_silu_bwd -- dx (batch, seqlen, dim), dw (dim, width), dbias
 * (dim), fp64, overwritten. Returns 0, -1 on bad arguments, -2 without memory. */
int oracle_conv1d_silu_bwd(int64_t batch, int64_t seqlen, int64_t dim, int64_t width,
                           int is_bf16, const void* x, const float* w, const float* bias,
                           int silu_on, const void* dout, double* dx, double* dw,
                           double* dbias) {
  if (batch < 0 || seqlen < 0 || dim < 0 || width < 1 || !x || !w || !dout || !dx || !dw ||
      !dbias)
    return -1;
  double* du = (double*)malloc((size_t)(seqlen > 0 ? seqlen : 1) * sizeof(double));
  if (!du) return -2;
  memset(dw, 0, (size_t)dim * width * sizeof(double));
  memset(dbias, 0, (size_t)dim * sizeof(double));
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t d = 0; d < dim; ++d) {
      for (int64_t t = 0; t < seqlen; ++t) {
        const double g = widen(dout, (b * seqlen + t) * dim + d, is_bf16);
        if (silu_on) {
          const double u = conv_u(x, w, bias, is_bf16, b, t, d, seqlen, dim, width);
          const double sg = sigmoid(u);
          du[t] = g * sg * (1.0 + u * (1.0 - sg));
        } else {
          du[t] = g;
        }
        dbias[d] += du[t];
        for (int64_t k = 0; k < width; ++k) {
          const int64_t s = t - (width - 1) + k;
          if (s >= 0) dw[d * width + k] += du[t] * widen(x, (b * seqlen + s) * dim + d, is_bf16);
        }
      }
      for (int64_t s = 0; s < seqlen; ++s) {
        double acc = 0.0;
        for (int64_t k = 0; k < width; ++k) {
          const int64_t t = s + (width - 1) - k;
          if (t < seqlen) acc += (double)w[d * width + k] * du[t];
        }
        dx[(b * seqlen + s) * dim + d] = acc;
      }
    }
  free(du);
  return 0;
}

/* oracle_conv1d_silu_update -- one decode step of the block's causal conv:
 * state (batch, dim, width-1) holds the last width-1 inputs of each channel,
 * oldest first (zero at the start of a sequence); x (batch, dim) is the new
 * input. out = SiLU(bias + sum_(k < width-1) w[d,k] state[k] + w[d,width-1] x)
 * (or without SiLU), then the state drops its oldest input and appends x.
 * The state is the oracle's own fp64 copy. Returns 0 or -1. */
int oracle_conv1d_silu_update(int64_t batch, int64_t dim, int64_t width, int is_bf16,
                              double* state, const void* x, const float* w, const float* bias,
                              int silu_on, double* out) {
  if (batch < 0 || dim < 0 || width < 1 || !state || !x || !w || !out) return -1;
  const int64_t S = width - 1;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t d = 0; d < dim; ++d) {
      double* st = state + (b * dim + d) * S;
      const double xv = widen(x, b * dim + d, is_bf16);
      double u = bias ? (double)bias[d] : 0.0;
      for (int64_t k = 0; k < S; ++k) u += (double)w[d * width + k] * st[k];
      u += (double)w[d * width + S] * xv;
      out[b * dim + d] = silu_on ? silu(u) : u;
      for (int64_t k = 0; k + 1 < S; ++k) st[k] = st[k + 1];
      if (S > 0) st[S - 1] = xv;
    }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Mamba-2 SSD scan (page "Mamba 논문 리뷰", §4.1 State Space Duality and
 * §4.2: multi-head, larger state). Head h of width P (headdim) has one scalar
 * A[h] and one step Delta[b,t,h]; B and C (N wide) are shared by every head.
 * The state of a head is an N x P matrix, held here as S[p][n]:
 *
 *   Delta      = softplus(dt[b,t,h] + dt_bias[h])   (or without softplus)
 *   S[p][n]    = exp(Delta A[h]) S[p][n] + Delta B[b,t,n] x[b,t,h,p]
 *   y[b,t,h,p] = sum_n C[b,t,n] S[p][n] + D[h] x[b,t,h,p]
 *
 * i.e. §4.1's h_t = A_t h_{t-1} + B_t x_t, y_t = C_t h_t with the scalar
 * A_t = exp(Delta_t A[h]) and the input term Delta_t B_t of §3.3, per head.
 * Layouts: x, y (batch, seqlen, nheads, headdim); dt (batch, seqlen, nheads);
 * B, C (batch, seqlen, dstate); A, D, dt_bias (nheads); h0, h_last
 * (batch, nheads, headdim, dstate). pairs (npairs x 2 int64: b, h) selects
 * the heads computed; y_out is (npairs, seqlen, headdim) and h_last_out
 * (npairs, headdim, dstate), fp64.
 * Returns 0, -1 on bad arguments, -2 without memory.
 */
int oracle_ssd_scan(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                    int64_t dstate, int is_bf16, const void* x, const void* dt, const float* A,
                    const void* Bm, const void* Cm, const float* D, const float* dt_bias,
                    int softplus_on, const float* h0, const int64_t* pairs, int64_t npairs,
                    double* y_out, double* h_last_out) {
  if (batch < 0 || seqlen < 0 || nheads < 0 || headdim < 1 || dstate < 1 || npairs < 0 ||
      !x || !dt || !A || !Bm || !Cm || !pairs || !y_out || !h_last_out)
    return -1;
  const int64_t P = headdim, N = dstate, H = nheads, L = seqlen;
  double* S = (double*)malloc((size_t)(P * N) * sizeof(double));
  if (!S) return -2;
  for (int64_t k = 0; k < npairs; ++k) {
    const int64_t b = pairs[2 * k], h = pairs[2 * k + 1];
    if (b < 0 || b >= batch || h < 0 || h >= H) {
      free(S);
      return -1;
    }
    for (int64_t p = 0; p < P; ++p)
      for (int64_t n = 0; n < N; ++n)
        S[p * N + n] = h0 ? (double)h0[((b * H + h) * P + p) * N + n] : 0.0;
    const double bias = dt_bias ? (double)dt_bias[h] : 0.0;
    const double Dh = D ? (double)D[h] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
      const double v = widen(dt, (b * L + t) * H + h, is_bf16) + bias;
      const double delta = softplus_on ? softplus(v) : v;
      const double a = exp(delta * (double)A[h]);
      for (int64_t p = 0; p < P; ++p) {
        const double xv = widen(x, ((b * L + t) * H + h) * P + p, is_bf16);
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          const double bn = widen(Bm, (b * L + t) * N + n, is_bf16);
          S[p * N + n] = a * S[p * N + n] + delta * bn * xv;
          acc += widen(Cm, (b * L + t) * N + n, is_bf16) * S[p * N + n];
        }
        y_out[(k * L + t) * P + p] = acc + Dh * xv;
      }
    }
    memcpy(h_last_out + k * P * N, S, (size_t)(P * N) * sizeof(double));
  }
  free(S);
  return 0;
}

/* oracle_ssd_state_update -- one decode step of the multi-head SSD: the
 * recurrent side of §4.1's duality (state update, O(1) per token), on the
 * oracle's own fp64 state (batch, nheads, headdim, dstate), in place.
 * x (batch, nheads, headdim), dt (batch, nheads), B, C (batch, dstate) in the
 * io type; A, D, dt_bias (nheads) fp32 (D, dt_bias nullable); y (batch,
 * nheads, headdim) fp64. Same arithmetic as one step of oracle_ssd_scan.
 * Returns 0 or -1. */
int oracle_ssd_state_update(int64_t batch, int64_t nheads, int64_t headdim, int64_t dstate,
                            int is_bf16, double* state, const void* x, const void* dt,
                            const float* A, const void* Bm, const void* Cm, const float* D,
                            const float* dt_bias, int softplus_on, double* y) {
  if (batch < 0 || nheads < 0 || headdim < 1 || dstate < 1 || !state || !x || !dt || !A ||
      !Bm || !Cm || !y)
    return -1;
  const int64_t H = nheads, P = headdim, N = dstate;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t h = 0; h < H; ++h) {
      const double v = widen(dt, b * H + h, is_bf16) + (dt_bias ? (double)dt_bias[h] : 0.0);
      const double delta = softplus_on ? softplus(v) : v;
      const double a = exp(delta * (double)A[h]);
      for (int64_t p = 0; p < P; ++p) {
        const double xv = widen(x, (b * H + h) * P + p, is_bf16);
        double* S = state + ((b * H + h) * P + p) * N;
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          S[n] = a * S[n] + delta * widen(Bm, b * N + n, is_bf16) * xv;
          acc += widen(Cm, b * N + n, is_bf16) * S[n];
        }
        y[(b * H + h) * P + p] = acc + (D ? (double)D[h] : 0.0) * xv;
      }
    }
  return 0;
}
