/*
 * oracle.c -- fp64 CPU reference of the selective scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py, never by the product path.  It shares no code
 * with the CUDA library.
 *
 * Sources (web pages on Mamba and state space models):
 *  [relay]  "Mamba is attention all you really need, part 2", section
 *           "The relay": two fade-and-add steps compose as
 *           (a1,b1) then (a2,b2) = (a1 a2, a2 b1 + b2); worked example
 *           (0.6,0.4) then (0.5,1.0) = (0.3,1.2).
 *  [eq]     "The State That Must Remember Everything", Part 2, "The
 *           Equation": x'(t) = A x + B u, y = C x + D u, discretised with
 *           step Delta to h_t = Abar h_{t-1} + Bbar u_t, y_t = C h_t
 *           (the readout uses the state after the update).
 *  [euler]  same page, Part 7: Mamba-1 corresponds to an exponential-Euler
 *           discretisation, i.e. Abar = exp(Delta A), Bbar = Delta B.
 *  [select] "State Space Models and the Post-Transformer Era", section
 *           "The Selection Mechanism": Delta, B and C are per-token inputs.
 *  [trap]   "The State That Must Remember Everything", Part 7: Mamba-3
 *           replaces the Euler step by a trapezoidal one with three terms,
 *           h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1} + gamma_t B_t x_t
 *           (alpha, beta, gamma not given there; read as the trapezoidal
 *           rule for the same ODE: alpha = exp(Delta A), beta = alpha
 *           Delta / 2, gamma = Delta / 2, no previous input at t = 0).
 *  [ssd]    "Mamba is attention all you really need, part 2", section
 *           "The evolution", and "State Space Models and the Post-Transformer
 *           Era", section "Mamba-2 and Structured State Space Duality":
 *           Mamba-2 restricts A to one number times the identity; the result
 *           is the same sequence map as attention under a 1-semiseparable
 *           causal mask, computable by the linear scan or by the quadratic
 *           matrix form.  Read here as: the channels of a head share Delta
 *           and the scalar A (so a head's channels form the matrix that the
 *           blockwise form multiplies), B and C are shared per group.
 *  The step-size nonlinearity Delta = softplus(delta + delta_bias) and the
 *  output gate y * silu(z) are not written out on the pages; this library
 *  uses the standard Mamba parameterisation for both.
 *
 * Parity of every function here is pinned by tests that do not re-use this
 * code: the page's worked example, brute-force unrolled sums, the LTI
 * convolution form, the N=1 gate closed form, Delta limits and special cases.
 */
#include "oracle.h"

#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

void oracle_combine_f64(double a1, double b1, double a2, double b2,
                        double *a_out, double *b_out) {
  /* [relay]: applying h -> a1 h + b1 and then h -> a2 h + b2 gives
   * h -> a2 (a1 h + b1) + b2 = (a1 a2) h + (a2 b1 + b2). */
  *a_out = a1 * a2;
  *b_out = a2 * b1 + b2;
}

double oracle_softplus_f64(double x) {
  /* log(1 + e^x) without overflow: max(x,0) + log1p(e^{-|x|}). */
  double ax = fabs(x);
  return (x > 0.0 ? x : 0.0) + log1p(exp(-ax));
}

double oracle_silu_f64(double z) {
  /* z * sigmoid(z) = z / (1 + e^{-z}). */
  return z / (1.0 + exp(-z));
}

static double step_size(double delta, double bias, int softplus) {
  /* [select]: Delta is the token's own step; softplus keeps it positive. */
  double x = delta + bias;
  return softplus ? oracle_softplus_f64(x) : x;
}

int oracle_selective_scan_f64(int64_t batch, int64_t dim, int64_t dstate,
                              int64_t seqlen, const double *u,
                              const double *delta, const double *A,
                              const double *B, const double *C,
                              const double *D, const double *z,
                              const double *delta_bias, int delta_softplus,
                              const double *h0, double *y,
                              double *last_state, const int32_t *cu_seqlens,
                              int64_t num_seqs, int trapezoid) {
  /* the per-channel state lives on the stack; 256 states is far above any
   * size the tests or the bench use */
  if (batch < 0 || dim < 0 || dstate < 1 || dstate > 256 || seqlen < 0)
    return -1;
  if (cu_seqlens && num_seqs < 1) return -1;
  const int64_t channels = batch * dim;

  /* Channels (b, d) are independent recurrences; OpenMP only distributes
   * them over cores.  Within a channel the loop over t is sequential. */
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t ch = 0; ch < channels; ++ch) {
    const int64_t b = ch / dim;
    const int64_t d = ch % dim;
    double hp[256];
    /* trapezoidal rule: B_{t-1}[n] u_{t-1}, 0 before the first step */
    double wprev[256];
    for (int64_t n = 0; n < dstate; ++n) wprev[n] = 0.0;
    /* h_{-1} = h0, or 0 ([eq]: the state starts empty). */
    for (int64_t n = 0; n < dstate; ++n)
      hp[n] = h0 ? h0[(b * dim + d) * dstate + n] : 0.0;

    const double bias = delta_bias ? delta_bias[d] : 0.0;
    const double dskip = D ? D[d] : 0.0;
    const double *urow = u + (b * dim + d) * seqlen;
    const double *drow = delta + (b * dim + d) * seqlen;
    const double *zrow = z ? z + (b * dim + d) * seqlen : NULL;
    double *yrow = y + (b * dim + d) * seqlen;
    const double *Bb = B + b * dstate * seqlen;
    const double *Cb = C + b * dstate * seqlen;

    int64_t next = 1; /* index of the next interior sequence start */
    for (int64_t t = 0; t < seqlen; ++t) {
      /* Packed independent sequences: the state starts empty again at every
       * interior start cu_seqlens[i], 0 < i < num_seqs. */
      if (cu_seqlens) {
        while (next < num_seqs && cu_seqlens[next] < t) ++next;
        if (next < num_seqs && cu_seqlens[next] == t)
          for (int64_t n = 0; n < dstate; ++n) hp[n] = wprev[n] = 0.0;
      }
      const double dt = step_size(drow[t], bias, delta_softplus);
      const double ut = urow[t];
      double acc = 0.0;
      for (int64_t n = 0; n < dstate; ++n) {
        /* [euler]: Abar = exp(Delta A[d,n]), Bbar u = Delta B_t[n] u_t. */
        const double abar = exp(dt * A[d * dstate + n]);
        if (trapezoid) {
          /* [trap]: three terms, the previous input decayed over the step
           * and the current one, weighted by half a step each. */
          const double w = Bb[n * seqlen + t] * ut;
          hp[n] = abar * hp[n] + 0.5 * dt * (abar * wprev[n] + w);
          wprev[n] = w;
          acc += Cb[n * seqlen + t] * hp[n];
          continue;
        }
        const double bbar_u = dt * Bb[n * seqlen + t] * ut;
        /* [eq]: h_t = Abar h_{t-1} + Bbar u_t. */
        hp[n] = abar * hp[n] + bbar_u;
        /* [eq]: y_t = C_t h_t, with the state after the update. */
        acc += Cb[n * seqlen + t] * hp[n];
      }
      /* [eq]: the D u skip term of y = C x + D u. */
      double yt = acc + dskip * ut;
      if (zrow) yt *= oracle_silu_f64(zrow[t]);
      yrow[t] = yt;
    }
    if (last_state)
      for (int64_t n = 0; n < dstate; ++n)
        last_state[(b * dim + d) * dstate + n] = hp[n];
  }
  return 0;
}

int oracle_selective_state_update_f64(int64_t batch, int64_t dim,
                                      int64_t dstate, double *state,
                                      const double *x, const double *dt,
                                      const double *A, const double *B,
                                      const double *C, const double *D,
                                      const double *z, const double *dt_bias,
                                      int dt_softplus, double *y) {
  /* One step of the same recurrence: a new token is a state update
   * ("Mamba: The State Space Models Challenging the Transformer", section
   * "What a state space model actually is"). */
  if (batch < 0 || dim < 0 || dstate < 1) return -1;
  for (int64_t b = 0; b < batch; ++b) {
    for (int64_t d = 0; d < dim; ++d) {
      const int64_t ch = b * dim + d;
      const double step = step_size(dt[ch], dt_bias ? dt_bias[d] : 0.0,
                                    dt_softplus);
      double acc = 0.0;
      for (int64_t n = 0; n < dstate; ++n) {
        double *hn = &state[ch * dstate + n];
        *hn = exp(step * A[d * dstate + n]) * (*hn) +
              step * B[b * dstate + n] * x[ch];
        acc += C[b * dstate + n] * (*hn);
      }
      double yt = acc + (D ? D[d] : 0.0) * x[ch];
      if (z) yt *= oracle_silu_f64(z[ch]);
      y[ch] = yt;
    }
  }
  return 0;
}

/* Gradient of the full selective scan by the chain rule, sequential over t
 * (reverse-time adjoint).  The backward pass recomputes the states it needs
 * from the inputs instead of receiving them from the forward pass ("Mamba
 * is attention all you really need, part 2", section "Keeping the pad on
 * the desk"; "The State That Must Remember Everything", Part 3, "The
 * Hardware-Aware Way Out", rematerialisation).  Here the recomputation is
 * simply a forward sweep that keeps every state of one channel.
 *
 * Loss: sum(dy * y) + sum(d_last * last_state).  With s_t = sum_n C_t[n]
 * h_t[n] + D u_t, g_t = silu(z_t) (1 without z), y_t = s_t g_t:
 *   lam_t[n] = ds_t C_t[n] + exp(Delta_{t+1} A[n]) lam_{t+1}[n],
 *              lam_{L-1} starting from d_last,        ds_t = dy_t g_t
 *   dDelta_t = sum_n lam_t[n] (A[n] a_t[n] h_{t-1}[n] + B_t[n] u_t)
 *   dA[d,n] += lam_t[n] Delta_t a_t[n] h_{t-1}[n]
 *   dB_t[n] += lam_t[n] Delta_t u_t        dC_t[n] += ds_t h_t[n]
 *   du_t     = ds_t D + sum_n lam_t[n] Delta_t B_t[n]
 *   dD      += ds_t u_t                     dz_t = dy_t s_t silu'(z_t)
 *   ddelta_t = dDelta_t sigmoid(delta_t + bias)   (dDelta_t without softplus)
 *   dbias   += ddelta_t                     dh0 = a_0 lam_0
 * dB, dC sum over channels, dA, dD, dbias over batch rows.  Every output
 * is overwritten (not accumulated into).  Returns 0, or -1 on a bad size
 * or allocation failure. */
static double dsilu(double z) {
  const double sg = 1.0 / (1.0 + exp(-z));
  return sg * (1.0 + z * (1.0 - sg));
}

int oracle_selective_scan_bwd_f64(
    int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
    const double *u, const double *delta, const double *A, const double *B,
    const double *C, const double *D, const double *z,
    const double *delta_bias, int delta_softplus, const double *h0,
    const double *dy, const double *d_last, double *du, double *ddelta,
    double *dA, double *dB, double *dC, double *dD, double *dz,
    double *ddelta_bias, double *dh0, const int32_t *cu_seqlens,
    int64_t num_seqs) {
  if (batch < 0 || dim < 0 || dstate < 1 || dstate > 256 || seqlen < 0)
    return -1;
  if (cu_seqlens && num_seqs < 1) return -1;
  const int64_t N = dstate, L = seqlen;
  /* Packed sequences: step t starts a sequence (the state before it is
   * empty, as in the forward oracle) when t is an interior start
   * cu_seqlens[i], 0 < i < num_seqs. */
  char *starts = calloc((size_t)(L + 1), 1);
  if (!starts) return -1;
  if (cu_seqlens)
    for (int64_t i = 1; i < num_seqs; ++i)
      if (cu_seqlens[i] >= 0 && cu_seqlens[i] < L) starts[cu_seqlens[i]] = 1;
  /* per batch row partial sums of the per-channel parameter gradients */
  double *pA = calloc((size_t)(batch * dim * N + 1), sizeof(double));
  double *pD = calloc((size_t)(batch * dim + 1), sizeof(double));
  double *pb = calloc((size_t)(batch * dim + 1), sizeof(double));
  if (!pA || !pD || !pb) {
    free(pA); free(pD); free(pb); free(starts);
    return -1;
  }
  memset(dB, 0, sizeof(double) * (size_t)(batch * N * L));
  memset(dC, 0, sizeof(double) * (size_t)(batch * N * L));
  int failed = 0;

  /* Batch rows own disjoint dB, dC slices, so they run in parallel; the
   * channels of one row are visited in order. */
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t b = 0; b < batch; ++b) {
    double *H = malloc(sizeof(double) * (size_t)((L + 1) * N));
    double *S = malloc(sizeof(double) * (size_t)(L + 1));
    double *Dt = malloc(sizeof(double) * (size_t)(L + 1));
    if (!H || !S || !Dt) {
      free(H); free(S); free(Dt);
#ifdef _OPENMP
#pragma omp atomic write
#endif
      failed = 1;
      continue;
    }
    const double *Bb = B + b * N * L, *Cb = C + b * N * L;
    double *dBb = dB + b * N * L, *dCb = dC + b * N * L;
    for (int64_t d = 0; d < dim; ++d) {
      const int64_t row = (b * dim + d) * L;
      const double bias = delta_bias ? delta_bias[d] : 0.0;
      const double dskip = D ? D[d] : 0.0;
      /* forward sweep keeping every state: H[t + 1] = h_t, H[0] = h_{-1} */
      for (int64_t n = 0; n < N; ++n)
        H[n] = h0 ? h0[(b * dim + d) * N + n] : 0.0;
      for (int64_t t = 0; t < L; ++t) {
        const double dt = step_size(delta[row + t], bias, delta_softplus);
        Dt[t] = dt;
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          /* the state entering step t: h_{t-1}, or empty at a start */
          const double hin = starts[t] ? 0.0 : H[t * N + n];
          const double h = exp(dt * A[d * N + n]) * hin +
                           dt * Bb[n * L + t] * u[row + t];
          H[(t + 1) * N + n] = h;
          acc += Cb[n * L + t] * h;
        }
        S[t] = acc + dskip * u[row + t];
      }
      /* reverse sweep */
      double lam[256];
      for (int64_t n = 0; n < N; ++n)
        lam[n] = d_last ? d_last[(b * dim + d) * N + n] : 0.0;
      double accD = 0.0, accb = 0.0;
      for (int64_t t = L - 1; t >= 0; --t) {
        const double ut = u[row + t], dt = Dt[t];
        const double g = z ? oracle_silu_f64(z[row + t]) : 1.0;
        const double ds = dy[row + t] * g;
        if (z && dz) dz[row + t] = dy[row + t] * S[t] * dsilu(z[row + t]);
        accD += ds * ut;
        double dut = ds * dskip, dDelta = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          const double an = A[d * N + n];
          /* at a start nothing flows back from step t to h_{t-1} (every
           * use of hprev below is multiplied by a) */
          const double a = starts[t] ? 0.0 : exp(dt * an);
          const double hprev = H[t * N + n];
          lam[n] += ds * Cb[n * L + t];
          dCb[n * L + t] += ds * H[(t + 1) * N + n];
          dDelta += lam[n] * (an * a * hprev + Bb[n * L + t] * ut);
          pA[(b * dim + d) * N + n] += lam[n] * dt * a * hprev;
          dBb[n * L + t] += lam[n] * dt * ut;
          dut += lam[n] * dt * Bb[n * L + t];
          lam[n] *= a;
        }
        du[row + t] = dut;
        const double x = delta[row + t] + bias;
        const double dd = delta_softplus ? dDelta / (1.0 + exp(-x)) : dDelta;
        ddelta[row + t] = dd;
        accb += dd;
      }
      if (dh0)
        for (int64_t n = 0; n < N; ++n) dh0[(b * dim + d) * N + n] = lam[n];
      pD[b * dim + d] = accD;
      pb[b * dim + d] = accb;
    }
    free(H); free(S); free(Dt);
  }
  if (!failed) {
    for (int64_t d = 0; d < dim; ++d) {
      double sD = 0.0, sb = 0.0;
      for (int64_t b = 0; b < batch; ++b) {
        sD += pD[b * dim + d];
        sb += pb[b * dim + d];
      }
      if (dD) dD[d] = sD;
      if (ddelta_bias) ddelta_bias[d] = sb;
      for (int64_t n = 0; n < N; ++n) {
        double s = 0.0;
        for (int64_t b = 0; b < batch; ++b) s += pA[(b * dim + d) * N + n];
        dA[d * N + n] = s;
      }
    }
  }
  free(pA); free(pD); free(pb); free(starts);
  return failed ? -1 : 0;
}

int oracle_ssd_scan_f64(int64_t batch, int64_t seqlen, int64_t nheads,
                        int64_t headdim, int64_t ngroups, int64_t dstate,
                        const double *x, const double *dt, const double *A,
                        const double *B, const double *C, const double *D,
                        const double *z, const double *dt_bias, int dt_softplus,
                        const double *h0, double *y, double *last_state) {
  if (batch < 0 || seqlen < 0 || nheads < 1 || headdim < 1 || ngroups < 1 ||
      dstate < 1 || nheads % ngroups != 0)
    return -1;
  const int64_t heads_per_group = nheads / ngroups;
  int failed = 0;
  /* (b, h) pairs are independent; OpenMP only distributes them. */
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t bh = 0; bh < batch * nheads; ++bh) {
    const int64_t b = bh / nheads;
    const int64_t h = bh % nheads;
    const int64_t g = h / heads_per_group;
    /* [ssd]: the state of one head is a headdim x dstate matrix. */
    double *S = (double *)malloc(sizeof(double) * headdim * dstate);
    if (!S) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      failed = 1;
      continue;
    }
    for (int64_t p = 0; p < headdim; ++p)
      for (int64_t n = 0; n < dstate; ++n)
        S[p * dstate + n] = h0 ? h0[((b * nheads + h) * headdim + p) * dstate + n] : 0.0;
    const double bias = dt_bias ? dt_bias[h] : 0.0;
    const double dskip = D ? D[h] : 0.0;
    for (int64_t t = 0; t < seqlen; ++t) {
      const double step = step_size(dt[(b * seqlen + t) * nheads + h], bias, dt_softplus);
      /* [ssd] + [euler]: one fade exp(Delta A[h]) for every state entry. */
      const double fade = exp(step * A[h]);
      const double *Bt = B + ((b * seqlen + t) * ngroups + g) * dstate;
      const double *Ct = C + ((b * seqlen + t) * ngroups + g) * dstate;
      const int64_t row = ((b * seqlen + t) * nheads + h) * headdim;
      for (int64_t p = 0; p < headdim; ++p) {
        const double xp = x[row + p];
        double acc = 0.0;
        for (int64_t n = 0; n < dstate; ++n) {
          /* [eq]: h_t = Abar h_{t-1} + Bbar x_t, per channel p. */
          S[p * dstate + n] = fade * S[p * dstate + n] + step * Bt[n] * xp;
          /* [eq]: read out with the state after the update. */
          acc += Ct[n] * S[p * dstate + n];
        }
        double yp = acc + dskip * xp;
        if (z) yp *= oracle_silu_f64(z[row + p]);
        y[row + p] = yp;
      }
    }
    if (last_state)
      memcpy(last_state + (b * nheads + h) * headdim * dstate, S,
             sizeof(double) * headdim * dstate);
    free(S);
  }
  return failed ? -1 : 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
