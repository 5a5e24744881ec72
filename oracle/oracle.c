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
                              int64_t num_seqs) {
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
          for (int64_t n = 0; n < dstate; ++n) hp[n] = 0.0;
      }
      const double dt = step_size(drow[t], bias, delta_softplus);
      const double ut = urow[t];
      double acc = 0.0;
      for (int64_t n = 0; n < dstate; ++n) {
        /* [euler]: Abar = exp(Delta A[d,n]), Bbar u = Delta B_t[n] u_t. */
        const double abar = exp(dt * A[d * dstate + n]);
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

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
