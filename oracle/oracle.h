/*
 * oracle.h -- fp64 CPU reference of the selective scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this code: only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py use it.  It shares no header, helper, table or
 * constant with the CUDA library and imports nothing from it.
 *
 * Every function computes the plain definition, in the order the sources
 * state it, in double precision.  Layouts (all row-major, contiguous):
 *   u, delta, z, y        (batch, dim, seqlen)
 *   B, C                  (batch, dstate, seqlen)   shared by all channels
 *   A                     (dim, dstate)
 *   D, delta_bias         (dim)
 *   h0, last_state        (batch, dim, dstate)
 * Optional pointers may be NULL (D, z, delta_bias, h0 -> treated as 0 /
 * "no gate"; last_state -> not written).
 */
#ifndef SSS48_ORACLE_H
#define SSS48_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Composition of two fade-and-add steps, "step 1 then step 2":
 * (a1, b1) then (a2, b2) = (a1*a2, a2*b1 + b2).
 * Page "Mamba is attention... part 2", section "The relay". */
void oracle_combine_f64(double a1, double b1, double a2, double b2,
                        double *a_out, double *b_out);

/* softplus(x) = log(1 + exp(x)), evaluated as max(x,0) + log1p(exp(-|x|)). */
double oracle_softplus_f64(double x);

/* silu(z) = z / (1 + exp(-z)). */
double oracle_silu_f64(double z);

/* Full selective scan, sequential over t (the recurrence as defined):
 *   Delta_t = softplus(delta_t + delta_bias[d])   (or delta_t + delta_bias[d]
 *                                                    when delta_softplus == 0)
 *   h_t[n]  = exp(Delta_t * A[d,n]) * h_{t-1}[n] + Delta_t * B_t[n] * u_t
 *   y_t     = sum_n C_t[n] * h_t[n] + D[d] * u_t
 *   y_t    *= silu(z_t)                            (when z != NULL)
 * with h_{-1} = h0 (or 0).  Packed sequences: when cu_seqlens is not NULL
 * (num_seqs + 1 increasing offsets, 0 ... seqlen, the same for every batch
 * row), h is set to 0 before every step t = cu_seqlens[i], 0 < i < num_seqs,
 * so each row holds num_seqs independent scans; h0 seeds the first and
 * last_state is the end of the last.  With trapezoid != 0 the update is the
 * three-term trapezoidal form
 *   h_t = a h_{t-1} + Delta_t / 2 * (a B_{t-1}[n] u_{t-1} + B_t[n] u_t),
 *   a = exp(Delta_t A[d,n]), no previous term at t = 0 or at a restart.
 * Returns 0, or -1 on a bad size. */
int oracle_selective_scan_f64(int64_t batch, int64_t dim, int64_t dstate,
                              int64_t seqlen, const double *u,
                              const double *delta, const double *A,
                              const double *B, const double *C,
                              const double *D, const double *z,
                              const double *delta_bias, int delta_softplus,
                              const double *h0, double *y,
                              double *last_state, const int32_t *cu_seqlens,
                              int64_t num_seqs, int trapezoid);

/* One decode step (the same recurrence for a single t), state updated in
 * place.  x, dt, z, y: (batch, dim); B, C: (batch, dstate);
 * state: (batch, dim, dstate).  Returns 0, or -1 on a bad size. */
int oracle_selective_state_update_f64(int64_t batch, int64_t dim,
                                      int64_t dstate, double *state,
                                      const double *x, const double *dt,
                                      const double *A, const double *B,
                                      const double *C, const double *D,
                                      const double *z, const double *dt_bias,
                                      int dt_softplus, double *y);

/* Gradient of the selective scan above (Euler update; packed sequences as
 * there, cu_seqlens NULL for none) for the loss
 * sum(dy * y) + sum(d_last * last_state): du, ddelta, dz (batch, dim,
 * seqlen), dA (dim, dstate), dB, dC (batch, dstate, seqlen), dD,
 * ddelta_bias (dim), dh0 (batch, dim, dstate).  d_last, dz, dD,
 * ddelta_bias and dh0 may be NULL.  Returns 0, or -1 on a bad size or an
 * allocation failure. */
int oracle_selective_scan_bwd_f64(
    int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
    const double *u, const double *delta, const double *A, const double *B,
    const double *C, const double *D, const double *z,
    const double *delta_bias, int delta_softplus, const double *h0,
    const double *dy, const double *d_last, double *du, double *ddelta,
    double *dA, double *dB, double *dC, double *dD, double *dz,
    double *ddelta_bias, double *dh0, const int32_t *cu_seqlens,
    int64_t num_seqs);

/* Mamba-2 (SSD): the same recurrence with A restricted to a scalar times
 * the identity per head, sequential over t.  headdim channels of a head
 * share its step Delta_t and its scalar A[h]; ngroups groups of B, C are
 * shared by nheads / ngroups consecutive heads each.  Token-major layouts:
 *   x, z, y            (batch, seqlen, nheads, headdim)
 *   dt                 (batch, seqlen, nheads)
 *   A, D, dt_bias      (nheads)
 *   B, C               (batch, seqlen, ngroups, dstate)
 *   h0, last_state     (batch, nheads, headdim, dstate)
 * For head h (group g = h / (nheads / ngroups)) and channel p:
 *   Delta_t   = softplus(dt_t + dt_bias[h])  (or dt_t + dt_bias[h])
 *   h_t[p,n]  = exp(Delta_t A[h]) h_{t-1}[p,n] + Delta_t B_t[g,n] x_t[p]
 *   y_t[p]    = sum_n C_t[g,n] h_t[p,n] + D[h] x_t[p],  times silu(z_t[p])
 * Returns 0, or -1 on a bad size. */
int oracle_ssd_scan_f64(int64_t batch, int64_t seqlen, int64_t nheads,
                        int64_t headdim, int64_t ngroups, int64_t dstate,
                        const double *x, const double *dt, const double *A,
                        const double *B, const double *C, const double *D,
                        const double *z, const double *dt_bias, int dt_softplus,
                        const double *h0, double *y, double *last_state);

/* Number of OpenMP threads the scan uses (1 when built without OpenMP). */
int oracle_num_threads(void);

/* Sets the number of OpenMP threads later calls use (n >= 1; for timing
 * the oracle on one core).  No effect when built without OpenMP. */
void oracle_set_num_threads(int n);

#ifdef __cplusplus
}
#endif

#endif
