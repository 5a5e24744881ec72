/*
 * ssd.h -- C ABI of the Mamba-2 (SSD) chunked scan in libsss48.so.
 *
 * What it computes.  The selective scan of selective_scan.h with A
 * restricted to one scalar per head times the identity ("Mamba is attention
 * all you really need, part 2", section "The evolution"): the headdim
 * channels p of head h share its step Delta_t and its scalar A[h], and the
 * nheads / ngroups consecutive heads of group g share B and C.  For every
 * batch row b, head h (group g = h / (nheads / ngroups)), channel p and
 * state n:
 *
 *   Delta_t   = softplus(dt[b,t,h] + dt_bias[h])            (softplus optional)
 *   h_t[p,n]  = exp(Delta_t A[h]) h_{t-1}[p,n] + Delta_t B[b,t,g,n] x[b,t,h,p]
 *   y[b,t,h,p]= (sum_n C[b,t,g,n] h_t[p,n] + D[h] x[b,t,h,p]) * silu(z[b,t,h,p])
 *
 * with h_{-1} = h0 (or 0) and the gate omitted when z is NULL.
 *
 * How.  "State Space Models and the Post-Transformer Era", section "Mamba-2
 * and Structured State Space Duality", and "The State That Must Remember
 * Everything", Part 4: the same map is attention under a 1-semiseparable
 * causal mask, so it can be evaluated blockwise by matrix products.  The
 * sequence is cut into chunks of 128 steps; per chunk and head, on the
 * tensor cores (bf16 operands, fp32 accumulation):
 *   scores   S = C B^T                             (128 x 128, K = dstate)
 *   diagonal Y = (S o decay mask o Delta) X        (K = 128 steps)
 *   carry    Y += diag(exp(cum_t)) C h_prev        (K = dstate)
 *   state    h = exp(cum_last) h_prev + B^T (w o X)  (K = 128 steps)
 * where cum_t is the running sum of Delta A inside the chunk.  The carried
 * state stays in fp32 on chip for the whole sequence; the mask, h_prev and
 * w o X enter their products rounded to bf16, so y matches the fp64
 * recurrence to about bf16 precision (a relative error of a few 1e-3 of
 * max |y|), not to fp32 precision.
 *
 * Layouts (row-major, dense, token-major as the chunked products read them):
 *   x, z, y          (batch, seqlen, nheads, headdim)   in_dtype (y: out_dtype)
 *   dt               (batch, seqlen, nheads)            in_dtype
 *   B, C             (batch, seqlen, ngroups, dstate)   in_dtype
 *   A, D, dt_bias    (nheads)                           fp32 (D, dt_bias optional)
 *   h0, last_state   (batch, nheads, headdim, dstate)   fp32, optional
 * A[h] is expected to be <= 0 (a decaying state, as in Mamba-2): the
 * kernel factors the decay between two steps into per-row and per-column
 * factors that stay below 1 only for A <= 0.
 * Supported here: in_dtype MSS_BF16, headdim 64, dstate 128 (other valid
 * sizes return MSS_ERR_UNSUPPORTED).  x, B, C, z and y must be 16-byte
 * aligned, dt 2-byte aligned (its bf16 elements), and the fp32 pointers
 * (A, D, dt_bias, h0, last_state) 4-byte aligned.  Outputs must not
 * overlap inputs.
 *
 * Ownership and streams as in selective_scan.h: device pointers owned by
 * the caller, nothing allocated, work enqueued on `stream` (a cudaStream_t
 * as void*, NULL = legacy default stream) without synchronising.
 *
 * Schedule.  One CTA per (batch row, head) sequence, one CTA per SM, so
 * the sequences run in waves.  When the last wave is at most half full
 * (r = batch * nheads mod the SM count, 0 < 2 r <= the SM count), at least
 * one wave is full and the sequence has at least two chunks, the last r
 * sequences are cut at chunk boundaries into min(round(SMs / r), full
 * waves + 1, chunks, 8) pieces, and the pieces are spread over the
 * schedule between the whole sequences, so the last wave runs short
 * pieces.  Each piece starts from the end state of the piece before (fp32,
 * in the workspace); the output is bit-identical to the uncut schedule.
 * Cutting needs the workspace below (mss_ssd_workspace_size() bytes);
 * without one (workspace NULL) every sequence runs whole.
 *
 * Errors.  Argument errors return MSS_ERR_INVALID_ARG / MSS_ERR_UNSUPPORTED
 * and enqueue nothing; a failed launch returns MSS_ERR_CUDA.  The kernel's
 * waits are bounded (spin_timeout_ns, 0 = 2 s); one that runs out records
 * MSS_ERR_TIMEOUT in a library status word read (and cleared) by
 * mss_ssd_status().
 */
#ifndef SSS48_SSD_H
#define SSS48_SSD_H

#include <stdint.h>

#include "selective_scan.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mss_ssd_args {
  int64_t batch;
  int64_t seqlen;
  int64_t nheads;
  int64_t headdim; /* 64 */
  int64_t ngroups; /* divides nheads */
  int64_t dstate;  /* 128 */
  mss_dtype in_dtype;
  mss_dtype out_dtype;
  const void *x;
  const void *dt;
  const float *A;
  const void *B;
  const void *C;
  const float *D;       /* NULL: no skip term */
  const void *z;        /* NULL: no gate */
  const float *dt_bias; /* NULL: 0 */
  int dt_softplus;
  const float *h0;      /* NULL: the state starts at 0 */
  void *y;
  float *last_state;    /* NULL: not written */
  uint64_t spin_timeout_ns;
  /* NULL (every sequence runs whole), or device memory of at least
     mss_ssd_workspace_size() bytes, 16-byte aligned, not shared with a call
     in flight: a work-item counter and flags (cleared by cudaMemsetAsync on
     `stream` at every call) and the end states of the pieces.
     Smaller than required: MSS_ERR_WORKSPACE. */
  void *workspace;
  size_t workspace_bytes;
} mss_ssd_args;

/* Workspace bytes that let mamba2_ssd_fwd cut the last wave's sequences
 * into pieces on the current device (0 when its schedule cuts nothing).  Reads only
 * batch, nheads and seqlen, and the current device's SM count. */
mss_status mss_ssd_workspace_size(const mss_ssd_args *args, size_t *bytes);

/* Chunked SSD forward: y (and last_state) for the arguments above. */
mss_status mamba2_ssd_fwd(const mss_ssd_args *args, void *stream);

/* Synchronises `stream` and returns the SSD kernels' device status word
 * (MSS_OK or MSS_ERR_TIMEOUT), clearing it.  The word is the library's own
 * (one per device): it covers every SSD call on this device that has
 * completed since the previous read.  Only `stream` is synchronised, so a
 * call still running on another stream is covered only once it has
 * completed (synchronise that stream, or the device, first); such a call
 * can also record its status after this read. */
mss_status mss_ssd_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SSS48_SSD_H */
