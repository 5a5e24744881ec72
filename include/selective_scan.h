/*
 * selective_scan.h -- C ABI of the B200 selective-scan (S6) library
 * (libsss48.so).
 *
 * What it computes.  For every batch row b, channel d in [0, dim) and state
 * n in [0, dstate), over time t in [0, seqlen):
 *
 *   Delta_t = softplus(delta[b,d,t] + delta_bias[d])      (softplus optional)
 *   h_t[n]  = exp(Delta_t * A[d,n]) * h_{t-1}[n] + Delta_t * B[b,n,t] * u[b,d,t]
 *   y[b,d,t]= (sum_n C[b,n,t] * h_t[n] + D[d] * u[b,d,t]) * silu(z[b,d,t])
 *
 * with h_{-1} = h0 (or 0), silu(z) = z / (1 + e^-z), and the gate omitted
 * when z is NULL.  Sources, by page and section:
 *  - the recurrence and readout h_t = Abar h_{t-1} + Bbar u_t, y = C h + D u:
 *    "The State That Must Remember Everything", Part 2, "The Equation";
 *  - Abar = exp(Delta A), Bbar = Delta B (exponential-Euler discretisation):
 *    same page, Part 7 "Mamba-3";
 *  - Delta, B, C chosen per token: "State Space Models and the
 *    Post-Transformer Era", section "The Selection Mechanism";
 *  - the scan over time by composing fade-and-add pairs
 *    (a1,b1) then (a2,b2) = (a1 a2, a2 b1 + b2): "Mamba is attention all you
 *    really need, part 2", section "The relay";
 *  - discretisation, scan and readout in one kernel, the state kept on chip
 *    and only y written back: same page, "Keeping the pad on the desk", and
 *    "The State That Must Remember Everything", "The Hardware-Aware Way Out";
 *  - decode as a single state update: "Mamba: The State Space Models
 *    Challenging the Transformer", section "What a state space model
 *    actually is".
 * The softplus step size, delta_bias and the silu(z) gate are not written
 * out on the pages; they follow the standard Mamba parameterisation.
 *
 * Memory and ownership.  Every pointer is a device pointer owned by the
 * caller.  The library never allocates or frees device or host memory.
 * Tensors are row-major (C order) with the shapes given below; the scan's
 * (batch, rows, seqlen) tensors may carry their own batch and row strides
 * (mss_scan_args.stride_*), everything else is dense.
 * Work is enqueued on the caller's stream (a cudaStream_t passed as void*,
 * NULL = legacy default stream) and is never synchronised, except in
 * mss_scan_status().
 *
 * Errors.  Argument checks happen before any launch; a failing check returns
 * MSS_ERR_INVALID_ARG or MSS_ERR_UNSUPPORTED and enqueues nothing.  A CUDA
 * launch error returns MSS_ERR_CUDA.  Errors detected on the device (a
 * bounded wait that ran out) are written to a status word, inside the
 * workspace for a scan split into chunks and in the library's own device
 * memory otherwise, and reported by mss_scan_status().
 *
 * Besides the scan above, the library offers packed sequences, strided
 * views, the three-term trapezoidal update and state checkpoints (fields of
 * mss_scan_args), the backward pass (mamba_selective_scan_bwd) and the
 * single-token decode step (selective_state_update).
 */
#ifndef SSS48_SELECTIVE_SCAN_H
#define SSS48_SELECTIVE_SCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MSS_ABI_VERSION 11

typedef enum {
  MSS_OK = 0,
  MSS_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or dtype   */
  MSS_ERR_UNSUPPORTED = 2, /* valid request this build does not implement   */
  MSS_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed          */
  MSS_ERR_TIMEOUT = 4,     /* a bounded device-side wait ran out            */
  MSS_ERR_WORKSPACE = 5    /* workspace missing or smaller than required    */
} mss_status;

typedef enum { MSS_F32 = 0, MSS_BF16 = 1 } mss_dtype;

/* Test-only flags (mss_scan_args.test_flags); 0 in production. */
#define MSS_TESTFLAG_DROP_PUBLISH 0x1u /* split scans: before composing the
                                          chunks' carries, the library waits
                                          for a publication that never
                                          comes, so its bounded wait
                                          (spin_timeout_ns) must run out    */
#define MSS_TESTFLAG_DEBUG_OOB 0x2u    /* checked build only: the first y
                                          store of the first thread block is
                                          aimed one tensor length past y; the
                                          bounds check must skip it and
                                          report MSS_ERR_INVALID_ARG.  No
                                          effect in the ordinary build.     */

/* Checked build.  Compiling the library with MSS_DEBUG=1 (the builder's
 * --debug option, libsss48_debug.so) adds a bounds check to every global
 * access at a computed index in the forward scan, the decode step and the
 * backward scan.  An index outside its tensor is skipped and recorded in
 * the device status word; the status calls then return MSS_ERR_INVALID_ARG
 * (ahead of MSS_ERR_TIMEOUT).  The checks never trap or assert.  Accesses
 * made by the TMA engine are bounds-checked by the hardware in either
 * build.  The ordinary build contains none of this code. */

/* Arguments of one forward scan.  Shapes:
 *   u, delta, z, y   (batch, dim, seqlen)   in_dtype (y: out_dtype)
 *   B, C             (batch, dstate, seqlen) in_dtype, shared by all channels
 *   A                (dim, dstate)          fp32, expected <= 0
 *   D, delta_bias    (dim)                  fp32
 *   h0, last_state   (batch, dim, dstate)   fp32
 * Optional (may be NULL): D (-> 0), z (-> no gate), delta_bias (-> 0),
 * h0 (-> zero initial state), last_state (-> not written).
 * Strides: u, delta, z, y, B and C may be views with any batch and row
 * (channel or state) strides, given in elements in stride_*[0] (batch) and
 * stride_*[1] (row); the time dimension must be contiguous.  {0, 0} means
 * packed, i.e. {rows * seqlen, seqlen}.  Input strides may be anything
 * non-negative (a zero batch stride shares one B or C between all batch
 * rows).  y's rows must not overlap (stride_y[1] >= seqlen when dim > 1),
 * nor its batches (stride_y[0] >= (dim - 1) * stride_y[1] + seqlen when
 * batch > 1), and y must not overlap any input; violations of the first two
 * return MSS_ERR_INVALID_ARG, the last is not checked.  This covers, for
 * instance, u and z taken as the two halves of one (batch, 2 dim, seqlen)
 * projection.
 * Alignment: every pointer must be aligned to its element size; 16-byte
 * alignment of u, delta, z, B, C with every stride (and seqlen) a multiple
 * of 16 bytes enables the TMA load path (otherwise plain loads run), and y
 * rows starting at multiples of 4 elements on a 16-byte (fp32) or 8-byte
 * (bf16) boundary enable vector stores.
 * h0 may alias last_state. */
typedef struct mss_scan_args {
  int64_t batch;   /* >= 1 */
  int64_t dim;     /* >= 1, channels D */
  int64_t dstate;  /* 1..16, states N per channel */
  int64_t seqlen;  /* >= 1, sequence length L */
  mss_dtype in_dtype;
  mss_dtype out_dtype;
  const void *u;
  const void *delta;
  const float *A;
  const void *B;
  const void *C;
  const float *D;
  const void *z;
  const float *delta_bias;
  int delta_softplus; /* 1: Delta = softplus(delta + bias); 0: delta + bias */
  const float *h0;
  void *y;
  float *last_state;
  void *workspace;        /* device, >= mss_scan_workspace_size() bytes,
                             256-byte aligned; may be NULL if that is 0 */
  size_t workspace_bytes;
  int plan_splits;        /* 0 = automatic; > 0 forces the number of
                             sequence chunks (tests use it to check that
                             the result does not depend on the grouping) */
  int plan_chunk_steps;   /* reserved, must be 0 */
  unsigned test_flags;    /* 0 in production */
  int64_t spin_timeout_ns;/* bound of the wait MSS_TESTFLAG_DROP_PUBLISH
                             provokes; 0 = 1 s (the pipeline's own waits
                             are bounded at 2 s) */
  /* element strides {batch, row} of the (batch, rows, seqlen) tensors; time
     is contiguous; {0, 0} = packed (see above) */
  int64_t stride_u[2];
  int64_t stride_delta[2];
  int64_t stride_z[2];
  int64_t stride_B[2];
  int64_t stride_C[2];
  int64_t stride_y[2];
  /* packed sequences: NULL, or num_seqs + 1 int32 offsets (device memory,
     0 = cu_seqlens[0] <= ... <= cu_seqlens[num_seqs] = seqlen) dividing
     every batch row into num_seqs independent sequences.  The state
     restarts from zero at each interior offset; h0 seeds the first
     sequence of a row and last_state receives the end of its last.
     Requires A <= 0 (a restart is a decay of exactly zero).  The offsets
     are read on the device and not validated there: offsets that are not
     ordered restart the state at the wrong steps but read nothing out of
     bounds. */
  const int32_t *cu_seqlens;
  int64_t num_seqs;     /* 0 when cu_seqlens is NULL */
  /* 1: the three-term trapezoidal update of Mamba-3 ("The State That Must
     Remember Everything", Part 7: h_t = alpha_t h_{t-1} + beta_t B_{t-1}
     x_{t-1} + gamma_t B_t x_t), read as the trapezoidal rule for the same
     ODE: h_t = a_t h_{t-1} + Delta_t / 2 (a_t B_{t-1} u_{t-1} + B_t u_t),
     a_t = exp(Delta_t A), no previous input before step 0; a chunk of a
     split sequence reads the step before it from u and B.  0: the Euler
     update above.  Not combined with cu_seqlens (MSS_ERR_UNSUPPORTED). */
  int trapezoid;
  /* NULL, or an output of 128 bytes per 16 steps of every channel (for
     dstate <= 16: 2 * tiles * ceil(seqlen / 16) * 4 * groups * 32 floats,
     the checkpoint part of mss_scan_bwd_workspace_size()) that receives two
     arrays of states in the layout mamba_selective_scan_bwd reads
     (mss_scan_bwd_args.checkpoints): the state of every channel at the
     start of every 16-step block, then the state entering its 9th step,
     each fp32 [tile][block][state][lane] with tile = b * ceil(dim / 32) +
     d / 32, block = t / 16, lane = d % 32, and states padded to 4, 8 or
     16.  A scan
     that writes checkpoints is never split into chunks; not combined with
     cu_seqlens or trapezoid (MSS_ERR_UNSUPPORTED). */
  float *checkpoints;
} mss_scan_args;

/* Bytes of device workspace the scan needs for these arguments (0 when the
 * sequence is not split).  Reads only sizes, dtypes and plan fields. */
mss_status mss_scan_workspace_size(const mss_scan_args *args, size_t *bytes);

/* Forward selective scan: validates, plans the launch (sequence split,
 * chunk length), clears the workspace's status word with cudaMemsetAsync
 * and launches on `stream` (a split scan: the chunks from a zero state, the
 * composition of their carries, then the carried terms, three kernels in
 * stream order).  Writes y and, if requested, last_state. */
mss_status mamba_selective_scan_fwd(const mss_scan_args *args, void *stream);

/* Synchronises `stream`, then reports the device-side status of the last
 * scan with these arguments: for a split scan the status word in
 * args->workspace, otherwise the library's own word, which is read and
 * cleared (so it reports every unsplit scan, and in the checked build every
 * decode step, since the previous call, on any stream of this device, once
 * that work has completed).  MSS_ERR_TIMEOUT: a bounded wait ran out;
 * MSS_ERR_INVALID_ARG: the checked build skipped an out-of-range access. */
mss_status mss_scan_status(const mss_scan_args *args, void *stream);

/* The same forward scan for callers that cannot allocate device memory:
 * plugins and runtimes that are handed only the tensors they own and have no
 * allocator of their own to call, code running under a memory pool it must
 * not re-enter, and latency-critical paths where cudaMalloc (which can
 * synchronise the device) is not allowed.  The pages have no counterpart;
 * this is a calling convenience of this library.
 *
 * A scan whose plan splits the sequence needs workspace
 * (mss_scan_workspace_size() > 0).  Here it uses an 8 MiB array that the
 * library keeps in device memory (every device that loads the library holds
 * it until the process exits) instead of args->workspace, which is ignored.
 * Inputs and outputs are still the caller's.  Plans needing more than 8 MiB
 * of workspace are rejected with MSS_ERR_WORKSPACE before anything is
 * enqueued.  Nothing is allocated or freed, by this call or by any library
 * it calls.
 *
 * The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture.  All
 * calls share the one array and its status word is cleared on the caller's stream
 * at the start of each call: two calls whose work overlaps on the GPU (on
 * different streams, or from different threads) race and must not be
 * issued.  A bounded device-side wait that runs out is recorded in a status
 * word (inside the array for a split plan) and y is then unspecified;
 * mss_scan_noalloc_status reports it.  mss_scan_status does not apply to
 * these calls: it reads args->workspace, which this entry point never
 * writes. */
mss_status mamba_selective_scan_fwd_noalloc(const mss_scan_args *args,
                                           void *stream);

/* Synchronises `stream`, then reports the device-side status of
 * mamba_selective_scan_fwd_noalloc calls with these arguments' plan:
 * MSS_ERR_TIMEOUT if a bounded wait ran out.  For a split plan it reads the
 * status word at the start of the library's array, which each such call
 * clears when it starts (so call this before the next one); otherwise the
 * library's own word, as mss_scan_status does.  The word read is cleared.
 * Like the scan, it allocates nothing.  The pages have no counterpart. */
mss_status mss_scan_noalloc_status(const mss_scan_args *args, void *stream);

/* Arguments of one decode step.  Shapes:
 *   state            (batch, dim, dstate) fp32, updated in place
 *   x, dt, z, y      (batch, dim)         in_dtype (y: out_dtype)
 *   B, C             (batch, dstate)      in_dtype
 *   A                (dim, dstate)        fp32
 *   D, dt_bias       (dim)                fp32, optional
 */
typedef struct mss_update_args {
  int64_t batch;
  int64_t dim;
  int64_t dstate; /* 1..16 */
  mss_dtype in_dtype;
  mss_dtype out_dtype;
  float *state;
  const void *x;
  const void *dt;
  const float *A;
  const void *B;
  const void *C;
  const float *D;
  const void *z;
  const float *dt_bias;
  int dt_softplus;
  void *y;
} mss_update_args;

/* Single-token state update (decode): one step of the recurrence above for
 * every (batch, channel), state updated in place, y written. */
mss_status selective_state_update(const mss_update_args *args, void *stream);

/* Arguments of one backward scan: the gradients of
 *   loss = sum(dy * y) + sum(d_last * last_state)
 * for the forward scan with the same inputs (shapes as in mss_scan_args;
 * the (batch, rows, seqlen) inputs and dy may be strided, and packed
 * sequences restart the state as in the forward scan, so no gradient flows
 * across a sequence start).  The states are not
 * taken from the forward pass but recomputed: a forward sweep stores the
 * state of every channel at the start of every 16-step block in the
 * workspace and a reverse sweep recomputes each block from it ("Mamba is
 * attention all you really need, part 2", section "Keeping the pad on the
 * desk"; "The State That Must Remember Everything", Part 3, "The
 * Hardware-Aware Way Out").  Inputs: dy (batch, dim, seqlen) fp32 and
 * d_last (batch, dim, dstate) fp32 or NULL.  Outputs, all fp32 and all
 * overwritten: du, ddelta, dz (batch, dim, seqlen; dz NULL when z is), dA
 * (dim, dstate), dB, dC (batch, dstate, seqlen), dD and ddelta_bias (dim;
 * NULL when D / delta_bias are), dh0 (batch, dim, dstate) or NULL.  dA, dB,
 * dC, dD and ddelta_bias are cleared with cudaMemsetAsync on the stream and
 * then accumulated with atomics, so their low bits depend on the order in
 * which blocks finish. */
typedef struct mss_scan_bwd_args {
  int64_t batch;
  int64_t dim;
  int64_t dstate;   /* 1..16 */
  int64_t seqlen;
  mss_dtype in_dtype; /* of u, delta, B, C, z */
  const void *u;
  const void *delta;
  const float *A;
  const void *B;
  const void *C;
  const float *D;
  const void *z;
  const float *delta_bias;
  int delta_softplus;
  const float *h0;
  const float *dy;
  const float *d_last;
  float *du;
  float *ddelta;
  float *dA;
  float *dB;
  float *dC;
  float *dD;
  float *dz;
  float *ddelta_bias;
  float *dh0;
  /* NULL, or the checkpoints written by the forward scan of the same
     inputs (mss_scan_args.checkpoints): the backward then skips its own
     forward sweep and needs no workspace. */
  const float *checkpoints;
  void *workspace;          /* device, >= mss_scan_bwd_workspace_size(),
                               256-byte aligned, not shared with a call in
                               flight; may be NULL with checkpoints (no
                               cut schedule then) */
  size_t workspace_bytes;
  /* element strides {batch, row} of u, delta, z, B, C and dy, with the
     same meaning and rules as the input strides of mss_scan_args ({0, 0}:
     packed); the gradients are always packed */
  int64_t stride_u[2];
  int64_t stride_delta[2];
  int64_t stride_z[2];
  int64_t stride_B[2];
  int64_t stride_C[2];
  int64_t stride_dy[2];
  /* packed sequences as in mss_scan_args (NULL / 0: one sequence per row);
     not combined with checkpoints */
  const int32_t *cu_seqlens;
  int64_t num_seqs;
} mss_scan_bwd_args;

/* Workspace bytes of the backward scan: the states of its own forward sweep
 * (64 bytes per 16 steps of every channel, for dstate <= 16, twice over --
 * block starts and mid-block -- without cu_seqlens, once with; none when
 * `checkpoints` is given), then the area of the cut schedule when it applies on the current
 * device.  A launch of batch * ceil(dim / 32) blocks whose last wave of
 * resident blocks is at most half full cuts the tiles of that wave in two
 * at their middle 16-step block: the first part's forward sweep, the second
 * part's sweeps and the first part's reverse sweep run as separate work
 * items (taken by ticket: the first pieces, every whole tile, the other
 * pieces), handing the state and
 * the adjoint over through the workspace; du, ddelta and dz are
 * bit-identical to the uncut schedule.  A workspace with the checkpoints
 * but not that area runs every tile whole.  Packed sequences are not cut.
 * A hand-over wait is bounded (2 s); one that runs out records a timeout in
 * the library's own status word (reported by mss_scan_status for an
 * unsplit scan's arguments). */
mss_status mss_scan_bwd_workspace_size(const mss_scan_bwd_args *args, size_t *bytes);

/* Backward selective scan on `stream`; argument errors return before any
 * work is enqueued. */
mss_status mamba_selective_scan_bwd(const mss_scan_bwd_args *args, void *stream);

/* Human-readable name of a status code (static string). */
const char *mss_status_string(mss_status status);

/* MSS_ABI_VERSION of the loaded library. */
int mss_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif
