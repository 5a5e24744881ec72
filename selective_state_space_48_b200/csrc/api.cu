// api.cu -- C ABI of the selective-scan library: argument checks, launch
// planning and dispatch.  Declarations and their documentation are in
// include/selective_scan.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "device_math.cuh"
#include "nvtx_range.cuh"
#include "scan_bwd.cuh"
#include "scan_fwd.cuh"
#include "selective_scan.h"

using namespace sss48;

namespace {

constexpr int64_t kMinChunk = 1024;  // shortest automatic sequence chunk
constexpr int kMaxDevices = 64;

bool aligned(const void *p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

size_t esize(mss_dtype t) { return t == MSS_BF16 ? 2 : 4; }

bool valid_dtype(mss_dtype t) { return t == MSS_F32 || t == MSS_BF16; }

struct Plan {
  int groups;
  int ch_tiles;
  int64_t tiles;
  int splits;
  int64_t chunk;
  size_t workspace;
};

int device_sms(int dev) {
  static int cache[kMaxDevices] = {0};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess ||
        n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

int blocks_per_sm(int dev, int in_bf16, int out_bf16, int groups) {
  static int cache[kMaxDevices][2][2][5] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= kMaxDevices) return 1;
  int &c = cache[dev][in_bf16][out_bf16][groups];
  if (c == 0) c = scan_blocks_per_sm(in_bf16, out_bf16, groups);
  return c;
}

// Element strides {batch, row} of a (batch, rows, seqlen) tensor whose
// time dimension is contiguous: {0, 0} means packed.  Inputs may overlap
// (a zero batch stride broadcasts one tensor to every batch row); the
// output's rows and batches must not.  False on a negative or absurdly
// large stride, or an overlapping output.
bool resolve_strides(const int64_t (&in)[2], int64_t batch, int64_t rows,
                     int64_t seqlen, bool output, int64_t (&out)[2]) {
  if (in[0] == 0 && in[1] == 0) {
    out[0] = rows * seqlen;
    out[1] = seqlen;
    return true;
  }
  const int64_t lim = int64_t(1) << 44;
  if (in[0] < 0 || in[1] < 0 || in[0] > lim || in[1] > lim) return false;
  if (output) {
    if (rows > 1 && in[1] < seqlen) return false;
    if (batch > 1 && in[0] < (rows - 1) * in[1] + seqlen) return false;
  }
  out[0] = in[0];
  out[1] = in[1];
  return true;
}

// All six stride pairs of a scan, resolved; false on the first bad one.
bool resolve_scan_strides(const mss_scan_args *a, ScanParams *p) {
  const int64_t Bt = a->batch, D = a->dim, N = a->dstate, L = a->seqlen;
  return resolve_strides(a->stride_u, Bt, D, L, false, p->su) &&
         resolve_strides(a->stride_delta, Bt, D, L, false, p->sdl) &&
         resolve_strides(a->stride_z, Bt, D, L, false, p->sz) &&
         resolve_strides(a->stride_B, Bt, N, L, false, p->sB) &&
         resolve_strides(a->stride_C, Bt, N, L, false, p->sC) &&
         resolve_strides(a->stride_y, Bt, D, L, true, p->sy);
}

mss_status check_scan_args(const mss_scan_args *a) {
  if (!a) return MSS_ERR_INVALID_ARG;
  if (a->batch < 1 || a->dim < 1 || a->seqlen < 1 || a->dstate < 1)
    return MSS_ERR_INVALID_ARG;
  if (a->dstate > kMaxStates) return MSS_ERR_UNSUPPORTED;
  if (!valid_dtype(a->in_dtype) || !valid_dtype(a->out_dtype))
    return MSS_ERR_INVALID_ARG;
  if (a->plan_splits < 0 || a->plan_chunk_steps != 0 || a->spin_timeout_ns < 0)
    return MSS_ERR_INVALID_ARG;
  // sizes whose element counts or grid would overflow
  const int64_t lim = int64_t(1) << 40;
  if (a->batch > lim / a->dim || a->batch * a->dim > lim / a->seqlen)
    return MSS_ERR_UNSUPPORTED;
  if (!a->u || !a->delta || !a->A || !a->B || !a->C || !a->y)
    return MSS_ERR_INVALID_ARG;
  {
    ScanParams probe{};
    if (!resolve_scan_strides(a, &probe)) return MSS_ERR_INVALID_ARG;
  }
  if (a->cu_seqlens ? (a->num_seqs < 1 || a->num_seqs > INT32_MAX ||
                       !aligned(a->cu_seqlens, 4))
                    : a->num_seqs != 0)
    return MSS_ERR_INVALID_ARG;
  if (a->trapezoid != 0 && a->trapezoid != 1) return MSS_ERR_INVALID_ARG;
  if (a->trapezoid && a->cu_seqlens) return MSS_ERR_UNSUPPORTED;
  if (a->checkpoints && (a->trapezoid || a->cu_seqlens)) return MSS_ERR_UNSUPPORTED;
  if (a->checkpoints && (!aligned(a->checkpoints, 4) || a->plan_splits > 1))
    return MSS_ERR_INVALID_ARG;
  const size_t ei = esize(a->in_dtype), eo = esize(a->out_dtype);
  if (!aligned(a->u, ei) || !aligned(a->delta, ei) || !aligned(a->B, ei) ||
      !aligned(a->C, ei) || (a->z && !aligned(a->z, ei)) ||
      !aligned(a->y, eo) || !aligned(a->A, 4) || (a->D && !aligned(a->D, 4)) ||
      (a->delta_bias && !aligned(a->delta_bias, 4)) ||
      (a->h0 && !aligned(a->h0, 4)) ||
      (a->last_state && !aligned(a->last_state, 4)))
    return MSS_ERR_INVALID_ARG;
  return MSS_OK;
}

mss_status make_plan(const mss_scan_args *a, Plan *pl) {
  pl->groups = static_cast<int>((a->dstate + 3) / 4);
  pl->ch_tiles = static_cast<int>((a->dim + kChannelsPerBlock - 1) /
                                  kChannelsPerBlock);
  pl->tiles = a->batch * pl->ch_tiles;
  int64_t want = a->plan_splits;
  // checkpoints hold the true state at every block: only an unsplit scan
  // has it before its carry correction
  if (a->checkpoints) want = 1;
  if (want == 0) {
    // Split the sequence only when there are fewer channel tiles than SMs:
    // a chunk that does not start the sequence pays a carry correction whose
    // length grows with the state's memory, so whole-sequence tiles are
    // preferred whenever they can occupy the chip.
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MSS_ERR_CUDA;
    const int64_t sms = device_sms(dev);
    const int64_t target =
        sms * blocks_per_sm(dev, a->in_dtype == MSS_BF16,
                            a->out_dtype == MSS_BF16, pl->groups);
    if (pl->tiles >= sms) {
      want = 1;
    } else {
      // as many chunks as keep every (tile, chunk) block resident at once:
      // one block more than the chip holds would run as a second wave
      want = std::max<int64_t>(1, target / pl->tiles);
      want = std::min<int64_t>(want, std::max<int64_t>(1, a->seqlen / kMinChunk));
    }
  }
  want = std::max<int64_t>(1, std::min<int64_t>(want, a->seqlen));
  int64_t chunk = (a->seqlen + want - 1) / want;
  chunk = ((chunk + kTimeBlock - 1) / kTimeBlock) * kTimeBlock;
  pl->chunk = chunk;
  pl->splits = static_cast<int>((a->seqlen + chunk - 1) / chunk);
  if (pl->tiles * pl->splits > int64_t(INT32_MAX)) return MSS_ERR_UNSUPPORTED;
  // the carry launch has one block per (tile, chunk, segment)
  const int64_t nseg = ((chunk + kTimeBlock - 1) / kTimeBlock + kSegBlocks - 1) / kSegBlocks;
  if (pl->splits > 1 && pl->tiles * pl->splits * nseg > int64_t(INT32_MAX))
    return MSS_ERR_UNSUPPORTED;
  pl->workspace = scan_workspace_bytes(pl->tiles, pl->splits, pl->chunk, pl->groups);
  return MSS_OK;
}

// Kernel parameters of a checked scan (everything but the status word and
// the workspace fields).
void fill_scan_params(const mss_scan_args *a, const Plan &pl, ScanParams *p) {
  p->batch = a->batch;
  p->dim = a->dim;
  p->dstate = a->dstate;
  p->seqlen = a->seqlen;
  p->u = a->u;
  p->delta = a->delta;
  p->A = a->A;
  p->B = a->B;
  p->C = a->C;
  p->D = a->D;
  p->z = a->z;
  p->delta_bias = a->delta_bias;
  p->softplus = a->delta_softplus ? 1 : 0;
  p->h0 = a->h0;
  p->y = a->y;
  p->last_state = a->last_state;
  resolve_scan_strides(a, p);  // checked in check_scan_args
  p->cu = a->cu_seqlens;
  p->nseq = a->cu_seqlens ? a->num_seqs : 0;
  p->trap = a->trapezoid;
  p->ckpt_out = a->checkpoints;
  p->chunk = pl.chunk;
  p->splits = pl.splits;
  p->ch_tiles = pl.ch_tiles;
  p->tiles = pl.tiles;
  p->test_flags = a->test_flags;
  p->spin_timeout_ns = a->spin_timeout_ns;
  auto ext = [&](const int64_t (&st)[2], int64_t rows) {
    return (a->batch - 1) * st[0] + (rows - 1) * st[1] + a->seqlen;
  };
  p->ext_u = ext(p->su, a->dim);
  p->ext_delta = ext(p->sdl, a->dim);
  p->ext_z = ext(p->sz, a->dim);
  p->ext_B = ext(p->sB, a->dstate);
  p->ext_C = ext(p->sC, a->dstate);
  p->ext_y = ext(p->sy, a->dim);
  // two arrays: block starts and mid-block states
  const size_t ck = scan_bwd_workspace_bytes(pl.tiles, a->seqlen, a->dstate);
  p->ext_ckpt = a->checkpoints ? static_cast<int64_t>(2 * ck / sizeof(float)) : 0;
}

}  // namespace

extern "C" {

mss_status mss_scan_workspace_size(const mss_scan_args *args, size_t *bytes) {
  if (!bytes) return MSS_ERR_INVALID_ARG;
  mss_status st = check_scan_args(args);
  if (st != MSS_OK) return st;
  Plan pl;
  st = make_plan(args, &pl);
  if (st != MSS_OK) return st;
  *bytes = pl.workspace;
  return MSS_OK;
}

mss_status mamba_selective_scan_fwd(const mss_scan_args *a, void *stream) {
  NvtxRange range("mamba_selective_scan_fwd");
  mss_status st = check_scan_args(a);
  if (st != MSS_OK) return st;
  Plan pl;
  st = make_plan(a, &pl);
  if (st != MSS_OK) return st;
  if (pl.workspace > 0 &&
      (!a->workspace || a->workspace_bytes < pl.workspace ||
       !aligned(a->workspace, 256)))
    return MSS_ERR_WORKSPACE;

  ScanParams p{};
  fill_scan_params(a, pl, &p);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pl.splits > 1) {
    scan_bind_workspace(p, a->workspace, pl.groups);
    if (cudaMemsetAsync(a->workspace, 0, scan_workspace_clear_bytes(), s) != cudaSuccess)
      return MSS_ERR_CUDA;
  } else {
    p.status = scan_status_word();
    if (!p.status) return MSS_ERR_CUDA;
  }
  if (launch_scan_fwd(p, a->in_dtype == MSS_BF16, a->out_dtype == MSS_BF16,
                      s) != cudaSuccess)
    return MSS_ERR_CUDA;
  return MSS_OK;
}

mss_status mss_scan_status(const mss_scan_args *a, void *stream) {
  mss_status st = check_scan_args(a);
  if (st != MSS_OK) return st;
  Plan pl;
  st = make_plan(a, &pl);
  if (st != MSS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MSS_ERR_CUDA;
  unsigned word = 0;
  if (pl.splits <= 1) {
    // scans without workspace report into the library's own word, which is
    // read and cleared here
    unsigned *w = scan_status_word();
    if (!w) return MSS_ERR_CUDA;
    if (cudaMemcpy(&word, w, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(w, 0, sizeof(word)) != cudaSuccess)
      return MSS_ERR_CUDA;
  } else {
    if (!a->workspace || a->workspace_bytes < pl.workspace)
      return MSS_ERR_WORKSPACE;
    if (cudaMemcpy(&word, a->workspace, sizeof(word), cudaMemcpyDeviceToHost) !=
        cudaSuccess)
      return MSS_ERR_CUDA;
  }
  if (word & kStatusBadIndex) return MSS_ERR_INVALID_ARG;
  if (word & kStatusTimeout) return MSS_ERR_TIMEOUT;
  return MSS_OK;
}

mss_status selective_state_update(const mss_update_args *a, void *stream) {
  NvtxRange range("selective_state_update");
  if (!a) return MSS_ERR_INVALID_ARG;
  if (a->batch < 1 || a->dim < 1 || a->dstate < 1) return MSS_ERR_INVALID_ARG;
  if (a->dstate > kMaxStates) return MSS_ERR_UNSUPPORTED;
  if (!valid_dtype(a->in_dtype) || !valid_dtype(a->out_dtype))
    return MSS_ERR_INVALID_ARG;
  if (a->batch > (int64_t(1) << 40) / a->dim) return MSS_ERR_UNSUPPORTED;
  if (!a->state || !a->x || !a->dt || !a->A || !a->B || !a->C || !a->y)
    return MSS_ERR_INVALID_ARG;
  const size_t ei = esize(a->in_dtype), eo = esize(a->out_dtype);
  if (!aligned(a->state, 4) || !aligned(a->x, ei) || !aligned(a->dt, ei) ||
      !aligned(a->B, ei) || !aligned(a->C, ei) || (a->z && !aligned(a->z, ei)) ||
      !aligned(a->y, eo) || !aligned(a->A, 4) || (a->D && !aligned(a->D, 4)) ||
      (a->dt_bias && !aligned(a->dt_bias, 4)))
    return MSS_ERR_INVALID_ARG;
  UpdateParams p{};
  p.batch = a->batch;
  p.dim = a->dim;
  p.dstate = a->dstate;
  p.state = a->state;
  p.x = a->x;
  p.dt = a->dt;
  p.A = a->A;
  p.B = a->B;
  p.C = a->C;
  p.D = a->D;
  p.z = a->z;
  p.dt_bias = a->dt_bias;
  p.softplus = a->dt_softplus ? 1 : 0;
  p.y = a->y;
  p.status = scan_status_word();
  if (!p.status) return MSS_ERR_CUDA;
  if (launch_state_update(p, a->in_dtype == MSS_BF16, a->out_dtype == MSS_BF16,
                          static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSS_ERR_CUDA;
  return MSS_OK;
}

}  // extern "C"

namespace {

// The six input stride pairs of a backward scan, resolved; false on the
// first bad one.
bool resolve_bwd_strides(const mss_scan_bwd_args *a, BwdParams *p) {
  const int64_t Bt = a->batch, D = a->dim, N = a->dstate, L = a->seqlen;
  return resolve_strides(a->stride_u, Bt, D, L, false, p->su) &&
         resolve_strides(a->stride_delta, Bt, D, L, false, p->sdl) &&
         resolve_strides(a->stride_z, Bt, D, L, false, p->sz) &&
         resolve_strides(a->stride_B, Bt, N, L, false, p->sB) &&
         resolve_strides(a->stride_C, Bt, N, L, false, p->sC) &&
         resolve_strides(a->stride_dy, Bt, D, L, false, p->sdy);
}

mss_status check_bwd_args(const mss_scan_bwd_args *a) {
  if (!a) return MSS_ERR_INVALID_ARG;
  if (a->batch < 1 || a->dim < 1 || a->seqlen < 1 || a->dstate < 1)
    return MSS_ERR_INVALID_ARG;
  if (a->dstate > kMaxStates) return MSS_ERR_UNSUPPORTED;
  if (!valid_dtype(a->in_dtype)) return MSS_ERR_INVALID_ARG;
  const int64_t lim = int64_t(1) << 40;
  if (a->batch > lim / a->dim || a->batch * a->dim > lim / a->seqlen)
    return MSS_ERR_UNSUPPORTED;
  if (!a->u || !a->delta || !a->A || !a->B || !a->C || !a->dy || !a->du ||
      !a->ddelta || !a->dA || !a->dB || !a->dC)
    return MSS_ERR_INVALID_ARG;
  {
    BwdParams probe{};
    if (!resolve_bwd_strides(a, &probe)) return MSS_ERR_INVALID_ARG;
  }
  if (a->cu_seqlens ? (a->num_seqs < 1 || a->num_seqs > INT32_MAX ||
                       !aligned(a->cu_seqlens, 4))
                    : a->num_seqs != 0)
    return MSS_ERR_INVALID_ARG;
  // the forward scan writes no checkpoints for packed sequences
  if (a->cu_seqlens && a->checkpoints) return MSS_ERR_UNSUPPORTED;
  // a gradient is requested exactly for the optional inputs that are given
  if ((a->D == nullptr) != (a->dD == nullptr) || (a->z == nullptr) != (a->dz == nullptr) ||
      (a->delta_bias == nullptr) != (a->ddelta_bias == nullptr))
    return MSS_ERR_INVALID_ARG;
  const size_t ei = esize(a->in_dtype);
  const void *in[] = {a->u, a->delta, a->B, a->C, a->z};
  for (const void *q : in)
    if (q && !aligned(q, ei)) return MSS_ERR_INVALID_ARG;
  const void *f32[] = {a->A, a->D, a->delta_bias, a->h0, a->dy, a->d_last, a->du,
                       a->ddelta, a->dA, a->dB, a->dC, a->dD, a->dz,
                       a->ddelta_bias, a->dh0, a->checkpoints};
  for (const void *q : f32)
    if (q && !aligned(q, 4)) return MSS_ERR_INVALID_ARG;
  return MSS_OK;
}

}  // namespace

extern "C" {

// The backward's cut schedule for these arguments on the current device.
static BwdCut bwd_cut_of(const mss_scan_bwd_args *a) {
  BwdParams q{};
  q.seqlen = a->seqlen;
  q.dstate = a->dstate;
  q.tiles = a->batch * ((a->dim + kBwdChannels - 1) / kBwdChannels);
  q.ckpt_given = a->checkpoints ? 1 : 0;
  q.cu = a->cu_seqlens;
  return plan_bwd_cut(q, a->in_dtype == MSS_BF16);
}

mss_status mss_scan_bwd_workspace_size(const mss_scan_bwd_args *a, size_t *bytes) {
  if (!bytes) return MSS_ERR_INVALID_ARG;
  const mss_status st = check_bwd_args(a);
  if (st != MSS_OK) return st;
  const int64_t tiles = a->batch * ((a->dim + kBwdChannels - 1) / kBwdChannels);
  // the own sweep of ordinary sequences keeps a second array of states at
  // mid-block
  const size_t arrays = a->checkpoints ? 0 : (a->cu_seqlens ? 1 : 2);
  *bytes = arrays * scan_bwd_workspace_bytes(tiles, a->seqlen, a->dstate) + bwd_cut_of(a).bytes;
  return MSS_OK;
}

mss_status mamba_selective_scan_bwd(const mss_scan_bwd_args *a, void *stream) {
  NvtxRange range("mamba_selective_scan_bwd");
  const mss_status st = check_bwd_args(a);
  if (st != MSS_OK) return st;
  const int64_t ntiles = a->batch * ((a->dim + kBwdChannels - 1) / kBwdChannels);
  const size_t ck_array = scan_bwd_workspace_bytes(ntiles, a->seqlen, a->dstate);
  const size_t ck_bytes = a->checkpoints ? 0 : (a->cu_seqlens ? 1 : 2) * ck_array;
  if (!a->checkpoints &&
      (!a->workspace || a->workspace_bytes < ck_bytes || !aligned(a->workspace, 256)))
    return MSS_ERR_WORKSPACE;
  // the cut schedule runs when the workspace also holds its area (after the
  // checkpoints); otherwise every tile runs whole
  BwdCut cut = bwd_cut_of(a);
  if (!a->workspace || !aligned(a->workspace, 256) || a->workspace_bytes < ck_bytes + cut.bytes)
    cut = BwdCut();
  BwdParams p{};
  p.batch = a->batch;
  p.dim = a->dim;
  p.dstate = a->dstate;
  p.seqlen = a->seqlen;
  p.u = a->u;
  p.delta = a->delta;
  p.A = a->A;
  p.B = a->B;
  p.C = a->C;
  p.D = a->D;
  p.z = a->z;
  p.delta_bias = a->delta_bias;
  p.softplus = a->delta_softplus ? 1 : 0;
  p.h0 = a->h0;
  p.dy = a->dy;
  p.d_last = a->d_last;
  p.du = a->du;
  p.ddelta = a->ddelta;
  p.dA = a->dA;
  p.dB = a->dB;
  p.dC = a->dC;
  p.dD = a->dD;
  p.dz = a->dz;
  p.ddelta_bias = a->ddelta_bias;
  p.dh0 = a->dh0;
  p.ckpt = a->checkpoints ? const_cast<float *>(a->checkpoints)
                          : static_cast<float *>(a->workspace);
  // the second array: the states entering step 8 of every block (written
  // by the backward's own sweep, or by the forward scan with its checkpoints)
  p.ckpt_mid = a->cu_seqlens ? nullptr
                             : reinterpret_cast<float *>(reinterpret_cast<unsigned char *>(p.ckpt) +
                                                         ck_array);
  p.ckpt_given = a->checkpoints ? 1 : 0;
  p.ch_tiles = static_cast<int>((a->dim + kBwdChannels - 1) / kBwdChannels);
  p.tiles = a->batch * p.ch_tiles;
  resolve_bwd_strides(a, &p);  // checked above
  auto ext = [&](const int64_t (&st)[2], int64_t rows) {
    return (a->batch - 1) * st[0] + (rows - 1) * st[1] + a->seqlen;
  };
  p.ext_u = ext(p.su, a->dim);
  p.ext_delta = ext(p.sdl, a->dim);
  p.ext_z = ext(p.sz, a->dim);
  p.ext_B = ext(p.sB, a->dstate);
  p.ext_C = ext(p.sC, a->dstate);
  p.ext_dy = ext(p.sdy, a->dim);
  p.cu = a->cu_seqlens;
  p.nseq = a->cu_seqlens ? a->num_seqs : 0;
  p.status = scan_status_word();
  if (!p.status) return MSS_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  p.ncut = cut.ncut;
  p.kcut = cut.kcut;
  p.gap0 = cut.gap0;
  p.gap1 = cut.gap1;
  if (cut.ncut) {
    unsigned char *area = static_cast<unsigned char *>(a->workspace) + ck_bytes;
    p.ticket = reinterpret_cast<unsigned *>(area);
    p.flag = reinterpret_cast<unsigned *>(area + 256);
    p.lam = reinterpret_cast<float *>(area + 256 + ((8 * static_cast<size_t>(cut.ncut) + 255) /
                                                    256) * 256);
    // the ticket and the flags start at zero on every call
    if (cudaMemsetAsync(area, 0, reinterpret_cast<unsigned char *>(p.lam) - area, s) !=
        cudaSuccess)
      return MSS_ERR_CUDA;
  }
  // the gradients that are sums over blocks are accumulated with atomics
  const size_t f = sizeof(float);
  const size_t nBC = static_cast<size_t>(a->batch * a->dstate * a->seqlen) * f;
  if (cudaMemsetAsync(a->dA, 0, static_cast<size_t>(a->dim * a->dstate) * f, s) != cudaSuccess ||
      cudaMemsetAsync(a->dB, 0, nBC, s) != cudaSuccess ||
      cudaMemsetAsync(a->dC, 0, nBC, s) != cudaSuccess ||
      (a->dD && cudaMemsetAsync(a->dD, 0, static_cast<size_t>(a->dim) * f, s) != cudaSuccess) ||
      (a->ddelta_bias &&
       cudaMemsetAsync(a->ddelta_bias, 0, static_cast<size_t>(a->dim) * f, s) != cudaSuccess))
    return MSS_ERR_CUDA;
  if (launch_scan_bwd(p, a->in_dtype == MSS_BF16, s) != cudaSuccess) return MSS_ERR_CUDA;
  return MSS_OK;
}

const char *mss_status_string(mss_status s) {
  switch (s) {
    case MSS_OK: return "MSS_OK";
    case MSS_ERR_INVALID_ARG: return "MSS_ERR_INVALID_ARG";
    case MSS_ERR_UNSUPPORTED: return "MSS_ERR_UNSUPPORTED";
    case MSS_ERR_CUDA: return "MSS_ERR_CUDA";
    case MSS_ERR_TIMEOUT: return "MSS_ERR_TIMEOUT";
    case MSS_ERR_WORKSPACE: return "MSS_ERR_WORKSPACE";
  }
  return "MSS_ERR_UNKNOWN";
}

int mss_abi_version(void) { return MSS_ABI_VERSION; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Scan without any allocation by the caller or the library: the workspace of
// a sequence-split scan lives in a fixed array in device memory that this
// library owns (see the declaration in selective_scan.h).

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

// Every device that loads the library holds this array until the process
// exits.  Host code must not use its name as an address: the device address
// is looked up once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array on the current device, looked up on the first
// call per device (nullptr if the lookup fails).
void *noalloc_scratch_address() {
  static void *addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = ptr;
  }
  return addr[dev];
}

}  // namespace

extern "C" mss_status mamba_selective_scan_fwd_noalloc(const mss_scan_args *a,
                                                       void *stream) {
  NvtxRange range("mamba_selective_scan_fwd_noalloc");
  mss_status st = check_scan_args(a);
  if (st != MSS_OK) return st;
  Plan pl;
  st = make_plan(a, &pl);
  if (st != MSS_OK) return st;
  if (pl.workspace > kNoAllocScratchBytes) return MSS_ERR_WORKSPACE;

  ScanParams p{};
  fill_scan_params(a, pl, &p);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pl.splits > 1) {
    void *ws = noalloc_scratch_address();
    if (!ws) return MSS_ERR_CUDA;
    scan_bind_workspace(p, ws, pl.groups);
    // the status word carries the previous call's value: clear it
    if (cudaMemsetAsync(ws, 0, scan_workspace_clear_bytes(), s) != cudaSuccess)
      return MSS_ERR_CUDA;
  } else {
    p.status = scan_status_word();
    if (!p.status) return MSS_ERR_CUDA;
  }
  if (launch_scan_fwd(p, a->in_dtype == MSS_BF16, a->out_dtype == MSS_BF16, s) !=
      cudaSuccess)
    return MSS_ERR_CUDA;
  return MSS_OK;
}

extern "C" mss_status mss_scan_noalloc_status(const mss_scan_args *a, void *stream) {
  mss_status st = check_scan_args(a);
  if (st != MSS_OK) return st;
  Plan pl;
  st = make_plan(a, &pl);
  if (st != MSS_OK) return st;
  if (pl.workspace > kNoAllocScratchBytes) return MSS_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MSS_ERR_CUDA;
  // unsplit plans report into the library's own word, split plans into the
  // word at the start of the array; both are read and cleared here
  unsigned *w = pl.splits > 1 ? static_cast<unsigned *>(noalloc_scratch_address())
                              : scan_status_word();
  if (!w) return MSS_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, w, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(w, 0, sizeof(word)) != cudaSuccess)
    return MSS_ERR_CUDA;
  if (word & kStatusBadIndex) return MSS_ERR_INVALID_ARG;
  return (word & kStatusTimeout) ? MSS_ERR_TIMEOUT : MSS_OK;
}
