// scan_bwd.cuh -- launch interface of the backward selective-scan kernel.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace sss48 {

constexpr int kBwdChannels = 32;   // channels per thread block
constexpr int kBwdTimeBlock = 16;  // steps between state checkpoints

struct BwdParams {
  int64_t batch, dim, dstate, seqlen;
  const void *u, *delta;
  const float *A;
  const void *B, *C;
  const float *D;
  const void *z;
  const float *delta_bias;
  int softplus;
  const float *h0;
  const float *dy;
  const float *d_last;
  float *du, *ddelta, *dA, *dB, *dC, *dD, *dz, *ddelta_bias, *dh0;
  float *ckpt;      // workspace: one state per channel and 16-step block
  float *ckpt_mid;  // ordinary sequences: the state entering step 8 of
                    // every block (same layout); null with packed sequences
  int ckpt_given;   // ckpt already holds the forward scan's states
  int ch_tiles;     // ceil(dim / kBwdChannels)
  int64_t tiles;    // batch * ch_tiles
  unsigned *status; // library status word (bounds checks of the checked build)
  // element strides {batch, row} of the (batch, rows, seqlen) inputs (time
  // contiguous; always resolved) and their extents (largest index + 1) for
  // the checked build; the gradients are packed
  int64_t su[2], sdl[2], sz[2], sB[2], sC[2], sdy[2];
  int64_t ext_u, ext_delta, ext_z, ext_B, ext_C, ext_dy;
  // packed sequences (nullptr: one sequence per row): interior offsets
  // cu[1 .. nseq-1] start a sequence with an empty state
  const int32_t *cu;
  int64_t nseq;
  // cut schedule (ncut == 0: one block per tile in blockIdx order).  The
  // last ncut tiles are cut after block kcut into work items taken by
  // ticket: the first part's forward sweep (no item when the checkpoints
  // are given), the second part's sweeps, the first part's reverse sweep,
  // with gap0 whole tiles after the first of them and gap1 after the second
  int ncut, kcut;
  int64_t gap0, gap1;
  unsigned *ticket;
  unsigned *flag;  // [2][ncut]: first part's states written, second part's adjoint written
  float *lam;      // [ncut][4 * groups][32]: the adjoint entering the second part
};

// The cut schedule of a launch: how many tiles are cut, where, and the
// workspace it needs beyond the checkpoints (0 bytes: nothing is cut).
struct BwdCut {
  int ncut = 0, kcut = 0;
  int64_t gap0 = 0, gap1 = 0;
  size_t bytes = 0;
};
BwdCut plan_bwd_cut(const BwdParams &p, int in_bf16);

// Warps per block (state groups of 4): 1, 2 or 4.
int bwd_groups(int64_t dstate);

// Workspace bytes of the state checkpoints (one array; the backward's own
// sweep of ordinary sequences keeps two, the second at mid-block).
size_t scan_bwd_workspace_bytes(int64_t tiles, int64_t seqlen, int64_t dstate);

// dA, dB, dC, dD and ddelta_bias are accumulated with atomics: the caller
// zeroes them first.
cudaError_t launch_scan_bwd(const BwdParams &p, int in_bf16, cudaStream_t stream);

}  // namespace sss48
