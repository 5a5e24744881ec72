// scan_fwd.cuh -- launch interface between the C ABI layer and the
// forward-scan / state-update kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace sss48 {

// Channels per thread block (one per lane) and states per lane.  A block has
// one warp per group of kStatesPerLane states, so every lane of a warp owns
// the same state indices and reads B_t[n], C_t[n] at warp-uniform addresses.
constexpr int kChannelsPerBlock = 32;
constexpr int kStatesPerLane = 4;
constexpr int kMaxStates = 16;
constexpr int kTimeBlock = 16;  // timesteps staged in shared memory at once

struct ScanParams {
  int64_t batch, dim, dstate, seqlen;
  const void *u, *delta;
  const float *A;
  const void *B, *C;
  const float *D;
  const void *z;
  const float *delta_bias;
  int softplus;
  const float *h0;
  void *y;
  float *last_state;
  // element strides {batch, row} of the (batch, rows, seqlen) tensors (time
  // is contiguous); always resolved, never 0
  int64_t su[2], sdl[2], sz[2], sB[2], sC[2], sy[2];
  // packed sequences (nullptr: one sequence per row): interior offsets
  // cu[1 .. nseq-1] restart the state
  const int32_t *cu;
  int64_t nseq;
  // three-term trapezoidal update (1) instead of the Euler one (0)
  int trap;
  // optional: state at the start of every block, [tile][block][4G][CH]
  float *ckpt_out;
  int y_vec;       // rows of y allow 4-element vector stores (set at launch)
  // launch plan
  int64_t chunk;   // timesteps per sequence chunk (multiple of kTimeBlock)
  int splits;      // number of sequence chunks
  int ch_tiles;    // ceil(dim / kChannelsPerBlock)
  int64_t tiles;   // batch * ch_tiles
  // device-side status word (workspace when split, library word otherwise)
  unsigned *status;
  // split-mode workspace: next item to hand out, then per item
  // (chunk-major: chunk * tiles + tile)
  unsigned *ticket;
  float *agg;      // decay product P over the chunk, then local end state e
  float *incl;     // true state at the end of the chunk
  float *sig;      // running sum of Delta at the start of every segment
  int segb;        // 16-step blocks per correction segment
  int nseg;        // segments per chunk
  unsigned test_flags;
  int64_t spin_timeout_ns;
  // element extents (largest index + 1) of the streamed tensors under their
  // strides and of the checkpoint buffer: the bounds of the checked build
  int64_t ext_u, ext_delta, ext_z, ext_B, ext_C, ext_y, ext_ckpt;
};

// TMA descriptors of the five streamed inputs (z unused without a gate).
struct TmaMaps {
  CUtensorMap u, delta, z, B, C;
};

// Blocks of kTimeBlock steps per correction segment of a split scan.
constexpr int kSegBlocks = 32;

// Workspace bytes for `splits` chunks of `chunk` steps over `tiles` tiles
// with `groups` state groups (0 when splits == 1).
size_t scan_workspace_bytes(int64_t tiles, int splits, int64_t chunk, int groups);

// Carves the workspace into the fields of `p`.
void scan_bind_workspace(ScanParams &p, void *ws, int groups);

// Bytes at the start of the workspace (the status word) that must be zero
// before a launch.
size_t scan_workspace_clear_bytes();

// Device address of the library's own status word (used when a scan has no
// workspace); nullptr on failure.
unsigned *scan_status_word();

// Thread blocks of the scan kernel that fit on one SM (for planning).
int scan_blocks_per_sm(int in_bf16, int out_bf16, int groups);

cudaError_t launch_scan_fwd(const ScanParams &p, int in_bf16, int out_bf16,
                            cudaStream_t stream);

struct UpdateParams {
  int64_t batch, dim, dstate;
  float *state;
  const void *x, *dt;
  const float *A;
  const void *B, *C;
  const float *D;
  const void *z;
  const float *dt_bias;
  int softplus;
  void *y;
  unsigned *status;  // library status word (bounds checks of the checked build)
};

cudaError_t launch_state_update(const UpdateParams &p, int in_bf16,
                                int out_bf16, cudaStream_t stream);

}  // namespace sss48
