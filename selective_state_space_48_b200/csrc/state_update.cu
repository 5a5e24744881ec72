// state_update.cu -- single-token selective state update (decode).
//
// Decoding advances the recurrence by one token: the fixed-size state is
// read, updated once and written back, whatever the length of the context
// before it (page "Mamba: The State Space Models Challenging the
// Transformer", section "What a state space model actually is").  One step
// of h = exp(Delta A) h + Delta B x with readout y = C h + D x, gated by
// silu(z).  The step is bound by reading and writing
// the fp32 state (8 * dstate bytes per channel).  With 16 states, four
// threads share a channel, each moving 4 states as one 16-byte vector, so a
// warp's loads and stores of its 8 channels are contiguous (512 bytes); the
// readout is summed over the four by shuffles.  Other state sizes take one
// thread per channel.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "device_math.cuh"
#include "scan_fwd.cuh"

namespace sss48 {
namespace {

template <typename InT>
__device__ __forceinline__ float ld(const void *base, int64_t i) {
  return to_f32<InT>(reinterpret_cast<const InT *>(base)[i]);
}

template <typename InT, typename OutT>
__global__ void __launch_bounds__(128) state_update_kernel(const UpdateParams p) {
  const int64_t ch = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (ch >= p.batch * p.dim) return;
  // checked build: every computed index of this channel lies in its tensor
  if (!dbg_index_ok((ch + 1) * p.dstate - 1, p.batch * p.dim * p.dstate, p.status) ||
      !dbg_index_ok((ch % p.dim + 1) * p.dstate - 1, p.dim * p.dstate, p.status) ||
      !dbg_index_ok((ch / p.dim + 1) * p.dstate - 1, p.batch * p.dstate, p.status))
    return;
  const int64_t b = ch / p.dim;
  const int64_t d = ch % p.dim;
  const int nst = static_cast<int>(p.dstate);
  float x = ld<InT>(p.x, ch);
  float s = ld<InT>(p.dt, ch);
  const float gate = p.z ? ld<InT>(p.z, ch) : 1.f;
  const float skip = p.D ? p.D[d] : 0.f;
  if (p.dt_bias) s += p.dt_bias[d];
  const float step = p.softplus ? softplus_f(s) : s;
  const float sx = step * x;
  float *st = p.state + ch * p.dstate;
  float acc = 0.f;
  for (int n = 0; n < nst; ++n) {
    const float a = ex2_mufu(step * p.A[d * p.dstate + n] * kLog2e);
    const float hn = fmaf(a, __ldcs(st + n), sx * ld<InT>(p.B, b * p.dstate + n));
    __stcs(st + n, hn);
    acc = fmaf(ld<InT>(p.C, b * p.dstate + n), hn, acc);
  }
  float yv = fmaf(skip, x, acc);
  if (p.z) yv *= silu_f(gate);
  reinterpret_cast<OutT *>(p.y)[ch] = from_f32<OutT>(yv);
}

// 16 states with the state, A, B and C 16-byte aligned: thread 4 ch + qd
// owns states 4 qd .. 4 qd + 3 of channel ch.  Idx is the index type: 32
// bits when every state index fits (a 64-bit division per thread is a long
// instruction sequence; the kernel is bound by issue, not by DRAM).  With
// ROWS the grid is (channel blocks, batch): the row is blockIdx.y and no
// thread divides at all.
constexpr int kRowsThreads = 128;  // threads of a block on the (channel blocks, rows) grid
template <typename InT, typename OutT, typename Idx, bool ROWS>
__global__ void __launch_bounds__(ROWS ? kRowsThreads : 256) state_update16_kernel(const UpdateParams p) {
  const Idx dim = static_cast<Idx>(p.dim);
  Idx ch;
  int qd;
  bool valid;  // every thread of a channel takes part in the shuffles below
  if constexpr (ROWS) {
    const Idx dl = static_cast<Idx>(blockIdx.x) * (kRowsThreads / 4) + (threadIdx.x >> 2);
    qd = static_cast<int>(threadIdx.x & 3);
    valid = dl < dim;
    ch = static_cast<Idx>(blockIdx.y) * dim + dl;
  } else {
    const Idx gt = static_cast<Idx>(blockIdx.x) * static_cast<Idx>(blockDim.x) + threadIdx.x;
    ch = gt >> 2;
    qd = static_cast<int>(gt & 3);
    valid = static_cast<int64_t>(ch) < p.batch * p.dim;
  }
  if (valid && (!dbg_index_ok((ch + 1) * 16 - 1, p.batch * p.dim * 16, p.status) ||
                !dbg_index_ok((ch % p.dim + 1) * 16 - 1, p.dim * 16, p.status) ||
                !dbg_index_ok((ch / p.dim + 1) * 16 - 1, p.batch * 16, p.status)))
    valid = false;
  const Idx c = valid ? ch : 0;
  Idx b, d;
  if constexpr (ROWS) {
    b = valid ? static_cast<Idx>(blockIdx.y) : 0;
    d = c - b * dim;
  } else {
    b = c / dim;
    d = c - b * dim;
  }
  float acc = 0.f, x = 0.f, gate = 1.f, skip = 0.f;
  if (valid) {
    // every load is issued before the arithmetic (the gate and skip inputs
    // too, by all four threads of the channel), so no thread waits on
    // memory twice
    x = ld<InT>(p.x, c);
    float s = ld<InT>(p.dt, c);
    if (p.z) gate = ld<InT>(p.z, c);
    if (p.D) skip = p.D[d];
    if (p.dt_bias) s += p.dt_bias[d];
    const float step = p.softplus ? softplus_f(s) : s;
    const float sx = step * x;
    float4 *st = reinterpret_cast<float4 *>(p.state + c * 16) + qd;
    // the state is read once and written once: streaming (evict-first)
    // accesses keep it from displacing A, B and C in the caches
    const float4 hv = __ldcs(st);
    const float4 av = reinterpret_cast<const float4 *>(p.A + d * 16)[qd];
    const float4 bv = load4_f32(static_cast<const InT *>(p.B) + b * 16 + 4 * qd);
    const float4 cv = load4_f32(static_cast<const InT *>(p.C) + b * 16 + 4 * qd);
    const float hs[4] = {hv.x, hv.y, hv.z, hv.w}, as[4] = {av.x, av.y, av.z, av.w},
                bs[4] = {bv.x, bv.y, bv.z, bv.w}, cs[4] = {cv.x, cv.y, cv.z, cv.w};
    float ho[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = ex2_mufu(step * as[j] * kLog2e);
      ho[j] = fmaf(a, hs[j], sx * bs[j]);
      acc = fmaf(cs[j], ho[j], acc);
    }
    __stcs(st, make_float4(ho[0], ho[1], ho[2], ho[3]));
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  if (valid && qd == 0) {
    float yv = fmaf(skip, x, acc);
    if (p.z) yv *= silu_f(gate);
    reinterpret_cast<OutT *>(p.y)[c] = from_f32<OutT>(yv);
  }
}

bool aligned16(const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; }

template <typename InT, typename OutT>
cudaError_t launch_typed(const UpdateParams &p, cudaStream_t s) {
  const int64_t n = p.batch * p.dim;
  if (p.dstate == 16 && aligned16(p.state) && aligned16(p.A) && aligned16(p.B) &&
      aligned16(p.C)) {
    const unsigned grid = static_cast<unsigned>((4 * n + 255) / 256);
    // 32-bit indices when the largest state index (16 n) and the thread
    // count (4 n, rounded up to the block) fit; a grid row per batch row
    // when the batch fits the grid's y extent
    const bool fits32 = 16 * n + 256 <= static_cast<int64_t>(UINT32_MAX);
    if (fits32 && p.batch <= 65535) {
      constexpr int cpb = kRowsThreads / 4;  // channels per block
      const dim3 g2(static_cast<unsigned>((p.dim + cpb - 1) / cpb), static_cast<unsigned>(p.batch));
      state_update16_kernel<InT, OutT, uint32_t, true><<<g2, kRowsThreads, 0, s>>>(p);
    } else if (fits32) {
      state_update16_kernel<InT, OutT, uint32_t, false><<<grid, 256, 0, s>>>(p);
    } else {
      state_update16_kernel<InT, OutT, int64_t, false><<<grid, 256, 0, s>>>(p);
    }
  } else {
    const unsigned grid = static_cast<unsigned>((n + 127) / 128);
    state_update_kernel<InT, OutT><<<grid, 128, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const UpdateParams &p, int in_bf16,
                                int out_bf16, cudaStream_t stream) {
  using BF = __nv_bfloat16;
  if (in_bf16)
    return out_bf16 ? launch_typed<BF, BF>(p, stream)
                    : launch_typed<BF, float>(p, stream);
  return out_bf16 ? launch_typed<float, BF>(p, stream)
                  : launch_typed<float, float>(p, stream);
}

}  // namespace sss48
