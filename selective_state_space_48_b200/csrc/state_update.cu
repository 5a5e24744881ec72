// state_update.cu -- single-token selective state update (decode).
//
// Decoding advances the recurrence by one token: the fixed-size state is
// read, updated once and written back, whatever the length of the context
// before it (page "Mamba: The State Space Models Challenging the
// Transformer", section "What a state space model actually is").  One step
// of h = exp(Delta A) h + Delta B x with readout y = C h + D x, gated by
// silu(z).  The step is bound by reading and writing
// the fp32 state (8 * dstate bytes per channel), so one thread owns one
// channel (b, d) and moves its state with 16-byte vector loads and stores.
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

template <typename InT, typename OutT, int N>
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
  if (p.dt_bias) s += p.dt_bias[d];
  const float step = p.softplus ? softplus_f(s) : s;
  const float sx = step * x;
  float *st = p.state + ch * p.dstate;
  float acc = 0.f;
  if (N == 16 && nst == 16 && (reinterpret_cast<uintptr_t>(st) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(p.A) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(p.B) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(p.C) & 15) == 0) {
    // 16 states: the state, A's row and the batch row's B and C move as
    // 16-byte vectors (B, C rows are shared by the channels of a batch row)
    const float *Ad = p.A + d * 16;
    const InT *Bb = static_cast<const InT *>(p.B) + b * 16;
    const InT *Cb = static_cast<const InT *>(p.C) + b * 16;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 hv = reinterpret_cast<const float4 *>(st)[q];
      const float4 av = reinterpret_cast<const float4 *>(Ad)[q];
      const float4 bv = load4_f32(Bb + 4 * q);
      const float4 cv = load4_f32(Cb + 4 * q);
      const float hs[4] = {hv.x, hv.y, hv.z, hv.w}, as[4] = {av.x, av.y, av.z, av.w},
                  bs[4] = {bv.x, bv.y, bv.z, bv.w}, cs[4] = {cv.x, cv.y, cv.z, cv.w};
      float ho[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = ex2_mufu(step * as[j] * kLog2e);
        ho[j] = fmaf(a, hs[j], sx * bs[j]);
        acc = fmaf(cs[j], ho[j], acc);
      }
      reinterpret_cast<float4 *>(st)[q] = make_float4(ho[0], ho[1], ho[2], ho[3]);
    }
  } else {
    for (int n = 0; n < nst; ++n) {
      const float a = ex2_mufu(step * p.A[d * p.dstate + n] * kLog2e);
      const float hn = fmaf(a, st[n], sx * ld<InT>(p.B, b * p.dstate + n));
      st[n] = hn;
      acc = fmaf(ld<InT>(p.C, b * p.dstate + n), hn, acc);
    }
  }
  float yv = acc + (p.D ? p.D[d] : 0.f) * x;
  if (p.z) yv *= silu_f(ld<InT>(p.z, ch));
  reinterpret_cast<OutT *>(p.y)[ch] = from_f32<OutT>(yv);
}

template <typename InT, typename OutT>
cudaError_t launch_typed(const UpdateParams &p, cudaStream_t s) {
  const int64_t n = p.batch * p.dim;
  const unsigned grid = static_cast<unsigned>((n + 127) / 128);
  if (p.dstate == 16)
    state_update_kernel<InT, OutT, 16><<<grid, 128, 0, s>>>(p);
  else
    state_update_kernel<InT, OutT, 0><<<grid, 128, 0, s>>>(p);
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
