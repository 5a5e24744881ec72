// scan_fwd.cu -- forward selective scan (S6) for sm_100a.
//
// One thread block handles 32 consecutive channels d of one batch row b and
// a chunk of the sequence.  Lane l of warp g owns channel d0 + l and the
// states n = 4g .. 4g+3, whose fp32 values h[n] stay in registers for the
// whole chunk ("Keeping the pad on the desk": the state never goes back to
// HBM; only y is written).  Time is walked in blocks of 32 steps:
//
//   prep   every (channel, t) of the block computes, once,
//          Delta = softplus(delta + delta_bias), Delta*u, D*u and silu(z),
//          and B_t[n], C_t[n] are widened to fp32 -- all into shared memory;
//   scan   each lane runs h = exp(Delta A) h + Delta B u over the 32 steps
//          for its 4 states and forms its share of y_t = sum_n C_t[n] h_t[n]
//          (page "The State That Must Remember Everything", "The Equation",
//          with the exponential-Euler discretisation of its Part 7);
//   epilogue the shares of the state groups are summed, the D*u skip added,
//          the silu(z) gate applied and y stored, coalesced along t.
//
// Long sequences with few channels are split into chunks that run in
// parallel ("The relay": fade-and-add steps compose associatively, so a
// chunk can be squashed into one pair (P, e) = (prod exp(Delta A), state
// reached from zero) without knowing the state it starts from).  A chunk
// publishes (P, e), looks back over its predecessors' pairs to obtain the
// true state h_in at its start (decoupled look-back, each wait bounded), and
// then adds the missing term sum_n C_t[n] exp(A[n] sigma_t) h_in[n] to the
// outputs it has written, until that term has decayed below 2^-64 of h_in
// (sigma_t is the running sum of Delta from the chunk start).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "device_math.cuh"
#include "scan_fwd.cuh"

namespace sss48 {
namespace {

constexpr int CH = kChannelsPerBlock;
constexpr int TB = kTimeBlock;
constexpr int ROW = TB + 4;  // padded row: lanes reading float4 at row l hit
                             // distinct bank groups
constexpr float kCutoffLog2 = -64.0f;

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) {
  return a < b ? a : b;
}

struct Smem {
  // offsets in floats into dynamic shared memory
  static constexpr int delta = 0;
  static constexpr int du = delta + CH * ROW;
  static constexpr int skip = du + CH * ROW;
  static constexpr int gate = skip + CH * ROW;
  static constexpr int part = gate + CH * ROW;
  // followed by part[G][CH][ROW], then sB[NP][TB], sC[NP][TB]
  static constexpr int bytes(int G) {
    return (part + G * CH * ROW + 2 * 4 * G * TB) * 4;
  }
};

template <typename InT>
__device__ __forceinline__ float ld_in(const void *base, int64_t idx) {
  return to_f32<InT>(reinterpret_cast<const InT *>(base)[idx]);
}

// Fill the shared-memory tiles of one time block [t0, t0 + nt).
template <typename InT, int G, bool HAS_Z>
__device__ __forceinline__ void prep_block(const ScanParams &p, float *sm,
                                           int64_t b, int64_t d0, int64_t t0,
                                           int nt, bool with_skip) {
  constexpr int NT = 32 * G;
  constexpr int NP = 4 * G;
  const int tid = threadIdx.x;
  float *sDelta = sm + Smem::delta;
  float *sDu = sm + Smem::du;
  float *sSkip = sm + Smem::skip;
  float *sGate = sm + Smem::gate;
  float *sB = sm + Smem::part + G * CH * ROW;
  float *sC = sB + NP * TB;
#pragma unroll 4
  for (int idx = tid; idx < CH * TB; idx += NT) {
    const int c = idx / TB;
    const int t = idx % TB;
    const int64_t d = d0 + c;
    float dl = 0.f, u = 0.f, g = 1.f, dskip = 0.f;
    if (d < p.dim && t < nt) {
      const int64_t off = (b * p.dim + d) * p.seqlen + t0 + t;
      u = ld_in<InT>(p.u, off);
      float x = ld_in<InT>(p.delta, off);
      if (p.delta_bias) x += p.delta_bias[d];
      dl = p.softplus ? softplus_f(x) : x;
      if (HAS_Z) g = silu_f(ld_in<InT>(p.z, off));
      if (p.D) dskip = p.D[d];
    }
    sDelta[c * ROW + t] = dl;
    sDu[c * ROW + t] = dl * u;
    if (with_skip) sSkip[c * ROW + t] = dskip * u;
    if (HAS_Z) sGate[c * ROW + t] = g;
  }
#pragma unroll 4
  for (int idx = tid; idx < NP * TB; idx += NT) {
    const int n = idx / TB;
    const int t = idx % TB;
    float bv = 0.f, cv = 0.f;
    if (n < p.dstate && t < nt) {
      const int64_t off = (b * p.dstate + n) * p.seqlen + t0 + t;
      bv = ld_in<InT>(p.B, off);
      cv = ld_in<InT>(p.C, off);
    }
    sB[n * TB + t] = bv;
    sC[n * TB + t] = cv;
  }
}

// Sum the state-group shares of y for the block and store (or accumulate
// into) y.
template <typename OutT, int G, bool HAS_Z, bool ACCUMULATE>
__device__ __forceinline__ void epilogue_block(const ScanParams &p, float *sm,
                                               int64_t b, int64_t d0,
                                               int64_t t0, int nt) {
  constexpr int NT = 32 * G;
  const float *sPart = sm + Smem::part;
  const float *sSkip = sm + Smem::skip;
  const float *sGate = sm + Smem::gate;
  OutT *y = reinterpret_cast<OutT *>(p.y);
  for (int idx = threadIdx.x; idx < CH * TB; idx += NT) {
    const int c = idx / TB;
    const int t = idx % TB;
    const int64_t d = d0 + c;
    if (d >= p.dim || t >= nt) continue;
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) s += sPart[(g * CH + c) * ROW + t];
    const int64_t off = (b * p.dim + d) * p.seqlen + t0 + t;
    if (ACCUMULATE) {
      if (HAS_Z) s *= sGate[c * ROW + t];
      y[off] = from_f32<OutT>(to_f32<OutT>(y[off]) + s);
    } else {
      s += sSkip[c * ROW + t];
      if (HAS_Z) s *= sGate[c * ROW + t];
      y[off] = from_f32<OutT>(s);
    }
  }
}

template <typename InT, typename OutT, int G, bool HAS_Z, bool SPLIT>
__global__ void __launch_bounds__(32 * G)
    scan_fwd_kernel(const ScanParams p) {
  extern __shared__ __align__(16) float sm[];
  constexpr int NP = 4 * G;
  __shared__ int s_item;
  __shared__ unsigned s_flag;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int g = tid >> 5;  // state group of this warp

  int64_t item;
  if (SPLIT) {
    if (tid == 0) s_item = static_cast<int>(atomicAdd(p.ticket, 1u));
    __syncthreads();
    item = s_item;
  } else {
    item = blockIdx.x;
  }
  const int64_t k = item / p.tiles;  // sequence chunk (chunk-major order)
  const int64_t tile = item % p.tiles;
  const int64_t b = tile / p.ch_tiles;
  const int64_t d0 = (tile % p.ch_tiles) * CH;
  const int64_t d = d0 + lane;
  const bool dvalid = d < p.dim;
  const int64_t t_begin = k * p.chunk;
  const int64_t t_end = min64(t_begin + p.chunk, p.seqlen);

  float alpha[4], h[4];
  bool live[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = 4 * g + i;
    live[i] = dvalid && n < p.dstate;
    alpha[i] = live[i] ? p.A[d * p.dstate + n] * kLog2e : 0.f;
    h[i] = (live[i] && k == 0 && p.h0) ? p.h0[(b * p.dim + d) * p.dstate + n]
                                       : 0.f;
  }
  float dsum = 0.f;

  const float *sDelta = sm + Smem::delta;
  const float *sDu = sm + Smem::du;
  float *sPart = sm + Smem::part;
  const float *sB = sm + Smem::part + G * CH * ROW;
  const float *sC = sB + NP * TB;

  for (int64_t t0 = t_begin; t0 < t_end; t0 += TB) {
    const int nt = static_cast<int>(min64(TB, t_end - t0));
    __syncthreads();
    prep_block<InT, G, HAS_Z>(p, sm, b, d0, t0, nt, true);
    __syncthreads();
    const int nq = (nt + 3) >> 2;
    for (int q = 0; q < nq; ++q) {
      const float4 dl = *reinterpret_cast<const float4 *>(&sDelta[lane * ROW + 4 * q]);
      const float4 du = *reinterpret_cast<const float4 *>(&sDu[lane * ROW + 4 * q]);
      const float dls[4] = {dl.x, dl.y, dl.z, dl.w};
      const float dus[4] = {du.x, du.y, du.z, du.w};
      float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = 4 * g + i;
        const float4 bq = *reinterpret_cast<const float4 *>(&sB[n * TB + 4 * q]);
        const float4 cq = *reinterpret_cast<const float4 *>(&sC[n * TB + 4 * q]);
        const float bs[4] = {bq.x, bq.y, bq.z, bq.w};
        const float cs[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a = ex2_mufu(dls[j] * alpha[i]);
          h[i] = fmaf(a, h[i], dus[j] * bs[j]);
          part[j] = fmaf(cs[j], h[i], part[j]);
        }
      }
      *reinterpret_cast<float4 *>(&sPart[(g * CH + lane) * ROW + 4 * q]) =
          make_float4(part[0], part[1], part[2], part[3]);
      if (SPLIT) dsum += (dls[0] + dls[1]) + (dls[2] + dls[3]);
    }
    __syncthreads();
    epilogue_block<OutT, G, HAS_Z, false>(p, sm, b, d0, t0, nt);
  }

  if (!SPLIT) {
    if (p.last_state) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (live[i]) p.last_state[(b * p.dim + d) * p.dstate + 4 * g + i] = h[i];
    }
    return;
  }

  // ---- split mode: publish, look back, publish the true end state, correct
  const int64_t stride = static_cast<int64_t>(2) * CH * NP;
  float *my_agg = p.agg + item * stride;
  float *my_incl = p.incl + item * static_cast<int64_t>(CH * NP);
  const bool drop = (p.test_flags & 1u) && k == 1 && tile == 0;
  float P[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) P[i] = ex2_mufu(alpha[i] * dsum);

  float h_in[4] = {0.f, 0.f, 0.f, 0.f};
  if (k == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) my_incl[(4 * g + i) * CH + lane] = h[i];
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      my_agg[(4 * g + i) * CH + lane] = P[i];
      my_agg[CH * NP + (4 * g + i) * CH + lane] = h[i];
    }
    __syncthreads();
    if (tid == 0 && !drop) {
      __threadfence();
      st_release_gpu(&p.flags[item], 1u);
    }
    float pacc[4] = {1.f, 1.f, 1.f, 1.f};
    for (int64_t j = k - 1; j >= 0; --j) {
      const int64_t pred = j * p.tiles + tile;
      if (tid == 0) {
        unsigned f = ld_acquire_gpu(&p.flags[pred]);
        const uint64_t start = global_timer_ns();
        const uint64_t limit = p.spin_timeout_ns > 0
                                   ? static_cast<uint64_t>(p.spin_timeout_ns)
                                   : 1000000000ull;
        for (uint32_t it = 0; f == 0u; ++it) {
          if ((it > 64u && global_timer_ns() - start > limit) || it > (1u << 30)) {
            atomicOr(p.status, kStatusTimeout);
            break;
          }
          __nanosleep(128);
          f = ld_acquire_gpu(&p.flags[pred]);
        }
        s_flag = f;
      }
      __syncthreads();
      const unsigned f = s_flag;
      bool done = true;
      if (f == 2u) {
        const float *pi = p.incl + pred * static_cast<int64_t>(CH * NP);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          h_in[i] = fmaf(pacc[i], __ldcg(&pi[(4 * g + i) * CH + lane]), h_in[i]);
      } else if (f == 1u) {
        const float *pa = p.agg + pred * stride;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          h_in[i] = fmaf(pacc[i], __ldcg(&pa[CH * NP + (4 * g + i) * CH + lane]), h_in[i]);
          pacc[i] *= __ldcg(&pa[(4 * g + i) * CH + lane]);
          if (live[i] && pacc[i] != 0.f) done = false;
        }
      }
      if (__syncthreads_and(done)) break;
    }
    // the true state at the end of this chunk: P * h_in + e
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      h[i] = fmaf(P[i], h_in[i], h[i]);
      my_incl[(4 * g + i) * CH + lane] = h[i];
    }
  }
  __syncthreads();
  if (tid == 0 && !drop) {
    __threadfence();
    st_release_gpu(&p.flags[item], 2u);
  }
  if (p.last_state && t_end == p.seqlen) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (live[i]) p.last_state[(b * p.dim + d) * p.dstate + 4 * g + i] = h[i];
  }
  if (k == 0) return;

  // correction: y_t += silu(z_t) * sum_n C_t[n] 2^(alpha[n] sigma_t) h_in[n]
  float sigma = 0.f;
  for (int64_t t0 = t_begin; t0 < t_end; t0 += TB) {
    bool need = false;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      need |= live[i] && h_in[i] != 0.f && !(alpha[i] * sigma < kCutoffLog2);
    if (!__syncthreads_or(need)) break;
    const int nt = static_cast<int>(min64(TB, t_end - t0));
    prep_block<InT, G, HAS_Z>(p, sm, b, d0, t0, nt, false);
    __syncthreads();
    const int nq = (nt + 3) >> 2;
    for (int q = 0; q < nq; ++q) {
      const float4 dl = *reinterpret_cast<const float4 *>(&sDelta[lane * ROW + 4 * q]);
      const float dls[4] = {dl.x, dl.y, dl.z, dl.w};
      float part[4] = {0.f, 0.f, 0.f, 0.f};
      float sig[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sigma += dls[j];
        sig[j] = sigma;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = 4 * g + i;
        const float4 cq = *reinterpret_cast<const float4 *>(&sC[n * TB + 4 * q]);
        const float cs[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          part[j] = fmaf(cs[j] * ex2_mufu(alpha[i] * sig[j]), h_in[i], part[j]);
      }
      *reinterpret_cast<float4 *>(&sPart[(g * CH + lane) * ROW + 4 * q]) =
          make_float4(part[0], part[1], part[2], part[3]);
    }
    __syncthreads();
    epilogue_block<OutT, G, HAS_Z, true>(p, sm, b, d0, t0, nt);
    __syncthreads();
  }
}

template <typename InT, typename OutT, int G, bool HAS_Z, bool SPLIT>
cudaError_t launch_typed(const ScanParams &p, cudaStream_t stream) {
  auto kern = scan_fwd_kernel<InT, OutT, G, HAS_Z, SPLIT>;
  const int smem = Smem::bytes(G);
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.tiles * p.splits;
  kern<<<static_cast<unsigned>(grid), 32 * G, smem, stream>>>(p);
  return cudaGetLastError();
}

template <typename InT, typename OutT, int G>
cudaError_t dispatch_z(const ScanParams &p, int has_z, cudaStream_t s) {
  const bool split = p.splits > 1;
  if (has_z)
    return split ? launch_typed<InT, OutT, G, true, true>(p, s)
                 : launch_typed<InT, OutT, G, true, false>(p, s);
  return split ? launch_typed<InT, OutT, G, false, true>(p, s)
               : launch_typed<InT, OutT, G, false, false>(p, s);
}

template <typename InT, typename OutT>
cudaError_t dispatch_g(const ScanParams &p, int has_z, cudaStream_t s) {
  const int G = static_cast<int>((p.dstate + 3) / 4);
  switch (G) {
    case 1: return dispatch_z<InT, OutT, 1>(p, has_z, s);
    case 2: return dispatch_z<InT, OutT, 2>(p, has_z, s);
    case 3: return dispatch_z<InT, OutT, 3>(p, has_z, s);
    default: return dispatch_z<InT, OutT, 4>(p, has_z, s);
  }
}

template <typename InT, typename OutT, int G, bool HAS_Z, bool SPLIT>
int occupancy_typed() {
  int n = 0;
  auto kern = scan_fwd_kernel<InT, OutT, G, HAS_Z, SPLIT>;
  const int smem = Smem::bytes(G);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * G, smem) !=
      cudaSuccess)
    return 1;
  return std::max(n, 1);
}

}  // namespace

size_t scan_workspace_clear_bytes(int64_t tiles, int splits) {
  const size_t items = static_cast<size_t>(tiles) * splits;
  return 256 + ((items * sizeof(unsigned) + 255) / 256) * 256;
}

size_t scan_workspace_bytes(int64_t tiles, int splits, int groups) {
  if (splits <= 1) return 0;
  const size_t items = static_cast<size_t>(tiles) * splits;
  const size_t np = 4 * static_cast<size_t>(groups);
  const size_t agg = items * 2 * CH * np * sizeof(float);
  const size_t incl = items * CH * np * sizeof(float);
  return scan_workspace_clear_bytes(tiles, splits) + ((agg + 255) / 256) * 256 +
         ((incl + 255) / 256) * 256;
}

void scan_bind_workspace(ScanParams &p, void *ws, int groups) {
  char *base = static_cast<char *>(ws);
  const size_t items = static_cast<size_t>(p.tiles) * p.splits;
  const size_t np = 4 * static_cast<size_t>(groups);
  p.status = reinterpret_cast<unsigned *>(base);
  p.ticket = reinterpret_cast<unsigned *>(base + 4);
  p.flags = reinterpret_cast<unsigned *>(base + 256);
  const size_t clear = scan_workspace_clear_bytes(p.tiles, p.splits);
  p.agg = reinterpret_cast<float *>(base + clear);
  const size_t agg = ((items * 2 * CH * np * sizeof(float) + 255) / 256) * 256;
  p.incl = reinterpret_cast<float *>(base + clear + agg);
}

int scan_blocks_per_sm(int in_bf16, int out_bf16, int has_z, int groups,
                       int split) {
  // Occupancy depends on registers and shared memory only; the z / split
  // variants are close enough that the z = true, split = false kernel
  // stands in for all of them.
  (void)has_z;
  (void)split;
  using BF = __nv_bfloat16;
  switch ((in_bf16 ? 2 : 0) + (out_bf16 ? 1 : 0)) {
    case 0:
      switch (groups) {
        case 1: return occupancy_typed<float, float, 1, true, false>();
        case 2: return occupancy_typed<float, float, 2, true, false>();
        case 3: return occupancy_typed<float, float, 3, true, false>();
        default: return occupancy_typed<float, float, 4, true, false>();
      }
    case 1:
      return occupancy_typed<float, BF, 4, true, false>();
    case 2:
      switch (groups) {
        case 1: return occupancy_typed<BF, float, 1, true, false>();
        case 2: return occupancy_typed<BF, float, 2, true, false>();
        case 3: return occupancy_typed<BF, float, 3, true, false>();
        default: return occupancy_typed<BF, float, 4, true, false>();
      }
    default:
      return occupancy_typed<BF, BF, 4, true, false>();
  }
}

cudaError_t launch_scan_fwd(const ScanParams &p, int in_bf16, int out_bf16,
                            int has_z, cudaStream_t stream) {
  using BF = __nv_bfloat16;
  if (in_bf16)
    return out_bf16 ? dispatch_g<BF, BF>(p, has_z, stream)
                    : dispatch_g<BF, float>(p, has_z, stream);
  return out_bf16 ? dispatch_g<float, BF>(p, has_z, stream)
                  : dispatch_g<float, float>(p, has_z, stream);
}

}  // namespace sss48
