// scan_bwd.cu -- backward pass of the selective scan (S6): gradients of
// sum(dy * y) + sum(d_last * last_state) with respect to every input.
//
// The states are not kept from the forward pass; they are recomputed
// ("Mamba is attention all you really need, part 2", section "Keeping the
// pad on the desk"; "The State That Must Remember Everything", Part 3, "The
// Hardware-Aware Way Out", rematerialisation).  One thread block owns 32
// channels (one per lane) of one batch row, one warp per group of 4 states,
// the same layout as the forward kernel:
//
//   forward sweep  walks the sequence in 16-step blocks and writes the state
//                  at the start of every block to the workspace (the only
//                  state that touches HBM: 64 B per channel and block);
//   reverse sweep  walks the blocks backwards; for each it reloads the inputs,
//                  recomputes the states of one half block (8 steps) from
//                  the checkpoint into registers, runs the adjoint
//                  lam_t = ds_t C_t + a_{t+1} lam_{t+1} backwards over them
//                  (re-evaluating each decay a_t), then does the same for
//                  the other half.
//
// With s_t = sum_n C_t[n] h_t[n] + D u_t, g_t = silu(z_t) and y_t = s_t g_t,
// ds_t = dy_t g_t:
//   dDelta_t = sum_n lam_t[n] (A[n] a_t[n] h_{t-1}[n] + B_t[n] u_t)
//   dA[n]   += lam_t[n] Delta_t a_t[n] h_{t-1}[n]
//   dB_t[n] += lam_t[n] Delta_t u_t       dC_t[n] += ds_t h_t[n]
//   du_t     = ds_t D + sum_n lam_t[n] Delta_t B_t[n]
//   dz_t     = dy_t s_t silu'(z_t),  ddelta_t = dDelta_t sigmoid(delta_t + bias)
// Sums over the 16 states go through shared memory (one share per warp);
// dB and dC, which sum over channels, are reduced across the warp's lanes
// by a shuffle reduce-scatter every four steps and added to HBM with one
// atomic per lane pair; dA, dD and dbias, which sum over channels of other
// blocks and over batch rows, with one atomic per channel at the end.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "device_math.cuh"
#include "scan_bwd.cuh"

namespace sss48 {
namespace {

constexpr int CH = 32;
constexpr int TB = 16;
constexpr int ROW = TB + 4;  // padded fp32 row (conflict-free float4 reads)

template <int G>
struct BwdSmem {
  static constexpr int NP = 4 * G;
  // per (channel, step) tiles [CH][ROW]
  float u[CH * ROW], dl[CH * ROW], du[CH * ROW], ds[CH * ROW], sg[CH * ROW],
      z[CH * ROW], dy[CH * ROW];
  // per (state, step) tiles [NP][TB]
  float B[NP * TB], C[NP * TB];
  // per warp shares [G][CH][ROW]: readout s_t, du_t, dDelta_t
  float ps[G * CH * ROW], pu[G * CH * ROW], pd[G * CH * ROW];
  float bias[CH], dskip[CH];
  float accD[CH], accB[CH];  // per-channel sums of ds u and ddelta
};

template <typename T> __device__ __forceinline__ float ld_f32(const T *p, int64_t i);
template <> __device__ __forceinline__ float ld_f32<float>(const float *p, int64_t i) {
  return p[i];
}
template <> __device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16 *p,
                                                                 int64_t i) {
  return __bfloat162float(p[i]);
}

// Component j (a compile-time constant after unrolling) of a float4.
__device__ __forceinline__ float comp(const float4 &v, int j) {
  return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}
__device__ __forceinline__ float4 ld4(const float *p) {
  return *reinterpret_cast<const float4 *>(p);
}

__device__ __forceinline__ float sigmoid_f(float x) {
  return __fdividef(1.0f, 1.0f + ex2_mufu(-x * kLog2e));
}

// silu'(z) = sigmoid(z) (1 + z (1 - sigmoid(z)))
__device__ __forceinline__ float dsilu_f(float z) {
  const float s = sigmoid_f(z);
  return s * fmaf(z, 1.0f - s, 1.0f);
}

// Sum over the 32 lanes of 16 values per lane (v[j], j = 4 i + tq): four
// halving rounds leave lane l with the sum over the 16 lanes that share its
// bit 0 for j = l >> 1; the last exchange completes it (both lanes of a pair
// return the full sum of j = l >> 1).
__device__ __forceinline__ float reduce_scatter16(float (&v)[16], int lane) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int half = 8 >> r;
    const int off = 16 >> r;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float send = upper ? v[j] : v[j + half];
      const float keep = upper ? v[j + half] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

template <typename InT, int G>
__global__ void __launch_bounds__(32 * G, 12 / G)  // 3 blocks of 4 warps per SM
    scan_bwd_kernel(const BwdParams p) {
  using Sm = BwdSmem<G>;
  constexpr int NP = Sm::NP;
  constexpr int NT = 32 * G;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Sm &s = *reinterpret_cast<Sm *>(smem_raw);

  const int tid = threadIdx.x, lane = tid & 31, g = tid >> 5;
  const int64_t tile = blockIdx.x;
  const int64_t b = tile / p.ch_tiles;
  const int64_t d0 = (tile % p.ch_tiles) * CH;
  const int64_t d = d0 + lane;
  const bool dvalid = d < p.dim;
  const int64_t L = p.seqlen;
  const int nblk = static_cast<int>((L + TB - 1) / TB);

  const InT *gu = static_cast<const InT *>(p.u);
  const InT *gd = static_cast<const InT *>(p.delta);
  const InT *gz = static_cast<const InT *>(p.z);
  const InT *gB = static_cast<const InT *>(p.B);
  const InT *gC = static_cast<const InT *>(p.C);

  if (tid < CH) {
    const bool ok = d0 + tid < p.dim;
    s.bias[tid] = (ok && p.delta_bias) ? p.delta_bias[d0 + tid] : 0.f;
    s.dskip[tid] = (ok && p.D) ? p.D[d0 + tid] : 0.f;
    s.accD[tid] = 0.f;
    s.accB[tid] = 0.f;
  }

  float alpha[4], an[4], h[4];
  bool live[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = 4 * g + i;
    live[i] = dvalid && n < p.dstate;
    an[i] = live[i] ? p.A[d * p.dstate + n] : 0.f;
    alpha[i] = an[i] * kLog2e;
    h[i] = (live[i] && p.h0) ? p.h0[(b * p.dim + d) * p.dstate + n] : 0.f;
  }
  // state 4g + i of lane at the start of block k:
  // ckpt[(k * NP + 4g + i) * CH + lane] (coalesced per warp)
  float *ckpt = p.ckpt + tile * static_cast<int64_t>(nblk) * NP * CH;

  // Block k of the inputs into the fp32 tiles with Delta and Delta*u (and,
  // for the reverse sweep, z, dy, ds = dy silu(z), sigmoid(delta + bias)
  // and C) -- all threads.
  auto load_block = [&](int k, bool full) {
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
    for (int idx = tid; idx < CH * TB; idx += NT) {
      const int c = idx / TB, t = idx % TB;
      const int64_t dd = d0 + c;
      const bool ok = dd < p.dim && t < nt;
      const int64_t off = (b * p.dim + dd) * L + t0 + t;
      const float uv = ok ? ld_f32(gu, off) : 0.f;
      const float x = ok ? ld_f32(gd, off) + s.bias[c] : 0.f;
      const float dl = ok ? (p.softplus ? softplus_f(x) : x) : 0.f;
      s.u[c * ROW + t] = uv;
      s.dl[c * ROW + t] = dl;
      s.du[c * ROW + t] = dl * uv;
      if (full) {
        const float zv = (ok && gz) ? ld_f32(gz, off) : 0.f;
        const float dyv = ok ? p.dy[off] : 0.f;
        s.z[c * ROW + t] = zv;
        s.dy[c * ROW + t] = dyv;
        s.ds[c * ROW + t] = gz ? dyv * silu_f(zv) : dyv;
        s.sg[c * ROW + t] = p.softplus ? sigmoid_f(x) : 1.f;
      }
    }
    for (int idx = tid; idx < NP * TB; idx += NT) {
      const int n = idx / TB, t = idx % TB;
      const bool ok = n < p.dstate && t < nt;
      const int64_t off = (b * p.dstate + n) * L + t0 + t;
      s.B[idx] = ok ? ld_f32(gB, off) : 0.f;
      if (full) s.C[idx] = ok ? ld_f32(gC, off) : 0.f;
    }
  };

  // The reverse sweep reads block k - 1 from HBM into registers while block
  // k is computed, and writes it to the tiles at the start of the next
  // iteration: fetch (loads only) and commit (math and shared stores).
  constexpr int E = CH * TB / NT;             // (channel, step) elements per thread
  constexpr int EB = (NP * TB + NT - 1) / NT; // (state, step) elements per thread
  struct Raw {
    float u[E], x[E], z[E], dy[E], B[EB], C[EB];
    unsigned ok;  // bit e: element e lies inside the tensors
  };
  auto fetch = [&](int k, Raw &r) {
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
    r.ok = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = tid + NT * e, c = idx / TB, t = idx % TB;
      const int64_t dd = d0 + c;
      const bool ok = dd < p.dim && t < nt;
      const int64_t off = (b * p.dim + dd) * L + t0 + t;
      r.u[e] = ok ? ld_f32(gu, off) : 0.f;
      r.x[e] = ok ? ld_f32(gd, off) : 0.f;
      r.z[e] = (ok && gz) ? ld_f32(gz, off) : 0.f;
      r.dy[e] = ok ? p.dy[off] : 0.f;
      if (ok) r.ok |= 1u << e;
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int idx = tid + NT * e;
      const int n = idx / TB, t = idx % TB;
      const bool ok = idx < NP * TB && n < p.dstate && t < nt;
      const int64_t off = (b * p.dstate + n) * L + t0 + t;
      r.B[e] = ok ? ld_f32(gB, off) : 0.f;
      r.C[e] = ok ? ld_f32(gC, off) : 0.f;
    }
  };
  auto commit = [&](const Raw &r) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = tid + NT * e, c = idx / TB, t = idx % TB;
      const bool ok = (r.ok >> e) & 1u;
      const float x = ok ? r.x[e] + s.bias[c] : 0.f;
      const float dl = ok ? (p.softplus ? softplus_f(x) : x) : 0.f;
      s.u[c * ROW + t] = r.u[e];
      s.dl[c * ROW + t] = dl;
      s.du[c * ROW + t] = dl * r.u[e];
      s.z[c * ROW + t] = r.z[e];
      s.dy[c * ROW + t] = r.dy[e];
      s.ds[c * ROW + t] = gz ? r.dy[e] * silu_f(r.z[e]) : r.dy[e];
      s.sg[c * ROW + t] = p.softplus ? sigmoid_f(x) : 1.f;
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int idx = tid + NT * e;
      if (idx < NP * TB) {
        s.B[idx] = r.B[e];
        s.C[idx] = r.C[e];
      }
    }
  };

  // ------------------------------------------------------ forward sweep
  // (skipped when the forward scan already wrote the checkpoints)
  __syncthreads();
  for (int k = 0; k < (p.ckpt_given ? 0 : nblk); ++k) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      ckpt[(static_cast<int64_t>(k) * NP + 4 * g + i) * CH + lane] = h[i];
    load_block(k, false);
    __syncthreads();
#pragma unroll
    for (int q = 0; q < TB / 4; ++q) {
      const float4 dl4 = ld4(&s.dl[lane * ROW + 4 * q]), du4 = ld4(&s.du[lane * ROW + 4 * q]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 b4 = ld4(&s.B[(4 * g + i) * TB + 4 * q]);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          h[i] = fmaf(ex2_mufu(comp(dl4, j) * alpha[i]), h[i], comp(du4, j) * comp(b4, j));
      }
    }
    __syncthreads();
  }

  // ------------------------------------------------------ reverse sweep
  float lam[4], dA[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lam[i] = (live[i] && p.d_last)
                 ? p.d_last[(b * p.dim + d) * p.dstate + 4 * g + i] : 0.f;
    dA[i] = 0.f;
  }
  // the checkpoint of the block after the current one is read a block early
  float hnext[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    hnext[i] = ckpt[(static_cast<int64_t>(nblk - 1) * NP + 4 * g + i) * CH + lane];
  Raw raw;
  fetch(nblk - 1, raw);
  for (int k = nblk - 1; k >= 0; --k) {
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
    commit(raw);
    float hc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hc[i] = hnext[i];
      if (k > 0) hnext[i] = ckpt[(static_cast<int64_t>(k - 1) * NP + 4 * g + i) * CH + lane];
    }
    __syncthreads();
    if (k > 0) fetch(k - 1, raw);  // in flight while block k is computed

    // Two halves of the block, the later one first.  For each: recompute
    // the states of its 8 steps from the checkpoint into registers (with
    // this warp's share of the readout s_t), then run the adjoint backwards
    // over them.  Keeping 8 steps instead of 16 halves the registers the
    // states need, for half a block of extra recomputation.
#pragma unroll
    for (int half = 1; half >= 0; --half) {
      const int tb = 8 * half;  // first step of this half
      float hs[4][8], hpre[4];  // states of steps tb..tb+7 and of step tb-1
      float hh[4] = {hc[0], hc[1], hc[2], hc[3]};
#pragma unroll
      for (int q = 0; q < tb / 4 + 2; ++q) {
        const float4 dl4 = ld4(&s.dl[lane * ROW + 4 * q]), du4 = ld4(&s.du[lane * ROW + 4 * q]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 b4 = ld4(&s.B[(4 * g + i) * TB + 4 * q]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int t = 4 * q + j;
            if (t == tb) hpre[i] = hh[i];
            hh[i] = fmaf(ex2_mufu(comp(dl4, j) * alpha[i]), hh[i], comp(du4, j) * comp(b4, j));
            if (t >= tb) hs[i][t - tb] = hh[i];
          }
        }
      }
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 c4 = ld4(&s.C[(4 * g + i) * TB + tb + 4 * qq]);
          acc.x = fmaf(c4.x, hs[i][4 * qq + 0], acc.x);
          acc.y = fmaf(c4.y, hs[i][4 * qq + 1], acc.y);
          acc.z = fmaf(c4.z, hs[i][4 * qq + 2], acc.z);
          acc.w = fmaf(c4.w, hs[i][4 * qq + 3], acc.w);
        }
        *reinterpret_cast<float4 *>(&s.ps[(g * CH + lane) * ROW + tb + 4 * qq]) = acc;
      }

      // adjoint, four steps at a time backwards
#pragma unroll
      for (int qq = 1; qq >= 0; --qq) {
        const int q = 2 * half + qq;
        float vB[16], vC[16];
        const int t4 = tb + 4 * qq;  // first step of this quad
        const float4 dl4 = ld4(&s.dl[lane * ROW + t4]), u4 = ld4(&s.u[lane * ROW + t4]),
                     ds4 = ld4(&s.ds[lane * ROW + t4]);
        float4 B4[4], C4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          B4[i] = ld4(&s.B[(4 * g + i) * TB + t4]);
          C4[i] = ld4(&s.C[(4 * g + i) * TB + t4]);
        }
        float4 pu4, pd4;
#pragma unroll
        for (int tq = 3; tq >= 0; --tq) {
          const int tl = 4 * qq + tq;  // step within the half
          const float dl = comp(dl4, tq), uu = comp(u4, tq), ds = comp(ds4, tq);
          float pdu = 0.f, pdd = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float Bv = comp(B4[i], tq), Cv = comp(C4[i], tq);
            const float hprev = tl > 0 ? hs[i][tl - 1] : hpre[i];
            const float a = ex2_mufu(dl * alpha[i]);
            lam[i] = fmaf(ds, Cv, lam[i]);
            vC[4 * i + tq] = ds * hs[i][tl];
            const float la = lam[i] * a * hprev;
            pdd = fmaf(lam[i], Bv * uu, fmaf(la, an[i], pdd));
            dA[i] = fmaf(la, dl, dA[i]);
            vB[4 * i + tq] = lam[i] * dl * uu;
            pdu = fmaf(lam[i] * dl, Bv, pdu);
            lam[i] *= a;
          }
          if (tq == 0) { pu4.x = pdu; pd4.x = pdd; }
          if (tq == 1) { pu4.y = pdu; pd4.y = pdd; }
          if (tq == 2) { pu4.z = pdu; pd4.z = pdd; }
          if (tq == 3) { pu4.w = pdu; pd4.w = pdd; }
        }
        *reinterpret_cast<float4 *>(&s.pu[(g * CH + lane) * ROW + t4]) = pu4;
        *reinterpret_cast<float4 *>(&s.pd[(g * CH + lane) * ROW + t4]) = pd4;
        // channel sums of dB, dC for states 4g + i, steps 4q + tq: the even
        // lane of each pair adds j = lane >> 1 = 4 i + tq
        const float rb = reduce_scatter16(vB, lane);
        const float rc = reduce_scatter16(vC, lane);
        const int j = lane >> 1, n = 4 * g + j / 4, t = 4 * q + j % 4;
        if ((lane & 1) == 0 && n < p.dstate && t < nt) {
          const int64_t off = (b * p.dstate + n) * L + t0 + t;
          atomicAdd(p.dB + off, rb);
          atomicAdd(p.dC + off, rc);
        }
      }
    }
    __syncthreads();

    // elementwise: du, ddelta, dz, and the per-channel sums of dD, dbias
    for (int idx = tid; idx < CH * TB; idx += NT) {
      const int c = idx / TB, t = idx % TB;
      const int64_t dd = d0 + c;
      if (dd >= p.dim || t >= nt) continue;
      float sp = 0.f, su = 0.f, sd = 0.f;
#pragma unroll
      for (int w = 0; w < G; ++w) {
        sp += s.ps[(w * CH + c) * ROW + t];
        su += s.pu[(w * CH + c) * ROW + t];
        sd += s.pd[(w * CH + c) * ROW + t];
      }
      const float uu = s.u[c * ROW + t], ds = s.ds[c * ROW + t];
      const int64_t off = (b * p.dim + dd) * L + t0 + t;
      p.du[off] = fmaf(ds, s.dskip[c], su);
      const float ddl = sd * s.sg[c * ROW + t];
      p.ddelta[off] = ddl;
      if (p.dz) {
        const float sv = fmaf(s.dskip[c], uu, sp);
        p.dz[off] = s.dy[c * ROW + t] * sv * dsilu_f(s.z[c * ROW + t]);
      }
      atomicAdd(&s.accD[c], ds * uu);
      atomicAdd(&s.accB[c], ddl);
    }
    __syncthreads();
  }

  // parameter gradients, summed over batch rows (and dh0 = lam_{-1})
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (!live[i]) continue;
    const int n = 4 * g + i;
    atomicAdd(p.dA + d * p.dstate + n, dA[i]);
    if (p.dh0) p.dh0[(b * p.dim + d) * p.dstate + n] = lam[i];
  }
  if (tid < CH && d0 + tid < p.dim) {
    if (p.dD) atomicAdd(p.dD + d0 + tid, s.accD[tid]);
    if (p.ddelta_bias) atomicAdd(p.ddelta_bias + d0 + tid, s.accB[tid]);
  }
}

template <typename InT, int G>
cudaError_t launch_typed(const BwdParams &p, cudaStream_t stream) {
  auto kern = scan_bwd_kernel<InT, G>;
  const int smem = static_cast<int>(sizeof(BwdSmem<G>));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(p.tiles), 32 * G, smem, stream>>>(p);
  return cudaGetLastError();
}

template <typename InT>
cudaError_t dispatch(const BwdParams &p, cudaStream_t stream) {
  switch (bwd_groups(p.dstate)) {
    case 1: return launch_typed<InT, 1>(p, stream);
    case 2: return launch_typed<InT, 2>(p, stream);
    default: return launch_typed<InT, 4>(p, stream);
  }
}

}  // namespace
}  // namespace sss48

namespace sss48 {

int bwd_groups(int64_t dstate) {
  const int g = static_cast<int>((dstate + 3) / 4);
  return g <= 1 ? 1 : (g == 2 ? 2 : 4);
}

size_t scan_bwd_workspace_bytes(int64_t tiles, int64_t seqlen, int64_t dstate) {
  const int64_t nblk = (seqlen + kBwdTimeBlock - 1) / kBwdTimeBlock;
  return static_cast<size_t>(tiles) * static_cast<size_t>(nblk) *
         static_cast<size_t>(4 * bwd_groups(dstate)) * kBwdChannels * sizeof(float);
}

cudaError_t launch_scan_bwd(const BwdParams &p, int in_bf16, cudaStream_t stream) {
  return in_bf16 ? dispatch<__nv_bfloat16>(p, stream) : dispatch<float>(p, stream);
}

}  // namespace sss48
