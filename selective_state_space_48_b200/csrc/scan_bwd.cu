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
//   reverse sweep  walks the blocks backwards; for each, the later half
//                  (8 steps) first: recompute the states from the block's
//                  checkpoint, keeping each step's state and decay a_t of the
//                  half in registers, then run the adjoint
//                  lam_t = ds_t C_t + a_{t+1} lam_{t+1} backwards over them
//                  with the kept decays (no exponential is evaluated twice
//                  within a half); then the earlier half the same way.
//
// Packed sequences (their own instantiation) take exp(Delta A) = 0 at every
// sequence start, in the forward sweep and the recompute alike: the state
// entering the start is then empty and the adjoint's lam_{t-1} = a_t lam_t
// gets nothing across it.  The inputs may be strided views (time
// contiguous); the gradients are packed.
//
// The arithmetic pairs the lane's states: two states advance together in
// one f32x2 instruction, so B_t and C_t sit in shared memory step-major
// ([t][n]) and a warp reads the four values of its states with one
// warp-uniform 16-byte load.
//
// With s_t = sum_n C_t[n] h_t[n] + D u_t, g_t = silu(z_t) and y_t = s_t g_t,
// ds_t = dy_t g_t, and the per-step sums over states
// Pb_t = sum_n lam_t[n] B_t[n], Pa_t = sum_n lam_t[n] A[n] a_t[n] h_{t-1}[n]:
//   du_t      = Delta_t Pb_t + ds_t D
//   dDelta_t  = Pa_t + u_t Pb_t,          ddelta_t = dDelta_t sigmoid(delta_t + bias)
//   dA[n]    += lam_t[n] Delta_t a_t[n] h_{t-1}[n]
//   dB_t[n]  += lam_t[n] Delta_t u_t,     dC_t[n] += ds_t h_t[n]
//   dz_t      = dy_t s_t silu'(z_t)
// Sums over the 16 states go through shared memory (one share per warp);
// dB and dC, which sum over channels, are reduced across the warp's lanes
// by a shuffle reduce-scatter every four steps and added to HBM with one
// atomic per lane pair; dA, dD and dbias, which sum over channels of other
// blocks and over batch rows, with one atomic per channel at the end.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "device_math.cuh"
#include "scan_bwd.cuh"

namespace sss48 {
namespace {

constexpr int CH = 32;
constexpr int TB = 16;
constexpr int ROW = TB + 4;  // padded fp32 row (conflict-free float4 reads)

// The fp32 tiles of one 16-step block (16-byte aligned: the tiles are
// read as float4, also in the second of two consecutive sets).
template <int G>
struct alignas(16) BwdTiles {
  static constexpr int NP = 4 * G;
  // per (channel, step) tiles [CH][ROW]; gz = dy silu'(z), so that
  // dz = gz s with s the readout (incl. D u)
  float u[CH * ROW], dl[CH * ROW], du[CH * ROW], ds[CH * ROW], sg[CH * ROW],
      gz[CH * ROW];
  // per (step, state) tiles [TB][NP]: a warp's four states are adjacent
  float B[TB * NP], C[TB * NP];
  // packed sequences: bit t set when step t of the block starts a sequence
  unsigned rmask;
};

// The raw inputs of one 16-step block as they lie in HBM (bf16 u, delta,
// z, B, C; fp32 dy), rows of 16 steps: the reverse sweep copies block k - 1
// here asynchronously while block k is computed.
template <int G>
struct BwdStage {
  static constexpr int NP = 4 * G;
  __nv_bfloat16 u[CH * TB], x[CH * TB], z[CH * TB];
  float dy[CH * TB];
  __nv_bfloat16 B[NP * TB], C[NP * TB];
};

template <int G>
struct BwdSmem {
  static constexpr int NP = 4 * G;
  static_assert(sizeof(BwdTiles<G>) % 16 == 0, "tile sets keep 16-byte alignment");
  // two sets of tiles: block k is computed from set k & 1 while the other
  // set still serves block k + 1's epilogue
  BwdTiles<G> tl[2];
  // per warp shares [G][CH][ROW]: readout s_t, Pb_t, Pa_t
  float ps[G * CH * ROW], pb[G * CH * ROW], pa[G * CH * ROW];
  float bias[CH], dskip[CH];
  float accD[CH], accB[CH];  // per-channel sums of ds u and ddelta
  alignas(16) BwdStage<G> st;  // bf16 inputs only
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
__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 ex2_pair(float2 x) {
  return make_float2(ex2_mufu(x.x), ex2_mufu(x.y));
}

// 16-byte asynchronous copy global -> shared (through L2 only), tracked by
// the thread's groups
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ bool aligned16(const void *q) {
  return (reinterpret_cast<uintptr_t>(q) & 15) == 0;
}

__device__ __forceinline__ float sigmoid_f(float x) {
  return __fdividef(1.0f, 1.0f + ex2_mufu(-x * kLog2e));
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

// Bit t (t < 16) set when step t0 + t (< L) is an interior sequence start.
// `nb` is the caller's cursor into cu (1 .. nseq), moved to the first
// interior start at or after t0: blocks are visited in order, forwards in the
// forward sweep and backwards in the reverse sweep, so it moves a step or two.
__device__ unsigned restart_mask(const BwdParams &p, int64_t t0, int64_t L, int64_t &nb) {
  while (nb > 1 && __ldg(p.cu + nb - 1) >= t0) --nb;
  while (nb < p.nseq && __ldg(p.cu + nb) < t0) ++nb;
  unsigned m = 0u;
  for (int64_t i = nb; i < p.nseq; ++i) {
    const int64_t t = __ldg(p.cu + i) - t0;
    if (t >= kBwdTimeBlock || t0 + t >= L) break;
    m |= 1u << t;
  }
  return m;
}

// Work item of a block under the cut schedule: tile and blocks [kb0, kb1),
// piece -1 (a whole tile), 0 (the first part's forward sweep), 1 (the
// second part: its forward sweep unless the checkpoints are given, and its
// reverse sweep) or 2 (the first part's reverse sweep), of cut tile si.
// Items in ticket order: the first pieces of the cut tiles, gap0 whole
// tiles, the next pieces, gap1 whole tiles, the last pieces.
struct BwdWork {
  int64_t tile;
  int kb0, kb1, piece, si;
};

__device__ BwdWork bwd_work(int64_t item, const BwdParams &p, int nblk) {
  BwdWork w{item, 0, nblk, -1, 0};
  const int64_t F = p.tiles - p.ncut;  // whole tiles
  const int first = p.ckpt_given ? 1 : 0;
  int64_t pos = item, full = 0;
  for (int j = first; j < 3; ++j) {
    if (pos < p.ncut) {
      w.si = static_cast<int>(pos);
      w.tile = F + w.si;
      w.piece = j;
      w.kb0 = j == 1 ? p.kcut : 0;
      w.kb1 = j == 1 ? nblk : p.kcut;
      return w;
    }
    pos -= p.ncut;
    if (j < 2) {
      const int64_t gs = j == first ? p.gap0 : p.gap1;
      if (pos < gs) {
        w.tile = full + pos;
        return w;
      }
      pos -= gs;
      full += gs;
    }
  }
  return w;  // not reached: the grid has F + (3 - first) * ncut items
}

// one thread waits (bounded) for a flag another block releases
__device__ void wait_flag(const unsigned *f, unsigned *status) {
  const uint64_t start = global_timer_ns();
  while (ld_acquire_gpu(f) == 0u) {
    if (global_timer_ns() - start > 2000000000ull) {
      atomicOr(status, kStatusTimeout);
      break;
    }
    __nanosleep(256);
  }
  __threadfence();
}

template <typename InT, int G, bool VARLEN, bool CUT, bool MID>
__global__ void __launch_bounds__(32 * G, 12 / G)  // 3 blocks of 4 warps per SM
    scan_bwd_kernel(const BwdParams p) {
  using Sm = BwdSmem<G>;
  constexpr int NP = Sm::NP;
  constexpr int NT = 32 * G;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Sm &s = *reinterpret_cast<Sm *>(smem_raw);

  const int tid = threadIdx.x, lane = tid & 31, g = tid >> 5;
  const int64_t L = p.seqlen;
  const int nblk = static_cast<int>((L + TB - 1) / TB);
  // the block's work: a whole tile, or with the cut schedule a ticket's item
  __shared__ int64_t s_item;
  if (CUT) {
    if (tid == 0) s_item = atomicAdd(p.ticket, 1u);
    __syncthreads();
  }
  const BwdWork wk = CUT ? bwd_work(s_item, p, nblk) : BwdWork{blockIdx.x, 0, nblk, -1, 0};
  const int kb0 = wk.kb0, kb1 = wk.kb1;
  const int64_t tile = wk.tile;
  const int64_t b = tile / p.ch_tiles;
  const int64_t d0 = (tile % p.ch_tiles) * CH;
  const int64_t d = d0 + lane;
  const bool dvalid = d < p.dim;

  // tensor sizes for the bounds checks of the checked build
  const int64_t nBDL = p.batch * p.dim * L, nBNL = p.batch * p.dstate * L;
  const int64_t nCk = p.tiles * static_cast<int64_t>(nblk) * NP * CH;
  // the block's checkpoints (a block-uniform condition: all threads leave)
  if (!dbg_index_ok((tile + 1) * static_cast<int64_t>(nblk) * NP * CH - 1, nCk, p.status))
    return;
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

  // this lane's states 4g .. 4g+3 as two pairs (4g, 4g+1), (4g+2, 4g+3)
  float2 al2[2], an2[2], h2[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    float av[2], hv[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 4 * g + 2 * q + e;
      const bool live = dvalid && n < p.dstate;
      av[e] = live ? p.A[d * p.dstate + n] : 0.f;
      hv[e] = (live && p.h0) ? p.h0[(b * p.dim + d) * p.dstate + n] : 0.f;
    }
    an2[q] = make_float2(av[0], av[1]);
    al2[q] = make_float2(av[0] * kLog2e, av[1] * kLog2e);
    h2[q] = make_float2(hv[0], hv[1]);
  }
  // state 4g + i of lane at the start of block k:
  // ckpt[(k * NP + 4g + i) * CH + lane] (coalesced per warp)
  float *ckpt = p.ckpt + tile * static_cast<int64_t>(nblk) * NP * CH;
  // ordinary scans also have the state after the 8th step of every block
  // (kept by the own forward sweep, or written by the forward scan with its
  // checkpoints), so the reverse sweep recomputes each half of a block from
  // its own start
  float *ckmid = MID ? p.ckpt_mid + tile * static_cast<int64_t>(nblk) * NP * CH : nullptr;
  // a second part with its own forward sweep starts from the state the
  // first part's sweep left at block kb0
  if (CUT && wk.piece == 1 && !p.ckpt_given) {
    if (tid == 0) wait_flag(p.flag + wk.si, p.status);
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 2; ++q)
      h2[q] = make_float2(__ldcg(&ckpt[(static_cast<int64_t>(kb0) * NP + 4 * g + 2 * q) * CH + lane]),
                          __ldcg(&ckpt[(static_cast<int64_t>(kb0) * NP + 4 * g + 2 * q + 1) * CH + lane]));
  }

  // The reverse sweep reads block k - 1 from HBM into registers while block
  // k's earlier half is computed and writes it to the other tile set right
  // after: fetch (loads only) and commit (math and shared stores).
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
      const int64_t ou = b * p.su[0] + dd * p.su[1] + t0 + t,
                    ox = b * p.sdl[0] + dd * p.sdl[1] + t0 + t,
                    oz = b * p.sz[0] + dd * p.sz[1] + t0 + t,
                    oy = b * p.sdy[0] + dd * p.sdy[1] + t0 + t;
      const bool ok = dd < p.dim && t < nt && dbg_index_ok(ou, p.ext_u, p.status) &&
                      dbg_index_ok(ox, p.ext_delta, p.status) &&
                      (!gz || dbg_index_ok(oz, p.ext_z, p.status)) &&
                      dbg_index_ok(oy, p.ext_dy, p.status);
      r.u[e] = ok ? ld_f32(gu, ou) : 0.f;
      r.x[e] = ok ? ld_f32(gd, ox) : 0.f;
      r.z[e] = (ok && gz) ? ld_f32(gz, oz) : 0.f;
      r.dy[e] = ok ? p.dy[oy] : 0.f;
      if (ok) r.ok |= 1u << e;
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int idx = tid + NT * e;
      const int n = idx / TB, t = idx % TB;
      const int64_t ob = b * p.sB[0] + n * p.sB[1] + t0 + t,
                    oc = b * p.sC[0] + n * p.sC[1] + t0 + t;
      const bool ok = idx < NP * TB && n < p.dstate && t < nt &&
                      dbg_index_ok(ob, p.ext_B, p.status) && dbg_index_ok(oc, p.ext_C, p.status);
      r.B[e] = ok ? ld_f32(gB, ob) : 0.f;
      r.C[e] = ok ? ld_f32(gC, oc) : 0.f;
    }
  };
  // the tiles of element (c, t) of a block from its raw values (zeros when
  // the element lies outside the tensors)
  auto put = [&](BwdTiles<G> &T, int c, int t, bool ok, float uu, float xr, float zv, float dyv) {
    const float x = ok ? xr + s.bias[c] : 0.f;
    const float dl = ok ? (p.softplus ? softplus_f(x) : x) : 0.f;
    T.u[c * ROW + t] = uu;
    T.dl[c * ROW + t] = dl;
    T.du[c * ROW + t] = dl * uu;
    // silu(z) = z sig(z) and silu'(z) = sig(z) (1 + z (1 - sig(z))) from
    // one sigmoid
    const float sz = gz ? sigmoid_f(zv) : 1.f;
    T.ds[c * ROW + t] = gz ? dyv * zv * sz : dyv;
    T.gz[c * ROW + t] = dyv * sz * fmaf(zv, 1.0f - sz, 1.0f);
    T.sg[c * ROW + t] = p.softplus ? sigmoid_f(x) : 1.f;
  };
  // packed sequences: the block's restart mask, written by thread 0 with its
  // tiles (no decay across a start: exp(Delta A) is taken as 0 there)
  int64_t mask_cursor = 1;
  auto put_mask = [&](int k, BwdTiles<G> &T) {
    if (VARLEN && tid == 0)
      T.rmask = restart_mask(p, static_cast<int64_t>(k) * TB, L, mask_cursor);
  };
  auto commit = [&](const Raw &r, BwdTiles<G> &T) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = tid + NT * e, c = idx / TB, t = idx % TB;
      put(T, c, t, (r.ok >> e) & 1u, r.u[e], r.x[e], r.z[e], r.dy[e]);
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int idx = tid + NT * e;
      if (idx < NP * TB) {
        const int n = idx / TB, t = idx % TB;
        T.B[t * NP + n] = r.B[e];
        T.C[t * NP + n] = r.C[e];
      }
    }
  };

  // bf16 inputs: the reverse sweep stages block k - 1's raw inputs in
  // shared memory by asynchronous copies (no registers held while block k
  // is computed), 16-byte pieces of the blocks' rows where rows are whole
  // and aligned, element loads elsewhere.
  constexpr bool kStaged = sizeof(InT) == 2;
  auto st16 = [](const int64_t(&sd)[2], int es) {
    return (sd[0] * es) % 16 == 0 && (sd[1] * es) % 16 == 0;
  };
  constexpr int ES = static_cast<int>(sizeof(InT));
  const bool rows16 = aligned16(p.u) && aligned16(p.delta) && (!gz || aligned16(p.z)) &&
                      aligned16(p.dy) && aligned16(p.B) && aligned16(p.C) &&
                      st16(p.su, ES) && st16(p.sdl, ES) && (!gz || st16(p.sz, ES)) &&
                      st16(p.sdy, 4) && st16(p.sB, ES) && st16(p.sC, ES);
  auto stage_fetch = [&](int k) {
    BwdStage<G> &st = s.st;
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
    constexpr int NR = CH * 2;                      // 8-element pieces of a bf16 tile
    constexpr int NCH = 3 * NR + CH * 4 + 2 * NP * 2;  // + 4-element pieces of dy
    for (int j = tid; j < NCH; j += NT) {
      const void *src;
      void *dst;
      int64_t off, ext;
      int row_ok, w, r;
      bool f32 = false;
      if (j < 3 * NR) {
        const int kind = j / NR, rr = j % NR, c = rr / 2, h = rr % 2;
        const InT *base = kind == 0 ? gu : (kind == 1 ? gd : gz);
        const int64_t(&sd)[2] = kind == 0 ? p.su : (kind == 1 ? p.sdl : p.sz);
        off = b * sd[0] + (d0 + c) * sd[1] + t0 + 8 * h;
        ext = kind == 0 ? p.ext_u : (kind == 1 ? p.ext_delta : p.ext_z);
        row_ok = d0 + c < p.dim && (kind < 2 || gz);
        w = 8 * h;
        src = base;
        __nv_bfloat16 *sb = kind == 0 ? st.u : (kind == 1 ? st.x : st.z);
        dst = sb + c * TB + 8 * h;
      } else if (j < 3 * NR + CH * 4) {
        r = j - 3 * NR;
        const int c = r / 4, h = r % 4;
        off = b * p.sdy[0] + (d0 + c) * p.sdy[1] + t0 + 4 * h;
        ext = p.ext_dy;
        row_ok = d0 + c < p.dim;
        w = 4 * h;
        src = p.dy;
        dst = st.dy + c * TB + 4 * h;
        f32 = true;
      } else {
        r = j - 3 * NR - CH * 4;
        const int kind = r / (2 * NP), rr = r % (2 * NP), n = rr / 2, h = rr % 2;
        const int64_t(&sd)[2] = kind == 0 ? p.sB : p.sC;
        off = b * sd[0] + n * sd[1] + t0 + 8 * h;
        ext = kind == 0 ? p.ext_B : p.ext_C;
        row_ok = n < p.dstate;
        w = 8 * h;
        src = kind == 0 ? gB : gC;
        dst = (kind == 0 ? st.B : st.C) + n * TB + 8 * h;
      }
      if (!row_ok) continue;
      const int cnt = f32 ? 4 : 8;
      if (rows16 && nt == TB && dbg_index_ok(off + cnt - 1, ext, p.status)) {
        cp_async16(dst, f32 ? static_cast<const void *>(static_cast<const float *>(src) + off)
                            : static_cast<const void *>(static_cast<const InT *>(src) + off));
      } else {
        for (int q = 0; q < cnt && w + q < nt; ++q) {
          if (!dbg_index_ok(off + q, ext, p.status)) break;
          if (f32)
            static_cast<float *>(dst)[q] = static_cast<const float *>(src)[off + q];
          else
            static_cast<InT *>(dst)[q] = static_cast<const InT *>(src)[off + q];
        }
      }
    }
    cp_async_commit();
  };
  // block k's tiles from the staged raw inputs (after every thread's copies
  // have landed and a barrier)
  auto stage_commit = [&](int k, BwdTiles<G> &T) {
    const BwdStage<G> &st = s.st;
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = tid + NT * e, c = idx / TB, t = idx % TB;
      const bool ok = d0 + c < p.dim && t < nt;
      const int i = c * TB + t;
      put(T, c, t, ok, ok ? ld_f32(reinterpret_cast<const InT *>(st.u), i) : 0.f,
          ok ? ld_f32(reinterpret_cast<const InT *>(st.x), i) : 0.f,
          (ok && gz) ? ld_f32(reinterpret_cast<const InT *>(st.z), i) : 0.f,
          ok ? st.dy[i] : 0.f);
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int idx = tid + NT * e;
      if (idx < NP * TB) {
        const int n = idx / TB, t = idx % TB;
        const bool ok = n < p.dstate && t < nt;
        T.B[t * NP + n] = ok ? ld_f32(reinterpret_cast<const InT *>(st.B), idx) : 0.f;
        T.C[t * NP + n] = ok ? ld_f32(reinterpret_cast<const InT *>(st.C), idx) : 0.f;
      }
    }
  };

  // ------------------------------------------------------ forward sweep
  // (skipped when the forward scan already wrote the checkpoints).  Block
  // k + 1's u, delta and B are read into registers while block k is
  // computed and committed to the other tile set next iteration, so one
  // barrier per block separates the phases.
  struct RawF {
    float u[E], x[E], B[EB];
    unsigned ok;
  };
  auto fetch_fwd = [&](int k, RawF &r) {
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
    r.ok = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = tid + NT * e, c = idx / TB, t = idx % TB;
      const int64_t dd = d0 + c;
      const int64_t ou = b * p.su[0] + dd * p.su[1] + t0 + t,
                    ox = b * p.sdl[0] + dd * p.sdl[1] + t0 + t;
      const bool ok = dd < p.dim && t < nt && dbg_index_ok(ou, p.ext_u, p.status) &&
                      dbg_index_ok(ox, p.ext_delta, p.status);
      r.u[e] = ok ? ld_f32(gu, ou) : 0.f;
      r.x[e] = ok ? ld_f32(gd, ox) : 0.f;
      if (ok) r.ok |= 1u << e;
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int idx = tid + NT * e;
      const int n = idx / TB, t = idx % TB;
      const int64_t ob = b * p.sB[0] + n * p.sB[1] + t0 + t;
      const bool ok = idx < NP * TB && n < p.dstate && t < nt &&
                      dbg_index_ok(ob, p.ext_B, p.status);
      r.B[e] = ok ? ld_f32(gB, ob) : 0.f;
    }
  };
  auto commit_fwd = [&](const RawF &r, BwdTiles<G> &T) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = tid + NT * e, c = idx / TB, t = idx % TB;
      const bool ok = (r.ok >> e) & 1u;
      const float x = ok ? r.x[e] + s.bias[c] : 0.f;
      const float dl = ok ? (p.softplus ? softplus_f(x) : x) : 0.f;
      T.dl[c * ROW + t] = dl;
      T.du[c * ROW + t] = dl * r.u[e];
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int idx = tid + NT * e;
      if (idx < NP * TB) T.B[(idx % TB) * NP + idx / TB] = r.B[e];
    }
  };
  __syncthreads();
  // bf16 forward sweep: block k + 2's u, delta and B are copied
  // asynchronously into one of two areas of the staging buffer while block
  // k is computed and block k + 1 is committed from the other area.
  constexpr int kFArea = 2 * CH * TB * 2 + NP * TB * 2;  // bytes of one area
  static_assert(2 * kFArea <= static_cast<int>(sizeof(BwdStage<G>)), "two areas fit");
  auto farea = [&](int a) {
    return reinterpret_cast<InT *>(reinterpret_cast<unsigned char *>(&s.st) + a * kFArea);
  };
  auto fstage_fetch = [&](int k, int a) {
    InT *su = farea(a), *sx = su + CH * TB, *sB = sx + CH * TB;
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
    constexpr int NR = CH * 2;  // 8-element pieces of a (channel, step) tile
    for (int j = tid; j < 2 * NR + NP * 2; j += NT) {
      const InT *src;
      InT *dst;
      int64_t off, ext;
      int w;
      if (j < 2 * NR) {
        const int kind = j / NR, rr = j % NR, c = rr / 2, h = rr % 2;
        if (d0 + c >= p.dim) continue;
        src = kind == 0 ? gu : gd;
        dst = (kind == 0 ? su : sx) + c * TB + 8 * h;
        const int64_t(&sd)[2] = kind == 0 ? p.su : p.sdl;
        off = b * sd[0] + (d0 + c) * sd[1] + t0 + 8 * h;
        ext = kind == 0 ? p.ext_u : p.ext_delta;
        w = 8 * h;
      } else {
        const int r = j - 2 * NR, n = r / 2, h = r % 2;
        if (n >= p.dstate) continue;
        src = gB;
        dst = sB + n * TB + 8 * h;
        off = b * p.sB[0] + n * p.sB[1] + t0 + 8 * h;
        ext = p.ext_B;
        w = 8 * h;
      }
      if (rows16 && nt == TB && dbg_index_ok(off + 7, ext, p.status)) {
        cp_async16(dst, src + off);
      } else {
        for (int q = 0; q < 8 && w + q < nt; ++q) {
          if (!dbg_index_ok(off + q, ext, p.status)) break;
          dst[q] = src[off + q];
        }
      }
    }
    cp_async_commit();
  };
  auto fstage_commit = [&](int k, int a, BwdTiles<G> &T) {
    const InT *su = farea(a), *sx = su + CH * TB, *sB = sx + CH * TB;
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = tid + NT * e, c = idx / TB, t = idx % TB;
      const bool ok = d0 + c < p.dim && t < nt;
      const float uu = ok ? ld_f32(su, c * TB + t) : 0.f;
      const float x = ok ? ld_f32(sx, c * TB + t) + s.bias[c] : 0.f;
      const float dl = ok ? (p.softplus ? softplus_f(x) : x) : 0.f;
      T.dl[c * ROW + t] = dl;
      T.du[c * ROW + t] = dl * uu;
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      const int idx = tid + NT * e;
      if (idx < NP * TB) {
        const int n = idx / TB, t = idx % TB;
        T.B[t * NP + n] = (n < p.dstate && t < nt) ? ld_f32(sB, idx) : 0.f;
      }
    }
  };
  // block k's recurrence from tile set T, state at its start in h2.  With
  // packed sequences only a block with a start in it takes the masked loop
  // (the test is uniform over the block); the ordinary kernel keeps its own
  // copy of the loop, whose register allocation a shared generic lambda
  // changed (0.7 % slower).
  auto fwd_block = [&](const BwdTiles<G> &T, int k) {
    if constexpr (VARLEN) {
      auto run = [&](auto masked) {
#pragma unroll
        for (int qd = 0; qd < TB / 4; ++qd) {
          const float4 dl4 = ld4(&T.dl[lane * ROW + 4 * qd]);
          const float4 du4 = ld4(&T.du[lane * ROW + 4 * qd]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float4 b4 = ld4(&T.B[(4 * qd + j) * NP + 4 * g]);
            const float2 D2 = f2(comp(dl4, j)), U2 = f2(comp(du4, j));
            float2 e0 = ex2_pair(__fmul2_rn(D2, al2[0])), e1 = ex2_pair(__fmul2_rn(D2, al2[1]));
            if (decltype(masked)::value && ((T.rmask >> (4 * qd + j)) & 1u))
              e0 = e1 = make_float2(0.f, 0.f);
            h2[0] = __ffma2_rn(e0, h2[0], __fmul2_rn(U2, make_float2(b4.x, b4.y)));
            h2[1] = __ffma2_rn(e1, h2[1], __fmul2_rn(U2, make_float2(b4.z, b4.w)));
          }
        }
      };
      if (T.rmask != 0u)
        run(std::true_type{});
      else
        run(std::false_type{});
    } else {
#pragma unroll
      for (int qd = 0; qd < TB / 4; ++qd) {
        const float4 dl4 = ld4(&T.dl[lane * ROW + 4 * qd]), du4 = ld4(&T.du[lane * ROW + 4 * qd]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 b4 = ld4(&T.B[(4 * qd + j) * NP + 4 * g]);
          const float2 D2 = f2(comp(dl4, j)), U2 = f2(comp(du4, j));
          float2 e0 = ex2_pair(__fmul2_rn(D2, al2[0])), e1 = ex2_pair(__fmul2_rn(D2, al2[1]));
          h2[0] = __ffma2_rn(e0, h2[0], __fmul2_rn(U2, make_float2(b4.x, b4.y)));
          h2[1] = __ffma2_rn(e1, h2[1], __fmul2_rn(U2, make_float2(b4.z, b4.w)));
        }
        if constexpr (MID) {
          if (qd == 1) {  // the state entering step 8 of block k
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              ckmid[(static_cast<int64_t>(k) * NP + 4 * g + 2 * q) * CH + lane] = h2[q].x;
              ckmid[(static_cast<int64_t>(k) * NP + 4 * g + 2 * q + 1) * CH + lane] = h2[q].y;
            }
          }
        }
      }
    }
  };
  auto put_ckpt = [&](int k) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      ckpt[(static_cast<int64_t>(k) * NP + 4 * g + 2 * q) * CH + lane] = h2[q].x;
      ckpt[(static_cast<int64_t>(k) * NP + 4 * g + 2 * q + 1) * CH + lane] = h2[q].y;
    }
  };
  const bool sweep = !p.ckpt_given && wk.piece != 2;
  if (sweep && kStaged) {
    fstage_fetch(kb0, kb0 & 1);
    cp_async_wait_all();
    __syncthreads();
    fstage_commit(kb0, kb0 & 1, s.tl[kb0 & 1]);
    put_mask(kb0, s.tl[kb0 & 1]);
    if (kb0 + 1 < kb1) fstage_fetch(kb0 + 1, (kb0 + 1) & 1);
    for (int k = kb0; k < kb1; ++k) {
      put_ckpt(k);
      // block k + 1's copies (this thread's) have landed; after the barrier
      // every thread's have, and block k's tiles are committed
      cp_async_wait_all();
      __syncthreads();
      // area k & 1 held block k, committed before the barrier; tile set
      // (k + 1) & 1 was last read by block k - 1, finished before it
      if (k + 2 < kb1) fstage_fetch(k + 2, k & 1);
      if (k + 1 < kb1) {
        fstage_commit(k + 1, (k + 1) & 1, s.tl[(k + 1) & 1]);
        put_mask(k + 1, s.tl[(k + 1) & 1]);
      }
      fwd_block(s.tl[k & 1], k);
    }
    __syncthreads();
  } else if (sweep) {
    RawF rf;
    fetch_fwd(kb0, rf);
    for (int k = kb0; k < kb1; ++k) {
      BwdTiles<G> &T = s.tl[k & 1];
      commit_fwd(rf, T);
      put_mask(k, T);
      put_ckpt(k);
      __syncthreads();
      if (k + 1 < kb1) fetch_fwd(k + 1, rf);  // in flight while block k is computed
      fwd_block(T, k);
      // no barrier here: block k + 1 is committed to the other tile set, and
      // this set is next written two blocks on, after the next barrier
    }
    __syncthreads();
  }
  if (CUT && wk.piece == 0) {
    // the first part's sweep ends here: its end state is the checkpoint of
    // block kb1, published for the second part
    put_ckpt(kb1);
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release_gpu(p.flag + wk.si, 1u);
    return;
  }

  // ------------------------------------------------------ reverse sweep
  float2 lam[2], dA2[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    float lv[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 4 * g + 2 * q + e;
      lv[e] = (dvalid && n < p.dstate && p.d_last)
                  ? p.d_last[(b * p.dim + d) * p.dstate + n] : 0.f;
    }
    lam[q] = make_float2(lv[0], lv[1]);
    dA2[q] = make_float2(0.f, 0.f);
  }
  // the first part's reverse sweep starts from the adjoint the second part
  // left at its first block
  if (CUT && wk.piece == 2) {
    if (tid == 0) wait_flag(p.flag + p.ncut + wk.si, p.status);
    __syncthreads();
    const float *lr = p.lam + static_cast<int64_t>(wk.si) * NP * CH;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float lv[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {  // written only for live (channel, state)
        const int n = 4 * g + 2 * q + e;
        lv[e] = (dvalid && n < p.dstate) ? __ldcg(&lr[n * CH + lane]) : 0.f;
      }
      lam[q] = make_float2(lv[0], lv[1]);
    }
  }
  // the checkpoint of the block after the current one is read a block early
  float2 hnext[2], hnextm[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    hnext[q] = make_float2(
        ckpt[(static_cast<int64_t>(kb1 - 1) * NP + 4 * g + 2 * q) * CH + lane],
        ckpt[(static_cast<int64_t>(kb1 - 1) * NP + 4 * g + 2 * q + 1) * CH + lane]);
    if constexpr (MID)
      hnextm[q] = make_float2(
          ckmid[(static_cast<int64_t>(kb1 - 1) * NP + 4 * g + 2 * q) * CH + lane],
          ckmid[(static_cast<int64_t>(kb1 - 1) * NP + 4 * g + 2 * q + 1) * CH + lane]);
  }
  Raw raw;
  if (kStaged) {
    stage_fetch(kb1 - 1);
    cp_async_wait_all();
    __syncthreads();
    stage_commit(kb1 - 1, s.tl[(kb1 - 1) & 1]);
    put_mask(kb1 - 1, s.tl[(kb1 - 1) & 1]);
  } else {
    fetch(kb1 - 1, raw);
    commit(raw, s.tl[(kb1 - 1) & 1]);
    put_mask(kb1 - 1, s.tl[(kb1 - 1) & 1]);
  }
  // this thread's shares of the per-channel sums (in registers when a
  // thread has few elements; otherwise added to shared memory per block)
  constexpr bool kRegAcc = E <= 4;
  constexpr int EA = kRegAcc ? E : 1;
  float accD[EA], accB[EA];
#pragma unroll
  for (int e = 0; e < EA; ++e) accD[e] = accB[e] = 0.f;
  for (int k = kb1 - 1; k >= kb0; --k) {
    const int64_t t0 = static_cast<int64_t>(k) * TB;
    const int nt = static_cast<int>(min(static_cast<int64_t>(TB), L - t0));
    BwdTiles<G> &T = s.tl[k & 1];
    float2 hc[2], hcm[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      hc[q] = hnext[q];
      if constexpr (MID) hcm[q] = hnextm[q];
      if (k > kb0) {
        hnext[q] = make_float2(
            ckpt[(static_cast<int64_t>(k - 1) * NP + 4 * g + 2 * q) * CH + lane],
            ckpt[(static_cast<int64_t>(k - 1) * NP + 4 * g + 2 * q + 1) * CH + lane]);
        if constexpr (MID)
          hnextm[q] = make_float2(
              ckmid[(static_cast<int64_t>(k - 1) * NP + 4 * g + 2 * q) * CH + lane],
              ckmid[(static_cast<int64_t>(k - 1) * NP + 4 * g + 2 * q + 1) * CH + lane]);
      }
    }
    __syncthreads();

    // Two halves of the block, the later one first.  For each: recompute
    // the states of its 8 steps from the checkpoint, keeping every step's
    // state and decay (with this warp's share of the readout s_t), then
    // run the adjoint backwards over them with the kept decays.
#pragma unroll
    for (int half = 1; half >= 0; --half) {
      const int tb = 8 * half;  // first step of this half
      // block k-1's inputs: in flight while the earlier half is computed
      if (half == 0 && k > kb0) {
        if (kStaged)
          stage_fetch(k - 1);
        else
          fetch(k - 1, raw);
      }
      float2 hs[2][8], as[2][8];
      float2 hh[2] = {hc[0], hc[1]};
      if constexpr (VARLEN) {
        // packed sequences: the masked loop only when this pass has a start
        auto recompute = [&](auto masked) {
#pragma unroll
          for (int qd = 0; qd < tb / 4 + 2; ++qd) {
            const float4 dl4 = ld4(&T.dl[lane * ROW + 4 * qd]);
            const float4 du4 = ld4(&T.du[lane * ROW + 4 * qd]);
            float4 ds4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (4 * qd >= tb) ds4 = ld4(&T.ds[lane * ROW + 4 * qd]);
            float4 sp4 = make_float4(0.f, 0.f, 0.f, 0.f);
            float vC[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int t = 4 * qd + j;
              const float4 b4 = ld4(&T.B[t * NP + 4 * g]);
              const float2 D2 = f2(comp(dl4, j)), U2 = f2(comp(du4, j));
              float2 a0 = ex2_pair(__fmul2_rn(D2, al2[0]));
              float2 a1 = ex2_pair(__fmul2_rn(D2, al2[1]));
              // a sequence start: nothing of the previous state survives it
              if (decltype(masked)::value && ((T.rmask >> t) & 1u))
                a0 = a1 = make_float2(0.f, 0.f);
              hh[0] = __ffma2_rn(a0, hh[0], __fmul2_rn(U2, make_float2(b4.x, b4.y)));
              hh[1] = __ffma2_rn(a1, hh[1], __fmul2_rn(U2, make_float2(b4.z, b4.w)));
              if (t >= tb) {
                as[0][t - tb] = a0;
                as[1][t - tb] = a1;
                hs[0][t - tb] = hh[0];
                hs[1][t - tb] = hh[1];
                const float4 c4 = ld4(&T.C[t * NP + 4 * g]);
                float2 r = __fmul2_rn(make_float2(c4.x, c4.y), hh[0]);
                r = __ffma2_rn(make_float2(c4.z, c4.w), hh[1], r);
                const float sv = r.x + r.y;
                if (j == 0) sp4.x = sv;
                if (j == 1) sp4.y = sv;
                if (j == 2) sp4.z = sv;
                if (j == 3) sp4.w = sv;
                // dC_t[n] = sum over channels of ds_t h_t[n]
                const float2 S2 = f2(comp(ds4, j));
                const float2 v0 = __fmul2_rn(S2, hh[0]), v1 = __fmul2_rn(S2, hh[1]);
                vC[0 + j] = v0.x;
                vC[4 + j] = v0.y;
                vC[8 + j] = v1.x;
                vC[12 + j] = v1.y;
              }
            }
            if (4 * qd >= tb) {
              *reinterpret_cast<float4 *>(&s.ps[(g * CH + lane) * ROW + 4 * qd]) = sp4;
              // channel sums of dC for states 4g + i, steps 4 qd + tq: the even
              // lane of each pair adds j = lane >> 1 = 4 i + tq
              const float rc = reduce_scatter16(vC, lane);
              const int jj = lane >> 1, n = 4 * g + jj / 4, t = 4 * qd + jj % 4;
              if ((lane & 1) == 0 && n < p.dstate && t < nt &&
                  dbg_index_ok((b * p.dstate + n) * L + t0 + t, nBNL, p.status))
                atomicAdd(p.dC + (b * p.dstate + n) * L + t0 + t, rc);
            }
          }
        };
        if ((T.rmask & (half ? 0xFFFFu : 0x00FFu)) != 0u)
          recompute(std::true_type{});
        else
          recompute(std::false_type{});
      } else {
        // with the mid-block states, the later half starts at step 8
        if constexpr (MID) {
          if (half == 1) {
            hh[0] = hcm[0];
            hh[1] = hcm[1];
          }
        }
#pragma unroll
        for (int qd = MID ? tb / 4 : 0; qd < tb / 4 + 2; ++qd) {
          const float4 dl4 = ld4(&T.dl[lane * ROW + 4 * qd]), du4 = ld4(&T.du[lane * ROW + 4 * qd]);
          float4 ds4 = make_float4(0.f, 0.f, 0.f, 0.f);
          if (4 * qd >= tb) ds4 = ld4(&T.ds[lane * ROW + 4 * qd]);
          float4 sp4 = make_float4(0.f, 0.f, 0.f, 0.f);
          float vC[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int t = 4 * qd + j;
            const float4 b4 = ld4(&T.B[t * NP + 4 * g]);
            const float2 D2 = f2(comp(dl4, j)), U2 = f2(comp(du4, j));
            float2 a0 = ex2_pair(__fmul2_rn(D2, al2[0]));
            float2 a1 = ex2_pair(__fmul2_rn(D2, al2[1]));
            hh[0] = __ffma2_rn(a0, hh[0], __fmul2_rn(U2, make_float2(b4.x, b4.y)));
            hh[1] = __ffma2_rn(a1, hh[1], __fmul2_rn(U2, make_float2(b4.z, b4.w)));
            if (t >= tb) {
              as[0][t - tb] = a0;
              as[1][t - tb] = a1;
              hs[0][t - tb] = hh[0];
              hs[1][t - tb] = hh[1];
              const float4 c4 = ld4(&T.C[t * NP + 4 * g]);
              float2 r = __fmul2_rn(make_float2(c4.x, c4.y), hh[0]);
              r = __ffma2_rn(make_float2(c4.z, c4.w), hh[1], r);
              const float sv = r.x + r.y;
              if (j == 0) sp4.x = sv;
              if (j == 1) sp4.y = sv;
              if (j == 2) sp4.z = sv;
              if (j == 3) sp4.w = sv;
              // dC_t[n] = sum over channels of ds_t h_t[n]
              const float2 S2 = f2(comp(ds4, j));
              const float2 v0 = __fmul2_rn(S2, hh[0]), v1 = __fmul2_rn(S2, hh[1]);
              vC[0 + j] = v0.x;
              vC[4 + j] = v0.y;
              vC[8 + j] = v1.x;
              vC[12 + j] = v1.y;
            }
          }
          if (4 * qd >= tb) {
            *reinterpret_cast<float4 *>(&s.ps[(g * CH + lane) * ROW + 4 * qd]) = sp4;
            // channel sums of dC for states 4g + i, steps 4 qd + tq: the even
            // lane of each pair adds j = lane >> 1 = 4 i + tq
            const float rc = reduce_scatter16(vC, lane);
            const int jj = lane >> 1, n = 4 * g + jj / 4, t = 4 * qd + jj % 4;
            if ((lane & 1) == 0 && n < p.dstate && t < nt &&
                dbg_index_ok((b * p.dstate + n) * L + t0 + t, nBNL, p.status))
              atomicAdd(p.dC + (b * p.dstate + n) * L + t0 + t, rc);
          }
        }
      }

      // adjoint, four steps at a time backwards; a_t h_{t-1} = h_t - Delta_t
      // u_t B_t needs no state of the previous step
#pragma unroll
      for (int qq = 1; qq >= 0; --qq) {
        const int q = 2 * half + qq;
        float vB[16];
        const int t4 = tb + 4 * qq;  // first step of this quad
        const float4 dl4 = ld4(&T.dl[lane * ROW + t4]), du4 = ld4(&T.du[lane * ROW + t4]),
                     ds4 = ld4(&T.ds[lane * ROW + t4]);
        float4 pb4, pa4;
#pragma unroll
        for (int tq = 3; tq >= 0; --tq) {
          const int tl = 4 * qq + tq;  // step within the half
          const float4 b4 = ld4(&T.B[(t4 + tq) * NP + 4 * g]);
          const float4 c4 = ld4(&T.C[(t4 + tq) * NP + 4 * g]);
          const float2 D2 = f2(comp(dl4, tq)), U2 = f2(comp(du4, tq)), S2 = f2(comp(ds4, tq));
          const float2 nU2 = f2(-comp(du4, tq));
          float2 qa = make_float2(0.f, 0.f), qb = make_float2(0.f, 0.f);
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {
            const float2 Bp = pr == 0 ? make_float2(b4.x, b4.y) : make_float2(b4.z, b4.w);
            const float2 Cp = pr == 0 ? make_float2(c4.x, c4.y) : make_float2(c4.z, c4.w);
            lam[pr] = __ffma2_rn(S2, Cp, lam[pr]);
            const float2 la = __fmul2_rn(lam[pr], __ffma2_rn(nU2, Bp, hs[pr][tl]));
            qa = __ffma2_rn(la, an2[pr], qa);
            qb = __ffma2_rn(lam[pr], Bp, qb);
            dA2[pr] = __ffma2_rn(la, D2, dA2[pr]);
            const float2 vb = __fmul2_rn(lam[pr], U2);
            vB[4 * (2 * pr) + tq] = vb.x;
            vB[4 * (2 * pr + 1) + tq] = vb.y;
            lam[pr] = __fmul2_rn(lam[pr], as[pr][tl]);
          }
          const float sa = qa.x + qa.y, sb = qb.x + qb.y;
          if (tq == 0) { pa4.x = sa; pb4.x = sb; }
          if (tq == 1) { pa4.y = sa; pb4.y = sb; }
          if (tq == 2) { pa4.z = sa; pb4.z = sb; }
          if (tq == 3) { pa4.w = sa; pb4.w = sb; }
        }
        *reinterpret_cast<float4 *>(&s.pa[(g * CH + lane) * ROW + t4]) = pa4;
        *reinterpret_cast<float4 *>(&s.pb[(g * CH + lane) * ROW + t4]) = pb4;
        // channel sums of dB for states 4g + i, steps 4q + tq (as for dC)
        const float rb = reduce_scatter16(vB, lane);
        const int j = lane >> 1, n = 4 * g + j / 4, t = 4 * q + j % 4;
        if ((lane & 1) == 0 && n < p.dstate && t < nt &&
            dbg_index_ok((b * p.dstate + n) * L + t0 + t, nBNL, p.status))
          atomicAdd(p.dB + (b * p.dstate + n) * L + t0 + t, rb);
      }
      // block k-1 into the other tile set, which is free: block k+1's
      // epilogue ended before this block's barrier
      if (!kStaged && half == 0 && k > kb0) {
        commit(raw, s.tl[(k - 1) & 1]);
        put_mask(k - 1, s.tl[(k - 1) & 1]);
      }
    }
    if (kStaged) cp_async_wait_all();
    __syncthreads();
    // staged inputs: block k-1 into the other tile set once every copy has
    // landed (the staging area is refilled only after the next barrier)
    if (kStaged && k > kb0) {
      stage_commit(k - 1, s.tl[(k - 1) & 1]);
      put_mask(k - 1, s.tl[(k - 1) & 1]);
    }

    // elementwise: du, ddelta, dz, and the per-channel sums of dD, dbias
    // (kept in registers: a thread's channels are the same in every block)
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int idx = tid + NT * e;
      const int c = idx / TB, t = idx % TB;
      const int64_t dd = d0 + c;
      if (dd >= p.dim || t >= nt) continue;
      float sp = 0.f, sb = 0.f, sa = 0.f;
#pragma unroll
      for (int w = 0; w < G; ++w) {
        sp += s.ps[(w * CH + c) * ROW + t];
        sb += s.pb[(w * CH + c) * ROW + t];
        sa += s.pa[(w * CH + c) * ROW + t];
      }
      const float uu = T.u[c * ROW + t], ds = T.ds[c * ROW + t];
      const int64_t off = (b * p.dim + dd) * L + t0 + t;
      if (!dbg_index_ok(off, nBDL, p.status)) continue;
      p.du[off] = fmaf(ds, s.dskip[c], T.dl[c * ROW + t] * sb);
      const float ddl = fmaf(uu, sb, sa) * T.sg[c * ROW + t];
      p.ddelta[off] = ddl;
      if (p.dz) {
        const float sv = fmaf(s.dskip[c], uu, sp);
        p.dz[off] = T.gz[c * ROW + t] * sv;
      }
      if (kRegAcc) {
        accD[e % EA] = fmaf(ds, uu, accD[e % EA]);
        accB[e % EA] += ddl;
      } else {
        atomicAdd(&s.accD[c], ds * uu);
        atomicAdd(&s.accB[c], ddl);
      }
    }
    // no barrier here: the next block is committed to the other tile set,
    // and the shares are rewritten only after the next block's barrier,
    // which every thread reaches after finishing this epilogue
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < (kRegAcc ? E : 0); ++e) {
    const int c = (tid + NT * e) / TB;
    atomicAdd(&s.accD[c], accD[e % EA]);
    atomicAdd(&s.accB[c], accB[e % EA]);
  }
  __syncthreads();

  // parameter gradients, summed over batch rows (and dh0 = lam_{-1})
#pragma unroll
  for (int q = 0; q < 2; ++q) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 4 * g + 2 * q + e;
      if (!dvalid || n >= p.dstate) continue;
      atomicAdd(p.dA + d * p.dstate + n, e == 0 ? dA2[q].x : dA2[q].y);
      if (CUT && wk.piece == 1)  // the adjoint handed to the first part
        p.lam[static_cast<int64_t>(wk.si) * NP * CH + (4 * g + 2 * q + e) * CH + lane] =
            e == 0 ? lam[q].x : lam[q].y;
      else if (p.dh0)
        p.dh0[(b * p.dim + d) * p.dstate + n] = e == 0 ? lam[q].x : lam[q].y;
    }
  }
  if (CUT && wk.piece == 1) {
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release_gpu(p.flag + p.ncut + wk.si, 1u);
  }
  if (tid < CH && d0 + tid < p.dim) {
    if (p.dD) atomicAdd(p.dD + d0 + tid, s.accD[tid]);
    if (p.ddelta_bias) atomicAdd(p.ddelta_bias + d0 + tid, s.accB[tid]);
  }
}

template <typename InT, int G, bool VARLEN, bool CUT, bool MID>
cudaError_t launch_kernel(const BwdParams &p, cudaStream_t stream) {
  auto kern = scan_bwd_kernel<InT, G, VARLEN, CUT, MID>;
  const int smem = static_cast<int>(sizeof(BwdSmem<G>));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // items: the whole tiles, and two or three pieces of every cut tile
  const int64_t items = p.tiles + (CUT ? (p.ckpt_given ? 1 : 2) * static_cast<int64_t>(p.ncut) : 0);
  kern<<<static_cast<unsigned>(items), 32 * G, smem, stream>>>(p);
  return cudaGetLastError();
}

// Ordinary scans read the mid-block states (from the backward's own sweep
// or the forward's checkpoints), and the cut schedule has its own
// instantiation; packed sequences keep block starts only and are not cut.
template <typename InT, int G, bool VARLEN>
cudaError_t launch_typed(const BwdParams &p, cudaStream_t stream) {
  if constexpr (!VARLEN) {
    return p.ncut ? launch_kernel<InT, G, false, true, true>(p, stream)
                  : launch_kernel<InT, G, false, false, true>(p, stream);
  } else {
    return launch_kernel<InT, G, true, false, false>(p, stream);
  }
}

template <typename InT, int G>
int blocks_per_sm() {
  int n = 0;
  const int smem = static_cast<int>(sizeof(BwdSmem<G>));
  auto kern = scan_bwd_kernel<InT, G, false, false, true>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * G, smem) != cudaSuccess)
    return 0;
  return n;
}

template <typename InT>
int blocks_per_sm_g(int groups) {
  switch (groups) {
    case 1: return blocks_per_sm<InT, 1>();
    case 2: return blocks_per_sm<InT, 2>();
    default: return blocks_per_sm<InT, 4>();
  }
}

// Packed sequences get their own instantiation, so their code never
// touches the kernel of ordinary scans.
template <typename InT, bool VARLEN>
cudaError_t dispatch_v(const BwdParams &p, cudaStream_t stream) {
  switch (bwd_groups(p.dstate)) {
    case 1: return launch_typed<InT, 1, VARLEN>(p, stream);
    case 2: return launch_typed<InT, 2, VARLEN>(p, stream);
    default: return launch_typed<InT, 4, VARLEN>(p, stream);
  }
}

template <typename InT>
cudaError_t dispatch(const BwdParams &p, cudaStream_t stream) {
  return p.cu ? dispatch_v<InT, true>(p, stream) : dispatch_v<InT, false>(p, stream);
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

// A launch of `tiles` blocks fills W full waves of the resident slots and a
// last wave of r blocks.  When that wave is at most half full (and a tile
// has two 16-step blocks or more), the last r tiles are cut in two at their
// middle block: the first part's forward sweep, the second part's sweeps
// and the first part's reverse sweep become separate work items, taken in
// the order: the first pieces, every whole tile, the remaining pieces
// (with checkpoints the first kind is not needed).  Packed sequences are
// not cut.
BwdCut plan_bwd_cut(const BwdParams &p, int in_bf16) {
  BwdCut c;
  const int nblk = static_cast<int>((p.seqlen + kBwdTimeBlock - 1) / kBwdTimeBlock);
  if (p.cu || nblk < 2) return c;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();  // no device: nothing is cut
    return c;
  }
  const int G = bwd_groups(p.dstate);
  const int per_sm = in_bf16 ? blocks_per_sm_g<__nv_bfloat16>(G) : blocks_per_sm_g<float>(G);
  const int64_t slots = static_cast<int64_t>(sms) * per_sm;
  if (slots < 1) return c;
  const int64_t W = p.tiles / slots, r = p.tiles % slots;
  if (W < 1 || r < 1 || 2 * r > slots) return c;
  c.ncut = static_cast<int>(r);
  c.kcut = nblk / 2;
  const int64_t F = p.tiles - r;
  c.gap0 = F;  // measured: 2.5 % faster than half of them here, half later
  c.gap1 = 0;
  const size_t NPc = static_cast<size_t>(4 * G);
  c.bytes = 256 + ((8 * static_cast<size_t>(r) + 255) / 256) * 256 +
            static_cast<size_t>(r) * NPc * kBwdChannels * sizeof(float);
  return c;
}

}  // namespace sss48
