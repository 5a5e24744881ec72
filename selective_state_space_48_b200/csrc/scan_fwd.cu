// scan_fwd.cu -- forward selective scan (S6) for sm_100a.
//
// One thread block handles 32 consecutive channels d of one batch row b and
// a chunk of the sequence.  Lane l of warp g owns channel d0 + l and the
// states n = 4g .. 4g+3, whose fp32 values h[n] stay in registers for the
// whole chunk ("Keeping the pad on the desk": the state never goes back to
// HBM; only y is written).  Time is walked in blocks of 16 steps.  Raw input
// tiles (u, delta, z, B, C) arrive in a five-stage shared-memory ring filled
// by TMA three blocks ahead (one thread issues five 3-D tensor copies per
// block; every wait on the ring's mbarriers is bounded).  Each block passes
// three phases:
//
//   prep     every (channel, t) of the block computes, once,
//            Delta = softplus(delta + delta_bias) and Delta*u, and B_t[n],
//            C_t[n] are widened to fp32, into shared memory;
//   scan     each lane runs h = exp(Delta A) h + Delta B u over the 16 steps
//            for its 4 states and forms its share of y_t = sum_n C_t[n] h_t[n]
//            (page "The State That Must Remember Everything", "The Equation",
//            with the exponential-Euler discretisation of its Part 7);
//   epilogue the shares of the state groups are summed, the D*u skip added,
//            the silu(z) gate applied and y stored, coalesced along t.
//
// The phases run in different warps at the same time: the scan warps (one
// per group of 4 states) do nothing but the recurrence, while four auxiliary
// warps issue the copies, prep block i+2 and finish block i.  Tiles and y
// shares are double buffered and handed over through mbarriers (every wait
// bounded), so the special-function work of prep and epilogue overlaps the
// recurrence.
//
// Long sequences with few channels are split into chunks that run in
// parallel ("The relay": fade-and-add steps compose associatively, so a
// chunk can be squashed into one pair (P, e) = (prod exp(Delta A), state
// reached from zero) without knowing the state it starts from).  Three
// launches on the stream, with no block ever waiting for another:
//
//   scan      every chunk runs from a zero state (the first from h0), writes
//             its outputs, its pair (P, e) and the running sum of Delta at
//             the start of every segment of 32 blocks;
//   prefix    one thread per (tile, state, channel) composes the pairs in
//             chunk order into the true state at the end of every chunk
//             (and the final state);
//   carry     one block per (tile, chunk after the first, segment) adds the
//             missing term sum_n C_t[n] exp(A[n] sigma_t) h_in[n] to the
//             segment's outputs (sigma_t: running sum of Delta from the
//             chunk start, h_in: true state at the chunk start), block by
//             block until the decay exp(A[n] sigma_t) of every state has
//             fallen below 2^-24, fp32's unit roundoff, in every channel: a
//             term dropped there is smaller than the rounding error of the
//             carried state itself.  Segments whose terms have all decayed
//             leave at once, so the work follows the states' memory and is
//             spread over the whole chip instead of trailing behind the
//             chunks that carry the longest.
//
// Shapes whose rows TMA cannot address (a row of seqlen elements that is
// not a multiple of 16 bytes, or unaligned pointers) take the same kernel
// with the tiles filled by plain coalesced loads instead.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "device_math.cuh"
#include "scan_fwd.cuh"

namespace sss48 {

__device__ unsigned g_scan_status;  // status of scans run without workspace

namespace {

constexpr int CH = kChannelsPerBlock;
constexpr int TB = kTimeBlock;
constexpr int ROW = TB + 4;  // padded fp32 row: float4 reads of 32 lanes at
                             // rows l spread over the bank groups
constexpr int STAGES = 5;    // raw tile ring: blocks i-1 .. i+3 alive at once
constexpr float kCutoffLog2 = -24.0f;
// States per lane (of 4) whose decay exp(Delta A) is evaluated by the
// FMA-pipe polynomial instead of the special-function unit; balances the
// two pipes (the unit's 16 results per clock per SM bound the scan).
constexpr int kPolyStates = 0;
constexpr uint64_t kTmaWaitNs = 2000000000ull;

constexpr int align128(int x) { return (x + 127) / 128 * 128; }

// Kernel variants: ordinary scans, packed sequences (restarts), and the
// three-term trapezoidal update.  Each is its own instantiation so the
// code of one never reaches the others.
constexpr int kModePlain = 0;
constexpr int kModeVarlen = 1;
constexpr int kModeTrap = 2;
constexpr int kModeCkpt = 3;  // ordinary scan that also writes checkpoints

template <typename InT, int G, bool TRAP = false>
struct Layout {
  static constexpr int NP = 4 * G;
  static constexpr int tileU = align128(CH * TB * static_cast<int>(sizeof(InT)));
  static constexpr int tileB = align128(NP * TB * static_cast<int>(sizeof(InT)));
  static constexpr int stage = 3 * tileU + 2 * tileB;   // u, delta, z, B, C
  static constexpr int raw = 0;
  // two sets of fp32 tiles: Delta, Delta*u [CH][ROW]; B, C [NP][TB]
  static constexpr int set0 = raw + STAGES * stage;
  static constexpr int oDelta = 0;
  static constexpr int oDu = CH * ROW * 4;
  static constexpr int oB = 2 * CH * ROW * 4;
  static constexpr int oC = oB + NP * TB * 4;
  // trapezoidal update only: Delta_t u_{t-1} / 2 [CH][ROW]
  static constexpr int oQ = oC + NP * TB * 4;
  static constexpr int set = oQ + (TRAP ? CH * ROW * 4 : 0);
  // two sets of state-group shares of y: [G][CH][ROW]
  static constexpr int part0 = set0 + 2 * set;
  static constexpr int part = G * CH * ROW * 4;
  static constexpr int bias = part0 + 2 * part;          // fp32 [CH]
  static constexpr int dskip = bias + CH * 4;            // fp32 [CH]
  static constexpr int bars = dskip + CH * 4;            // u64 [STAGES]
  static constexpr int hand = bars + STAGES * 8;         // u64 [8] handoffs
  static constexpr int misc = hand + 8 * 8;              // int [4]
  static constexpr int bytes = misc + 16;
};

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) {
  return a < b ? a : b;
}

template <typename InT, typename OutT, int G, bool TMA, int MODE>
struct Scan {
  static constexpr bool VARLEN = MODE == kModeVarlen;
  static constexpr bool TRAP = MODE == kModeTrap;
  using Lay = Layout<InT, G, TRAP>;
  static constexpr int NP = 4 * G;

  const ScanParams &p;
  const TmaMaps &maps;
  unsigned char *smem;
  int64_t b, d0, t_begin, t_end;
  bool has_z;

  __device__ Scan(const ScanParams &p_, const TmaMaps &m_, unsigned char *s_)
      : p(p_), maps(m_), smem(s_), b(0), d0(0), t_begin(0), t_end(0),
        has_z(p_.z != nullptr) {}

  __device__ float *f32(int off) const { return reinterpret_cast<float *>(smem + off); }
  __device__ float *fset(int set, int off) const {
    return f32(Lay::set0 + set * Lay::set + off);
  }
  __device__ float *fpart(int set) const { return f32(Lay::part0 + set * Lay::part); }
  __device__ InT *raw(int stage, int which) const {
    const int off = Lay::raw + stage * Lay::stage +
                    (which < 3 ? which * Lay::tileU : 3 * Lay::tileU + (which - 3) * Lay::tileB);
    return reinterpret_cast<InT *>(smem + off);
  }
  __device__ uint64_t *bar(int stage) const {
    return reinterpret_cast<uint64_t *>(smem + Lay::bars) + stage;
  }
  // handoff barrier `kind` (0 tiles ready, 1 tiles free, 2 shares ready,
  // 3 shares free) of buffer set `set`
  __device__ uint64_t *hand(int kind, int set) const {
    return reinterpret_cast<uint64_t *>(smem + Lay::hand) + 2 * kind + set;
  }
  __device__ int64_t t0_of(int blk) const { return t_begin + static_cast<int64_t>(blk) * TB; }
  __device__ int nt_of(int blk) const {
    return static_cast<int>(min64(TB, t_end - t0_of(blk)));
  }

  // ---- packed sequences.  Index of the first interior start cu[i]
  // (1 <= i < nseq) at or after step pos, nseq when there is none.
  __device__ int64_t first_start_from(int64_t pos) const {
    int64_t lo = 1, hi = p.nseq;
    while (lo < hi) {
      const int64_t mid = lo + (hi - lo) / 2;
      if (__ldg(p.cu + mid) < pos) lo = mid + 1; else hi = mid;
    }
    return lo;
  }
  // Offset of interior start nb (nseq fits 32 bits, checked on the host).
  __device__ int start_at(int nb) const { return nb < p.nseq ? __ldg(p.cu + nb) : 0; }
  // Bit j (j < 4) set when step pos + j (< t_end) starts a sequence.  The
  // caller's cursor (nb, next = start_at(nb)) only moves forward, so a
  // window with no start in it costs one compare and no load.
  __device__ uint32_t restarts4(int64_t pos, int &nb, int &next) const {
    uint32_t m = 0;
    while (nb < p.nseq && next < pos + 4) {
      if (next >= pos && next < t_end) m |= 1u << (next - pos);
      next = start_at(++nb);
    }
    return m;
  }
  // A restart is a step of infinite Delta: exp(Delta A) = 0 while the
  // input term keeps the finite Delta (written to the Delta*u tile first).
  static __device__ __forceinline__ void mark_restarts(float4 &dl, uint32_t m) {
    const float inf = __int_as_float(0x7f800000);
    if (m & 1u) dl.x = inf;
    if (m & 2u) dl.y = inf;
    if (m & 4u) dl.z = inf;
    if (m & 8u) dl.w = inf;
  }

  // thread 0: start the TMA copies of block `blk` into `stage`
  __device__ void issue(int stage, int blk) const {
    const uint32_t bytes = static_cast<uint32_t>(
        (2 + (has_z ? 1 : 0)) * CH * TB * sizeof(InT) + 2 * NP * TB * sizeof(InT));
    uint64_t *bb = bar(stage);
    mbar_expect_tx(bb, bytes);
    const int x = static_cast<int>(t0_of(blk)), yd = static_cast<int>(d0),
              zb = static_cast<int>(b);
    tma_load_3d(raw(stage, 0), &maps.u, x, yd, zb, bb);
    tma_load_3d(raw(stage, 1), &maps.delta, x, yd, zb, bb);
    if (has_z) tma_load_3d(raw(stage, 2), &maps.z, x, yd, zb, bb);
    tma_load_3d(raw(stage, 3), &maps.B, x, 0, zb, bb);
    tma_load_3d(raw(stage, 4), &maps.C, x, 0, zb, bb);
  }

  // all threads: fill `stage` with block `blk` by plain loads (zero outside
  // the tensors); visible to other threads after the next barrier
  __device__ void load_plain(int stage, int blk, int ti, int nth) const {
    const int64_t t0 = t0_of(blk);
    const int nt = nt_of(blk);
    const InT zero = from_f32<InT>(0.f);
    const InT *gu = static_cast<const InT *>(p.u);
    const InT *gd = static_cast<const InT *>(p.delta);
    const InT *gz = static_cast<const InT *>(p.z);
    InT *ru = raw(stage, 0), *rd = raw(stage, 1), *rz = raw(stage, 2);
    for (int idx = ti; idx < CH * TB; idx += nth) {
      const int c = idx / TB, t = idx % TB;
      const bool ok = d0 + c < p.dim && t < nt;
      const int64_t d = d0 + c, tt = t0 + t;
      const int64_t iu = b * p.su[0] + d * p.su[1] + tt, idl = b * p.sdl[0] + d * p.sdl[1] + tt,
                    iz = b * p.sz[0] + d * p.sz[1] + tt;
      ru[idx] = ok && dbg_index_ok(iu, p.ext_u, p.status) ? gu[iu] : zero;
      rd[idx] = ok && dbg_index_ok(idl, p.ext_delta, p.status) ? gd[idl] : zero;
      if (has_z) rz[idx] = ok && dbg_index_ok(iz, p.ext_z, p.status) ? gz[iz] : zero;
    }
    const InT *gb = static_cast<const InT *>(p.B);
    const InT *gc = static_cast<const InT *>(p.C);
    InT *rb = raw(stage, 3), *rc = raw(stage, 4);
    for (int idx = ti; idx < NP * TB; idx += nth) {
      const int n = idx / TB, t = idx % TB;
      const bool ok = n < p.dstate && t < nt;
      const int64_t tt = t0 + t;
      const int64_t ib = b * p.sB[0] + n * p.sB[1] + tt, ic = b * p.sC[0] + n * p.sC[1] + tt;
      rb[idx] = ok && dbg_index_ok(ib, p.ext_B, p.status) ? gb[ib] : zero;
      rc[idx] = ok && dbg_index_ok(ic, p.ext_C, p.status) ? gc[ic] : zero;
    }
  }

  // Fill the raw stage of block `blk` (blocks past the chunk: nothing).
  // TMA: thread ti == 0 starts the copies, which complete the stage's
  // mbarrier.  Plain: the group of nth threads loads and each thread then
  // arrives on the mbarrier, whose arrival count is that group's size.
  __device__ void produce(int blk, int nblk, int ti, int nth) const {
    if (blk >= nblk) return;
    const int stage = blk % STAGES;
    if (TMA) {
      if (ti == 0) issue(stage, blk);
    } else {
      load_plain(stage, blk, ti, nth);
      mbar_arrive(bar(stage));
    }
  }

  // Wait (bounded) until the raw stage of block `blk` is complete; true
  // when it is.  Every thread that waits tracks the stage phases itself.
  __device__ bool wait_raw(int blk, int stage_base, uint32_t &phase) const {
    const int stage = (stage_base + blk) % STAGES;
    const bool ok = mbar_wait_bounded(bar(stage), (phase >> stage) & 1u, kTmaWaitNs);
    phase ^= 1u << stage;
    return ok;
  }

  // ---- main-pass prep/epilogue on fixed slots.  With 64 threads per role
  // and TB/4 groups of four steps per channel row, thread ti always owns the
  // groups ti + 64k (k < kSlots): channel row (ti + 64k) / (TB/4), steps
  // 4 (ti % (TB/4)) .. +3 of every block.  Everything that depends only on
  // the slot (rows, pointers, bias, D) is computed once per kernel.
  static constexpr int QT = TB / 4;
  static constexpr int kSlots = CH * QT / 64;
  static_assert(kSlots * 64 == CH * QT && 64 % QT == 0,
                "every slot of a thread must cover the same steps");
  struct Slots {
    int c[kSlots];
    int t;
    bool ok[kSlots];
    float bias[kSlots], dk[kSlots];
    OutT *yrow[kSlots];  // y of (b, d0 + c) at step t_begin + t
  };
  __device__ Slots make_slots(int ti) const {
    Slots sl;
    sl.t = 4 * (ti % QT);
    OutT *y = static_cast<OutT *>(p.y);
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
      const int c = (ti + 64 * k) / QT;
      const int64_t d = d0 + c;
      sl.c[k] = c;
      sl.ok[k] = d < p.dim;
      sl.bias[k] = (sl.ok[k] && p.delta_bias) ? p.delta_bias[d] : 0.f;
      sl.dk[k] = (sl.ok[k] && p.D) ? p.D[d] : 0.f;
      sl.yrow[k] = y + b * p.sy[0] + (sl.ok[k] ? d : d0) * p.sy[1] + t_begin + sl.t;
    }
    return sl;
  }

  // uprev0[k]: u of the step before the block for slot k (trapezoidal
  // update, slots starting the block only).
  __device__ void prep_slots(int stage, int set, int nt, const Slots &sl, int ti,
                             uint32_t restarts, const float (&uprev0)[kSlots]) const {
    const InT *ru = raw(stage, 0), *rd = raw(stage, 1);
    float *sDelta = fset(set, Lay::oDelta), *sDu = fset(set, Lay::oDu);
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
      const int c = sl.c[k], t = sl.t;
      const float4 u = load4_f32(ru + c * TB + t);
      const float4 dd = load4_f32(rd + c * TB + t);
      const float bias = sl.bias[k];
      float4 dl = make_float4(dd.x + bias, dd.y + bias, dd.z + bias, dd.w + bias);
      if (p.softplus) {
        const float2 a = softplus2_f(make_float2(dl.x, dl.y));
        const float2 a2 = softplus2_f(make_float2(dl.z, dl.w));
        dl = make_float4(a.x, a.y, a2.x, a2.y);
      }
      if (t + 4 > nt) {
        if (t >= nt) dl.x = 0.f;
        if (t + 1 >= nt) dl.y = 0.f;
        if (t + 2 >= nt) dl.z = 0.f;
        if (t + 3 >= nt) dl.w = 0.f;
      }
      if (TRAP) {
        // half-step weights: Delta_t u_t / 2 and Delta_t u_{t-1} / 2
        const float up = t > 0 ? to_f32<InT>(ru[c * TB + t - 1]) : uprev0[k];
        *reinterpret_cast<float4 *>(sDu + c * ROW + t) = make_float4(
            0.5f * dl.x * u.x, 0.5f * dl.y * u.y, 0.5f * dl.z * u.z, 0.5f * dl.w * u.w);
        *reinterpret_cast<float4 *>(fset(set, Lay::oQ) + c * ROW + t) = make_float4(
            0.5f * dl.x * up, 0.5f * dl.y * u.x, 0.5f * dl.z * u.y, 0.5f * dl.w * u.z);
      } else {
        *reinterpret_cast<float4 *>(sDu + c * ROW + t) =
            make_float4(dl.x * u.x, dl.y * u.y, dl.z * u.z, dl.w * u.w);
      }
      if (restarts) mark_restarts(dl, restarts);
      *reinterpret_cast<float4 *>(sDelta + c * ROW + t) = dl;
    }
    const InT *rb = raw(stage, 3), *rc = raw(stage, 4);
    float *sB = fset(set, Lay::oB), *sC = fset(set, Lay::oC);
#pragma unroll
    for (int k = 0; k < (2 * NP * TB + 4 * 64 - 1) / (4 * 64); ++k) {
      const int idx = 4 * (ti + 64 * k);
      if (idx >= 2 * NP * TB) break;
      if (idx < NP * TB) store4(sB + idx, load4_f32(rb + idx));
      else store4(sC + idx - NP * TB, load4_f32(rc + idx - NP * TB));
    }
  }

  __device__ void epilogue_slots(int stage, int set, int blk, const Slots &sl) const {
    const int nt = nt_of(blk);
    const int64_t toff = static_cast<int64_t>(blk) * TB;
    const InT *ru = raw(stage, 0), *rz = raw(stage, 2);
    const float *sPart = fpart(set);
    const int t = sl.t;
    if (t >= nt) return;
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
      if (!sl.ok[k]) continue;
      const int c = sl.c[k];
      // sum of the state-group shares, steps (t, t+1) and (t+2, t+3) paired
      float4 s = *reinterpret_cast<const float4 *>(sPart + c * ROW + t);
      float2 s01 = make_float2(s.x, s.y), s23 = make_float2(s.z, s.w);
#pragma unroll
      for (int g = 1; g < G; ++g) {
        const float4 v = *reinterpret_cast<const float4 *>(sPart + (g * CH + c) * ROW + t);
        s01 = __fadd2_rn(s01, make_float2(v.x, v.y));
        s23 = __fadd2_rn(s23, make_float2(v.z, v.w));
      }
      const float4 u = load4_f32(ru + c * TB + t);
      const float2 dk = make_float2(sl.dk[k], sl.dk[k]);
      s01 = __ffma2_rn(dk, make_float2(u.x, u.y), s01);
      s23 = __ffma2_rn(dk, make_float2(u.z, u.w), s23);
      if (has_z) {
        const float4 z = load4_f32(rz + c * TB + t);
        s01 = __fmul2_rn(s01, make_float2(silu_f(z.x), silu_f(z.y)));
        s23 = __fmul2_rn(s23, make_float2(silu_f(z.z), silu_f(z.w)));
      }
      s = make_float4(s01.x, s01.y, s23.x, s23.y);
      OutT *yr = sl.yrow[k] + toff;
#if MSS_DEBUG
      {
        int64_t yi = yr - static_cast<OutT *>(p.y);
        // test flag: the store of channel d0, steps 0..3 of the first block
        // aims one tensor length past y (the check must catch and skip it)
        if ((p.test_flags & 2u) && blockIdx.x == 0 && blk == 0 && sl.c[k] == 0 && t == 0) {
          yi += p.ext_y;
          yr += p.ext_y;
        }
        if (!dbg_index_ok(yi + min64(nt - t, 4) - 1, p.ext_y, p.status)) continue;
      }
#endif
      if (p.y_vec && t + 4 <= nt) {
        store4(yr, s);
      } else {
        const float sv[4] = {s.x, s.y, s.z, s.w};
        for (int j = 0; j < 4 && t + j < nt; ++j) yr[j] = from_f32<OutT>(sv[j]);
      }
    }
  }

  // The recurrence over one block for this lane's channel and 4 states:
  // h = exp(Delta A) h + Delta B u, with this warp's share of
  // y_t = sum_n C_t[n] h_t[n] written to part set `set`.  Exponents and
  // inputs of steps (t, t+1) go through one paired f32x2 instruction, as do
  // the shares of y.
  // Trapezoidal update: the input term of step t gains the previous input,
  // decayed over the step, e_t (Delta_t u_{t-1} / 2) B_{t-1}[n]; bprev holds
  // B_{t-1}[n] of this lane's states across quads and blocks.
  // steps 4 q0 .. 4 q1 - 1 of the block (the whole block: 0, TB / 4)
  __device__ void scan(int set, int g, int lane, float (&h)[4],
                       const float2 (&al2)[4], float &dsum, bool split,
                       float (&bprev)[4], int q0 = 0, int q1 = TB / 4) const {
    const float *sDelta = fset(set, Lay::oDelta), *sDu = fset(set, Lay::oDu);
    const float *sB = fset(set, Lay::oB), *sC = fset(set, Lay::oC);
    float *sPart = fpart(set);
#pragma unroll
    for (int q = q0; q < q1; ++q) {
      const float4 dl = *reinterpret_cast<const float4 *>(&sDelta[lane * ROW + 4 * q]);
      const float4 du = *reinterpret_cast<const float4 *>(&sDu[lane * ROW + 4 * q]);
      const float2 dl01 = make_float2(dl.x, dl.y), dl23 = make_float2(dl.z, dl.w);
      const float2 du01 = make_float2(du.x, du.y), du23 = make_float2(du.z, du.w);
      float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (TRAP) qv = *reinterpret_cast<const float4 *>(&fset(set, Lay::oQ)[lane * ROW + 4 * q]);
      float2 p01 = make_float2(0.f, 0.f), p23 = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = 4 * g + i;
        const float4 bq = *reinterpret_cast<const float4 *>(&sB[n * TB + 4 * q]);
        const float4 cq = *reinterpret_cast<const float4 *>(&sC[n * TB + 4 * q]);
        const float2 x01 = __fmul2_rn(dl01, al2[i]);
        const float2 x23 = __fmul2_rn(dl23, al2[i]);
        float2 b01 = __fmul2_rn(du01, make_float2(bq.x, bq.y));
        float2 b23 = __fmul2_rn(du23, make_float2(bq.z, bq.w));
        // the last kPolyStates states of the group take their decays from
        // the FMA-pipe polynomial, the others from the special-function unit
        float2 e01, e23;
        if (i >= 4 - kPolyStates) {
          e01 = exp2_poly2(x01);
          e23 = exp2_poly2(x23);
        } else {
          e01 = make_float2(ex2_mufu(x01.x), ex2_mufu(x01.y));
          e23 = make_float2(ex2_mufu(x23.x), ex2_mufu(x23.y));
        }
        if (TRAP) {
          const float2 q01 = __fmul2_rn(make_float2(qv.x, qv.y), make_float2(bprev[i], bq.x));
          const float2 q23 = __fmul2_rn(make_float2(qv.z, qv.w), make_float2(bq.y, bq.z));
          b01 = __ffma2_rn(e01, q01, b01);
          b23 = __ffma2_rn(e23, q23, b23);
          bprev[i] = bq.w;
        }
        float2 h01, h23;
        h01.x = fmaf(e01.x, h[i], b01.x);
        h01.y = fmaf(e01.y, h01.x, b01.y);
        h23.x = fmaf(e23.x, h01.y, b23.x);
        h23.y = fmaf(e23.y, h23.x, b23.y);
        h[i] = h23.y;
        p01 = __ffma2_rn(make_float2(cq.x, cq.y), h01, p01);
        p23 = __ffma2_rn(make_float2(cq.z, cq.w), h23, p23);
      }
      *reinterpret_cast<float4 *>(&sPart[(g * CH + lane) * ROW + 4 * q]) =
          make_float4(p01.x, p01.y, p23.x, p23.y);
      if (split) dsum += (dl.x + dl.y) + (dl.z + dl.w);
    }
  }

};

// Warp roles of one block: G scan warps (one per group of 4 states), two
// prep warps and two epilogue warps.  They hand tiles and y shares over
// through mbarriers in shared memory (one per kind and buffer set), so each
// warp waits only for the data it needs and never for its siblings; every
// wait is bounded.
constexpr int kPrepWarps = 2;  // the slot layout of prep/epilogue assumes
constexpr int kEpiWarps = 2;   // 64 threads per role
constexpr int kAuxWarps = kPrepWarps + kEpiWarps;
constexpr int kTilesReady = 0;  // prep -> scan: fp32 tiles of a block written
constexpr int kTilesFree = 1;   // scan -> prep: tiles of a block consumed
constexpr int kPartReady = 2;   // scan -> epi: y shares of a block written
constexpr int kPartFree = 3;    // epi -> scan: y shares of a block consumed
constexpr int kBarEpi = 1;      // named barrier of the epilogue warps only
constexpr uint64_t kHandoffWaitNs = 2000000000ull;

// (checkpoint mode: 4 blocks per SM asked for, so the extra stores of the
// mid-block states do not cost a resident block; the other modes give ptxas
// no minimum, which keeps their register allocation)
template <typename InT, typename OutT, int G, bool TMA, int MODE>
__global__ void __launch_bounds__(32 * (G + kAuxWarps), MODE == kModeCkpt ? 4 : 0)
    scan_fwd_kernel(const ScanParams p, const __grid_constant__ TmaMaps maps) {
  using S = Scan<InT, OutT, G, TMA, MODE>;
  constexpr bool VARLEN = S::VARLEN;
  constexpr bool TRAP = S::TRAP;
  constexpr bool CKPT = MODE == kModeCkpt;
  using Lay = typename S::Lay;
  constexpr int NP = 4 * G;
  constexpr int NSCAN = 32 * G;
  constexpr int NPREP = 32 * kPrepWarps;
  constexpr int NEPI = 32 * kEpiWarps;
  extern __shared__ __align__(128) unsigned char smem[];
  S sc(p, maps, smem);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const bool is_scan = tid < NSCAN;
  const int g = is_scan ? (tid >> 5) : 0;  // state group of a scan warp
  const bool is_prep = !is_scan && tid < NSCAN + NPREP;
  const int tp = tid - NSCAN;              // index within the prep warps
  const int te = tid - NSCAN - NPREP;      // index within the epilogue warps
  const bool split = p.splits > 1;

  int *misc = reinterpret_cast<int *>(smem + Lay::misc);
  if (tid == 0) {
    // split scans hand out items (chunk-major) in the order blocks start
    misc[0] = split ? static_cast<int>(atomicAdd(p.ticket, 1u))
                    : static_cast<int>(blockIdx.x);
    // a raw stage completes when its TMA bytes land (one arrival) or when
    // every epilogue thread has stored its share of the plain loads
    for (int s = 0; s < STAGES; ++s) mbar_init(sc.bar(s), TMA ? 1 : NEPI);
    for (int set = 0; set < 2; ++set) {
      mbar_init(sc.hand(kTilesReady, set), NPREP);
      mbar_init(sc.hand(kTilesFree, set), NSCAN);
      mbar_init(sc.hand(kPartReady, set), NSCAN);
      mbar_init(sc.hand(kPartFree, set), NEPI);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int64_t item = misc[0];
  const int64_t k = item / p.tiles;  // sequence chunk (chunk-major order)
  const int64_t tile = item % p.tiles;
  sc.b = tile / p.ch_tiles;
  sc.d0 = (tile % p.ch_tiles) * CH;
  sc.t_begin = k * p.chunk;
  sc.t_end = min64(sc.t_begin + p.chunk, p.seqlen);
  const int64_t b = sc.b, d0 = sc.d0;
  const int64_t d = d0 + lane;
  const bool dvalid = is_scan && d < p.dim;
  const int nblk = static_cast<int>((sc.t_end - sc.t_begin + TB - 1) / TB);
  if (tid < CH) {
    const bool ok = d0 + tid < p.dim;
    sc.f32(Lay::bias)[tid] = (ok && p.delta_bias) ? p.delta_bias[d0 + tid] : 0.f;
    sc.f32(Lay::dskip)[tid] = (ok && p.D) ? p.D[d0 + tid] : 0.f;
  }

  float alpha[4], h[4];
  bool live[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = 4 * g + i;
    live[i] = dvalid && n < p.dstate;
    live[i] = live[i] && dbg_index_ok(d * p.dstate + n, p.dim * p.dstate, p.status);
    alpha[i] = live[i] ? p.A[d * p.dstate + n] * kLog2e : 0.f;
    // with packed sequences a restart multiplies alpha by an infinite
    // Delta: keep A = 0 states at a decay of exactly 1 elsewhere but 0 there
    if (VARLEN && alpha[i] == 0.f) alpha[i] = -1e-30f;
    const int64_t si = (b * p.dim + d) * p.dstate + n;
    live[i] = live[i] && dbg_index_ok(si, p.batch * p.dim * p.dstate, p.status);
    h[i] = (live[i] && k == 0 && p.h0) ? p.h0[si] : 0.f;
  }
  // trapezoidal update: B_{t-1}[n] of the step before this chunk (none
  // before the sequence starts)
  float bprev[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bprev[i] = 0.f;
    if (TRAP && live[i] && sc.t_begin > 0)
      bprev[i] = to_f32<InT>(static_cast<const InT *>(p.B)[b * p.sB[0] + (4 * g + i) * p.sB[1] +
                                                          sc.t_begin - 1]);
  }
  float dsum = 0.f;
  float2 al2[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) al2[i] = make_float2(alpha[i], alpha[i]);
  uint32_t phase = 0;

  // ------------------------------------------------------------ main pass
  // Scan warps only run the recurrence.  Prep warps turn raw block i+2 into
  // fp32 tiles while block i is scanned; epilogue warps write the outputs of
  // block i and then refill its raw stage with block i+STAGES.  Tiles and y
  // shares are double buffered (set = block & 1).  A wait that runs out is
  // recorded and the pipeline carries on, so no warp is ever left waiting.
  __syncthreads();  // bias / D tiles, barrier initialisation
  bool ok = true;
  uint32_t hp = 0;  // parities of the handoff barriers this thread waits on
  auto wait_hand = [&](int kind, int set) {
    const int bit = 2 * kind + set;
    ok &= mbar_wait_bounded(sc.hand(kind, set), (hp >> bit) & 1u, kHandoffWaitNs);
    hp ^= 1u << bit;
  };
  if (is_scan) {
    for (int i = 0; i < nblk; ++i) {
      const int s = i & 1;
      wait_hand(kTilesReady, s);
      if (i >= 2) wait_hand(kPartFree, s);
      if (CKPT) {
        // state before block i for the backward pass (unsplit plans only),
        // and in the second array the state entering its step 8
        const int64_t ci = ((item * nblk + i) * NP + 4 * g) * static_cast<int64_t>(CH) + lane;
        const int64_t arr = p.tiles * static_cast<int64_t>(nblk) * NP * CH;
        float *ck = p.ckpt_out + ci;
        const bool ok = dbg_index_ok(ci + 3 * CH, p.ext_ckpt, p.status) &&
                        dbg_index_ok(arr + ci + 3 * CH, p.ext_ckpt, p.status);
        if (ok) {
#pragma unroll
          for (int j = 0; j < 4; ++j) ck[j * CH] = h[j];
        }
        sc.scan(s, g, lane, h, al2, dsum, split, bprev, 0, TB / 8);
        if (ok) {
#pragma unroll
          for (int j = 0; j < 4; ++j) ck[arr + j * CH] = h[j];
        }
        sc.scan(s, g, lane, h, al2, dsum, split, bprev, TB / 8, TB / 4);
      } else {
        sc.scan(s, g, lane, h, al2, dsum, split, bprev);
      }
      if (i + 2 < nblk) mbar_arrive(sc.hand(kTilesFree, s));
      mbar_arrive(sc.hand(kPartReady, s));
    }
  } else if (is_prep) {
    const typename S::Slots sl = sc.make_slots(tp);
    // cursor into the sequence offsets for this thread's steps
    int nb = VARLEN ? static_cast<int>(sc.first_start_from(sc.t_begin + sl.t)) : 0;
    int next_start = VARLEN ? sc.start_at(nb) : 0;
    // split scans: this thread's share of each slot's running sum of Delta;
    // the four threads of a channel row write the sum at every segment
    // start for the carry launch
    float psum[S::kSlots];
#pragma unroll
    for (int k = 0; k < S::kSlots; ++k) psum[k] = 0.f;
    for (int blk = 0; blk < nblk; ++blk) {
      if (split && blk % kSegBlocks == 0) {
#pragma unroll
        for (int k = 0; k < S::kSlots; ++k) {
          float v = psum[k] + __shfl_xor_sync(0xffffffffu, psum[k], 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          if (sl.t == 0 && sl.ok[k])
            p.sig[(item * p.nseg + blk / kSegBlocks) * CH + sl.c[k]] = v;
        }
      }
      if (blk >= 2) wait_hand(kTilesFree, blk & 1);
      const uint32_t rs = VARLEN ? sc.restarts4(sc.t0_of(blk) + sl.t, nb, next_start) : 0u;
      // trapezoidal update: u of the step before the block, for the slots
      // that start it (read from HBM/L2: the previous raw stage may already
      // be refilled)
      float up0[S::kSlots];
#pragma unroll
      for (int k = 0; k < S::kSlots; ++k) {
        up0[k] = 0.f;
        const int64_t tp0 = sc.t0_of(blk) - 1;
        if (TRAP && sl.t == 0 && sl.ok[k] && tp0 >= 0)
          up0[k] = to_f32<InT>(static_cast<const InT *>(p.u)[b * p.su[0] +
                                                             (d0 + sl.c[k]) * p.su[1] + tp0]);
      }
      ok &= sc.wait_raw(blk, 0, phase);
      sc.prep_slots(blk % STAGES, blk & 1, sc.nt_of(blk), sl, tp, rs, up0);
      if (split) {
        const float *sDelta = sc.fset(blk & 1, Lay::oDelta);
#pragma unroll
        for (int k = 0; k < S::kSlots; ++k) {
          const float4 dl = *reinterpret_cast<const float4 *>(sDelta + sl.c[k] * ROW + sl.t);
          psum[k] += (dl.x + dl.y) + (dl.z + dl.w);
        }
      }
      mbar_arrive(sc.hand(kTilesReady, blk & 1));
    }
  } else {
    const typename S::Slots sl = sc.make_slots(te);
    for (int j = 0; j < STAGES; ++j) sc.produce(j, nblk, te, NEPI);
    for (int i = 0; i < nblk; ++i) {
      const int s = i & 1;
      wait_hand(kPartReady, s);
      ok &= sc.wait_raw(i, 0, phase);
      sc.epilogue_slots(i % STAGES, s, i, sl);
      if (i + 2 < nblk) mbar_arrive(sc.hand(kPartFree, s));
      // the raw stage of block i is free once every epilogue thread is done
      bar_sync(kBarEpi, NEPI);
      sc.produce(i + STAGES, nblk, te, NEPI);
    }
  }
  if (!ok) atomicOr(p.status, kStatusTimeout);

  if (!split) {
    if (p.last_state) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (live[i]) p.last_state[(b * p.dim + d) * p.dstate + 4 * g + i] = h[i];
    }
    return;
  }

  // ---- split mode: the chunk's pair (P, e) for the prefix launch, which
  // also writes the final state; the carried terms are added by the carry
  // launch
  float *my_agg = p.agg + item * static_cast<int64_t>(2) * CH * NP;
  if (is_scan) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      my_agg[(4 * g + i) * CH + lane] = ex2_mufu(alpha[i] * dsum);
      my_agg[CH * NP + (4 * g + i) * CH + lane] = h[i];
    }
  }
}

// ------------------------------------------------------ split: prefix
// One block of 32 x 32 threads per (tile, state) composes the chunks'
// pairs in chunk order into incl_k = P_k incl_{k-1} + e_k, the true state at
// the end of chunk k (incl_0 = e_0: the first chunk started from h0), and
// writes the final state.  Thread (c, j) holds channel c (rows of the pairs
// are read coalesced) and the j-th run of consecutive chunks: it composes
// its run, the runs' pairs are scanned per channel through shared memory
// (composition is associative: "The relay"), and the thread replays its
// run from the state before it.  Under MSS_TESTFLAG_DROP_PUBLISH the first
// thread first waits for a word of the workspace that nothing sets, bounded
// by the caller's spin timeout, and records the timeout in the status word.
__global__ void __launch_bounds__(1024) scan_prefix_kernel(const ScanParams p, int np) {
  __shared__ float sP[32][33], sE[32][33];
  const int c = threadIdx.x, j = threadIdx.y;
  const int64_t tile = blockIdx.x / np;
  const int n = static_cast<int>(blockIdx.x % np);
  if ((p.test_flags & 1u) && blockIdx.x == 0 && c == 0 && j == 0) {
    const uint64_t limit = p.spin_timeout_ns > 0 ? static_cast<uint64_t>(p.spin_timeout_ns)
                                                 : 1000000000ull;
    const uint64_t start = global_timer_ns();
    while (ld_acquire_gpu(p.status + 2) == 0u) {
      if (global_timer_ns() - start > limit) {
        atomicOr(p.status, kStatusTimeout);
        break;
      }
      __nanosleep(1000);
    }
  }
  const int64_t per_tile = static_cast<int64_t>(np) * CH;
  const int r = n * CH + c;
  const int64_t stride = 2 * per_tile;
  const int run = (p.splits + 31) / 32;
  const int k0 = min(p.splits, j * run), k1 = min(p.splits, k0 + run);
  auto pair = [&](int k, float &P, float &e) {
    const int64_t item = static_cast<int64_t>(k) * p.tiles + tile;
    P = k == 0 ? 0.f : p.agg[item * stride + r];  // nothing precedes chunk 0
    e = p.agg[item * stride + per_tile + r];
  };
  // this thread's run as one pair: h -> P h + E (pairs read eight at a time
  // so their loads overlap)
  float P = 1.f, E = 0.f;
  for (int k = k0; k < k1; k += 8) {
    float pk[8], ek[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      pk[q] = 1.f;
      ek[q] = 0.f;
      if (k + q < k1) pair(k + q, pk[q], ek[q]);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      E = fmaf(pk[q], E, ek[q]);
      P *= pk[q];
    }
  }
  sP[j][c] = P;
  sE[j][c] = E;
  __syncthreads();
  // warp j scans channel j's runs (lane = run), the earlier pair first,
  // and leaves the state before each run
  {
    float q = sP[c][j], x = sE[c][j];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float qo = __shfl_up_sync(0xffffffffu, q, o);
      const float xo = __shfl_up_sync(0xffffffffu, x, o);
      if (c >= o) {
        x = fmaf(q, xo, x);
        q *= qo;
      }
    }
    const float before = __shfl_up_sync(0xffffffffu, x, 1);
    __syncthreads();
    sE[c][j] = c == 0 ? 0.f : before;
  }
  __syncthreads();
  float h = sE[j][c];
  for (int k = k0; k < k1; k += 8) {
    float pk[8], ek[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (k + q < k1) pair(k + q, pk[q], ek[q]);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (k + q >= k1) break;
      h = fmaf(pk[q], h, ek[q]);
      p.incl[(static_cast<int64_t>(k + q) * p.tiles + tile) * per_tile + r] = h;
    }
  }
  if (p.last_state && k1 == p.splits && k0 < k1) {
    const int64_t b = tile / p.ch_tiles, d = (tile % p.ch_tiles) * CH + c;
    if (d < p.dim && n < p.dstate) p.last_state[(b * p.dim + d) * p.dstate + n] = h;
  }
}

// ------------------------------------------------------- split: carry
// 16-byte asynchronous copy global -> shared (through L2 only), tracked by
// the thread's groups.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// wait until at most N of this thread's committed groups are in flight
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The piece of a 16-step row that thread-level copy unit `w` (elements
// w .. w + 16/sizeof(T) - 1) covers: one asynchronous copy when the row is
// whole and aligned, element loads of the steps inside the chunk otherwise.
template <typename T>
__device__ __forceinline__ void stage_piece(T *dst, const T *row, int w, int nt, bool vec) {
  constexpr int EL = 16 / static_cast<int>(sizeof(T));
  if (vec && nt == TB) {
    cp_async16(dst + w, row + w);
  } else {
    for (int e = 0; e < EL && w + e < nt; ++e) dst[w + e] = row[w + e];
  }
}

// One block per (tile, chunk k >= 1, segment of kSegBlocks blocks): adds
// silu(z_t) * sum_n C_t[n] 2^(alpha[n] sigma_t) h_in[n] to the segment's y,
// block by block, until every term has decayed below the cutoff.  Warp g
// takes the states g + G i (i < 4), so every warp holds slow and fast
// states, and skips a state once its term is below the cutoff in all its
// lanes (lane = channel).  The raw delta, z, C and old y of a block are
// staged in shared memory two blocks ahead (three buffers).
template <typename InT, typename OutT, int G, bool VARLEN>
__global__ void __launch_bounds__(32 * G) scan_carry_kernel(const ScanParams p) {
  constexpr int NP = 4 * G;
  constexpr int NT = 32 * G;
  constexpr int QT = TB / 4;
  __shared__ __align__(16) InT rD[3][CH * TB];
  __shared__ __align__(16) InT rZ[3][CH * TB];
  __shared__ __align__(16) InT rC[3][NP * TB];
  __shared__ __align__(16) OutT rY[3][CH * TB];
  __shared__ __align__(16) float sDl[CH * ROW];
  __shared__ __align__(16) float sPart[G][CH * ROW];
  __shared__ float sBias[CH];

  const int tid = threadIdx.x, lane = tid & 31, g = tid >> 5;
  const int64_t unit = blockIdx.x;
  const int seg = static_cast<int>(unit % p.nseg);
  const int64_t rest = unit / p.nseg;
  const int64_t tile = rest % p.tiles;
  const int64_t k = rest / p.tiles + 1;
  const int64_t item = k * p.tiles + tile;
  const int64_t b = tile / p.ch_tiles, d0 = (tile % p.ch_tiles) * CH;
  const int64_t t_begin = k * p.chunk;
  const int64_t t_end = min64(t_begin + p.chunk, p.seqlen);
  const int nblk = static_cast<int>((t_end - t_begin + TB - 1) / TB);
  const int blk0 = seg * p.segb;
  if (blk0 >= nblk) return;
  const int blk1 = min(nblk, blk0 + p.segb);

  // this lane's states g + G i: rate, carried state, still-active mask
  const int64_t d = d0 + lane;
  const bool dvalid = d < p.dim;
  float sigma = p.sig[(item * p.nseg + seg) * CH + lane];
  float alpha[4], hin[4];
  unsigned act = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = g + G * i;
    const bool live = dvalid && n < p.dstate &&
                      dbg_index_ok(d * p.dstate + n, p.dim * p.dstate, p.status);
    alpha[i] = live ? p.A[d * p.dstate + n] * kLog2e : 0.f;
    if (VARLEN && alpha[i] == 0.f) alpha[i] = -1e-30f;
    hin[i] = live ? p.incl[(item - p.tiles) * NP * CH + n * CH + lane] : 0.f;
    if (__any_sync(0xffffffffu, hin[i] != 0.f && !(alpha[i] * sigma < kCutoffLog2)))
      act |= 1u << i;
  }
  if (tid < CH) {
    const bool ok = d0 + tid < p.dim;
    sBias[tid] = (ok && p.delta_bias) ? p.delta_bias[d0 + tid] : 0.f;
  }
  if (!__syncthreads_or(act != 0u)) return;

  const bool has_z = p.z != nullptr;
  auto vec_ok = [&](const void *ptr, const int64_t (&st)[2], int es) {
    return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0 && (st[0] * es) % 16 == 0 &&
           (st[1] * es) % 16 == 0;
  };
  const bool vD = vec_ok(p.delta, p.sdl, sizeof(InT));
  const bool vZ = has_z && vec_ok(p.z, p.sz, sizeof(InT));
  const bool vC = vec_ok(p.C, p.sC, sizeof(InT));
  const bool vY = vec_ok(p.y, p.sy, sizeof(OutT));
  constexpr int PI = TB * static_cast<int>(sizeof(InT)) / 16;   // copy units per input row
  constexpr int PO = TB * static_cast<int>(sizeof(OutT)) / 16;  // per y row
  constexpr int EI = 16 / static_cast<int>(sizeof(InT)), EO = 16 / static_cast<int>(sizeof(OutT));
  constexpr int NU = 2 * CH * PI + NP * PI + CH * PO;
  auto stage = [&](int j, int buf) {
    const int64_t t0 = t_begin + static_cast<int64_t>(j) * TB;
    const int nt = static_cast<int>(min64(TB, t_end - t0));
    for (int q = tid; q < NU; q += NT) {
      if (q < CH * PI) {
        const int c = q / PI, w = (q % PI) * EI;
        if (d0 + c < p.dim)
          stage_piece(rD[buf] + c * TB, static_cast<const InT *>(p.delta) + b * p.sdl[0] +
                                            (d0 + c) * p.sdl[1] + t0,
                      w, nt, vD);
      } else if (q < 2 * CH * PI) {
        const int qq = q - CH * PI, c = qq / PI, w = (qq % PI) * EI;
        if (has_z && d0 + c < p.dim)
          stage_piece(rZ[buf] + c * TB, static_cast<const InT *>(p.z) + b * p.sz[0] +
                                            (d0 + c) * p.sz[1] + t0,
                      w, nt, vZ);
      } else if (q < 2 * CH * PI + NP * PI) {
        const int qq = q - 2 * CH * PI, n = qq / PI, w = (qq % PI) * EI;
        if (n < p.dstate)
          stage_piece(rC[buf] + n * TB,
                      static_cast<const InT *>(p.C) + b * p.sC[0] + n * p.sC[1] + t0, w, nt, vC);
      } else {
        const int qq = q - 2 * CH * PI - NP * PI, c = qq / PO, w = (qq % PO) * EO;
        if (d0 + c < p.dim)
          stage_piece(rY[buf] + c * TB, static_cast<const OutT *>(p.y) + b * p.sy[0] +
                                            (d0 + c) * p.sy[1] + t0,
                      w, nt, vY);
      }
    }
    cp_async_commit();
  };

  stage(blk0, 0);
  if (blk0 + 1 < blk1)
    stage(blk0 + 1, 1);
  else
    cp_async_commit();
  for (int j = blk0; j < blk1; ++j) {
    const int buf = (j - blk0) % 3;
    const int64_t t0 = t_begin + static_cast<int64_t>(j) * TB;
    const int nt = static_cast<int>(min64(TB, t_end - t0));
    // block j's copies (this thread's, then everyone's) have landed; block
    // j - 1 is consumed, so its buffer may take block j + 2
    cp_async_wait<1>();
    __syncthreads();
    if (j + 2 < blk1)
      stage(j + 2, (j - blk0 + 2) % 3);
    else
      cp_async_commit();
    // Delta = softplus(delta + bias), zero past the chunk, infinite where a
    // packed sequence restarts
    for (int qd = tid; qd < CH * QT; qd += NT) {
      const int c = qd / QT, t = 4 * (qd % QT);
      float4 dl = make_float4(0.f, 0.f, 0.f, 0.f);
      if (d0 + c < p.dim && t < nt) {
        const InT *r = rD[buf] + c * TB + t;
        const float bias = sBias[c];
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = t + e < nt ? to_f32<InT>(r[e]) + bias : 0.f;
        if (p.softplus) {
          const float2 a = softplus2_f(make_float2(v[0], v[1]));
          const float2 c2 = softplus2_f(make_float2(v[2], v[3]));
          v[0] = a.x; v[1] = a.y; v[2] = c2.x; v[3] = c2.y;
        }
        dl = make_float4(t < nt ? v[0] : 0.f, t + 1 < nt ? v[1] : 0.f, t + 2 < nt ? v[2] : 0.f,
                         t + 3 < nt ? v[3] : 0.f);
        if (VARLEN && p.cu) {
          // binary search for the first sequence start at or after t0 + t
          const int64_t pos = t0 + t;
          int64_t lo = 1, hi = p.nseq;
          while (lo < hi) {
            const int64_t mid = lo + (hi - lo) / 2;
            if (__ldg(p.cu + mid) < pos) lo = mid + 1; else hi = mid;
          }
          const float inf = __int_as_float(0x7f800000);
          for (int64_t nb = lo; nb < p.nseq && __ldg(p.cu + nb) < pos + 4; ++nb) {
            const int e = static_cast<int>(__ldg(p.cu + nb) - pos);
            if (e == 0) dl.x = inf;
            if (e == 1) dl.y = inf;
            if (e == 2) dl.z = inf;
            if (e == 3) dl.w = inf;
          }
        }
      }
      *reinterpret_cast<float4 *>(sDl + c * ROW + t) = dl;
    }
    __syncthreads();
    // this warp's share of the carried terms of block j
    {
      float *share = sPart[g];
      if (act == 0u) {
#pragma unroll
        for (int q = 0; q < QT; ++q)
          *reinterpret_cast<float4 *>(share + lane * ROW + 4 * q) = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
#pragma unroll
        for (int q = 0; q < QT; ++q) {
          const float4 dl = *reinterpret_cast<const float4 *>(sDl + lane * ROW + 4 * q);
          float2 s01, s23;  // sigma after steps 4q .. 4q + 3
          sigma += dl.x;
          s01.x = sigma;
          sigma += dl.y;
          s01.y = sigma;
          sigma += dl.z;
          s23.x = sigma;
          sigma += dl.w;
          s23.y = sigma;
          float2 p01 = make_float2(0.f, 0.f), p23 = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (!((act >> i) & 1u)) continue;
            const float4 cq = load4_f32(rC[buf] + (g + G * i) * TB + 4 * q);
            const float2 a2 = make_float2(alpha[i], alpha[i]), h2 = make_float2(hin[i], hin[i]);
            const float2 x01 = __fmul2_rn(a2, s01), x23 = __fmul2_rn(a2, s23);
            p01 = __ffma2_rn(__fmul2_rn(make_float2(cq.x, cq.y), h2),
                             make_float2(ex2_mufu(x01.x), ex2_mufu(x01.y)), p01);
            p23 = __ffma2_rn(__fmul2_rn(make_float2(cq.z, cq.w), h2),
                             make_float2(ex2_mufu(x23.x), ex2_mufu(x23.y)), p23);
          }
          *reinterpret_cast<float4 *>(share + lane * ROW + 4 * q) =
              make_float4(p01.x, p01.y, p23.x, p23.y);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (!__any_sync(0xffffffffu, hin[i] != 0.f && !(alpha[i] * sigma < kCutoffLog2)))
            act &= ~(1u << i);
      }
    }
    const bool more = __syncthreads_or(act != 0u);
    // y += silu(z) * (sum of the shares), four steps of one channel per thread
    for (int qd = tid; qd < CH * QT; qd += NT) {
      const int c = qd / QT, t = 4 * (qd % QT);
      if (d0 + c >= p.dim || t >= nt) continue;
      float4 sv = *reinterpret_cast<const float4 *>(sPart[0] + c * ROW + t);
#pragma unroll
      for (int w = 1; w < G; ++w) {
        const float4 v = *reinterpret_cast<const float4 *>(sPart[w] + c * ROW + t);
        sv.x += v.x; sv.y += v.y; sv.z += v.z; sv.w += v.w;
      }
      float o[4] = {sv.x, sv.y, sv.z, sv.w};
      const OutT *yo = rY[buf] + c * TB + t;
      const InT *zr = rZ[buf] + c * TB + t;
      const int64_t yi = b * p.sy[0] + (d0 + c) * p.sy[1] + t0 + t;
      OutT *yr = static_cast<OutT *>(p.y) + yi;
      if (!dbg_index_ok(yi + min(nt - t, 4) - 1, p.ext_y, p.status)) continue;
      if (t + 4 <= nt) {
        if (has_z) {
          const float4 z = load4_f32(zr);
          const float2 g01 = silu2_f(make_float2(z.x, z.y));
          const float2 g23 = silu2_f(make_float2(z.z, z.w));
          o[0] *= g01.x; o[1] *= g01.y; o[2] *= g23.x; o[3] *= g23.y;
        }
        const float4 old = load4_f32(yo);
        const float4 nv = make_float4(old.x + o[0], old.y + o[1], old.z + o[2], old.w + o[3]);
        if (p.y_vec) {
          store4(yr, nv);
        } else {
          const float nvs[4] = {nv.x, nv.y, nv.z, nv.w};
          for (int e = 0; e < 4; ++e) yr[e] = from_f32<OutT>(nvs[e]);
        }
      } else {
        for (int e = 0; e < 4 && t + e < nt; ++e) {
          const float gate = has_z ? silu_f(to_f32<InT>(zr[e])) : 1.f;
          yr[e] = from_f32<OutT>(to_f32<OutT>(yo[e]) + o[e] * gate);
        }
      }
    }
    if (!more) break;
  }
  cp_async_wait<0>();  // no copy may land after the block has left
}

// ------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool encode_3d(CUtensorMap *m, const void *ptr, bool bf16, uint64_t len,
               uint64_t rows, uint64_t batch, const int64_t (&st)[2], uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const uint64_t es = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {len, rows, batch};
  cuuint64_t strides[2] = {static_cast<uint64_t>(st[1]) * es, static_cast<uint64_t>(st[0]) * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(TB), box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
             3, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tma_eligible(const ScanParams &p, int in_bf16) {
  const uint64_t es = in_bf16 ? 2 : 4;
  auto al = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  if ((p.seqlen * es) % 16 != 0) return false;
  // TMA strides are multiples of 16 bytes below 2^40
  auto st_ok = [&](const int64_t (&s)[2]) {
    return (s[0] * static_cast<int64_t>(es)) % 16 == 0 &&
           (s[1] * static_cast<int64_t>(es)) % 16 == 0 &&
           s[0] * static_cast<int64_t>(es) < (int64_t(1) << 40);
  };
  if (!st_ok(p.su) || !st_ok(p.sdl) || !st_ok(p.sB) || !st_ok(p.sC) || (p.z && !st_ok(p.sz)))
    return false;
  if (p.seqlen >= (int64_t(1) << 31) || p.dim >= (int64_t(1) << 31) ||
      p.batch >= (int64_t(1) << 31))
    return false;
  if (!al(p.u) || !al(p.delta) || !al(p.B) || !al(p.C) || (p.z && !al(p.z)))
    return false;
  return tensor_map_encoder() != nullptr;
}

bool build_maps(const ScanParams &p, int in_bf16, int groups, TmaMaps *m) {
  const uint32_t np = 4 * groups;
  const uint64_t L = p.seqlen, D = p.dim, N = p.dstate, Bt = p.batch;
  if (!encode_3d(&m->u, p.u, in_bf16, L, D, Bt, p.su, CH)) return false;
  if (!encode_3d(&m->delta, p.delta, in_bf16, L, D, Bt, p.sdl, CH)) return false;
  if (p.z && !encode_3d(&m->z, p.z, in_bf16, L, D, Bt, p.sz, CH)) return false;
  if (!encode_3d(&m->B, p.B, in_bf16, L, N, Bt, p.sB, np)) return false;
  if (!encode_3d(&m->C, p.C, in_bf16, L, N, Bt, p.sC, np)) return false;
  return true;
}

template <typename InT, typename OutT, int G, bool TMA, int MODE>
cudaError_t launch_typed(const ScanParams &p, const TmaMaps &maps, cudaStream_t s) {
  auto kern = scan_fwd_kernel<InT, OutT, G, TMA, MODE>;
  const int smem = Layout<InT, G, MODE == kModeTrap>::bytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.tiles * p.splits;
  kern<<<static_cast<unsigned>(grid), 32 * (G + kAuxWarps), smem, s>>>(p, maps);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.splits <= 1) return e;
  // split scans: the chunks' true start states, then the carried terms
  scan_prefix_kernel<<<static_cast<unsigned>(p.tiles * 4 * G), dim3(32, 32), 0, s>>>(p, 4 * G);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t units = p.tiles * (p.splits - 1) * p.nseg;
  scan_carry_kernel<InT, OutT, G, MODE == kModeVarlen>
      <<<static_cast<unsigned>(units), 32 * G, 0, s>>>(p);
  return cudaGetLastError();
}

// Packed sequences and the trapezoidal update get their own instantiations,
// so their code never touches the kernels of ordinary scans.
template <typename InT, typename OutT, int MODE>
cudaError_t dispatch_v(const ScanParams &p, bool tma, const TmaMaps &maps, cudaStream_t s) {
  const int G = static_cast<int>((p.dstate + 3) / 4);
  if (tma) {
    switch (G) {
      case 1: return launch_typed<InT, OutT, 1, true, MODE>(p, maps, s);
      case 2: return launch_typed<InT, OutT, 2, true, MODE>(p, maps, s);
      default: return launch_typed<InT, OutT, 4, true, MODE>(p, maps, s);
    }
  }
  switch (G) {
    case 1: return launch_typed<InT, OutT, 1, false, MODE>(p, maps, s);
    case 2: return launch_typed<InT, OutT, 2, false, MODE>(p, maps, s);
    default: return launch_typed<InT, OutT, 4, false, MODE>(p, maps, s);
  }
}

template <typename InT, typename OutT>
cudaError_t dispatch(const ScanParams &p, bool tma, const TmaMaps &maps, cudaStream_t s) {
  if (p.cu) return dispatch_v<InT, OutT, kModeVarlen>(p, tma, maps, s);
  if (p.trap) return dispatch_v<InT, OutT, kModeTrap>(p, tma, maps, s);
  if (p.ckpt_out) return dispatch_v<InT, OutT, kModeCkpt>(p, tma, maps, s);
  return dispatch_v<InT, OutT, kModePlain>(p, tma, maps, s);
}

template <typename InT, typename OutT, int G>
int occupancy_typed() {
  int n = 0;
  auto kern = scan_fwd_kernel<InT, OutT, G, true, kModePlain>;
  const int smem = Layout<InT, G>::bytes;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 32 * (G + kAuxWarps), smem) !=
      cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

template <typename InT, typename OutT>
int occupancy_g(int groups) {
  switch (groups) {
    case 1: return occupancy_typed<InT, OutT, 1>();
    case 2: return occupancy_typed<InT, OutT, 2>();
    default: return occupancy_typed<InT, OutT, 4>();
  }
}

}  // namespace

// groups 3 runs on the 4-group kernel (the fourth group's states are padding)
static int kernel_groups(int groups) { return groups == 3 ? 4 : groups; }

size_t scan_workspace_clear_bytes() { return 256; }

static int64_t segments_per_chunk(int64_t chunk) {
  const int64_t nblk = (chunk + TB - 1) / TB;
  return (nblk + kSegBlocks - 1) / kSegBlocks;
}

static size_t round256(size_t n) { return ((n + 255) / 256) * 256; }

size_t scan_workspace_bytes(int64_t tiles, int splits, int64_t chunk, int groups) {
  if (splits <= 1) return 0;
  const size_t items = static_cast<size_t>(tiles) * splits;
  const size_t np = 4 * static_cast<size_t>(kernel_groups(groups));
  const size_t agg = items * 2 * CH * np * sizeof(float);
  const size_t incl = items * CH * np * sizeof(float);
  const size_t sig = items * static_cast<size_t>(segments_per_chunk(chunk)) * CH * sizeof(float);
  return scan_workspace_clear_bytes() + round256(agg) + round256(incl) + round256(sig);
}

// Layout: status word, ticket and the word the test flag waits for in the
// first 256 bytes, then the chunks' pairs, their true end states and the running
// sums of Delta at the segment starts.
void scan_bind_workspace(ScanParams &p, void *ws, int groups) {
  char *base = static_cast<char *>(ws);
  const size_t items = static_cast<size_t>(p.tiles) * p.splits;
  const size_t np = 4 * static_cast<size_t>(kernel_groups(groups));
  p.status = reinterpret_cast<unsigned *>(base);
  p.ticket = reinterpret_cast<unsigned *>(base + 4);
  size_t off = scan_workspace_clear_bytes();
  p.agg = reinterpret_cast<float *>(base + off);
  off += round256(items * 2 * CH * np * sizeof(float));
  p.incl = reinterpret_cast<float *>(base + off);
  off += round256(items * CH * np * sizeof(float));
  p.sig = reinterpret_cast<float *>(base + off);
  p.segb = kSegBlocks;
  p.nseg = static_cast<int>(segments_per_chunk(p.chunk));
}

// The word's device address, looked up once per device (with that device
// current) and cached.
unsigned *scan_status_word() {
  constexpr int kDevices = 64;
  static unsigned *addr[kDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < kDevices && addr[dev]) return addr[dev];
  void *ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_scan_status) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < kDevices) addr[dev] = static_cast<unsigned *>(ptr);
  return static_cast<unsigned *>(ptr);
}

int scan_blocks_per_sm(int in_bf16, int out_bf16, int groups) {
  using BF = __nv_bfloat16;
  const int G = kernel_groups(groups);
  switch ((in_bf16 ? 2 : 0) + (out_bf16 ? 1 : 0)) {
    case 0: return occupancy_g<float, float>(G);
    case 1: return occupancy_g<float, BF>(G);
    case 2: return occupancy_g<BF, float>(G);
    default: return occupancy_g<BF, BF>(G);
  }
}

cudaError_t launch_scan_fwd(const ScanParams &params, int in_bf16, int out_bf16,
                            cudaStream_t stream) {
  using BF = __nv_bfloat16;
  ScanParams p = params;
  const uintptr_t yv = 4 * (out_bf16 ? 2 : 4);
  p.y_vec = (p.sy[0] % 4 == 0) && (p.sy[1] % 4 == 0) &&
            (reinterpret_cast<uintptr_t>(p.y) % yv == 0);
  TmaMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const int groups = kernel_groups(static_cast<int>((p.dstate + 3) / 4));
  const bool tma = tma_eligible(p, in_bf16) && build_maps(p, in_bf16, groups, &maps);
  if (in_bf16)
    return out_bf16 ? dispatch<BF, BF>(p, tma, maps, stream)
                    : dispatch<BF, float>(p, tma, maps, stream);
  return out_bf16 ? dispatch<float, BF>(p, tma, maps, stream)
                  : dispatch<float, float>(p, tma, maps, stream);
}

}  // namespace sss48
