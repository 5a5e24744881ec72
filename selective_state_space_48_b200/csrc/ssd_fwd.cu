// ssd_fwd.cu -- Mamba-2 (SSD) chunked scan on the sm_100a tensor cores.
//
// With A a scalar per head, the scan of one head over a chunk of Q = 128
// steps is four matrix products ("State Space Models and the
// Post-Transformer Era", section "Mamba-2 and Structured State Space
// Duality"; "The State That Must Remember Everything", Part 4):
//
//   S  = C B^T                       M = t, N = s, K = n   (both K-major)
//   Y  = S' X,   S'[t,s] = S[t,s] 2^(c_t - c_s) Delta_s  for s <= t, else 0
//                                    M = t, N = p, K = s   (A in tensor memory,
//                                                         B operand MN-major)
//   YO = C Hp,   Hp = the state before the chunk (bf16 copy)
//                                    M = t, N = p, K = n   (B operand MN-major)
//   H  = 2^(c_last) H + B^T X'',  X''[s,p] = X[s,p] Delta_s 2^(c_last - c_s)
//                                    M = n, N = p, K = s   (both MN-major)
//
// with c_t the running sum of Delta A log2(e) inside the chunk, and the
// output y_t = Y_t + 2^(c_t) YO_t + D x_t (times silu(z_t)).  One CTA owns
// one (batch row, head) and walks its chunks in order, so the state H is
// carried in tensor memory (fp32) across the whole sequence and never
// touches HBM.  Warp roles: warp 0 issues the TMA loads of the C, B and X
// tiles (two stages), warp 1 allocates tensor memory and issues the
// tcgen05.mma products (one thread), warps 2-17 (512 threads, four warps
// per tensor memory lane quarter, which split the columns) compute
// the step sizes and their running sum, build the operand S' in tensor
// memory and X'' and Hp in shared memory, rescale H, and write y.  The state products (YO and H)
// are issued as soon as Hp and X'' are ready, so they run while the
// epilogue builds the masked scores S'.
//
// The grid has one CTA per sequence, so batch * nheads CTAs fill the SMs in
// waves.  When the last wave is at most half full (r sequences), those r
// sequences are cut at chunk boundaries into `parts` pieces (about SMs / r,
// at most the number of full waves + 1) and the pieces are spread over the
// schedule: CTAs take work items in ticket order, and the order is piece 0
// of the r sequences, a share of the whole sequences, piece 1, another
// share, ..., the last piece.  A piece therefore starts only after the
// piece before it was taken by a running CTA, normally long after that one
// ended, and the last wave holds short pieces instead of whole sequences.
// A piece publishes its end state (fp32, in the caller's workspace) with a
// release flag; the next piece loads it as its initial state.  Every piece
// runs exactly the per-chunk arithmetic of the whole sequence, so the output
// is the same bit for bit.
//
// Shared memory tiles are [128 rows][64 bf16] with the 128-byte swizzle that
// the TMA writes and the tensor core reads: 16-byte chunk j of row r sits at
// chunk position j ^ (r % 8).  Every wait on an mbarrier is bounded; a wait
// that runs out records a timeout in the status word and the CTA finishes
// its loop without waiting further, so no CTA can hang.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "device_math.cuh"
#include "nvtx_range.cuh"
#include "selective_scan.h"
#include "ssd.h"

namespace sss48 {
namespace ssd {

constexpr int Q = 128;   // chunk length
constexpr int P = 64;    // headdim
constexpr int NS = 128;  // dstate
constexpr int kThreads = 576;  // 2 issue warps + 16 epilogue warps
constexpr int kEpi = 512;
constexpr int kEpiBarrier = 1;  // named barrier of the sixteen epilogue warps
constexpr int kHalfBarrier = 2; // + half: named barrier of the eight warps of a y half

constexpr int kTile = Q * 64 * 2;      // one [128][64] bf16 tile
constexpr int kStage = 5 * kTile;      // C (two n halves), B (two), X
constexpr int oC = 0, oB = 2 * kTile, oX = 4 * kTile;
constexpr int oXpp = 2 * kStage;       // X''
constexpr int oHp = oXpp + kTile;      // bf16 copy of the state, [n][p]
constexpr int oCum = oHp + kTile;      // float c_s [Q]
constexpr int oStep = oCum + Q * 4;    // float Delta_s [Q]
constexpr int oColf = oStep + Q * 4;   // float column factors [Q]
constexpr int oTot = oColf + Q * 4;    // float warp totals [4]
constexpr int oBar = oTot + 16;        // 10 mbarriers
constexpr int oTmemSlot = oBar + 10 * 8;
constexpr int oAbort = oTmemSlot + 4;
constexpr int oItem = oAbort + 4;      // this CTA's work item
constexpr int kSmemUsed = oAbort + 12;
constexpr int kSmemBytes = kSmemUsed + 1024;  // room to align the base
static_assert(kSmemBytes <= 232448, "shared memory above the per-block limit");

// tensor memory columns (fp32, lane = row)
constexpr uint32_t kColS = 0, kColY = 128, kColYO = 192, kColH = 256;
constexpr uint32_t kColSp = 320;  // S' as bf16 pairs: 64 columns
constexpr uint32_t kTmemCols = 512;

// barrier indices: tiles landed / released (per stage), scores S done,
// masked scores S' ready, Hp ready, the state update's operands ready (X'',
// H rescaled), the output products Y and YO done, the state update done
constexpr int kFull = 0, kEmpty = 2, kSFull = 4, kReadyScores = 5, kReadyState = 6,
              kDoneY = 7, kDoneH = 8, kReadyHp = 9;

struct Params {
  int64_t batch, L, H, G;
  const __nv_bfloat16 *dt;
  const float *A, *D, *dt_bias;
  int softplus;
  const __nv_bfloat16 *z;
  const float *h0;
  void *y;
  int y_bf16;
  float *last;
  unsigned *status;
  uint64_t spin_ns;
  // cut sequences: the last ncut of the batch * nheads order, in `parts`
  // pieces, with gfull whole sequences between two pieces (the rest before
  // the last piece); ticket, flags and end states in the workspace
  int ncut, parts;
  int64_t gfull;
  unsigned *ticket;
  unsigned *flag;  // [(parts - 1) * ncut]: 1 once the piece's end state is written
  float *mid;      // [(parts - 1) * ncut][P][NS]: end states of all but the last pieces
};

struct Maps {
  CUtensorMap x, B, C, y;
};

__device__ unsigned g_ssd_status;

// ---------------------------------------------------------------- PTX

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, int c3, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_addr(bar))
      : "memory");
}

// 4-D tiled TMA store of a shared-memory box (rows past the tensor's end
// are not written), tracked by this thread's bulk group
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *map, const void *src, int c0,
                                             int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_addr(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the shared memory of this thread's bulk stores may be overwritten
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// this thread's bulk stores are complete
__device__ __forceinline__ void tma_store_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// generic-proxy shared-memory writes -> visible to the tensor core
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 in, fp32 accumulate)
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: A is M lanes of K bf16 values packed two
// per 32-bit column (K slice kk at column offset 8 kk)
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive on `bar` once every tcgen05.mma issued so far by this thread is done
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// 32 consecutive fp32 columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr));
}

// 16 consecutive fp32 columns of this thread's lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

// The loaded registers are valid only after tcgen05.wait::ld; threading
// them through the wait keeps the compiler from using them earlier.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]),
                 "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                 "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]),
                 "+r"(v[27]), "+r"(v[28]), "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&v)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------ UMMA descriptors

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2),
// version 1; addresses and offsets in 16-byte units.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFF) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) | (uint64_t(1) << 46) |
         (uint64_t(2) << 61);
}

// K-major operand stored as two [128 rows][64] tiles (K = 0..63, 64..127):
// the 16-wide K slice kk starts 32 bytes into a row of tile kk / 4; rows
// advance 128 bytes, 8-row groups 1024.
__device__ __forceinline__ uint64_t desc_k(uint32_t tile0, int kk) {
  return smem_desc(tile0 + (kk >> 2) * kTile + (kk & 3) * 32, 16, 1024);
}

// MN-major operand: rows are K, 64 MN values per 128-byte row, 16 K rows
// per instruction (2048 bytes), a second 64-wide MN block `lbo` bytes on.
__device__ __forceinline__ uint64_t desc_mn(uint32_t tile, int kk, uint32_t lbo) {
  return smem_desc(tile + kk * 2048, lbo, 1024);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&u);
  return __bfloat1622float2(v);
}

// byte offset of 16-byte chunk j of row r in a swizzled [128][64] tile
__device__ __forceinline__ uint32_t swz(int r, int j) {
  return static_cast<uint32_t>(r * 128 + ((j ^ (r & 7)) << 4));
}

// ------------------------------------------------------------- kernel

struct Sync {
  uint64_t *bar;
  volatile int *abort;
  unsigned *status;
  uint64_t limit;
  // bounded wait; after the first timeout in the CTA every wait returns at
  // once (the results are then garbage, but nothing hangs)
  __device__ void wait(int i, uint32_t parity) const {
    if (*abort) return;
    if (!mbar_wait_bounded(bar + i, parity, limit)) {
      *abort = 1;
      atomicOr(status, static_cast<unsigned>(MSS_ERR_TIMEOUT));
    }
  }
  // bounded wait that is not skipped after a timeout: used before exit for
  // copies and products still in flight
  __device__ void drain(int i, uint32_t parity) const {
    if (!mbar_wait_bounded(bar + i, parity, limit)) {
      *abort = 1;
      atomicOr(status, static_cast<unsigned>(MSS_ERR_TIMEOUT));
    }
  }
};

// Step sizes of chunk c (row r of the e = 0 warps), their running sum c_t
// in log2 units and the column factors 2^(c_end - c_s) Delta_s, c_end the
// last step of s's 32-step block, into shared memory.  `dt_next` holds
// the bits of chunk c's raw bf16 step on entry and chunk c + 1's on exit
// (converted only when used, so the load's latency is not waited for here).
// Ends with every epilogue thread past the second barrier.
struct StepPlan {
  float *cum_s, *step_s, *colf_s, *tot_s;
  const __nv_bfloat16 *dtp;
  int64_t L, H;
  float A2, bias;
  int softplus;
  __device__ void run(int c, int q, int e, int lane, int r, unsigned short &dt_next) const {
    const int64_t t = static_cast<int64_t>(c) * Q + r;
    float cw = 0.0f, step = 0.0f;
    if (e == 0) {
      if (t < L) {
        const float v = __uint_as_float(static_cast<uint32_t>(dt_next) << 16) + bias;
        step = softplus ? softplus_f(v) : v;
      }
      if (t + Q < L)
        dt_next = *reinterpret_cast<const unsigned short *>(dtp + (t + Q) * H);
      cw = step * A2;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, cw, o);
        if (lane >= o) cw += u;
      }
      if (lane == 31) tot_s[q] = cw;
    }
    bar_sync(kEpiBarrier, kEpi);
    if (e == 0) {
      float base = 0.0f;
      for (int j = 0; j < q; ++j) base += tot_s[j];
      const float cum = base + cw;
      const float cend = base + __shfl_sync(0xffffffffu, cw, 31);
      cum_s[r] = cum;
      step_s[r] = step;
      colf_s[r] = ex2_mufu(cend - cum) * step;
    }
    bar_sync(kEpiBarrier, kEpi);
  }
};

// Work item -> sequence bh and its chunks [c0, c0 + nc), and the state
// slots of a piece: `in` holds its initial state, `out` receives its end
// state (-1: the caller's h0 / last_state).  Items in ticket order: piece 0
// of the cut sequences, gfull whole sequences, piece 1, gfull more, ...,
// the remaining whole sequences, the last piece.
struct Work {
  int64_t bh;
  int c0, nc, in, out;
  static __device__ Work of(int item, const Params &p, int nchunks) {
    Work w{item, 0, nchunks, -1, -1};
    if (!p.ncut) return w;
    const int64_t F = p.batch * p.H - p.ncut;  // whole sequences
    int64_t pos = item, full = 0;
    for (int j = 0; j < p.parts; ++j) {
      if (pos < p.ncut) {  // piece j of cut sequence si
        const int si = static_cast<int>(pos);
        w.bh = F + si;
        w.c0 = static_cast<int>(static_cast<int64_t>(j) * nchunks / p.parts);
        w.nc = static_cast<int>(static_cast<int64_t>(j + 1) * nchunks / p.parts) - w.c0;
        w.in = j > 0 ? (j - 1) * p.ncut + si : -1;
        w.out = j < p.parts - 1 ? j * p.ncut + si : -1;
        return w;
      }
      pos -= p.ncut;
      if (j < p.parts - 1) {
        const int64_t gs = j < p.parts - 2 ? p.gfull : F - p.gfull * (p.parts - 2);
        if (pos < gs) {
          w.bh = full + pos;
          return w;
        }
        pos -= gs;
        full += gs;
      }
    }
    return w;  // not reached: the grid has F + parts * ncut items
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    ssd_fwd_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nchunks = static_cast<int>((p.L + Q - 1) / Q);

  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + oBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + oTmemSlot);
  volatile int *abort = reinterpret_cast<volatile int *>(sm + oAbort);
  float *cum_s = reinterpret_cast<float *>(sm + oCum);
  float *step_s = reinterpret_cast<float *>(sm + oStep);
  float *colf_s = reinterpret_cast<float *>(sm + oColf);
  float *tot_s = reinterpret_cast<float *>(sm + oTot);
  const Sync sy{bar, abort, p.status, p.spin_ns};

  if (tid == 0) {
    mbar_init(bar + kFull, 1);
    mbar_init(bar + kFull + 1, 1);
    mbar_init(bar + kEmpty, kEpi);
    mbar_init(bar + kEmpty + 1, kEpi);
    mbar_init(bar + kSFull, 1);
    mbar_init(bar + kReadyScores, kEpi);
    mbar_init(bar + kReadyState, kEpi);
    mbar_init(bar + kReadyHp, kEpi);
    mbar_init(bar + kDoneY, 1);
    mbar_init(bar + kDoneH, 1);
    *abort = 0;
    *reinterpret_cast<int *>(sm + oItem) =
        p.ncut ? static_cast<int>(atomicAdd(p.ticket, 1u)) : static_cast<int>(blockIdx.x);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const Work wk = Work::of(*reinterpret_cast<const int *>(sm + oItem), p, nchunks);
  const int c0 = wk.c0, nc = wk.nc;
  const int b = static_cast<int>(wk.bh / p.H), h = static_cast<int>(wk.bh % p.H);
  const int g = static_cast<int>(h / (p.H / p.G));

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer
    if (lane == 0) {
      for (int i = 0; i < nc; ++i) {
        const int st = i & 1;
        if (i >= 2) sy.wait(kEmpty + st, ((i >> 1) - 1) & 1);
        unsigned char *s = sm + st * kStage;
        uint64_t *full = bar + kFull + st;
        mbar_expect_tx(full, kStage);
        const int t0 = (c0 + i) * Q;
        tma_load_4d(s + oC, &maps.C, 0, g, t0, b, full);
        tma_load_4d(s + oC + kTile, &maps.C, 64, g, t0, b, full);
        tma_load_4d(s + oB, &maps.B, 0, g, t0, b, full);
        tma_load_4d(s + oB + kTile, &maps.B, 64, g, t0, b, full);
        tma_load_4d(s + oX, &maps.x, 0, h, t0, b, full);
      }
      // no copy may still be landing when the CTA exits
      for (int i = nc > 2 ? nc - 2 : 0; i < nc; ++i) sy.drain(kFull + (i & 1), (i >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------- tensor-core issue
    // Descriptors of the 16-wide K slices differ from slice 0's only in the
    // start-address field (16-byte units), by compile-time offsets.
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idY = idesc_bf16(128, 64, 0, 1);
      constexpr uint32_t idH = idesc_bf16(128, 64, 1, 1);
      const uint64_t dHp = desc_mn(sbase + oHp, 0, kTile);
      const uint64_t dXpp = desc_mn(sbase + oXpp, 0, kTile);
      // S = C B^T of this CTA's i-th chunk (stage i % 2), after its tiles
      // have landed
      auto scores = [&](int i) {
        const uint32_t s = sbase + (i & 1) * kStage;
        const uint64_t dC = desc_k(s + oC, 0), dBk = desc_k(s + oB, 0);
        sy.wait(kFull + (i & 1), (i >> 1) & 1);
        tc_fence_after();
        if (!*abort) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ko = (kk >> 2) * (kTile >> 4) + (kk & 3) * 2;
            umma_bf16(tmem + kColS, dC + ko, dBk + ko, idS, kk > 0);
          }
        }
        umma_commit(bar + kSFull);
      };
      // The tensor pipe runs products in issue order: Y, then YO as soon as
      // Hp is written, then the next chunk's scores, then this chunk's state
      // update, which is needed only after the next chunk's masked scores
      // are built.
      if (nc > 0) scores(0);
      for (int i = 0; i < nc; ++i) {
        const uint32_t s = sbase + (i & 1) * kStage;
        const uint64_t dC = desc_k(s + oC, 0);
        const uint64_t dBm = desc_mn(s + oB, 0, kTile), dX = desc_mn(s + oX, 0, kTile);
        sy.wait(kReadyScores, i & 1);
        tc_fence_after();
        if (!*abort) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // Y = S' X, S' from tensor memory
            umma_bf16_ts(tmem + kColY, tmem + kColSp + 8 * kk, dX + kk * 128, idY, kk > 0);
        }
        sy.wait(kReadyHp, i & 1);
        tc_fence_after();
        if (!*abort) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // YO = C Hp
            umma_bf16(tmem + kColYO, dC + (kk >> 2) * (kTile >> 4) + (kk & 3) * 2,
                      dHp + kk * 128, idY, kk > 0);
        }
        umma_commit(bar + kDoneY);
        if (i + 1 < nc) scores(i + 1);
        sy.wait(kReadyState, i & 1);
        tc_fence_after();
        if (!*abort) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // H += B^T X''
            umma_bf16(tmem + kColH, dBm + kk * 128, dXpp + kk * 128, idH, 1);
        }
        umma_commit(bar + kDoneH);
      }
      // every product done before the tensor memory is freed
      if (nc > 0) sy.drain(kDoneH, (nc - 1) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- epilogue
    // Four warps per tensor-memory lane quarter: e = 0 .. 3 takes columns
    // 16e .. 16e + 15 of the 64-wide products and score block e of the
    // masked scores; y is written in two 32-column halves (e / 2).
    const int q = warp & 3;
    const int e = (warp - 2) >> 2;
    const int half = e >> 1, sub = e & 1;
    const int r = 32 * q + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const float Dh = p.D ? p.D[h] : 0.0f;
    const int64_t H = p.H;
    // one thread per half issues the half's y stores (first lane of one of
    // the half's warps)
    const bool writer = lane == 0 && q == 2 && sub == 0;
    const StepPlan plan{cum_s, step_s, colf_s, tot_s,
                        p.dt + static_cast<int64_t>(b) * p.L * H + h, p.L, H,
                        p.A[h] * kLog2e, p.dt_bias ? p.dt_bias[h] : 0.0f, p.softplus};

    // the initial state into H (row n = r, columns 16e .. 16e + 15): the
    // caller's h0, or for a later piece the end state of the piece before,
    // once published (one thread waits, bounded; the barrier passes it on)
    {
      const float *h0 = p.h0 ? p.h0 + (static_cast<int64_t>(b) * H + h) * P * NS : nullptr;
      if (wk.in >= 0) {
        if (tid == 64) {
          const uint64_t start = global_timer_ns();
          while (ld_acquire_gpu(p.flag + wk.in) == 0u) {
            if (global_timer_ns() - start > p.spin_ns) {
              *abort = 1;
              atomicOr(p.status, static_cast<unsigned>(MSS_ERR_TIMEOUT));
              break;
            }
            __nanosleep(256);
          }
          __threadfence();
        }
        bar_sync(kEpiBarrier, kEpi);
        h0 = p.mid + static_cast<int64_t>(wk.in) * P * NS;
      }
      uint32_t v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        v[j] = __float_as_uint(h0 ? __ldcg(h0 + (e * 16 + j) * NS + r) : 0.0f);
      tmem_st16(tl + kColH + 16 * e, v);
      tmem_wait_st();
    }

    // raw steps are loaded one chunk ahead
    unsigned short dt_next = 0;
    const int64_t tfirst = static_cast<int64_t>(c0) * Q + r;
    if (e == 0 && tfirst < p.L)
      dt_next = *reinterpret_cast<const unsigned short *>(plan.dtp + tfirst * H);
    plan.run(c0, q, e, lane, r, dt_next);
    float cum = cum_s[r], cl = cum_s[Q - 1];

    // chunk c = c0 + i of the sequence; barrier phases and stages follow i
    for (int i = 0; i < nc; ++i) {
      const int c = c0 + i;
      const int st = i & 1;
      unsigned char *s = sm + st * kStage;
      const int64_t t = static_cast<int64_t>(c) * Q + r;

      // S' row t, block gb = e of 32 columns: below the diagonal
      // S 2^(c_t - c_end(gb)) colf[s] (both factors <= 1); on the diagonal
      // S 2^(c_t - c_s) Delta_s for s <= t, factored the same way when that
      // cannot overflow; above it zero
      sy.wait(kSFull, i & 1);
      tc_fence_after();
      {
        const int gb = e;
        uint32_t pk[16];
        if (gb < q) {
          uint32_t v[32];
          tmem_ld32(tl + kColS + 32 * gb, v);
          const float rf = ex2_mufu(cum - cum_s[32 * gb + 31]);
          tmem_wait_ld(v);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const int s0 = 32 * gb + j;
            pk[j >> 1] = pack_bf16(__uint_as_float(v[j]) * rf * colf_s[s0],
                                   __uint_as_float(v[j + 1]) * rf * colf_s[s0 + 1]);
          }
        } else if (gb == q) {
          uint32_t v[32];
          tmem_ld32(tl + kColS + 32 * gb, v);
          const float cend = cum_s[32 * gb + 31];
          // the same two factors when the block decays by less than 2^64
          // (2^(c_t - c_end) <= 2^64 cannot overflow); else one 2^x each
          const bool fact = cum_s[32 * gb] - cend < 64.0f;  // warp-uniform
          const float rf = ex2_mufu(cum - cend);
          tmem_wait_ld(v);
          if (fact) {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const int s0 = 32 * gb + j;
              const float f0 = j <= lane ? __uint_as_float(v[j]) * rf * colf_s[s0] : 0.0f;
              const float f1 =
                  j + 1 <= lane ? __uint_as_float(v[j + 1]) * rf * colf_s[s0 + 1] : 0.0f;
              pk[j >> 1] = pack_bf16(f0, f1);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const int s0 = 32 * gb + j;
              const float f0 = j <= lane ? __uint_as_float(v[j]) *
                                               ex2_mufu(cum - cum_s[s0]) * step_s[s0]
                                         : 0.0f;
              const float f1 = j + 1 <= lane ? __uint_as_float(v[j + 1]) *
                                                   ex2_mufu(cum - cum_s[s0 + 1]) * step_s[s0 + 1]
                                             : 0.0f;
              pk[j >> 1] = pack_bf16(f0, f1);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) pk[j] = 0u;
        }
        tmem_st16(tl + kColSp + 16 * gb, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar + kReadyScores);

      // the previous chunk's state update is done: its tiles (B read by it,
      // C holding the staged y) may be released once the y store has read
      // the staging tile
      if (i >= 1) {
        sy.wait(kDoneH, (i - 1) & 1);
        tc_fence_after();
        if (writer) {
          tma_store_wait_read();
          mbar_arrive(bar + kEmpty + ((i - 1) & 1));
        }
      }
      sy.wait(kFull + st, (i >> 1) & 1);

      // Hp row n = r (columns 16e .. 16e + 15): bf16 copy of the state
      // before this chunk; then the state decays over the chunk:
      // H *= 2^(c_last)
      {
        const float gam = ex2_mufu(cl);
        uint32_t v[16];
        tmem_ld16(tl + kColH + 16 * e, v);
        tmem_wait_ld(v);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          uint4 o;
          o.x = pack_bf16(__uint_as_float(v[8 * k + 0]), __uint_as_float(v[8 * k + 1]));
          o.y = pack_bf16(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3]));
          o.z = pack_bf16(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5]));
          o.w = pack_bf16(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7]));
          *reinterpret_cast<uint4 *>(sm + oHp + swz(r, e * 2 + k)) = o;
        }
        // the carried-state readout YO = C Hp may start now
        fence_async_smem();
        mbar_arrive(bar + kReadyHp);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * gam);
        tmem_st16(tl + kColH + 16 * e, v);
        tmem_wait_st();
      }
      // X'' row s = r, two of its eight 16-byte chunks (the XOR with the
      // row keeps the eight rows of a shared-memory phase on distinct banks)
      {
        const float w = step_s[r] * ex2_mufu(cl - cum);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint32_t off = static_cast<uint32_t>(r * 128 + (((e * 2 + k) ^ (r & 7)) << 4));
          const uint4 xv = *reinterpret_cast<const uint4 *>(s + oX + off);
          const float2 a0 = unpack_bf16(xv.x), a1 = unpack_bf16(xv.y);
          const float2 a2 = unpack_bf16(xv.z), a3 = unpack_bf16(xv.w);
          *reinterpret_cast<uint4 *>(sm + oXpp + off) =
              make_uint4(pack_bf16(a0.x * w, a0.y * w), pack_bf16(a1.x * w, a1.y * w),
                         pack_bf16(a2.x * w, a2.y * w), pack_bf16(a3.x * w, a3.y * w));
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar + kReadyState);

      // the next chunk's steps, while the output products run
      const float cum_t = cum;
      if (i + 1 < nc) {
        plan.run(c + 1, q, e, lane, r, dt_next);
        cum = cum_s[r];
        cl = cum_s[Q - 1];
      }

      // y row t, columns 16e .. 16e + 15: Y + 2^(c_t) YO + D x, gated
      sy.wait(kDoneY, i & 1);
      tc_fence_after();
      {
        const float eo = ex2_mufu(cum_t);
        uint32_t yv[16], ov[16];
        tmem_ld16(tl + kColY + 16 * e, yv);
        tmem_ld16(tl + kColYO + 16 * e, ov);
        tmem_wait_ld(yv);
        tmem_wait_ld(ov);
        float out[16];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint4 xv = *reinterpret_cast<const uint4 *>(s + oX + swz(r, e * 2 + k));
          const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 xf = unpack_bf16(xw[i]);
            const int j = 8 * k + 2 * i;
            out[j] = fmaf(eo, __uint_as_float(ov[j]), __uint_as_float(yv[j])) + Dh * xf.x;
            out[j + 1] =
                fmaf(eo, __uint_as_float(ov[j + 1]), __uint_as_float(yv[j + 1])) + Dh * xf.y;
          }
        }
        if (p.z && t < p.L) {
          const int64_t row = ((static_cast<int64_t>(b) * p.L + t) * H + h) * P + 16 * e;
          const uint4 *zr = reinterpret_cast<const uint4 *>(p.z + row);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint4 zv = zr[k];
            const uint32_t zw[4] = {zv.x, zv.y, zv.z, zv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 zf = unpack_bf16(zw[i]);
              out[8 * k + 2 * i] *= silu_f(zf.x);
              out[8 * k + 2 * i + 1] *= silu_f(zf.y);
            }
          }
        }
        // stage row t of the half's 32 columns in the stage's C tile (free
        // once the output products are done) and store the half's 128 x 32
        // box with one TMA store
        unsigned char *yt = s + oC + half * kTile;
        if (p.y_bf16) {
          // 64-byte rows, 64-byte swizzle: chunk k at k ^ ((t / 2) % 4)
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int j = 2 * sub + k;
            *reinterpret_cast<uint4 *>(yt + r * 64 + ((j ^ ((r >> 1) & 3)) << 4)) =
                make_uint4(pack_bf16(out[8 * k], out[8 * k + 1]),
                           pack_bf16(out[8 * k + 2], out[8 * k + 3]),
                           pack_bf16(out[8 * k + 4], out[8 * k + 5]),
                           pack_bf16(out[8 * k + 6], out[8 * k + 7]));
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<float4 *>(yt + swz(r, 4 * sub + k)) =
                make_float4(out[4 * k], out[4 * k + 1], out[4 * k + 2], out[4 * k + 3]);
        }
        fence_async_smem();
        bar_sync(kHalfBarrier + half, kEpi / 2);
        if (writer) tma_store_4d(&maps.y, yt, 32 * half, h, c * Q, b);
      }
      tc_fence_before();
      // the writer releases the stage in the next chunk, after the state
      // update and its store's read of the staging tile
      if (!writer) mbar_arrive(bar + kEmpty + st);
    }

    if (writer) tma_store_wait_all();
    // the state after the last chunk (columns 16e .. 16e + 15): the
    // caller's last_state, or a piece's end state for the next piece
    if (nc > 0) {
      sy.wait(kDoneH, (nc - 1) & 1);
      tc_fence_after();
    }
    // (the work item is decoded again: nothing of it stays live in the loop)
    const Work we = Work::of(*reinterpret_cast<volatile int *>(sm + oItem), p, nchunks);
    float *lr = we.out >= 0 ? p.mid + static_cast<int64_t>(we.out) * P * NS
                            : (p.last ? p.last + we.bh * P * NS : nullptr);
    if (lr) {
      uint32_t v[16];
      tmem_ld16(tl + kColH + 16 * e, v);
      tmem_wait_ld(v);
#pragma unroll
      for (int j = 0; j < 16; ++j) lr[(e * 16 + j) * NS + r] = __uint_as_float(v[j]);
    }
    if (we.out >= 0) {
      // every epilogue thread's stores are visible before the flag is set
      // (published after a timeout too, so the next piece never waits for
      // nothing)
      __threadfence();
      bar_sync(kEpiBarrier, kEpi);
      if (tid == 64) st_release_gpu(p.flag + we.out, 1u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor (d0 innermost, ..., d3), dense; box {64, 1, Q, 1}, 128-byte
// swizzle, rows past the end of the sequence read as zeros
bool encode_4d(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t d3) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(Q), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// y: (batch, seqlen, nheads, 64) fp32 or bf16; box {32, 1, Q, 1}, the
// swizzle matching the 128- (fp32) or 64-byte (bf16) rows of the box
bool encode_y(CUtensorMap *m, void *ptr, bool bf16, uint64_t H, uint64_t L, uint64_t Bt) {
  auto enc = encoder();
  if (!enc) return false;
  const uint64_t es = bf16 ? 2 : 4;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(P), H, L, Bt};
  cuuint64_t strides[3] = {P * es, P * H * es, P * H * L * es};
  cuuint32_t box[4] = {32, 1, static_cast<cuuint32_t>(Q), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ptr,
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool al16(const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; }
bool al4(const void *q) { return (reinterpret_cast<uintptr_t>(q) & 3) == 0; }

mss_status check(const mss_ssd_args *a) {
  if (!a) return MSS_ERR_INVALID_ARG;
  if (a->batch < 1 || a->seqlen < 1 || a->nheads < 1 || a->headdim < 1 || a->ngroups < 1 ||
      a->dstate < 1 || a->nheads % a->ngroups != 0)
    return MSS_ERR_INVALID_ARG;
  if ((a->in_dtype != MSS_F32 && a->in_dtype != MSS_BF16) ||
      (a->out_dtype != MSS_F32 && a->out_dtype != MSS_BF16))
    return MSS_ERR_INVALID_ARG;
  if (!a->x || !a->dt || !a->A || !a->B || !a->C || !a->y) return MSS_ERR_INVALID_ARG;
  if (a->in_dtype != MSS_BF16 || a->headdim != P || a->dstate != NS)
    return MSS_ERR_UNSUPPORTED;
  if (!al16(a->x) || !al16(a->B) || !al16(a->C) || !al16(a->y) || (a->z && !al16(a->z)))
    return MSS_ERR_INVALID_ARG;
  if (!al4(a->A) || (a->D && !al4(a->D)) || (a->dt_bias && !al4(a->dt_bias)) ||
      (a->h0 && !al4(a->h0)) || (a->last_state && !al4(a->last_state)) ||
      (reinterpret_cast<uintptr_t>(a->dt) & 1))
    return MSS_ERR_INVALID_ARG;
  // grid of batch * nheads CTAs; TMA coordinates are 32-bit
  if (a->batch * a->nheads >= (int64_t(1) << 31) - 65536 || a->seqlen >= (int64_t(1) << 31) - Q)
    return MSS_ERR_UNSUPPORTED;
  return MSS_OK;
}

// The cut schedule (one CTA per SM: a CTA's shared memory is above half an
// SM's).  With W full waves and r sequences left over (0 < 2 r <= SMs,
// W >= 1: the pieces need whole sequences to run between them), the r
// sequences are cut into min(round(SMs / r), W + 1, chunks, 8) >= 2
// pieces.  Workspace: the work-item counter at byte 0, the flags from byte
// 256, the end states after them; the first `clear` bytes are cleared per
// call.
struct Plan {
  int ncut = 0, parts = 0;
  int64_t gfull = 0;
  size_t clear = 0, bytes = 0;
};

mss_status plan_of(const mss_ssd_args *a, Plan *pl) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MSS_ERR_CUDA;
  *pl = Plan();
  if (sms < 1) return MSS_OK;
  const int64_t BH = a->batch * a->nheads;
  const int64_t nchunks = (a->seqlen + Q - 1) / Q;
  const int64_t W = BH / sms, r = BH % sms;
  if (W < 1 || r < 1 || 2 * r > sms || nchunks < 2) return MSS_OK;
  int64_t parts = (sms + r / 2) / r;  // round(SMs / r) >= 2
  parts = std::min<int64_t>(std::min<int64_t>(parts, W + 1), std::min<int64_t>(nchunks, 8));
  if (parts < 2) return MSS_OK;
  const size_t slots = static_cast<size_t>(r) * static_cast<size_t>(parts - 1);
  pl->ncut = static_cast<int>(r);
  pl->parts = static_cast<int>(parts);
  pl->gfull = (BH - r) / (parts - 1);
  pl->clear = 256 + ((4 * slots + 255) / 256) * 256;
  pl->bytes = pl->clear + slots * P * NS * sizeof(float);
  return MSS_OK;
}

}  // namespace ssd
}  // namespace sss48

using namespace sss48;

extern "C" mss_status mamba2_ssd_fwd(const mss_ssd_args *a, void *stream) {
  sss48::NvtxRange range("mamba2_ssd_fwd");
  const mss_status st = ssd::check(a);
  if (st != MSS_OK) return st;
  ssd::Maps maps;
  const uint64_t L = static_cast<uint64_t>(a->seqlen), H = static_cast<uint64_t>(a->nheads),
                 G = static_cast<uint64_t>(a->ngroups), Bt = static_cast<uint64_t>(a->batch);
  if (!ssd::encode_4d(&maps.x, a->x, ssd::P, H, L, Bt) ||
      !ssd::encode_4d(&maps.B, a->B, ssd::NS, G, L, Bt) ||
      !ssd::encode_4d(&maps.C, a->C, ssd::NS, G, L, Bt) ||
      !ssd::encode_y(&maps.y, a->y, a->out_dtype == MSS_BF16, H, L, Bt))
    return MSS_ERR_CUDA;
  ssd::Plan plan;
  const mss_status pst = ssd::plan_of(a, &plan);
  if (pst != MSS_OK) return pst;
  if (!a->workspace) plan = ssd::Plan();  // no workspace: every sequence whole
  if (plan.ncut && (a->workspace_bytes < plan.bytes)) return MSS_ERR_WORKSPACE;
  if (plan.ncut && !ssd::al16(a->workspace)) return MSS_ERR_INVALID_ARG;
  unsigned *status = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void **>(&status), ssd::g_ssd_status) !=
      cudaSuccess)
    return MSS_ERR_CUDA;
  ssd::Params p;
  p.batch = a->batch;
  p.L = a->seqlen;
  p.H = a->nheads;
  p.G = a->ngroups;
  p.dt = static_cast<const __nv_bfloat16 *>(a->dt);
  p.A = a->A;
  p.D = a->D;
  p.dt_bias = a->dt_bias;
  p.softplus = a->dt_softplus ? 1 : 0;
  p.z = static_cast<const __nv_bfloat16 *>(a->z);
  p.h0 = a->h0;
  p.y = a->y;
  p.y_bf16 = a->out_dtype == MSS_BF16;
  p.last = a->last_state;
  p.status = status;
  p.spin_ns = a->spin_timeout_ns ? a->spin_timeout_ns : 2000000000ull;
  unsigned char *ws = static_cast<unsigned char *>(a->workspace);
  p.ncut = plan.ncut;
  p.parts = plan.parts;
  p.gfull = plan.gfull;
  p.ticket = plan.ncut ? reinterpret_cast<unsigned *>(ws) : nullptr;
  p.flag = plan.ncut ? reinterpret_cast<unsigned *>(ws + 256) : nullptr;
  p.mid = plan.ncut ? reinterpret_cast<float *>(ws + plan.clear) : nullptr;
  // per launch: the attribute belongs to the current device
  if (cudaFuncSetAttribute(ssd::ssd_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           ssd::kSmemBytes) != cudaSuccess)
    return MSS_ERR_CUDA;
  if (plan.ncut &&
      cudaMemsetAsync(ws, 0, plan.clear, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSS_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(a->batch * a->nheads +
                                              static_cast<int64_t>(plan.parts - 1) * plan.ncut);
  ssd::ssd_fwd_kernel<<<grid, ssd::kThreads, ssd::kSmemBytes,
                        static_cast<cudaStream_t>(stream)>>>(maps, p);
  return cudaGetLastError() == cudaSuccess ? MSS_OK : MSS_ERR_CUDA;
}

extern "C" mss_status mss_ssd_workspace_size(const mss_ssd_args *a, size_t *bytes) {
  if (!a || !bytes || a->batch < 1 || a->seqlen < 1 || a->nheads < 1) return MSS_ERR_INVALID_ARG;
  ssd::Plan plan;
  const mss_status st = ssd::plan_of(a, &plan);
  if (st != MSS_OK) return st;
  *bytes = plan.bytes;
  return MSS_OK;
}

extern "C" mss_status mss_ssd_status(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSS_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, ssd::g_ssd_status, sizeof(v)) != cudaSuccess)
    return MSS_ERR_CUDA;
  const unsigned zero = 0;
  if (v && cudaMemcpyToSymbol(ssd::g_ssd_status, &zero, sizeof(zero)) != cudaSuccess)
    return MSS_ERR_CUDA;
  return v ? MSS_ERR_TIMEOUT : MSS_OK;
}
