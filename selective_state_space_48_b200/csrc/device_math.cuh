// device_math.cuh -- device helpers of the selective-scan kernels: the
// special-function arithmetic of the step size, decay and gate, and the
// PTX wrappers for TMA loads, mbarriers and release/acquire flags.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#ifndef MSS_DEBUG
#define MSS_DEBUG 0
#endif

namespace sss48 {

// Device status bits (read by the status entry points): a bounded wait
// that ran out, and (checked builds only) an access outside its tensor.
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusBadIndex = 2u;

// Bounds check of a global access at element index i of a tensor with n
// elements.  In builds with MSS_DEBUG=1 an index outside [0, n) is
// recorded in *status (kStatusBadIndex) and false is returned, so the
// caller skips the access; no trap, no assert.  In ordinary builds it is
// always true and generates no code.
__device__ __forceinline__ bool dbg_index_ok(int64_t i, int64_t n, unsigned *status) {
#if MSS_DEBUG
  if (i >= 0 && i < n) return true;
  if (status) atomicOr(status, kStatusBadIndex);
  return false;
#else
  (void)i;
  (void)n;
  (void)status;
  return true;
#endif
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// 2^x on the special-function unit (subnormal results flush to zero).
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for two arguments at once on the FMA pipe, for x in [-126, 127]
// (clamped there).  x = j + f with j = round(x) and |f| <= 1/2: adding
// 1.5 * 2^23 leaves j in the low mantissa bits; 2^f comes from a degree-5
// polynomial with constant term exactly 1 (so 2^0 = 1 exactly) whose other
// coefficients were fitted for this library, minimax in relative error on
// [-1/2, 1/2]: 9.1e-8 in exact arithmetic, 1.7e-7 after fp32 rounding; 2^j
// is applied by adding j to the exponent field.  Used beside ex2.approx to
// move part of the exponentials off the special-function unit.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  x.x = fminf(fmaxf(x.x, -126.0f), 127.0f);
  x.y = fminf(fmaxf(x.y, -126.0f), 127.0f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
  const float2 j = __fadd2_rn(t, make_float2(-kRound, -kRound));
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);
  float2 q = __ffma2_rn(f, make_float2(1.326472731e-03f, 1.326472731e-03f),
                        make_float2(9.671512991e-03f, 9.671512991e-03f));
  q = __ffma2_rn(q, f, make_float2(5.550733581e-02f, 5.550733581e-02f));
  q = __ffma2_rn(q, f, make_float2(2.402224243e-01f, 2.402224243e-01f));
  q = __ffma2_rn(q, f, make_float2(6.931470037e-01f, 6.931470037e-01f));
  q = __ffma2_rn(q, f, make_float2(1.0f, 1.0f));
  return make_float2(
      __int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
      __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// log1p(e) / e for e in [0, 1]: a degree-7 polynomial with constant term
// exactly 1 (so the ratio tends to 1 as e -> 0) whose other coefficients
// were fitted for this library, minimax in relative error on [0, 1]:
// 2.2e-7 in exact arithmetic, 3.7e-7 for e * P(e) after fp32 rounding.
__device__ __forceinline__ float log1p_ratio(float e) {
  float q = fmaf(-8.778954856e-03f, e, 4.498663917e-02f);
  q = fmaf(q, e, -1.090229079e-01f);
  q = fmaf(q, e, 1.784720868e-01f);
  q = fmaf(q, e, -2.453686595e-01f);
  q = fmaf(q, e, 3.328406513e-01f);
  q = fmaf(q, e, -4.999817908e-01f);
  return fmaf(q, e, 1.0f);
}
__device__ __forceinline__ float2 log1p_ratio2(float2 e) {
  auto c = [](float v) { return make_float2(v, v); };
  float2 q = __ffma2_rn(c(-8.778954856e-03f), e, c(4.498663917e-02f));
  q = __ffma2_rn(q, e, c(-1.090229079e-01f));
  q = __ffma2_rn(q, e, c(1.784720868e-01f));
  q = __ffma2_rn(q, e, c(-2.453686595e-01f));
  q = __ffma2_rn(q, e, c(3.328406513e-01f));
  q = __ffma2_rn(q, e, c(-4.999817908e-01f));
  return __ffma2_rn(q, e, c(1.0f));
}

// softplus(x) = log(1 + e^x) = max(x, 0) + log1p(e) with e = e^-|x| in
// (0, 1], and log1p(e) = e * (log1p(e) / e) from the polynomial above: one
// exponential, no logarithm and no branch.  Relative error a few 1e-7 for
// |x| up to ~20 (the rounding of -|x| log2(e) grows with |x|); +-inf and
// NaN give inf, 0 and NaN.
__device__ __forceinline__ float softplus_f(float x) {
  const float e = ex2_mufu(-fabsf(x) * kLog2e);
  return fmaf(e, log1p_ratio(e), fmaxf(x, 0.0f));
}

// silu(z) = z / (1 + e^-z); e^-z overflowing to inf gives -0, as it should.
__device__ __forceinline__ float silu_f(float z) {
  return __fdividef(z, 1.0f + ex2_mufu(-z * kLog2e));
}

// softplus of two values, same formula as softplus_f, the polynomial
// evaluated with paired f32x2 instructions.
__device__ __forceinline__ float2 softplus2_f(float2 x) {
  const float2 e = make_float2(ex2_mufu(-fabsf(x.x) * kLog2e), ex2_mufu(-fabsf(x.y) * kLog2e));
  return __ffma2_rn(e, log1p_ratio2(e), make_float2(fmaxf(x.x, 0.0f), fmaxf(x.y, 0.0f)));
}

// silu of two values with e^-z on the FMA pipe; the polynomial saturates at
// 2^127 for z < -88, where silu(z) is -0 to fp32 precision anyway.
__device__ __forceinline__ float2 silu2_f(float2 z) {
  const float2 e = exp2_poly2(__fmul2_rn(z, make_float2(-kLog2e, -kLog2e)));
  return make_float2(__fdividef(z.x, 1.0f + e.x), __fdividef(z.y, 1.0f + e.y));
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Two / four consecutive elements, widened to fp32 (p suitably aligned).
__device__ __forceinline__ float2 load2_f32(const float *p) {
  return *reinterpret_cast<const float2 *>(p);
}
__device__ __forceinline__ float2 load2_f32(const __nv_bfloat16 *p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ float4 load4_f32(const float *p) {
  return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ float4 load4_f32(const __nv_bfloat16 *p) {
  const uint2 v = *reinterpret_cast<const uint2 *>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void store4(float *p, float4 v) {
  *reinterpret_cast<float4 *>(p) = v;
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t *>(&a);
  w.y = *reinterpret_cast<uint32_t *>(&b);
  *reinterpret_cast<uint2 *>(p) = w;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned *p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---- named barriers between warp groups of one block

// Non-aligned forms: correct even if the warp is not converged here.
__device__ __forceinline__ void bar_sync(int id, int nthreads) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void bar_arrive(int id, int nthreads) {
  asm volatile("barrier.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- mbarrier + TMA (no clusters: every CTA is its own cluster of one)

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Plain arrival (release of this thread's earlier shared-memory writes).
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Like mbar_try_wait, but a thread whose phase is not complete yet is
// suspended (it issues nothing) until the phase completes or about
// `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of `bar` to complete, giving up after
// `limit_ns` nanoseconds (returns false then).  Waiting threads sleep in
// slices of up to 100 us instead of spinning, so they take no issue slots
// from the warps doing work.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
    if (global_timer_ns() - start > limit_ns) return false;
  }
}

// 3-D tiled TMA load of box {c0 (innermost), c1, c2} into shared memory,
// completing `bar`'s transaction count.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map,
                                            int c0, int c1, int c2,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2),
      "r"(smem_addr(bar))
      : "memory");
}

}  // namespace sss48
