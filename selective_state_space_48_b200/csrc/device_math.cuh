// device_math.cuh -- small device helpers of the selective-scan kernels.
//
// Only the arithmetic the scan needs: the base-2 exponential used for the
// decay exp(Delta*A), the softplus step size and the silu gate.  The decay
// uses the MUFU ex2 unit; fp32 accuracy of the scan is checked by the parity
// tests against the fp64 oracle.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace sss48 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// 2^x on the special-function unit (flushes subnormal results to zero).
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(x) = log(1 + e^x).  Above 15 it equals x to fp32 precision.
__device__ __forceinline__ float softplus_f(float x) {
  return x > 15.0f ? x : log1pf(__expf(x));
}

// silu(z) = z / (1 + e^-z); e^-z overflowing to inf gives -0, as it should.
__device__ __forceinline__ float silu_f(float z) {
  return __fdividef(z, 1.0f + __expf(-z));
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

}  // namespace sss48
