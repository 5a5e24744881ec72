// Test kernel: evaluates the library's device exponentials on an array so a
// GPU test can compare them with float64 references.  Built by the test.
#include "device_math.cuh"

__global__ void eval(const float *x, float *poly, float *mufu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = sss48::exp2_poly2(make_float2(x[i], x[i + 1]));
    poly[i] = r.x;
    poly[i + 1] = r.y;
    mufu[i] = sss48::ex2_mufu(x[i]);
    mufu[i + 1] = sss48::ex2_mufu(x[i + 1]);
  }
}

extern "C" int eval_exp2(const float *x, float *poly, float *mufu, int n) {
  eval<<<(n / 2 + 255) / 256, 256>>>(x, poly, mufu, n);
  return (int)cudaGetLastError();
}

// softplus (paired and scalar) and silu (paired and scalar) of every
// element.
__global__ void eval_act(const float *x, float *sp_pair, float *sp_scalar,
                         float *si_pair, float *si_scalar, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 v = make_float2(x[i], x[i + 1]);
    const float2 a = sss48::softplus2_f(v);
    const float2 s = sss48::silu2_f(v);
    sp_pair[i] = a.x;
    sp_pair[i + 1] = a.y;
    sp_scalar[i] = sss48::softplus_f(v.x);
    sp_scalar[i + 1] = sss48::softplus_f(v.y);
    si_pair[i] = s.x;
    si_pair[i + 1] = s.y;
    si_scalar[i] = sss48::silu_f(v.x);
    si_scalar[i + 1] = sss48::silu_f(v.y);
  }
}

extern "C" int eval_activations(const float *x, float *sp_pair, float *sp_scalar,
                                float *si_pair, float *si_scalar, int n) {
  eval_act<<<(n / 2 + 255) / 256, 256>>>(x, sp_pair, sp_scalar, si_pair, si_scalar, n);
  return (int)cudaGetLastError();
}
