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
