// exp2_poly_probe.cu -- test-only: evaluates the prefill kernel's FMA-pipe exponential
// (sm100::exp2_poly2) and the device's exp2f on the same inputs, so a test can compare
// both with the exact value of 2^x.  Built by tests/test_exp2_poly.py into a temporary
// directory; never part of the library.
#include <cuda_runtime.h>

#include "sm100.cuh"

__global__ void exp2_poly_probe_kernel(const float* x, float* y_poly, float* y_lib, int n_pairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pairs) return;
  const float2 v = make_float2(x[2 * i], x[2 * i + 1]);
  const float2 r = sm100::exp2_poly2(v);
  y_poly[2 * i] = r.x;
  y_poly[2 * i + 1] = r.y;
  y_lib[2 * i] = exp2f(v.x);
  y_lib[2 * i + 1] = exp2f(v.y);
}

// x, y_poly, y_lib: device arrays of 2 * n_pairs floats.  Returns the launch status.
extern "C" __attribute__((visibility("default"))) int exp2_poly_eval(const float* x, float* y_poly, float* y_lib,
                                                                      int n_pairs, void* stream) {
  if (n_pairs <= 0) return 0;
  const int threads = 256;
  exp2_poly_probe_kernel<<<(n_pairs + threads - 1) / threads, threads, 0, (cudaStream_t)stream>>>(x, y_poly, y_lib,
                                                                                                  n_pairs);
  return (int)cudaGetLastError();
}
