// Test-only probe: evaluates the prefill softmax's exp2_poly2 (pa_fastmath.cuh)
// on a buffer of inputs so that a test can compare it with CUDA's exp2.
#include <cuda_runtime.h>

#include "pa_fastmath.cuh"

__global__ void exp2_poly_probe_kernel(const float* x, float* y, long n_pairs) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pairs) return;
  const uint64_t r = pa::exp2_poly2(pa::f2(x[2 * i], x[2 * i + 1]));
  float a, b;
  pa::f2_split(r, a, b);
  y[2 * i] = a;
  y[2 * i + 1] = b;
}

// x, y: device arrays of 2 * n_pairs floats.  Returns a cudaError_t value.
extern "C" int exp2_poly_probe(const float* x, float* y, long n_pairs) {
  if (n_pairs <= 0) return 0;
  const int threads = 256;
  const long blocks = (n_pairs + threads - 1) / threads;
  exp2_poly_probe_kernel<<<(unsigned)blocks, threads>>>(x, y, n_pairs);
  return (int)cudaGetLastError();
}
