// selftest.cu -- device self-test of the HyperDual number type.
//
// f1 = a sin a and f2 = a sin b + b cos a are the worked examples of the page
// "How to Implement Automatic Differentiation Using the $autodiff Block for
// Custom Kernels" (Code Examples section), which states their gradients in
// closed form; f3 = sqrt(a^2 + b^2) and f4 = a / b exercise sqrt and division.
// Output per input: 4 functions x (value, d/da, d/db, d2/da2, d2/dadb, d2/db2).
#include "dual.cuh"
#include "mad_internal.h"

namespace mad {
namespace {

__device__ void put(const HyperDual<double, 2>& f, double* o) {
  o[0] = f.v;
  o[1] = f.g[0];
  o[2] = f.g[1];
  o[3] = f.h[Tri<2>::idx(0, 0)];
  o[4] = f.h[Tri<2>::idx(0, 1)];
  o[5] = f.h[Tri<2>::idx(1, 1)];
}

__global__ void k_selftest(int n, const double* __restrict__ ab, double* __restrict__ out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const HyperDual<double, 2> a = hd_var<double, 2>(ab[2 * i], 0);
  const HyperDual<double, 2> b = hd_var<double, 2>(ab[2 * i + 1], 1);
  double* o = out + (size_t)i * 24;
  put(a * sin(a), o);
  put(a * sin(b) + b * cos(a), o + 6);
  put(sqrt(sq(a) + sq(b)), o + 12);
  put(a / b, o + 18);
}

}  // namespace

cudaError_t selftest_dual(int n, const double* ab_dev, double* out_dev) {
  if (n <= 0) return cudaSuccess;
  k_selftest<<<(n + 127) / 128, 128>>>(n, ab_dev, out_dev);
  return cudaGetLastError();
}

}  // namespace mad
