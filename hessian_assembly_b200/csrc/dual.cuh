// dual.cuh -- forward-mode AD number type with a compile-time tangent width.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法, key design 1: forward mode rather than reverse
// mode, because every local term has few inputs; the primal, the directional
// derivatives and the local Jacobian/Hessian all stay in registers, so the
// only global traffic is reading the mesh and writing the final sparse
// derivatives.
//
// HyperDual<T, N> carries a value, its gradient with respect to N seeded
// inputs and the packed symmetric N x N Hessian (upper triangle, row-major),
// and propagates all three through every operation by the first- and
// second-order chain rules.  N is a template parameter, so every loop below
// unrolls and the whole number lives in registers.
#pragma once

#include <cuda_runtime.h>

namespace mad {

template <int N>
struct Tri {
  static constexpr int size = N * (N + 1) / 2;
  // packed index of (i, j), i <= j
  __host__ __device__ static constexpr int idx(int i, int j) {
    return i * N - (i * (i - 1)) / 2 + (j - i);
  }
};

template <typename T, int N>
struct HyperDual {
  T v;
  T g[N];
  T h[Tri<N>::size];
};

// ---- construction --------------------------------------------------------
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> hd_const(T c) {
  HyperDual<T, N> r;
  r.v = c;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = T(0);
#pragma unroll
  for (int i = 0; i < Tri<N>::size; ++i) r.h[i] = T(0);
  return r;
}

// input number k of N: tangent e_k, zero Hessian
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> hd_var(T val, int k) {
  HyperDual<T, N> r = hd_const<T, N>(val);
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = (i == k) ? T(1) : T(0);
  return r;
}

// ---- linear operations -----------------------------------------------------
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator+(const HyperDual<T, N>& a,
                                                              const HyperDual<T, N>& b) {
  HyperDual<T, N> r;
  r.v = a.v + b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] + b.g[i];
#pragma unroll
  for (int i = 0; i < Tri<N>::size; ++i) r.h[i] = a.h[i] + b.h[i];
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator-(const HyperDual<T, N>& a,
                                                              const HyperDual<T, N>& b) {
  HyperDual<T, N> r;
  r.v = a.v - b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] - b.g[i];
#pragma unroll
  for (int i = 0; i < Tri<N>::size; ++i) r.h[i] = a.h[i] - b.h[i];
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator-(const HyperDual<T, N>& a) {
  HyperDual<T, N> r;
  r.v = -a.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = -a.g[i];
#pragma unroll
  for (int i = 0; i < Tri<N>::size; ++i) r.h[i] = -a.h[i];
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator+(const HyperDual<T, N>& a, T c) {
  HyperDual<T, N> r = a;
  r.v = a.v + c;
  return r;
}
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator+(T c, const HyperDual<T, N>& a) {
  return a + c;
}
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator-(const HyperDual<T, N>& a, T c) {
  HyperDual<T, N> r = a;
  r.v = a.v - c;
  return r;
}
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator-(T c, const HyperDual<T, N>& a) {
  HyperDual<T, N> r = -a;
  r.v = c - a.v;
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator*(const HyperDual<T, N>& a, T c) {
  HyperDual<T, N> r;
  r.v = a.v * c;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] * c;
#pragma unroll
  for (int i = 0; i < Tri<N>::size; ++i) r.h[i] = a.h[i] * c;
  return r;
}
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator*(T c, const HyperDual<T, N>& a) {
  return a * c;
}

// ---- products --------------------------------------------------------------
// (ab)'' = a b'' + b a'' + a' b'^T + b' a'^T
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator*(const HyperDual<T, N>& a,
                                                              const HyperDual<T, N>& b) {
  HyperDual<T, N> r;
  r.v = a.v * b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.v * b.g[i] + b.v * a.g[i];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) {
      const int q = Tri<N>::idx(i, j);
      r.h[q] = a.v * b.h[q] + b.v * a.h[q] + a.g[i] * b.g[j] + a.g[j] * b.g[i];
    }
  return r;
}

// a^2, cheaper than a * a
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> sq(const HyperDual<T, N>& a) {
  HyperDual<T, N> r;
  r.v = a.v * a.v;
  const T two_v = T(2) * a.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = two_v * a.g[i];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) {
      const int q = Tri<N>::idx(i, j);
      r.h[q] = two_v * a.h[q] + T(2) * a.g[i] * a.g[j];
    }
  return r;
}

// f(a) for a scalar function with value f0 and derivatives f1, f2 at a.v:
// f(a)' = f1 a',  f(a)'' = f1 a'' + f2 a' a'^T
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> chain(const HyperDual<T, N>& a, T f0, T f1,
                                                          T f2) {
  HyperDual<T, N> r;
  r.v = f0;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = f1 * a.g[i];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) {
      const int q = Tri<N>::idx(i, j);
      r.h[q] = f1 * a.h[q] + f2 * a.g[i] * a.g[j];
    }
  return r;
}

// ---- elementary functions (IEEE sqrt and division) -------------------------
__host__ __device__ __forceinline__ float sq(float a) { return a * a; }
__host__ __device__ __forceinline__ double sq(double a) { return a * a; }
__host__ __device__ __forceinline__ float inv(float a) { return 1.0f / a; }
__host__ __device__ __forceinline__ double inv(double a) { return 1.0 / a; }
__host__ __device__ __forceinline__ float sqrt(float a) { return ::sqrtf(a); }
__host__ __device__ __forceinline__ double sqrt(double a) { return ::sqrt(a); }
// 1/sqrt(a) from the CUDA math library (a few ulp, not correctly rounded)
__device__ __forceinline__ float rsqrt(float a) { return ::rsqrtf(a); }
__device__ __forceinline__ double rsqrt(double a) { return ::rsqrt(a); }

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> sqrt(const HyperDual<T, N>& a) {
  const T f0 = ::sqrt(a.v);
  const T r0 = T(1) / f0;
  const T f1 = T(0.5) * r0;            // d sqrt = 1 / (2 sqrt v)
  const T f2 = T(-0.25) * r0 * r0 * r0;  // d2 sqrt = -1 / (4 v^{3/2})
  return chain(a, f0, f1, f2);
}

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> inv(const HyperDual<T, N>& a) {
  const T f0 = T(1) / a.v;
  const T f1 = -f0 * f0;
  const T f2 = T(-2) * f1 * f0;  // 2 / v^3
  return chain(a, f0, f1, f2);
}

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator/(const HyperDual<T, N>& a,
                                                              const HyperDual<T, N>& b) {
  return a * inv(b);
}

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> sin(const HyperDual<T, N>& a) {
  const T s = ::sin(a.v), c = ::cos(a.v);
  return chain(a, s, c, -s);
}

template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> cos(const HyperDual<T, N>& a) {
  const T s = ::sin(a.v), c = ::cos(a.v);
  return chain(a, c, -s, -c);
}

// ---- affine quantities ------------------------------------------------------
// A value that is affine in the seeded inputs (the inputs themselves, their
// differences, constant linear maps of them) has an identically zero
// Hessian.  Lin<T, N> carries only value and gradient, so no arithmetic is
// spent on those zeros; products and squares of Lin values produce the first
// non-zero Hessians.  This is exact (no approximation): it only drops terms
// that are zero by construction.
template <typename T, int N>
struct Lin {
  T v;
  T g[N];
};

template <typename T, int N>
__host__ __device__ __forceinline__ Lin<T, N> lin_var(T val, int k) {
  Lin<T, N> r;
  r.v = val;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = (i == k) ? T(1) : T(0);
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ Lin<T, N> operator+(const Lin<T, N>& a, const Lin<T, N>& b) {
  Lin<T, N> r;
  r.v = a.v + b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] + b.g[i];
  return r;
}
template <typename T, int N>
__host__ __device__ __forceinline__ Lin<T, N> operator-(const Lin<T, N>& a, const Lin<T, N>& b) {
  Lin<T, N> r;
  r.v = a.v - b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] - b.g[i];
  return r;
}
template <typename T, int N>
__host__ __device__ __forceinline__ Lin<T, N> operator*(const Lin<T, N>& a, T c) {
  Lin<T, N> r;
  r.v = a.v * c;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] * c;
  return r;
}

// promotion
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> to_hd(const Lin<T, N>& a) {
  HyperDual<T, N> r;
  r.v = a.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i];
#pragma unroll
  for (int i = 0; i < Tri<N>::size; ++i) r.h[i] = T(0);
  return r;
}

// a^2 of an affine value: Hessian 2 a' a'^T
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> sq(const Lin<T, N>& a) {
  HyperDual<T, N> r;
  r.v = a.v * a.v;
  const T two_v = T(2) * a.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = two_v * a.g[i];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) r.h[Tri<N>::idx(i, j)] = T(2) * (a.g[i] * a.g[j]);
  return r;
}

// product of two affine values: Hessian a' b'^T + b' a'^T
template <typename T, int N>
__host__ __device__ __forceinline__ HyperDual<T, N> operator*(const Lin<T, N>& a, const Lin<T, N>& b) {
  HyperDual<T, N> r;
  r.v = a.v * b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.v * b.g[i] + b.v * a.g[i];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) r.h[Tri<N>::idx(i, j)] = a.g[i] * b.g[j] + a.g[j] * b.g[i];
  return r;
}

// Hessian entry (i, j) of a packed HyperDual, any order of i and j
template <typename T, int N>
__host__ __device__ __forceinline__ T hess(const HyperDual<T, N>& a, int i, int j) {
  return i <= j ? a.h[Tri<N>::idx(i, j)] : a.h[Tri<N>::idx(j, i)];
}

}  // namespace mad
