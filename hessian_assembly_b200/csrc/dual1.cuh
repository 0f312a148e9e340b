// dual1.cuh -- first-order forward-mode AD number: a value and its gradient
// with respect to N seeded inputs.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法: for a vector-valued objective each local term
// yields its local Jacobian J_j, which forward mode delivers for all N stencil
// inputs in one pass when every residual component carries an N-wide tangent
// (key design 1: the number lives in registers).  This is HyperDual without
// the Hessian part; every operation applies the first-order chain rule.
#pragma once

#include <cuda_runtime.h>

namespace mad {

template <typename T, int N>
struct Dual {
  T v;
  T g[N];
};

template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> d_const(T c) {
  Dual<T, N> r;
  r.v = c;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = T(0);
  return r;
}

// input number k of N: tangent e_k
template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> d_var(T val, int k) {
  Dual<T, N> r;
  r.v = val;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = (i == k) ? T(1) : T(0);
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> operator+(const Dual<T, N>& a, const Dual<T, N>& b) {
  Dual<T, N> r;
  r.v = a.v + b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] + b.g[i];
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> operator-(const Dual<T, N>& a, const Dual<T, N>& b) {
  Dual<T, N> r;
  r.v = a.v - b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] - b.g[i];
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> operator-(const Dual<T, N>& a) {
  Dual<T, N> r;
  r.v = -a.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = -a.g[i];
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> operator*(const Dual<T, N>& a, T s) {
  Dual<T, N> r;
  r.v = a.v * s;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] * s;
  return r;
}

// (ab)' = a' b + a b'
template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> operator*(const Dual<T, N>& a, const Dual<T, N>& b) {
  Dual<T, N> r;
  r.v = a.v * b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = a.g[i] * b.v + a.v * b.g[i];
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> operator-(const Dual<T, N>& a, T s) {
  Dual<T, N> r = a;
  r.v -= s;
  return r;
}

// f(a) with value f0 and derivative f1 at a.v: f(a)' = f1 a'
template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> chain1(const Dual<T, N>& a, T f0, T f1) {
  Dual<T, N> r;
  r.v = f0;
#pragma unroll
  for (int i = 0; i < N; ++i) r.g[i] = f1 * a.g[i];
  return r;
}

template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> sqrt(const Dual<T, N>& a) {
  const T s = ::sqrt(a.v);
  return chain1(a, s, T(0.5) / s);  // d sqrt = 1 / (2 sqrt v)
}

template <typename T, int N>
__host__ __device__ __forceinline__ Dual<T, N> inv(const Dual<T, N>& a) {
  const T f0 = T(1) / a.v;
  return chain1(a, f0, -f0 * f0);  // d (1/v) = -1 / v^2
}

}  // namespace mad
