// sparse_ad.cuh -- forward-mode AD numbers whose sparsity is known at compile
// time.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法, key design 1: a local term is differentiated in
// forward mode with its tangents in registers.  When the seeded inputs are
// single variables (a one-hot tangent) or differences of two of them, most of
// the gradient entries of the first intermediates and most of their Hessian
// entries are zero by construction.  A multiplication by such a zero cannot
// be removed by the compiler under IEEE semantics (x * 0 is NaN for x = inf
// and -0 for negative x), so the dense HyperDual spends instructions on them.
//
// SLin<T, N, G> and SHD<T, N, G, H> carry the same value, gradient and packed
// Hessian as Lin and HyperDual, plus two masks as template arguments: bit i
// of G set when gradient entry i may be non-zero, bit Tri<N>::idx(i, j) of H
// when Hessian entry (i, j) may be.  Each operation computes the masks of its
// result from those of its operands (union for sums, the outer product of the
// gradient masks for products and chain steps) and evaluates only the
// entries that are set; an entry outside the mask is exactly zero and is
// never read.  The derivatives are identical to the dense types': only terms
// that are zero by construction are dropped, and the order of the remaining
// additions is the same.
#pragma once

#include <stdint.h>

#include "dual.cuh"

namespace mad {

__host__ __device__ constexpr bool mbit(uint64_t m, int i) { return ((m >> i) & 1u) != 0; }

// Hessian mask of u' v'^T + v' u'^T for gradient masks a and b
template <int N>
__host__ __device__ constexpr uint64_t outer_mask(uint32_t a, uint32_t b) {
  uint64_t m = 0;
  for (int i = 0; i < N; ++i)
    for (int j = i; j < N; ++j)
      if ((mbit(a, i) && mbit(b, j)) || (mbit(a, j) && mbit(b, i)))
        m |= uint64_t(1) << Tri<N>::idx(i, j);
  return m;
}

template <typename T, int N, uint32_t G>
struct SLin {
  T v;
  T g[N];
};

template <typename T, int N, uint32_t G, uint64_t H>
struct SHD {
  static_assert(Tri<N>::size <= 64, "packed Hessian mask holds at most 64 entries");
  T v;
  T g[N];
  T h[Tri<N>::size];
};

// input number K of N: tangent e_K
template <typename T, int N, int K>
__device__ __forceinline__ SLin<T, N, (1u << K)> slin_var(T val) {
  SLin<T, N, (1u << K)> r;
  r.v = val;
  r.g[K] = T(1);
  return r;
}

template <typename T, int N, uint32_t A, uint32_t B>
__device__ __forceinline__ SLin<T, N, (A | B)> operator-(const SLin<T, N, A>& a,
                                                         const SLin<T, N, B>& b) {
  SLin<T, N, (A | B)> r;
  r.v = a.v - b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    if (mbit(A, i) && mbit(B, i)) r.g[i] = a.g[i] - b.g[i];
    else if (mbit(A, i)) r.g[i] = a.g[i];
    else if (mbit(B, i)) r.g[i] = -b.g[i];
  }
  return r;
}

// (ab)'' = a' b'^T + b' a'^T for affine a, b
template <typename T, int N, uint32_t A, uint32_t B>
__device__ __forceinline__ SHD<T, N, (A | B), outer_mask<N>(A, B)> operator*(
    const SLin<T, N, A>& a, const SLin<T, N, B>& b) {
  SHD<T, N, (A | B), outer_mask<N>(A, B)> r;
  r.v = a.v * b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    if (mbit(A, i) && mbit(B, i)) r.g[i] = a.v * b.g[i] + b.v * a.g[i];
    else if (mbit(B, i)) r.g[i] = a.v * b.g[i];
    else if (mbit(A, i)) r.g[i] = b.v * a.g[i];
  }
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) {
      const bool t1 = mbit(A, i) && mbit(B, j), t2 = mbit(A, j) && mbit(B, i);
      const int q = Tri<N>::idx(i, j);
      if (t1 && t2) r.h[q] = a.g[i] * b.g[j] + a.g[j] * b.g[i];
      else if (t1) r.h[q] = a.g[i] * b.g[j];
      else if (t2) r.h[q] = a.g[j] * b.g[i];
    }
  return r;
}

// a^2 of an affine value: Hessian 2 a' a'^T
template <typename T, int N, uint32_t A>
__device__ __forceinline__ SHD<T, N, A, outer_mask<N>(A, A)> sq(const SLin<T, N, A>& a) {
  SHD<T, N, A, outer_mask<N>(A, A)> r;
  r.v = a.v * a.v;
  const T two_v = T(2) * a.v;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (mbit(A, i)) r.g[i] = two_v * a.g[i];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j)
      if (mbit(A, i) && mbit(A, j)) r.h[Tri<N>::idx(i, j)] = T(2) * (a.g[i] * a.g[j]);
  return r;
}

template <typename T, int N, uint32_t GA, uint64_t HA, uint32_t GB, uint64_t HB>
__device__ __forceinline__ SHD<T, N, (GA | GB), (HA | HB)> operator+(const SHD<T, N, GA, HA>& a,
                                                                     const SHD<T, N, GB, HB>& b) {
  SHD<T, N, (GA | GB), (HA | HB)> r;
  r.v = a.v + b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    if (mbit(GA, i) && mbit(GB, i)) r.g[i] = a.g[i] + b.g[i];
    else if (mbit(GA, i)) r.g[i] = a.g[i];
    else if (mbit(GB, i)) r.g[i] = b.g[i];
  }
#pragma unroll
  for (int q = 0; q < Tri<N>::size; ++q) {
    if (mbit(HA, q) && mbit(HB, q)) r.h[q] = a.h[q] + b.h[q];
    else if (mbit(HA, q)) r.h[q] = a.h[q];
    else if (mbit(HB, q)) r.h[q] = b.h[q];
  }
  return r;
}

template <typename T, int N, uint32_t GA, uint64_t HA, uint32_t GB, uint64_t HB>
__device__ __forceinline__ SHD<T, N, (GA | GB), (HA | HB)> operator-(const SHD<T, N, GA, HA>& a,
                                                                     const SHD<T, N, GB, HB>& b) {
  SHD<T, N, (GA | GB), (HA | HB)> r;
  r.v = a.v - b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    if (mbit(GA, i) && mbit(GB, i)) r.g[i] = a.g[i] - b.g[i];
    else if (mbit(GA, i)) r.g[i] = a.g[i];
    else if (mbit(GB, i)) r.g[i] = -b.g[i];
  }
#pragma unroll
  for (int q = 0; q < Tri<N>::size; ++q) {
    if (mbit(HA, q) && mbit(HB, q)) r.h[q] = a.h[q] - b.h[q];
    else if (mbit(HA, q)) r.h[q] = a.h[q];
    else if (mbit(HB, q)) r.h[q] = -b.h[q];
  }
  return r;
}

// (ab)'' = a b'' + b a'' + a' b'^T + b' a'^T
template <typename T, int N, uint32_t GA, uint64_t HA, uint32_t GB, uint64_t HB>
__device__ __forceinline__ SHD<T, N, (GA | GB), (HA | HB | outer_mask<N>(GA, GB))> operator*(
    const SHD<T, N, GA, HA>& a, const SHD<T, N, GB, HB>& b) {
  SHD<T, N, (GA | GB), (HA | HB | outer_mask<N>(GA, GB))> r;
  r.v = a.v * b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    if (mbit(GA, i) && mbit(GB, i)) r.g[i] = a.v * b.g[i] + b.v * a.g[i];
    else if (mbit(GB, i)) r.g[i] = a.v * b.g[i];
    else if (mbit(GA, i)) r.g[i] = b.v * a.g[i];
  }
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) {
      const int q = Tri<N>::idx(i, j);
      // the four terms in the dense product's order, each only where it can be non-zero
      const bool t0 = mbit(HB, q), t1 = mbit(HA, q);
      const bool t2 = mbit(GA, i) && mbit(GB, j), t3 = mbit(GA, j) && mbit(GB, i);
      T acc = T(-0.0);
      if (t0) acc = a.v * b.h[q];
      if (t1) acc = t0 ? acc + b.v * a.h[q] : b.v * a.h[q];
      if (t2) acc = (t0 || t1) ? acc + a.g[i] * b.g[j] : a.g[i] * b.g[j];
      if (t3) acc = (t0 || t1 || t2) ? acc + a.g[j] * b.g[i] : a.g[j] * b.g[i];
      if (t0 || t1 || t2 || t3) r.h[q] = acc;
    }
  return r;
}

// a^2: (a^2)'' = 2 a a'' + 2 a' a'^T
template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ SHD<T, N, G, (H | outer_mask<N>(G, G))> sq(const SHD<T, N, G, H>& a) {
  SHD<T, N, G, (H | outer_mask<N>(G, G))> r;
  r.v = a.v * a.v;
  const T two_v = T(2) * a.v;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (mbit(G, i)) r.g[i] = two_v * a.g[i];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) {
      const int q = Tri<N>::idx(i, j);
      const bool hh = mbit(H, q), gg = mbit(G, i) && mbit(G, j);
      if (hh && gg) r.h[q] = two_v * a.h[q] + T(2) * a.g[i] * a.g[j];
      else if (hh) r.h[q] = two_v * a.h[q];
      else if (gg) r.h[q] = T(2) * a.g[i] * a.g[j];
    }
  return r;
}

// f(a) with f0, f1, f2 the value and first two derivatives of f at a.v:
// f(a)' = f1 a',  f(a)'' = f1 a'' + f2 a' a'^T
template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ SHD<T, N, G, (H | outer_mask<N>(G, G))> chain(
    const SHD<T, N, G, H>& a, T f0, T f1, T f2) {
  SHD<T, N, G, (H | outer_mask<N>(G, G))> r;
  r.v = f0;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (mbit(G, i)) r.g[i] = f1 * a.g[i];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = i; j < N; ++j) {
      const int q = Tri<N>::idx(i, j);
      const bool hh = mbit(H, q), gg = mbit(G, i) && mbit(G, j);
      if (hh && gg) r.h[q] = f1 * a.h[q] + f2 * a.g[i] * a.g[j];
      else if (hh) r.h[q] = f1 * a.h[q];
      else if (gg) r.h[q] = f2 * a.g[i] * a.g[j];
    }
  return r;
}

// ---- elementary functions and scalar operations ----------------------------
// sqrt and 1/x as chain-rule steps with their own first and second
// derivatives, as for the dense numbers (dual.cuh); -a and a + c, a - c.
template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ auto sqrt(const SHD<T, N, G, H>& a) {
  const T f0 = ::sqrt(a.v);
  const T r0 = T(1) / f0;
  return chain(a, f0, T(0.5) * r0, T(-0.25) * r0 * r0 * r0);
}

template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ auto inv(const SHD<T, N, G, H>& a) {
  const T f0 = T(1) / a.v;
  const T f1 = -f0 * f0;
  return chain(a, f0, f1, T(-2) * f1 * f0);
}

template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ SHD<T, N, G, H> operator-(const SHD<T, N, G, H>& a) {
  SHD<T, N, G, H> r;
  r.v = -a.v;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (mbit(G, i)) r.g[i] = -a.g[i];
#pragma unroll
  for (int q = 0; q < Tri<N>::size; ++q)
    if (mbit(H, q)) r.h[q] = -a.h[q];
  return r;
}

template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ SHD<T, N, G, H> operator+(const SHD<T, N, G, H>& a, T c) {
  SHD<T, N, G, H> r = a;
  r.v = a.v + c;
  return r;
}

template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ SHD<T, N, G, H> operator-(const SHD<T, N, G, H>& a, T c) {
  SHD<T, N, G, H> r = a;
  r.v = a.v - c;
  return r;
}

template <typename T, int N, uint32_t G>
__device__ __forceinline__ SLin<T, N, G> operator-(const SLin<T, N, G>& a) {
  SLin<T, N, G> r;
  r.v = -a.v;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (mbit(G, i)) r.g[i] = -a.g[i];
  return r;
}

// an affine value as a number with a (structurally zero) Hessian
template <typename T, int N, uint32_t G>
__device__ __forceinline__ SHD<T, N, G, 0> to_shd(const SLin<T, N, G>& a) {
  SHD<T, N, G, 0> r;
  r.v = a.v;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (mbit(G, i)) r.g[i] = a.g[i];
  return r;
}

template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ SHD<T, N, G, H> operator*(const SHD<T, N, G, H>& a, T c) {
  SHD<T, N, G, H> r;
  r.v = a.v * c;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (mbit(G, i)) r.g[i] = a.g[i] * c;
#pragma unroll
  for (int q = 0; q < Tri<N>::size; ++q)
    if (mbit(H, q)) r.h[q] = a.h[q] * c;
  return r;
}

// |u|^2 of D = 2 or 3 seeded inputs u[a] (input a of D)
template <typename T, int D>
__device__ __forceinline__ auto sqnorm_m(const T* u) {
  static_assert(D == 2 || D == 3, "dof 2 or 3");
  const auto s = sq(slin_var<T, D, 0>(u[0])) + sq(slin_var<T, D, 1>(u[1]));
  if constexpr (D == 3) return s + sq(slin_var<T, D, 2>(u[2]));
  else return s;
}

// |xa - xb|^2 with xa[a] seeded as input a and xb[a] as input D + a of 2D
template <typename T, int D>
__device__ __forceinline__ auto sqdist_m(const T* xa, const T* xb) {
  static_assert(D == 2 || D == 3, "dof 2 or 3");
  constexpr int N = 2 * D;
  const auto s = sq(slin_var<T, N, 0>(xa[0]) - slin_var<T, N, D>(xb[0])) +
                 sq(slin_var<T, N, 1>(xa[1]) - slin_var<T, N, D + 1>(xb[1]));
  if constexpr (D == 3) return s + sq(slin_var<T, N, 2>(xa[2]) - slin_var<T, N, 5>(xb[2]));
  else return s;
}

// Gradient entry i and Hessian entry (i, j), any order.  An entry outside
// the mask reads as -0, the exact additive identity (x + -0 = x for every
// x, +0 and -0 included), so a sum that takes it costs no instruction.
template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ T sgrad(const SHD<T, N, G, H>& a, int i) {
  return mbit(G, i) ? a.g[i] : T(-0.0);
}
template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ T shess(const SHD<T, N, G, H>& a, int i, int j) {
  const int q = i <= j ? Tri<N>::idx(i, j) : Tri<N>::idx(j, i);
  return mbit(H, q) ? a.h[q] : T(-0.0);
}

}  // namespace mad
