// terms.cuh -- local energy terms, written once and evaluated on HyperDual
// numbers, and the evaluators that turn one term into its local gradient and
// Hessian blocks.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法: the user writes only local energy terms on
// vertices, edges, faces or runtime pairs; the framework evaluates,
// differentiates (forward mode, key design 1) and assembles them.  The
// energies below are those of the page's applications (section 实验结果):
// mass-spring cloth with inertia, runtime contact-style pairs, and the
// parameterization energy; the page names them but prints no formulas, so
// the standard forms are used:
//   spring / pair   1/2 k (|d| - L0)^2,  d = x_a - x_b
//   inertia         1/2 w |x - xt|^2
//   sym. Dirichlet  A (|J|_F^2 + |J^-1|_F^2) = A a (1 + 1/det(J)^2), a = |J|_F^2
//
// Two seeding strategies give the same derivatives (the AD forms of
// kAdReduced, kAdFull and kAdGeneric below):
//  * full: tangents on every stencil DOF (width 2*dof for an edge or pair
//    term, 3*dof for a face term); the energy is evaluated through the
//    stencil-to-variable map in HyperDual arithmetic;
//  * reduced (default): tangents on the term's natural variables (the edge
//    vector d, width dof; the Jacobian J, width 4) and the constant linear
//    map A from stencil DOFs to those variables is applied afterwards:
//    g_j = A^T grad, H_j = A^T Hess A.  For an edge term A = [I, -I], so the
//    four blocks are K, -K, -K, K.
#pragma once

#include <type_traits>

#include "../../include/mad.h"
#include "dual.cuh"
#include "sparse_ad.cuh"

namespace mad {

// ------------------------------------------------- forms of the local AD
// Template argument AD of the evaluators and kernels:
//  * kAdReduced: tangents on the term's natural variables; the spring,
//    symmetric Dirichlet and area energies use one univariate chain-rule step
//    with its derivatives written out (spring_of_s, symdir_scale, area_of_s);
//  * kAdFull: tangents on every stencil DOF (MAD_EVAL_FULL_STENCIL_AD);
//  * kAdGeneric: tangents as kAdReduced, and every energy written as a plain
//    expression of its inputs, differentiated by the number types' own
//    operations and elementary functions (sqrt, 1/x) alone
//    (MAD_EVAL_GENERIC_AD).
constexpr int kAdReduced = 0;
constexpr int kAdFull = 1;
constexpr int kAdGeneric = 2;
__host__ __device__ constexpr int ad_form(uint32_t flags) {
  return (flags & MAD_EVAL_FULL_STENCIL_AD) ? kAdFull
         : (flags & MAD_EVAL_GENERIC_AD)    ? kAdGeneric
                                            : kAdReduced;
}


// ---------------------------------------------------------------- energies
// S is the number type of the inputs (plain T, Lin or HyperDual); products
// of affine inputs become HyperDual, so the results are `auto`.
// Spring: E = k/2 (|d| - L0)^2 depends on d only through s = d.d, so it is
// evaluated as the univariate function f(s) = k/2 (sqrt(s) - L0)^2 of the AD
// number s, with f'(s) = k (l - L0) / (2 l) and f''(s) = k L0 / (4 l^3),
// l = sqrt(s): one chain-rule step instead of sqrt, square and product steps.
template <typename T>
__device__ __forceinline__ T spring_of_s(T s, T L0, T k) {
  const T r = sqrt(s) - L0;
  return (T(0.5) * k) * (r * r);
}
template <typename S, typename T>
__device__ __forceinline__ auto spring_chain(const S& s, T L0, T k) {
  const T il = rsqrt(s.v);
  const T l = s.v * il;
  const T r = l - L0;
  const T hk = T(0.5) * k;
  const T f1 = hk * r * il;
  const T f2 = (T(0.5) * hk) * L0 * (il * il * il);
  return chain(s, hk * (r * r), f1, f2);
}
template <typename T, int N>
__device__ __forceinline__ HyperDual<T, N> spring_of_s(const HyperDual<T, N>& s, T L0, T k) {
  return spring_chain(s, L0, k);
}
template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ auto spring_of_s(const SHD<T, N, G, H>& s, T L0, T k) {
  return spring_chain(s, L0, k);
}

template <typename S, int D, typename T>
__device__ __forceinline__ auto spring_energy(const S (&d)[D], T L0, T k) {
  auto s = sq(d[0]);
#pragma unroll
  for (int a = 1; a < D; ++a) s = s + sq(d[a]);
  return spring_of_s(s, L0, k);
}

// s(det) = A (1 + det^-2), the factor that multiplies ||J||_F^2 in the
// symmetric Dirichlet energy.  For HyperDual inputs it is one chain-rule step
// with s' = -2 A det^-3 and s'' = 6 A det^-4.
template <typename T>
__device__ __forceinline__ T symdir_scale(T det, T A) {
  const T r = inv(det);
  return A + A * (r * r);
}
template <typename S, typename T>
__device__ __forceinline__ auto symdir_scale_chain(const S& det, T A) {
  const T r = T(1) / det.v;
  const T Ar2 = A * (r * r);
  return chain(det, A + Ar2, T(-2) * Ar2 * r, T(6) * Ar2 * (r * r));
}
template <typename T, int N>
__device__ __forceinline__ HyperDual<T, N> symdir_scale(const HyperDual<T, N>& det, T A) {
  return symdir_scale_chain(det, A);
}
template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ auto symdir_scale(const SHD<T, N, G, H>& det, T A) {
  return symdir_scale_chain(det, A);
}

// j = (J00, J01, J10, J11): E = ||J||_F^2 (1 + det(J)^-2) A, which equals
// A (||J||_F^2 + ||J^-1||_F^2) for 2x2 J
template <typename S, typename T>
__device__ __forceinline__ auto symdir_energy(const S (&j)[4], T A) {
  auto a = sq(j[0]) + sq(j[1]) + sq(j[2]) + sq(j[3]);
  auto det = j[0] * j[3] - j[1] * j[2];
  return a * symdir_scale(det, A);
}

// As-rigid-as-possible parameterization energy, E = A |J - R(J)|_F^2 with
// R(J) the rotation closest to J.  That rotation maximises tr(R^T J), whose
// maximum over 2D rotations is s = sqrt((J00 + J11)^2 + (J10 - J01)^2), so
// E = A (|J|_F^2 - 2 s + 2); s > 0 whenever det J > 0 (s^2 = |J|^2 + 2 det J).
template <typename S, typename T>
__device__ __forceinline__ auto arap_energy(const S (&j)[4], T A) {
  auto a = sq(j[0]) + sq(j[1]) + sq(j[2]) + sq(j[3]);
  auto s = sq(j[0] + j[3]) + sq(j[2] - j[1]);
  return (a - sqrt(s) * T(2) + T(2)) * A;
}

// Symmetric Dirichlet on masked AD numbers (sparse_ad.cuh), where each
// component of vec J = (j0, j1, j2, j3) has its own type.
template <typename J0, typename J1, typename J2, typename J3, typename T>
__device__ __forceinline__ auto symdir_energy_m(const J0& j0, const J1& j1, const J2& j2,
                                                const J3& j3, T A) {
  const auto a = sq(j0) + sq(j1) + sq(j2) + sq(j3);
  const auto det = j0 * j3 - j1 * j2;
  return a * symdir_scale(det, A);
}

// The dof-2 face energies on the same inputs (J, rest area), summed as
// selected by kind: bit 0 symmetric Dirichlet, bit 1 ARAP.  kind is the same
// for every thread of a launch.
constexpr int kFaceSymDir = 1;
constexpr int kFaceArap = 2;
__host__ __device__ constexpr int face2_kind(uint32_t mask) {
  return ((mask & MAD_TERM_SYMDIR) ? kFaceSymDir : 0) | ((mask & MAD_TERM_ARAP) ? kFaceArap : 0);
}
template <int KIND, typename S, typename T>
__device__ __forceinline__ auto face2_energy(const S (&j)[4], T A) {
  static_assert(KIND >= 1 && KIND <= 3, "face energy selector");
  if constexpr (KIND == kFaceSymDir) return symdir_energy(j, A);
  else if constexpr (KIND == kFaceArap) return arap_energy(j, A);
  else return symdir_energy(j, A) + arap_energy(j, A);
}
// the same with the selector known only at run time (plain-value energies)
template <typename S, typename T>
__device__ __forceinline__ auto face2_energy(const S (&j)[4], T A, int kind) {
  decltype(symdir_energy(j, A)) e;
  if (kind == kFaceSymDir) e = face2_energy<kFaceSymDir>(j, A);
  else if (kind == kFaceArap) e = face2_energy<kFaceArap>(j, A);
  else e = face2_energy<kFaceSymDir | kFaceArap>(j, A);
  return e;
}
// calls f(std::integral_constant<int, KIND>) for a run-time selector, so that
// the face loop is compiled once per energy set
template <typename F>
__device__ __forceinline__ void with_face2_kind(int kind, F&& f) {
  if (kind == kFaceSymDir) f(std::integral_constant<int, kFaceSymDir>{});
  else if (kind == kFaceArap) f(std::integral_constant<int, kFaceArap>{});
  else f(std::integral_constant<int, kFaceSymDir | kFaceArap>{});
}

// Value, gradient and Hessian in J space of the dof-2 face energies selected
// by KIND at J = Jv, seeded on vec J.  Symmetric Dirichlet runs on the masked
// AD numbers (25.1 against 27.1 us per 500^2 eval); ARAP, alone or summed,
// on the dense ones, which measured faster for it (27.1 against 37.2 us).
template <int KIND, int AD, typename T>
__device__ __forceinline__ HyperDual<T, 4> face2_hd(const T (&Jv)[4], T A) {
  if constexpr (KIND == kFaceSymDir) {
    const auto j0 = slin_var<T, 4, 0>(Jv[0]);
    const auto j1 = slin_var<T, 4, 1>(Jv[1]);
    const auto j2 = slin_var<T, 4, 2>(Jv[2]);
    const auto j3 = slin_var<T, 4, 3>(Jv[3]);
    const auto m = [&] {
      if constexpr (AD == kAdGeneric) return symdir_energy_g(j0, j1, j2, j3, A);
      else return symdir_energy_m(j0, j1, j2, j3, A);
    }();
    HyperDual<T, 4> e;
    e.v = m.v;
#pragma unroll
    for (int p = 0; p < 4; ++p) e.g[p] = sgrad(m, p);
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int q = p; q < 4; ++q) e.h[Tri<4>::idx(p, q)] = shess(m, p, q);
    return e;
  } else {
    Lin<T, 4> j[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) j[p] = lin_var<T, 4>(Jv[p], p);
    return face2_energy<KIND>(j, A);
  }
}

// Area preservation of a 3D triangle: with n = e1 x e2 (e1 = x1 - x0,
// e2 = x2 - x0) and s = n.n, A = sqrt(s) / 2 and E = k/2 (A - A0)^2 / A0 is a
// univariate function of s: f'(s) = (k/A0)(A - A0) / (8A), f''(s) =
// k / (64 A^3) (from dA/ds = 1/(8A), d2A/ds2 = -1/(64 A^3)), applied as one
// chain step on the AD number s.
template <typename T>
__device__ __forceinline__ T area_of_s(T s, T A0, T k) {
  const T A = T(0.5) * sqrt(s);
  return (T(0.5) * k / A0) * (A - A0) * (A - A0);
}
template <typename S, typename T>
__device__ __forceinline__ auto area_chain(const S& s, T A0, T k) {
  const T A = T(0.5) * ::sqrt(s.v);
  const T iA = T(1) / A;
  const T f1 = (k / A0) * (A - A0) * (T(0.125) * iA);
  const T f2 = k * (T(1) / T(64)) * (iA * iA * iA);
  return chain(s, (T(0.5) * k / A0) * (A - A0) * (A - A0), f1, f2);
}
template <typename T, int N>
__device__ __forceinline__ HyperDual<T, N> area_of_s(const HyperDual<T, N>& s, T A0, T k) {
  return area_chain(s, A0, k);
}
template <typename T, int N, uint32_t G, uint64_t H>
__device__ __forceinline__ auto area_of_s(const SHD<T, N, G, H>& s, T A0, T k) {
  return area_chain(s, A0, k);
}

template <typename S, typename T>
__device__ __forceinline__ auto area_energy(const S (&e1)[3], const S (&e2)[3], T A0, T k) {
  auto n0 = e1[1] * e2[2] - e1[2] * e2[1];
  auto n1 = e1[2] * e2[0] - e1[0] * e2[2];
  auto n2 = e1[0] * e2[1] - e1[1] * e2[0];
  auto s = sq(n0) + sq(n1) + sq(n2);
  return area_of_s(s, A0, k);
}
// The same energy on masked AD numbers (sparse_ad.cuh), where each component
// of e1 and e2 has its own type.
template <typename A0_, typename A1_, typename A2_, typename B0_, typename B1_, typename B2_,
          typename T>
__device__ __forceinline__ auto area_energy_m(const A0_& a0, const A1_& a1, const A2_& a2,
                                              const B0_& b0, const B1_& b1, const B2_& b2, T A0,
                                              T k) {
  const auto n0 = a1 * b2 - a2 * b1;
  const auto n1 = a2 * b0 - a0 * b2;
  const auto n2 = a0 * b1 - a1 * b0;
  return area_of_s(sq(n0) + sq(n1) + sq(n2), A0, k);
}

// The energies as plain expressions (kAdGeneric), on masked AD numbers.
// spring / pair: k/2 (|d| - L0)^2
template <typename T, int D>
__device__ __forceinline__ auto spring_energy_g(const T* d, T L0, T k) {
  const auto l = sqrt(sqnorm_m<T, D>(d));
  return sq(l - L0) * (T(0.5) * k);
}
// symmetric Dirichlet: A (|J|_F^2 + |J^-1|_F^2) with J^-1 = adj(J) / det(J)
template <typename J0, typename J1, typename J2, typename J3, typename T>
__device__ __forceinline__ auto symdir_energy_g(const J0& j0, const J1& j1, const J2& j2,
                                                const J3& j3, T A) {
  const auto a = sq(j0) + sq(j1) + sq(j2) + sq(j3);
  const auto idet = inv(j0 * j3 - j1 * j2);
  const auto b = sq(to_shd(j3) * idet) + sq(to_shd(-j1) * idet) + sq(to_shd(-j2) * idet) +
                 sq(to_shd(j0) * idet);
  return (a + b) * A;
}
// area preservation: k/2 (A - A0)^2 / A0 with A = |e1 x e2| / 2
template <typename A0_, typename A1_, typename A2_, typename B0_, typename B1_, typename B2_,
          typename T>
__device__ __forceinline__ auto area_energy_g(const A0_& a0, const A1_& a1, const A2_& a2,
                                              const B0_& b0, const B1_& b1, const B2_& b2, T A0,
                                              T k) {
  const auto n0 = a1 * b2 - a2 * b1;
  const auto n1 = a2 * b0 - a0 * b2;
  const auto n2 = a0 * b1 - a1 * b0;
  const auto A = sqrt(sq(n0) + sq(n1) + sq(n2)) * T(0.5);
  return sq(A - A0) * (T(0.5) * k / A0);
}
// the area energy of a reduced-seeded row in either form
template <int AD, typename A0_, typename A1_, typename A2_, typename B0_, typename B1_,
          typename B2_, typename T>
__device__ __forceinline__ auto area_energy_ad(const A0_& a0, const A1_& a1, const A2_& a2,
                                               const B0_& b0, const B1_& b1, const B2_& b2, T A0,
                                               T k) {
  if constexpr (AD == kAdGeneric) return area_energy_g(a0, a1, a2, b0, b1, b2, A0, k);
  else return area_energy_m(a0, a1, a2, b0, b1, b2, A0, k);
}

// ---------------------------------------------------------------- results
// Edge / pair term: blocks are D x D row-major; the (b, a) block is the
// transpose of Hab.
template <typename T, int D>
struct EdgeDerivs {
  T E;
  T ga[D], gb[D];
  T Haa[D * D], Hab[D * D], Hbb[D * D];
};

// the spring energy of the edge vector d in the reduced or generic form
template <int AD, typename T, int D>
__device__ __forceinline__ auto spring_energy_ad(const T* d, T L0, T k) {
  if constexpr (AD == kAdGeneric) return spring_energy_g<T, D>(d, L0, k);
  else return spring_of_s(sqnorm_m<T, D>(d), L0, k);
}

template <typename T, int D, int AD>
__device__ __forceinline__ void eval_edge(const T* xa, const T* xb, T L0, T k,
                                          EdgeDerivs<T, D>& o) {
  if constexpr (AD != kAdFull) {
    T d[D];
#pragma unroll
    for (int a = 0; a < D; ++a) d[a] = xa[a] - xb[a];
    const auto e = spring_energy_ad<AD, T, D>(d, L0, k);
    o.E = e.v;
#pragma unroll
    for (int a = 0; a < D; ++a) {
      o.ga[a] = sgrad(e, a);
      o.gb[a] = -sgrad(e, a);
    }
#pragma unroll
    for (int a = 0; a < D; ++a)
#pragma unroll
      for (int b = 0; b < D; ++b) {
        const T K = shess(e, a, b);
        o.Haa[a * D + b] = K;
        o.Hbb[a * D + b] = K;
        o.Hab[a * D + b] = -K;
      }
  } else {
    const auto e = spring_of_s(sqdist_m<T, D>(xa, xb), L0, k);
    o.E = e.v;
#pragma unroll
    for (int a = 0; a < D; ++a) {
      o.ga[a] = sgrad(e, a);
      o.gb[a] = sgrad(e, D + a);
    }
#pragma unroll
    for (int a = 0; a < D; ++a)
#pragma unroll
      for (int b = 0; b < D; ++b) {
        o.Haa[a * D + b] = shess(e, a, b);
        o.Hab[a * D + b] = shess(e, a, D + b);
        o.Hbb[a * D + b] = shess(e, D + a, D + b);
      }
  }
}

// Compact per-term result kept in registers between the evaluation of all of
// a thread's edge terms and the colour phases that add them into the rows.
// Reduced seeding: K = d2E/dd2 (packed symmetric), g = dE/dd; the blocks are
// (a,a) = (b,b) = K, (a,b) = (b,a) = -K and g_a = g = -g_b.
template <typename T, int D, int AD>
struct EdgeRes {
  T K[Tri<D>::size];
  T g[D];
  T E;
};
template <typename T, int D>
struct EdgeRes<T, D, kAdFull> {
  EdgeDerivs<T, D> d;
};

template <typename T, int D, int AD>
__device__ __forceinline__ void eval_edge_res(const T* xa, const T* xb, T L0, T k,
                                              EdgeRes<T, D, AD>& R) {
  if constexpr (AD != kAdFull) {
    T d[D];
#pragma unroll
    for (int a = 0; a < D; ++a) d[a] = xa[a] - xb[a];
    const auto e = spring_energy_ad<AD, T, D>(d, L0, k);
    R.E = e.v;
#pragma unroll
    for (int a = 0; a < D; ++a) R.g[a] = sgrad(e, a);
#pragma unroll
    for (int a = 0; a < D; ++a)
#pragma unroll
      for (int b = a; b < D; ++b) R.K[Tri<D>::idx(a, b)] = shess(e, a, b);
  } else {
    eval_edge<T, D, kAdFull>(xa, xb, L0, k, R.d);
  }
}

// Add side `side` (0 = endpoint a, 1 = endpoint b) of an edge term into an
// owned row: the diagonal block goes to the row's packed symmetric
// accumulator `dacc`, the off-diagonal block to `off` (stored when the term
// is the block's only contributor, else added), the gradient to `gr`.
template <bool STORE, typename T>
__device__ __forceinline__ void put(T& dst, T v) {
  if constexpr (STORE) dst = v; else dst += v;
}

template <bool STORE_OFF, typename T, int D, int AD>
__device__ __forceinline__ void apply_edge_side(const EdgeRes<T, D, AD>& R, int side, T* dacc,
                                                T* off, T* gr) {
  if constexpr (AD != kAdFull) {
    const T sg = side == 0 ? T(1) : T(-1);
#pragma unroll
    for (int q = 0; q < Tri<D>::size; ++q) dacc[q] += R.K[q];
#pragma unroll
    for (int a = 0; a < D; ++a) {
#pragma unroll
      for (int b = 0; b < D; ++b)
        put<STORE_OFF>(off[a * D + b], -(a <= b ? R.K[Tri<D>::idx(a, b)] : R.K[Tri<D>::idx(b, a)]));
      gr[a] += sg * R.g[a];
    }
  } else {
#pragma unroll
    for (int a = 0; a < D; ++a) {
#pragma unroll
      for (int b = a; b < D; ++b)
        dacc[Tri<D>::idx(a, b)] += side == 0 ? R.d.Haa[a * D + b] : R.d.Hbb[a * D + b];
#pragma unroll
      for (int b = 0; b < D; ++b)
        put<STORE_OFF>(off[a * D + b], side == 0 ? R.d.Hab[a * D + b] : R.d.Hab[b * D + a]);
      gr[a] += side == 0 ? R.d.ga[a] : R.d.gb[a];
    }
  }
}

template <typename T, int D, int AD>
__device__ __forceinline__ T edge_energy(const EdgeRes<T, D, AD>& R) {
  if constexpr (AD != kAdFull) return R.E; else return R.d.E;
}

// Inertia: reduced seeding on r = x - xt (width D)
template <typename T, int D>
__device__ __forceinline__ void eval_inertia(const T* x, const T* xt, T w, T& E, T* g,
                                             T* Hd) {
  T r[D];
#pragma unroll
  for (int a = 0; a < D; ++a) r[a] = x[a] - xt[a];
  const auto e = sqnorm_m<T, D>(r) * (T(0.5) * w);
  E = e.v;
#pragma unroll
  for (int a = 0; a < D; ++a) g[a] = sgrad(e, a);
#pragma unroll
  for (int a = 0; a < D; ++a)
#pragma unroll
    for (int b = 0; b < D; ++b) Hd[a * D + b] = shess(e, a, b);
}

// Symmetric Dirichlet face term in 2D.  u0, u1, u2 are the corners' UV, M the
// row-major Dm^-1, A the rest area.  Output g[6] (corner-major) and the 3x3
// grid of 2x2 blocks H[k][l][4].
template <typename T>
struct FaceDerivs {
  T E;
  T g[6];
  T H[3][3][4];
};

// (AD: kAdReduced or kAdFull; the dense number types)
template <typename T, int AD, int KIND = kFaceSymDir>
__device__ __forceinline__ void eval_symdir(const T* u0, const T* u1, const T* u2,
                                            const T* M, T A, FaceDerivs<T>& o) {
  static_assert(AD != kAdGeneric, "the generic form runs on the row kernels");
  // corner weights w_k: dJ[al][ga]/du_k[be] = delta(al, be) w_k[ga]
  const T w[3][2] = {{-(M[0] + M[2]), -(M[1] + M[3])}, {M[0], M[1]}, {M[2], M[3]}};
  if constexpr (AD != kAdFull) {
    T Jv[4];
#pragma unroll
    for (int al = 0; al < 2; ++al)
#pragma unroll
      for (int ga = 0; ga < 2; ++ga)
        Jv[2 * al + ga] = (u1[al] - u0[al]) * M[ga] + (u2[al] - u0[al]) * M[2 + ga];
    Lin<T, 4> j[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) j[p] = lin_var<T, 4>(Jv[p], p);
    HyperDual<T, 4> e = face2_energy<KIND>(j, A);
    o.E = e.v;
#pragma unroll
    for (int k = 0; k < 3; ++k)
#pragma unroll
      for (int al = 0; al < 2; ++al)
        o.g[2 * k + al] = e.g[2 * al] * w[k][0] + e.g[2 * al + 1] * w[k][1];
#pragma unroll
    for (int k = 0; k < 3; ++k)
#pragma unroll
      for (int l = 0; l < 3; ++l)
#pragma unroll
        for (int al = 0; al < 2; ++al)
#pragma unroll
          for (int be = 0; be < 2; ++be) {
            T s = T(0);
#pragma unroll
            for (int ga = 0; ga < 2; ++ga)
#pragma unroll
              for (int de = 0; de < 2; ++de)
                s += hess(e, 2 * al + ga, 2 * be + de) * (w[k][ga] * w[l][de]);
            o.H[k][l][2 * al + be] = s;
          }
  } else {
    Lin<T, 6> u[3][2];
#pragma unroll
    for (int al = 0; al < 2; ++al) {
      u[0][al] = lin_var<T, 6>(u0[al], 0 + al);
      u[1][al] = lin_var<T, 6>(u1[al], 2 + al);
      u[2][al] = lin_var<T, 6>(u2[al], 4 + al);
    }
    Lin<T, 6> j[4];
#pragma unroll
    for (int al = 0; al < 2; ++al)
#pragma unroll
      for (int ga = 0; ga < 2; ++ga)
        j[2 * al + ga] = (u[1][al] - u[0][al]) * M[ga] + (u[2][al] - u[0][al]) * M[2 + ga];
    HyperDual<T, 6> e = face2_energy<KIND>(j, A);
    o.E = e.v;
#pragma unroll
    for (int q = 0; q < 6; ++q) o.g[q] = e.g[q];
#pragma unroll
    for (int k = 0; k < 3; ++k)
#pragma unroll
      for (int l = 0; l < 3; ++l)
#pragma unroll
        for (int al = 0; al < 2; ++al)
#pragma unroll
          for (int be = 0; be < 2; ++be)
            o.H[k][l][2 * al + be] = hess(e, 2 * k + al, 2 * l + be);
  }
}

// One corner's share of a symmetric Dirichlet face term, for the row of that
// corner's vertex i: the gradient g_i, the blocks H_ii, H_ij, H_ik (row-major
// 2x2 each) and the energy.  The face's corners in order are (i, j, k) rotated
// by c: i is corner c, j corner c+1, k corner c+2 (mod 3).  J is formed from
// the face's own edge differences in its own corner order, as eval_symdir
// does, so every corner row sees the same J up to rounding.
template <typename T>
struct FaceRow {
  T E;
  T g[2];
  T H[3][4];  // (i,i), (i,j), (i,k)
};

template <typename T>
__device__ __forceinline__ T sel3(int c, T a, T b, T d) {
  return c == 0 ? a : (c == 1 ? b : d);
}

// The share of corner i of a dof-2 face term given its value, gradient and
// Hessian in J space (e, J in the face's own corner order): the corner
// weights wr of i, j, k (rotated from those of corners 0, 1, 2) map
// g_i[al] = sum_ga dE/dJ[al][ga] w_i[ga] and block (i, l)[al][be] =
// sum_{ga,de} H_J[(al,ga),(be,de)] w_i[ga] w_l[de].
template <typename T>
__device__ __forceinline__ void project_face_row(const HyperDual<T, 4>& e, const T (&wr)[3][2],
                                                 FaceRow<T>& o) {
  o.E = e.v;
#pragma unroll
  for (int al = 0; al < 2; ++al) o.g[al] = e.g[2 * al] * wr[0][0] + e.g[2 * al + 1] * wr[0][1];
  // q[al][be][de] = sum_ga H_J[(al,ga),(be,de)] w_i[ga]
  T q[2][2][2];
#pragma unroll
  for (int al = 0; al < 2; ++al)
#pragma unroll
    for (int be = 0; be < 2; ++be)
#pragma unroll
      for (int de = 0; de < 2; ++de)
        q[al][be][de] = hess(e, 2 * al + 0, 2 * be + de) * wr[0][0] +
                        hess(e, 2 * al + 1, 2 * be + de) * wr[0][1];
#pragma unroll
  for (int l = 0; l < 3; ++l)
#pragma unroll
    for (int al = 0; al < 2; ++al)
#pragma unroll
      for (int be = 0; be < 2; ++be)
        o.H[l][2 * al + be] = q[al][be][0] * wr[l][0] + q[al][be][1] * wr[l][1];
}

// the corner weights of i, j, k for the row of corner c of a face with Dm^-1 M
template <typename T>
__device__ __forceinline__ void rotated_weights(const T* M, int c, T (&wr)[3][2]) {
  const T w[3][2] = {{-(M[0] + M[2]), -(M[1] + M[3])}, {M[0], M[1]}, {M[2], M[3]}};
#pragma unroll
  for (int ga = 0; ga < 2; ++ga) {
    wr[0][ga] = sel3(c, w[0][ga], w[1][ga], w[2][ga]);
    wr[1][ga] = sel3(c, w[1][ga], w[2][ga], w[0][ga]);
    wr[2][ga] = sel3(c, w[2][ga], w[0][ga], w[1][ga]);
  }
}

template <typename T, int AD, int KIND>
__device__ __forceinline__ void eval_symdir_row(const T* xi, const T* xj, const T* xk, int c,
                                                const T* M, T A, FaceRow<T>& o) {
  // corner weights of corners 0, 1, 2; then those of i, j, k
  const T w[3][2] = {{-(M[0] + M[2]), -(M[1] + M[3])}, {M[0], M[1]}, {M[2], M[3]}};
  if constexpr (AD != kAdFull) {
    T wr[3][2];
#pragma unroll
    for (int ga = 0; ga < 2; ++ga) {
      wr[0][ga] = sel3(c, w[0][ga], w[1][ga], w[2][ga]);
      wr[1][ga] = sel3(c, w[1][ga], w[2][ga], w[0][ga]);
      wr[2][ga] = sel3(c, w[2][ga], w[0][ga], w[1][ga]);
    }
    T Jv[4];
#pragma unroll
    for (int al = 0; al < 2; ++al) {
      // corners 0, 1, 2 of the face: c = 0 -> (i, j, k), 1 -> (k, i, j), 2 -> (j, k, i)
      const T u0 = sel3(c, xi[al], xk[al], xj[al]);
      const T u1 = sel3(c, xj[al], xi[al], xk[al]);
      const T u2 = sel3(c, xk[al], xj[al], xi[al]);
#pragma unroll
      for (int ga = 0; ga < 2; ++ga) Jv[2 * al + ga] = (u1 - u0) * M[ga] + (u2 - u0) * M[2 + ga];
    }
    const HyperDual<T, 4> e = face2_hd<KIND, AD>(Jv, A);
    project_face_row<T>(e, wr, o);
  } else {
    // width-6 AD over (x_i, x_j, x_k)
    Lin<T, 6> ui[2], uj[2], uk[2];
#pragma unroll
    for (int al = 0; al < 2; ++al) {
      ui[al] = lin_var<T, 6>(xi[al], 0 + al);
      uj[al] = lin_var<T, 6>(xj[al], 2 + al);
      uk[al] = lin_var<T, 6>(xk[al], 4 + al);
    }
    Lin<T, 6> j[4];
#pragma unroll
    for (int al = 0; al < 2; ++al) {
      const Lin<T, 6> u0 = c == 0 ? ui[al] : (c == 1 ? uk[al] : uj[al]);
      const Lin<T, 6> u1 = c == 0 ? uj[al] : (c == 1 ? ui[al] : uk[al]);
      const Lin<T, 6> u2 = c == 0 ? uk[al] : (c == 1 ? uj[al] : ui[al]);
#pragma unroll
      for (int ga = 0; ga < 2; ++ga) j[2 * al + ga] = (u1 - u0) * M[ga] + (u2 - u0) * M[2 + ga];
    }
    HyperDual<T, 6> e = face2_energy<KIND>(j, A);
    o.E = e.v;
    o.g[0] = e.g[0];
    o.g[1] = e.g[1];
#pragma unroll
    for (int l = 0; l < 3; ++l)
#pragma unroll
      for (int al = 0; al < 2; ++al)
#pragma unroll
        for (int be = 0; be < 2; ++be) o.H[l][2 * al + be] = hess(e, al, 2 * l + be);
  }
}

// One corner's share of an area-preservation face (dof 3): gradient g_i and
// the blocks (i,i), (i,j), (i,k) (row-major 3x3) for the row of vertex i,
// with (i, j, k) the face's corners rotated so that i comes first.  A cyclic
// rotation leaves n = e1 x e2 unchanged, so the row evaluates the face with
// e1 = x_j - x_i and e2 = x_k - x_i.  Reduced seeding on (e1, e2) (width 6):
// corner i's coefficients on (e1, e2) are (-1, -1), j's (1, 0) and k's
// (0, 1), so block (a, b) = sum_{s,t} p_s[a] p_t[b] H_(s,t) becomes
//   (i,i) = H11 + H12 + H21 + H22,  (i,j) = -(H11 + H21),  (i,k) = -(H12 + H22).
// Both seedings run on the masked AD numbers: the e components are single
// variables (reduced) or differences of two (full).
template <typename T>
struct FaceRow3 {
  T E;
  T g[3];
  T H[3][9];  // (i,i), (i,j), (i,k)
};

template <typename T, int AD>
__device__ __forceinline__ void eval_area_row(const T* xi, const T* xj, const T* xk, T A0, T k,
                                              FaceRow3<T>& o) {
  if constexpr (AD != kAdFull) {
    const auto e = area_energy_ad<AD>(
        slin_var<T, 6, 0>(xj[0] - xi[0]), slin_var<T, 6, 1>(xj[1] - xi[1]),
        slin_var<T, 6, 2>(xj[2] - xi[2]), slin_var<T, 6, 3>(xk[0] - xi[0]),
        slin_var<T, 6, 4>(xk[1] - xi[1]), slin_var<T, 6, 5>(xk[2] - xi[2]), A0, k);
    o.E = e.v;
#pragma unroll
    for (int al = 0; al < 3; ++al) o.g[al] = -(sgrad(e, al) + sgrad(e, 3 + al));
#pragma unroll
    for (int al = 0; al < 3; ++al)
#pragma unroll
      for (int be = 0; be < 3; ++be) {
        const T h11 = shess(e, al, be), h12 = shess(e, al, 3 + be);
        const T h21 = shess(e, 3 + al, be), h22 = shess(e, 3 + al, 3 + be);
        o.H[0][3 * al + be] = (h11 + h12) + (h21 + h22);
        o.H[1][3 * al + be] = -(h11 + h21);
        o.H[2][3 * al + be] = -(h12 + h22);
      }
  } else {
    // width-9 AD over (x_i, x_j, x_k)
    const auto i0 = slin_var<T, 9, 0>(xi[0]);
    const auto i1 = slin_var<T, 9, 1>(xi[1]);
    const auto i2 = slin_var<T, 9, 2>(xi[2]);
    const auto e = area_energy_m(slin_var<T, 9, 3>(xj[0]) - i0, slin_var<T, 9, 4>(xj[1]) - i1,
                                 slin_var<T, 9, 5>(xj[2]) - i2, slin_var<T, 9, 6>(xk[0]) - i0,
                                 slin_var<T, 9, 7>(xk[1]) - i1, slin_var<T, 9, 8>(xk[2]) - i2,
                                 A0, k);
    o.E = e.v;
#pragma unroll
    for (int al = 0; al < 3; ++al) o.g[al] = sgrad(e, al);
#pragma unroll
    for (int m = 0; m < 3; ++m)
#pragma unroll
      for (int al = 0; al < 3; ++al)
#pragma unroll
        for (int be = 0; be < 3; ++be) o.H[m][3 * al + be] = shess(e, al, 3 * m + be);
  }
}

// (H v) of one area-preservation face for its three corners (face order):
// out[3a + al].  Reduced form: t = H_e dE with dE = (v1 - v0, v2 - v0), then
// corner a takes p1[a] t_e1 + p2[a] t_e2 with p1 = (-1, 1, 0), p2 = (-1, 0, 1).
template <typename T, int AD>
__device__ __forceinline__ void hv_area_face(const T* u0, const T* u1, const T* u2,
                                             const T* v0, const T* v1, const T* v2, T A0, T k,
                                             T* out) {
  if constexpr (AD != kAdFull) {
    const auto e = area_energy_ad<AD>(
        slin_var<T, 6, 0>(u1[0] - u0[0]), slin_var<T, 6, 1>(u1[1] - u0[1]),
        slin_var<T, 6, 2>(u1[2] - u0[2]), slin_var<T, 6, 3>(u2[0] - u0[0]),
        slin_var<T, 6, 4>(u2[1] - u0[1]), slin_var<T, 6, 5>(u2[2] - u0[2]), A0, k);
    T d[6];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      d[a] = v1[a] - v0[a];
      d[3 + a] = v2[a] - v0[a];
    }
    T t[6];
#pragma unroll
    for (int p = 0; p < 6; ++p) {
      T s = shess(e, p, 0) * d[0];
#pragma unroll
      for (int q = 1; q < 6; ++q) s += shess(e, p, q) * d[q];
      t[p] = s;
    }
#pragma unroll
    for (int al = 0; al < 3; ++al) {
      out[al] = -(t[al] + t[3 + al]);
      out[3 + al] = t[al];
      out[6 + al] = t[3 + al];
    }
  } else {
    const auto a0 = slin_var<T, 9, 0>(u0[0]);
    const auto a1 = slin_var<T, 9, 1>(u0[1]);
    const auto a2 = slin_var<T, 9, 2>(u0[2]);
    const auto e = area_energy_m(slin_var<T, 9, 3>(u1[0]) - a0, slin_var<T, 9, 4>(u1[1]) - a1,
                                 slin_var<T, 9, 5>(u1[2]) - a2, slin_var<T, 9, 6>(u2[0]) - a0,
                                 slin_var<T, 9, 7>(u2[1]) - a1, slin_var<T, 9, 8>(u2[2]) - a2,
                                 A0, k);
    const T* vv[3] = {v0, v1, v2};
#pragma unroll
    for (int p = 3; p < 9; ++p) {
      T s = shess(e, p, 0) * vv[0][0];
#pragma unroll
      for (int q = 1; q < 9; ++q) s += shess(e, p, q) * vv[q / 3][q % 3];
      out[p] = s;
    }
    // the term is translation invariant: corner 0 is minus corners 1 and 2
#pragma unroll
    for (int al = 0; al < 3; ++al) out[al] = -(out[3 + al] + out[6 + al]);
  }
}

// (H v) of one symmetric Dirichlet face for all three corners: out[2k + al]
// = sum_l (H_kl v_l)[al], with u and v the corners' positions and direction
// in face order.  The reduced form contracts in J space: dJ = sum_k v_k w_k^T,
// t = H_J dJ, out_k = t projected on w_k.
template <typename T, int AD, int KIND>
__device__ __forceinline__ void hv_symdir_face(const T* u0, const T* u1, const T* u2,
                                               const T* v0, const T* v1, const T* v2,
                                               const T* M, T A, T* out) {
  if constexpr (AD != kAdFull) {
    const T w[3][2] = {{-(M[0] + M[2]), -(M[1] + M[3])}, {M[0], M[1]}, {M[2], M[3]}};
    T Jv[4], dJ[4];
#pragma unroll
    for (int al = 0; al < 2; ++al)
#pragma unroll
      for (int ga = 0; ga < 2; ++ga) {
        Jv[2 * al + ga] = (u1[al] - u0[al]) * M[ga] + (u2[al] - u0[al]) * M[2 + ga];
        dJ[2 * al + ga] = (v1[al] - v0[al]) * M[ga] + (v2[al] - v0[al]) * M[2 + ga];
      }
    const HyperDual<T, 4> e = face2_hd<KIND, AD>(Jv, A);
    T t[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      T s = T(0);
#pragma unroll
      for (int q = 0; q < 4; ++q) s += hess(e, p, q) * dJ[q];
      t[p] = s;
    }
#pragma unroll
    for (int k = 0; k < 3; ++k)
#pragma unroll
      for (int al = 0; al < 2; ++al) out[2 * k + al] = t[2 * al] * w[k][0] + t[2 * al + 1] * w[k][1];
  } else {
    FaceDerivs<T> o;
    eval_symdir<T, kAdFull, KIND>(u0, u1, u2, M, A, o);
    const T* vv[3] = {v0, v1, v2};
#pragma unroll
    for (int k = 0; k < 3; ++k)
#pragma unroll
      for (int al = 0; al < 2; ++al) {
        T s = T(0);
#pragma unroll
        for (int l = 0; l < 3; ++l)
          s += o.H[k][l][2 * al] * vv[l][0] + o.H[k][l][2 * al + 1] * vv[l][1];
        out[2 * k + al] = s;
      }
  }
}

}  // namespace mad
