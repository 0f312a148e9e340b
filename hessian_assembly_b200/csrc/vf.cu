// vf.cu -- vertex-face terms: a vertex p and the three corners (a, b, c) of a
// mesh face, a 4-vertex stencil with 12 variables and sixteen 3x3 blocks.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法 (key design 4: runtime terms whose blocks are
// inserted into the CSR on the GPU) and section 实验结果 (the contact shell,
// whose vertex-face terms change every step).  The energy is
//   E = 1/2 k (d - r)^2,  d = (p - a) . n / |n|,  n = (b - a) x (c - a),
// the signed distance of p to the face's plane against a rest offset r.
//
// The blocks between p and the corners are the three vertex pairs of each
// term, inserted by mad_add_pairs; the blocks among the corners are mesh
// blocks.  One thread evaluates one term, after the row kernel has written
// every row, and adds its gradient, blocks and energy with atomics: the
// scatter form of the pages' key design 4.  Contributions of several terms to
// one block therefore add in no fixed order.
//
// Forward-mode AD on masked numbers (sparse_ad.cuh) seeded on the natural
// variables z = (u, e1, e2) = (p - a, b - a, c - a), width 9; the stencil's
// coefficients on z are p: (1, 0, 0), a: (-1, -1, -1), b: (0, 1, 0),
// c: (0, 0, 1), so block (i, j) = sum_{s,t} c_i[s] c_j[t] H_z(s, t).
#include <cuda_runtime.h>
#include <stdint.h>

#include "mad_internal.h"
#include "sparse_ad.cuh"

namespace mad {
namespace {

constexpr int kVfThreads = 256;

// coefficient of stencil vertex v (p, a, b, c) on natural variable s (u, e1, e2)
__host__ __device__ constexpr int vf_coef(int v, int s) {
  return v == 0 ? (s == 0 ? 1 : 0) : v == 1 ? -1 : (v - 1 == s ? 1 : 0);
}

// E and its derivatives in z of one term: value, gradient [9], Hessian
// (packed).  GEN: E written as a plain expression, d = (u . n) / sqrt(n . n)
// and E = k/2 (d - r)^2, differentiated by the number types' operations and
// elementary functions alone; otherwise 1/|n| and the final square are
// single chain-rule steps with their derivatives written out.
template <typename T, bool GEN>
__device__ __forceinline__ auto vf_energy(const T* p, const T* a, const T* b, const T* c, T r,
                                          T k) {
  const auto u0 = to_shd(slin_var<T, 9, 0>(p[0] - a[0]));
  const auto u1 = to_shd(slin_var<T, 9, 1>(p[1] - a[1]));
  const auto u2 = to_shd(slin_var<T, 9, 2>(p[2] - a[2]));
  const auto e10 = slin_var<T, 9, 3>(b[0] - a[0]);
  const auto e11 = slin_var<T, 9, 4>(b[1] - a[1]);
  const auto e12 = slin_var<T, 9, 5>(b[2] - a[2]);
  const auto e20 = slin_var<T, 9, 6>(c[0] - a[0]);
  const auto e21 = slin_var<T, 9, 7>(c[1] - a[1]);
  const auto e22 = slin_var<T, 9, 8>(c[2] - a[2]);
  const auto n0 = e11 * e22 - e12 * e21;
  const auto n1 = e12 * e20 - e10 * e22;
  const auto n2 = e10 * e21 - e11 * e20;
  const auto un = u0 * n0 + u1 * n1 + u2 * n2;
  const auto nn = sq(n0) + sq(n1) + sq(n2);
  if constexpr (GEN) {
    const auto d = un * inv(sqrt(nn));
    return sq(d - r) * (T(0.5) * k);
  } else {
    // 1/|n| as one chain step: s^(-1/2), -1/2 s^(-3/2), 3/4 s^(-5/2)
    const T is = T(1) / ::sqrt(nn.v);
    const T is2 = is * is;
    const auto inv_m = chain(nn, is, T(-0.5) * is * is2, T(0.75) * is * is2 * is2);
    const auto d = un * inv_m;
    const T dev = d.v - r;
    return chain(d, T(0.5) * k * dev * dev, k * dev, k);
  }
}

__device__ __forceinline__ int find_col(const int32_t* __restrict__ rp,
                                        const int32_t* __restrict__ ci, int row, int col) {
  int lo = rp[row], hi = rp[row + 1];
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (ci[mid] < col) lo = mid + 1;
    else hi = mid;
  }
  return (lo < rp[row + 1] && ci[lo] == col) ? lo : -1;
}

// dst[0..n-1] += v[0..n-1] for n = 3 (a vertex's gradient) or 9 (a block).
// fp32: pairs of adds as one 8-byte vector reduction
// (red.global.add.v2.f32), starting at element 0 when dst is 8-byte aligned
// and at element 1 otherwise, so that every pair is 8-byte aligned; the one
// element left over takes a scalar add.  fp64: scalar adds.
__device__ __forceinline__ void red_add2(float* a, float x, float y) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(a), "f"(x), "f"(y) : "memory");
}
template <int NV, typename T>
__device__ __forceinline__ void add_vec(T* dst, const T (&v)[NV]) {
  static_assert(NV % 2 == 1, "odd length: one scalar add");
  if constexpr (sizeof(T) == 4) {
    if ((reinterpret_cast<uintptr_t>(dst) & 7u) == 0) {
#pragma unroll
      for (int q = 0; q + 1 < NV; q += 2) red_add2(dst + q, v[q], v[q + 1]);
      atomicAdd(dst + NV - 1, v[NV - 1]);
    } else {
      atomicAdd(dst, v[0]);
#pragma unroll
      for (int q = 1; q + 1 < NV + 1; q += 2) red_add2(dst + q, v[q], v[q + 1]);
    }
  } else {
#pragma unroll
    for (int q = 0; q < NV; ++q) atomicAdd(dst + q, v[q]);
  }
}

template <typename T>
__device__ __forceinline__ bool load_term(int t, const int32_t* __restrict__ vf,
                                          const int32_t* __restrict__ F, int nF, int V,
                                          const T* __restrict__ x, int vid[4], T X[4][3]) {
  const int p = vf[2 * t], f = vf[2 * t + 1];
  if (p < 0 || p >= V || f < 0 || f >= nF) return false;
  vid[0] = p;
  vid[1] = F[3 * f];
  vid[2] = F[3 * f + 1];
  vid[3] = F[3 * f + 2];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int al = 0; al < 3; ++al) X[q][al] = x[(int64_t)vid[q] * 3 + al];
  return true;
}

template <typename T, bool GEN>
__global__ void __launch_bounds__(kVfThreads) k_vf_eval(
    int n, const int32_t* __restrict__ vf, const T* __restrict__ rest, T k,
    const int32_t* __restrict__ F, int nF, int V, const T* __restrict__ x,
    const int32_t* __restrict__ rp, const int32_t* __restrict__ ci, T* __restrict__ g,
    T* __restrict__ H, double* energy, int32_t* status) {
  const int t = blockIdx.x * kVfThreads + threadIdx.x;
  double e = 0.0;
  int vid[4];
  T X[4][3];
  if (t < n) {
    if (!load_term<T>(t, vf, F, nF, V, x, vid, X)) {
      atomicOr(status, kStatusIndex);
    } else {
      const auto z = vf_energy<T, GEN>(X[0], X[1], X[2], X[3], rest[t], k);
      e = (double)z.v;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        T gi[3];
#pragma unroll
        for (int al = 0; al < 3; ++al) {
          T s = T(-0.0);
#pragma unroll
          for (int sv = 0; sv < 3; ++sv)
            if (vf_coef(i, sv) != 0) s += T(vf_coef(i, sv)) * sgrad(z, 3 * sv + al);
          gi[al] = s;
        }
        add_vec<3>(g + (int64_t)vid[i] * 3, gi);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int pos = find_col(rp, ci, vid[i], vid[j]);
          if (pos < 0) {
            atomicOr(status, kStatusIndex);
            continue;
          }
          T bv[9];
#pragma unroll
          for (int al = 0; al < 3; ++al)
#pragma unroll
            for (int be = 0; be < 3; ++be) {
              T s = T(-0.0);
#pragma unroll
              for (int sv = 0; sv < 3; ++sv)
#pragma unroll
                for (int tv = 0; tv < 3; ++tv)
                  if (vf_coef(i, sv) * vf_coef(j, tv) != 0)
                    s += T(vf_coef(i, sv) * vf_coef(j, tv)) * shess(z, 3 * sv + al, 3 * tv + be);
              bv[3 * al + be] = s;
            }
          add_vec<9>(H + (int64_t)pos * 9, bv);
        }
    }
  }
  if (energy) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e += __shfl_down_sync(0xFFFFFFFFu, e, o);
    if ((threadIdx.x & 31) == 0 && e != 0.0) atomicAdd(energy, e);
  }
}

template <typename T, bool GEN>
__global__ void __launch_bounds__(kVfThreads) k_vf_hvp(
    int n, const int32_t* __restrict__ vf, const T* __restrict__ rest, T k,
    const int32_t* __restrict__ F, int nF, int V, const T* __restrict__ x,
    const T* __restrict__ v, T* __restrict__ y, int32_t* status) {
  const int t = blockIdx.x * kVfThreads + threadIdx.x;
  if (t >= n) return;
  int vid[4];
  T X[4][3];
  if (!load_term<T>(t, vf, F, nF, V, x, vid, X)) {
    atomicOr(status, kStatusIndex);
    return;
  }
  const auto z = vf_energy<T, GEN>(X[0], X[1], X[2], X[3], rest[t], k);
  // dz_s = sum_j c_j[s] v_j, t = H_z dz, y_i = sum_s c_i[s] t_s
  T dz[9];
#pragma unroll
  for (int sv = 0; sv < 3; ++sv)
#pragma unroll
    for (int al = 0; al < 3; ++al) {
      T s = T(-0.0);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (vf_coef(j, sv) != 0) s += T(vf_coef(j, sv)) * v[(int64_t)vid[j] * 3 + al];
      dz[3 * sv + al] = s;
    }
  T tz[9];
#pragma unroll
  for (int q = 0; q < 9; ++q) {
    T s = shess(z, q, 0) * dz[0];
#pragma unroll
    for (int w = 1; w < 9; ++w) s += shess(z, q, w) * dz[w];
    tz[q] = s;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    T yi[3];
#pragma unroll
    for (int al = 0; al < 3; ++al) {
      T s = T(-0.0);
#pragma unroll
      for (int sv = 0; sv < 3; ++sv)
        if (vf_coef(i, sv) != 0) s += T(vf_coef(i, sv)) * tz[3 * sv + al];
      yi[al] = s;
    }
    add_vec<3>(y + (int64_t)vid[i] * 3, yi);
  }
}

// ---------------------------------------------------------------------------
// Installed term sets (mad_add_vf): the gather form.  Every term is listed in
// the rows of its four vertices; one thread per row evaluates the row's
// terms and adds only the row's share (its gradient and its four blocks) to
// g and H, which the row kernel has just written.  No two threads touch the
// same row, so no atomics are needed and the sums are reproducible.
//
// Entry of row i (32 bytes): term t and role r (which stencil vertex i is:
// p, a, b or c) packed as t | r << 30, then the block positions of the
// stencil's four vertices p, a, b, c in row i of the active pattern (-1:
// missing, the entry is skipped).

__device__ __forceinline__ bool vf_term(int t, const int32_t* __restrict__ terms,
                                        const int32_t* __restrict__ F, int nF, int V,
                                        int vid[4]) {
  const int p = terms[2 * t], f = terms[2 * t + 1];
  if (p < 0 || p >= V || f < 0 || f >= nF) return false;
  vid[0] = p;
  vid[1] = F[3 * f];
  vid[2] = F[3 * f + 1];
  vid[3] = F[3 * f + 2];
  return p != vid[1] && p != vid[2] && p != vid[3];
}

// N values at p (N a multiple of 4; p 16-byte aligned) in 16-byte accesses
template <typename T, int N>
__device__ __forceinline__ void store_rec(T* p, const T* r) {
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int q = 0; q < N; q += 4)
      reinterpret_cast<float4*>(p)[q / 4] = make_float4(r[q], r[q + 1], r[q + 2], r[q + 3]);
  } else {
#pragma unroll
    for (int q = 0; q < N; q += 2) reinterpret_cast<double2*>(p)[q / 2] = make_double2(r[q], r[q + 1]);
  }
}
template <typename T, int N>
__device__ __forceinline__ void load_rec(const T* p, T* r) {
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int q = 0; q < N; q += 4) {
      const float4 v4 = reinterpret_cast<const float4*>(p)[q / 4];
      r[q] = v4.x;
      r[q + 1] = v4.y;
      r[q + 2] = v4.z;
      r[q + 3] = v4.w;
    }
  } else {
#pragma unroll
    for (int q = 0; q < N; q += 2) {
      const double2 v2 = reinterpret_cast<const double2*>(p)[q / 2];
      r[q] = v2.x;
      r[q + 1] = v2.y;
    }
  }
}

// the terms' (vertex, corner) pairs for the insertion, and a copy of the terms
__global__ void __launch_bounds__(kVfThreads) k_vf_expand(int n, const int32_t* __restrict__ vf,
                                                          const int32_t* __restrict__ F, int nF,
                                                          int V, int32_t* pairs,
                                                          int32_t* terms) {
  const int t = blockIdx.x * kVfThreads + threadIdx.x;
  if (t >= n) return;
  const int p = vf[2 * t], f = vf[2 * t + 1];
  terms[2 * t] = p;
  terms[2 * t + 1] = f;
  int vid[4];
  const bool ok = vf_term(t, terms, F, nF, V, vid);
#pragma unroll
  for (int c = 0; c < 3; ++c) {  // a bad term gives pairs the insertion rejects
    pairs[2 * (3 * t + c)] = ok ? p : -1;
    pairs[2 * (3 * t + c) + 1] = ok ? vid[1 + c] : -1;
  }
}

__global__ void __launch_bounds__(kVfThreads) k_vf_count(int n, const int32_t* __restrict__ terms,
                                                         const int32_t* __restrict__ F, int nF,
                                                         int V, int32_t* cnt) {
  const int t = blockIdx.x * kVfThreads + threadIdx.x;
  int vid[4];
  if (t >= n || !vf_term(t, terms, F, nF, V, vid)) return;
#pragma unroll
  for (int r = 0; r < 4; ++r) atomicAdd(&cnt[vid[r]], 1);
}

// each incidence takes a slot of its row, counting the row counter back to 0
__global__ void __launch_bounds__(kVfThreads) k_vf_fill(int n, const int32_t* __restrict__ terms,
                                                        const int32_t* __restrict__ F, int nF,
                                                        int V, const int32_t* __restrict__ vrow,
                                                        int32_t* cnt, int32_t* ent) {
  const int t = blockIdx.x * kVfThreads + threadIdx.x;
  int vid[4];
  if (t >= n || !vf_term(t, terms, F, nF, V, vid)) return;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int slot = vrow[vid[r]] + atomicSub(&cnt[vid[r]], 1) - 1;
    ent[8 * slot] = t | (r << 30);
  }
}

// per row: entries in (term, role) order, then the block positions, and
// for every (term, role) its entry's index (where the term pass writes that
// vertex's share)
__global__ void __launch_bounds__(kVfThreads) k_vf_finalize(
    int V, const int32_t* __restrict__ vrow, int32_t* ent, const int32_t* __restrict__ terms,
    const int32_t* __restrict__ F, int nF, const int32_t* __restrict__ rp,
    const int32_t* __restrict__ ci, int32_t* vslot, int32_t* status) {
  const int i = blockIdx.x * kVfThreads + threadIdx.x;
  if (i >= V) return;
  const int b = vrow[i], e = vrow[i + 1];
  for (int q = b + 1; q < e; ++q) {  // insertion sort: rows hold few entries
    const int32_t key = ent[8 * q];
    int j = q - 1;
    while (j >= b && ent[8 * j] > key) {
      ent[8 * (j + 1)] = ent[8 * j];
      --j;
    }
    ent[8 * (j + 1)] = key;
  }
  const int r0 = rp[i];
  for (int q = b; q < e; ++q) {
    const int t = ent[8 * q] & 0x3FFFFFFF;
    int vid[4];
    vf_term(t, terms, F, nF, V, vid);
    int4 w = make_int4(0, 0, 0, 0);
    bool all = true;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int pos = find_col(rp, ci, i, vid[k]);
      all &= pos >= 0;
      const int rel = pos < 0 ? -1 : pos - r0;
      if (k < 3) (k == 0 ? w.x : k == 1 ? w.y : w.z) = rel;
      else w.w = rel;
    }
    if (!all) atomicOr(status, kStatusIndex);
    vslot[4 * t + (int)((uint32_t)ent[8 * q] >> 30)] = q;
    reinterpret_cast<int4*>(ent)[2 * q] = make_int4(ent[8 * q], w.x, w.y, w.z);
    reinterpret_cast<int4*>(ent)[2 * q + 1] = make_int4(w.w, all ? 1 : 0, 0, 0);
  }
}

// Term pass of an installed set: one thread per term differentiates it once
// and writes, for each of its four vertices (role p, a, b, c), that
// vertex's share: its gradient (3) and its blocks with the four stencil
// vertices (4 x 9), then E in the last of kVfRoleVals values.  A row then
// only adds its role's slice.
constexpr int kVfRoleVals = 40;             // 3 + 36 + E

template <typename T, bool GEN>
__global__ void __launch_bounds__(kVfThreads) k_vf_term_rec(
    int n, const int32_t* __restrict__ terms, const int32_t* __restrict__ F, int nF, int V,
    const int32_t* __restrict__ vslot, const T* __restrict__ rest, T k,
    const T* __restrict__ x, T* __restrict__ rec, double* epart) {
  const int t = blockIdx.x * kVfThreads + threadIdx.x;
  double e = 0.0;
  int vid[4];
  if (t < n && vf_term(t, terms, F, nF, V, vid)) {
    T X[4][3];
#pragma unroll
    for (int v4 = 0; v4 < 4; ++v4)
#pragma unroll
      for (int al = 0; al < 3; ++al) X[v4][al] = x[(int64_t)vid[v4] * 3 + al];
    const auto z = vf_energy<T, GEN>(X[0], X[1], X[2], X[3], rest[t], k);
    e = (double)z.v;
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      T r[kVfRoleVals];
#pragma unroll
      for (int al = 0; al < 3; ++al) {
        T s2 = T(-0.0);
#pragma unroll
        for (int sv = 0; sv < 3; ++sv)
          if (vf_coef(rr, sv) != 0) s2 += T(vf_coef(rr, sv)) * sgrad(z, 3 * sv + al);
        r[al] = s2;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int al = 0; al < 3; ++al)
#pragma unroll
          for (int be = 0; be < 3; ++be) {
            T s2 = T(-0.0);
#pragma unroll
            for (int sv = 0; sv < 3; ++sv)
#pragma unroll
              for (int tv = 0; tv < 3; ++tv)
                if (vf_coef(rr, sv) * vf_coef(j, tv) != 0)
                  s2 += T(vf_coef(rr, sv) * vf_coef(j, tv)) * shess(z, 3 * sv + al, 3 * tv + be);
            r[3 + 9 * j + 3 * al + be] = s2;
          }
      r[kVfRoleVals - 1] = z.v;
      store_rec<T, kVfRoleVals>(rec + (int64_t)vslot[4 * t + rr] * kVfRoleVals, r);
    }
  }
  if (epart) {
    __shared__ double red[kVfThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e += __shfl_down_sync(0xFFFFFFFFu, e, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = e;
    __syncthreads();
    if (threadIdx.x == 0) {
      double s2 = 0.0;
      for (int w = 0; w < kVfThreads / 32; ++w) s2 += red[w];
      epart[blockIdx.x] = s2;
    }
  }
}

// Row pass (used when the row kernel does not gather the terms itself): one
// thread per row adds its role's slice of each of its terms to its gradient
// and blocks; each term's four blocks are read before any is written.
template <typename T>
__global__ void __launch_bounds__(kVfThreads) k_vf_rows(int V, const int32_t* __restrict__ vrow,
                                                        const int32_t* __restrict__ ent,
                                                        const T* __restrict__ rec,
                                                        const int32_t* __restrict__ rp,
                                                        T* __restrict__ g, T* __restrict__ H) {
  const int i = blockIdx.x * kVfThreads + threadIdx.x;
  if (i >= V) return;
  const int b = vrow[i], en = vrow[i + 1];
  if (en <= b) return;
  const int64_t r0 = rp[i];
  T gacc[3] = {T(0), T(0), T(0)};
  for (int q = b; q < en; ++q) {
    const int4 w0 = reinterpret_cast<const int4*>(ent)[2 * q];
    const int4 w1 = reinterpret_cast<const int4*>(ent)[2 * q + 1];
    if (!w1.y) continue;
    T r[kVfRoleVals];
    load_rec<T, kVfRoleVals>(rec + (int64_t)q * kVfRoleVals, r);
    const int pos[4] = {w0.y, w0.z, w0.w, w1.x};
    T cur[4][9];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q9 = 0; q9 < 9; ++q9) cur[j][q9] = H[(r0 + pos[j]) * 9 + q9];
#pragma unroll
    for (int al = 0; al < 3; ++al) gacc[al] += r[al];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q9 = 0; q9 < 9; ++q9) cur[j][q9] += r[3 + 9 * j + q9];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q9 = 0; q9 < 9; ++q9) H[(r0 + pos[j]) * 9 + q9] = cur[j][q9];
  }
#pragma unroll
  for (int al = 0; al < 3; ++al) g[(int64_t)i * 3 + al] += gacc[al];
}

// Product, term pass: each term's (H v) restricted to each of its four
// vertices, written per role (12 values, padded to 16).
constexpr int kVfHvRec = 16;
template <typename T, bool GEN>
__global__ void __launch_bounds__(kVfThreads) k_vf_term_hv(
    int n, const int32_t* __restrict__ terms, const int32_t* __restrict__ F, int nF, int V,
    const T* __restrict__ rest, T k, const T* __restrict__ x, const T* __restrict__ v,
    T* __restrict__ rec) {
  const int t = blockIdx.x * kVfThreads + threadIdx.x;
  int vid[4];
  if (t >= n || !vf_term(t, terms, F, nF, V, vid)) return;
  T X[4][3], W[4][3];
#pragma unroll
  for (int v4 = 0; v4 < 4; ++v4)
#pragma unroll
    for (int al = 0; al < 3; ++al) {
      X[v4][al] = x[(int64_t)vid[v4] * 3 + al];
      W[v4][al] = v[(int64_t)vid[v4] * 3 + al];
    }
  const auto z = vf_energy<T, GEN>(X[0], X[1], X[2], X[3], rest[t], k);
  T dz[9];
#pragma unroll
  for (int sv = 0; sv < 3; ++sv)
#pragma unroll
    for (int al = 0; al < 3; ++al) {
      T s2 = T(-0.0);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (vf_coef(j, sv) != 0) s2 += T(vf_coef(j, sv)) * W[j][al];
      dz[3 * sv + al] = s2;
    }
  T tz[9];
#pragma unroll
  for (int q = 0; q < 9; ++q) {
    T s2 = shess(z, q, 0) * dz[0];
#pragma unroll
    for (int w = 1; w < 9; ++w) s2 += shess(z, q, w) * dz[w];
    tz[q] = s2;
  }
  T r[kVfHvRec];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr)
#pragma unroll
    for (int al = 0; al < 3; ++al) {
      T s2 = T(-0.0);
#pragma unroll
      for (int sv = 0; sv < 3; ++sv)
        if (vf_coef(rr, sv) != 0) s2 += T(vf_coef(rr, sv)) * tz[3 * sv + al];
      r[3 * rr + al] = s2;
    }
#pragma unroll
  for (int q = 12; q < kVfHvRec; ++q) r[q] = T(0);
  store_rec<T, kVfHvRec>(rec + (int64_t)t * kVfHvRec, r);
}

template <typename T>
__global__ void __launch_bounds__(kVfThreads) k_vf_rows_hvp(int V,
                                                            const int32_t* __restrict__ vrow,
                                                            const int32_t* __restrict__ ent,
                                                            const T* __restrict__ rec,
                                                            T* __restrict__ y) {
  const int i = blockIdx.x * kVfThreads + threadIdx.x;
  if (i >= V) return;
  const int b = vrow[i], en = vrow[i + 1];
  if (en <= b) return;
  T yacc[3] = {T(0), T(0), T(0)};
  for (int q = b; q < en; ++q) {
    const int4 w0 = reinterpret_cast<const int4*>(ent)[2 * q];
    const int4 w1 = reinterpret_cast<const int4*>(ent)[2 * q + 1];
    if (!w1.y) continue;
    const int t = w0.x & 0x3FFFFFFF, role = (int)((uint32_t)w0.x >> 30);
    const T* rr = rec + (int64_t)t * kVfHvRec + 3 * role;
#pragma unroll
    for (int al = 0; al < 3; ++al) yacc[al] += rr[al];
  }
#pragma unroll
  for (int al = 0; al < 3; ++al) y[(int64_t)i * 3 + al] += yacc[al];
}

__global__ void k_energy_add(const double* __restrict__ part, int n, double* out) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += part[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    *out += t;
  }
}

}  // namespace

cudaError_t launch_vf_install_expand(const VfSet& S, int n, const int32_t* vf, int V,
                                     const int32_t* F, int nF, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const unsigned nb = (unsigned)((n + kVfThreads - 1) / kVfThreads);
  k_vf_expand<<<nb, kVfThreads, 0, s>>>(n, vf, F, nF, V, S.pairs, S.terms);
  return cudaGetLastError();
}

cudaError_t launch_vf_install_tables(const VfSet& S, int n, int V, const int32_t* F, int nF,
                                     const int32_t* rp, const int32_t* ci, int32_t* cnt,
                                     int32_t* status, cudaStream_t s) {
  cudaError_t e;
  const unsigned nb = (unsigned)((n + kVfThreads - 1) / kVfThreads);
  const unsigned nr = (unsigned)((V + kVfThreads - 1) / kVfThreads);
  if (n > 0) {
    k_vf_count<<<nb, kVfThreads, 0, s>>>(n, S.terms, F, nF, V, cnt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = scan_exclusive(cnt, S.vrow, V, S.scan_tmp, s)) != cudaSuccess) return e;
  if (n > 0) {
    k_vf_fill<<<nb, kVfThreads, 0, s>>>(n, S.terms, F, nF, V, S.vrow, cnt, S.ent);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_vf_finalize<<<nr, kVfThreads, 0, s>>>(V, S.vrow, S.ent, S.terms, F, nF, rp, ci, S.vslot,
                                            status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T, bool GEN>
cudaError_t vf_rows_t(const VfSet& S, const VfLaunch& L, void* g, void* H, double* energy,
                      cudaStream_t s) {
  const unsigned nt = (unsigned)((S.n + kVfThreads - 1) / kVfThreads);
  const unsigned nr = (unsigned)((L.V + kVfThreads - 1) / kVfThreads);
  if (S.n > 0) {
    k_vf_term_rec<T, GEN><<<nt, kVfThreads, 0, s>>>(S.n, S.terms, L.F, L.nF, L.V, S.vslot,
                                                    (const T*)L.rest, (T)L.k, (const T*)L.x,
                                                    (T*)S.rec, energy ? S.epart : nullptr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (energy) {  // E of the terms, summed once per term
      k_energy_add<<<1, 1024, 0, s>>>(S.epart, (int)nt, energy);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  k_vf_rows<T><<<nr, kVfThreads, 0, s>>>(L.V, S.vrow, S.ent, (const T*)S.rec, L.rp, (T*)g,
                                         (T*)H);
  return cudaGetLastError();
}

template <typename T, bool GEN>
cudaError_t vf_rows_hvp_t(const VfSet& S, const VfLaunch& L, const void* v, void* y,
                          cudaStream_t s) {
  const unsigned nt = (unsigned)((S.n + kVfThreads - 1) / kVfThreads);
  const unsigned nr = (unsigned)((L.V + kVfThreads - 1) / kVfThreads);
  if (S.n > 0) {
    k_vf_term_hv<T, GEN><<<nt, kVfThreads, 0, s>>>(S.n, S.terms, L.F, L.nF, L.V,
                                                   (const T*)L.rest, (T)L.k, (const T*)L.x,
                                                   (const T*)v, (T*)S.rec);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  k_vf_rows_hvp<T><<<nr, kVfThreads, 0, s>>>(L.V, S.vrow, S.ent, (const T*)S.rec, (T*)y);
  return cudaGetLastError();
}

cudaError_t launch_vf_term_pass(int dtype, const VfSet& S, const VfLaunch& L, cudaStream_t s) {
  if (S.n <= 0) return cudaSuccess;
  const unsigned nt = (unsigned)((S.n + kVfThreads - 1) / kVfThreads);
  if (dtype == MAD_F64) {
    if (L.generic)
      k_vf_term_rec<double, true><<<nt, kVfThreads, 0, s>>>(S.n, S.terms, L.F, L.nF, L.V, S.vslot,
                                                             (const double*)L.rest, L.k,
                                                             (const double*)L.x, (double*)S.rec,
                                                             nullptr);
    else
      k_vf_term_rec<double, false><<<nt, kVfThreads, 0, s>>>(S.n, S.terms, L.F, L.nF, L.V, S.vslot,
                                                              (const double*)L.rest, L.k,
                                                              (const double*)L.x,
                                                              (double*)S.rec, nullptr);
  } else {
    if (L.generic)
      k_vf_term_rec<float, true><<<nt, kVfThreads, 0, s>>>(S.n, S.terms, L.F, L.nF, L.V, S.vslot,
                                                            (const float*)L.rest, (float)L.k,
                                                            (const float*)L.x, (float*)S.rec,
                                                            nullptr);
    else
      k_vf_term_rec<float, false><<<nt, kVfThreads, 0, s>>>(S.n, S.terms, L.F, L.nF, L.V, S.vslot,
                                                             (const float*)L.rest, (float)L.k,
                                                             (const float*)L.x, (float*)S.rec,
                                                             nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_vf_rows_eval(int dtype, const VfSet& S, const VfLaunch& L, void* g, void* H,
                                double* energy, cudaStream_t s) {
  if (L.V <= 0) return cudaSuccess;
  if (dtype == MAD_F64)
    return L.generic ? vf_rows_t<double, true>(S, L, g, H, energy, s)
                     : vf_rows_t<double, false>(S, L, g, H, energy, s);
  return L.generic ? vf_rows_t<float, true>(S, L, g, H, energy, s)
                   : vf_rows_t<float, false>(S, L, g, H, energy, s);
}

cudaError_t launch_vf_rows_hvp(int dtype, const VfSet& S, const VfLaunch& L, const void* v,
                               void* y, cudaStream_t s) {
  if (L.V <= 0) return cudaSuccess;
  if (dtype == MAD_F64)
    return L.generic ? vf_rows_hvp_t<double, true>(S, L, v, y, s)
                     : vf_rows_hvp_t<double, false>(S, L, v, y, s);
  return L.generic ? vf_rows_hvp_t<float, true>(S, L, v, y, s)
                   : vf_rows_hvp_t<float, false>(S, L, v, y, s);
}

template <typename T, bool GEN>
void vf_eval_t(const VfLaunch& L, unsigned nb, void* g, void* H, double* energy, cudaStream_t s) {
  k_vf_eval<T, GEN><<<nb, kVfThreads, 0, s>>>(L.n, L.vf, (const T*)L.rest, (T)L.k, L.F, L.nF, L.V,
                                              (const T*)L.x, L.rp, L.ci, (T*)g, (T*)H, energy,
                                              L.status);
}

template <typename T, bool GEN>
void vf_hvp_t(const VfLaunch& L, unsigned nb, const void* v, void* y, cudaStream_t s) {
  k_vf_hvp<T, GEN><<<nb, kVfThreads, 0, s>>>(L.n, L.vf, (const T*)L.rest, (T)L.k, L.F, L.nF, L.V,
                                             (const T*)L.x, (const T*)v, (T*)y, L.status);
}

cudaError_t launch_vf_eval(int dtype, const VfLaunch& L, void* g, void* H, double* energy,
                           cudaStream_t s) {
  if (L.n <= 0) return cudaSuccess;
  const unsigned nb = (unsigned)((L.n + kVfThreads - 1) / kVfThreads);
  if (dtype == MAD_F64) {
    if (L.generic) vf_eval_t<double, true>(L, nb, g, H, energy, s);
    else vf_eval_t<double, false>(L, nb, g, H, energy, s);
  } else {
    if (L.generic) vf_eval_t<float, true>(L, nb, g, H, energy, s);
    else vf_eval_t<float, false>(L, nb, g, H, energy, s);
  }
  return cudaGetLastError();
}

cudaError_t launch_vf_hvp(int dtype, const VfLaunch& L, const void* v, void* y, cudaStream_t s) {
  if (L.n <= 0) return cudaSuccess;
  const unsigned nb = (unsigned)((L.n + kVfThreads - 1) / kVfThreads);
  if (dtype == MAD_F64) {
    if (L.generic) vf_hvp_t<double, true>(L, nb, v, y, s);
    else vf_hvp_t<double, false>(L, nb, v, y, s);
  } else {
    if (L.generic) vf_hvp_t<float, true>(L, nb, v, y, s);
    else vf_hvp_t<float, false>(L, nb, v, y, s);
  }
  return cudaGetLastError();
}

}  // namespace mad
