// jacobian.cu -- residual vector and sparse Jacobian of a vector-valued
// objective built from the mesh terms.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法: a vector-valued objective assembles the sparse
// Jacobian J = sum_j P_j^T J_j S_j (S_j selects the term's stencil, P_j places
// its residuals in the global residual vector); the highlights note that
// materialising J explicitly pays off for large geometry problems.
//
// Residual form of each term, chosen so that F = 1/2 |r|^2 is the term's
// scalar energy (J^T r is then the gradient and J^T J the Gauss-Newton part
// of the Hessian):
//   spring   r = sqrt(k) (|d| - L0),  d = x_a - x_b      1 row
//   inertia  r = sqrt(w) (x_v - xt_v)                     dof rows
//   SymDir   r = sqrt(2A) (vec J, vec J^-1)               8 rows
// Each term owns its rows (P_j is a contiguous row range), so a thread per
// term writes its rows directly: no assembly conflicts, no atomics.  The
// local Jacobian comes from first-order forward AD (Dual) seeded on the
// term's natural variables (d, or vec J), mapped to the stencil's columns.
//
// Layout: rows term-major -- springs (edge order), inertia (vertex order,
// dof rows each), faces (face order, 8 rows each); within a row the columns
// vertex*dof + component ascending (stencil vertices sorted by index).  Every
// row of a term type has the same number of nonzeros, so the row pointers of
// a segment are an arithmetic sequence.
#include <algorithm>

#include "dual1.cuh"
#include "mad_internal.h"

namespace mad {
namespace {

constexpr int kJT = 256;
// spring rows per thread of the residual/Jacobian kernel
#ifndef MAD_JAC_EDGES_PER_THREAD
#define MAD_JAC_EDGES_PER_THREAD 2
#endif
constexpr int kJE = MAD_JAC_EDGES_PER_THREAD;

inline unsigned jgrid(int64_t n) {
  int64_t b = (n + kJT - 1) / kJT;
  if (b < 1) b = 1;
  if (b > 65535LL * 16) b = 65535LL * 16;
  return (unsigned)b;
}

struct Segs {
  int64_t r_sp, r_in, r_fa, rows;  // first row of each segment, total rows
  int64_t z_sp, z_in, z_fa, nnz;   // first nonzero of each segment, total
  int nsp, nin, nfa;               // nonzeros per row of each segment
};

__host__ __device__ inline Segs make_segs(int V, int dof, unsigned mask, int nE, int nF) {
  Segs s{};
  const int64_t E = (mask & MAD_TERM_SPRING) ? nE : 0;
  const int64_t R = (mask & MAD_TERM_INERTIA) ? (int64_t)V * dof : 0;
  const int64_t Fr = (mask & MAD_TERM_SYMDIR) ? (int64_t)nF * 8 : 0;
  s.nsp = 2 * dof;
  s.nin = 1;
  s.nfa = 3 * dof;
  s.r_sp = 0;
  s.r_in = E;
  s.r_fa = E + R;
  s.rows = E + R + Fr;
  s.z_sp = 0;
  s.z_in = E * s.nsp;
  s.z_fa = s.z_in + R;
  s.nnz = s.z_fa + Fr * s.nfa;
  return s;
}

// sorted corner order of a face: o[0..2] = corner indices by vertex id
__device__ __forceinline__ void sort3(const int32_t* v, int* o) {
  o[0] = 0;
  o[1] = 1;
  o[2] = 2;
  if (v[o[1]] < v[o[0]]) { const int t = o[0]; o[0] = o[1]; o[1] = t; }
  if (v[o[2]] < v[o[1]]) { const int t = o[1]; o[1] = o[2]; o[2] = t; }
  if (v[o[1]] < v[o[0]]) { const int t = o[0]; o[0] = o[1]; o[1] = t; }
}

__global__ void __launch_bounds__(kJT) k_jac_pattern(Segs S, int dof, int V,
                                                     const int32_t* __restrict__ edges,
                                                     const int32_t* __restrict__ F,
                                                     int64_t* __restrict__ rp,
                                                     int32_t* __restrict__ ci) {
  for (int64_t row = blockIdx.x * (int64_t)kJT + threadIdx.x; row < S.rows;
       row += (int64_t)gridDim.x * kJT) {
    if (row < S.r_in) {  // spring e: columns of a then b (edges have a < b)
      const int64_t z = S.z_sp + row * S.nsp;
      rp[row] = z;
      const int32_t a = edges[2 * row], b = edges[2 * row + 1];
      for (int c = 0; c < dof; ++c) {
        ci[z + c] = a * dof + c;
        ci[z + dof + c] = b * dof + c;
      }
    } else if (row < S.r_fa) {  // inertia: the row's own column
      const int64_t q = row - S.r_in;
      rp[row] = S.z_in + q;
      ci[S.z_in + q] = (int32_t)q;
    } else {  // face row: its 3 corners' columns in vertex order
      const int64_t q = row - S.r_fa;
      const int64_t f = q / 8;
      const int64_t z = S.z_fa + q * S.nfa;
      rp[row] = z;
      int32_t v[3] = {F[3 * f], F[3 * f + 1], F[3 * f + 2]};
      int o[3];
      sort3(v, o);
      for (int s = 0; s < 3; ++s)
        for (int c = 0; c < dof; ++c) ci[z + s * dof + c] = v[o[s]] * dof + c;
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) rp[S.rows] = S.nnz;
  (void)V;
}

__device__ __forceinline__ void jbulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  const uint32_t sa = (uint32_t)__cvta_generic_to_shared(ssrc);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(sa), "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Springs and inertia in one launch: blocks [0, nbs) take kJT * kJE edges
// each, the rest kJT inertia rows each.  A block's spring rows (2*DOF values
// per edge, contiguous in J) are staged in shared memory and leave with one 1-D bulk
// copy when its first value and its size are 16-byte aligned; otherwise
// every thread stores its own row.
template <typename T, int DOF>
__global__ void __launch_bounds__(kJT) k_jac_edges_vertices(
    Segs S, int nE, int nbs, int64_t nin, const int32_t* __restrict__ edges,
    const T* __restrict__ x, const T* __restrict__ L0, T sk, const T* __restrict__ xt, T sw,
    T* __restrict__ r, T* __restrict__ J) {
  __shared__ __align__(16) T stage[kJT * kJE * 2 * DOF];
  if ((int)blockIdx.x < nbs) {
    // kJE edges per thread (edges e0 + h*kJT + thread), every load of them
    // issued before the first is used
    const int64_t e0 = (int64_t)blockIdx.x * kJT * kJE;
    const int cnt = (int)((nE - e0) < kJT * kJE ? (nE - e0) : kJT * kJE);
    int2 ab[kJE];
    T l0[kJE], xa[kJE][DOF], xb[kJE][DOF];
#pragma unroll
    for (int h = 0; h < kJE; ++h) {
      const int64_t e = e0 + h * kJT + threadIdx.x;
      if (e < nE) {
        ab[h] = reinterpret_cast<const int2*>(edges)[e];
        l0[h] = L0[e];
      }
    }
#pragma unroll
    for (int h = 0; h < kJE; ++h) {
      if (e0 + h * kJT + threadIdx.x >= nE) continue;
#pragma unroll
      for (int c = 0; c < DOF; ++c) {
        xa[h][c] = x[(int64_t)ab[h].x * DOF + c];
        xb[h][c] = x[(int64_t)ab[h].y * DOF + c];
      }
    }
#pragma unroll
    for (int h = 0; h < kJE; ++h) {
      const int64_t e = e0 + h * kJT + threadIdx.x;
      if (e >= nE) continue;
      Dual<T, DOF> s = d_const<T, DOF>(T(0));
#pragma unroll
      for (int c = 0; c < DOF; ++c) {
        const Dual<T, DOF> d = d_var<T, DOF>(xa[h][c] - xb[h][c], c);
        s = s + d * d;
      }
      const Dual<T, DOF> res = (sqrt(s) - l0[h]) * sk;
      r[S.r_sp + e] = res.v;
      // dr/dx_a = dr/dd, dr/dx_b = -dr/dd
      T* st = stage + (h * kJT + threadIdx.x) * 2 * DOF;
#pragma unroll
      for (int c = 0; c < DOF; ++c) {
        st[c] = res.g[c];
        st[DOF + c] = -res.g[c];
      }
    }
    __syncthreads();
    T* dst = J + S.z_sp + e0 * (2 * DOF);
    const uint32_t bytes = (uint32_t)(cnt * 2 * DOF * sizeof(T));
    if (((((uintptr_t)dst) | bytes) & 15u) == 0) {
      if (threadIdx.x == 0) jbulk_store(dst, stage, bytes);
    } else {
      for (int q = threadIdx.x; q < cnt * 2 * DOF; q += kJT) dst[q] = stage[q];
    }
  } else {
    const int64_t q = (int64_t)(blockIdx.x - nbs) * kJT + threadIdx.x;
    if (q < nin) {
      const Dual<T, 1> res = (d_var<T, 1>(x[q], 0) - xt[q]) * sw;
      r[S.r_in + q] = res.v;
      J[S.z_in + q] = res.g[0];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kJT) k_jac_faces(Segs S, int nF, const int32_t* __restrict__ F,
                                                   const T* __restrict__ x,
                                                   const T* __restrict__ Minv,
                                                   const T* __restrict__ area,
                                                   T* __restrict__ r, T* __restrict__ J) {
  for (int64_t f = blockIdx.x * (int64_t)kJT + threadIdx.x; f < nF;
       f += (int64_t)gridDim.x * kJT) {
    int32_t v[3] = {F[3 * f], F[3 * f + 1], F[3 * f + 2]};
    T M[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) M[q] = Minv[4 * f + q];
    const T s = ::sqrt(T(2) * area[f]);
    T u[3][2];
#pragma unroll
    for (int k = 0; k < 3; ++k)
#pragma unroll
      for (int al = 0; al < 2; ++al) u[k][al] = x[(int64_t)v[k] * 2 + al];
    // seeds on vec J = (J00, J01, J10, J11)
    Dual<T, 4> j[4];
#pragma unroll
    for (int al = 0; al < 2; ++al)
#pragma unroll
      for (int ga = 0; ga < 2; ++ga)
        j[2 * al + ga] = d_var<T, 4>(
            (u[1][al] - u[0][al]) * M[ga] + (u[2][al] - u[0][al]) * M[2 + ga], 2 * al + ga);
    const Dual<T, 4> id = inv(j[0] * j[3] - j[1] * j[2]);
    // J^-1 = cof(J)^T / det = [[J11, -J01], [-J10, J00]] / det
    Dual<T, 4> res[8] = {j[0] * s, j[1] * s, j[2] * s, j[3] * s,
                         (j[3] * id) * s, (-(j[1] * id)) * s, (-(j[2] * id)) * s,
                         (j[0] * id) * s};
    // dvecJ[2al+ga]/du_k[be] = delta(al,be) w_k[ga]: column (k, be) of a row
    // is sum_ga dres/dJ[be][ga] w_k[ga]
    const T w[3][2] = {{-(M[0] + M[2]), -(M[1] + M[3])}, {M[0], M[1]}, {M[2], M[3]}};
    int o[3];
    sort3(v, o);
    const int64_t row0 = 8 * f;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      r[S.r_fa + row0 + p] = res[p].v;
      T* out = J + S.z_fa + (row0 + p) * 6;
#pragma unroll
      for (int sidx = 0; sidx < 3; ++sidx) {
        const int k = o[sidx];
#pragma unroll
        for (int be = 0; be < 2; ++be)
          out[2 * sidx + be] = res[p].g[2 * be + 0] * w[k][0] + res[p].g[2 * be + 1] * w[k][1];
      }
    }
  }
}

}  // namespace

void jac_shape(int V, int dof, unsigned mask, int nE, int nF, int64_t* rows, int64_t* nnz) {
  const Segs S = make_segs(V, dof, mask, nE, nF);
  *rows = S.rows;
  *nnz = S.nnz;
}

cudaError_t launch_jac_pattern(int V, int dof, unsigned mask, int nE, const int32_t* edges,
                               int nF, const int32_t* F, int64_t* rp, int32_t* ci,
                               cudaStream_t s) {
  const Segs S = make_segs(V, dof, mask, nE, nF);
  k_jac_pattern<<<jgrid(S.rows), kJT, 0, s>>>(S, dof, V, edges, F, rp, ci);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t jac_values(int V, int dof, unsigned mask, int nE, const int32_t* edges,
                              int nF, const int32_t* F, const mad_terms& t, const void* x,
                              void* r, void* J, cudaStream_t s) {
  const Segs S = make_segs(V, dof, mask, nE, nF);
  const int64_t ne = (mask & MAD_TERM_SPRING) ? nE : 0;
  const int64_t nin = (mask & MAD_TERM_INERTIA) ? (int64_t)V * dof : 0;
  if (ne + nin > 0) {
    const int nbs = (int)((ne + kJT * kJE - 1) / (kJT * kJE));
    const int nbi = (int)((nin + kJT - 1) / kJT);
    const T sk = (T)std::sqrt(t.spring_k), sw = (T)std::sqrt(t.inertia_w);
    if (dof == 3)
      k_jac_edges_vertices<T, 3><<<nbs + nbi, kJT, 0, s>>>(
          S, (int)ne, nbs, nin, edges, (const T*)x, (const T*)t.spring_rest, sk,
          (const T*)t.inertia_xt, sw, (T*)r, (T*)J);
    else
      k_jac_edges_vertices<T, 2><<<nbs + nbi, kJT, 0, s>>>(
          S, (int)ne, nbs, nin, edges, (const T*)x, (const T*)t.spring_rest, sk,
          (const T*)t.inertia_xt, sw, (T*)r, (T*)J);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if ((mask & MAD_TERM_SYMDIR) && nF > 0) {
    k_jac_faces<T><<<jgrid(nF), kJT, 0, s>>>(S, nF, F, (const T*)x, (const T*)t.face_Minv,
                                            (const T*)t.face_area, (T*)r, (T*)J);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_jacobian(int dtype, int V, int dof, unsigned mask, int nE,
                            const int32_t* edges, int nF, const int32_t* F, const mad_terms& t,
                            const void* x, void* r, void* J, cudaStream_t s) {
  if (dtype == MAD_F64) return jac_values<double>(V, dof, mask, nE, edges, nF, F, t, x, r, J, s);
  return jac_values<float>(V, dof, mask, nE, edges, nF, F, t, x, r, J, s);
}

}  // namespace mad
