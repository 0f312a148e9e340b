// noalloc.cu -- energy evaluation that allocates no memory at all.
//
// mad_eval computes the total energy with one partial sum per CUDA block,
// kept in scratch memory that mad_create allocates in the context, and a
// final deterministic sum.  mad_energy_noalloc is the same reduction for
// callers that cannot allocate device memory and so have no context: the
// per-block partial sums live in a file-scope device array of fixed size.
// The caller passes every input (device pointers) and the output.
#include <cuda_runtime.h>

#include <mutex>

#include "mad_internal.h"
#include "terms.cuh"

namespace mad {
namespace {

constexpr int kNaThreads = 256;
// One partial sum per block of 256 terms: at most kNaMaxBlocks blocks, so at
// most kNaMaxBlocks * 256 terms (springs + vertices + faces + pairs) per call.
constexpr int kNaMaxBlocks = 65536;
constexpr int kNaMaxDevices = 64;

// Shared by every call on a device; each call overwrites the slots it uses.
static __device__ __align__(256) double g_partials[kNaMaxBlocks];

double* g_partials_addr[kNaMaxDevices] = {};
std::mutex g_setup_mutex;

// Device address of g_partials on the current device (host code must not
// use the symbol itself as an address).  A call on a stream that is not
// being captured looks the address up again, so a context created anew on
// the device (after cudaDeviceReset) is picked up; a call under capture
// takes the address the last uncaptured call found.
cudaError_t partials_address(cudaStream_t s, double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNaMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (cs == cudaStreamCaptureStatusNone || !g_partials_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_partials);
    if (e != cudaSuccess) return e;
    g_partials_addr[dev] = (double*)p;
  }
  *out = g_partials_addr[dev];
  return cudaSuccess;
}

// A vertex index the term may read: in [0, V).  A term with any other index
// is skipped and contributes a NaN, so the returned energy shows it.
__device__ __forceinline__ bool vok(int v, int V) { return (unsigned)v < (unsigned)V; }

template <typename T>
struct NaArgs {
  int V, nE, nF, nP;
  const T* x;
  const int32_t* edges;
  const T* L0;
  T k;
  const T* xt;
  T w;
  const int32_t* F;
  const T* Minv;
  const T* area;
  const int32_t* pairs;
  const T* prest;
  T kp;
  T ka;
  unsigned mask;
  double* partials;
};

// Terms are numbered springs, then vertices, then faces, then pairs; thread
// t evaluates term t.
template <typename T, int DOF>
__global__ void __launch_bounds__(kNaThreads) k_energy_terms(const NaArgs<T> A) {
  const int64_t t = (int64_t)blockIdx.x * kNaThreads + threadIdx.x;
  const int64_t nS = (A.mask & MAD_TERM_SPRING) ? A.nE : 0;
  const int64_t nI = (A.mask & MAD_TERM_INERTIA) ? A.V : 0;
  const int64_t nFc = ((DOF == 2 && (A.mask & (MAD_TERM_SYMDIR | MAD_TERM_ARAP))) ||
                       (DOF == 3 && (A.mask & MAD_TERM_AREA)))
                          ? A.nF
                          : 0;
  const int64_t nPr = (A.mask & MAD_TERM_PAIR) ? A.nP : 0;
  double e = 0.0;
  const double bad = __longlong_as_double(0x7FF8000000000000LL);  // quiet NaN
  if (t < nS) {
    const int a = A.edges[2 * t], b = A.edges[2 * t + 1];
    if (vok(a, A.V) && vok(b, A.V)) {
      T d[DOF];
#pragma unroll
      for (int c = 0; c < DOF; ++c) d[c] = A.x[(int64_t)a * DOF + c] - A.x[(int64_t)b * DOF + c];
      e = (double)spring_energy(d, A.L0[t], A.k);
    } else {
      e = bad;
    }
  } else if (t < nS + nI) {
    const int64_t i = t - nS;
    T s = T(0);
#pragma unroll
    for (int c = 0; c < DOF; ++c) s += sq(A.x[i * DOF + c] - A.xt[i * DOF + c]);
    e = (double)(s * (T(0.5) * A.w));
  } else if (t < nS + nI + nFc) {
    const int64_t f = t - nS - nI;
    const int c0 = A.F[3 * f], c1 = A.F[3 * f + 1], c2 = A.F[3 * f + 2];
    if (!(vok(c0, A.V) && vok(c1, A.V) && vok(c2, A.V))) {
      e = bad;
    } else if constexpr (DOF == 2) {
      const T* u0 = A.x + (int64_t)c0 * 2;
      const T* u1 = A.x + (int64_t)c1 * 2;
      const T* u2 = A.x + (int64_t)c2 * 2;
      const T* M = A.Minv + 4 * f;
      T j[4];
#pragma unroll
      for (int al = 0; al < 2; ++al)
#pragma unroll
        for (int ga = 0; ga < 2; ++ga)
          j[2 * al + ga] = (u1[al] - u0[al]) * M[ga] + (u2[al] - u0[al]) * M[2 + ga];
      e = (double)face2_energy(j, A.area[f], face2_kind(A.mask));
    } else {
      const T* u0 = A.x + (int64_t)c0 * 3;
      const T* u1 = A.x + (int64_t)c1 * 3;
      const T* u2 = A.x + (int64_t)c2 * 3;
      T e1[3], e2[3];
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        e1[a] = u1[a] - u0[a];
        e2[a] = u2[a] - u0[a];
      }
      e = (double)area_energy(e1, e2, A.area[f], A.ka);
    }
  } else if (t < nS + nI + nFc + nPr) {
    const int64_t p = t - nS - nI - nFc;
    const int a = A.pairs[2 * p], b = A.pairs[2 * p + 1];
    if (vok(a, A.V) && vok(b, A.V)) {
      T d[DOF];
#pragma unroll
      for (int c = 0; c < DOF; ++c) d[c] = A.x[(int64_t)a * DOF + c] - A.x[(int64_t)b * DOF + c];
      e = (double)spring_energy(d, A.prest[p], A.kp);
    } else {
      e = bad;
    }
  }
  __shared__ double red[kNaThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) e += __shfl_down_sync(0xffffffffu, e, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = e;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < kNaThreads / 32; ++i) s += red[i];
    A.partials[blockIdx.x] = s;  // every slot below gridDim.x is written
  }
}

__global__ void k_energy_final(const double* __restrict__ partials, int n, double* out) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += partials[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    *out = t;
  }
}

template <typename T>
cudaError_t run(const NaArgs<T>& A, int dof, int blocks, double* energy, cudaStream_t s) {
  if (blocks > 0) {
    if (dof == 2)
      k_energy_terms<T, 2><<<blocks, kNaThreads, 0, s>>>(A);
    else
      k_energy_terms<T, 3><<<blocks, kNaThreads, 0, s>>>(A);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  k_energy_final<<<1, 1024, 0, s>>>(A.partials, blocks, energy);
  return cudaGetLastError();
}

}  // namespace
}  // namespace mad

extern "C" mad_status mad_energy_noalloc(int32_t V, int32_t dof, mad_dtype dt, const void* x,
                                         const mad_terms* t, int32_t nE, const int32_t* edges,
                                         int32_t nF, const int32_t* F, int32_t nP,
                                         const int32_t* pairs, const void* pair_rest,
                                         double* energy, void* stream) {
  if (V < 0 || nE < 0 || nF < 0 || nP < 0 || (dof != 2 && dof != 3) ||
      (dt != MAD_F32 && dt != MAD_F64) || !t || !energy) {
    return MAD_ERR_INVALID_ARG;
  }
  const unsigned known = MAD_TERM_SPRING | MAD_TERM_INERTIA | MAD_TERM_SYMDIR | MAD_TERM_PAIR |
                         MAD_TERM_AREA | MAD_TERM_ARAP | MAD_TERM_VF;
  if (t->mask & ~known) {
    return MAD_ERR_INVALID_ARG;
  }
  if (t->mask & MAD_TERM_VF) {
    return MAD_ERR_UNIMPLEMENTED;
  }
  const bool sp = (t->mask & MAD_TERM_SPRING) && nE > 0;
  const bool in = (t->mask & MAD_TERM_INERTIA) && V > 0;
  const bool sd = (t->mask & MAD_TERM_SYMDIR) && nF > 0;
  const bool rp = (t->mask & MAD_TERM_ARAP) && nF > 0;
  const bool ar = (t->mask & MAD_TERM_AREA) && nF > 0;
  const bool fa = sd || rp || ar;
  const bool pa = (t->mask & MAD_TERM_PAIR) && nP > 0;
  if (((t->mask & (MAD_TERM_SYMDIR | MAD_TERM_ARAP)) && dof != 2) ||
      ((t->mask & MAD_TERM_AREA) && dof != 3)) {
    return MAD_ERR_UNIMPLEMENTED;
  }
  if ((V > 0 && !x) || (sp && (!edges || !t->spring_rest)) || (in && !t->inertia_xt) ||
      ((sd || rp) && (!F || !t->face_Minv || !t->face_area)) || (ar && (!F || !t->face_area)) ||
      (pa && (!pairs || !pair_rest))) {
    return MAD_ERR_INVALID_ARG;
  }
  const int64_t terms = (sp ? (int64_t)nE : 0) + (in ? (int64_t)V : 0) + (fa ? (int64_t)nF : 0) +
                        (pa ? (int64_t)nP : 0);
  const int64_t blocks = (terms + mad::kNaThreads - 1) / mad::kNaThreads;
  if (blocks > mad::kNaMaxBlocks) {
    return MAD_ERR_CAPACITY;
  }
  double* partials = nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = mad::partials_address(s, &partials);
  if (e != cudaSuccess) {
    return MAD_ERR_CUDA;
  }
  const unsigned mask = (sp ? MAD_TERM_SPRING : 0u) | (in ? MAD_TERM_INERTIA : 0u) |
                        (sd ? MAD_TERM_SYMDIR : 0u) | (rp ? MAD_TERM_ARAP : 0u) |
                        (ar ? MAD_TERM_AREA : 0u) |
                        (pa ? MAD_TERM_PAIR : 0u);
  if (dt == MAD_F64) {
    mad::NaArgs<double> A{V, nE, nF, nP, (const double*)x, edges, (const double*)t->spring_rest,
                     t->spring_k, (const double*)t->inertia_xt, t->inertia_w, F,
                     (const double*)t->face_Minv, (const double*)t->face_area, pairs,
                     (const double*)pair_rest, t->pair_k, t->area_k, mask, partials};
    e = mad::run(A, dof, (int)blocks, energy, s);
  } else {
    mad::NaArgs<float> A{V, nE, nF, nP, (const float*)x, edges, (const float*)t->spring_rest,
                    (float)t->spring_k, (const float*)t->inertia_xt, (float)t->inertia_w, F,
                    (const float*)t->face_Minv, (const float*)t->face_area, pairs,
                    (const float*)pair_rest, (float)t->pair_k, (float)t->area_k, mask,
                    partials};
    e = mad::run(A, dof, (int)blocks, energy, s);
  }
  if (e != cudaSuccess) {
    return MAD_ERR_CUDA;
  }
  return MAD_OK;
}

