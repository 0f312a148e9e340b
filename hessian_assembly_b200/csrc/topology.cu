// topology.cu -- block-CSR pattern and edge list of a triangle mesh, on the GPU.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法, key design 3: the Hessian's block sparsity is
// fully determined by mesh connectivity and the declared (1-ring)
// neighbourhoods, so it is preallocated once as CSR by a parallel analysis
// and a prefix sum for the offsets.  Steps here:
//   count   each face corner adds its two neighbours to its row (+1 diagonal)
//   scan    row offsets of the (duplicated) neighbour lists
//   fill    every corner writes its two neighbours; every row its diagonal
//   unique  per-row sort + de-duplication (the result is independent of the
//           atomic fill order, so the pattern is deterministic)
//   scan    final row_ptr;  copy -> col_idx, diagonal positions
//   edges   the upper-triangle entries (i < j) in row order = the unique
//           undirected edges sorted by (i, j)
#include "mad_internal.h"

namespace mad {
namespace {

constexpr int kT = 256;

inline unsigned grid_for(int64_t n) {
  int64_t b = (n + kT - 1) / kT;
  if (b < 1) b = 1;
  if (b > 65535LL * 8) b = 65535LL * 8;
  return (unsigned)b;
}

__global__ void k_fill_value(int32_t* a, int64_t n, int32_t v) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    a[i] = v;
}

__global__ void k_face_count(const int32_t* __restrict__ F, int64_t nF, int32_t* cnt) {
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < 3 * nF;
       c += (int64_t)gridDim.x * blockDim.x)
    atomicAdd(&cnt[F[c]], 2);
}

__global__ void k_face_fill(const int32_t* __restrict__ F, int64_t nF,
                            const int32_t* __restrict__ tptr, int32_t* cur,
                            int32_t* tmp) {
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < 3 * nF;
       c += (int64_t)gridDim.x * blockDim.x) {
    int64_t f = c / 3;
    int k = (int)(c - 3 * f);
    int32_t v = F[c];
    int32_t slot = tptr[v] + atomicAdd(&cur[v], 2);
    tmp[slot] = F[3 * f + (k + 1) % 3];
    tmp[slot + 1] = F[3 * f + (k + 2) % 3];
  }
}

// Diagonal entry in the last slot of each row, then sort + unique in place.
__global__ void k_row_unique(int V, const int32_t* __restrict__ tptr, int32_t* tmp,
                             int32_t* ulen) {
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < V;
       v += (int64_t)gridDim.x * blockDim.x) {
    int32_t b = tptr[v], e = tptr[v + 1];
    tmp[e - 1] = (int32_t)v;
    for (int32_t i = b + 1; i < e; ++i) {  // insertion sort
      int32_t key = tmp[i];
      int32_t j = i - 1;
      while (j >= b && tmp[j] > key) {
        tmp[j + 1] = tmp[j];
        --j;
      }
      tmp[j + 1] = key;
    }
    int32_t u = b;
    for (int32_t i = b; i < e; ++i)
      if (i == b || tmp[i] != tmp[u - 1]) tmp[u++] = tmp[i];
    ulen[v] = u - b;
  }
}

__global__ void k_row_copy(int V, const int32_t* __restrict__ tptr,
                           const int32_t* __restrict__ tmp, const int32_t* __restrict__ rp,
                           int32_t* ci, int32_t* diag, int32_t* up) {
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < V;
       v += (int64_t)gridDim.x * blockDim.x) {
    int32_t b = tptr[v], o = rp[v], n = rp[v + 1] - rp[v];
    int32_t d = -1;
    for (int32_t i = 0; i < n; ++i) {
      int32_t c = tmp[b + i];
      ci[o + i] = c;
      if (c == (int32_t)v) d = o + i;
    }
    diag[v] = d;
    up[v] = rp[v + 1] - 1 - d;
  }
}

__global__ void k_edges(int V, const int32_t* __restrict__ rp, const int32_t* __restrict__ ci,
                        const int32_t* __restrict__ diag, const int32_t* __restrict__ eptr,
                        int32_t* edges) {
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < V;
       v += (int64_t)gridDim.x * blockDim.x) {
    int32_t e = eptr[v];
    for (int32_t q = diag[v] + 1; q < rp[v + 1]; ++q, ++e) {
      edges[2 * (int64_t)e] = (int32_t)v;
      edges[2 * (int64_t)e + 1] = ci[q];
    }
  }
}

#define MAD_CK(x)                                              \
  do {                                                         \
    cudaError_t e_ = (x);                                      \
    if (e_ != cudaSuccess) {                                   \
      err = std::string(#x) + ": " + cudaGetErrorString(e_);   \
      goto done;                                               \
    }                                                          \
  } while (0)

}  // namespace

std::string build_pattern_gpu(int V, int nF, const int32_t* F_dev, cudaStream_t s,
                              PatternDev& out) {
  std::string err;
  int32_t *cnt = nullptr, *cur = nullptr, *tptr = nullptr, *tmp = nullptr,
          *ulen = nullptr, *up = nullptr, *eptr = nullptr, *stmp = nullptr;
  int64_t ntmp = 6 * (int64_t)nF + V;
  int32_t h[2] = {0, 0};
  out = PatternDev{nullptr, nullptr, nullptr, nullptr, 0, 0};
  if (ntmp >= (int64_t)1 << 31) return "mesh too large for int32 pattern offsets";
  MAD_CK(cudaMalloc(&cnt, sizeof(int32_t) * (V + 1)));
  MAD_CK(cudaMalloc(&cur, sizeof(int32_t) * (V + 1)));
  MAD_CK(cudaMalloc(&tptr, sizeof(int32_t) * (V + 1)));
  MAD_CK(cudaMalloc(&ulen, sizeof(int32_t) * (V + 1)));
  MAD_CK(cudaMalloc(&up, sizeof(int32_t) * (V + 1)));
  MAD_CK(cudaMalloc(&eptr, sizeof(int32_t) * (V + 1)));
  MAD_CK(cudaMalloc(&tmp, sizeof(int32_t) * (ntmp > 0 ? ntmp : 1)));
  MAD_CK(cudaMalloc(&stmp, sizeof(int32_t) * scan_tmp_elems(V)));
  MAD_CK(cudaMalloc(&out.rp, sizeof(int32_t) * (V + 1)));
  MAD_CK(cudaMalloc(&out.diag, sizeof(int32_t) * (V > 0 ? V : 1)));
  if (V > 0) {
    k_fill_value<<<grid_for(V), kT, 0, s>>>(cnt, V, 1);
    MAD_CK(cudaGetLastError());
    MAD_CK(cudaMemsetAsync(cur, 0, sizeof(int32_t) * (V + 1), s));
    if (nF > 0) {
      k_face_count<<<grid_for(3 * (int64_t)nF), kT, 0, s>>>(F_dev, nF, cnt);
      MAD_CK(cudaGetLastError());
    }
  }
  MAD_CK(scan_exclusive(cnt, tptr, V, stmp, s));
  if (nF > 0) {
    k_face_fill<<<grid_for(3 * (int64_t)nF), kT, 0, s>>>(F_dev, nF, tptr, cur, tmp);
    MAD_CK(cudaGetLastError());
  }
  if (V > 0) {
    k_row_unique<<<grid_for(V), kT, 0, s>>>(V, tptr, tmp, ulen);
    MAD_CK(cudaGetLastError());
  }
  MAD_CK(scan_exclusive(ulen, out.rp, V, stmp, s));
  MAD_CK(cudaMemcpyAsync(&h[0], out.rp + V, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  MAD_CK(cudaStreamSynchronize(s));
  out.nnzb = h[0];
  MAD_CK(cudaMalloc(&out.ci, sizeof(int32_t) * (out.nnzb > 0 ? out.nnzb : 1)));
  if (V > 0) {
    k_row_copy<<<grid_for(V), kT, 0, s>>>(V, tptr, tmp, out.rp, out.ci, out.diag, up);
    MAD_CK(cudaGetLastError());
  }
  MAD_CK(scan_exclusive(up, eptr, V, stmp, s));
  MAD_CK(cudaMemcpyAsync(&h[1], eptr + V, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  MAD_CK(cudaStreamSynchronize(s));
  out.E = h[1];
  MAD_CK(cudaMalloc(&out.edges, sizeof(int32_t) * 2 * (out.E > 0 ? out.E : 1)));
  if (V > 0) {
    k_edges<<<grid_for(V), kT, 0, s>>>(V, out.rp, out.ci, out.diag, eptr, out.edges);
    MAD_CK(cudaGetLastError());
  }
  MAD_CK(cudaStreamSynchronize(s));
done:
  cudaFree(cnt);
  cudaFree(cur);
  cudaFree(tptr);
  cudaFree(ulen);
  cudaFree(up);
  cudaFree(eptr);
  cudaFree(tmp);
  cudaFree(stmp);
  if (!err.empty()) {
    cudaFree(out.rp);
    cudaFree(out.ci);
    cudaFree(out.diag);
    cudaFree(out.edges);
    out = PatternDev{nullptr, nullptr, nullptr, nullptr, 0, 0};
  }
  return err;
}

}  // namespace mad
