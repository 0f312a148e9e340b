// pairs.cu -- GPU insertion of runtime vertex-vertex pair blocks into the
// double-buffered block CSR.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法, key design 4: interactions that appear at run
// time (contact, proximity: Op::VV) add off-diagonal Hessian blocks; the system
// decouples interaction discovery from evaluation and, with a double-buffered
// CSR and reserved storage, inserts the new nonzeros in parallel on the GPU and
// swaps the buffers, with no CPU round trip.
//
// Steps (all stream-ordered, no host synchronisation):
//   count   pair entries per row (each pair lands in the rows of both ends)
//   scan    -> prow, the per-row pair-entry offsets
//   fill    each pair writes (partner, pair id) into both rows
//   rows    per row: sort entries by (partner, pair id), merge with the mesh
//           row, give every entry the position of its block in the merged
//           row, mark the entries that create a block, count new blocks
//   scan    -> per-row block shift; capacity check on the total
//   write   new row_ptr = mesh row_ptr + shift, merged col_idx; a warp whose
//           32 rows gained nothing copies their columns as one coalesced run
//   restore on capacity overflow: the new buffer receives a copy of the
//           previous pattern and pair set instead
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

#define GRID_STRIDE(i, n)                                                    \
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (n); \
       i += (int64_t)gridDim.x * blockDim.x)

__global__ void k_pair_count(const int32_t* __restrict__ ij, int n, int V, int32_t* cnt,
                             int32_t* status) {
  GRID_STRIDE(p, n) {
    const int32_t i = ij[2 * p], j = ij[2 * p + 1];
    if (i < 0 || i >= V || j < 0 || j >= V || i == j) {
      atomicOr(status, kStatusIndex);
      continue;
    }
    atomicAdd(&cnt[i], 1);
    atomicAdd(&cnt[j], 1);
  }
}

__global__ void k_pair_fill(const int32_t* __restrict__ ij, int n, int V,
                            const int32_t* __restrict__ prow, int32_t* cur, int32_t* pe_col,
                            int32_t* pe_pid) {
  GRID_STRIDE(p, n) {
    const int32_t i = ij[2 * p], j = ij[2 * p + 1];
    if (i < 0 || i >= V || j < 0 || j >= V || i == j) continue;
    int32_t s = prow[i] + atomicAdd(&cur[i], 1);
    pe_col[s] = j;
    pe_pid[s] = (int32_t)p;
    s = prow[j] + atomicAdd(&cur[j], 1);
    pe_col[s] = i;
    pe_pid[s] = (int32_t)p;
  }
}

template <typename T>
__global__ void k_pair_rows(int V, const int32_t* __restrict__ prow,
                            const int32_t* __restrict__ base_rp,
                            const int32_t* __restrict__ base_ci, int32_t* pe_col,
                            int32_t* pe_pid, int32_t* pe_pos, T* pe_rest,
                            const T* __restrict__ rest, int32_t* newcnt) {
  GRID_STRIDE(v, V) {
    const int32_t b = prow[v], e = prow[v + 1];
    if (b == e) {
      newcnt[v] = 0;
      continue;
    }
    for (int32_t i = b + 1; i < e; ++i) {  // insertion sort by (col, pid)
      const int32_t kc = pe_col[i], kp = pe_pid[i];
      int32_t j = i - 1;
      while (j >= b && (pe_col[j] > kc || (pe_col[j] == kc && pe_pid[j] > kp))) {
        pe_col[j + 1] = pe_col[j];
        pe_pid[j + 1] = pe_pid[j];
        --j;
      }
      pe_col[j + 1] = kc;
      pe_pid[j + 1] = kp;
    }
    const int32_t r0 = base_rp[v], blen = base_rp[v + 1] - r0;
    int32_t kb = 0, kn = 0, prev_col = -1;
    bool prev_new = false;
    for (int32_t i = b; i < e; ++i) {
      const int32_t c = pe_col[i];
      const bool first = (c != prev_col);
      if (first && prev_new) ++kn;  // the previous group added one block
      while (kb < blen && base_ci[r0 + kb] < c) ++kb;
      const bool in_mesh = kb < blen && base_ci[r0 + kb] == c;
      if (first) prev_new = !in_mesh;
      pe_pos[i] = (kb + kn) | ((first && !in_mesh) ? kPairNewBlock : 0);
      pe_rest[i] = rest[pe_pid[i]];
      prev_col = c;
    }
    if (prev_new) ++kn;
    newcnt[v] = kn;
  }
}

__global__ void k_check_capacity(const int32_t* __restrict__ shift, int V, int nnzb_base,
                                 int capacity, int32_t* nnzb_out, int32_t* flag,
                                 int32_t* status) {
  const int64_t total = (int64_t)nnzb_base + shift[V];
  if (total > capacity) {
    *flag = 1;
    atomicOr(status, kStatusCapacity);
  } else {
    *flag = 0;
    *nnzb_out = (int32_t)total;
  }
}

// One warp per 32 consecutive rows.
__global__ void k_write_pattern(int V, const int32_t* __restrict__ base_rp,
                                const int32_t* __restrict__ base_ci,
                                const int32_t* __restrict__ shift,
                                const int32_t* __restrict__ newcnt,
                                const int32_t* __restrict__ prow,
                                const int32_t* __restrict__ pe_col,
                                const int32_t* __restrict__ pe_pos, const int32_t* flag,
                                int32_t* rp, int32_t* ci) {
  if (*flag) return;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t w = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; w * 32 < V;
       w += warps) {
    const int64_t v = w * 32 + lane;
    const bool valid = v < V;
    const int32_t sh = valid ? shift[v] : 0;
    const int32_t nc = valid ? newcnt[v] : 0;
    if (valid) rp[v] = base_rp[v] + sh;
    if (v == V - 1) rp[V] = base_rp[V] + shift[V];
    const unsigned any_new = __ballot_sync(0xffffffffu, nc != 0);
    if (!any_new) {
      // rows w*32 .. w*32+31 gained nothing: one contiguous shifted run
      const int64_t v0 = w * 32, v1 = v0 + 32 < V ? v0 + 32 : V;
      const int32_t s0 = __shfl_sync(0xffffffffu, sh, 0);
      const int32_t a = base_rp[v0], z = base_rp[v1];
      for (int32_t q = a + lane; q < z; q += 32) ci[q + s0] = base_ci[q];
    } else if (valid) {
      const int32_t r0 = base_rp[v], r1 = base_rp[v + 1];
      int32_t o = r0 + sh;
      int32_t kb = r0;
      for (int32_t e = prow[v]; e < prow[v + 1]; ++e) {
        if (!(pe_pos[e] & kPairNewBlock)) continue;
        const int32_t c = pe_col[e];
        while (kb < r1 && base_ci[kb] < c) ci[o++] = base_ci[kb++];
        ci[o++] = c;
      }
      while (kb < r1) ci[o++] = base_ci[kb++];
    }
  }
}

// Capacity overflow: make the new buffer a copy of the previous state.
template <typename T>
__global__ void k_restore_prev(int V, const int32_t* flag, const int32_t* prev_rp,
                               const int32_t* prev_ci, const int32_t* prev_nnzb,
                               const int32_t* prev_prow, const int32_t* prev_pe_col,
                               const int32_t* prev_pe_pos, const T* prev_pe_rest,
                               int32_t* rp, int32_t* ci, int32_t* nnzb, int32_t* prow,
                               int32_t* pe_col, int32_t* pe_pos, T* pe_rest) {
  if (*flag == 0) return;
  const int32_t nb = *prev_nnzb;
  GRID_STRIDE(i, (int64_t)V + 1) {
    rp[i] = prev_rp[i];
    prow[i] = prev_prow ? prev_prow[i] : 0;
  }
  GRID_STRIDE(i, nb) ci[i] = prev_ci[i];
  if (prev_prow) {
    const int32_t ne = prev_prow[V];
    GRID_STRIDE(i, ne) {
      pe_col[i] = prev_pe_col[i];
      pe_pos[i] = prev_pe_pos[i];
      pe_rest[i] = prev_pe_rest[i];
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *nnzb = nb;
}

#define CK(x)                              \
  do {                                     \
    cudaError_t e_ = (x);                  \
    if (e_ != cudaSuccess) return e_;      \
  } while (0)

template <typename T>
cudaError_t add_pairs_t(const PairLaunch& L, int n, const int32_t* ij, const void* rest,
                        const DynBuf& nb, const DynBuf* prev, const int32_t* base_nnzb_dev,
                        cudaStream_t s) {
  const int V = L.V;
  CK(cudaMemsetAsync(L.cnt, 0, sizeof(int32_t) * (V + 1), s));
  CK(cudaMemsetAsync(L.cur, 0, sizeof(int32_t) * (V + 1), s));
  k_pair_count<<<grid_for(n), kT, 0, s>>>(ij, n, V, L.cnt, L.status);
  CK(cudaGetLastError());
  CK(scan_exclusive(L.cnt, nb.prow, V, L.scan_tmp, s));
  k_pair_fill<<<grid_for(n), kT, 0, s>>>(ij, n, V, nb.prow, L.cur, nb.pe_col, L.pe_pid);
  CK(cudaGetLastError());
  k_pair_rows<T><<<grid_for(V), kT, 0, s>>>(V, nb.prow, L.base_rp, L.base_ci, nb.pe_col,
                                            L.pe_pid, nb.pe_pos, (T*)nb.pe_rest,
                                            (const T*)rest, L.newcnt);
  CK(cudaGetLastError());
  CK(scan_exclusive(L.newcnt, L.shift, V, L.scan_tmp, s));
  k_check_capacity<<<1, 1, 0, s>>>(L.shift, V, L.nnzb_base, L.capacity, nb.nnzb, L.flag,
                                   L.status);
  CK(cudaGetLastError());
  k_write_pattern<<<grid_for((int64_t)V), kT, 0, s>>>(V, L.base_rp, L.base_ci, L.shift,
                                                       L.newcnt, nb.prow, nb.pe_col,
                                                       nb.pe_pos, L.flag, nb.rp, nb.ci);
  CK(cudaGetLastError());
  const int64_t most = (int64_t)(L.capacity > V + 1 ? L.capacity : V + 1);
  if (prev)
    k_restore_prev<T><<<grid_for(most), kT, 0, s>>>(
        V, L.flag, prev->rp, prev->ci, prev->nnzb, prev->prow, prev->pe_col, prev->pe_pos,
        (const T*)prev->pe_rest, nb.rp, nb.ci, nb.nnzb, nb.prow, nb.pe_col, nb.pe_pos,
        (T*)nb.pe_rest);
  else
    k_restore_prev<T><<<grid_for(most), kT, 0, s>>>(
        V, L.flag, L.base_rp, L.base_ci, base_nnzb_dev, nullptr, nullptr, nullptr, nullptr,
        nb.rp, nb.ci, nb.nnzb, nb.prow, nb.pe_col, nb.pe_pos, (T*)nb.pe_rest);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_add_pairs(const PairLaunch& L, int n, const int32_t* ij, const void* rest,
                             const DynBuf& nb, const DynBuf* prev, cudaStream_t s) {
  if (L.dtype == MAD_F64)
    return add_pairs_t<double>(L, n, ij, rest, nb, prev, L.base_nnzb_dev, s);
  return add_pairs_t<float>(L, n, ij, rest, nb, prev, L.base_nnzb_dev, s);
}

}  // namespace mad
