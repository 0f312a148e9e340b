// eval.cu -- fused evaluate / differentiate / assemble kernel, and the
// matrix-free Hessian-vector product, one CUDA block per patch.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法:
//   flowchart: patch-parallel kernel execution -> forward-mode AD in
//   registers / shared memory -> scatter-add into the global sparse g and H;
//   key design 1 (forward mode, everything local stays on chip, global traffic
//   = read the mesh + write the final sparse derivatives), key design 2 (one
//   CUDA block per patch, ribbon ghosts), key design 3 (preallocated CSR),
//   key design 4 (runtime pair blocks, accumulation points only where terms
//   meet).
//
// One block = one patch:
//  1. stage the positions of the patch's owned and ribbon vertices in shared
//     memory; lay the owned rows of H (in the CURRENT pattern, pair blocks
//     included) out contiguously in shared memory and zero them; rows that do
//     not fit the staging budget are assembled in place in global memory;
//  2. for each colour of edge terms, then of face terms: one thread per term
//     evaluates E, g_j, H_j with HyperDual numbers in registers and adds the
//     blocks that belong to owned rows into the staged rows (a colour never
//     has two terms on one owned vertex, so no atomics are needed);
//  3. one thread per owned row adds that row's runtime pair terms;
//  4. the staged rows are written to H with coalesced stores (consecutive
//     rows of consecutive vertices are consecutive in H), g likewise.
// Every block writes only its owned rows, so H and g need no zeroing pass
// and no global atomics, and the result does not depend on scheduling.
#include <algorithm>

#include "mad_internal.h"
#include "terms.cuh"

namespace mad {
namespace {

constexpr int kThreads = 256;

template <typename T>
struct KArgs {
  const PatchHdr* hdr;
  const int32_t* vgid;
  const uint32_t* meta;
  const EdgeLut* elut;
  const int32_t* eid;
  const int32_t* ecol;
  const FaceLut* flut;
  const int32_t* fcol;
  const int32_t* rp;
  const int32_t* prow;
  const int32_t* pe_col;
  const int32_t* pe_pos;
  const T* pe_rest;
  const T* x;
  const T* v;
  T* g;
  T* H;
  T* y;
  const T* L0;
  T k;
  const T* xt;
  T w;
  const T* Minv;
  const T* area;
  T kp;
  unsigned mask;
  double* epart;
  int nv_max, no_max, stage_cap;  // stage_cap in elements of T
};

template <typename T, int DOF>
struct Smem {
  T* x;      // [nv_max][DOF]
  T* v;      // [nv_max][DOF]   (HVP)
  T* g;      // [no_max][DOF]   gradient or y accumulators
  int32_t* where;  // [no_max] offset of the row in `stage`, -1 = assembled in place
  int32_t* gid;   // [no_max]
  int32_t* dst;   // [no_max] first block of the row in the current pattern
  int32_t* len;   // [no_max] row length in the current pattern
  uint32_t* meta; // [no_max]
  int32_t* pb;    // [no_max] first pair entry
  int32_t* pn;    // [no_max] pair entries
  int32_t* nins;  // [no_max] blocks inserted into the row by pairs
  double* red;    // [32]
  T* stage;       // [stage_cap]
};

__host__ __device__ inline size_t align16(size_t b) { return (b + 15) & ~size_t(15); }

template <typename T, int DOF>
__host__ __device__ size_t smem_layout(int nv_max, int no_max, int stage_cap, bool hvp,
                                       char* base, Smem<T, DOF>* s) {
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align16(o + bytes);
    return base ? base + at : nullptr;
  };
  char* px = take(sizeof(T) * nv_max * DOF);
  char* pv = hvp ? take(sizeof(T) * nv_max * DOF) : nullptr;
  char* pg = take(sizeof(T) * no_max * DOF);
  char* pwh = take(sizeof(int32_t) * no_max);
  char* pgid = take(sizeof(int32_t) * no_max);
  char* pdst = take(sizeof(int32_t) * no_max);
  char* plen = take(sizeof(int32_t) * no_max);
  char* pmeta = take(sizeof(uint32_t) * no_max);
  char* ppb = take(sizeof(int32_t) * no_max);
  char* ppn = take(sizeof(int32_t) * no_max);
  char* pins = take(sizeof(int32_t) * no_max);
  char* pred = take(sizeof(double) * 32);
  char* pst = hvp ? nullptr : take(sizeof(T) * (size_t)stage_cap);
  if (s) {
    s->x = (T*)px;
    s->v = (T*)pv;
    s->g = (T*)pg;
    s->where = (int32_t*)pwh;
    s->gid = (int32_t*)pgid;
    s->dst = (int32_t*)pdst;
    s->len = (int32_t*)plen;
    s->meta = (uint32_t*)pmeta;
    s->pb = (int32_t*)ppb;
    s->pn = (int32_t*)ppn;
    s->nins = (int32_t*)pins;
    s->red = (double*)pred;
    s->stage = (T*)pst;
  }
  return o;
}

// Position, in the current pattern's row, of the block that sits at position
// p of the mesh-pattern row.  Rows that received new pair blocks are shifted
// past those blocks (their positions are ascending in the pair entries).
__device__ __forceinline__ int row_pos(const int32_t* __restrict__ pe_pos, int pb, int pn,
                                       int nins, int p) {
  if (nins == 0) return p;
  for (int e = pb; e < pb + pn; ++e) {
    const int32_t wv = pe_pos[e];
    if ((wv & kPairNewBlock) && (wv & kPairPosMask) <= p) ++p;
  }
  return p;
}

template <int B, typename T>
__device__ __forceinline__ void add_block(T* dst, const T* blk) {
#pragma unroll
  for (int i = 0; i < B; ++i) dst[i] += blk[i];
}

template <int D, typename T>
__device__ __forceinline__ void add_block_t(T* dst, const T* blk) {  // dst += blk^T
#pragma unroll
  for (int a = 0; a < D; ++a)
#pragma unroll
    for (int b = 0; b < D; ++b) dst[a * D + b] += blk[b * D + a];
}

__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (lane == 0) red[w] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < kThreads / 32; ++i) s += red[i];
  return s;
}

// Exclusive scan of one int per thread across the block.
__device__ __forceinline__ int block_excl_scan_int(int v, int* total) {
  __shared__ int ws[kThreads / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) ws[w] = incl;
  __syncthreads();
  if (w == 0) {
    int s = lane < kThreads / 32 ? ws[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += t;
    }
    if (lane < kThreads / 32) ws[lane] = s;
  }
  __syncthreads();
  const int base = w > 0 ? ws[w - 1] : 0;
  *total = ws[kThreads / 32 - 1];
  __syncthreads();
  return base + incl - v;
}

// ---------------------------------------------------------------------------
template <typename T, int DOF, bool FULL>
__global__ void __launch_bounds__(kThreads) k_eval(const KArgs<T> A) {
  constexpr int B = DOF * DOF;
  extern __shared__ __align__(16) char smem_raw[];
  Smem<T, DOF> S;
  smem_layout<T, DOF>(A.nv_max, A.no_max, A.stage_cap, false, smem_raw, &S);
  const PatchHdr hd = A.hdr[blockIdx.x];
  const int tid = threadIdx.x;
  // pair terms are evaluated when requested; the pair layout (shifted rows)
  // applies whenever the current pattern holds pair blocks
  const bool pairs = (A.mask & MAD_TERM_PAIR) && A.prow != nullptr;
  double energy = 0.0;
  // first element of owned row r: staged in shared memory or in place in H
#define ROW(r) (S.where[r] >= 0 ? S.stage + S.where[r] : A.H + (int64_t)S.dst[r] * B)

  // ---- 1a. positions of owned + ribbon vertices --------------------------
  for (int e = tid; e < hd.nv * DOF; e += kThreads) {
    const int lv = e / DOF, c = e - lv * DOF;
    S.x[e] = A.x[(int64_t)A.vgid[hd.vbeg + lv] * DOF + c];
  }
  // ---- 1b. owned rows: destination, length, pair entries -------------------
  for (int r = tid; r < hd.no; r += kThreads) {
    const int gid = A.vgid[hd.vbeg + r];
    const uint32_t m = A.meta[hd.vbeg + r];
    const int d0 = A.rp[gid], d1 = A.rp[gid + 1];
    S.gid[r] = gid;
    S.meta[r] = m;
    S.dst[r] = d0;
    S.len[r] = d1 - d0;
    S.nins[r] = (d1 - d0) - (int)(m & 0xFFFFu);
    if (A.prow != nullptr) {
      const int p0 = A.prow[gid];
      S.pb[r] = p0;
      S.pn[r] = A.prow[gid + 1] - p0;
    } else {
      S.pb[r] = 0;
      S.pn[r] = 0;
    }
  }
  __syncthreads();
  // ---- 1c. staging layout: rows in order; rows past the budget are
  //      assembled in place in global memory ------------------------------
  __shared__ int s_staged;
  {
    const int R = (hd.no + kThreads - 1) / kThreads;
    const int r0 = min(hd.no, tid * R), r1 = min(hd.no, r0 + R);
    int sum = 0;
    for (int r = r0; r < r1; ++r) sum += S.len[r] * B;
    int total;
    int off = block_excl_scan_int(sum, &total);
    for (int r = r0; r < r1; ++r) {
      const int n = S.len[r] * B;
      S.where[r] = (off + n <= A.stage_cap) ? off : -1;
      off += n;
    }
    if (tid == 0) s_staged = min(total, A.stage_cap);
  }
  __syncthreads();
  for (int e = tid; e < s_staged; e += kThreads) S.stage[e] = T(0);
  for (int r = tid; r < hd.no; r += kThreads) {
    if (S.where[r] < 0) {
      T* row = A.H + (int64_t)S.dst[r] * B;
      for (int e = 0; e < S.len[r] * B; ++e) row[e] = T(0);
    }
  }
  __syncthreads();
  // ---- inertia initialises the diagonal and g -----------------------------
  const bool inertia = A.mask & MAD_TERM_INERTIA;
  for (int r = tid; r < hd.no; r += kThreads) {
    if (inertia) {
      T xr[DOF], xtr[DOF], Ei, gi[DOF], Hi[B];
#pragma unroll
      for (int a = 0; a < DOF; ++a) {
        xr[a] = S.x[r * DOF + a];
        xtr[a] = A.xt[(int64_t)S.gid[r] * DOF + a];
      }
      eval_inertia<T, DOF>(xr, xtr, A.w, Ei, gi, Hi);
      energy += (double)Ei;
      const int dp = row_pos(A.pe_pos, S.pb[r], S.pn[r], S.nins[r], (int)(S.meta[r] >> 16));
      add_block<B>(ROW(r) + dp * B, Hi);
#pragma unroll
      for (int a = 0; a < DOF; ++a) S.g[r * DOF + a] = gi[a];
    } else {
#pragma unroll
      for (int a = 0; a < DOF; ++a) S.g[r * DOF + a] = T(0);
    }
  }
  __syncthreads();

  // ---- 2a. edge terms (springs), colour by colour ---------------------------
  if (A.mask & MAD_TERM_SPRING) {
    for (int c = 0; c < hd.nce; ++c) {
      const int lo = A.ecol[hd.ecbeg + c], hi = A.ecol[hd.ecbeg + c + 1];
      for (int t = lo + tid; t < hi; t += kThreads) {
        const EdgeLut L = A.elut[hd.ebeg + t];
        const T L0 = A.L0[A.eid[hd.ebeg + t]];
        EdgeDerivs<T, DOF> o;
        eval_edge<T, DOF, FULL>(S.x + L.la * DOF, S.x + L.lb * DOF, L0, A.k, o);
        // each owned endpoint takes half of the term's energy
        if (L.pab != kNotOwned) {
          const int r = L.la;
          T* row = ROW(r);
          const int pb = S.pb[r], pn = S.pn[r], ni = S.nins[r];
          add_block<B>(row + row_pos(A.pe_pos, pb, pn, ni, (int)(S.meta[r] >> 16)) * B, o.Haa);
          add_block<B>(row + row_pos(A.pe_pos, pb, pn, ni, L.pab) * B, o.Hab);
#pragma unroll
          for (int a = 0; a < DOF; ++a) S.g[r * DOF + a] += o.ga[a];
          energy += 0.5 * (double)o.E;
        }
        if (L.pba != kNotOwned) {
          const int r = L.lb;
          T* row = ROW(r);
          const int pb = S.pb[r], pn = S.pn[r], ni = S.nins[r];
          add_block<B>(row + row_pos(A.pe_pos, pb, pn, ni, (int)(S.meta[r] >> 16)) * B, o.Hbb);
          add_block_t<DOF>(row + row_pos(A.pe_pos, pb, pn, ni, L.pba) * B, o.Hab);
#pragma unroll
          for (int a = 0; a < DOF; ++a) S.g[r * DOF + a] += o.gb[a];
          energy += 0.5 * (double)o.E;
        }
      }
      __syncthreads();
    }
  }
  // ---- 2b. face terms (symmetric Dirichlet, dof 2) -------------------------
  if constexpr (DOF == 2) {
    if (A.mask & MAD_TERM_SYMDIR) {
      for (int c = 0; c < hd.ncf; ++c) {
        const int lo = A.fcol[hd.fcbeg + c], hi = A.fcol[hd.fcbeg + c + 1];
        for (int t = lo + tid; t < hi; t += kThreads) {
          const FaceLut L = A.flut[hd.fbeg + t];
          T M[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) M[q] = A.Minv[(int64_t)L.fid * 4 + q];
          const T ar = A.area[L.fid];
          FaceDerivs<T> o;
          eval_symdir<T, FULL>(S.x + L.l[0] * 2, S.x + L.l[1] * 2, S.x + L.l[2] * 2, M, ar, o);
#pragma unroll
          for (int kk = 0; kk < 3; ++kk) {
            if (L.pos[kk][0] == kNotOwned) continue;
            const int r = L.l[kk];
            T* row = ROW(r);
            const int pb = S.pb[r], pn = S.pn[r], ni = S.nins[r];
#pragma unroll
            for (int m = 0; m < 3; ++m)
              add_block<4>(row + row_pos(A.pe_pos, pb, pn, ni, L.pos[kk][m]) * 4, o.H[kk][m]);
            S.g[r * 2 + 0] += o.g[2 * kk + 0];
            S.g[r * 2 + 1] += o.g[2 * kk + 1];
            energy += (double)o.E * (1.0 / 3.0);
          }
        }
        __syncthreads();
      }
    }
  }
  // ---- 3. runtime pairs: one thread per owned row ---------------------------
  if (pairs) {
    for (int r = tid; r < hd.no; r += kThreads) {
      const int pb = S.pb[r], pn = S.pn[r];
      if (pn == 0) continue;
      T* row = ROW(r);
      const int dp = row_pos(A.pe_pos, pb, pn, S.nins[r], (int)(S.meta[r] >> 16));
      for (int e = pb; e < pb + pn; ++e) {
        const int j = A.pe_col[e];
        const int pos = A.pe_pos[e] & kPairPosMask;
        T xj[DOF];
#pragma unroll
        for (int a = 0; a < DOF; ++a) xj[a] = A.x[(int64_t)j * DOF + a];
        EdgeDerivs<T, DOF> o;
        eval_edge<T, DOF, FULL>(S.x + r * DOF, xj, A.pe_rest[e], A.kp, o);
        add_block<B>(row + dp * B, o.Haa);
        add_block<B>(row + pos * B, o.Hab);
#pragma unroll
        for (int a = 0; a < DOF; ++a) S.g[r * DOF + a] += o.ga[a];
        energy += 0.5 * (double)o.E;
      }
    }
  }
  __syncthreads();
  // ---- 4. write the staged rows and g --------------------------------------
  {
    const int lane = tid & 31, wid = tid >> 5;
    for (int r = wid; r < hd.no; r += kThreads / 32) {
      if (S.where[r] < 0) continue;  // assembled in place
      const T* src = S.stage + S.where[r];
      T* dst = A.H + (int64_t)S.dst[r] * B;
      const int n = S.len[r] * B;
      for (int e = lane; e < n; e += 32) dst[e] = src[e];
    }
    for (int e = tid; e < hd.no * DOF; e += kThreads) {
      const int r = e / DOF, c = e - r * DOF;
      A.g[(int64_t)S.gid[r] * DOF + c] = S.g[e];
    }
  }
  if (A.epart) {
    const double s = block_sum(energy, S.red);
    if (tid == 0) A.epart[blockIdx.x] = s;
  }
#undef ROW
}

// ---------------------------------------------------------------------------
// y = H v restricted to the owned rows, without forming H.
template <typename T, int DOF>
__device__ __forceinline__ void mv_add(T* y, const T* Hblk, const T* vv) {
#pragma unroll
  for (int a = 0; a < DOF; ++a) {
    T s = T(0);
#pragma unroll
    for (int b = 0; b < DOF; ++b) s += Hblk[a * DOF + b] * vv[b];
    y[a] += s;
  }
}
template <typename T, int DOF>
__device__ __forceinline__ void mvt_add(T* y, const T* Hblk, const T* vv) {  // y += H^T v
#pragma unroll
  for (int a = 0; a < DOF; ++a) {
    T s = T(0);
#pragma unroll
    for (int b = 0; b < DOF; ++b) s += Hblk[b * DOF + a] * vv[b];
    y[a] += s;
  }
}

template <typename T, int DOF, bool FULL>
__global__ void __launch_bounds__(kThreads) k_hvp(const KArgs<T> A) {
  constexpr int B = DOF * DOF;
  extern __shared__ __align__(16) char smem_raw[];
  Smem<T, DOF> S;
  smem_layout<T, DOF>(A.nv_max, A.no_max, 0, true, smem_raw, &S);
  const PatchHdr hd = A.hdr[blockIdx.x];
  const int tid = threadIdx.x;
  const bool pairs = (A.mask & MAD_TERM_PAIR) && A.prow != nullptr;

  for (int e = tid; e < hd.nv * DOF; e += kThreads) {
    const int lv = e / DOF, c = e - lv * DOF;
    const int64_t gi = (int64_t)A.vgid[hd.vbeg + lv] * DOF + c;
    S.x[e] = A.x[gi];
    S.v[e] = A.v[gi];
  }
  __syncthreads();
  const bool inertia = A.mask & MAD_TERM_INERTIA;
  for (int r = tid; r < hd.no; r += kThreads) {
    const int gid = A.vgid[hd.vbeg + r];
    S.gid[r] = gid;
    if (pairs) {
      const int p0 = A.prow[gid];
      S.pb[r] = p0;
      S.pn[r] = A.prow[gid + 1] - p0;
    } else {
      S.pn[r] = 0;
    }
    T yr[DOF];
#pragma unroll
    for (int a = 0; a < DOF; ++a) yr[a] = T(0);
    if (inertia) {
      T xr[DOF], xtr[DOF], Ei, gi[DOF], Hi[B];
#pragma unroll
      for (int a = 0; a < DOF; ++a) {
        xr[a] = S.x[r * DOF + a];
        xtr[a] = A.xt[(int64_t)gid * DOF + a];
      }
      eval_inertia<T, DOF>(xr, xtr, A.w, Ei, gi, Hi);
      mv_add<T, DOF>(yr, Hi, S.v + r * DOF);
    }
#pragma unroll
    for (int a = 0; a < DOF; ++a) S.g[r * DOF + a] = yr[a];
  }
  __syncthreads();
  if (A.mask & MAD_TERM_SPRING) {
    for (int c = 0; c < hd.nce; ++c) {
      const int lo = A.ecol[hd.ecbeg + c], hi = A.ecol[hd.ecbeg + c + 1];
      for (int t = lo + tid; t < hi; t += kThreads) {
        const EdgeLut L = A.elut[hd.ebeg + t];
        const T L0 = A.L0[A.eid[hd.ebeg + t]];
        EdgeDerivs<T, DOF> o;
        eval_edge<T, DOF, FULL>(S.x + L.la * DOF, S.x + L.lb * DOF, L0, A.k, o);
        const T* va = S.v + L.la * DOF;
        const T* vb = S.v + L.lb * DOF;
        if (L.pab != kNotOwned) {
          T* yr = S.g + L.la * DOF;
          mv_add<T, DOF>(yr, o.Haa, va);
          mv_add<T, DOF>(yr, o.Hab, vb);
        }
        if (L.pba != kNotOwned) {
          T* yr = S.g + L.lb * DOF;
          mvt_add<T, DOF>(yr, o.Hab, va);
          mv_add<T, DOF>(yr, o.Hbb, vb);
        }
      }
      __syncthreads();
    }
  }
  if constexpr (DOF == 2) {
    if (A.mask & MAD_TERM_SYMDIR) {
      for (int c = 0; c < hd.ncf; ++c) {
        const int lo = A.fcol[hd.fcbeg + c], hi = A.fcol[hd.fcbeg + c + 1];
        for (int t = lo + tid; t < hi; t += kThreads) {
          const FaceLut L = A.flut[hd.fbeg + t];
          T M[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) M[q] = A.Minv[(int64_t)L.fid * 4 + q];
          FaceDerivs<T> o;
          eval_symdir<T, FULL>(S.x + L.l[0] * 2, S.x + L.l[1] * 2, S.x + L.l[2] * 2, M,
                               A.area[L.fid], o);
#pragma unroll
          for (int kk = 0; kk < 3; ++kk) {
            if (L.pos[kk][0] == kNotOwned) continue;
            T* yr = S.g + L.l[kk] * 2;
#pragma unroll
            for (int m = 0; m < 3; ++m) mv_add<T, 2>(yr, o.H[kk][m], S.v + L.l[m] * 2);
          }
        }
        __syncthreads();
      }
    }
  }
  if (pairs) {
    for (int r = tid; r < hd.no; r += kThreads) {
      const int pb = S.pb[r], pn = S.pn[r];
      for (int e = pb; e < pb + pn; ++e) {
        const int j = A.pe_col[e];
        T xj[DOF], vj[DOF];
#pragma unroll
        for (int a = 0; a < DOF; ++a) {
          xj[a] = A.x[(int64_t)j * DOF + a];
          vj[a] = A.v[(int64_t)j * DOF + a];
        }
        EdgeDerivs<T, DOF> o;
        eval_edge<T, DOF, FULL>(S.x + r * DOF, xj, A.pe_rest[e], A.kp, o);
        mv_add<T, DOF>(S.g + r * DOF, o.Haa, S.v + r * DOF);
        mv_add<T, DOF>(S.g + r * DOF, o.Hab, vj);
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < hd.no * DOF; e += kThreads) {
    const int r = e / DOF, c = e - r * DOF;
    A.y[(int64_t)S.gid[r] * DOF + c] = S.g[e];
  }
}

// Deterministic sum of the per-patch energies.
__global__ void k_energy_sum(const double* __restrict__ part, int n, double* out) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += part[i];
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
KArgs<T> make_args(const EvalLaunch& L, const mad_terms& t, const void* x, const void* v,
                   void* g, void* H, void* y, bool energy) {
  KArgs<T> A;
  A.hdr = L.hdr;
  A.vgid = L.vgid;
  A.meta = L.meta;
  A.elut = L.elut;
  A.eid = L.eid;
  A.ecol = L.ecol;
  A.flut = L.flut;
  A.fcol = L.fcol;
  A.rp = L.rp;
  A.prow = L.prow;
  A.pe_col = L.pe_col;
  A.pe_pos = L.pe_pos;
  A.pe_rest = (const T*)L.pe_rest;
  A.x = (const T*)x;
  A.v = (const T*)v;
  A.g = (T*)g;
  A.H = (T*)H;
  A.y = (T*)y;
  A.L0 = (const T*)t.spring_rest;
  A.k = (T)t.spring_k;
  A.xt = (const T*)t.inertia_xt;
  A.w = (T)t.inertia_w;
  A.Minv = (const T*)t.face_Minv;
  A.area = (const T*)t.face_area;
  A.kp = (T)t.pair_k;
  A.mask = t.mask;
  A.epart = energy ? L.epart : nullptr;
  A.nv_max = L.nv_max;
  A.no_max = L.no_max;
  A.stage_cap = L.stage_cap * L.dof * L.dof;
  return A;
}

template <typename T, int DOF>
cudaError_t run_eval(const EvalLaunch& L, const mad_terms& t, const void* x, void* g,
                     void* H, double* energy, cudaStream_t s) {
  KArgs<T> A = make_args<T>(L, t, x, nullptr, g, H, nullptr, energy != nullptr);
  const size_t smem = eval_smem_bytes(L, false);
  if (t.flags & MAD_EVAL_FULL_STENCIL_AD)
    k_eval<T, DOF, true><<<L.n_patches, kThreads, smem, s>>>(A);
  else
    k_eval<T, DOF, false><<<L.n_patches, kThreads, smem, s>>>(A);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !energy) return e;
  k_energy_sum<<<1, 1024, 0, s>>>(L.epart, L.n_patches, energy);
  return cudaGetLastError();
}

template <typename T, int DOF>
cudaError_t run_hvp(const EvalLaunch& L, const mad_terms& t, const void* x, const void* v,
                    void* y, cudaStream_t s) {
  KArgs<T> A = make_args<T>(L, t, x, v, nullptr, nullptr, y, false);
  const size_t smem = eval_smem_bytes(L, true);
  if (t.flags & MAD_EVAL_FULL_STENCIL_AD)
    k_hvp<T, DOF, true><<<L.n_patches, kThreads, smem, s>>>(A);
  else
    k_hvp<T, DOF, false><<<L.n_patches, kThreads, smem, s>>>(A);
  return cudaGetLastError();
}

template <typename T, int DOF>
cudaError_t set_limits(size_t bytes) {
  cudaError_t e;
  e = cudaFuncSetAttribute(k_eval<T, DOF, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_eval<T, DOF, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_hvp<T, DOF, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)bytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_hvp<T, DOF, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes);
}

}  // namespace

size_t eval_smem_bytes(const EvalLaunch& L, bool hvp) {
  const int B = L.dof * L.dof;
  if (L.dtype == MAD_F64) {
    if (L.dof == 2)
      return smem_layout<double, 2>(L.nv_max, L.no_max, L.stage_cap * B, hvp, nullptr, nullptr);
    return smem_layout<double, 3>(L.nv_max, L.no_max, L.stage_cap * B, hvp, nullptr, nullptr);
  }
  if (L.dof == 2)
    return smem_layout<float, 2>(L.nv_max, L.no_max, L.stage_cap * B, hvp, nullptr, nullptr);
  return smem_layout<float, 3>(L.nv_max, L.no_max, L.stage_cap * B, hvp, nullptr, nullptr);
}

cudaError_t eval_set_smem_limits(int dtype, int dof, size_t bytes) {
  if (dtype == MAD_F64) return dof == 2 ? set_limits<double, 2>(bytes) : set_limits<double, 3>(bytes);
  return dof == 2 ? set_limits<float, 2>(bytes) : set_limits<float, 3>(bytes);
}

cudaError_t launch_eval(const EvalLaunch& L, const mad_terms& t, const void* x, void* g,
                        void* H, double* energy, cudaStream_t s) {
  if (L.n_patches == 0) {
    if (energy) return cudaMemsetAsync(energy, 0, sizeof(double), s);
    return cudaSuccess;
  }
  if (L.dtype == MAD_F64)
    return L.dof == 2 ? run_eval<double, 2>(L, t, x, g, H, energy, s)
                      : run_eval<double, 3>(L, t, x, g, H, energy, s);
  return L.dof == 2 ? run_eval<float, 2>(L, t, x, g, H, energy, s)
                    : run_eval<float, 3>(L, t, x, g, H, energy, s);
}

cudaError_t launch_hvp(const EvalLaunch& L, const mad_terms& t, const void* x, const void* v,
                       void* y, cudaStream_t s) {
  if (L.n_patches == 0) return cudaSuccess;
  if (L.dtype == MAD_F64)
    return L.dof == 2 ? run_hvp<double, 2>(L, t, x, v, y, s) : run_hvp<double, 3>(L, t, x, v, y, s);
  return L.dof == 2 ? run_hvp<float, 2>(L, t, x, v, y, s) : run_hvp<float, 3>(L, t, x, v, y, s);
}

}  // namespace mad
