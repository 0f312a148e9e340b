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
//   key design 4 (runtime pair blocks).
//
// One block = one patch, one thread = one owned vertex (= one Hessian row):
//  1. prologue: every global load the patch needs is issued before the only
//     barrier: positions of owned + ribbon vertices into shared memory; per
//     row its place in H, its row slots (column, edge id) and their rest
//     lengths, its inertia target and pair entries;
//  2. per row, in registers: the inertia term, then every edge term of the
//     row (HyperDual AD); the off-diagonal block of each edge is stored into
//     the row staged in shared memory (the edge is the block's only mesh
//     contributor), the diagonal block and the gradient accumulate in
//     registers (the gather form of g = sum S^T g_j, H = sum S^T H_j S_j:
//     each edge term is evaluated once per owned endpoint);
//     [face terms are scattered colour by colour: no two faces of a colour
//     share an owned vertex, so the adds need no atomics];
//  3. per row: runtime pair terms, then the diagonal block;
//  4. write-back: consecutive owned vertices have consecutive rows in H
//     ("runs"); each run was staged contiguously at the same offset modulo
//     16 bytes as in H and leaves with one 1-D bulk (TMA) copy.
// A block writes only its owned rows: no zeroing pass over H, no global
// atomics, and results that do not depend on scheduling.
#include <algorithm>

#include "mad_internal.h"
#include "terms.cuh"

namespace mad {
namespace {

// Asynchronous copies of single elements from global to shared memory
// (cp.async, 4 or 8 bytes): the staging of a patch's positions is issued in
// one go, without a register round trip per element, and is in flight while
// the thread loads its row's tables; cp_async_wait_all() then waits for the
// thread's own copies (a block barrier after it publishes them to all).
template <typename T>
__device__ __forceinline__ void cp_async_elem(T* sdst, const T* gsrc) {
  static_assert(sizeof(T) == 4 || sizeof(T) == 8, "4- or 8-byte elements");
  const uint32_t sa = (uint32_t)__cvta_generic_to_shared(sdst);
  if constexpr (sizeof(T) == 4)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sa), "l"(gsrc) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

constexpr int kThreads = 256;
constexpr int kUnr = 8;  // row slots loaded and evaluated together
#ifndef MAD_EVAL_MIN_BLOCKS
#define MAD_EVAL_MIN_BLOCKS 2  // resident blocks per SM the register budget targets
#endif

template <typename T>
struct KArgs {
  const PatchHdr* hdr;
  const int32_t* vgid;
  const uint2* meta;
  const uint32_t* runs;
  const EdgeLut* elut;
  const int32_t* eid;
  const int32_t* ecol;
  const FaceLut* flut;
  const int32_t* fcol;
  const uint16_t* slot_lidx;
  const int32_t* slot_eid;
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
  unsigned flags;
  double* epart;
  int nv_max, no_max, stage_cap, rho;  // stage_cap in elements of T
};

template <typename T, int DOF>
struct Smem {
  T* x;        // [nv_max][DOF] positions of owned + ribbon vertices
  T* v;        // [nv_max][DOF] HVP direction
  T* g;        // [no_max][DOF] gradient (or y) of owned rows
  T* dacc;     // [no_max][DOF(DOF+1)/2] diagonal blocks (colour-phase modes)
  int32_t* where;  // [no_max] staged offset of the row, -1 = in place in H
  int32_t* dst;    // [no_max] first block of the row in the current pattern
  int32_t* len;    // [no_max] row length in the current pattern
  int32_t* gid;    // [no_max]
  double* red;     // [32]
  T* stage;        // [stage_cap]
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
  char* pd = hvp ? nullptr : take(sizeof(T) * no_max * Tri<DOF>::size);
  char* pwh = take(sizeof(int32_t) * no_max);
  char* pdst = take(sizeof(int32_t) * no_max);
  char* plen = take(sizeof(int32_t) * no_max);
  char* pgid = take(sizeof(int32_t) * no_max);
  char* pred = take(sizeof(double) * 32);
  char* pst = hvp ? nullptr : take(sizeof(T) * (size_t)stage_cap);
  if (s) {
    s->x = (T*)px;
    s->v = (T*)pv;
    s->g = (T*)pg;
    s->dacc = (T*)pd;
    s->where = (int32_t*)pwh;
    s->dst = (int32_t*)pdst;
    s->len = (int32_t*)plen;
    s->gid = (int32_t*)pgid;
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

// Colour of term t (terms are sorted by colour; col has ncol+1 offsets).
__device__ __forceinline__ int colour_of(const int32_t* __restrict__ col, int ncol, int t) {
  int c = 0;
  while (c + 1 < ncol && col[c + 1] <= t) ++c;
  return c;
}

// ---- 1-D bulk (TMA) stores from shared to global memory -------------------
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  const uint32_t sa = (uint32_t)__cvta_generic_to_shared(ssrc);
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(sa), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_and_wait_read() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Per-row state the prologue loads (one owned row per thread).
template <typename T>
struct RowIn {
  int gid = 0, blen = 0, dpos = 0, q = 0, run = 0;
  int d0 = 0, d1 = 0, dq = 0;  // row start / end, run start in the pattern
  int pb = 0, pn = 0;          // pair entries
  int lb[kUnr];                // first kUnr slots: column local index (-1 none)
  T l0[kUnr];                  // ... and edge rest length
};

template <typename T, int DOF>
__device__ __forceinline__ void load_row(const KArgs<T>& A, const PatchHdr& hd, int r,
                                         bool springs, bool pairs_layout, RowIn<T>& in) {
  in.gid = A.vgid[hd.vbeg + r];
  const uint2 m = A.meta[hd.vbeg + r];
  in.blen = (int)(m.x & 0xFFFFu);
  in.dpos = (int)(m.x >> 16);
  in.q = (int)(m.y & 0xFFFFu);
  in.run = (int)(m.y >> 16);
  int eidv[kUnr];
  const int so = hd.sbeg + r * hd.stride;
#pragma unroll
  for (int j = 0; j < kUnr; ++j) {
    in.lb[j] = -1;
    eidv[j] = -1;
    if (springs && j < hd.stride) {
      const uint16_t lj = A.slot_lidx[so + j];
      eidv[j] = A.slot_eid[so + j];
      in.lb[j] = (lj == kNoSlot || eidv[j] < 0) ? -1 : (int)lj;
    }
  }
  in.d0 = A.rp[in.gid];
  in.d1 = A.rp[in.gid + 1];
  in.dq = A.rp[in.gid - (r - in.q)];  // the run's vertices have consecutive ids
#pragma unroll
  for (int j = 0; j < kUnr; ++j)
    if (in.lb[j] >= 0) in.l0[j] = A.L0[eidv[j]];
  if (pairs_layout) {
    in.pb = A.prow[in.gid];
    in.pn = A.prow[in.gid + 1] - in.pb;
  }
}

// Staging room per row: (stride + rho) blocks rounded up to 16 bytes, so that
// every run window below starts on a 16-byte boundary.
__host__ __device__ inline int row_stage_elems(int stride, int rho, int dof, int esz) {
  const int vec = 16 / esz;
  return (((stride + rho) * dof * dof + vec - 1) / vec) * vec;
}

// Staged offset of the row (or -1 to assemble it in place): the run's window
// starts at q*RS + run*VEC (16-byte aligned) and holds the run's rows
// contiguously from the same offset modulo 16 bytes as in H, so the
// write-back's bulk copy has both ends 16-byte aligned; the window holds the
// run when its rows have at most stride + rho blocks each.
template <typename T, int DOF>
__device__ __forceinline__ int stage_offset(const KArgs<T>& A, const PatchHdr& hd,
                                            const RowIn<T>& in) {
  constexpr int B = DOF * DOF;
  constexpr int VEC = 16 / (int)sizeof(T);
  const int RS = row_stage_elems(hd.stride, A.rho, DOF, (int)sizeof(T));
  const int mis = (int)(((uintptr_t)(A.H + (int64_t)in.dq * B) / sizeof(T)) % VEC);
  if (A.rho > 0 || in.d1 - in.d0 > hd.stride) {  // rows may outgrow the window
    const uint32_t rn = A.runs[hd.rbeg + in.run];
    const int rows = (int)(rn >> 16);
    if (mis + (in.d1 - in.dq) * B > rows * RS) return -1;
  }
  return in.q * RS + in.run * VEC + mis + (in.d0 - in.dq) * B;
}

// The row's edge terms (gather): every mesh-pattern block of the row except
// the diagonal is one edge (r, b).  on_term(R, p, lb) gets the derivatives of
// the term at slot p with column local index lb.
template <typename T, int DOF, bool FULL, typename OnTerm>
__device__ __forceinline__ void gather_row_edges(const KArgs<T>& A, const PatchHdr& hd,
                                                 const T* sx, int r, const RowIn<T>& in,
                                                 OnTerm on_term) {
  const T* xr = sx + r * DOF;
#pragma unroll
  for (int j = 0; j < kUnr; ++j) {
    if (in.lb[j] < 0) continue;
    EdgeRes<T, DOF, FULL> R;
    eval_edge_res<T, DOF, FULL>(xr, sx + in.lb[j] * DOF, in.l0[j], A.k, R);
    on_term(R, j, in.lb[j]);
  }
  // rows longer than kUnr (valence >= kUnr): the rest, kUnr at a time
  const int so = hd.sbeg + r * hd.stride;
  for (int p0 = kUnr; p0 < in.blen; p0 += kUnr) {
    int lb[kUnr];
    T l0[kUnr];
#pragma unroll
    for (int j = 0; j < kUnr; ++j) {
      const int p = p0 + j;
      lb[j] = -1;
      if (p < in.blen && p != in.dpos) {
        lb[j] = A.slot_lidx[so + p];
        l0[j] = A.L0[A.slot_eid[so + p]];
      }
    }
#pragma unroll
    for (int j = 0; j < kUnr; ++j) {
      if (lb[j] < 0) continue;
      EdgeRes<T, DOF, FULL> R;
      eval_edge_res<T, DOF, FULL>(xr, sx + lb[j] * DOF, l0[j], A.k, R);
      on_term(R, p0 + j, lb[j]);
    }
  }
}

// ---------------------------------------------------------------------------
// GENERAL = false: edge terms gathered per row, inertia and pairs only (no
// colour phases); GENERAL = true adds the scatter-mode edges and face terms.
template <typename T, int DOF, bool FULL, bool GENERAL>
__global__ void __launch_bounds__(kThreads, MAD_EVAL_MIN_BLOCKS) k_eval(const KArgs<T> A) {
  constexpr int B = DOF * DOF;
  constexpr int TD = Tri<DOF>::size;
  constexpr int VEC = 16 / (int)sizeof(T);
  constexpr int MAXT = FULL ? 1 : 4;  // scatter mode: terms per thread per chunk
  constexpr int CHUNK = kThreads * MAXT;
  extern __shared__ __align__(16) char smem_raw[];
  Smem<T, DOF> S;
  smem_layout<T, DOF>(A.nv_max, A.no_max, A.stage_cap, false, smem_raw, &S);
  const PatchHdr hd = A.hdr[blockIdx.x];
  const int tid = threadIdx.x;
  const bool pairs_layout = A.prow != nullptr;  // the pattern holds pair blocks
  const bool pairs = (A.mask & MAD_TERM_PAIR) && pairs_layout;
  const bool springs = (A.mask & MAD_TERM_SPRING) && hd.ne > 0;
  const bool gather = springs && !(A.flags & MAD_EVAL_EDGE_SCATTER);
  const bool scatter = GENERAL && springs && !gather;
  const bool faces = GENERAL && DOF == 2 && (A.mask & MAD_TERM_SYMDIR) && hd.nf > 0;
  const bool inertia = A.mask & MAD_TERM_INERTIA;
  // Every off-diagonal mesh block of a row belongs to exactly one edge, so
  // when the gathered springs write a row first they store its blocks and the
  // row needs no zeroing; blocks inserted by pairs, and every block when the
  // springs do not store, start from zero.
  const bool zero_rows = pairs_layout || !gather;
  const bool colour_phases = scatter || faces;
  double energy = 0.0;

  // ---- 1. prologue: all global loads of the patch --------------------------
  // the positions of the owned and ribbon vertices, staged by cp.async
  for (int lv = tid; lv < hd.nv; lv += kThreads) {
    const int64_t gv = (int64_t)A.vgid[hd.vbeg + lv] * DOF;
#pragma unroll
    for (int c = 0; c < DOF; ++c) cp_async_elem<T>(&S.x[lv * DOF + c], &A.x[gv + c]);
  }
  RowIn<T> in;
  const bool has_row = tid < hd.no;
  if (has_row) load_row<T, DOF>(A, hd, tid, gather, pairs_layout, in);
  T xt[DOF];
  if (has_row && inertia) {
#pragma unroll
    for (int a = 0; a < DOF; ++a) xt[a] = A.xt[(int64_t)in.gid * DOF + a];
  }
  int where = -1;
  if (has_row) {
    where = stage_offset<T, DOF>(A, hd, in);
    S.where[tid] = where;
    S.dst[tid] = in.d0;
    S.len[tid] = in.d1 - in.d0;
    S.gid[tid] = in.gid;
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- 2. per row: inertia, then the row's edge terms (gather mode) --------
  const int nins = in.d1 - in.d0 - in.blen;
  T* row = has_row ? (where >= 0 ? S.stage + where : A.H + (int64_t)in.d0 * B) : nullptr;
  T acc[TD], gr[DOF];
  if (has_row) {
    if (zero_rows)
      for (int e = 0; e < (in.d1 - in.d0) * B; ++e) row[e] = T(0);
    if (inertia) {
      T Ei, Hi[B];
      eval_inertia<T, DOF>(S.x + tid * DOF, xt, A.w, Ei, gr, Hi);
      energy += (double)Ei;
#pragma unroll
      for (int a = 0; a < DOF; ++a)
#pragma unroll
        for (int b = a; b < DOF; ++b) acc[Tri<DOF>::idx(a, b)] = Hi[a * DOF + b];
    } else {
#pragma unroll
      for (int a = 0; a < DOF; ++a) gr[a] = T(0);
#pragma unroll
      for (int q = 0; q < TD; ++q) acc[q] = T(0);
    }
    if (gather) {
      gather_row_edges<T, DOF, FULL>(
          A, hd, S.x, tid, in, [&](const EdgeRes<T, DOF, FULL>& R, int p, int) {
            const int op = nins == 0 ? p : row_pos(A.pe_pos, in.pb, in.pn, nins, p);
            apply_edge_side<true>(R, 0, acc, row + op * B, gr);
            energy += 0.5 * (double)edge_energy(R);
          });
    }
  }

  // ---- 2s. colour phases (scatter-mode edges, face terms): accumulators in
  //      shared memory, one colour at a time ----------------------------------
  if (GENERAL && colour_phases) {
    if (has_row) {
#pragma unroll
      for (int q = 0; q < TD; ++q) S.dacc[tid * TD + q] = acc[q];
#pragma unroll
      for (int a = 0; a < DOF; ++a) S.g[tid * DOF + a] = gr[a];
    }
    __syncthreads();
    // row of owned local vertex r (staged or in place)
#define ROW(r) (S.where[r] >= 0 ? S.stage + S.where[r] : A.H + (int64_t)S.dst[r] * B)
    if (scatter) {
      const int32_t* col = A.ecol + hd.ecbeg;
      for (int base = 0; base < hd.ne; base += CHUNK) {
        EdgeLut L[MAXT];
        T L0v[MAXT];
#pragma unroll
        for (int k = 0; k < MAXT; ++k) {
          const int t = base + tid + k * kThreads;
          if (t < hd.ne) {
            L[k] = A.elut[hd.ebeg + t];
            L0v[k] = A.L0[A.eid[hd.ebeg + t]];
          }
        }
        EdgeRes<T, DOF, FULL> R[MAXT];
#pragma unroll
        for (int k = 0; k < MAXT; ++k) {
          const int t = base + tid + k * kThreads;
          if (t < hd.ne)
            eval_edge_res<T, DOF, FULL>(S.x + L[k].la * DOF, S.x + L[k].lb * DOF, L0v[k], A.k,
                                        R[k]);
        }
        const int last = min(hd.ne, base + CHUNK) - 1;
        const int c0 = colour_of(col, hd.nce, base), c1 = colour_of(col, hd.nce, last);
        for (int c = c0; c <= c1; ++c) {
          const int lo = col[c], hi = col[c + 1];
#pragma unroll
          for (int k = 0; k < MAXT; ++k) {
            const int t = base + tid + k * kThreads;
            if (t < lo || t >= hi) continue;
#pragma unroll
            for (int side = 0; side < 2; ++side) {
              const int pos = side == 0 ? L[k].pab : L[k].pba;
              if (pos == kNotOwned) continue;
              const int r = side == 0 ? L[k].la : L[k].lb;
              const int ni = S.len[r] - (int)(A.meta[hd.vbeg + r].x & 0xFFFFu);
              int op = pos;
              if (ni != 0) {
                const int gr0 = S.gid[r];
                const int pb0 = A.prow[gr0];
                op = row_pos(A.pe_pos, pb0, A.prow[gr0 + 1] - pb0, ni, pos);
              }
              apply_edge_side<false>(R[k], side, S.dacc + r * TD, ROW(r) + op * B, S.g + r * DOF);
              energy += 0.5 * (double)edge_energy(R[k]);
            }
          }
          __syncthreads();
        }
      }
    }
    if constexpr (DOF == 2) {
      if (faces) {
        for (int c = 0; c < hd.ncf; ++c) {
          const int lo = A.fcol[hd.fcbeg + c], hi = A.fcol[hd.fcbeg + c + 1];
          for (int t = lo + tid; t < hi; t += kThreads) {
            const FaceLut Lf = A.flut[hd.fbeg + t];
            T M[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) M[q] = A.Minv[(int64_t)Lf.fid * 4 + q];
            const T ar = A.area[Lf.fid];
            FaceDerivs<T> o;
            eval_symdir<T, FULL>(S.x + Lf.l[0] * 2, S.x + Lf.l[1] * 2, S.x + Lf.l[2] * 2, M, ar,
                                 o);
#pragma unroll
            for (int kk = 0; kk < 3; ++kk) {
              if (Lf.pos[kk][0] == kNotOwned) continue;
              const int r = Lf.l[kk];
              const int ni = S.len[r] - (int)(A.meta[hd.vbeg + r].x & 0xFFFFu);
              int pb0 = 0, pn0 = 0;
              if (ni != 0) {
                pb0 = A.prow[S.gid[r]];
                pn0 = A.prow[S.gid[r] + 1] - pb0;
              }
              T* dacc = S.dacc + r * TD;
              dacc[0] += o.H[kk][kk][0];
              dacc[1] += o.H[kk][kk][1];
              dacc[2] += o.H[kk][kk][3];
              T* rw = ROW(r);
#pragma unroll
              for (int m = 0; m < 3; ++m) {
                if (m == kk) continue;
                add_block<4>(rw + row_pos(A.pe_pos, pb0, pn0, ni, Lf.pos[kk][m]) * 4, o.H[kk][m]);
              }
              S.g[r * 2 + 0] += o.g[2 * kk + 0];
              S.g[r * 2 + 1] += o.g[2 * kk + 1];
              energy += (double)o.E * (1.0 / 3.0);
            }
          }
          __syncthreads();
        }
      }
    }
#undef ROW
    if (has_row) {
#pragma unroll
      for (int q = 0; q < TD; ++q) acc[q] = S.dacc[tid * TD + q];
#pragma unroll
      for (int a = 0; a < DOF; ++a) gr[a] = S.g[tid * DOF + a];
    }
  }

  // ---- 3. per row: runtime pairs, then the diagonal block and g -----------
  if (has_row) {
    if (pairs) {
      for (int e = in.pb; e < in.pb + in.pn; ++e) {
        const int j = A.pe_col[e];
        const int pos = A.pe_pos[e] & kPairPosMask;
        T xj[DOF];
#pragma unroll
        for (int a = 0; a < DOF; ++a) xj[a] = A.x[(int64_t)j * DOF + a];
        EdgeRes<T, DOF, FULL> Rp;
        eval_edge_res<T, DOF, FULL>(S.x + tid * DOF, xj, A.pe_rest[e], A.kp, Rp);
        apply_edge_side<false>(Rp, 0, acc, row + pos * B, gr);
        energy += 0.5 * (double)edge_energy(Rp);
      }
    }
    const int dp = row_pos(A.pe_pos, in.pb, in.pn, nins, in.dpos);
    T* d = row + dp * B;
#pragma unroll
    for (int a = 0; a < DOF; ++a)
#pragma unroll
      for (int b = 0; b < DOF; ++b)
        d[a * DOF + b] = a <= b ? acc[Tri<DOF>::idx(a, b)] : acc[Tri<DOF>::idx(b, a)];
#pragma unroll
    for (int a = 0; a < DOF; ++a) S.g[tid * DOF + a] = gr[a];
  }
  // ---- 4. write-back -------------------------------------------------------
  fence_async_smem();
  __syncthreads();
  {
    bool issued = false;
    for (int t = tid; t < hd.nruns; t += kThreads) {
      const uint32_t rn = A.runs[hd.rbeg + t];
      const int q = (int)(rn & 0xFFFFu), nr = (int)(rn >> 16);
      if (S.where[q] < 0) continue;
      int e = q;
      while (e + 1 < q + nr && S.where[e + 1] >= 0) ++e;  // staged prefix of the run
      const int n = (S.dst[e] + S.len[e] - S.dst[q]) * B;
      const T* src = S.stage + S.where[q];
      T* dst = A.H + (int64_t)S.dst[q] * B;
      const int mis = (int)(((uintptr_t)dst / sizeof(T)) % VEC);
      const int head = min(n, (VEC - mis) % VEC);
      const int body = ((n - head) / VEC) * VEC;
      for (int i = 0; i < head; ++i) dst[i] = src[i];
      for (int i = head + body; i < n; ++i) dst[i] = src[i];
      if (body > 0) {
        // the layout makes both ends 16-byte aligned; plain stores otherwise
        if ((((uintptr_t)(dst + head) | (uintptr_t)(src + head)) & 15u) == 0) {
          bulk_store(dst + head, src + head, (uint32_t)(body * sizeof(T)));
          issued = true;
        } else {
          for (int i = head; i < head + body; ++i) dst[i] = src[i];
        }
      }
    }
    for (int e = tid; e < hd.no * DOF; e += kThreads) {
      const int r = e / DOF, c = e - r * DOF;
      A.g[(int64_t)S.gid[r] * DOF + c] = S.g[e];
    }
    if (issued) bulk_commit_and_wait_read();
  }
  if (A.epart) {
    const double s = block_sum(energy, S.red);
    if (tid == 0) A.epart[blockIdx.x] = s;
  }
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

// y_a += H_aa v_a + H_ab v_b for one edge term seen from endpoint a
template <typename T, int DOF, int AD>
__device__ __forceinline__ void edge_hv(const EdgeRes<T, DOF, AD>& R, const T* va, const T* vb,
                                        T* y) {
  if constexpr (AD != kAdFull) {
    T dv[DOF];
#pragma unroll
    for (int a = 0; a < DOF; ++a) dv[a] = va[a] - vb[a];
#pragma unroll
    for (int a = 0; a < DOF; ++a) {
      T s = T(0);
#pragma unroll
      for (int b = 0; b < DOF; ++b)
        s += (a <= b ? R.K[Tri<DOF>::idx(a, b)] : R.K[Tri<DOF>::idx(b, a)]) * dv[b];
      y[a] += s;
    }
  } else {
    mv_add<T, DOF>(y, R.d.Haa, va);
    mv_add<T, DOF>(y, R.d.Hab, vb);
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
  const bool springs = (A.mask & MAD_TERM_SPRING) && hd.ne > 0;
  const bool faces = DOF == 2 && (A.mask & MAD_TERM_SYMDIR) && hd.nf > 0;
  const bool inertia = A.mask & MAD_TERM_INERTIA;

  // positions and direction of the owned and ribbon vertices, by cp.async
  for (int lv = tid; lv < hd.nv; lv += kThreads) {
    const int64_t gv = (int64_t)A.vgid[hd.vbeg + lv] * DOF;
#pragma unroll
    for (int c = 0; c < DOF; ++c) {
      cp_async_elem<T>(&S.x[lv * DOF + c], &A.x[gv + c]);
      cp_async_elem<T>(&S.v[lv * DOF + c], &A.v[gv + c]);
    }
  }
  RowIn<T> in;
  const bool has_row = tid < hd.no;
  if (has_row) load_row<T, DOF>(A, hd, tid, springs, pairs, in);
  T xt[DOF];
  if (has_row && inertia) {
#pragma unroll
    for (int a = 0; a < DOF; ++a) xt[a] = A.xt[(int64_t)in.gid * DOF + a];
  }
  if (has_row) S.gid[tid] = in.gid;
  cp_async_wait_all();
  __syncthreads();
  T yr[DOF];
#pragma unroll
  for (int a = 0; a < DOF; ++a) yr[a] = T(0);
  if (has_row) {
    const T* vr = S.v + tid * DOF;
    if (inertia) {
      T Ei, gi[DOF], Hi[B];
      eval_inertia<T, DOF>(S.x + tid * DOF, xt, A.w, Ei, gi, Hi);
      mv_add<T, DOF>(yr, Hi, vr);
    }
    if (springs) {
      gather_row_edges<T, DOF, FULL>(
          A, hd, S.x, tid, in,
          [&](const EdgeRes<T, DOF, FULL>& R, int, int lb) { edge_hv(R, vr, S.v + lb * DOF, yr); });
    }
    if (pairs) {
      for (int e = in.pb; e < in.pb + in.pn; ++e) {
        const int j = A.pe_col[e];
        T xj[DOF], vj[DOF];
#pragma unroll
        for (int a = 0; a < DOF; ++a) {
          xj[a] = A.x[(int64_t)j * DOF + a];
          vj[a] = A.v[(int64_t)j * DOF + a];
        }
        EdgeRes<T, DOF, FULL> Rp;
        eval_edge_res<T, DOF, FULL>(S.x + tid * DOF, xj, A.pe_rest[e], A.kp, Rp);
        edge_hv(Rp, vr, vj, yr);
      }
    }
  }
  if constexpr (DOF == 2) {
    if (faces) {
      if (has_row) {
        S.g[tid * 2 + 0] = yr[0];
        S.g[tid * 2 + 1] = yr[1];
      }
      __syncthreads();
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
            T* y = S.g + L.l[kk] * 2;
#pragma unroll
            for (int m = 0; m < 3; ++m) mv_add<T, 2>(y, o.H[kk][m], S.v + L.l[m] * 2);
          }
        }
        __syncthreads();
      }
      if (has_row) {
        yr[0] = S.g[tid * 2 + 0];
        yr[1] = S.g[tid * 2 + 1];
      }
    }
  }
  if (has_row) {
#pragma unroll
    for (int a = 0; a < DOF; ++a) S.g[tid * DOF + a] = yr[a];
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
  A.runs = L.runs;
  A.elut = L.elut;
  A.eid = L.eid;
  A.ecol = L.ecol;
  A.flut = L.flut;
  A.fcol = L.fcol;
  A.slot_lidx = L.slot_lidx;
  A.slot_eid = L.slot_eid;
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
  A.flags = t.flags;
  A.epart = energy ? L.epart : nullptr;
  A.nv_max = L.nv_max;
  A.no_max = L.no_max;
  A.stage_cap = L.stage_cap;
  A.rho = L.rho;
  return A;
}

template <typename T, int DOF>
cudaError_t run_eval(const EvalLaunch& L, const mad_terms& t, const void* x, void* g,
                     void* H, double* energy, cudaStream_t s) {
  KArgs<T> A = make_args<T>(L, t, x, nullptr, g, H, nullptr, energy != nullptr);
  const size_t smem = eval_smem_bytes(L, false);
  const bool general = (t.mask & MAD_TERM_SYMDIR) || (t.flags & MAD_EVAL_EDGE_SCATTER);
  const bool full = t.flags & MAD_EVAL_FULL_STENCIL_AD;
  if (full && general)
    k_eval<T, DOF, true, true><<<L.n_patches, kThreads, smem, s>>>(A);
  else if (full)
    k_eval<T, DOF, true, false><<<L.n_patches, kThreads, smem, s>>>(A);
  else if (general)
    k_eval<T, DOF, false, true><<<L.n_patches, kThreads, smem, s>>>(A);
  else
    k_eval<T, DOF, false, false><<<L.n_patches, kThreads, smem, s>>>(A);
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
  e = cudaFuncSetAttribute(k_eval<T, DOF, false, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_eval<T, DOF, true, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_eval<T, DOF, false, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_eval<T, DOF, true, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_hvp<T, DOF, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)bytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(k_hvp<T, DOF, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes);
}

}  // namespace

int eval_grid(const EvalLaunch&) { return 0; }  // one block per patch

size_t patch_stage_elems(const PatchHdr& h, int dof, int esz, int rho) {
  return (size_t)h.no * (size_t)row_stage_elems(h.stride, rho, dof, esz) +
         (size_t)h.nruns * (16 / esz);
}

size_t eval_smem_bytes(const EvalLaunch& L, bool hvp) {
  if (L.dtype == MAD_F64) {
    if (L.dof == 2)
      return smem_layout<double, 2>(L.nv_max, L.no_max, L.stage_cap, hvp, nullptr, nullptr);
    return smem_layout<double, 3>(L.nv_max, L.no_max, L.stage_cap, hvp, nullptr, nullptr);
  }
  if (L.dof == 2)
    return smem_layout<float, 2>(L.nv_max, L.no_max, L.stage_cap, hvp, nullptr, nullptr);
  return smem_layout<float, 3>(L.nv_max, L.no_max, L.stage_cap, hvp, nullptr, nullptr);
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
