// rows.cu -- row-streaming assembly: one warp per 32 consecutive Hessian rows,
// no block-wide barriers.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法: per-term forward-mode AD in registers (key
// design 1), assembly g = sum S^T g_j, H = sum S^T H_j S_j into the
// preallocated CSR (key design 3), runtime pair blocks (key design 4).
//
// This kernel is the gather form of that assembly.  Thread = row i (vertex
// i): it evaluates the inertia term of i, every edge term (i, b) of its row
// and every face term with i as a corner with HyperDual numbers, keeps the
// diagonal block and the gradient in registers, and writes each off-diagonal
// block once.  Each edge term is evaluated once per endpoint and each face
// term once per corner, for that corner's row only.  Rows 32w .. 32w+31 are consecutive in H, so warp w stages
// them contiguously in its own slice of shared memory, at the same offset
// modulo 16 bytes as in H, and writes them back with one 1-D bulk (TMA) copy.
// Neighbour positions are read through the L1/L2 caches.  Warps never wait
// for each other, so memory latency is hidden across the resident warps.
// A thread writes only its own row: no zeroing pass, no atomics.
//
// This header holds the kernels and their launchers; each rows_<dtype>_d<dof>.cu
// translation unit includes it and instantiates one (dtype, dof), so the
// instantiations compile in parallel.
#pragma once
#include <algorithm>
#include <type_traits>

#include "mad_internal.h"
#include "rows_common.h"
#include "terms.cuh"

namespace mad {
namespace {

constexpr int kS0Max = 8;         // most slots per row in the slot table
#ifndef MAD_ROWS_MIN_BLOCKS
#define MAD_ROWS_MIN_BLOCKS 6  // resident blocks per SM (fp32) the register budget targets
#endif
// FACES: 0 none; 1, 2 face terms (their evaluators need more registers);
// 4 installed vertex-face terms, whose branch runs on few rows and is held
// to the budget of the plain kernel (it may spill rather than lower the
// occupancy of every row)
// The area face rows (dof 3) are held to 6 blocks per SM (80 registers, no
// spill): 131.5 us against 139.9 us at 4 per 1000x1000 eval.
#ifndef MAD_ROWS_FACES3_MIN_BLOCKS
#define MAD_ROWS_FACES3_MIN_BLOCKS 6
#endif
template <typename T, int FACES, int DOF = 2>
constexpr int rows_min_blocks() {
  return (FACES == 1 || FACES == 2)
             ? (sizeof(T) == 4 ? (DOF == 3 ? MAD_ROWS_FACES3_MIN_BLOCKS : 4) : 2)
             : (sizeof(T) == 4 ? MAD_ROWS_MIN_BLOCKS : 3);
}

template <typename T>
struct RArgs {
  // installed vertex-face terms (FACES == 4): per-row entries and the term
  // pass's records (see vf.cu)
  const int32_t* vrow;
  const int32_t* vent;
  const T* vrec;
  const int32_t* fcslots;
  const int32_t* fcofl;
  const T* fhv;
  const int4* fslots;
  const int32_t* fofl_ptr;
  const int4* fofl;
  const T* Minv;
  const T* area;
  const int2* slots;
  const uint32_t* meta;
  const int32_t* ofl_ptr;
  const int2* ofl;
  // compact slot tables (rows_compact.cu; nullptr when absent): the product
  // reads its edge terms from them
  const int4* ctile;
  const uint32_t* cslots;
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
  T kp;
  T ka;  // area-preservation stiffness
  unsigned mask;
  double* epart;
  int V, s0, sf, wstage;  // wstage: staging elements per warp
};

// New-block positions of a row with inserted pair blocks, in increasing
// order: the first kRowNew in registers, the rest read from pe_pos.
constexpr int kRowNew = 4;
struct RowNew {
  int np[kRowNew];  // merged-row positions, 0x7FFFFFFF past the row's count
};

__device__ __forceinline__ void load_row_new(const int32_t* __restrict__ pe_pos, int pb, int pn,
                                             int nins, RowNew& rn) {
#pragma unroll
  for (int k = 0; k < kRowNew; ++k) rn.np[k] = 0x7FFFFFFF;
  if (nins == 0) return;
  int k = 0;
  for (int e = pb; e < pb + pn && k < kRowNew; ++e) {
    const int32_t wv = pe_pos[e];
    if (wv & kPairNewBlock) {
#pragma unroll
      for (int q = 0; q < kRowNew; ++q)
        if (q == k) rn.np[q] = wv & kPairPosMask;
      ++k;
    }
  }
}

__device__ __forceinline__ int row_pos(const int32_t* __restrict__ pe_pos, int pb, int pn,
                                       int nins, int p);

// Merged-row position of mesh-pattern position p.
__device__ __forceinline__ int row_pos_new(const RowNew& rn, const int32_t* __restrict__ pe_pos,
                                           int pb, int pn, int nins, int p) {
  if (nins > kRowNew) return row_pos(pe_pos, pb, pn, nins, p);
#pragma unroll
  for (int k = 0; k < kRowNew; ++k) p += rn.np[k] <= p;
  return p;
}

__device__ __forceinline__ int row_pos(const int32_t* __restrict__ pe_pos, int pb, int pn,
                                       int nins, int p) {
  if (nins == 0) return p;
  for (int e = pb; e < pb + pn; ++e) {
    const int32_t wv = pe_pos[e];
    if ((wv & kPairNewBlock) && (wv & kPairPosMask) <= p) ++p;
  }
  return p;
}

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

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  return v;
}

// Per-block energy partial (all threads of the block call it).
__device__ __forceinline__ void block_energy(double e, double* out) {
  __shared__ double red[kWarps];
  e = warp_sum(e);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = e;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < kWarps; ++i) s += red[i];
    *out = s;
  }
}

// 1: the product reads its edge terms from the compact slot tables when the
// context has them (0: always the wide ones)
#ifndef MAD_HVP_COMPACT
#define MAD_HVP_COMPACT 1
#endif

// Compact slot word: column minus row (low 16 bits), edge id minus the
// tile's first edge id (high 16 bits), both signed; 0 marks an empty slot.
__device__ __forceinline__ int slot_dcol(uint32_t w) { return (int)(int16_t)(w & 0xFFFFu); }
__device__ __forceinline__ int slot_deid(uint32_t w) { return (int)(int16_t)(w >> 16); }

// Calls on_term(R, col) for every edge term (i, col) of row i, read from the
// compact slot tables (positions are not needed: the product).
template <typename T, int DOF, int AD, int S0, typename OnTerm>
__device__ __forceinline__ void row_edges_c(const RArgs<T>& A, int i, int tile, int lane,
                                            const T* xi, OnTerm on_term) {
  const int4 th = A.ctile[tile];
  uint32_t sw[S0];
#pragma unroll
  for (int k = 0; k < S0; ++k)
    sw[k] = k < A.s0 ? A.cslots[(uint32_t)((tile * A.s0 + k) * 32 + lane)] : 0u;
  T xb[S0][DOF];
  T l0[S0];
#pragma unroll
  for (int k = 0; k < S0; ++k) {
    if (sw[k] == 0u) continue;
    const int col = i + slot_dcol(sw[k]);
#pragma unroll
    for (int a = 0; a < DOF; ++a) xb[k][a] = A.x[(uint32_t)(col * DOF + a)];
    l0[k] = A.L0[th.y + slot_deid(sw[k])];
  }
#pragma unroll
  for (int k = 0; k < S0; ++k) {
    if (sw[k] == 0u) continue;
    EdgeRes<T, DOF, AD> R;
    eval_edge_res<T, DOF, AD>(xi, xb[k], l0[k], A.k, R);
    on_term(R, i + slot_dcol(sw[k]));
  }
  if (((uint32_t)th.z >> lane) & 1u) {  // rows longer than the slot table
    const int o0 = A.ofl_ptr[i], o1 = A.ofl_ptr[i + 1];
    for (int q = o0; q < o1; ++q) {
      const int2 e = A.ofl[q];
      T xo[DOF];
#pragma unroll
      for (int a = 0; a < DOF; ++a) xo[a] = A.x[(uint32_t)(e.x * DOF + a)];
      EdgeRes<T, DOF, AD> R;
      eval_edge_res<T, DOF, AD>(xi, xo, A.L0[e.y], A.k, R);
      on_term(R, e.x);
    }
  }
}

// Calls on_term(R, p, col) for every edge term (i, col) of row i, where p is
// the block position of column col in the mesh-pattern row.
// S0 (compile time) >= the slot table's row width A.s0.
template <typename T, int DOF, int AD, int S0, typename OnTerm>
__device__ __forceinline__ void row_edges(const RArgs<T>& A, int i, int tile, int lane,
                                          uint32_t m, const T* xi, OnTerm on_term) {
  const int noff = (int)(m & 0xFFFFu), dpos = (int)(m >> 16);
  int2 sl[S0];
#pragma unroll
  for (int k = 0; k < S0; ++k) {
    sl[k] = make_int2(-1, -1);
    if (k < A.s0) sl[k] = A.slots[(uint32_t)((tile * A.s0 + k) * 32 + lane)];
  }
  T xb[S0][DOF];
  T l0[S0];
#pragma unroll
  for (int k = 0; k < S0; ++k) {
    if (sl[k].x < 0) continue;
#pragma unroll
    for (int a = 0; a < DOF; ++a) xb[k][a] = A.x[(uint32_t)(sl[k].x * DOF + a)];
    l0[k] = A.L0[sl[k].y];
  }
#pragma unroll
  for (int k = 0; k < S0; ++k) {
    if (sl[k].x < 0) continue;
    EdgeRes<T, DOF, AD> R;
    eval_edge_res<T, DOF, AD>(xi, xb[k], l0[k], A.k, R);
    on_term(R, k < dpos ? k : k + 1, sl[k].x);
  }
  if (noff > A.s0) {  // rows longer than the slot table: the overflow slots
    const int o0 = A.ofl_ptr[i];
    for (int k = A.s0; k < noff; ++k) {
      const int2 e = A.ofl[o0 + k - A.s0];
      T xo[DOF];
#pragma unroll
      for (int a = 0; a < DOF; ++a) xo[a] = A.x[(uint32_t)(e.x * DOF + a)];
      EdgeRes<T, DOF, AD> R;
      eval_edge_res<T, DOF, AD>(xi, xo, A.L0[e.y], A.k, R);
      on_term(R, k < dpos ? k : k + 1, e.x);
    }
  }
}

// Four consecutive values starting at p (16-byte loads when p allows them).
template <typename T>
__device__ __forceinline__ void load4(const T* __restrict__ p, T* o) {
  if ((((uintptr_t)p) & 15u) == 0) {
    if constexpr (sizeof(T) == 4) {
      const float4 v = *reinterpret_cast<const float4*>(p);
      o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else {
      const double2 a = reinterpret_cast<const double2*>(p)[0];
      const double2 b = reinterpret_cast<const double2*>(p)[1];
      o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = p[q];
  }
}

// Calls on_face(xj, xk, j, k, c, pj, pk, M, area) for every face term with
// vertex i as a corner (dof 2): j and k are the other two corners (corner
// c+1 and c+2 of the face when i is corner c), pj and pk their mesh-pattern
// block positions in row i, M the face's Dm^-1 and area its rest area.  The
// loop is not unrolled (a small body stays in the instruction cache); the
// next table entry is loaded while the current face is evaluated.
template <typename T, typename OnFace>
__device__ __forceinline__ void row_faces(const RArgs<T>& A, int i, int tile, int lane,
                                          OnFace on_face) {
  constexpr uint32_t kPm = (1u << kFacePosBits) - 1u;
  auto one = [&](const int4& e) {
    const int j = e.y, k = e.z & 0x7FFFFFFF;
    const uint32_t w = (uint32_t)e.w;
    T xj[2], xk[2], M[4];
    xj[0] = A.x[(uint32_t)(j * 2)];
    xj[1] = A.x[(uint32_t)(j * 2 + 1)];
    xk[0] = A.x[(uint32_t)(k * 2)];
    xk[1] = A.x[(uint32_t)(k * 2 + 1)];
    load4<T>(A.Minv + (uint32_t)e.x * 4u, M);
    const T ar = A.area[e.x];
    on_face(xj, xk, j, k, (int)(w & 3u), (int)((w >> 2) & kPm), (int)(w >> (2 + kFacePosBits)),
            M, ar);
  };
  const int4* p = A.fslots + (uint32_t)(tile * A.sf * 32 + lane);
  int4 e = p[0];
  bool more = false;
#pragma unroll 1
  for (int k = 0; k < A.sf; ++k) {  // a row's entries fill a prefix of its slots
    if (e.x < 0) break;
    const int4 en = k + 1 < A.sf ? p[(uint32_t)((k + 1) * 32)] : make_int4(-1, 0, 0, 0);
    if (k == kFaceRowSlots - 1) more = e.z < 0;  // the overflow mark
    one(e);
    e = en;
  }
  if (more) {
    const int o0 = A.fofl_ptr[i], o1 = A.fofl_ptr[i + 1];
#pragma unroll 1
    for (int q = o0; q < o1; ++q) one(A.fofl[q]);
  }
}

// The dof-3 face terms of row i: calls on_face(xj, xk, c, pj, pk, A0) for
// every face with vertex i as a corner (same table as row_faces).
template <typename T, typename OnFace>
__device__ __forceinline__ void row_faces3(const RArgs<T>& A, int i, int tile, int lane,
                                           OnFace on_face) {
  constexpr uint32_t kPm = (1u << kFacePosBits) - 1u;
  auto one = [&](const int4& e) {
    const int j = e.y, k = e.z & 0x7FFFFFFF;
    const uint32_t w = (uint32_t)e.w;
    T xj[3], xk[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      xj[a] = A.x[(uint32_t)(j * 3 + a)];
      xk[a] = A.x[(uint32_t)(k * 3 + a)];
    }
    on_face(xj, xk, (int)(w & 3u), (int)((w >> 2) & kPm), (int)(w >> (2 + kFacePosBits)),
            A.area[e.x]);
  };
  const int4* p = A.fslots + (uint32_t)(tile * A.sf * 32 + lane);
  int4 e = p[0];
  bool more = false;
#pragma unroll 1
  for (int k = 0; k < A.sf; ++k) {  // a row's entries fill a prefix of its slots
    if (e.x < 0) break;
    const int4 en = k + 1 < A.sf ? p[(uint32_t)((k + 1) * 32)] : make_int4(-1, 0, 0, 0);
    if (k == kFaceRowSlots - 1) more = e.z < 0;  // the overflow mark
    one(e);
    e = en;
  }
  if (more) {
    const int o0 = A.fofl_ptr[i], o1 = A.fofl_ptr[i + 1];
#pragma unroll 1
    for (int q = o0; q < o1; ++q) one(A.fofl[q]);
  }
}

// Vertex-face records of the term pass (vf.cu): per term and role (the
// term's vertex p, a, b or c) kVfRoleVals values: that vertex's gradient
// (3), its blocks with p, a, b, c (4 x 9, row-major), and E.
constexpr int kVfRoleVals = 40;

// b[0..8] += v[0..8]
template <typename T>
__device__ __forceinline__ void add9(T* b, const T* v) {
#pragma unroll
  for (int q = 0; q < 9; ++q) b[q] += v[q];
}

// b[0..3] += v[0..3] (16-byte accesses when b allows them)
template <typename T>
__device__ __forceinline__ void add4(T* b, const T* v) {
  if constexpr (sizeof(T) == 4) {
    if ((((uintptr_t)b) & 15u) == 0) {
      float4 t = *reinterpret_cast<float4*>(b);
      t.x += v[0]; t.y += v[1]; t.z += v[2]; t.w += v[3];
      *reinterpret_cast<float4*>(b) = t;
      return;
    }
  } else {
    if ((((uintptr_t)b) & 15u) == 0) {
      double2 t0 = reinterpret_cast<double2*>(b)[0], t1 = reinterpret_cast<double2*>(b)[1];
      t0.x += v[0]; t0.y += v[1]; t1.x += v[2]; t1.y += v[3];
      reinterpret_cast<double2*>(b)[0] = t0;
      reinterpret_cast<double2*>(b)[1] = t1;
      return;
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) b[q] += v[q];
}

// The work of one row, writing the row's blocks through `row` (a shared-memory
// staging slot or, for rows that do not fit, the row's place in H).
template <typename T, int DOF, int AD, bool ENERGY, int S0, int FACES, bool PAIRS>
__device__ __forceinline__ void rows_eval_row(const RArgs<T>& A, int i, int tile, int lane,
                                              uint32_t m, int d0, int d1, int pb, int pn,
                                              int vb, int ve, const T* xi, const T* xti, T* row,
                                              double& energy) {
  constexpr int B = DOF * DOF;
  constexpr int TD = Tri<DOF>::size;
  const bool pairs = PAIRS && (A.mask & MAD_TERM_PAIR);
  const bool springs = A.mask & MAD_TERM_SPRING;
  const int nins = (d1 - d0) - ((int)(m & 0xFFFFu) + 1);
  T acc[TD], gr[DOF];
  RowNew rn;
  if constexpr (PAIRS) load_row_new(A.pe_pos, pb, pn, nins, rn);
  if constexpr (FACES == 4) {
    // the row's first vertex-face share and entry, asked of L1 now, read
    // after the edge terms
    if (ve > vb && (A.mask & MAD_TERM_VF)) {
      const char* p = reinterpret_cast<const char*>(A.vrec + (size_t)vb * kVfRoleVals);
#pragma unroll
      for (int l = 0; l < (int)(kVfRoleVals * sizeof(T)); l += 128)
        asm volatile("prefetch.global.L1 [%0];" ::"l"(p + l));
      asm volatile("prefetch.global.L1 [%0];" ::"l"(A.vent + 8 * (size_t)vb));
    }
  }
  // The row's first pair entry is loaded before the edge terms are evaluated,
  // so that its partner's position (a random vertex) arrives meanwhile.
  int pc0 = 0, pw0 = 0;
  T pr0 = T(0), xp0[DOF];
  if (pairs && pn > 0) {
    pc0 = A.pe_col[pb];
    pw0 = A.pe_pos[pb];
    pr0 = A.pe_rest[pb];
#pragma unroll
    for (int a = 0; a < DOF; ++a) xp0[a] = A.x[(uint32_t)(pc0 * DOF + a)];
  }
  // Blocks that no edge term stores start at 0: the whole row without edge
  // terms, else only the blocks that pairs inserted.
  if (!springs || S0 == 0) {
    for (int e = 0; e < (d1 - d0) * B; ++e) row[e] = T(0);
  } else if (PAIRS && nins > 0) {
#pragma unroll
    for (int k = 0; k < kRowNew; ++k)
      if (k < nins) {
        T* b = row + rn.np[k] * B;
#pragma unroll
        for (int q = 0; q < B; ++q) b[q] = T(0);
      }
    if (nins > kRowNew) {
      for (int e = pb; e < pb + pn; ++e) {
        const int32_t wv = A.pe_pos[e];
        if (wv & kPairNewBlock) {
          T* b = row + (wv & kPairPosMask) * B;
#pragma unroll
          for (int q = 0; q < B; ++q) b[q] = T(0);
        }
      }
    }
  }
  if (A.mask & MAD_TERM_INERTIA) {
    T Ei, Hi[B];
    eval_inertia<T, DOF>(xi, xti, A.w, Ei, gr, Hi);
    if (ENERGY) energy += (double)Ei;
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
  if constexpr (S0 > 0) {  // S0 == 0: an instantiation without edge terms
    if (springs) {
      row_edges<T, DOF, AD, S0>(A, i, tile, lane, m, xi,
                              [&](const EdgeRes<T, DOF, AD>& R, int p, int) {
                                const int op =
                                    !PAIRS || nins == 0 ? p : row_pos_new(rn, A.pe_pos, pb, pn, nins, p);
                                apply_edge_side<true>(R, 0, acc, row + op * B, gr);
                                if (ENERGY) energy += 0.5 * (double)edge_energy(R);
                              });
    }
  }
  if constexpr (FACES == 1 && DOF == 3) {
    // area preservation after the edge terms, which store their blocks
    if (A.mask & MAD_TERM_AREA) {
      row_faces3<T>(A, i, tile, lane,
                    [&](const T* xj, const T* xk, int, int pj, int pk, T A0) {
                      FaceRow3<T> o;
                      eval_area_row<T, AD>(xi, xj, xk, A0, A.ka, o);
#pragma unroll
                      for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int b = a; b < 3; ++b) acc[Tri<3>::idx(a, b)] += o.H[0][3 * a + b];
#pragma unroll
                      for (int a = 0; a < 3; ++a) gr[a] += o.g[a];
                      const int oj = PAIRS ? row_pos_new(rn, A.pe_pos, pb, pn, nins, pj) : pj;
                      const int ok = PAIRS ? row_pos_new(rn, A.pe_pos, pb, pn, nins, pk) : pk;
                      add9<T>(row + oj * B, o.H[1]);
                      add9<T>(row + ok * B, o.H[2]);
                      if (ENERGY) energy += (double)o.E * (1.0 / 3.0);
                    });
    }
  }
  if constexpr ((FACES == 1 || FACES == 2) && DOF == 2) {
    // after the edge terms, which store their blocks: faces add to them
    if (A.mask & (MAD_TERM_SYMDIR | MAD_TERM_ARAP)) {
      auto faces = [&](auto kc) {
        constexpr int KIND = decltype(kc)::value;
        row_faces<T>(A, i, tile, lane,
                     [&](const T* xj, const T* xk, int, int, int c, int pj, int pk, const T* M,
                         T ar) {
                       FaceRow<T> o;
                       eval_symdir_row<T, AD, KIND>(xi, xj, xk, c, M, ar, o);
                       acc[0] += o.H[0][0];
                       acc[1] += o.H[0][1];
                       acc[2] += o.H[0][3];
                       gr[0] += o.g[0];
                       gr[1] += o.g[1];
                       const int oj = PAIRS ? row_pos_new(rn, A.pe_pos, pb, pn, nins, pj) : pj;
                       const int ok = PAIRS ? row_pos_new(rn, A.pe_pos, pb, pn, nins, pk) : pk;
                       add4<T>(row + oj * B, o.H[1]);
                       add4<T>(row + ok * B, o.H[2]);
                       if (ENERGY) energy += (double)o.E * (1.0 / 3.0);
                     });
      };
      if constexpr (FACES == 1) {
        faces(std::integral_constant<int, kFaceSymDir>{});
      } else {
        if (!(A.mask & MAD_TERM_SYMDIR)) faces(std::integral_constant<int, kFaceArap>{});
        else faces(std::integral_constant<int, kFaceSymDir | kFaceArap>{});
      }
    }
  }
  if (pairs) {
    for (int e = pb; e < pb + pn; ++e) {
      int pw;
      T xj[DOF], rest;
      if (e == pb) {
        pw = pw0;
        rest = pr0;
#pragma unroll
        for (int a = 0; a < DOF; ++a) xj[a] = xp0[a];
      } else {
        const int j = A.pe_col[e];
        pw = A.pe_pos[e];
        rest = A.pe_rest[e];
#pragma unroll
        for (int a = 0; a < DOF; ++a) xj[a] = A.x[(uint32_t)(j * DOF + a)];
      }
      EdgeRes<T, DOF, AD> Rp;
      eval_edge_res<T, DOF, AD>(xi, xj, rest, A.kp, Rp);
      apply_edge_side<false>(Rp, 0, acc, row + (pw & kPairPosMask) * B, gr);
      if (ENERGY) energy += 0.5 * (double)edge_energy(Rp);
    }
  }
  if constexpr (FACES == 4 && DOF == 3 && PAIRS) {
    // installed vertex-face terms: this row's share of each of its terms,
    // written by the term pass before this kernel (its role's slice: the
    // gradient, its four blocks, E); the blocks go to the staged row, the
    // diagonal block to the register accumulator
    if (A.mask & MAD_TERM_VF) {
      for (int q = vb; q < ve; ++q) {
        const int4 w0 = reinterpret_cast<const int4*>(A.vent)[2 * q];
        const int4 w1 = reinterpret_cast<const int4*>(A.vent)[2 * q + 1];
        if (!w1.y) continue;
        const int role = (int)((uint32_t)w0.x >> 30);
        // the slice is read a block at a time (few registers: this branch
        // runs on few rows and must not lower every row's occupancy)
        const T* r = A.vrec + (size_t)q * kVfRoleVals;
        if (ENERGY) energy += 0.25 * (double)r[kVfRoleVals - 1];
#pragma unroll
        for (int a = 0; a < 3; ++a) gr[a] += r[a];
        const int pos[4] = {w0.y, w0.z, w0.w, w1.x};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          T b9[9];
#pragma unroll
          for (int q9 = 0; q9 < 9; ++q9) b9[q9] = r[3 + 9 * j + q9];
          if (j == role) {
#pragma unroll
            for (int a = 0; a < 3; ++a)
#pragma unroll
              for (int b2 = a; b2 < 3; ++b2) acc[Tri<3>::idx(a, b2)] += b9[3 * a + b2];
          } else {
            add9<T>(row + pos[j] * B, b9);
          }
        }
      }
    }
  }
  const int dp = PAIRS ? row_pos_new(rn, A.pe_pos, pb, pn, nins, (int)(m >> 16)) : (int)(m >> 16);
  T* d = row + dp * B;
#pragma unroll
  for (int a = 0; a < DOF; ++a)
#pragma unroll
    for (int b = 0; b < DOF; ++b)
      d[a * DOF + b] = a <= b ? acc[Tri<DOF>::idx(a, b)] : acc[Tri<DOF>::idx(b, a)];
#pragma unroll
  for (int a = 0; a < DOF; ++a) A.g[(uint32_t)(i * DOF + a)] = gr[a];
}

template <typename T, int DOF, int AD, bool ENERGY, int S0, int FACES, bool PAIRS>
__global__ void __launch_bounds__(kRowThreads, rows_min_blocks<T, FACES, DOF>()) k_rows_eval(const RArgs<T> A) {
  constexpr int B = DOF * DOF;
  constexpr int VEC = 16 / (int)sizeof(T);
  extern __shared__ __align__(16) char smem_raw[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int tile = blockIdx.x * kWarps + wib;
  const int i = tile * 32 + lane;
  const bool tile_live = tile * 32 < A.V;
  const bool has = i < A.V;
  T* stage = (T*)smem_raw + wib * A.wstage;
  double energy = 0.0;

  int d0 = 0, d1 = 0, pb = 0, pn = 0, vb = 0, ve = 0;
  uint32_t m = 0;
  T xi[DOF], xti[DOF];
  if (has) {
    d0 = A.rp[i];
    d1 = A.rp[i + 1];
    m = A.meta[i];
#pragma unroll
    for (int a = 0; a < DOF; ++a) xi[a] = A.x[(uint32_t)(i * DOF + a)];
    if (A.mask & MAD_TERM_INERTIA) {
#pragma unroll
      for (int a = 0; a < DOF; ++a) xti[a] = A.xt[(uint32_t)(i * DOF + a)];
    }
    if constexpr (PAIRS) {
      pb = A.prow[i];
      pn = A.prow[i + 1] - pb;
    }
    if constexpr (FACES == 4) {
      if (A.vrow) {
        vb = A.vrow[i];
        ve = A.vrow[i + 1];
      }
    }
  }
  // the warp's rows are consecutive in H: stage them from the first one
  const int dfirst = __shfl_sync(0xffffffffu, d0, 0);
  const int mis = (int)(((uintptr_t)(A.H + (uint32_t)(dfirst * B)) / sizeof(T)) % VEC);
  const int off = mis + (d0 - dfirst) * B;
  const bool staged = has && off + (d1 - d0) * B <= A.wstage;
  // rows that do not fit their warp's slice are assembled in place in H
  if (has)
    rows_eval_row<T, DOF, AD, ENERGY, S0, FACES, PAIRS>(A, i, tile, lane, m, d0, d1, pb, pn, vb, ve, xi, xti,
                                        staged ? stage + off : A.H + (uint32_t)(d0 * B), energy);
  // ---- write-back of the warp's staged rows (a prefix of its 32 rows) -------
  fence_async_smem();
  __syncwarp();
  if (tile_live) {
    const unsigned st = __ballot_sync(0xffffffffu, staged);
    if (st) {
      const int last = 31 - __clz(st);  // staged rows form a prefix
      const int dend = __shfl_sync(0xffffffffu, d1, last);
      const int n = (dend - dfirst) * B;
      T* dst = A.H + (uint32_t)(dfirst * B);
      const T* src = stage + mis;
      const int head = min(n, (VEC - mis) % VEC);
      const int body = ((n - head) / VEC) * VEC;
      for (int e = lane; e < head; e += 32) dst[e] = src[e];
      for (int e = head + body + lane; e < n; e += 32) dst[e] = src[e];
      const bool aligned = ((((uintptr_t)(dst + head)) | ((uintptr_t)(src + head))) & 15u) == 0;
      if (body > 0 && !aligned)
        for (int e = head + lane; e < head + body; e += 32) dst[e] = src[e];
      if (lane == 0 && body > 0 && aligned) {
        bulk_store(dst + head, src + head, (uint32_t)(body * sizeof(T)));
        bulk_commit_and_wait_read();
      }
    }
  }
  if (ENERGY) block_energy(energy, A.epart + blockIdx.x);
}

// y += the per-face pass's result for incidence q = 3f + c (DOF values)
template <typename T, int DOF>
__device__ __forceinline__ void add_corner_hv(const T* __restrict__ fhv, uint32_t q, T* yr) {
  if constexpr (DOF == 2) {
    using T2 = typename std::conditional<sizeof(T) == 4, float2, double2>::type;
    const T2 c = reinterpret_cast<const T2*>(fhv)[q];
    yr[0] += c.x;
    yr[1] += c.y;
  } else {
    // dof 3 (area faces): the pass stores corners 1 and 2 only; corner 0's
    // result is minus their sum (the term is translation invariant, and the
    // pass computes corner 0 that way)
    const uint32_t f = q / 3u, c = q - 3u * f;
    const T* h = fhv + 6 * (size_t)f;
    if (c == 0) {
#pragma unroll
      for (int a = 0; a < 3; ++a) yr[a] -= h[a] + h[3 + a];
    } else {
#pragma unroll
      for (int a = 0; a < 3; ++a) yr[a] += h[3 * (c - 1) + a];
    }
  }
}

// Resident blocks per SM the product's row pass with face terms is compiled
// for (fp32); the pass is latency-bound, so occupancy pays.
#ifndef MAD_HVP_FACES_MIN_BLOCKS
#define MAD_HVP_FACES_MIN_BLOCKS 4
#endif
template <typename T, bool FACES>
constexpr int hvp_min_blocks() {
  return FACES ? (sizeof(T) == 4 ? MAD_HVP_FACES_MIN_BLOCKS : 2) : rows_min_blocks<T, 0>();
}

template <typename T, int DOF, int AD, int S0, bool FACES>
__global__ void __launch_bounds__(kRowThreads, hvp_min_blocks<T, FACES>()) k_rows_hvp(const RArgs<T> A) {
  constexpr int TD = Tri<DOF>::size;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int tile = blockIdx.x * kWarps + wib;
  const int i = tile * 32 + lane;
  if (i >= A.V) return;
  const bool pairs = (A.mask & MAD_TERM_PAIR) && A.prow != nullptr;
  // the row's own position, direction and slot meta are needed only by the
  // vertex, edge and pair terms (face terms come from the per-face pass)
  const bool own = A.mask & (MAD_TERM_INERTIA | MAD_TERM_SPRING | MAD_TERM_PAIR);
  T xi[DOF], vi[DOF], yr[DOF];
  uint32_t m = 0;
#pragma unroll
  for (int a = 0; a < DOF; ++a) {
    xi[a] = T(0);
    vi[a] = T(0);
    yr[a] = T(0);
  }
  if (own) {
#pragma unroll
    for (int a = 0; a < DOF; ++a) {
      xi[a] = A.x[(uint32_t)(i * DOF + a)];
      vi[a] = A.v[(uint32_t)(i * DOF + a)];
    }
    if (!(MAD_HVP_COMPACT && A.cslots)) m = A.meta[i];
  }
  // face terms: the row's incidence entries (3f + c) of the per-face pass
  constexpr int SF = kFaceRowSlots;
  const bool face_terms =
      FACES && (A.mask & (DOF == 2 ? (MAD_TERM_SYMDIR | MAD_TERM_ARAP) : MAD_TERM_AREA));
  int32_t fe[SF];
#pragma unroll
  for (int k = 0; k < SF; ++k)
    fe[k] = face_terms && k < A.sf ? A.fcslots[(uint32_t)((tile * A.sf + k) * 32 + lane)] : -1;
  if (A.mask & MAD_TERM_INERTIA) {
    T xti[DOF], Ei, gi[DOF], Hi[DOF * DOF];
#pragma unroll
    for (int a = 0; a < DOF; ++a) xti[a] = A.xt[(uint32_t)(i * DOF + a)];
    eval_inertia<T, DOF>(xi, xti, A.w, Ei, gi, Hi);
#pragma unroll
    for (int a = 0; a < DOF; ++a)
#pragma unroll
      for (int b = 0; b < DOF; ++b) yr[a] += Hi[a * DOF + b] * vi[b];
  }
  auto hv = [&](const EdgeRes<T, DOF, AD>& R, const T* vj) {
    if constexpr (AD != kAdFull) {
#pragma unroll
      for (int a = 0; a < DOF; ++a) {
        T s = T(0);
#pragma unroll
        for (int b = 0; b < DOF; ++b)
          s += (a <= b ? R.K[Tri<DOF>::idx(a, b)] : R.K[Tri<DOF>::idx(b, a)]) * (vi[b] - vj[b]);
        yr[a] += s;
      }
    } else {
#pragma unroll
      for (int a = 0; a < DOF; ++a)
#pragma unroll
        for (int b = 0; b < DOF; ++b)
          yr[a] += R.d.Haa[a * DOF + b] * vi[b] + R.d.Hab[a * DOF + b] * vj[b];
    }
  };
  if constexpr (S0 > 0) {
    if (A.mask & MAD_TERM_SPRING) {
      auto edge = [&](const EdgeRes<T, DOF, AD>& R, int col) {
        T vj[DOF];
#pragma unroll
        for (int a = 0; a < DOF; ++a) vj[a] = A.v[(uint32_t)(col * DOF + a)];
        hv(R, vj);
      };
      if (MAD_HVP_COMPACT && A.cslots)
        row_edges_c<T, DOF, AD, S0>(A, i, tile, lane, xi, edge);
      else
        row_edges<T, DOF, AD, S0>(A, i, tile, lane, m, xi,
                                  [&](const EdgeRes<T, DOF, AD>& R, int, int col) { edge(R, col); });
    }
  }
  if (pairs) {
    const int pb = A.prow[i], pe = A.prow[i + 1];
    for (int e = pb; e < pe; ++e) {
      const int j = A.pe_col[e];
      T xj[DOF], vj[DOF];
#pragma unroll
      for (int a = 0; a < DOF; ++a) {
        xj[a] = A.x[(uint32_t)(j * DOF + a)];
        vj[a] = A.v[(uint32_t)(j * DOF + a)];
      }
      EdgeRes<T, DOF, AD> Rp;
      eval_edge_res<T, DOF, AD>(xi, xj, A.pe_rest[e], A.kp, Rp);
      hv(Rp, vj);
    }
  }
  if constexpr (FACES) {
    if (face_terms) {
      // the row's corners' results of the per-face pass (k_face_hv), whose
      // table entries were loaded above
#pragma unroll
      for (int k = 0; k < SF; ++k) {
        if (fe[k] == -1) continue;
        add_corner_hv<T, DOF>(A.fhv, (uint32_t)fe[k] & 0x7FFFFFFFu, yr);
      }
      if (fe[SF - 1] != -1 && fe[SF - 1] < 0) {  // the row continues in the overflow table
        const int o0 = A.fofl_ptr[i], o1 = A.fofl_ptr[i + 1];
        for (int q = o0; q < o1; ++q) add_corner_hv<T, DOF>(A.fhv, (uint32_t)A.fcofl[q], yr);
      }
    }
  }
  (void)TD;
#pragma unroll
  for (int a = 0; a < DOF; ++a) A.y[(uint32_t)(i * DOF + a)] = yr[a];
}

// Per-face pass of the Hessian-vector product for area-preservation faces
// (dof 3): each thread takes kAreaHvFaces faces (their loads issued
// together) and writes (H_f v_f) of corners 1 and 2 of each.
#ifndef MAD_AREA_HV_FACES
#define MAD_AREA_HV_FACES 1
#endif
constexpr int kAreaHvFaces = MAD_AREA_HV_FACES;

template <typename T, int AD>
__global__ void __launch_bounds__(256) k_face_hv_area(int nF, const int32_t* __restrict__ F,
                                                      const T* __restrict__ x,
                                                      const T* __restrict__ v,
                                                      const T* __restrict__ area, T ka,
                                                      T* __restrict__ out) {
  T u[kAreaHvFaces][3][3], w[kAreaHvFaces][3][3], ar[kAreaHvFaces];
  int64_t fs[kAreaHvFaces];
#pragma unroll
  for (int h = 0; h < kAreaHvFaces; ++h) {
    const int64_t f = ((int64_t)blockIdx.x * kAreaHvFaces + h) * 256 + threadIdx.x;
    fs[h] = f;
    if (f >= nF) continue;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      const int32_t vid = F[3 * f + c];
#pragma unroll
      for (int a = 0; a < 3; ++a) {
        u[h][c][a] = x[(int64_t)vid * 3 + a];
        w[h][c][a] = v[(int64_t)vid * 3 + a];
      }
    }
    ar[h] = area[f];
  }
#pragma unroll
  for (int h = 0; h < kAreaHvFaces; ++h) {
    const int64_t f = fs[h];
    if (f >= nF) continue;
    T o[9];
    hv_area_face<T, AD>(u[h][0], u[h][1], u[h][2], w[h][0], w[h][1], w[h][2], ar[h], ka, o);
    // corners 1 and 2; the row pass takes corner 0 as minus their sum
#pragma unroll
    for (int q = 3; q < 9; ++q) out[6 * f + q - 3] = o[q];
  }
}

constexpr int kFacesPerThread = 2;

// Per-face pass of the Hessian-vector product: one thread per face computes
// (H_f v_f) for its three corners once; the row kernel then adds, for each
// row, its corners' results.  Each face is differentiated once instead of
// once per corner, and no atomics are needed.
template <typename T, int AD>
__global__ void __launch_bounds__(256) k_face_hv(int nF, bool vec2, const int32_t* __restrict__ F,
                                                 const T* __restrict__ x, const T* __restrict__ v,
                                                 const T* __restrict__ Minv,
                                                 const T* __restrict__ area, T* __restrict__ out,
                                                 int kind) {
  // kFacesPerThread faces per thread, their loads issued together: the
  // grid is about one wave, and each thread overlaps its faces' latencies
  using T2 = typename std::conditional<sizeof(T) == 4, float2, double2>::type;
  T u[kFacesPerThread][3][2], w[kFacesPerThread][3][2], M[kFacesPerThread][4],
      ar[kFacesPerThread];
  int64_t fs[kFacesPerThread];
#pragma unroll
  for (int h = 0; h < kFacesPerThread; ++h) {
    const int64_t f = ((int64_t)blockIdx.x * kFacesPerThread + h) * 256 + threadIdx.x;
    fs[h] = f;
    if (f >= nF) continue;
    const int32_t vid[3] = {F[3 * f], F[3 * f + 1], F[3 * f + 2]};
    // [V][2] arrays: a vertex's pair is one 2-element load when both arrays
    // are aligned to it (the caller's pointers need not be)
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      if (vec2) {
        const T2 xu = reinterpret_cast<const T2*>(x)[vid[k]];
        const T2 xv = reinterpret_cast<const T2*>(v)[vid[k]];
        u[h][k][0] = xu.x;
        u[h][k][1] = xu.y;
        w[h][k][0] = xv.x;
        w[h][k][1] = xv.y;
      } else {
#pragma unroll
        for (int al = 0; al < 2; ++al) {
          u[h][k][al] = x[(int64_t)vid[k] * 2 + al];
          w[h][k][al] = v[(int64_t)vid[k] * 2 + al];
        }
      }
    }
    load4<T>(Minv + 4 * f, M[h]);
    ar[h] = area[f];
  }
#pragma unroll
  for (int h = 0; h < kFacesPerThread; ++h) {
    const int64_t f = fs[h];
    if (f >= nF) continue;
    T o[6];
    with_face2_kind(kind, [&](auto kc) {
      hv_symdir_face<T, AD, decltype(kc)::value>(u[h][0], u[h][1], u[h][2], w[h][0], w[h][1],
                                                 w[h][2], M[h], ar[h], o);
    });
    T2* o2 = reinterpret_cast<T2*>(out) + 3 * f;  // one corner's pair per 8 (16) bytes
#pragma unroll
    for (int c2 = 0; c2 < 3; ++c2) {
      T2 v2;
      v2.x = o[2 * c2];
      v2.y = o[2 * c2 + 1];
      o2[c2] = v2;
    }
  }
}

template <typename T>
RArgs<T> make_rargs(const RowsLaunch& L, const mad_terms& t, const void* x, const void* v,
                    void* g, void* H, void* y, bool energy) {
  RArgs<T> A;
  A.vrow = L.vrow;
  A.vent = L.vent;
  A.vrec = (const T*)L.vrec;
  A.fcslots = L.fcslots;
  A.fcofl = L.fcofl;
  A.fhv = (const T*)L.fhv;
  A.fslots = L.fslots;
  A.fofl_ptr = L.fofl_ptr;
  A.fofl = L.fofl;
  A.Minv = (const T*)t.face_Minv;
  A.area = (const T*)t.face_area;
  A.sf = L.sf;
  A.slots = L.slots;
  A.ctile = L.ctile;
  A.cslots = L.cslots;
  A.meta = L.meta;
  A.ofl_ptr = L.ofl_ptr;
  A.ofl = L.ofl;
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
  A.kp = (T)t.pair_k;
  A.ka = (T)t.area_k;
  A.mask = t.mask;
  A.epart = energy ? L.epart : nullptr;
  A.V = L.V;
  A.s0 = L.s0;
  A.wstage = (int)wstage_elems(L);
  return A;
}

__global__ void k_energy_sum_rows(const double* __restrict__ part, int n, double* out) {
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

// One instantiation of the assembly kernel, chosen by whether the active
// pattern holds pair blocks; also sets (or, with set, only sets) its shared
// memory limit.
template <typename T, int DOF, int AD, bool ENERGY, int S0, int FACES>
cudaError_t eval_k(const RArgs<T>& A, bool pairs, int nb, size_t smem, cudaStream_t s,
                   bool set = false) {
  const void* kp = (const void*)k_rows_eval<T, DOF, AD, ENERGY, S0, FACES, true>;
  const void* kn = (const void*)k_rows_eval<T, DOF, AD, ENERGY, S0, FACES, false>;
  if (set) {
    cudaError_t e = cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(kn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  }
  if (pairs)
    k_rows_eval<T, DOF, AD, ENERGY, S0, FACES, true><<<nb, kRowThreads, smem, s>>>(A);
  else
    k_rows_eval<T, DOF, AD, ENERGY, S0, FACES, false><<<nb, kRowThreads, smem, s>>>(A);
  return cudaGetLastError();
}

// calls f(std::integral_constant<int, AD>) for the run-time AD form
template <typename F>
cudaError_t with_ad(int ad, F&& f) {
  if (ad == kAdFull) return f(std::integral_constant<int, kAdFull>{});
  if (ad == kAdGeneric) return f(std::integral_constant<int, kAdGeneric>{});
  return f(std::integral_constant<int, kAdReduced>{});
}

// Every (AD, ENERGY) instantiation for one S0 and FACES.  FACES: 0 no face
// terms; 1 the face term of the dof (symmetric Dirichlet for dof 2, area
// preservation for dof 3); 2 (dof 2) ARAP alone or with symmetric Dirichlet,
// an instantiation of its own so that the symmetric Dirichlet kernel keeps
// its register budget; 4 (dof 3) the installed vertex-face terms gathered
// from the term pass's records.
template <typename T, int DOF, int S0, int FACES>
cudaError_t eval_k4(const RArgs<T>& A, int ad, bool energy, bool pairs, int nb, size_t smem,
                    cudaStream_t s, bool set = false) {
  if (set) {
    for (int a : {kAdReduced, kAdFull, kAdGeneric}) {
      const cudaError_t e = with_ad(a, [&](auto adc) {
        constexpr int AD = decltype(adc)::value;
        const cudaError_t e1 = eval_k<T, DOF, AD, true, S0, FACES>(A, pairs, nb, smem, s, true);
        if (e1 != cudaSuccess) return e1;
        return eval_k<T, DOF, AD, false, S0, FACES>(A, pairs, nb, smem, s, true);
      });
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  return with_ad(ad, [&](auto adc) {
    constexpr int AD = decltype(adc)::value;
    if (energy) return eval_k<T, DOF, AD, true, S0, FACES>(A, pairs, nb, smem, s);
    return eval_k<T, DOF, AD, false, S0, FACES>(A, pairs, nb, smem, s);
  });
}

template <typename T, int DOF>
cudaError_t run_rows_eval(const RowsLaunch& L, const mad_terms& t, const void* x, void* g,
                          void* H, double* energy, cudaStream_t s) {
  RArgs<T> A = make_rargs<T>(L, t, x, nullptr, g, H, nullptr, energy != nullptr);
  const int nb = rows_blocks(L.V);
  const size_t smem = rows_smem_bytes(L);
  const int ad = ad_form(t.flags);
  const bool pairs = L.prow != nullptr;
  const bool en = energy != nullptr;
  cudaError_t e;
  if (DOF == 3 && L.vrow && pairs && (t.mask & MAD_TERM_VF) && !(t.mask & MAD_TERM_AREA) &&
      L.cslots == nullptr) {
    // installed vertex-face terms gathered into the rows (FACES == 4); with
    // compact slot tables the compact kernel does the same (below)
    if (t.mask & MAD_TERM_SPRING)
      e = eval_k4<T, DOF, kS0Max, 4>(A, ad, en, pairs, nb, smem, s);
    else
      e = eval_k4<T, DOF, 0, 4>(A, ad, en, pairs, nb, smem, s);
  } else if ((DOF == 2 && (t.mask & (MAD_TERM_SYMDIR | MAD_TERM_ARAP))) ||
      (DOF == 3 && (t.mask & MAD_TERM_AREA))) {
    // face terms: the face-row instantiations; without edge terms the kernel
    // carries no edge-slot code (S0 = 0)
    auto faces_k = [&](auto s0c) {
      constexpr int S0F = decltype(s0c)::value;
      if constexpr (DOF == 2) {
        if (t.mask & MAD_TERM_ARAP) return eval_k4<T, DOF, S0F, 2>(A, ad, en, pairs, nb, smem, s);
      }
      return eval_k4<T, DOF, S0F, 1>(A, ad, en, pairs, nb, smem, s);
    };
    if ((t.mask & MAD_TERM_SPRING) && L.s0 <= 6)
      e = faces_k(std::integral_constant<int, 6>{});  // valence <= 6: fewer registers
    else if (t.mask & MAD_TERM_SPRING)
      e = faces_k(std::integral_constant<int, kS0Max>{});
    else
      e = faces_k(std::integral_constant<int, 0>{});
  } else if (L.cslots != nullptr) {
    // edge, vertex and pair terms with compact slot tables
    return rows_eval_compact_t<T, DOF>(L, t, x, g, H, energy, s);
  } else if (L.s0 <= 6) {
    // slot-table rows of width <= 6 (triangle meshes of valence <= 6) use the
    // narrower instantiation: fewer registers
    e = eval_k4<T, DOF, 6, 0>(A, ad, en, pairs, nb, smem, s);
  } else {
    e = eval_k4<T, DOF, kS0Max, 0>(A, ad, en, pairs, nb, smem, s);
  }
  if (e != cudaSuccess || !energy) return e;
  k_energy_sum_rows<<<1, 1024, 0, s>>>(L.epart, nb, energy);
  return cudaGetLastError();
}

template <typename T, int DOF>
cudaError_t run_rows_hvp(const RowsLaunch& L, const mad_terms& t, const void* x, const void* v,
                         void* y, cudaStream_t s) {
  RArgs<T> A = make_rargs<T>(L, t, x, v, nullptr, nullptr, y, false);
  const int nb = rows_blocks(L.V);
  return with_ad(ad_form(t.flags), [&](auto adc) -> cudaError_t {
    constexpr int AD = decltype(adc)::value;
    const bool sp = t.mask & MAD_TERM_SPRING;
    // the row pass after a per-face pass (face terms), or alone
    // the row pass after the per-face pass, or alone
    auto rows = [&](auto facesc) {
      constexpr bool FC = decltype(facesc)::value;
      // slot tables of width <= 6 (triangle meshes of valence <= 6) take the
      // narrower instantiation: fewer registers
      if (sp && L.s0 <= 6) k_rows_hvp<T, DOF, AD, 6, FC><<<nb, kRowThreads, 0, s>>>(A);
      else if (sp) k_rows_hvp<T, DOF, AD, kS0Max, FC><<<nb, kRowThreads, 0, s>>>(A);
      else k_rows_hvp<T, DOF, AD, 0, FC><<<nb, kRowThreads, 0, s>>>(A);
      return cudaGetLastError();
    };
    if constexpr (DOF == 2) {
      if (t.mask & (MAD_TERM_SYMDIR | MAD_TERM_ARAP)) {
        if (L.nF > 0) {
          const unsigned nbf = (unsigned)((L.nF + 256 * kFacesPerThread - 1) / (256 * kFacesPerThread));
          const bool vec2 = ((((uintptr_t)x) | ((uintptr_t)v)) % (2 * sizeof(T))) == 0;
          k_face_hv<T, AD><<<nbf, 256, 0, s>>>(L.nF, vec2, L.F, (const T*)x, (const T*)v,
                                               (const T*)t.face_Minv, (const T*)t.face_area,
                                               (T*)L.fhv, face2_kind(t.mask));
          const cudaError_t e = cudaGetLastError();
          if (e != cudaSuccess) return e;
        }
        return rows(std::true_type{});
      }
    }
    if constexpr (DOF == 3) {
      if (t.mask & MAD_TERM_AREA) {
        if (L.nF > 0) {
          const unsigned nbf = (unsigned)((L.nF + 256 * kAreaHvFaces - 1) / (256 * kAreaHvFaces));
          k_face_hv_area<T, AD><<<nbf, 256, 0, s>>>(L.nF, L.F, (const T*)x, (const T*)v,
                                                    (const T*)t.face_area, (T)t.area_k,
                                                    (T*)L.fhv);
          const cudaError_t e = cudaGetLastError();
          if (e != cudaSuccess) return e;
        }
        return rows(std::true_type{});
      }
    }
    if (L.s0 <= 6) k_rows_hvp<T, DOF, AD, 6, false><<<nb, kRowThreads, 0, s>>>(A);
    else k_rows_hvp<T, DOF, AD, kS0Max, false><<<nb, kRowThreads, 0, s>>>(A);
    return cudaGetLastError();
  });
}

template <typename T, int DOF>
cudaError_t set_rows_limits(size_t bytes) {
  RArgs<T> A{};
  cudaError_t e;
  if ((e = eval_k4<T, DOF, 6, 0>(A, false, false, false, 0, bytes, 0, true)) != cudaSuccess)
    return e;
  if ((e = eval_k4<T, DOF, kS0Max, 0>(A, false, false, false, 0, bytes, 0, true)) != cudaSuccess)
    return e;
  if ((e = eval_k4<T, DOF, 6, 1>(A, false, false, false, 0, bytes, 0, true)) != cudaSuccess)
    return e;
  if ((e = eval_k4<T, DOF, kS0Max, 1>(A, false, false, false, 0, bytes, 0, true)) != cudaSuccess)
    return e;
  if ((e = eval_k4<T, DOF, 0, 1>(A, false, false, false, 0, bytes, 0, true)) != cudaSuccess)
    return e;
  if constexpr (DOF == 3) {
    if ((e = eval_k4<T, DOF, kS0Max, 4>(A, false, false, false, 0, bytes, 0, true)) !=
        cudaSuccess)
      return e;
    if ((e = eval_k4<T, DOF, 0, 4>(A, false, false, false, 0, bytes, 0, true)) != cudaSuccess)
      return e;
  }
  if constexpr (DOF == 2) {
    if ((e = eval_k4<T, DOF, 6, 2>(A, false, false, false, 0, bytes, 0, true)) != cudaSuccess)
      return e;
    if ((e = eval_k4<T, DOF, kS0Max, 2>(A, false, false, false, 0, bytes, 0, true)) !=
        cudaSuccess)
      return e;
    if ((e = eval_k4<T, DOF, 0, 2>(A, false, false, false, 0, bytes, 0, true)) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

}  // namespace

// Entry points of one (dtype, dof), instantiated by the rows_*.cu units.
template <typename T, int DOF>
cudaError_t rows_eval_t(const RowsLaunch& L, const mad_terms& t, const void* x, void* g, void* H,
                        double* energy, cudaStream_t s) {
  return run_rows_eval<T, DOF>(L, t, x, g, H, energy, s);
}
template <typename T, int DOF>
cudaError_t rows_hvp_t(const RowsLaunch& L, const mad_terms& t, const void* x, const void* v,
                       void* y, cudaStream_t s) {
  return run_rows_hvp<T, DOF>(L, t, x, v, y, s);
}
template <typename T, int DOF>
cudaError_t rows_limits_t(size_t bytes) {
  return set_rows_limits<T, DOF>(bytes);
}

}  // namespace mad
