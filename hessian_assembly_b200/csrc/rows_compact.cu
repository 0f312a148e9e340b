// rows_compact.cu -- the row-streaming assembly of edge and vertex terms
// driven by the compact slot tables.
//
// Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
// Computations", section 方法, key design 1: the only global traffic of the
// step should be reading the mesh and writing the final sparse derivatives;
// key design 3: the CSR block offsets come from a table built once per
// topology, so assembly needs no search.
//
// Same work as k_rows_eval (rows_impl.cuh) for a term set of springs,
// inertia and runtime pairs: one thread per Hessian row, the row's edge
// terms evaluated with forward-mode AD numbers in registers, each row staged
// in its warp's slice of shared memory and written back with one 1-D bulk
// copy per warp.  The row tables it reads are the compact ones
// (HostRowTables::cslots): 4 bytes per slot instead of 8 and no per-row
// row_ptr or meta word.  A row's block positions follow from its slots
// (columns ascend, the diagonal sits after the columns below the row), and
// the row's first block from the tile's row_ptr plus a warp prefix sum of
// the row lengths.  With runtime pairs active (method section, key design 4:
// blocks inserted into the pattern between steps) the rows come from the
// active row_ptr instead, and a mesh block's position is moved past the
// pair blocks inserted before it in its row.
#include "rows_impl.cuh"

namespace mad {
namespace {

template <typename T>
struct CArgs {
  const int4* ctile;
  const uint32_t* cslots;
  const int32_t* ofl_ptr;
  const int2* ofl;
  const T* x;
  T* g;
  T* H;
  const T* L0;
  T k;
  const T* xt;
  T w;
  // runtime pairs (the active pattern's row_ptr, per-row inserted-block
  // masks and pair entries)
  const int32_t* rp;
  const uint32_t* pmask;
  const int32_t* prow;
  const int32_t* pe_col;
  const int32_t* pe_pos;
  const T* pe_xr;  // per entry: partner position (zero padded to 4) + rest length
  T kp;
  // installed vertex-face terms: per-row entries and the term pass's
  // per-role shares (see vf.cu)
  const int32_t* vrow;
  const int32_t* vent;
  const T* vrec;
  unsigned mask;
  double* epart;
  int V, s0, wstage;
};

// A launch over the rows of one shard (mad_eval_shard): tiles from tile0,
// rows below row_hi; positions of shard s at xp[s] (rows rbeg[s] ..
// rbeg[s+1]); g and H hold the shard's rows and blocks only (g's first row
// is rbeg[own], H's first block hoff).
template <typename T>
struct ShardArgs {
  int tile0, row_hi, own, nparts;
  int64_t hoff;
  int rbeg[MAD_MAX_SHARDS + 1];
  const T* xp[MAD_MAX_SHARDS];
};

// Positions of vertex v: the own shard's part, else the owner's.
template <typename T, int DOF>
__device__ __forceinline__ const T* shard_x(const ShardArgs<T>& S, int v) {
  const int rb = S.rbeg[S.own], re = S.rbeg[S.own + 1];
  if ((unsigned)(v - rb) < (unsigned)(re - rb)) return S.xp[S.own] + (uint32_t)((v - rb) * DOF);
  int o = 0;
  while (o + 1 < S.nparts && v >= S.rbeg[o + 1]) ++o;
  return S.xp[o] + (uint32_t)((v - S.rbeg[o]) * DOF);
}

// Tiles ahead of its own whose slot, position and target lines a warp asks
// the L2 to fetch before it starts (0: none).  Tiles run in about index
// order, so tile t + D starts roughly D / (resident warps) waves later.
#ifndef MAD_ROWSC_PREFETCH_TILES
#define MAD_ROWSC_PREFETCH_TILES 512
#endif
// Also ask for the later tile's rest lengths of the edges above its rows
// (their ids start at that tile's first edge id, read at the start and used
// once this tile's terms are done).
#ifndef MAD_ROWSC_PREFETCH_L0
#define MAD_ROWSC_PREFETCH_L0 0
#endif
// With pairs: each row's first block read from the active row_ptr (1), or
// the tile's first block plus a warp prefix sum of the row lengths (0).
#ifndef MAD_ROWSC_PAIRS_RP
#define MAD_ROWSC_PAIRS_RP 1
#endif

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Entry e's partner position (DOF values) and rest length, gathered by
// k_pair_gather: four values, one 16-byte load for fp32, two for fp64.
template <typename T, int DOF>
__device__ __forceinline__ void load_xr(const T* __restrict__ xr, int e, T* xj, T& rest) {
  if constexpr (sizeof(T) == 4) {
    const float4 q = reinterpret_cast<const float4*>(xr)[e];
    xj[0] = q.x;
    xj[1] = q.y;
    if constexpr (DOF == 3) xj[2] = q.z;
    rest = q.w;
  } else {
    const double2 q0 = reinterpret_cast<const double2*>(xr)[2 * e];
    const double2 q1 = reinterpret_cast<const double2*>(xr)[2 * e + 1];
    xj[0] = q0.x;
    xj[1] = q0.y;
    if constexpr (DOF == 3) xj[2] = q1.x;
    rest = q1.y;
  }
}

// Before an assembly with pairs: for every live pair entry e (prow[V] of
// them) the partner's position and the entry's rest length, side by side.
// The row kernel then finds them next to the entry's position word instead
// of behind a dependent load at a random vertex.
constexpr int kGatherBlocks = 4 * 148;
template <typename T, int DOF>
__global__ void __launch_bounds__(256) k_pair_gather(const int32_t* __restrict__ nent,
                                                     const int32_t* __restrict__ pe_col,
                                                     const T* __restrict__ pe_rest,
                                                     const T* __restrict__ x, T* __restrict__ xr) {
  const int n = *nent;
  const int stride = gridDim.x * blockDim.x;
#pragma unroll 1
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += 2 * stride) {
    const int e2 = e + stride;
    const int j0 = pe_col[e];
    const int j1 = e2 < n ? pe_col[e2] : j0;
    T q0[4] = {T(0), T(0), T(0), T(0)}, q1[4] = {T(0), T(0), T(0), T(0)};
#pragma unroll
    for (int a = 0; a < DOF; ++a) {
      q0[a] = x[(uint32_t)(j0 * DOF + a)];
      q1[a] = x[(uint32_t)(j1 * DOF + a)];
    }
    q0[3] = pe_rest[e];
    q1[3] = e2 < n ? pe_rest[e2] : T(0);
    if constexpr (sizeof(T) == 4) {
      reinterpret_cast<float4*>(xr)[e] = make_float4(q0[0], q0[1], q0[2], q0[3]);
      if (e2 < n) reinterpret_cast<float4*>(xr)[e2] = make_float4(q1[0], q1[1], q1[2], q1[3]);
    } else {
      reinterpret_cast<double2*>(xr)[2 * e] = make_double2(q0[0], q0[1]);
      reinterpret_cast<double2*>(xr)[2 * e + 1] = make_double2(q0[2], q0[3]);
      if (e2 < n) {
        reinterpret_cast<double2*>(xr)[2 * e2] = make_double2(q1[0], q1[1]);
        reinterpret_cast<double2*>(xr)[2 * e2 + 1] = make_double2(q1[2], q1[3]);
      }
    }
  }
}


template <typename T, int DOF, int AD, bool ENERGY, int S0, bool SHARD, bool PAIRS, bool VF>
__device__ __forceinline__ void rows_c_body(const CArgs<T>& A, const ShardArgs<T>* S) {
  static_assert(!(SHARD && PAIRS), "a shard launch carries no pairs");
  static_assert(!VF || (PAIRS && DOF == 3), "vertex-face terms come with their pair blocks");
  constexpr int B = DOF * DOF;
  constexpr int TD = Tri<DOF>::size;
  constexpr int VEC = 16 / (int)sizeof(T);
  extern __shared__ __align__(16) char smem_raw[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int tile = (SHARD ? S->tile0 : 0) + blockIdx.x * kWarps + wib;
  const int i = tile * 32 + lane;
  const int row_hi = SHARD ? S->row_hi : A.V;
  const int goff = SHARD ? S->rbeg[S->own] : 0;   // g's first row
  const int64_t hoff = SHARD ? S->hoff : 0;        // H's first block
  const bool tile_live = tile * 32 < row_hi;
  const bool has = i < row_hi;
  T* stage = (T*)smem_raw + wib * A.wstage;
  double energy = 0.0;
  const bool springs = A.mask & MAD_TERM_SPRING;
  if constexpr (MAD_ROWSC_PREFETCH_TILES > 0 && !SHARD) {
    // one 128-byte line per lane: the later tile's slot words, then its
    // positions and targets (lines past the arrays' ends are skipped)
    const int tp = tile + MAD_ROWSC_PREFETCH_TILES;
    constexpr int XL = 32 * DOF * (int)sizeof(T) / 128;  // lines of a tile's rows
    if (tp * 32 < A.V) {
      const int64_t nx = (int64_t)A.V * DOF;
      if (lane < A.s0) {
        prefetch_l2(A.cslots + (size_t)(tp * A.s0 + lane) * 32);
      } else if (lane >= 8 && lane < 8 + XL) {
        const int64_t e = (int64_t)tp * 32 * DOF + (lane - 8) * (128 / (int)sizeof(T));
        if (e < nx) prefetch_l2(A.x + e);
      } else if (lane >= 16 && lane < 16 + XL && (A.mask & MAD_TERM_INERTIA)) {
        const int64_t e = (int64_t)tp * 32 * DOF + (lane - 16) * (128 / (int)sizeof(T));
        if (e < nx) prefetch_l2(A.xt + e);
      } else if (PAIRS && lane == 28) {
        prefetch_l2(A.pmask + (size_t)tp * 32);
      } else if (PAIRS && lane == 29) {
        prefetch_l2(A.prow + (size_t)tp * 32);
      }
    }
  }

  int4 th = make_int4(0, 0, 0, 0);
  if (tile_live) th = A.ctile[tile];
  constexpr bool kPfL0 = MAD_ROWSC_PREFETCH_TILES > 0 && MAD_ROWSC_PREFETCH_L0 && !SHARD;
  int pf_e0 = -1, pf_e1 = -1;  // the later tile's first edge id and the next tile's
  if constexpr (kPfL0) {
    const int tp = tile + MAD_ROWSC_PREFETCH_TILES;
    if (lane == 24 && (tp + 1) * 32 < A.V && springs) {
      pf_e0 = A.ctile[tp].y;
      pf_e1 = A.ctile[tp + 1].y;
    }
  }
  uint32_t sw[S0];
#pragma unroll
  for (int k = 0; k < S0; ++k) {
    sw[k] = 0u;
    if (has && k < A.s0) sw[k] = A.cslots[(uint32_t)((tile * A.s0 + k) * 32 + lane)];
  }
  // the row's inserted blocks and pair entries, the tile's first block in
  // the active pattern
  int pb = 0, pn = 0, prp = 0, pd0 = 0, pd1 = 0, vb = 0, ve = 0;
  uint32_t pm = 0u;
  if (VF && has) {
    vb = A.vrow[i];
    ve = A.vrow[i + 1];
  }
  if (PAIRS) {
    if (has) {
      pm = A.pmask[i];
      pb = A.prow[i];
      pn = A.prow[i + 1] - pb;
      if (MAD_ROWSC_PAIRS_RP) {
        pd0 = A.rp[i];
        pd1 = A.rp[i + 1];
      }
    }
    if (!MAD_ROWSC_PAIRS_RP && lane == 0 && tile_live) prp = A.rp[tile * 32];
  }
  T xi[DOF], xti[DOF];
  if (has) {
    const T* xs = SHARD ? shard_x<T, DOF>(*S, i) : A.x + (uint32_t)(i * DOF);
#pragma unroll
    for (int a = 0; a < DOF; ++a) xi[a] = xs[a];
    if (A.mask & MAD_TERM_INERTIA) {
#pragma unroll
      for (int a = 0; a < DOF; ++a) xti[a] = A.xt[(uint32_t)(i * DOF + a)];
    }
  }
  // positions and rest lengths behind the slots
  T xb[S0][DOF];
  T l0[S0];
#pragma unroll
  for (int k = 0; k < S0; ++k) {
    if (sw[k] == 0u || !springs) continue;
    const int col = i + slot_dcol(sw[k]);
    const T* xs = SHARD ? shard_x<T, DOF>(*S, col) : A.x + (uint32_t)(col * DOF);
#pragma unroll
    for (int a = 0; a < DOF; ++a) xb[k][a] = xs[a];
    l0[k] = A.L0[th.y + slot_deid(sw[k])];
  }
  const bool pairs = PAIRS && (A.mask & MAD_TERM_PAIR);
  if constexpr (VF) {
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
  // row length (off-diagonal slots + overflow + the diagonal) and the row's
  // first block: the tile's row_ptr plus the lengths of the rows before it
  int noff = 0, dpos = 0, o0 = 0, no = 0;
#pragma unroll
  for (int k = 0; k < S0; ++k) {
    noff += sw[k] != 0u;
    dpos += sw[k] != 0u && slot_dcol(sw[k]) < 0;
  }
  if (has && ((uint32_t)th.z >> lane) & 1u) {
    o0 = A.ofl_ptr[i];
    no = A.ofl_ptr[i + 1] - o0;
    for (int q = 0; q < no; ++q) dpos += A.ofl[o0 + q].x < i;
  }
  noff += no;
  // blocks the pairs inserted into the row (their positions are the set bits
  // of pm, or, past the mask's reach, the flagged pair entries)
  const bool pofl = PAIRS && (pm & kPmaskOverflow);
  const int nins = !PAIRS ? 0 : (pofl ? (int)(pm & ~kPmaskOverflow) : __popc(pm));
  int d0, d1;
  if (PAIRS && MAD_ROWSC_PAIRS_RP) {
    d0 = pd0;
    d1 = pd1;
  } else {
    const int len = has ? noff + 1 + nins : 0;
    int incl = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    d0 = (PAIRS ? __shfl_sync(0xffffffffu, prp, 0) : th.x) + incl - len;
    d1 = d0 + len;
  }
  // the first kRowNew inserted positions, ascending (0x7FFFFFFF past them)
  RowNew rn;
  if constexpr (PAIRS) {
    uint32_t m = pofl ? 0u : pm;
#pragma unroll
    for (int k = 0; k < kRowNew; ++k) {
      rn.np[k] = m ? __ffs(m) - 1 : 0x7FFFFFFF;
      m &= m - 1u;
    }
  }
  // a mesh block's position in the active row: past the inserted blocks at
  // or before it
  auto at = [&](int p) {
    if constexpr (PAIRS) {
      if (nins > kRowNew) {
        if (pofl) return row_pos(A.pe_pos, pb, pn, nins, p);
        for (uint32_t m = pm; m; m &= m - 1u) {
          if (__ffs(m) - 1 > p) break;
          ++p;
        }
        return p;
      }
#pragma unroll
      for (int k = 0; k < kRowNew; ++k) p += rn.np[k] <= p;
    }
    return p;
  };
  const int dfirst = __shfl_sync(0xffffffffu, d0, 0);
  T* const h0 = A.H + (uint32_t)((dfirst - hoff) * B);  // the warp's first block in H
  const int mis = (int)(((uintptr_t)h0 / sizeof(T)) % VEC);
  const int off = mis + (d0 - dfirst) * B;
  const bool staged = has && off + (d1 - d0) * B <= A.wstage;
  if (has) {
    T* row = staged ? stage + off : h0 + (uint32_t)((d0 - dfirst) * B);
    if (PAIRS && springs && nins > 0) {
      // inserted blocks no edge term stores start at 0
      if (!pofl) {
#pragma unroll
        for (int k = 0; k < kRowNew; ++k)
          if (k < nins) {
            T* b = row + rn.np[k] * B;
#pragma unroll
            for (int q = 0; q < B; ++q) b[q] = T(0);
          }
        if (nins > kRowNew) {
          uint32_t m = pm;
          for (int k = 0; k < kRowNew; ++k) m &= m - 1u;
          for (; m; m &= m - 1u) {
            T* b = row + (__ffs(m) - 1) * B;
#pragma unroll
            for (int q = 0; q < B; ++q) b[q] = T(0);
          }
        }
      } else {
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
    T acc[TD], gr[DOF];
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
    if (springs) {
#pragma unroll
      for (int k = 0; k < S0; ++k) {
        if (sw[k] == 0u) continue;
        EdgeRes<T, DOF, AD> R;
        eval_edge_res<T, DOF, AD>(xi, xb[k], l0[k], A.k, R);
        // block position: the slots before it plus the diagonal when the
        // column lies above the row
        const int p = at(k + (slot_dcol(sw[k]) > 0));
        apply_edge_side<true>(R, 0, acc, row + p * B, gr);
        if (ENERGY) energy += 0.5 * (double)edge_energy(R);
      }
      for (int q = 0; q < no; ++q) {  // rows longer than the slot table
        const int2 e = A.ofl[o0 + q];
        const T* xs = SHARD ? shard_x<T, DOF>(*S, e.x) : A.x + (uint32_t)(e.x * DOF);
        T xo[DOF];
#pragma unroll
        for (int a = 0; a < DOF; ++a) xo[a] = xs[a];
        EdgeRes<T, DOF, AD> R;
        eval_edge_res<T, DOF, AD>(xi, xo, A.L0[e.y], A.k, R);
        const int p = at(A.s0 + q + (e.x > i));
        apply_edge_side<true>(R, 0, acc, row + p * B, gr);
        if (ENERGY) energy += 0.5 * (double)edge_energy(R);
      }
    } else {
      // without edge terms every off-diagonal block of the row is zero
      for (int e = 0; e < (d1 - d0) * B; ++e) row[e] = T(0);
    }
    if (pairs) {
      // the gathered entries (L2 hits: the gather kernel has just written
      // them) are read after the edge terms, not ahead of them: asked for
      // early they held registers through the edge terms for little gain
      for (int e = pb; e < pb + pn; ++e) {
        const int pw = A.pe_pos[e];
        T xj[DOF], rest;
        load_xr<T, DOF>(A.pe_xr, e, xj, rest);
        EdgeRes<T, DOF, AD> Rp;
        eval_edge_res<T, DOF, AD>(xi, xj, rest, A.kp, Rp);
        apply_edge_side<false>(Rp, 0, acc, row + (pw & kPairPosMask) * B, gr);
        if (ENERGY) energy += 0.5 * (double)edge_energy(Rp);
      }
    }
    if constexpr (VF) {
      // installed vertex-face terms: this row's share of each of its terms
      // (its role's slice: the gradient, its four blocks, E); the blocks go
      // to the staged row, the diagonal block to the register accumulator
      if (A.mask & MAD_TERM_VF) {
        for (int q = vb; q < ve; ++q) {
          const int4 w0 = reinterpret_cast<const int4*>(A.vent)[2 * q];
          const int4 w1 = reinterpret_cast<const int4*>(A.vent)[2 * q + 1];
          if (!w1.y) continue;
          const int role = (int)((uint32_t)w0.x >> 30);
          // the slice is read a block at a time (few live registers)
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
    T* d = row + at(dpos) * B;
#pragma unroll
    for (int a = 0; a < DOF; ++a)
#pragma unroll
      for (int b = 0; b < DOF; ++b)
        d[a * DOF + b] = a <= b ? acc[Tri<DOF>::idx(a, b)] : acc[Tri<DOF>::idx(b, a)];
#pragma unroll
    for (int a = 0; a < DOF; ++a) A.g[(uint32_t)((i - goff) * DOF + a)] = gr[a];
  }
  if constexpr (kPfL0) {
    if (pf_e0 >= 0)
      for (int e = pf_e0; e < pf_e1; e += 128 / (int)sizeof(T)) prefetch_l2(A.L0 + e);
  }
  // ---- write-back of the warp's staged rows (a prefix of its 32 rows) ------
  fence_async_smem();
  __syncwarp();
  if (tile_live) {
    const unsigned st = __ballot_sync(0xffffffffu, staged);
    if (st) {
      const int last = 31 - __clz(st);
      const int dend = __shfl_sync(0xffffffffu, d1, last);
      const int n = (dend - dfirst) * B;
      T* dst = h0;
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

template <typename T, int DOF, int AD, bool ENERGY, int S0, bool PAIRS, bool VF>
__global__ void __launch_bounds__(kRowThreads, rows_min_blocks<T, 0>())
    k_rows_eval_c(const CArgs<T> A) {
  rows_c_body<T, DOF, AD, ENERGY, S0, false, PAIRS, VF>(A, nullptr);
}

template <typename T, int DOF, int AD, bool ENERGY, int S0>
__global__ void __launch_bounds__(kRowThreads, rows_min_blocks<T, 0>())
    k_rows_eval_cs(const CArgs<T> A, const __grid_constant__ ShardArgs<T> S) {
  rows_c_body<T, DOF, AD, ENERGY, S0, true, false, false>(A, &S);
}

// Shared-memory carve-out asked for the kernel, in percent of the unified
// L1 / shared memory (-1: the driver's choice); a smaller carve-out fits
// fewer blocks per SM and leaves more L1 for the neighbour gathers.
#ifndef MAD_ROWSC_CARVEOUT
#define MAD_ROWSC_CARVEOUT -1
#endif

template <typename T, int DOF, int AD, bool ENERGY, int S0>
cudaError_t launch_c(const CArgs<T>& A, const ShardArgs<T>* S, bool pairs, bool vf, int nb,
                     size_t smem, cudaStream_t s, bool set) {
  constexpr bool kVf = DOF == 3;  // vertex-face terms have dof 3
  if (set) {
    const void* ks[4] = {(const void*)k_rows_eval_c<T, DOF, AD, ENERGY, S0, false, false>,
                         (const void*)k_rows_eval_c<T, DOF, AD, ENERGY, S0, true, false>,
                         (const void*)k_rows_eval_c<T, DOF, AD, ENERGY, S0, true, kVf>,
                         (const void*)k_rows_eval_cs<T, DOF, AD, ENERGY, S0>};
    for (const void* k : ks) {
      cudaError_t e;
      if (MAD_ROWSC_CARVEOUT >= 0) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 MAD_ROWSC_CARVEOUT);
        if (e != cudaSuccess) return e;
      }
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (S)
    k_rows_eval_cs<T, DOF, AD, ENERGY, S0><<<nb, kRowThreads, smem, s>>>(A, *S);
  else if (pairs && vf && kVf)
    k_rows_eval_c<T, DOF, AD, ENERGY, S0, true, kVf><<<nb, kRowThreads, smem, s>>>(A);
  else if (pairs)
    k_rows_eval_c<T, DOF, AD, ENERGY, S0, true, false><<<nb, kRowThreads, smem, s>>>(A);
  else
    k_rows_eval_c<T, DOF, AD, ENERGY, S0, false, false><<<nb, kRowThreads, smem, s>>>(A);
  return cudaGetLastError();
}

template <typename T, int DOF, int S0>
cudaError_t launch_c4(const CArgs<T>& A, const ShardArgs<T>* S, bool pairs, bool vf, int ad,
                      bool energy, int nb, size_t smem, cudaStream_t s, bool set) {
  if (set) {
    for (int a : {kAdReduced, kAdFull, kAdGeneric}) {
      const cudaError_t e = with_ad(a, [&](auto adc) {
        constexpr int AD = decltype(adc)::value;
        const cudaError_t e1 =
            launch_c<T, DOF, AD, true, S0>(A, S, false, false, nb, smem, s, true);
        if (e1 != cudaSuccess) return e1;
        return launch_c<T, DOF, AD, false, S0>(A, S, false, false, nb, smem, s, true);
      });
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  return with_ad(ad, [&](auto adc) {
    constexpr int AD = decltype(adc)::value;
    if (energy) return launch_c<T, DOF, AD, true, S0>(A, S, pairs, vf, nb, smem, s, false);
    return launch_c<T, DOF, AD, false, S0>(A, S, pairs, vf, nb, smem, s, false);
  });
}

template <typename T>
CArgs<T> make_cargs(const RowsLaunch& L, const mad_terms& t, const void* x, void* g, void* H,
                    bool energy) {
  CArgs<T> A;
  A.ctile = L.ctile;
  A.cslots = L.cslots;
  A.ofl_ptr = L.ofl_ptr;
  A.ofl = L.ofl;
  A.x = (const T*)x;
  A.g = (T*)g;
  A.H = (T*)H;
  A.L0 = (const T*)t.spring_rest;
  A.k = (T)t.spring_k;
  A.xt = (const T*)t.inertia_xt;
  A.w = (T)t.inertia_w;
  A.rp = L.rp;
  A.pmask = L.pmask;
  A.prow = L.prow;
  A.pe_col = L.pe_col;
  A.pe_pos = L.pe_pos;
  A.pe_xr = (const T*)L.pe_xr;
  A.kp = (T)t.pair_k;
  A.vrow = L.vrow;
  A.vent = L.vent;
  A.vrec = (const T*)L.vrec;
  A.mask = t.mask;
  A.epart = energy ? L.epart : nullptr;
  A.V = L.V;
  A.s0 = L.s0;
  A.wstage = (int)wstage_elems(L);
  return A;
}

template <typename T, int DOF>
cudaError_t dispatch_c(const RowsLaunch& L, const CArgs<T>& A, const ShardArgs<T>* S, int ad,
                       double* energy, int nb, cudaStream_t s) {
  const size_t smem = rows_smem_bytes(L);
  const bool pairs = !S && L.prow != nullptr;
  // installed vertex-face shares gathered into the rows (their blocks are
  // pair blocks of the active pattern)
  const bool vf = pairs && DOF == 3 && L.vrow != nullptr && (A.mask & MAD_TERM_VF);
  cudaError_t e =
      L.s0 <= 6
          ? launch_c4<T, DOF, 6>(A, S, pairs, vf, ad, energy != nullptr, nb, smem, s, false)
          : launch_c4<T, DOF, kS0Max>(A, S, pairs, vf, ad, energy != nullptr, nb, smem, s,
                                      false);
  if (e != cudaSuccess || !energy) return e;
  k_energy_sum_rows<<<1, 1024, 0, s>>>(L.epart, nb, energy);
  return cudaGetLastError();
}

}  // namespace

template <typename T, int DOF>
cudaError_t rows_eval_compact_t(const RowsLaunch& L, const mad_terms& t, const void* x, void* g,
                                void* H, double* energy, cudaStream_t s) {
  const CArgs<T> A = make_cargs<T>(L, t, x, g, H, energy != nullptr);
  if (L.prow && (t.mask & MAD_TERM_PAIR)) {
    // four blocks per SM (148 on a B200) stride over the live entries
    k_pair_gather<T, DOF><<<kGatherBlocks, 256, 0, s>>>(L.prow + L.V, L.pe_col, (const T*)L.pe_rest,
                                                  (const T*)x, (T*)L.pe_xr);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return dispatch_c<T, DOF>(L, A, nullptr, ad_form(t.flags), energy,
                            rows_blocks(L.V), s);
}

template <typename T, int DOF>
cudaError_t rows_eval_shard_t(const RowsLaunch& L, const mad_terms& t, int nranks,
                              const int32_t* row_begin, int64_t block_lo,
                              const void* const* x_parts, int rank, void* g, void* H,
                              double* energy, cudaStream_t s) {
  const int lo = row_begin[rank], hi = row_begin[rank + 1];
  if (hi <= lo) return energy ? cudaMemsetAsync(energy, 0, sizeof(double), s) : cudaSuccess;
  const CArgs<T> A = make_cargs<T>(L, t, nullptr, g, H, energy != nullptr);
  ShardArgs<T> S{};
  S.tile0 = lo / 32;
  S.row_hi = hi;
  S.own = rank;
  S.nparts = nranks;
  S.hoff = block_lo;
  for (int r = 0; r <= nranks; ++r) S.rbeg[r] = row_begin[r];
  for (int r = 0; r < nranks; ++r) S.xp[r] = (const T*)x_parts[r];
  const int tiles = (hi - lo + 31) / 32;
  const int nb = (tiles + kWarps - 1) / kWarps;
  return dispatch_c<T, DOF>(L, A, &S, ad_form(t.flags), energy, nb, s);
}

template <typename T, int DOF>
cudaError_t rows_compact_limits_t(size_t bytes) {
  CArgs<T> A{};
  cudaError_t e =
      launch_c4<T, DOF, 6>(A, nullptr, false, false, kAdReduced, false, 0, bytes, 0, true);
  if (e != cudaSuccess) return e;
  return launch_c4<T, DOF, kS0Max>(A, nullptr, false, false, kAdReduced, false, 0, bytes, 0, true);
}

template cudaError_t rows_eval_compact_t<float, 2>(const RowsLaunch&, const mad_terms&, const void*,
                                                   void*, void*, double*, cudaStream_t);
template cudaError_t rows_eval_compact_t<float, 3>(const RowsLaunch&, const mad_terms&, const void*,
                                                   void*, void*, double*, cudaStream_t);
template cudaError_t rows_eval_compact_t<double, 2>(const RowsLaunch&, const mad_terms&,
                                                    const void*, void*, void*, double*,
                                                    cudaStream_t);
template cudaError_t rows_eval_compact_t<double, 3>(const RowsLaunch&, const mad_terms&,
                                                    const void*, void*, void*, double*,
                                                    cudaStream_t);
#define MAD_SHARD_INST(T, D)                                                                    \
  template cudaError_t rows_eval_shard_t<T, D>(const RowsLaunch&, const mad_terms&, int,          \
                                               const int32_t*, int64_t, const void* const*, int, \
                                               void*, void*, double*, cudaStream_t);
MAD_SHARD_INST(float, 2)
MAD_SHARD_INST(float, 3)
MAD_SHARD_INST(double, 2)
MAD_SHARD_INST(double, 3)
#undef MAD_SHARD_INST
template cudaError_t rows_compact_limits_t<float, 2>(size_t);
template cudaError_t rows_compact_limits_t<float, 3>(size_t);
template cudaError_t rows_compact_limits_t<double, 2>(size_t);
template cudaError_t rows_compact_limits_t<double, 3>(size_t);

}  // namespace mad
