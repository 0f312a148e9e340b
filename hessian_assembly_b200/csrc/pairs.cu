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
// Six kernels and one small memset, stream-ordered, no host synchronisation,
// no block waiting on another block.  One row per thread; rows are grouped in
// blocks of kB rows and super tiles of kSuper blocks, whose counts give every
// block its prefix from a few hundred values.
//   count   pair entries per row (each pair lands in the rows of both ends)
//   sums    entries per block and per super tile
//   scan    prow = exclusive prefix of the row counts
//   fill    each pair writes (partner, pair id) into both rows, counting the
//           row counters back down to zero (they are zero again afterwards)
//   rows    per row, in registers: sort the entries by (partner, pair id),
//           merge them with the mesh row, give every entry the position of
//           its block in the merged row, mark the entries that create a
//           block; new blocks per row, block and super tile; the row's
//           inserted positions as a bit mask (DynBuf::pmask)
//   write   per block: total and prefix of the new-block counts, capacity
//           check, new row_ptr, merged
//           col_idx (mesh columns copied with coalesced loads, each to its
//           shifted place; new columns scattered).  On capacity overflow
//           every block instead copies its share of the previous pattern and
//           pair set into the new buffer.
#include "mad_internal.h"

namespace mad {
namespace {

constexpr int kB = 256;        // rows per block unit (one per thread)
constexpr int kSuper = 8;      // block units per super tile
constexpr int kU = 4;          // block units per block of the row passes (rows per thread)
constexpr int kRegEntries = 4; // pair entries of a row merged in registers
constexpr int kRegMesh = 8;    // mesh columns of a row held in registers
constexpr int kRegNew = 4;     // new columns of a row the write kernel keeps in registers
constexpr int kMapPerWarp = 256;  // mesh columns of 32 rows the write kernel maps in smem
// resident blocks per SM the merge and write kernels are compiled for
#ifndef MAD_PAIR_ROWS_MINB
#define MAD_PAIR_ROWS_MINB 4
#endif
#ifndef MAD_WRITE_MINB
#define MAD_WRITE_MINB 4
#endif

inline unsigned grid_for(int64_t n) {
  int64_t b = (n + kB - 1) / kB;
  if (b < 1) b = 1;
  if (b > 65535LL * 8) b = 65535LL * 8;
  return (unsigned)b;
}

#define GRID_STRIDE(i, n)                                                    \
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (n); \
       i += (int64_t)gridDim.x * blockDim.x)

__device__ __forceinline__ bool pair_ok(int32_t i, int32_t j, int V) {
  return i >= 0 && i < V && j >= 0 && j < V && i != j;
}

// Sum over the block (every thread gets the total).
__device__ __forceinline__ int block_sum(int v) {
  __shared__ int red[kB / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  int s = 0;
#pragma unroll
  for (int w = 0; w < kB / 32; ++w) s += red[w];
  return s;
}

// Two sums over the block at once.
__device__ __forceinline__ int2 block_sum2(int a, int b) {
  __shared__ int2 red2[kB / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red2[threadIdx.x >> 5] = make_int2(a, b);
  __syncthreads();
  int2 s = make_int2(0, 0);
#pragma unroll
  for (int w = 0; w < kB / 32; ++w) {
    s.x += red2[w].x;
    s.y += red2[w].y;
  }
  return s;
}

// Four sums over the block at once.
__device__ __forceinline__ int4 block_sum4(int4 v) {
  __shared__ int4 red4[kB / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
    v.z += __shfl_xor_sync(0xffffffffu, v.z, o);
    v.w += __shfl_xor_sync(0xffffffffu, v.w, o);
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red4[threadIdx.x >> 5] = v;
  __syncthreads();
  int4 s = make_int4(0, 0, 0, 0);
#pragma unroll
  for (int w = 0; w < kB / 32; ++w) {
    s.x += red4[w].x;
    s.y += red4[w].y;
    s.z += red4[w].z;
    s.w += red4[w].w;
  }
  return s;
}

__device__ __forceinline__ int& lane_of(int4& v, int u) {
  return u == 0 ? v.x : (u == 1 ? v.y : (u == 2 ? v.z : v.w));
}

// Exclusive scan of one value per thread over the block; *total = sum.
__device__ __forceinline__ int block_excl_scan(int v, int* total) {
  __shared__ int ws[kB / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();
  if (lane == 31) ws[w] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int q = 0; q < kB / 32; ++q) {
    before += q < w ? ws[q] : 0;
    all += ws[q];
  }
  *total = all;
  return before + incl - v;
}

__global__ void __launch_bounds__(kB) k_pair_count(const int32_t* __restrict__ ij, int n, int V,
                                                   int32_t* cnt, int32_t* status) {
  GRID_STRIDE(p, n) {
    const int32_t i = ij[2 * p], j = ij[2 * p + 1];
    if (!pair_ok(i, j, V)) {
      atomicOr(status, kStatusIndex);
      continue;
    }
    atomicAdd(&cnt[i], 1);
    atomicAdd(&cnt[j], 1);
  }
}

// Entries per block unit (and per super tile): block b covers units
// kU*b .. kU*b + kU-1, thread t row t of each.
__global__ void __launch_bounds__(kB) k_block_sums(const int32_t* __restrict__ cnt, int V,
                                                   int nunits, int32_t* blk, int32_t* sup) {
  const int64_t base = (int64_t)blockIdx.x * kU * kB + threadIdx.x;
  int4 x = make_int4(0, 0, 0, 0);
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int64_t v = base + (int64_t)u * kB;
    lane_of(x, u) = v < V ? cnt[v] : 0;
  }
  int4 sm = block_sum4(x);
  if (threadIdx.x == 0) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int unit = blockIdx.x * kU + u;
      const int su = lane_of(sm, u);
      if (unit < nunits) {
        blk[unit] = su;
        if (su) atomicAdd(&sup[unit / kSuper], su);
      }
    }
  }
}

// prow[v] = sum of cnt[0 .. v); prow[V] = total.  Block b scans rows
// [b*kU*kB, (b+1)*kU*kB), thread t rows kU*t .. kU*t + kU-1 of them.
__global__ void __launch_bounds__(kB) k_scan_rows(const int32_t* __restrict__ cnt, int V,
                                                  const int32_t* __restrict__ sup,
                                                  const int32_t* __restrict__ blk,
                                                  int32_t* __restrict__ prow) {
  const int U0 = blockIdx.x * kU, S = U0 / kSuper;
  const int64_t r0 = (int64_t)blockIdx.x * kU * kB + (int64_t)threadIdx.x * kU;
  int4 c = make_int4(0, 0, 0, 0);
  if (r0 + kU <= V) {
    c = *reinterpret_cast<const int4*>(cnt + r0);  // 16-byte aligned: r0 % 4 == 0
  } else {
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (r0 + u < V) lane_of(c, u) = cnt[r0 + u];
  }
  // counts of every unit before this block: whole super tiles, then the
  // units of this block's super tile
  int s = 0;
  for (int q = threadIdx.x; q < S; q += kB) s += sup[q];
  if ((int)threadIdx.x < U0 - S * kSuper) s += blk[S * kSuper + threadIdx.x];
  const int off = block_sum(s);
  int total;
  int pre = off + block_excl_scan(c.x + c.y + c.z + c.w, &total);
  int4 o;
  o.x = pre;
  o.y = o.x + c.x;
  o.z = o.y + c.y;
  o.w = o.z + c.z;
  if (r0 + kU <= V) {
    *reinterpret_cast<int4*>(prow + r0) = o;
  } else {
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (r0 + u < V) prow[r0 + u] = lane_of(o, u);
  }
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) prow[V] = off + total;
}

template <typename T>
__global__ void __launch_bounds__(kB) k_pair_fill(const int32_t* __restrict__ ij, int n, int V,
                                                  const int32_t* __restrict__ prow,
                                                  int32_t* cnt, int32_t* pe_col,
                                                  int32_t* pe_pid, T* pe_rest,
                                                  const T* __restrict__ rest) {
  GRID_STRIDE(p, n) {
    const int32_t i = ij[2 * p], j = ij[2 * p + 1];
    if (!pair_ok(i, j, V)) continue;
    const T r = rest[p];
    // both slots are claimed before either entry is written, so that the two
    // atomics' round trips overlap
    const int32_t ci = atomicSub(&cnt[i], 1), cj = atomicSub(&cnt[j], 1);
    int32_t s = prow[i] + ci - 1;
    pe_col[s] = j;
    pe_pid[s] = (int32_t)p;
    pe_rest[s] = r;
    s = prow[j] + cj - 1;
    pe_col[s] = i;
    pe_pid[s] = (int32_t)p;
    pe_rest[s] = r;
  }
}

// Merge of one row with more entries, or a longer mesh row, than the
// register path holds: in place in global memory.
// The bit of merged position `pos` in a row's inserted-block mask, or the
// overflow bit when the position does not fit.
__device__ __forceinline__ uint32_t pmask_bit(int pos) {
  return pos < 31 ? (1u << pos) : kPmaskOverflow;
}

// A row's mask word: the inserted positions, or (when one of them is 31 or
// more) the overflow bit and the count of inserted blocks.
__device__ __forceinline__ uint32_t pmask_word(uint32_t bits, int kn) {
  return (bits & kPmaskOverflow) ? (kPmaskOverflow | (uint32_t)kn) : bits;
}

template <typename T>
__device__ int row_merge_global(int32_t b, int32_t e, const int32_t* __restrict__ base_ci,
                                int32_t r0, int32_t blen, int32_t* pe_col, int32_t* pe_pid,
                                int32_t* pe_pos, T* pe_rest, const T* __restrict__ rest,
                                uint32_t& mask) {
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
    if (first && !in_mesh) mask |= pmask_bit(kb + kn);
    pe_rest[i] = rest[pe_pid[i]];
    prev_col = c;
  }
  if (prev_new) ++kn;
  mask = pmask_word(mask, kn);
  return kn;
}

// Position of the j-th (from 0) set bit of m; j < popc(m).
__device__ __forceinline__ int nth_set_bit(unsigned m, int j) {
  int pos = 0;
#pragma unroll
  for (int w = 16; w > 0; w >>= 1) {
    const unsigned low = m & ((1u << w) - 1u);
    const int c = __popc(low);
    if (j >= c) {
      j -= c;
      m >>= w;
      pos += w;
    } else {
      m = low;
    }
  }
  return pos;
}

// One row: sort its entries, merge them with the mesh row, positions;
// returns the row's new blocks.
template <typename T>
__device__ __forceinline__ int merge_row(int32_t b, int32_t e, int32_t r0, int32_t r1,
                                         const int32_t* __restrict__ base_ci, int32_t* pe_col,
                                         int32_t* pe_pid, int32_t* pe_pos, T* pe_rest,
                                         const T* __restrict__ rest, uint32_t& mask) {
  const int32_t blen = r1 - r0;
  const int n = e - b;
  mask = 0u;
  if (n > kRegEntries || blen > kRegMesh)
    return row_merge_global<T>(b, e, base_ci, r0, blen, pe_col, pe_pid, pe_pos, pe_rest, rest,
                               mask);
  int kn = 0;
  int32_t col[kRegEntries], pid[kRegEntries], bc[kRegMesh];
  T rs[kRegEntries];
#pragma unroll
  for (int q = 0; q < kRegEntries; ++q) {
    col[q] = 0x7FFFFFFF;
    pid[q] = 0x7FFFFFFF;
    rs[q] = T(0);
    if (q < n) {
      col[q] = pe_col[b + q];
      pid[q] = pe_pid[b + q];
      rs[q] = pe_rest[b + q];
    }
  }
#pragma unroll
  for (int q = 0; q < kRegMesh; ++q) bc[q] = q < blen ? base_ci[r0 + q] : 0x7FFFFFFF;
  // sort by (col, pid): odd-even transposition, n passes
#pragma unroll
  for (int pass = 0; pass < kRegEntries; ++pass) {
    if (pass >= n) break;
#pragma unroll
    for (int q = pass & 1; q + 1 < kRegEntries; q += 2) {
      const bool sw = col[q] > col[q + 1] || (col[q] == col[q + 1] && pid[q] > pid[q + 1]);
      if (sw) {
        const int32_t tc = col[q], tp = pid[q];
        const T tr = rs[q];
        col[q] = col[q + 1]; pid[q] = pid[q + 1]; rs[q] = rs[q + 1];
        col[q + 1] = tc; pid[q + 1] = tp; rs[q + 1] = tr;
      }
    }
  }
  // position in the merged row = mesh columns below c + new columns below
  // c; entries with the same column (repeated pairs) share it
  int prev_col = -1, kn_group = 0;
#pragma unroll
  for (int q = 0; q < kRegEntries; ++q) {
    if (q < n) {
      const int c = col[q];
      int kb = 0;
      bool in_mesh = false;
#pragma unroll
      for (int m = 0; m < kRegMesh; ++m) {
        kb += bc[m] < c;
        in_mesh |= bc[m] == c;
      }
      const bool first = c != prev_col;
      const bool fresh = first && !in_mesh;
      if (first) kn_group = kn;
      pe_col[b + q] = c;
      pe_pos[b + q] = (kb + kn_group) | (fresh ? kPairNewBlock : 0);
      pe_rest[b + q] = rs[q];
      if (fresh) {
        mask |= pmask_bit(kb + kn_group);
        ++kn;
      }
      prev_col = c;
    }
  }
  mask = pmask_word(mask, kn);
  return kn;
}

// Per row: merge; new blocks per row, block unit and super tile.  Block b
// covers units kU*b .. kU*b + kU-1, thread t row t of each; the row
// pointers of all kU rows are loaded together.  Few rows have pair entries,
// so each warp deals its rows that have them out to its lanes, one per lane,
// and runs the merge once per 32 such rows.
template <typename T>
__global__ void __launch_bounds__(kB, MAD_PAIR_ROWS_MINB) k_pair_rows(int V, int nunits,
                                                  const int32_t* __restrict__ prow,
                                                  const int32_t* __restrict__ base_rp,
                                                  const int32_t* __restrict__ base_ci,
                                                  int32_t* pe_col, int32_t* pe_pid,
                                                  int32_t* pe_pos, T* pe_rest,
                                                  const T* __restrict__ rest, int32_t* newcnt,
                                                  uint32_t* pmask, int32_t* nblk,
                                                  int32_t* nsupc) {
  __shared__ int s_unit[kU];
  const int lane = threadIdx.x & 31;
  const int64_t base = (int64_t)blockIdx.x * kU * kB + threadIdx.x;
  int32_t b[kU], e[kU], r0[kU], r1[kU];
  unsigned has[kU];
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int64_t v = base + (int64_t)u * kB;
    const bool ok = v < V;
    b[u] = ok ? prow[v] : 0;
    e[u] = ok ? prow[v + 1] : 0;
    r0[u] = ok ? base_rp[v] : 0;
    r1[u] = ok ? base_rp[v + 1] : 0;
  }
  if (threadIdx.x < kU) s_unit[threadIdx.x] = 0;
  int total = 0;
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int64_t v = base + (int64_t)u * kB;
    has[u] = __ballot_sync(0xffffffffu, e[u] > b[u]);
    total += __popc(has[u]);
    if (v < V && e[u] <= b[u]) {
      newcnt[v] = 0;
      pmask[v] = 0u;
    }
  }
  __syncthreads();
  for (int round = 0; round * 32 < total; ++round) {
    // this lane's row: the j-th set bit over has[0], has[1], ...
    int j = round * 32 + lane, uu = -1, src = 0;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = __popc(has[u]);
      if (uu < 0 && j < c) {
        uu = u;
        src = nth_set_bit(has[u], j);
      } else if (uu < 0) {
        j -= c;
      }
    }
    int32_t rb = 0, re = 0, rr0 = 0, rr1 = 0;
#pragma unroll
    for (int u = 0; u < kU; ++u) {  // every lane takes part in every shuffle
      const int32_t xb = __shfl_sync(0xffffffffu, b[u], src);
      const int32_t xe = __shfl_sync(0xffffffffu, e[u], src);
      const int32_t x0 = __shfl_sync(0xffffffffu, r0[u], src);
      const int32_t x1 = __shfl_sync(0xffffffffu, r1[u], src);
      if (u == uu) {
        rb = xb;
        re = xe;
        rr0 = x0;
        rr1 = x1;
      }
    }
    if (uu >= 0) {
      const int64_t v = (int64_t)blockIdx.x * kU * kB + (int64_t)uu * kB +
                        (threadIdx.x - lane) + src;
      uint32_t mask;
      const int kn = merge_row<T>(rb, re, rr0, rr1, base_ci, pe_col, pe_pid, pe_pos, pe_rest,
                                  rest, mask);
      newcnt[v] = kn;
      pmask[v] = mask;
      if (kn) atomicAdd(&s_unit[uu], kn);
    }
  }
  __syncthreads();
  if (threadIdx.x < kU) {
    const int unit = blockIdx.x * kU + threadIdx.x;
    const int su = s_unit[threadIdx.x];
    if (unit < nunits) {
      nblk[unit] = su;
      if (su) atomicAdd(&nsupc[unit / kSuper], su);
    }
  }
}

// Block b writes rows [b*kB, (b+1)*kB) of the new pattern (one warp per 32
// rows), or on capacity overflow its share of the copy of the previous state.
// Every load that does not depend on the new-block prefix is issued first,
// so that a block waits for memory about twice.
template <typename T>
__global__ void __launch_bounds__(kB, MAD_WRITE_MINB) k_write_pattern(
    int V, int nnzb_base, int capacity, const int32_t* __restrict__ base_rp,
    const int32_t* __restrict__ base_ci, const int32_t* __restrict__ newcnt,
    int nsup, const int32_t* __restrict__ nsupc, const int32_t* __restrict__ nblk,
    const int32_t* __restrict__ prow,
    const int32_t* __restrict__ pe_col, const int32_t* __restrict__ pe_pos, int32_t* rp,
    int32_t* ci, int32_t* nnzb, int32_t* status,
    // the previous state (prev_prow == nullptr: the mesh pattern, no pairs)
    const int32_t* __restrict__ prev_rp, const int32_t* __restrict__ prev_ci,
    const int32_t* __restrict__ prev_nnzb, const int32_t* __restrict__ prev_prow,
    const int32_t* __restrict__ prev_pe_col, const int32_t* __restrict__ prev_pe_pos,
    const T* __restrict__ prev_pe_rest, const uint32_t* __restrict__ prev_pmask,
    int32_t* out_prow, int32_t* out_pe_col, int32_t* out_pe_pos, T* out_pe_rest,
    uint32_t* out_pmask) {
  constexpr int kBatch = kMapPerWarp / 32;  // mesh columns per lane held in registers
  __shared__ int32_t s_shift[kB + 1];
  __shared__ int32_t s_dst[kB / 32][kMapPerWarp];
  const int64_t R0 = (int64_t)blockIdx.x * kB;
  const int nrows = (int)((V - R0) < kB ? (V - R0) : kB);
  const int r = threadIdx.x;
  const bool valid = r < nrows;
  const int64_t v = R0 + r;
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const bool warp_live = g * 32 < nrows;
  const int gend = g * 32 + 32 < nrows ? g * 32 + 32 : nrows;
  // ---- round 1: row pointers, counts, pair offsets, the warp's column range
  const int32_t b0 = valid ? base_rp[v] : 0x7FFFFFFF;
  const int32_t b1r = valid ? base_rp[v + 1] : 0x7FFFFFFF;
  const int32_t nc0 = valid ? newcnt[v] : 0;
  const int32_t pr0 = valid ? prow[v] : 0;
  const int32_t pr1 = valid ? prow[v + 1] : 0;
  const int32_t a = warp_live ? base_rp[R0 + g * 32] : 0;
  const int32_t z = warp_live ? base_rp[R0 + gend] : 0;
  const int S = blockIdx.x / kSuper;
  int all = 0, bef = 0;
  for (int q = threadIdx.x; q < nsup; q += kB) {
    const int c = nsupc[q];
    all += c;
    if (q < S) bef += c;
  }
  if (r < (int)blockIdx.x - S * kSuper) bef += nblk[S * kSuper + r];
  // ---- round 2: the warp's mesh columns, and for rows that gained blocks
  // their pair entries and their own mesh columns
  const bool mapped = warp_live && z - a <= kMapPerWarp;
  int32_t cv[kBatch];
#pragma unroll
  for (int k = 0; k < kBatch; ++k) {
    const int32_t q = a + 32 * k + lane;
    cv[k] = mapped && q < z ? base_ci[q] : 0;
  }
  int32_t w4[kRegNew], c4[kRegNew], cr[kRegMesh];
#pragma unroll
  for (int m = 0; m < kRegNew; ++m) {
    w4[m] = 0;
    c4[m] = 0;
    if (nc0 && pr0 + m < pr1) {
      w4[m] = pe_pos[pr0 + m];
      c4[m] = pe_col[pr0 + m];
    }
  }
#pragma unroll
  for (int k = 0; k < kRegMesh; ++k) cr[k] = nc0 && b0 + k < b1r ? base_ci[b0 + k] : 0;
  // ---- prefix of the new-block counts; capacity check
  const int2 sums = block_sum2(all, bef);
  const int64_t total = (int64_t)nnzb_base + sums.x;
  if (total > capacity) {
    // overflow: the new buffer becomes a copy of the previous state
    const int32_t nb = *prev_nnzb;
    const int64_t tid = (int64_t)blockIdx.x * kB + threadIdx.x, step = (int64_t)gridDim.x * kB;
    for (int64_t i = tid; i <= V; i += step) {
      rp[i] = prev_rp[i];
      out_prow[i] = prev_prow ? prev_prow[i] : 0;
      if (i < V) out_pmask[i] = prev_pmask ? prev_pmask[i] : 0u;
    }
    for (int64_t i = tid; i < nb; i += step) ci[i] = prev_ci[i];
    if (prev_prow) {
      const int32_t ne = prev_prow[V];
      for (int64_t i = tid; i < ne; i += step) {
        out_pe_col[i] = prev_pe_col[i];
        out_pe_pos[i] = prev_pe_pos[i];
        out_pe_rest[i] = prev_pe_rest[i];
      }
    }
    if (tid == 0) {
      *nnzb = nb;
      atomicOr(status, kStatusCapacity);
    }
    return;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *nnzb = (int32_t)total;
  {
    int tot;
    s_shift[r] = sums.y + block_excl_scan(nc0, &tot);
    if (r == 0) s_shift[kB] = sums.y + tot;
  }
  __syncthreads();
  const int32_t sh = s_shift[r];
  const int32_t nc = s_shift[r + 1] - sh;
  if (valid) rp[v] = b0 + sh;
  if (R0 + nrows == V && r == 0) rp[V] = base_rp[V] + s_shift[kB];
  if (!warp_live) return;
  const unsigned any_new = __ballot_sync(0xffffffffu, nc != 0);
  if (!any_new) {  // one contiguous shifted run
    const int32_t s0 = __shfl_sync(0xffffffffu, sh, 0);
    if (mapped) {
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int32_t q = a + 32 * k + lane;
        if (q < z) ci[q + s0] = cv[k];
      }
    } else {
      for (int32_t q = a + lane; q < z; q += 32) ci[q + s0] = base_ci[q];
    }
    return;
  }
  // each lane's new columns (in column order), placed at their merged
  // positions; the first kRegNew kept in registers
  int32_t nw[kRegNew];
#pragma unroll
  for (int k = 0; k < kRegNew; ++k) nw[k] = 0x7FFFFFFF;
  const int32_t o0 = b0 + sh;
  if (valid && nc) {
    int k = 0;
#pragma unroll
    for (int m = 0; m < kRegNew; ++m) {
      if (w4[m] & kPairNewBlock) {
        ci[o0 + (w4[m] & kPairPosMask)] = c4[m];
#pragma unroll
        for (int q = 0; q < kRegNew; ++q)
          if (q == k) nw[q] = c4[m];
        ++k;
      }
    }
    for (int32_t e = pr0 + kRegNew; e < pr1; ++e) {
      const int32_t w = pe_pos[e];
      if (w & kPairNewBlock) {
        const int32_t c = pe_col[e];
        ci[o0 + (w & kPairPosMask)] = c;
#pragma unroll
        for (int q = 0; q < kRegNew; ++q)
          if (q == k) nw[q] = c;
        ++k;
      }
    }
  }
  // the new place of a mesh column of this lane's row: after the new
  // columns that sort before it
  auto new_place = [&](int32_t c, int32_t o) {
#pragma unroll
    for (int k = 0; k < kRegNew; ++k) o += nw[k] < c;
    if (nc > kRegNew) {  // the columns past the registers
      int k = 0;
      for (int32_t e = pr0; e < pr1; ++e)
        if (pe_pos[e] & kPairNewBlock) {
          if (k >= kRegNew && pe_col[e] < c) ++o;
          ++k;
        }
    }
    return o;
  };
  if (mapped) {
    // owners write the destination of each of their mesh columns into the
    // warp's map; then the loaded columns are stored
    int32_t* map = s_dst[g];
    if (valid) {
      if (nc == 0) {
        for (int32_t q = b0; q < b1r; ++q) map[q - a] = q + sh;
      } else {
#pragma unroll
        for (int k = 0; k < kRegMesh; ++k)
          if (b0 + k < b1r) map[b0 + k - a] = new_place(cr[k], b0 + k + sh);
        for (int32_t q = b0 + kRegMesh; q < b1r; ++q) map[q - a] = new_place(base_ci[q], q + sh);
      }
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int32_t q = a + 32 * k + lane;
      if (q < z) ci[map[q - a]] = cv[k];
    }
    return;
  }
  // long rows: look up each column's row within the warp
  for (int32_t qb = a; qb < z; qb += 32) {
    const int32_t q = qb + lane;
    const int32_t c = q < z ? base_ci[q] : 0;
    int lo = 0;  // the last lane whose row starts at or before q
#pragma unroll
    for (int st = 16; st > 0; st >>= 1) {
      const int32_t bs = __shfl_sync(0xffffffffu, b0, lo + st);
      if (bs <= q) lo += st;
    }
    // the owner's new columns that sort before c, read by shuffles
    int32_t extra = 0;
#pragma unroll
    for (int k = 0; k < kRegNew; ++k) extra += __shfl_sync(0xffffffffu, nw[k], lo) < c;
    const int32_t shr = __shfl_sync(0xffffffffu, sh, lo);
    const int32_t ncr = __shfl_sync(0xffffffffu, nc, lo);
    if (q < z) {
      int32_t dst = q + shr + extra;
      if (ncr > kRegNew) {
        const int64_t vr = R0 + g * 32 + lo;
        int k = 0;
        for (int32_t e = prow[vr]; e < prow[vr + 1]; ++e)
          if (pe_pos[e] & kPairNewBlock) {
            if (k >= kRegNew && pe_col[e] < c) ++dst;
            ++k;
          }
      }
      ci[dst] = c;
    }
  }
}

#define CK(x)                              \
  do {                                     \
    cudaError_t e_ = (x);                  \
    if (e_ != cudaSuccess) return e_;      \
  } while (0)

int n_blocks(int V) { return V > 0 ? (V + kB - 1) / kB : 1; }
int n_super(int V) { return (n_blocks(V) + kSuper - 1) / kSuper; }

template <typename T>
cudaError_t add_pairs_t(const PairLaunch& L, int n, const int32_t* ij, const void* rest,
                        const DynBuf& nb, const DynBuf* prev, cudaStream_t s) {
  const int V = L.V;
  const int nblocks = n_blocks(V), nsup = n_super(V);
  // scratch: [super entries | super new blocks | block entries | block new blocks]
  int32_t* sup_c = L.tsum;
  int32_t* sup_n = sup_c + nsup;
  int32_t* blk_c = sup_n + nsup;
  int32_t* blk_n = blk_c + nblocks;
  CK(cudaMemsetAsync(sup_c, 0, sizeof(int32_t) * 2 * nsup, s));
  k_pair_count<<<grid_for(n), kB, 0, s>>>(ij, n, V, L.cnt, L.status);
  CK(cudaGetLastError());
  const int ngroups = (nblocks + kU - 1) / kU;
  k_block_sums<<<ngroups, kB, 0, s>>>(L.cnt, V, nblocks, blk_c, sup_c);
  CK(cudaGetLastError());
  k_scan_rows<<<ngroups, kB, 0, s>>>(L.cnt, V, sup_c, blk_c, nb.prow);
  CK(cudaGetLastError());
  k_pair_fill<T><<<grid_for(n), kB, 0, s>>>(ij, n, V, nb.prow, L.cnt, nb.pe_col, L.pe_pid,
                                            (T*)nb.pe_rest, (const T*)rest);
  CK(cudaGetLastError());
  k_pair_rows<T><<<ngroups, kB, 0, s>>>(V, nblocks, nb.prow, L.base_rp, L.base_ci, nb.pe_col,
                                        L.pe_pid, nb.pe_pos, (T*)nb.pe_rest, (const T*)rest,
                                        L.newcnt, nb.pmask, blk_n, sup_n);
  CK(cudaGetLastError());
  if (prev)
    k_write_pattern<T><<<nblocks, kB, 0, s>>>(
        V, L.nnzb_base, L.capacity, L.base_rp, L.base_ci, L.newcnt, nsup, sup_n, blk_n,
        nb.prow, nb.pe_col, nb.pe_pos, nb.rp, nb.ci, nb.nnzb, L.status, prev->rp, prev->ci,
        prev->nnzb, prev->prow, prev->pe_col, prev->pe_pos, (const T*)prev->pe_rest,
        prev->pmask, nb.prow, nb.pe_col, nb.pe_pos, (T*)nb.pe_rest, nb.pmask);
  else
    k_write_pattern<T><<<nblocks, kB, 0, s>>>(
        V, L.nnzb_base, L.capacity, L.base_rp, L.base_ci, L.newcnt, nsup, sup_n, blk_n,
        nb.prow, nb.pe_col, nb.pe_pos, nb.rp, nb.ci, nb.nnzb, L.status, L.base_rp, L.base_ci,
        L.base_nnzb_dev, nullptr, nullptr, nullptr, nullptr, nullptr, nb.prow, nb.pe_col,
        nb.pe_pos, (T*)nb.pe_rest, nb.pmask);
  return cudaGetLastError();
}

}  // namespace

size_t pair_scratch_elems(int V) { return 2 * (size_t)n_super(V) + 2 * (size_t)n_blocks(V); }

cudaError_t launch_add_pairs(const PairLaunch& L, int n, const int32_t* ij, const void* rest,
                             const DynBuf& nb, const DynBuf* prev, cudaStream_t s) {
  cudaError_t e = L.dtype == MAD_F64 ? add_pairs_t<double>(L, n, ij, rest, nb, prev, s)
                                     : add_pairs_t<float>(L, n, ij, rest, nb, prev, s);
  // the row counters must be zero for the next call, whatever failed
  if (e != cudaSuccess) cudaMemsetAsync(L.cnt, 0, sizeof(int32_t) * (L.V + 1), s);
  return e;
}

}  // namespace mad
