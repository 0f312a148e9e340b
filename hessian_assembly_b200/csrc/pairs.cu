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
//           block; new blocks per row, block and super tile
//   write   per block: total and prefix of the new-block counts, capacity
//           check, new row_ptr, merged
//           col_idx (mesh columns copied with coalesced loads, each to its
//           shifted place; new columns scattered).  On capacity overflow
//           every block instead copies its share of the previous pattern and
//           pair set into the new buffer.
#include "mad_internal.h"

namespace mad {
namespace {

constexpr int kB = 256;        // rows per block (one per thread)
constexpr int kSuper = 8;      // blocks per super tile
constexpr int kRegEntries = 4; // pair entries of a row merged in registers
constexpr int kRegMesh = 8;    // mesh columns of a row held in registers
constexpr int kRegNew = 4;     // new columns of a row the write kernel keeps in registers
constexpr int kMapPerWarp = 512;  // mesh columns of 32 rows the write kernel maps in smem

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

// Sum of the counts of every block before this one: whole super tiles, then
// the blocks of this block's super tile.
__device__ __forceinline__ int blocks_before(const int32_t* __restrict__ sup,
                                             const int32_t* __restrict__ blk) {
  const int b = blockIdx.x, S = b / kSuper;
  int s = 0;
  for (int q = threadIdx.x; q < S; q += kB) s += sup[q];
  if ((int)threadIdx.x < b - S * kSuper) s += blk[S * kSuper + threadIdx.x];
  return block_sum(s);
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

__global__ void __launch_bounds__(kB) k_block_sums(const int32_t* __restrict__ cnt, int V,
                                                   int32_t* blk, int32_t* sup) {
  const int64_t v = (int64_t)blockIdx.x * kB + threadIdx.x;
  const int s = block_sum(v < V ? cnt[v] : 0);
  if (threadIdx.x == 0) {
    blk[blockIdx.x] = s;
    if (s) atomicAdd(&sup[blockIdx.x / kSuper], s);
  }
}

// prow[v] = sum of cnt[0 .. v); prow[V] = total.
__global__ void __launch_bounds__(kB) k_scan_rows(const int32_t* __restrict__ cnt, int V,
                                                  const int32_t* __restrict__ sup,
                                                  const int32_t* __restrict__ blk,
                                                  int32_t* __restrict__ prow) {
  const int off = blocks_before(sup, blk);
  const int64_t v = (int64_t)blockIdx.x * kB + threadIdx.x;
  const int c = v < V ? cnt[v] : 0;
  int total;
  const int pre = off + block_excl_scan(c, &total);
  if (v < V) prow[v] = pre;
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
    int32_t s = prow[i] + atomicSub(&cnt[i], 1) - 1;
    pe_col[s] = j;
    pe_pid[s] = (int32_t)p;
    pe_rest[s] = r;
    s = prow[j] + atomicSub(&cnt[j], 1) - 1;
    pe_col[s] = i;
    pe_pid[s] = (int32_t)p;
    pe_rest[s] = r;
  }
}

// Merge of one row with more entries, or a longer mesh row, than the
// register path holds: in place in global memory.
template <typename T>
__device__ int row_merge_global(int32_t b, int32_t e, const int32_t* __restrict__ base_ci,
                                int32_t r0, int32_t blen, int32_t* pe_col, int32_t* pe_pid,
                                int32_t* pe_pos, T* pe_rest, const T* __restrict__ rest) {
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
    pe_rest[i] = rest[pe_pid[i]];
    prev_col = c;
  }
  if (prev_new) ++kn;
  return kn;
}

// Per row: sort, merge, positions; new blocks per row, block and super tile.
template <typename T>
__global__ void __launch_bounds__(kB) k_pair_rows(int V,
                                                  const int32_t* __restrict__ prow,
                                                  const int32_t* __restrict__ base_rp,
                                                  const int32_t* __restrict__ base_ci,
                                                  int32_t* pe_col, int32_t* pe_pid,
                                                  int32_t* pe_pos, T* pe_rest,
                                                  const T* __restrict__ rest, int32_t* newcnt,
                                                  int32_t* nblk, int32_t* nsupc) {
  const int64_t v = (int64_t)blockIdx.x * kB + threadIdx.x;
  int kn = 0;
  // both row pointers at once: the mesh row is loaded in the same round trip
  // as the pair entries
  const int32_t b = v < V ? prow[v] : 0, e = v < V ? prow[v + 1] : 0;
  const int32_t r0 = v < V ? base_rp[v] : 0, r1 = v < V ? base_rp[v + 1] : 0;
  if (e > b) {
    const int32_t blen = r1 - r0;
    const int n = e - b;
    if (n <= kRegEntries && blen <= kRegMesh) {
      int32_t col[kRegEntries], pid[kRegEntries], bc[kRegMesh];
      T rs[kRegEntries];
#pragma unroll
      for (int q = 0; q < kRegEntries; ++q) {
        col[q] = 0x7FFFFFFF;
        pid[q] = 0x7FFFFFFF;
        if (q < n) {
          col[q] = pe_col[b + q];
          pid[q] = pe_pid[b + q];
        }
      }
#pragma unroll
      for (int q = 0; q < kRegMesh; ++q) bc[q] = q < blen ? base_ci[r0 + q] : 0x7FFFFFFF;
#pragma unroll
      for (int q = 0; q < kRegEntries; ++q) rs[q] = q < n ? pe_rest[b + q] : T(0);
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
      // position in the merged row = mesh columns below c + new columns
      // below c; entries with the same column (repeated pairs) share it
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
          if (fresh) ++kn;
          prev_col = c;
        }
      }
    } else {
      kn = row_merge_global<T>(b, e, base_ci, r0, blen, pe_col, pe_pid, pe_pos, pe_rest, rest);
    }
  }
  if (v < V) newcnt[v] = kn;
  const int s = block_sum(kn);
  if (threadIdx.x == 0) {
    nblk[blockIdx.x] = s;
    if (s) atomicAdd(&nsupc[blockIdx.x / kSuper], s);
  }
}

// Block b writes rows [b*kB, (b+1)*kB) of the new pattern (one warp per 32
// rows), or on capacity overflow its share of the copy of the previous state.
template <typename T>
__global__ void __launch_bounds__(kB, 4) k_write_pattern(
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
    const T* __restrict__ prev_pe_rest, int32_t* out_prow, int32_t* out_pe_col,
    int32_t* out_pe_pos, T* out_pe_rest) {
  __shared__ int32_t s_shift[kB + 1];
  __shared__ int32_t s_dst[kB / 32][kMapPerWarp];
  const int64_t R0 = (int64_t)blockIdx.x * kB;
  const int nrows = (int)((V - R0) < kB ? (V - R0) : kB);
  const int r = threadIdx.x;
  const bool valid = r < nrows;
  const int64_t v = R0 + r;
  // the row's own loads first: they do not depend on the counts below
  const int32_t b0 = valid ? base_rp[v] : 0x7FFFFFFF;
  const int32_t nc0 = valid ? newcnt[v] : 0;
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int gend = g * 32 + 32 < nrows ? g * 32 + 32 : nrows;
  const int32_t z = g * 32 < nrows ? base_rp[R0 + gend] : 0;
  // the row's pair entries (the new-block count is known only after the scan)
  int32_t pr0 = 0, pr1 = 0;
  if (valid && nc0) {
    pr0 = prow[v];
    pr1 = prow[v + 1];
  }
  // total new blocks (capacity check) and the new blocks of earlier blocks
  int2 sums;
  {
    const int S = blockIdx.x / kSuper;
    int all = 0, bef = 0;
    for (int q = threadIdx.x; q < nsup; q += kB) {
      const int c = nsupc[q];
      all += c;
      if (q < S) bef += c;
    }
    if (r < (int)blockIdx.x - S * kSuper) bef += nblk[S * kSuper + r];
    sums = block_sum2(all, bef);
  }
  const int64_t total = (int64_t)nnzb_base + sums.x;
  if (total > capacity) {
    // overflow: the new buffer becomes a copy of the previous state
    const int32_t nb = *prev_nnzb;
    const int64_t tid = (int64_t)blockIdx.x * kB + threadIdx.x, step = (int64_t)gridDim.x * kB;
    for (int64_t i = tid; i <= V; i += step) {
      rp[i] = prev_rp[i];
      out_prow[i] = prev_prow ? prev_prow[i] : 0;
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
  // one warp per 32 rows
  if (g * 32 >= nrows) return;
  const int32_t a = __shfl_sync(0xffffffffu, b0, 0);
  const unsigned any_new = __ballot_sync(0xffffffffu, nc != 0);
  if (!any_new) {  // one contiguous shifted run
    const int32_t s0 = __shfl_sync(0xffffffffu, sh, 0);
    for (int32_t q = a + lane; q < z; q += 32) ci[q + s0] = base_ci[q];
    return;
  }
  // each lane's new columns (in column order), placed at their merged
  // positions and kept in registers
  int32_t nw[kRegNew];
#pragma unroll
  for (int k = 0; k < kRegNew; ++k) nw[k] = 0x7FFFFFFF;
  const int32_t o0 = b0 + sh;
  if (valid && nc) {
    // the first kRegNew entries in one round trip, the rest one by one
    int32_t w4[kRegNew], c4[kRegNew];
#pragma unroll
    for (int m = 0; m < kRegNew; ++m) {
      w4[m] = 0;
      c4[m] = 0;
      if (pr0 + m < pr1) {
        w4[m] = pe_pos[pr0 + m];
        c4[m] = pe_col[pr0 + m];
      }
    }
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
  // the new place of every mesh column of a row that gained blocks: after
  // the new columns that sort before it
  auto new_place = [&](int32_t q, int32_t c, int32_t o) {
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
  if (z - a <= kMapPerWarp) {
    // owners write the destination of each of their mesh columns into the
    // warp's map; then the copy runs with coalesced loads
    int32_t* map = s_dst[g];
    const int32_t nxt = __shfl_down_sync(0xffffffffu, b0, 1);
    const int32_t b1 = (lane == 31 || g * 32 + lane + 1 >= gend) ? z : nxt;
    if (valid) {
      if (nc == 0) {
        for (int32_t q = b0; q < b1; ++q) map[q - a] = q + sh;
      } else {
        // the row's columns in one round trip (the first kRegMesh of them)
        int32_t cr[kRegMesh];
#pragma unroll
        for (int k = 0; k < kRegMesh; ++k) cr[k] = b0 + k < b1 ? base_ci[b0 + k] : 0;
#pragma unroll
        for (int k = 0; k < kRegMesh; ++k)
          if (b0 + k < b1) map[b0 + k - a] = new_place(b0 + k, cr[k], b0 + k + sh);
        for (int32_t q = b0 + kRegMesh; q < b1; ++q)
          map[q - a] = new_place(q, base_ci[q], q + sh);
      }
    }
    __syncwarp();
    // the copy, loads of a batch first
    constexpr int kBatch = 8;
    for (int32_t qb = a; qb < z; qb += 32 * kBatch) {
      int32_t cv[kBatch], dv[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int32_t q = qb + 32 * k + lane;
        if (q < z) {
          cv[k] = base_ci[q];
          dv[k] = map[q - a];
        }
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int32_t q = qb + 32 * k + lane;
        if (q < z) ci[dv[k]] = cv[k];
      }
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
  k_block_sums<<<nblocks, kB, 0, s>>>(L.cnt, V, blk_c, sup_c);
  CK(cudaGetLastError());
  k_scan_rows<<<nblocks, kB, 0, s>>>(L.cnt, V, sup_c, blk_c, nb.prow);
  CK(cudaGetLastError());
  k_pair_fill<T><<<grid_for(n), kB, 0, s>>>(ij, n, V, nb.prow, L.cnt, nb.pe_col, L.pe_pid,
                                            (T*)nb.pe_rest, (const T*)rest);
  CK(cudaGetLastError());
  k_pair_rows<T><<<nblocks, kB, 0, s>>>(V, nb.prow, L.base_rp, L.base_ci, nb.pe_col,
                                        L.pe_pid, nb.pe_pos, (T*)nb.pe_rest, (const T*)rest,
                                        L.newcnt, blk_n, sup_n);
  CK(cudaGetLastError());
  if (prev)
    k_write_pattern<T><<<nblocks, kB, 0, s>>>(
        V, L.nnzb_base, L.capacity, L.base_rp, L.base_ci, L.newcnt, nsup, sup_n, blk_n,
        nb.prow, nb.pe_col, nb.pe_pos, nb.rp, nb.ci, nb.nnzb, L.status, prev->rp, prev->ci,
        prev->nnzb, prev->prow, prev->pe_col, prev->pe_pos, (const T*)prev->pe_rest, nb.prow,
        nb.pe_col, nb.pe_pos, (T*)nb.pe_rest);
  else
    k_write_pattern<T><<<nblocks, kB, 0, s>>>(
        V, L.nnzb_base, L.capacity, L.base_rp, L.base_ci, L.newcnt, nsup, sup_n, blk_n,
        nb.prow, nb.pe_col, nb.pe_pos, nb.rp, nb.ci, nb.nnzb, L.status, L.base_rp, L.base_ci,
        L.base_nnzb_dev, nullptr, nullptr, nullptr, nullptr, nb.prow, nb.pe_col, nb.pe_pos,
        (T*)nb.pe_rest);
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
