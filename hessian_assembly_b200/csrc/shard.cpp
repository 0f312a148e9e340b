// shard.cpp -- host-side planning of owner-computes sharding: which rows of
// the block-CSR Hessian each GPU owns, and which positions of other GPUs'
// vertices those rows read.
//
// The page "Locality-Aware Automatic Differentiation on the GPU for
// Mesh-Based Computations" runs on one GPU; sharding one mesh across GPUs
// follows from its own structure (section 方法, key design 2): a term is
// evaluated by every owner of one of its vertices and writes only owned
// rows, so shards need no reduction, only the positions of the vertices
// across their borders.  Rows are split into contiguous ranges (so each
// shard's Hessian values are one contiguous range of blocks) balanced by
// block count, at multiples of 32 rows (the row kernels' tile).
#include <algorithm>
#include <cstdint>
#include <vector>

#include "../../include/mad.h"

namespace {

constexpr int kTile = 32;

// Mesh-pattern row lengths (diagonal + distinct face neighbours) and, when
// `adj` is non-null, the sorted neighbours of every row (CSR in adj_ptr/adj).
bool mesh_rows(int32_t V, int32_t nF, const int32_t* F, std::vector<int64_t>& row_ptr,
               std::vector<int32_t>* adj) {
  std::vector<uint64_t> keys;
  keys.reserve((size_t)nF * 6);
  for (int64_t f = 0; f < nF; ++f) {
    const int32_t a = F[3 * f], b = F[3 * f + 1], c = F[3 * f + 2];
    if (a < 0 || a >= V || b < 0 || b >= V || c < 0 || c >= V || a == b || b == c || a == c)
      return false;
    const int32_t v[3] = {a, b, c};
    for (int s = 0; s < 3; ++s) {
      const uint64_t p = (uint32_t)v[s], q = (uint32_t)v[(s + 1) % 3];
      keys.push_back(p << 32 | q);
      keys.push_back(q << 32 | p);
    }
  }
  std::sort(keys.begin(), keys.end());
  keys.erase(std::unique(keys.begin(), keys.end()), keys.end());
  row_ptr.assign((size_t)V + 1, 0);
  for (uint64_t k : keys) ++row_ptr[(k >> 32) + 1];
  for (int32_t v = 0; v < V; ++v) row_ptr[v + 1] += row_ptr[v] + 1;  // + the diagonal
  if (adj) {
    adj->resize(keys.size());
    for (size_t q = 0; q < keys.size(); ++q) (*adj)[q] = (int32_t)(keys[q] & 0xFFFFFFFFu);
  }
  return true;
}

}  // namespace

extern "C" mad_status mad_shard_plan(int32_t V, int32_t nF, const int32_t* F, int32_t nranks,
                                     int32_t* row_begin, int64_t* block_begin) {
  if (V < 0 || nF < 0 || (nF > 0 && !F) || nranks < 1 || nranks > MAD_MAX_SHARDS || !row_begin)
    return MAD_ERR_INVALID_ARG;
  std::vector<int64_t> rp;
  if (!mesh_rows(V, nF, F, rp, nullptr)) return MAD_ERR_INVALID_ARG;
  const int64_t nnzb = rp[V];
  row_begin[0] = 0;
  for (int r = 1; r < nranks; ++r) {
    // the first tile boundary whose blocks before it reach r / nranks of all
    const int64_t target = (nnzb * r + nranks / 2) / nranks;
    int32_t b = row_begin[r - 1];
    while (b < V && rp[b] < target) b = std::min<int64_t>((int64_t)b + kTile, V);
    // a boundary inside the last tile of the mesh is the end of the mesh
    row_begin[r] = b;
  }
  row_begin[nranks] = V;
  if (block_begin)
    for (int r = 0; r <= nranks; ++r) block_begin[r] = rp[row_begin[r]];
  return MAD_OK;
}

extern "C" mad_status mad_shard_halo(int32_t V, int32_t nF, const int32_t* F, int32_t row_lo,
                                     int32_t row_hi, int32_t* n_halo, int32_t* halo,
                                     int32_t cap) {
  if (V < 0 || nF < 0 || (nF > 0 && !F) || row_lo < 0 || row_hi < row_lo || row_hi > V ||
      !n_halo || cap < 0 || (cap > 0 && !halo))
    return MAD_ERR_INVALID_ARG;
  std::vector<int64_t> rp;
  std::vector<int32_t> adj;
  if (!mesh_rows(V, nF, F, rp, &adj)) return MAD_ERR_INVALID_ARG;
  // adj holds the off-diagonal neighbours row by row: row v's start is
  // rp[v] - v (rp counts the diagonals too)
  std::vector<int32_t> out;
  for (int32_t v = row_lo; v < row_hi; ++v)
    for (int64_t q = rp[v] - v; q < rp[v + 1] - (v + 1); ++q) {
      const int32_t u = adj[q];
      if (u < row_lo || u >= row_hi) out.push_back(u);
    }
  std::sort(out.begin(), out.end());
  out.erase(std::unique(out.begin(), out.end()), out.end());
  *n_halo = (int32_t)out.size();
  if ((int64_t)out.size() > cap) return cap == 0 ? MAD_OK : MAD_ERR_CAPACITY;
  std::copy(out.begin(), out.end(), halo);
  return MAD_OK;
}
