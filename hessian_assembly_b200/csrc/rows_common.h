// rows_common.h -- launch geometry of the row-streaming assembly kernels
// (rows_impl.cuh) shared with their host-side dispatch (rows.cu).
#pragma once

#include <stddef.h>

#include "mad_internal.h"

namespace mad {

constexpr int kRowThreads = 128;  // 4 warps per block
constexpr int kWarps = kRowThreads / 32;

// Staging elements per warp: 32 mesh rows of s0 + 1 blocks, plus, when the
// active pattern has inserted pair blocks, kWarpSpare blocks for them
// (shared by the warp's rows; rows past the reserve are assembled in place),
// rounded to 16 bytes, plus 16 bytes of alignment room.
constexpr int kWarpSpare = 16;
inline size_t wstage_elems(const RowsLaunch& L) {
  const int vec = L.dtype == MAD_F64 ? 2 : 4;
  const int blocks = 32 * (L.s0 + 1) + (L.rho > 0 ? kWarpSpare : 0);
  const int elems = blocks * L.dof * L.dof;
  return (size_t)(((elems + vec - 1) / vec) * vec + vec);
}

// One (dtype, dof) of the row kernels; defined in rows_impl.cuh and
// instantiated once per unit rows_<dtype>_d<dof>.cu.
template <typename T, int DOF>
cudaError_t rows_eval_t(const RowsLaunch& L, const mad_terms& t, const void* x, void* g, void* H,
                        double* energy, cudaStream_t s);
template <typename T, int DOF>
cudaError_t rows_hvp_t(const RowsLaunch& L, const mad_terms& t, const void* x, const void* v,
                       void* y, cudaStream_t s);
template <typename T, int DOF>
cudaError_t rows_limits_t(size_t bytes);
// The same assembly for edge and vertex terms on the mesh pattern, driven by
// the compact slot tables (rows_compact.cu); needs L.cslots.
template <typename T, int DOF>
cudaError_t rows_eval_compact_t(const RowsLaunch& L, const mad_terms& t, const void* x, void* g,
                                void* H, double* energy, cudaStream_t s);
template <typename T, int DOF>
cudaError_t rows_compact_limits_t(size_t bytes);
// The rows [row_begin[rank], row_begin[rank+1]) of the same assembly, with
// the positions of shard r at x_parts[r]; g and H hold the shard's rows and
// blocks only (H's first block is block_lo of the mesh pattern).
template <typename T, int DOF>
cudaError_t rows_eval_shard_t(const RowsLaunch& L, const mad_terms& t, int nranks,
                              const int32_t* row_begin, int64_t block_lo,
                              const void* const* x_parts, int rank, void* g, void* H,
                              double* energy, cudaStream_t s);

}  // namespace mad
