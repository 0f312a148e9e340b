// rows.cu -- host-side dispatch of the row-streaming assembly kernels
// (rows_impl.cuh) by dtype and dof.
#include <algorithm>

#include "rows_common.h"

namespace mad {

int rows_blocks(int V) {
  const int tiles = (V + 31) / 32;
  return std::max(1, (tiles + kWarps - 1) / kWarps);
}

size_t rows_smem_bytes(const RowsLaunch& L) {
  return (size_t)kWarps * wstage_elems(L) * (L.dtype == MAD_F64 ? 8 : 4);
}

cudaError_t rows_set_smem_limits(int dtype, int dof, size_t bytes) {
  cudaError_t e;
  if (dtype == MAD_F64) {
    e = dof == 2 ? rows_limits_t<double, 2>(bytes) : rows_limits_t<double, 3>(bytes);
    if (e != cudaSuccess) return e;
    return dof == 2 ? rows_compact_limits_t<double, 2>(bytes)
                    : rows_compact_limits_t<double, 3>(bytes);
  }
  e = dof == 2 ? rows_limits_t<float, 2>(bytes) : rows_limits_t<float, 3>(bytes);
  if (e != cudaSuccess) return e;
  return dof == 2 ? rows_compact_limits_t<float, 2>(bytes) : rows_compact_limits_t<float, 3>(bytes);
}

cudaError_t launch_rows_eval(const RowsLaunch& L, const mad_terms& t, const void* x, void* g,
                             void* H, double* energy, cudaStream_t s) {
  if (L.V == 0) {
    if (energy) return cudaMemsetAsync(energy, 0, sizeof(double), s);
    return cudaSuccess;
  }
  if (L.dtype == MAD_F64)
    return L.dof == 2 ? rows_eval_t<double, 2>(L, t, x, g, H, energy, s)
                      : rows_eval_t<double, 3>(L, t, x, g, H, energy, s);
  return L.dof == 2 ? rows_eval_t<float, 2>(L, t, x, g, H, energy, s)
                    : rows_eval_t<float, 3>(L, t, x, g, H, energy, s);
}

cudaError_t launch_rows_hvp(const RowsLaunch& L, const mad_terms& t, const void* x,
                            const void* v, void* y, cudaStream_t s) {
  if (L.V == 0) return cudaSuccess;
  if (L.dtype == MAD_F64)
    return L.dof == 2 ? rows_hvp_t<double, 2>(L, t, x, v, y, s)
                      : rows_hvp_t<double, 3>(L, t, x, v, y, s);
  return L.dof == 2 ? rows_hvp_t<float, 2>(L, t, x, v, y, s)
                    : rows_hvp_t<float, 3>(L, t, x, v, y, s);
}

cudaError_t launch_rows_eval_shard(const RowsLaunch& L, const mad_terms& t, int nranks,
                                   const int32_t* row_begin, int64_t block_lo,
                                   const void* const* x_parts, int rank, void* g, void* H,
                                   double* energy, cudaStream_t s) {
  if (L.dtype == MAD_F64)
    return L.dof == 2 ? rows_eval_shard_t<double, 2>(L, t, nranks, row_begin, block_lo, x_parts,
                                                     rank, g, H, energy, s)
                      : rows_eval_shard_t<double, 3>(L, t, nranks, row_begin, block_lo, x_parts,
                                                     rank, g, H, energy, s);
  return L.dof == 2 ? rows_eval_shard_t<float, 2>(L, t, nranks, row_begin, block_lo, x_parts, rank,
                                                  g, H, energy, s)
                    : rows_eval_shard_t<float, 3>(L, t, nranks, row_begin, block_lo, x_parts, rank,
                                                  g, H, energy, s);
}

}  // namespace mad
