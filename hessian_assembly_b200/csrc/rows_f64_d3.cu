// rows_f64_d3.cu -- the row-streaming assembly kernels for double with dof 3.
#include "rows_impl.cuh"

namespace mad {
template cudaError_t rows_eval_t<double, 3>(const RowsLaunch&, const mad_terms&, const void*, void*,
                                         void*, double*, cudaStream_t);
template cudaError_t rows_hvp_t<double, 3>(const RowsLaunch&, const mad_terms&, const void*,
                                        const void*, void*, cudaStream_t);
template cudaError_t rows_limits_t<double, 3>(size_t);
}  // namespace mad
