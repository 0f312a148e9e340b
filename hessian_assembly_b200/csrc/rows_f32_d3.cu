// rows_f32_d3.cu -- the row-streaming assembly kernels for float with dof 3.
#include "rows_impl.cuh"

namespace mad {
template cudaError_t rows_eval_t<float, 3>(const RowsLaunch&, const mad_terms&, const void*, void*,
                                         void*, double*, cudaStream_t);
template cudaError_t rows_hvp_t<float, 3>(const RowsLaunch&, const mad_terms&, const void*,
                                        const void*, void*, cudaStream_t);
template cudaError_t rows_limits_t<float, 3>(size_t);
}  // namespace mad
