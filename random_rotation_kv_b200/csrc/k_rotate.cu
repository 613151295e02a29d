// Instantiates the rotate kernels for the three input element types.
#include "quant_kernels.cuh"

namespace rrq {
template cudaError_t rotate_typed<__half>(const __half*, int64_t, int, uint64_t, int, float, float*,
                                          cudaStream_t);
template cudaError_t rotate_typed<__nv_bfloat16>(const __nv_bfloat16*, int64_t, int, uint64_t, int,
                                                 float, float*, cudaStream_t);
template cudaError_t rotate_typed<float>(const float*, int64_t, int, uint64_t, int, float, float*,
                                         cudaStream_t);
}  // namespace rrq
