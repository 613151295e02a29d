// Instantiates the bf16-output decode kernels (split per element type to build in parallel).
#include "batch_kernels.cuh"

namespace rrq {
template cudaError_t decode_typed<__nv_bfloat16>(const uint8_t*, const float*, int64_t, int,
                                        const QuantParams&, __nv_bfloat16*, cudaStream_t);
}  // namespace rrq
