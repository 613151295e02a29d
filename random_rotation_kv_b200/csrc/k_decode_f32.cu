// Instantiates the f32-output decode kernels (split per element type to build in parallel).
#include "batch_kernels.cuh"

namespace rrq {
template cudaError_t decode_typed<float>(const uint8_t*, const float*, int64_t, int,
                                        const QuantParams&, float*, cudaStream_t);
}  // namespace rrq
