// Instantiates the f32 encode kernels (split per element type to build in parallel).
#include "batch_kernels.cuh"

namespace rrq {
template cudaError_t encode_typed<float>(const float*, int64_t, int, const QuantParams&, uint8_t*,
                                        float*, cudaStream_t);
}  // namespace rrq
