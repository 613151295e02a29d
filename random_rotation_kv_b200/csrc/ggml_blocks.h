// ggml_blocks.h — launchers of the GGML block-type kernels (ggml_blocks.cu),
// called by the C ABI (api.cpp) and by the q4_0 encoder entry (q4_0.cu).  Both
// are asynchronous on `stream`; `type` is one of the RRQ_GGML_* block types.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "rrq.h"

namespace rrq {

cudaError_t launch_ggml_blocks(const void* x, int dtype, int64_t n, int d, uint64_t seed, int rotate,
                               int type, float inv_sqrt_d, void* blocks, cudaStream_t stream);
cudaError_t launch_ggml_blocks_decode(const void* blocks, int type, int64_t n, int d, uint64_t seed,
                                      int rotate, float inv_sqrt_d, void* out, int out_dtype,
                                      cudaStream_t stream);

}  // namespace rrq
