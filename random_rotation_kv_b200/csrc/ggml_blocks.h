// ggml_blocks.h — launchers of the GGML block-type kernels (ggml_blocks.cu),
// called by the C ABI (api.cpp).  Both are asynchronous on `stream`; `type` is
// one of RRQ_GGML_Q4_1, RRQ_GGML_Q5_0, RRQ_GGML_Q5_1, RRQ_GGML_Q8_0.
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
