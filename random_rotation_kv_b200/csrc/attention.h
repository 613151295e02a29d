// attention.h — arguments and launcher of the decode-attention kernel over a
// quantised K/V cache (attention.cu), called by the C ABI (api.cpp).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rrq_params.h"

namespace rrq {

struct AttnArgs {
  const __half* q;          // [hq × 128] query heads (unrotated)
  const uint8_t* k_codes;   // [T·hkv × 64] 4-bit K codes, row t·hkv + g
  const float* k_norms;     // [T·hkv]
  const uint8_t* v_codes;   // [T·hkv × 64] 4-bit V codes
  const float* v_norms;     // [T·hkv]
  float* out;               // [hq × 128]
  int64_t T;
  int hq, hkv, group;
  float scale;
  QuantParams pk, pv;       // K and V codebooks and rotation seeds
};

// Asynchronous on `stream`; d = 128, 4-bit K and V codes, group ∈ {1, 2, 4, 8}.
// Launched as clusters of up to 16 CTAs per kv head.
cudaError_t launch_attention_decode(const AttnArgs& a, cudaStream_t stream);

}  // namespace rrq
