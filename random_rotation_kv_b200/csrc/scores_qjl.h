// scores_qjl.h — arguments and launcher of the unbiased score kernel
// (scores_qjl.cu), called by the C ABI (api.cpp).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rrq_params.h"

namespace rrq {

struct QjlScoreArgs {
  const __half* q;              // [hq × 128] query heads
  const uint8_t* codes;         // [T·hkv × 16·bits] MSE codes, row t·hkv + g
  const float* norms;           // [T·hkv] ν
  const uint8_t* bits;          // [T·hkv × 16] QJL sign bits
  const float* rnorm;           // [T·hkv] residual norms ρ
  const __nv_bfloat16* S;       // [128 × 128] projection, row-major
  float* scores;                // [hq × T]
  int64_t T;
  int hq, hkv, group;
  float scale;
  QuantParams p;
};

// Asynchronous on `stream`; d = 128, group ∈ {1, 2, 4, 8}, bits 1..4.
cudaError_t launch_qk_scores_qjl(const QjlScoreArgs& a, cudaStream_t stream);

}  // namespace rrq
