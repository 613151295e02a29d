// rrq_params.h — parameter block passed by value to the rrq kernels, and the
// internal launcher interface between the C ABI (api.cpp) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "rrq.h"

namespace rrq {

constexpr int kMaxLevels = 16;  // bits <= 4
constexpr int kMaxCells = 64;   // cell-table search: at most 64 + 1 cells

// Cell table for the code search of the batch encoder.  The decision value
// u = y'/ν is mapped to s = sat(u·A + 1/2) ∈ [0, 1] with A = 1/(2R), R a
// power of two above every |τ_k|; the thresholds in that domain are
// t_k = fp32(τ_k·A + 1/2).  Cell j (j = 0..N) is the closed interval
// [(j − 1/2)/N, (j + 1/2)/N], the values s with round(s·N) = j.  `lo[j]` =
// #{k : t_k < (j − 1/2)/N} and `thr[j]` = the one t_k inside cell j, or 2 when
// the cell holds none, so code = lo[j] + (s > thr[j]) = #{k : s > t_k}.
// cells = 0: some cell of every allowed size would hold two thresholds, and
// the encoder uses its compare/select search instead.
struct CellTable {
  int cells;                      // N (16, 32 or 64), or 0
  float a;                        // A = 1/(2R) (a power of two)
  float thr[kMaxCells + 1];
  uint32_t lo[kMaxCells + 1];
};

// Codebook and rotation constants of one call.  levels: ascending c_0..c_{L-1};
// thr: τ_k = (c_k + c_{k+1})/2 for k = 0..L-2.  sym: the codebook is exactly
// symmetric (c_k = −c_{L−1−k}), so τ_{L/2−1} = 0 and the positive half of the
// thresholds decides every code.
struct QuantParams {
  uint64_t seed;
  float levels[kMaxLevels];
  float thr[kMaxLevels];
  int bits;
  int sym;
  float inv_sqrt_d;  // fp32(1/√d)
  float inv_d;       // 1/d (exact)
  // Per-vector value the encoders store: 0 = ν = ‖x‖₂; with a ±1 one-bit
  // codebook, DRIVE's scale S times √d ("History", DRIVE bullet): 1 = biased,
  // S = ‖Πx‖₁/d (stored ‖y'‖₁/d); 2 = unbiased, S = ‖x‖₂²/‖Πx‖₁ (stored
  // ‖x‖₂²·d/‖y'‖₁, 0 when y' = 0).  The decoder and score paths read the stored
  // value as ν, so x̂ = S·Πᵀ·sign(Πx) and ⟨q, x̂⟩ = S·⟨Πq, sign(Πx)⟩.
  int norm_mode;
  CellTable cell;
};

// Launchers (one per kernel family); all asynchronous on `stream`.
cudaError_t launch_rotate(const void* x, int dtype, int64_t n, int d, uint64_t seed, int inverse,
                          float inv_sqrt_d, float* y, cudaStream_t stream);
cudaError_t launch_encode(const void* x, int dtype, int64_t n, int d, const QuantParams& p,
                          uint8_t* codes, float* norms, cudaStream_t stream);
cudaError_t launch_decode(const uint8_t* codes, const float* norms, int64_t n, int d,
                          const QuantParams& p, void* out, int out_dtype, cudaStream_t stream);
cudaError_t launch_qk_scores(const void* q, int hq, const uint8_t* codes, const float* norms,
                             int64_t T, int hkv, int d, const QuantParams& p, float scale,
                             float* scores, cudaStream_t stream);
// Whether rrq_qk_scores supports (d, bits, hq, hkv): hkv a power of two and
// the kernel's shared-memory footprint within one CTA's limit.
bool qk_scores_supported(int d, int bits, int hq, int hkv);
cudaError_t launch_q4_0(const void* x, int dtype, int64_t n, int d, uint64_t seed, int rotate,
                        float inv_sqrt_d, void* blocks, cudaStream_t stream);
cudaError_t launch_q4_0_decode(const void* blocks, int64_t n, int d, uint64_t seed, int rotate,
                               float inv_sqrt_d, void* out, int out_dtype, cudaStream_t stream);
cudaError_t launch_encode_qjl(const void* x, int dtype, int64_t n, int d, const QuantParams& p,
                              const uint16_t* S, uint8_t* codes, float* norms, uint8_t* qjl_bits,
                              float* qjl_rnorm, cudaStream_t stream);

// Grid size for a grid-stride kernel: enough blocks for `work_blocks` units of
// work, capped at (resident blocks per SM) × (SM count) of the current device.
int grid_for(const void* kernel, int threads, size_t smem, int64_t work_blocks);

}  // namespace rrq
