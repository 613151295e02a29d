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
  unsigned* counters;       // [hkv] in the workspace, zero between calls
  float* states;            // [hkv × splits × G·131] in the workspace
  int64_t T;
  int hq, hkv, group, splits;
  float scale;
  QuantParams pk, pv;       // K and V codebooks and rotation seeds
};

// Token ranges per kv head for a cache of T tokens on the current device (as
// many CTAs as the device has SMs, one each), and the
// workspace bytes a call needs: hkv counters (padded to 256 bytes), then
// hq × splits × 131 floats of partial states (per head: m, l, M and 128 sums).
int attention_splits(int hkv, int group, int64_t T);
size_t attention_workspace_bytes(int hq, int hkv, int64_t T);

// Asynchronous on `stream`; d = 128, 4-bit K and V codes, group ∈ {1, 2, 4, 8}.
cudaError_t launch_attention_decode(const AttnArgs& a, cudaStream_t stream);

// The same with the workspace in a fixed device array of the library
// (kAttentionScratchBytes); a.counters / a.states are set here.  The caller has
// checked attention_workspace_bytes(...) ≤ kAttentionScratchBytes.
constexpr size_t kAttentionScratchBytes = size_t(4) << 20;
cudaError_t launch_attention_decode_in_scratch(AttnArgs a, cudaStream_t stream);
// That array's address on the current device (looked up once per device).
cudaError_t attention_scratch(void** addr);

// ---- every other shape (attention_gen.cu): d ∈ {64, 128, 256, 512}, 1- to 4-bit
// K and V codes, group ∈ {1, 2, 4, 8} (d = 512 with group ≤ 4), K widths the
// score kernel takes.  The scores go to the workspace first.
struct AttnGenArgs {
  const void* q;            // [hq × d] fp16 query heads (unrotated)
  const uint8_t* k_codes;   // [T·hkv × d·kb/8], row t·hkv + g
  const float* k_norms;     // [T·hkv]
  const uint8_t* v_codes;   // [T·hkv × d·vb/8]
  const float* v_norms;     // [T·hkv]
  float* out;               // [hq × d]
  unsigned* counters;       // set by launch_attention_general
  float* states;            // set by launch_attention_general
  float* scores;            // set by launch_attention_general
  int64_t T;
  int hq, hkv, group, splits, d;
  float scale;
  QuantParams pk, pv;
};
bool attention_general_supported(int d, int k_bits, int hq, int hkv);
int attention_general_splits(int hkv, int group, int d, int v_bits, int64_t T);
// counters (256-byte padded), partial states, then hq × T fp32 scores
size_t attention_general_workspace_bytes(int hq, int hkv, int d, int v_bits, int64_t T);
// Asynchronous on `stream`: the score launch, then the value launch.  The
// workspace's counters are zero before the call and after it.
cudaError_t launch_attention_general(AttnGenArgs a, void* workspace, cudaStream_t stream);

}  // namespace rrq
